// The C ABI (include/sketch_attn.h): argument validation, workspace layout,
// and dispatch to the kernels.  Host-side only; no allocation anywhere.
#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>
#include <cstdio>

#include "sa_internal.cuh"
#include "stca_internal.cuh"

namespace sa {

// ---------------------------------------------------------------- errors
static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }
sa_status fail(sa_status st, const std::string& msg) {
  set_error(msg);
  return st;
}
sa_status cuda_fail(cudaError_t e, const char* what) {
  set_error(std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")");
  return SA_ERR_CUDA;
}

__device__ int g_device_status;

int* device_status_word() {
  static std::mutex mu;
  static int* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    addr[dev] = (int*)p;
  }
  return addr[dev];
}

const DeviceInfo& device_info() {
  static std::mutex mu;
  static DeviceInfo info[64];
  static bool have[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    DeviceInfo d;
    d.device = dev;
    cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (d.sm_count <= 0) d.sm_count = 148;
    info[dev] = d;
    have[dev] = true;
  }
  return info[dev];
}

// ---------------------------------------------------------------- measurement
static std::atomic<long long> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {
struct ProfState {
  std::mutex mu;
  bool on = false;
  struct Pending { std::string name; cudaEvent_t a, b; };
  std::vector<Pending> pending;
  std::vector<cudaEvent_t> pool;
  std::vector<std::string> names;
  std::vector<double> ms;
  std::vector<long long> count;
  cudaEvent_t open_evt = nullptr;
  cudaEvent_t get() {
    if (!pool.empty()) { cudaEvent_t e = pool.back(); pool.pop_back(); return e; }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
  void settle() {
    for (auto& p : pending) {
      float t = 0.f;
      cudaEventSynchronize(p.b);
      cudaEventElapsedTime(&t, p.a, p.b);
      size_t i = 0;
      while (i < names.size() && names[i] != p.name) ++i;
      if (i == names.size()) { names.push_back(p.name); ms.push_back(0.0); count.push_back(0); }
      ms[i] += t;
      count[i] += 1;
      pool.push_back(p.a);
      pool.push_back(p.b);
    }
    pending.clear();
  }
};
ProfState& prof() { static ProfState s; return s; }
}  // namespace

void prof_begin(const char* name, cudaStream_t st) {
  (void)name;
  ProfState& p = prof();
  if (!p.on) return;
  std::lock_guard<std::mutex> lock(p.mu);
  p.open_evt = p.get();
  cudaEventRecord(p.open_evt, st);
}

void prof_end(const char* name, cudaStream_t st) {
  ProfState& p = prof();
  if (!p.on) return;
  std::lock_guard<std::mutex> lock(p.mu);
  if (!p.open_evt) return;
  cudaEvent_t b = p.get();
  cudaEventRecord(b, st);
  p.pending.push_back({name, p.open_evt, b});
  p.open_evt = nullptr;
  if (p.pending.size() > 4096) p.settle();
}

sa_status stca_fuse_run(const float* z_r, const float* z_u, const float* W_F, const float* b_F,
                        int64_t C, int D, float* out, cudaStream_t st);

namespace {

sa_status check_offsets(const int64_t* off, int B, const char* name) {
  if (!off) return fail(SA_ERR_INVALID_ARG, std::string(name) + " is NULL");
  if (off[0] != 0) return fail(SA_ERR_INVALID_ARG, std::string(name) + "[0] must be 0");
  for (int u = 0; u < B; ++u)
    if (off[u + 1] < off[u])
      return fail(SA_ERR_INVALID_ARG, std::string(name) + " must be non-decreasing (user " +
                                          std::to_string(u) + ")");
  return SA_OK;
}

sa_status check_ptr(const void* p, const char* name, bool nullable = false) {
  if (!p) return nullable ? SA_OK : fail(SA_ERR_INVALID_ARG, std::string(name) + " is NULL");
  if (!aligned16(p)) return fail(SA_ERR_INVALID_ARG, std::string(name) + " is not 16-byte aligned");
  return SA_OK;
}

#define SA_TRY(expr)                 \
  do {                               \
    sa_status _s = (expr);           \
    if (_s != SA_OK) return _s;      \
  } while (0)

sa_status check_sa_shape(int B, int k, int d, sa_dtype dt) {
  if (B < 1) return fail(SA_ERR_INVALID_ARG, "B must be >= 1");
  if (dt != SA_F32 && dt != SA_BF16) return fail(SA_ERR_INVALID_ARG, "unknown x_dtype");
  if (k < 1 || k > 4096) return fail(SA_ERR_UNSUPPORTED, "k must be in [1, 4096]");
  if (d != 64 && d != 128) return fail(SA_ERR_UNSUPPORTED, "d must be 64 or 128");
  return SA_OK;
}

// ---------------------------------------------------------------- layouts
bool use_tc(sa_dtype dt, int k, int d) { return sa_tc_supported(dt, k, d); }

size_t layout_fwd(void* base, int B, int64_t n, int k, int d, sa_dtype dt, SaFwdWork* w) {
  const DeviceInfo& di = device_info();
  Chunking ch;
  if (use_tc(dt, k, d)) {
    ch = make_chunking(n, sa_tc_num_chunks(k), 1);
  } else {
    const int kblocks = (k + 31) / 32;
    int target = std::max(1, 4 * di.sm_count / kblocks);
    target = (int)std::min<int64_t>(target, std::max<int64_t>(1, n / 256));
    ch = make_chunking(n, target, 1);
  }
  Carve c(base);
  SaFwdWork v;
  v.ch = ch;
  v.T = c.take<float>((size_t)d * d);
  v.Pf = c.take<float>((size_t)k * d);
  v.Pb = c.take<__nv_bfloat16>((size_t)k * d);
  v.lse = c.take<float>((size_t)std::max<int64_t>(n, 1));
  v.Muser = c.take<float>((size_t)B * k);
  v.slotH = c.take<float>((size_t)std::max(ch.G, 1) * 2 * k * d);
  v.slotM = c.take<float>((size_t)std::max(ch.G, 1) * 2 * k);
  v.Hhat = c.take<float>((size_t)B * k * d);
  if (dt == SA_BF16 && d == 128) {
    v.Hhi = c.take<__nv_bfloat16>((size_t)B * k * d);
    v.Hlo = c.take<__nv_bfloat16>((size_t)B * k * d);
    v.Vhi = c.take<__nv_bfloat16>((size_t)d * d);
    v.Vlo = c.take<__nv_bfloat16>((size_t)d * d);
  }
  if (w) *w = v;
  return c.bytes();
}

size_t layout_bwd(void* base, int B, int64_t n, int k, int d, sa_dtype dt, SaBwdWork* w) {
  const DeviceInfo& di = device_info();
  const bool tc = sa_bwd_tc_supported(dt, k, d);
  int target = tc ? sa_bwd_tc_dx_chunks() : 8 * di.sm_count;
  target = (int)std::min<int64_t>(target, std::max<int64_t>(1, n / 64));
  Chunking ch = make_chunking(n, target, 1);
  int targetE = tc ? sa_bwd_tc_e_chunks(k) : std::max(1, 4 * di.sm_count / ((k + 15) / 16));
  targetE = (int)std::min<int64_t>(targetE, std::max<int64_t>(1, n / 256));
  Chunking chE = make_chunking(n, targetE, 1);
  Carve c(base);
  SaBwdWork v;
  v.ch = ch;
  v.chE = chE;
  v.T = c.take<float>((size_t)d * d);
  v.Pf = c.take<float>((size_t)k * d);
  v.Pb = c.take<__nv_bfloat16>((size_t)k * d);
  v.lse = c.take<float>((size_t)std::max<int64_t>(n, 1));
  v.cbuf = c.take<float>((size_t)std::max<int64_t>(n, 1));
  v.dHh = c.take<float>((size_t)B * k * d);
  v.Hhat = c.take<float>((size_t)B * k * d);
  v.dH = c.take<float>((size_t)B * k * d);
  v.dHb = tc ? c.take<__nv_bfloat16>((size_t)B * k * d) : nullptr;
  v.dHlo = tc ? c.take<__nv_bfloat16>((size_t)B * k * d) : nullptr;
  v.dm = c.take<float>((size_t)B * k);
  v.dmc = tc ? c.take<float>((size_t)B * k) : nullptr;
  v.Epart = c.take<float>((size_t)std::max(chE.G, 1) * k * d);
  v.E = c.take<float>((size_t)k * d);
  v.dQ = c.take<float>((size_t)k * d);
  v.Q = c.take<float>((size_t)k * d);
  v.gsplit = c.take<float>((size_t)kMaxSplit * d * d);
  if (tc) {
    v.dShi = c.take<__nv_bfloat16>((size_t)B * k * d);
    v.dSlo = c.take<__nv_bfloat16>((size_t)B * k * d);
    v.Hhi = c.take<__nv_bfloat16>((size_t)B * k * d);
    v.Hlo = c.take<__nv_bfloat16>((size_t)B * k * d);
    v.Vhi = c.take<__nv_bfloat16>((size_t)d * d);
    v.Vlo = c.take<__nv_bfloat16>((size_t)d * d);
  }
  if (w) *w = v;
  return c.bytes();
}

size_t layout_stca(void* base, int B, int64_t C, int D, int heads, int d_h, StcaWork* w) {
  Carve c(base);
  StcaWork v = stca_attn_carve(c, B, C, D, heads, d_h);
  if (w) *w = v;
  return c.bytes();
}

}  // namespace
}  // namespace sa

using namespace sa;

extern "C" {

int sa_version(void) { return 100; }

long long sa_launch_count(void) { return g_launches.load(); }

sa_status sa_profile(int enable) {
  ProfState& p = prof();
  std::lock_guard<std::mutex> lock(p.mu);
  if (enable) {
    p.settle();
    p.names.clear();
    p.ms.clear();
    p.count.clear();
    p.on = true;
  } else {
    p.on = false;
  }
  return SA_OK;
}

int sa_profile_read(int i, char* name, int name_len, double* total_ms, long long* launches) {
  ProfState& p = prof();
  std::lock_guard<std::mutex> lock(p.mu);
  p.settle();
  if (i < 0 || i >= (int)p.names.size()) return 0;
  if (name && name_len > 0) {
    std::snprintf(name, (size_t)name_len, "%s", p.names[i].c_str());
  }
  if (total_ms) *total_ms = p.ms[i];
  if (launches) *launches = p.count[i];
  return 1;
}

const char* sa_last_error(void) { return g_last_error.c_str(); }

sa_status sa_poll_device_status(sa_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int* w = device_status_word();
  if (!w) return fail(SA_ERR_CUDA, "device status word unavailable");
  int v = 0;
  e = cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read device status");
  if (v != 0) {
    int zero = 0;
    cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (v & DEV_ERR_TIMEOUT) return fail(SA_ERR_TIMEOUT, "a device-side wait expired");
    if (v & DEV_ERR_INDEX) return fail(SA_ERR_INVALID_ARG, "an embedding id was out of range (its row was zeroed)");
    if (v & DEV_ERR_RANGE)
      return fail(SA_ERR_UNSUPPORTED, "a value of the full STCA layer's fp16 operands exceeded the fp16 range "
                                      "(|x| > 65504); scale the inputs down or use fp32 inputs");
    return fail(SA_ERR_CUDA, "device error word " + std::to_string(v));
  }
  return SA_OK;
}

size_t sa_forward_workspace(int B, int64_t n_total, int k, int d, sa_dtype x_dtype) {
  if (B < 1 || k < 1 || d < 1 || n_total < 0) return 0;
  return layout_fwd(nullptr, B, n_total, k, d, x_dtype, nullptr);
}

sa_status sa_forward(const void* X, sa_dtype x_dtype, const int64_t* offsets_host,
                     const int64_t* offsets_dev, int B, int k, int d, const float* P,
                     const float* W_Q, const float* W_K, const float* W_V, float eps, float* S,
                     float* mass, float* H, void* S_bf16, float* lse, void* workspace,
                     size_t ws_bytes, sa_stream_t stream) {
  SA_TRY(check_sa_shape(B, k, d, x_dtype));
  SA_TRY(check_offsets(offsets_host, B, "offsets_host"));
  const int64_t n = offsets_host[B];
  if (!(eps >= 0.f)) return fail(SA_ERR_INVALID_ARG, "eps must be >= 0");
  SA_TRY(check_ptr(X, "X", n == 0));
  SA_TRY(check_ptr(offsets_dev, "offsets_dev"));
  SA_TRY(check_ptr(P, "P"));
  SA_TRY(check_ptr(W_Q, "W_Q"));
  SA_TRY(check_ptr(W_K, "W_K"));
  SA_TRY(check_ptr(W_V, "W_V"));
  SA_TRY(check_ptr(S, "S"));
  SA_TRY(check_ptr(mass, "mass"));
  SA_TRY(check_ptr(H, "H", true));
  SA_TRY(check_ptr(S_bf16, "S_bf16", true));
  SA_TRY(check_ptr(lse, "lse", true));
  if (H == S) return fail(SA_ERR_INVALID_ARG, "H must not alias S");
  const size_t need = layout_fwd(nullptr, B, n, k, d, x_dtype, nullptr);
  if (!workspace || ws_bytes < need)
    return fail(SA_ERR_WORKSPACE, "workspace needs " + std::to_string(need) + " bytes");
  SA_TRY(check_ptr(workspace, "workspace"));
  SaFwdWork w;
  layout_fwd(workspace, B, n, k, d, x_dtype, &w);
  SaFwdArgs a{X, x_dtype, offsets_dev, B, n, k, d, P, W_Q, W_K, W_V, eps, S, mass, H, S_bf16, lse};
  cudaStream_t st = (cudaStream_t)stream;
  SA_TRY(sa_fold(k, d, P, W_Q, W_K, w.T, w.Pf, w.Pb, st));
  if (n > 0) {
    if (use_tc(x_dtype, k, d)) SA_TRY(sa_tc_forward(a, w, st));
    else SA_TRY(sa_simt_forward(a, w, st));
  }
  return sa_reduce_and_project(a, w, st);
}

size_t sa_forward_tokenwise_workspace(int B, int64_t n_total, int k, int d, sa_dtype x_dtype) {
  if (B < 1 || k < 1 || d < 1 || n_total < 0 || x_dtype != SA_BF16 || d != 128) return 0;
  return tokenwise_layout(nullptr, B, k, d, nullptr);
}

sa_status sa_forward_tokenwise(const void* X, sa_dtype x_dtype, const int64_t* offsets_host,
                               const int64_t* offsets_dev, int B, int k, int d, const float* P,
                               const float* W_Q, const float* W_K, const float* W_V, float eps,
                               float* S, float* mass, float* H, void* S_bf16, void* workspace,
                               size_t ws_bytes, sa_stream_t stream) {
  SA_TRY(check_sa_shape(B, k, d, x_dtype));
  if (x_dtype != SA_BF16 || d != 128)
    return fail(SA_ERR_UNSUPPORTED, "sa_forward_tokenwise needs bf16 X and d = 128");
  SA_TRY(check_offsets(offsets_host, B, "offsets_host"));
  const int64_t n = offsets_host[B];
  if (n >= (1LL << 31) || (int64_t)B * k >= (1LL << 31))
    return fail(SA_ERR_UNSUPPORTED, "n_total and B * k must be < 2^31");
  if (!(eps >= 0.f)) return fail(SA_ERR_INVALID_ARG, "eps must be >= 0");
  SA_TRY(check_ptr(X, "X", n == 0));
  SA_TRY(check_ptr(offsets_dev, "offsets_dev"));
  SA_TRY(check_ptr(P, "P"));
  SA_TRY(check_ptr(W_Q, "W_Q"));
  SA_TRY(check_ptr(W_K, "W_K"));
  SA_TRY(check_ptr(W_V, "W_V"));
  SA_TRY(check_ptr(S, "S"));
  SA_TRY(check_ptr(mass, "mass"));
  SA_TRY(check_ptr(H, "H", true));
  SA_TRY(check_ptr(S_bf16, "S_bf16", true));
  if (H == S) return fail(SA_ERR_INVALID_ARG, "H must not alias S");
  const size_t need = tokenwise_layout(nullptr, B, k, d, nullptr);
  if (!workspace || ws_bytes < need)
    return fail(SA_ERR_WORKSPACE, "workspace needs " + std::to_string(need) + " bytes");
  SA_TRY(check_ptr(workspace, "workspace"));
  TokenwiseWork w;
  tokenwise_layout(workspace, B, k, d, &w);
  SaFwdArgs a{X, x_dtype, offsets_dev, B, n, k, d, P, W_Q, W_K, W_V, eps, S, mass, H, S_bf16, nullptr};
  return sa_tokenwise_run(a, w, (cudaStream_t)stream);
}

size_t sa_refine_workspace(int B, int64_t n_total, int k, int d, sa_dtype x_dtype) {
  if (B < 1 || k < 1 || d < 1 || n_total < 0 || !sa_tc_supported(x_dtype, k, d)) return 0;
  return refine_layout(nullptr, B, n_total, k, d, nullptr, nullptr);
}

sa_status sa_refine_forward(const void* X, sa_dtype x_dtype, const int64_t* offsets_host,
                            const int64_t* offsets_dev, int B, int k, int d, const float* P0,
                            int n_iter, const sa_refine_layer* layers, float ln_eps,
                            float* sketch, void* workspace, size_t ws_bytes,
                            sa_stream_t stream) {
  SA_TRY(check_sa_shape(B, k, d, x_dtype));
  if (!sa_tc_supported(x_dtype, k, d))
    return fail(SA_ERR_UNSUPPORTED, "sa_refine_forward needs bf16 X, d = 128 and k a multiple of 128");
  SA_TRY(check_offsets(offsets_host, B, "offsets_host"));
  const int64_t n = offsets_host[B];
  if (n >= (1LL << 31)) return fail(SA_ERR_UNSUPPORTED, "n_total must be < 2^31");
  if (n_iter < 1) return fail(SA_ERR_INVALID_ARG, "n_iter must be >= 1");
  if (!layers) return fail(SA_ERR_INVALID_ARG, "layers is NULL");
  if (!(ln_eps > 0.f)) return fail(SA_ERR_INVALID_ARG, "ln_eps must be > 0");
  if ((int64_t)B * k >= (1LL << 31)) return fail(SA_ERR_UNSUPPORTED, "B * k must be < 2^31");
  SA_TRY(check_ptr(X, "X", n == 0));
  SA_TRY(check_ptr(offsets_dev, "offsets_dev"));
  SA_TRY(check_ptr(P0, "P0"));
  SA_TRY(check_ptr(sketch, "sketch"));
  for (int i = 0; i < n_iter; ++i) {
    const sa_refine_layer& L = layers[i];
    SA_TRY(check_ptr(L.W_Q, "layers[].W_Q"));
    SA_TRY(check_ptr(L.W_K, "layers[].W_K"));
    SA_TRY(check_ptr(L.W1, "layers[].W1"));
    SA_TRY(check_ptr(L.W3, "layers[].W3"));
    SA_TRY(check_ptr(L.W2, "layers[].W2"));
    SA_TRY(check_ptr(L.ln1_g, "layers[].ln1_g", true));
    SA_TRY(check_ptr(L.ln1_b, "layers[].ln1_b", true));
    SA_TRY(check_ptr(L.ln2_g, "layers[].ln2_g", true));
    SA_TRY(check_ptr(L.ln2_b, "layers[].ln2_b", true));
  }
  const size_t need = refine_layout(nullptr, B, n, k, d, nullptr, nullptr);
  if (!workspace || ws_bytes < need)
    return fail(SA_ERR_WORKSPACE, "workspace needs " + std::to_string(need) + " bytes");
  SA_TRY(check_ptr(workspace, "workspace"));
  SaFwdWork w;
  RefineWork r;
  refine_layout(workspace, B, n, k, d, &w, &r);
  return sa_refine_run(X, x_dtype, offsets_dev, B, n, k, d, P0, n_iter, layers, ln_eps, sketch, w, r,
                       (cudaStream_t)stream);
}

size_t sa_refine_backward_workspace(int B, int64_t n_total, int k, int d, int n_iter, sa_dtype x_dtype) {
  if (B < 1 || n_total < 0 || n_iter < 1 || n_iter > 8 || !sa_tc_supported(x_dtype, k, d)) return 0;
  return refine_bwd_layout(nullptr, B, n_total, k, d, n_iter, nullptr);
}

sa_status sa_refine_backward(const void* X, sa_dtype x_dtype, const int64_t* offsets_host,
                             const int64_t* offsets_dev, int B, int k, int d, const float* P0,
                             int n_iter, const sa_refine_layer* layers, float ln_eps,
                             const float* dsketch, float* dX, float* dP0,
                             const sa_refine_layer_grad* grads, void* workspace, size_t ws_bytes,
                             sa_stream_t stream) {
  SA_TRY(check_sa_shape(B, k, d, x_dtype));
  if (!sa_tc_supported(x_dtype, k, d))
    return fail(SA_ERR_UNSUPPORTED, "sa_refine_backward needs bf16 X, d = 128 and k a multiple of 128");
  SA_TRY(check_offsets(offsets_host, B, "offsets_host"));
  const int64_t n = offsets_host[B];
  if (n >= (1LL << 31)) return fail(SA_ERR_UNSUPPORTED, "n_total must be < 2^31");
  if (n_iter < 1 || n_iter > 8) return fail(SA_ERR_UNSUPPORTED, "n_iter must be 1..8");
  if (!layers || !grads) return fail(SA_ERR_INVALID_ARG, "layers or grads is NULL");
  if (!(ln_eps > 0.f)) return fail(SA_ERR_INVALID_ARG, "ln_eps must be > 0");
  if ((int64_t)B * k >= (1LL << 31)) return fail(SA_ERR_UNSUPPORTED, "B * k must be < 2^31");
  SA_TRY(check_ptr(X, "X", n == 0));
  SA_TRY(check_ptr(offsets_dev, "offsets_dev"));
  SA_TRY(check_ptr(P0, "P0"));
  SA_TRY(check_ptr(dsketch, "dsketch"));
  SA_TRY(check_ptr(dX, "dX", n == 0));
  SA_TRY(check_ptr(dP0, "dP0"));
  for (int i = 0; i < n_iter; ++i) {
    const sa_refine_layer& L = layers[i];
    const sa_refine_layer_grad& G = grads[i];
    SA_TRY(check_ptr(L.W_Q, "layers[].W_Q"));
    SA_TRY(check_ptr(L.W_K, "layers[].W_K"));
    SA_TRY(check_ptr(L.W1, "layers[].W1"));
    SA_TRY(check_ptr(L.W3, "layers[].W3"));
    SA_TRY(check_ptr(L.W2, "layers[].W2"));
    SA_TRY(check_ptr(G.dW_Q, "grads[].dW_Q"));
    SA_TRY(check_ptr(G.dW_K, "grads[].dW_K"));
    SA_TRY(check_ptr(G.dW1, "grads[].dW1"));
    SA_TRY(check_ptr(G.dW3, "grads[].dW3"));
    SA_TRY(check_ptr(G.dW2, "grads[].dW2"));
    const float* opt[4] = {L.ln1_g, L.ln1_b, L.ln2_g, L.ln2_b};
    float* const gopt[4] = {G.dln1_g, G.dln1_b, G.dln2_g, G.dln2_b};
    for (int j = 0; j < 4; ++j) {
      SA_TRY(check_ptr(opt[j], "a LayerNorm parameter", true));
      if (opt[j]) SA_TRY(check_ptr(gopt[j], "the gradient of a LayerNorm parameter"));
    }
  }
  const size_t need = refine_bwd_layout(nullptr, B, n, k, d, n_iter, nullptr);
  if (!workspace || ws_bytes < need)
    return fail(SA_ERR_WORKSPACE, "workspace needs " + std::to_string(need) + " bytes");
  SA_TRY(check_ptr(workspace, "workspace"));
  return sa_refine_backward_run(X, offsets_host, offsets_dev, B, n, k, d, P0, n_iter, layers, ln_eps, dsketch,
                                dX, dP0, grads, workspace, (cudaStream_t)stream);
}

size_t sa_backward_workspace(int B, int64_t n_total, int k, int d, sa_dtype x_dtype) {
  if (B < 1 || k < 1 || d < 1 || n_total < 0) return 0;
  return layout_bwd(nullptr, B, n_total, k, d, x_dtype, nullptr);
}

}  // extern "C"

namespace {
sa_status backward_impl(const void* X, sa_dtype x_dtype, const int64_t* offsets_host,
                        const int64_t* offsets_dev, int B, int k, int d, const float* P,
                        const float* W_Q, const float* W_K, const float* W_V, float eps,
                        const float* H, const float* mass, const float* dS, const float* dmass,
                        const float* lse, void* dX, float* dP, float* dW_Q, float* dW_K,
                        float* dW_V, void* workspace, size_t ws_bytes, sa_stream_t stream,
                        bool accumulate) {
  SA_TRY(check_sa_shape(B, k, d, x_dtype));
  SA_TRY(check_offsets(offsets_host, B, "offsets_host"));
  const int64_t n = offsets_host[B];
  if (!(eps >= 0.f)) return fail(SA_ERR_INVALID_ARG, "eps must be >= 0");
  SA_TRY(check_ptr(X, "X", n == 0));
  SA_TRY(check_ptr(dX, "dX", n == 0));
  SA_TRY(check_ptr(offsets_dev, "offsets_dev"));
  SA_TRY(check_ptr(P, "P"));
  SA_TRY(check_ptr(W_Q, "W_Q"));
  SA_TRY(check_ptr(W_K, "W_K"));
  SA_TRY(check_ptr(W_V, "W_V"));
  SA_TRY(check_ptr(H, "H"));
  SA_TRY(check_ptr(mass, "mass"));
  SA_TRY(check_ptr(dS, "dS"));
  SA_TRY(check_ptr(dmass, "dmass", true));
  SA_TRY(check_ptr(lse, "lse", true));
  SA_TRY(check_ptr(dP, "dP"));
  SA_TRY(check_ptr(dW_Q, "dW_Q"));
  SA_TRY(check_ptr(dW_K, "dW_K"));
  SA_TRY(check_ptr(dW_V, "dW_V"));
  const size_t need = layout_bwd(nullptr, B, n, k, d, x_dtype, nullptr);
  if (!workspace || ws_bytes < need)
    return fail(SA_ERR_WORKSPACE, "workspace needs " + std::to_string(need) + " bytes");
  SA_TRY(check_ptr(workspace, "workspace"));
  SaBwdWork w;
  layout_bwd(workspace, B, n, k, d, x_dtype, &w);
  SaBwdArgs a{X, x_dtype, offsets_dev, B, n, k, d, P, W_Q, W_K, W_V, eps,
              H, mass, dS, dmass, lse, dX, dP, dW_Q, dW_K, dW_V};
  a.accumulate = accumulate;
  cudaStream_t st = (cudaStream_t)stream;
  SA_TRY(sa_fold(k, d, P, W_Q, W_K, w.T, w.Pf, w.Pb, st));
  return sa_backward_run(a, w, sa_bwd_tc_supported(x_dtype, k, d), st);
}
}  // namespace

extern "C" {

sa_status sa_backward(const void* X, sa_dtype x_dtype, const int64_t* offsets_host,
                      const int64_t* offsets_dev, int B, int k, int d, const float* P,
                      const float* W_Q, const float* W_K, const float* W_V, float eps,
                      const float* H, const float* mass, const float* dS, const float* dmass,
                      const float* lse, void* dX, float* dP, float* dW_Q, float* dW_K,
                      float* dW_V, void* workspace, size_t ws_bytes, sa_stream_t stream) {
  return backward_impl(X, x_dtype, offsets_host, offsets_dev, B, k, d, P, W_Q, W_K, W_V, eps, H, mass,
                       dS, dmass, lse, dX, dP, dW_Q, dW_K, dW_V, workspace, ws_bytes, stream, false);
}

sa_status sa_backward_accumulate(const void* X, sa_dtype x_dtype, const int64_t* offsets_host,
                                 const int64_t* offsets_dev, int B, int k, int d, const float* P,
                                 const float* W_Q, const float* W_K, const float* W_V, float eps,
                                 const float* H, const float* mass, const float* dS,
                                 const float* dmass, const float* lse, void* dX, float* dP,
                                 float* dW_Q, float* dW_K, float* dW_V, void* workspace,
                                 size_t ws_bytes, sa_stream_t stream) {
  return backward_impl(X, x_dtype, offsets_host, offsets_dev, B, k, d, P, W_Q, W_K, W_V, eps, H, mass,
                       dS, dmass, lse, dX, dP, dW_Q, dW_K, dW_V, workspace, ws_bytes, stream, true);
}

size_t stca_forward_workspace(int B, int64_t C_total, int D, int heads, int d_h, sa_dtype dtype) {
  (void)dtype;
  if (B < 1 || C_total < 0 || D < 1 || heads < 1 || d_h < 1) return 0;
  return layout_stca(nullptr, B, C_total, D, heads, d_h, nullptr);
}

}  // extern "C"

namespace {
// Checks shared by stca_forward and stca_forward_full; fills a (less the
// layers) and the number of query tiles and of key rows.
sa_status stca_check(const void* q, sa_dtype dtype, const int64_t* cand_offsets_host,
                     const int64_t* cand_offsets_dev, int B, const void* kv, int64_t kv_rows,
                     const int64_t* kv_begin_host, const int64_t* kv_end_host,
                     const int64_t* kv_begin_dev, const int64_t* kv_end_dev, int D, int heads,
                     int d_h, int n_layers, const stca_layer* const* attn, float* out, StcaArgs* a,
                     int* max_tiles, int64_t* kv_total, bool out_optional = false) {
  if (B < 1) return fail(SA_ERR_INVALID_ARG, "B must be >= 1");
  if (dtype != SA_F32 && dtype != SA_BF16) return fail(SA_ERR_INVALID_ARG, "unknown dtype");
  if (D != 128) return fail(SA_ERR_UNSUPPORTED, "D must be 128");
  if (heads < 1 || d_h < 1 || (int64_t)heads * d_h > 4096)
    return fail(SA_ERR_UNSUPPORTED, "need heads >= 1, d_h >= 1, heads*d_h <= 4096");
  if (n_layers < 1 || !attn) return fail(SA_ERR_INVALID_ARG, "need n_layers >= 1 and layers");
  if (kv_rows < 0) return fail(SA_ERR_INVALID_ARG, "kv_rows must be >= 0");
  SA_TRY(check_offsets(cand_offsets_host, B, "cand_offsets_host"));
  if (!kv_begin_host || !kv_end_host) return fail(SA_ERR_INVALID_ARG, "kv ranges are NULL");
  int64_t max_rows = 0, kv_sum = 0;
  for (int u = 0; u < B; ++u) {
    if (kv_begin_host[u] < 0 || kv_end_host[u] < kv_begin_host[u] || kv_end_host[u] > kv_rows)
      return fail(SA_ERR_INVALID_ARG, "bad key range of user " + std::to_string(u));
    max_rows = std::max(max_rows, (cand_offsets_host[u + 1] - cand_offsets_host[u]) * heads);
    kv_sum += kv_end_host[u] - kv_begin_host[u];
  }
  const int64_t C = cand_offsets_host[B];
  SA_TRY(check_ptr(q, "q", C == 0));
  SA_TRY(check_ptr(kv, "kv", kv_rows == 0));
  SA_TRY(check_ptr(cand_offsets_dev, "cand_offsets_dev"));
  SA_TRY(check_ptr(kv_begin_dev, "kv_begin_dev"));
  SA_TRY(check_ptr(kv_end_dev, "kv_end_dev"));
  SA_TRY(check_ptr(out, "out", C == 0 || out_optional));
  for (int l = 0; l < n_layers; ++l) {
    const stca_layer& L = *attn[l];
    SA_TRY(check_ptr(L.W_Q, "layers[].W_Q"));
    SA_TRY(check_ptr(L.W_K, "layers[].W_K"));
    SA_TRY(check_ptr(L.W_V, "layers[].W_V"));
    SA_TRY(check_ptr(L.W_O, "layers[].W_O", true));
    if (!L.W_O && heads * d_h != D)
      return fail(SA_ERR_INVALID_ARG, "W_O = NULL needs heads*d_h == D");
  }
  const int tq = stca_tc_supported(dtype, D) ? 128 : 32;
  int64_t tiles = 0;
  for (int u = 0; u < B; ++u)
    tiles += ((cand_offsets_host[u + 1] - cand_offsets_host[u]) * heads + tq - 1) / tq;
  if (tiles > (1LL << 30)) return fail(SA_ERR_UNSUPPORTED, "too many query tiles");
  *max_tiles = (int)std::max<int64_t>(tiles, 1);
  *kv_total = kv_sum;
  *a = StcaArgs{q, dtype, cand_offsets_dev, B, C, kv, kv_rows, kv_begin_dev, kv_end_dev,
                D, heads, d_h, n_layers, nullptr, out, max_rows};
  return SA_OK;
}
}  // namespace

extern "C" {

sa_status stca_forward(const void* q, sa_dtype dtype, const int64_t* cand_offsets_host,
                       const int64_t* cand_offsets_dev, int B, const void* kv, int64_t kv_rows,
                       const int64_t* kv_begin_host, const int64_t* kv_end_host,
                       const int64_t* kv_begin_dev, const int64_t* kv_end_dev, int D, int heads,
                       int d_h, int n_layers, const stca_layer* layers, float* out,
                       void* workspace, size_t ws_bytes, sa_stream_t stream) {
  if (n_layers < 1 || !layers) return fail(SA_ERR_INVALID_ARG, "need n_layers >= 1 and layers");
  std::vector<const stca_layer*> attn(n_layers);
  for (int l = 0; l < n_layers; ++l) attn[l] = &layers[l];
  StcaArgs a;
  int max_tiles = 0;
  int64_t kv_total = 0;
  SA_TRY(stca_check(q, dtype, cand_offsets_host, cand_offsets_dev, B, kv, kv_rows, kv_begin_host,
                    kv_end_host, kv_begin_dev, kv_end_dev, D, heads, d_h, n_layers, attn.data(), out,
                    &a, &max_tiles, &kv_total));
  const int64_t C = cand_offsets_host[B];
  const size_t need = layout_stca(nullptr, B, C, D, heads, d_h, nullptr);
  if (!workspace || ws_bytes < need)
    return fail(SA_ERR_WORKSPACE, "workspace needs " + std::to_string(need) + " bytes");
  SA_TRY(check_ptr(workspace, "workspace"));
  StcaWork w;
  layout_stca(workspace, B, C, D, heads, d_h, &w);
  w.max_tiles = max_tiles;
  a.layers = layers;
  return stca_run(a, w, (cudaStream_t)stream);
}

size_t stca_forward_full_workspace(int B, int64_t C_total, int64_t kv_total, int D, int heads,
                                   int d_h, sa_dtype dtype) {
  if (B < 1 || C_total < 0 || kv_total < 0 || D < 1 || heads < 1 || d_h < 1) return 0;
  if (dtype != SA_F32 && dtype != SA_BF16) return 0;
  return stca_full_layout(nullptr, B, C_total, kv_total, D, heads, d_h, dtype, nullptr);
}

sa_status stca_forward_full(const void* q, sa_dtype dtype, const int64_t* cand_offsets_host,
                            const int64_t* cand_offsets_dev, int B, const void* kv, int64_t kv_rows,
                            const int64_t* kv_begin_host, const int64_t* kv_end_host,
                            const int64_t* kv_begin_dev, const int64_t* kv_end_dev, int D, int heads,
                            int d_h, int n_layers, const stca_full_layer* layers, float* out,
                            void* workspace, size_t ws_bytes, sa_stream_t stream) {
  if (n_layers < 1 || !layers) return fail(SA_ERR_INVALID_ARG, "need n_layers >= 1 and layers");
  std::vector<const stca_layer*> attn(n_layers);
  for (int l = 0; l < n_layers; ++l) {
    const stca_full_layer& L = layers[l];
    attn[l] = &L.attn;
    const int nh = !!L.hist_W1 + !!L.hist_W3 + !!L.hist_W2, nq = !!L.q_W1 + !!L.q_W3 + !!L.q_W2;
    if ((nh != 0 && nh != 3) || (nq != 0 && nq != 3))
      return fail(SA_ERR_INVALID_ARG, "layer " + std::to_string(l) + ": an FFN is partly given");
    for (const float* wp : {L.hist_W1, L.hist_W3, L.hist_W2, L.q_W1, L.q_W3, L.q_W2})
      SA_TRY(check_ptr(wp, "layers[] FFN weight", true));
  }
  StcaArgs a;
  int max_tiles = 0;
  int64_t kv_total = 0;
  SA_TRY(stca_check(q, dtype, cand_offsets_host, cand_offsets_dev, B, kv, kv_rows, kv_begin_host,
                    kv_end_host, kv_begin_dev, kv_end_dev, D, heads, d_h, n_layers, attn.data(), out,
                    &a, &max_tiles, &kv_total));
  const int64_t C = cand_offsets_host[B];
  const size_t need = stca_full_layout(nullptr, B, C, kv_total, D, heads, d_h, dtype, nullptr);
  if (!workspace || ws_bytes < need)
    return fail(SA_ERR_WORKSPACE, "workspace needs " + std::to_string(need) + " bytes");
  SA_TRY(check_ptr(workspace, "workspace"));
  StcaFullWork w;
  stca_full_layout(workspace, B, C, kv_total, D, heads, d_h, dtype, &w);
  w.attn.max_tiles = max_tiles;
  return stca_full_run(a, layers, kv_total, w, (cudaStream_t)stream);
}

}  // extern "C"

namespace {
// Shape of a backward call from its host offsets (no validation beyond sizes).
StcaBwdShape bwd_shape(int B, const int64_t* cand, const int64_t* kb, const int64_t* ke, int D, int heads,
                       int d_h, int n_layers, sa_dtype dtype) {
  StcaBwdShape sh{};
  sh.C = cand[B];
  for (int u = 0; u < B; ++u) {
    sh.kv_total += ke[u] - kb[u];
    sh.max_rows_x_keys =
        std::max(sh.max_rows_x_keys, (cand[u + 1] - cand[u]) * heads * score_pitch(ke[u] - kb[u]));
  }
  sh.D = D; sh.heads = heads; sh.d_h = d_h; sh.n_layers = n_layers; sh.dtype = dtype;
  return sh;
}
}  // namespace

extern "C" {

sa_status sa_measure_exp2_rate(int mode, double* per_second, sa_stream_t stream) {
  if ((mode != 0 && mode != 1) || !per_second) return fail(SA_ERR_INVALID_ARG, "mode must be 0 or 1, per_second non-NULL");
  return measure_exp2_rate(mode, per_second, (cudaStream_t)stream);
}

sa_status sa_selftest_bounded_wait(long long budget_cycles, sa_stream_t stream) {
  if (budget_cycles < 1 || budget_cycles > 4000000000LL) return fail(SA_ERR_INVALID_ARG, "budget out of range");
  return selftest_bounded_wait(budget_cycles, (cudaStream_t)stream);
}

sa_status sa_gather_events(const void* item_table, int64_t vocab, const void* action_table, int n_actions,
                           const int32_t* item_ids, const uint8_t* action_ids, int64_t n, int d, void* X,
                           sa_stream_t stream) {
  if (n < 0 || vocab < 1 || n_actions < 1 || n_actions > 256) return fail(SA_ERR_INVALID_ARG, "bad sizes");
  if (d < 8 || d % 8 != 0) return fail(SA_ERR_UNSUPPORTED, "d must be a positive multiple of 8");
  SA_TRY(check_ptr(item_table, "item_table"));
  SA_TRY(check_ptr(action_table, "action_table"));
  // the ids are read element by element: any alignment of their type will do
  if (n > 0 && (!item_ids || !action_ids)) return fail(SA_ERR_INVALID_ARG, "item_ids or action_ids is NULL");
  if (((uintptr_t)item_ids & 3) != 0) return fail(SA_ERR_INVALID_ARG, "item_ids is not 4-byte aligned");
  SA_TRY(check_ptr(X, "X", n == 0));
  return gather_events_run(item_table, vocab, action_table, n_actions, item_ids, action_ids, n, d, X,
                           (cudaStream_t)stream);
}

size_t sa_gather_events_fused_workspace(int n_actions, int d, int d_ff) {
  if (n_actions < 1 || n_actions > 16 || d != 128 || d_ff != 2 * d) return 0;
  return events_ffn_layout(nullptr, n_actions, nullptr);
}

sa_status sa_gather_events_fused(const void* item_table, int64_t vocab, const void* action_table, int n_actions,
                                 const int32_t* item_ids, const uint8_t* action_ids, int64_t n, int d,
                                 const float* W1, const float* W3, const float* W2, int d_ff, void* X,
                                 void* workspace, size_t ws_bytes, sa_stream_t stream) {
  if (n < 0 || vocab < 1 || n_actions < 1) return fail(SA_ERR_INVALID_ARG, "bad sizes");
  if (d != 128 || d_ff != 2 * d || n_actions > 16)
    return fail(SA_ERR_UNSUPPORTED, "the fused event rows take d = 128, d_ff = 256 and 1..16 action types");
  SA_TRY(check_ptr(item_table, "item_table"));
  SA_TRY(check_ptr(action_table, "action_table"));
  if (n > 0 && (!item_ids || !action_ids)) return fail(SA_ERR_INVALID_ARG, "item_ids or action_ids is NULL");
  if (((uintptr_t)item_ids & 3) != 0) return fail(SA_ERR_INVALID_ARG, "item_ids is not 4-byte aligned");
  SA_TRY(check_ptr(W1, "W1"));
  SA_TRY(check_ptr(W3, "W3"));
  SA_TRY(check_ptr(W2, "W2"));
  SA_TRY(check_ptr(X, "X", n == 0));
  const size_t need = events_ffn_layout(nullptr, n_actions, nullptr);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return fail(SA_ERR_WORKSPACE, "workspace too small or unaligned: need " + std::to_string(need) + " bytes");
  EventsFfnWork w;
  events_ffn_layout(workspace, n_actions, &w);
  return events_ffn_run((const __nv_bfloat16*)item_table, vocab, (const __nv_bfloat16*)action_table, n_actions,
                        item_ids, action_ids, n, W1, W3, W2, (__nv_bfloat16*)X, w, (cudaStream_t)stream);
}

size_t stca_backward_full_workspace(int B, const int64_t* cand_offsets_host, const int64_t* kv_begin_host,
                                    const int64_t* kv_end_host, int D, int heads, int d_h, int n_layers,
                                    sa_dtype dtype) {
  if (B < 1 || !cand_offsets_host || !kv_begin_host || !kv_end_host || D < 1 || heads < 1 || d_h < 1 ||
      n_layers < 1 || (dtype != SA_F32 && dtype != SA_BF16))
    return 0;
  for (int u = 0; u < B; ++u)
    if (kv_end_host[u] < kv_begin_host[u] || cand_offsets_host[u + 1] < cand_offsets_host[u]) return 0;
  return stca_bwd_layout(nullptr, bwd_shape(B, cand_offsets_host, kv_begin_host, kv_end_host, D, heads, d_h,
                                            n_layers, dtype), nullptr);
}

sa_status stca_backward_full(const void* q, sa_dtype dtype, const int64_t* cand_offsets_host,
                             const int64_t* cand_offsets_dev, int B, const void* kv, int64_t kv_rows,
                             const int64_t* kv_begin_host, const int64_t* kv_end_host,
                             const int64_t* kv_begin_dev, const int64_t* kv_end_dev, int D, int heads,
                             int d_h, int n_layers, const stca_full_layer* layers, const float* dout,
                             float* dq, float* dkv, const stca_full_layer_grad* grads, void* workspace,
                             size_t ws_bytes, sa_stream_t stream) {
  if (n_layers < 1 || !layers) return fail(SA_ERR_INVALID_ARG, "need n_layers >= 1 and layers");
  if (!grads) return fail(SA_ERR_INVALID_ARG, "grads is NULL");
  std::vector<const stca_layer*> attn(n_layers);
  for (int l = 0; l < n_layers; ++l) {
    const stca_full_layer& L = layers[l];
    const stca_full_layer_grad& G = grads[l];
    attn[l] = &L.attn;
    const int nh = !!L.hist_W1 + !!L.hist_W3 + !!L.hist_W2, nq = !!L.q_W1 + !!L.q_W3 + !!L.q_W2;
    if ((nh != 0 && nh != 3) || (nq != 0 && nq != 3))
      return fail(SA_ERR_INVALID_ARG, "layer " + std::to_string(l) + ": an FFN is partly given");
    const float* need[] = {G.dW_Q, G.dW_K, G.dW_V};
    for (const float* g : need) SA_TRY(check_ptr(g, "grads[] attention weight gradient"));
    if (L.attn.W_O) SA_TRY(check_ptr(G.dW_O, "grads[].dW_O"));
    if (nh) for (const float* g : {G.hist_dW1, G.hist_dW3, G.hist_dW2}) SA_TRY(check_ptr(g, "grads[] history FFN gradient"));
    if (nq) for (const float* g : {G.q_dW1, G.q_dW3, G.q_dW2}) SA_TRY(check_ptr(g, "grads[] query FFN gradient"));
  }
  StcaArgs a;
  int max_tiles = 0;
  int64_t kv_total = 0;
  SA_TRY(stca_check(q, dtype, cand_offsets_host, cand_offsets_dev, B, kv, kv_rows, kv_begin_host,
                    kv_end_host, kv_begin_dev, kv_end_dev, D, heads, d_h, n_layers, attn.data(), nullptr,
                    &a, &max_tiles, &kv_total, true));
  const int64_t C = cand_offsets_host[B];
  SA_TRY(check_ptr(dout, "dout", C == 0));
  SA_TRY(check_ptr(dq, "dq", true));
  SA_TRY(check_ptr(dkv, "dkv", true));
  const StcaBwdShape sh = bwd_shape(B, cand_offsets_host, kv_begin_host, kv_end_host, D, heads, d_h, n_layers, dtype);
  if (sh.max_rows_x_keys >= (1LL << 31) || sh.kv_total >= (1LL << 31) || C * heads >= (1LL << 31))
    return fail(SA_ERR_UNSUPPORTED, "a user's score matrix or the row counts must be < 2^31 elements");
  const size_t need = stca_bwd_layout(nullptr, sh, nullptr);
  if (!workspace || ws_bytes < need)
    return fail(SA_ERR_WORKSPACE, "workspace needs " + std::to_string(need) + " bytes");
  SA_TRY(check_ptr(workspace, "workspace"));
  StcaBwdWork w;
  stca_bwd_layout(workspace, sh, &w);
  std::vector<int64_t> kpre(B + 1, 0);
  for (int u = 0; u < B; ++u) kpre[u + 1] = kpre[u] + (kv_end_host[u] - kv_begin_host[u]);
  StcaBwdHost hst{cand_offsets_host, kv_begin_host, kv_end_host, kpre.data(), kv_total};
  return stca_backward_run(a, hst, layers, grads, dout, dq, dkv, w, (cudaStream_t)stream);
}

sa_status stca_fuse(const float* z_r, const float* z_u, const float* W_F, const float* b_F,
                    int64_t C, int D, float* out, sa_stream_t stream) {
  if (C < 0 || D < 1) return fail(SA_ERR_INVALID_ARG, "bad sizes");
  if (C > 0) {
    SA_TRY(check_ptr(z_r, "z_r"));
    SA_TRY(check_ptr(z_u, "z_u"));
    SA_TRY(check_ptr(out, "out"));
  }
  SA_TRY(check_ptr(W_F, "W_F"));
  SA_TRY(check_ptr(b_F, "b_F", true));
  return stca_fuse_run(z_r, z_u, W_F, b_F, C, D, out, (cudaStream_t)stream);
}

}  // extern "C"
