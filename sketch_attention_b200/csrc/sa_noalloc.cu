// sa_forward_noalloc: the tensor-core SA forward for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc or any allocating routine: code that
// runs inside a memory pool it does not own, a plugin whose host application
// forbids device allocations, or a step recorded once and replayed where an
// allocation would break the recording.  This entry point takes the same
// inputs and outputs as sa_forward but no workspace: its scratch memory is the
// file-scope device array below, a fixed 8 MiB that every GPU which loads the
// library holds until the process exits.
//
// Limits (larger sizes return SA_ERR_UNSUPPORTED before any GPU work): bf16
// X, d = 128, k a multiple of 128 with k <= 512, B <= 8 users, any n_total
// < 2^31.  Fewer token chunks are used than sa_forward uses (at most 8
// token chunks), so it is slower than sa_forward on large batches.
//
// Every call shares the array and it keeps the last call's contents.  Nothing
// in it needs to start at zero: every word a call reads was written earlier
// in the same call.  Calls whose work overlaps on the GPU (concurrent streams,
// or several host threads) race on the array; serialise them.
//
// The first call on each device looks up the array's device address with
// cudaGetSymbolAddress (a host-side symbol is not a device address), with
// that device current; make that first call before any stream capture.
#include <mutex>

#include "sa_internal.cuh"

namespace sa {
namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;
constexpr int kMaxUsers = 8, kMaxK = 512, kMaxChunks = 8, kD = 128;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch[64] = {};

sa_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(SA_ERR_UNSUPPORTED, "device index above 63");
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    g_scratch[dev] = p;
  }
  *out = g_scratch[dev];
  return SA_OK;
}

// Scratch views inside the array (same roles as sa_forward's workspace).
// n_lse: tokens whose log-sum-exp needs scratch (0 when the caller passes lse)
size_t layout(void* base, int B, int k, const Chunking& ch, int64_t n_lse, SaFwdWork* w) {
  Carve c(base);
  SaFwdWork v;
  v.ch = ch;
  v.T = c.take<float>((size_t)kD * kD);
  v.Pf = c.take<float>((size_t)k * kD);
  v.Pb = c.take<__nv_bfloat16>((size_t)k * kD);
  v.lse = n_lse > 0 ? c.take<float>((size_t)n_lse) : nullptr;
  v.Muser = c.take<float>((size_t)B * k);
  v.slotH = c.take<float>((size_t)std::max(ch.G, 1) * 2 * k * kD);
  v.slotM = c.take<float>((size_t)std::max(ch.G, 1) * 2 * k);
  v.Hhat = c.take<float>((size_t)B * k * kD);
  if (w) *w = v;
  return c.bytes();
}

}  // namespace
}  // namespace sa

using namespace sa;

extern "C" sa_status sa_forward_noalloc(const void* X, sa_dtype x_dtype,
                                        const int64_t* offsets_host, const int64_t* offsets_dev,
                                        int B, int k, int d, const float* P, const float* W_Q,
                                        const float* W_K, const float* W_V, float eps, float* S,
                                        float* mass, float* H, void* S_bf16, float* lse,
                                        sa_stream_t stream) {
  if (x_dtype != SA_BF16 || d != kD || k < 128 || k % 128 != 0 || k > kMaxK || B < 1 || B > kMaxUsers)
    return fail(SA_ERR_UNSUPPORTED,
                "sa_forward_noalloc takes bf16 X, d = 128, k a multiple of 128 up to 512 and "
                "1..8 users; use sa_forward with a workspace otherwise");
  if (!offsets_host || offsets_host[0] != 0) return fail(SA_ERR_INVALID_ARG, "offsets_host[0] must be 0");
  for (int u = 0; u < B; ++u)
    if (offsets_host[u + 1] < offsets_host[u])
      return fail(SA_ERR_INVALID_ARG, "offsets_host must be non-decreasing");
  const int64_t n = offsets_host[B];
  if (n >= (1LL << 31)) return fail(SA_ERR_UNSUPPORTED, "n_total must be < 2^31");
  if (!(eps >= 0.f)) return fail(SA_ERR_INVALID_ARG, "eps must be >= 0");
  const void* need[] = {offsets_dev, P, W_Q, W_K, W_V, S, mass};
  for (const void* q : need)
    if (!q || !aligned16(q)) return fail(SA_ERR_INVALID_ARG, "a required pointer is NULL or not 16-byte aligned");
  if (n > 0 && (!X || !aligned16(X))) return fail(SA_ERR_INVALID_ARG, "X is NULL or not 16-byte aligned");
  const void* opt[] = {H, S_bf16, lse};
  for (const void* q : opt)
    if (q && !aligned16(q)) return fail(SA_ERR_INVALID_ARG, "an optional output is not 16-byte aligned");
  if (H == S) return fail(SA_ERR_INVALID_ARG, "H must not alias S");

  const Chunking ch = make_chunking(n, std::min(kMaxChunks, sa_tc_num_chunks(k)), 1);
  const int64_t n_lse = lse ? 0 : n;
  if (layout(nullptr, B, k, ch, n_lse, nullptr) > kScratchBytes)
    return fail(SA_ERR_UNSUPPORTED, "sizes exceed the 8 MiB scratch array (pass lse to take "
                                    "the per-token log-sum-exp out of it)");
  void* scratch = nullptr;
  sa_status s = scratch_address(&scratch);
  if (s != SA_OK) return s;
  SaFwdWork w;
  layout(scratch, B, k, ch, n_lse, &w);
  SaFwdArgs a{X, x_dtype, offsets_dev, B, n, k, d, P, W_Q, W_K, W_V, eps, S, mass, H, S_bf16, lse};
  cudaStream_t st = (cudaStream_t)stream;
  if ((s = sa_fold(k, d, P, W_Q, W_K, w.T, w.Pf, w.Pb, st)) != SA_OK) return s;
  if (n > 0 && (s = sa_tc_forward(a, w, st)) != SA_OK) return s;
  return sa_reduce_and_project(a, w, st);
}
