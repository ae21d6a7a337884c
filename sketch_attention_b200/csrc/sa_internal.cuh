// Internal interfaces between the C-ABI layer (api.cu) and the SA kernels.
#pragma once
#include "common.cuh"
#include "gemm.cuh"

namespace sa {

struct SaFwdArgs {
  const void* X; sa_dtype x_dtype;
  const int64_t* off_dev; int B; int64_t n_total;
  int k, d;
  const float *P, *W_Q, *W_K, *W_V;
  float eps;
  float* S; float* mass; float* H; void* S_bf16; float* lse_out;
  int p_user_rows = 0;   // k: P is [B, k, d], one set of prototypes per user; 0: P is [k, d]
};

// Workspace views of sa_forward.
struct SaFwdWork {
  Chunking ch;
  float* T;             // [d, d]   W_Q W_K^T
  float* Pf;            // [k, d]   folded prototypes, log2 units, fp32
  __nv_bfloat16* Pb;    // [k, d]   same, bf16 (tensor-core operand)
  float* lse;           // [n_total] per-token log2-sum-exp (NULL: the caller's lse output holds it)
  float* Muser;         // [B, k]   mass of users that lie in one chunk
  float* slotH;         // [G, 2, k, d]
  float* slotM;         // [G, 2, k]
  float* Hhat;          // [B, k, d] H/(m+eps)
  // the output projection on the tensor cores (bf16 inputs, d = 128; NULL: the fp32 GEMM):
  // hi + lo bf16 splits of Hhat [B, k, d] and of W_V [d, d]
  __nv_bfloat16* Hhi = nullptr;
  __nv_bfloat16* Hlo = nullptr;
  __nv_bfloat16* Vhi = nullptr;
  __nv_bfloat16* Vlo = nullptr;
};

struct SaBwdArgs {
  const void* X; sa_dtype x_dtype;
  const int64_t* off_dev; int B; int64_t n_total;
  int k, d;
  const float *P, *W_Q, *W_K, *W_V;
  float eps;
  const float *H, *mass, *dS, *dmass, *lse_in;
  void* dX; float *dP, *dW_Q, *dW_K, *dW_V;
  bool accumulate = false;   // add the weight gradients into dP, dW_Q, dW_K, dW_V
  float* dX32 = nullptr;     // tensor-core path: dX as fp32 [n, d] instead of dX (added to when dX_acc)
  bool dX_acc = false;
  // tensor-core path with per-user prototypes (the refinement's later iterations): user u's
  // folded prototypes are rows u k.. of w.Pb, and E is kept per user (w.Euser) instead of
  // summed over the batch
  bool per_user = false;
};

struct SaBwdWork {
  Chunking ch;          // chunks of the per-token kernel
  Chunking chE;         // chunks of the E = dZ X accumulation
  float* T;             // [d, d]
  float* Pf;            // [k, d]
  __nv_bfloat16* Pb;    // [k, d]
  float* lse;           // [n_total]
  float* cbuf;          // [n_total]  c_t
  float* dHh;           // [B, k, d]  dS W_V^T
  float* Hhat;          // [B, k, d]
  float* dH;            // [B, k, d]
  __nv_bfloat16* dHb;   // [B, k, d]  bf16 copy (tensor-core path)
  __nv_bfloat16* dHlo;  // [B, k, d]  bf16 residual dH - dHb (tensor-core path)
  float* dm;            // [B, k]
  float* dmc;           // [B, k]     dm centred per user (tensor-core path)
  float* Epart;         // [chE.G, k, d]
  // the projection GEMMs on the tensor cores (bf16 inputs, d = 128; NULL: fp32 GEMMs): hi + lo
  // bf16 splits of dS and Hhat [B, k, d] and of W_V [d, d]
  __nv_bfloat16* dShi = nullptr;
  __nv_bfloat16* dSlo = nullptr;
  __nv_bfloat16* Hhi = nullptr;
  __nv_bfloat16* Hlo = nullptr;
  __nv_bfloat16* Vhi = nullptr;
  __nv_bfloat16* Vlo = nullptr;
  float* Euser;         // per_user: [B, k, d] each user's E
  float* slotE;         // per_user: [chE.G, 2, k, d] pieces of users that span E chunks
  float* E;             // [k, d]
  float* dQ;            // [k, d]
  float* Q;             // [k, d]
  float* gsplit;        // [kMaxSplit, d, d] split-K partials of the weight-gradient GEMMs
};
constexpr int kMaxSplit = 256;

sa_status sa_fold(int k, int d, const float* P, const float* W_Q, const float* W_K, float* T,
                  float* Pf, __nv_bfloat16* Pb, cudaStream_t st);
sa_status sa_simt_forward(const SaFwdArgs& a, const SaFwdWork& w, cudaStream_t st);
// Stacked refinement (sa_refine.cu): buffers besides the forward's workspace.
struct RefineWork {
  float* Huser;   // [B, k, d] the forward's per-user accumulator
  float* H;       // [B, k, d] A X
  float* mass;    // [B, k]
  float* Xbar;    // [B, k, d]
  float* G1;      // [B, k, 2d]
  float* G3;      // [B, k, 2d]
  float* U;       // [B, k, 2d]
  float* F;       // [B, k, d]
};
// Lays out the forward workspace (P' per user) and the refinement buffers;
// returns the bytes needed.
size_t refine_layout(void* base, int B, int64_t n, int k, int d, SaFwdWork* w, RefineWork* r);
sa_status sa_refine_run(const void* X, sa_dtype x_dtype, const int64_t* off_dev, int B, int64_t n,
                        int k, int d, const float* P0, int n_iter, const sa_refine_layer* layers,
                        float ln_eps, float* sketch, const SaFwdWork& w, const RefineWork& r,
                        cudaStream_t st);

// Backward of the stacked refinement (sa_refine_bwd.cu).
size_t refine_bwd_layout(void* base, int B, int64_t n, int k, int d, int n_iter, void* views);
sa_status sa_refine_backward_run(const void* X, const int64_t* off_host, const int64_t* off_dev, int B,
                                 int64_t n, int k, int d, const float* P0, int n_iter,
                                 const sa_refine_layer* layers, float ln_eps, const float* dsketch,
                                 float* dX, float* dP0, const sa_refine_layer_grad* grads, void* workspace,
                                 cudaStream_t st);

// Token-wise normalisation variant (sa_tokenwise.cu).
struct TokenwiseWork {
  float* T;              // [d, d]
  float* Pf;             // [k, d]
  __nv_bfloat16* Pb;     // [k, d]
  __nv_bfloat16* Ub;     // [B, k, d] P' for every user (the attention's queries)
  float* Y;              // [B, k, d] A X
  float* Hhat;           // [B, k, d]
  int64_t* cand;         // [B+1] u k
  int* prefix;           // [B+1] query tiles before user u
};
size_t tokenwise_layout(void* base, int B, int k, int d, TokenwiseWork* w);
sa_status sa_tokenwise_run(const SaFwdArgs& a, const TokenwiseWork& w, cudaStream_t st);

// Sums the split-n partials into H (if a.H), the mass and H/(m+eps) (w.Hhat).
sa_status sa_reduce(const SaFwdArgs& a, const SaFwdWork& w, cudaStream_t st);
// exponentials per second over the whole GPU: mode 0 all on the MUFU, mode 1 the
// SA forward's mix (one pair in four on the FMA pipe)
sa_status measure_exp2_rate(int mode, double* per_second, cudaStream_t st);
// a kernel whose only mbarrier wait cannot complete: exercises the bounded-wait path
sa_status selftest_bounded_wait(long long budget_cycles, cudaStream_t st);
// x_i = item[id_i] + action[a_i] for n bf16 rows of width d (a multiple of 8)
sa_status gather_events_run(const void* item, int64_t vocab, const void* action, int n_actions,
                            const int32_t* ids, const uint8_t* acts, int64_t n, int d, void* X,
                            cudaStream_t st);
// out[r] = LN(a[r or r % a_rows] + b[r]) * g + beta over rows of d = 128 (a_rows > 0: a holds
// a_rows rows shared by every block of a_rows output rows); g, beta nullable
sa_status sa_residual_ln(const float* a, int a_rows, const float* b, const float* g, const float* beta, float eps,
                         int64_t rows, int d, float* out, cudaStream_t st);
// out[e] = sum_{g < G} part[g][e] in a fixed order (zeros when G = 0)
sa_status sa_sum_slices(const float* part, int G, int64_t n, float* out, cudaStream_t st);
// U = SiLU(G1) * G3 elementwise over n fp32 values (n a multiple of 4, 16-byte aligned)
sa_status sa_swiglu(const float* G1, const float* G3, int64_t n, float* U, cudaStream_t st);
sa_status sa_reduce_and_project(const SaFwdArgs& a, const SaFwdWork& w, cudaStream_t st);
sa_status sa_backward_run(const SaBwdArgs& a, const SaBwdWork& w, bool tc, cudaStream_t st);
sa_status sa_bwd_weight_grads(const SaBwdArgs& a, const SaBwdWork& w, cudaStream_t st);

// Tensor-core backward (sa_bwd_tc.cu).
bool sa_bwd_tc_supported(sa_dtype x_dtype, int k, int d);
int sa_bwd_tc_dx_chunks();
int sa_bwd_tc_e_chunks(int k);
sa_status sa_bwd_tc_run(const SaBwdArgs& a, const SaBwdWork& w, cudaStream_t st);

// Tensor-core forward (sa_tc.cu).
bool sa_tc_supported(sa_dtype x_dtype, int k, int d);
int sa_tc_num_chunks(int k);       // token chunks of the aggregation kernel (one CTA per slice and chunk)
sa_status sa_tc_forward(const SaFwdArgs& a, const SaFwdWork& w, cudaStream_t st);

}  // namespace sa
