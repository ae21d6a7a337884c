// Token-wise normalisation variant of Sketch Attention: the same affinities as
// SA (SequenceO1 Sec. 3.1, eq. (6)), normalised over each prototype's tokens
// instead of over each token's prototypes -- the "vanilla attention" baseline
// the pages compare SA with (Table 1; Perceiver-style latent queries, Sec. 2).
//   A_{j,i} = exp S_{j,i} / sum_i' exp S_{j,i'},  H = A X,  m_j = sum_i A_{j,i}
//   S_out = diag(1/(m+eps)) H W_V
// This is attention with the k folded prototypes as queries and the user's
// events as keys and values, so it runs on the STCA tensor-core attention
// kernel: one query row per (user, prototype), key range = the user's events.
#include <algorithm>

#include "gemm.cuh"
#include "sa_internal.cuh"
#include "stca_internal.cuh"

namespace sa {

namespace {
// cand[u] = u k (query rows of user u), prefix[u] = u ceil(k/128) (query
// tiles), and Ub = P' repeated for every user.
__global__ void __launch_bounds__(256) tokenwise_setup_kernel(const __nv_bfloat16* __restrict__ Pb, int B,
                                                              int k, int d, int64_t* __restrict__ cand,
                                                              int* __restrict__ prefix,
                                                              __nv_bfloat16* __restrict__ Ub) {
  const int64_t per = (int64_t)k * d;
  const int tiles = (k + 127) / 128;
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < (int64_t)B * per;
       i += (int64_t)gridDim.x * 256)
    Ub[i] = Pb[i % per];
  if (blockIdx.x == 0)
    for (int u = threadIdx.x; u <= B; u += 256) {
      cand[u] = (int64_t)u * k;
      prefix[u] = u * tiles;
    }
}

// mass = 1 for a user with events (0 without), H copied out, Hhat = H/(m+eps)
__global__ void __launch_bounds__(256) tokenwise_finish_kernel(const int64_t* __restrict__ off, int k, int d,
                                                               float eps, const float* __restrict__ Y,
                                                               float* __restrict__ H, float* __restrict__ mass,
                                                               float* __restrict__ Hhat, int64_t rows) {
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < rows * d; i += (int64_t)gridDim.x * 256) {
    const int64_t r = i / d;
    const int u = (int)(r / k);
    const float m = off[u + 1] > off[u] ? 1.f : 0.f;
    const float den = m + eps;
    const float y = Y[i];
    if (H) H[i] = y;
    Hhat[i] = den > 0.f ? y / den : 0.f;
    if (i % d == 0) mass[r] = m;
  }
}

unsigned blocks_for(int64_t n) {
  return (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 1 << 16));
}
}  // namespace

size_t tokenwise_layout(void* base, int B, int k, int d, TokenwiseWork* w) {
  Carve c(base);
  TokenwiseWork v;
  const size_t bkd = (size_t)B * k * d;
  v.T = c.take<float>((size_t)d * d);
  v.Pf = c.take<float>((size_t)k * d);
  v.Pb = c.take<__nv_bfloat16>((size_t)k * d);
  v.Ub = c.take<__nv_bfloat16>(bkd);
  v.Y = c.take<float>(bkd);
  v.Hhat = c.take<float>(bkd);
  v.cand = c.take<int64_t>((size_t)B + 1);
  v.prefix = c.take<int>((size_t)B + 1);
  if (w) *w = v;
  return c.bytes();
}

sa_status sa_tokenwise_run(const SaFwdArgs& a, const TokenwiseWork& w, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * a.k;
  sa_status s;
  // P' = P W_Q W_K^T log2(e)/sqrt(d): the affinities of eq. (6) in base-2 units
  if ((s = sa_fold(a.k, a.d, a.P, a.W_Q, a.W_K, w.T, w.Pf, w.Pb, st)) != SA_OK) return s;
  SA_TIMED("tokenwise_setup_kernel", st,
           (tokenwise_setup_kernel<<<blocks_for(rows * a.d), 256, 0, st>>>(w.Pb, a.B, a.k, a.d, w.cand,
                                                                           w.prefix, w.Ub)));
  // attention of each prototype over its user's events (K = V = X): Y = A X
  StcaArgs sa_args{};
  sa_args.dtype = SA_BF16;
  sa_args.cand_dev = w.cand;
  sa_args.B = a.B;
  sa_args.C_total = rows;
  sa_args.kv = a.X;
  sa_args.kv_rows = a.n_total;
  sa_args.kvb_dev = a.off_dev;          // the user's events: [off[u], off[u+1])
  sa_args.kve_dev = a.off_dev + 1;
  sa_args.D = a.d;
  sa_args.heads = 1;
  sa_args.d_h = a.d;
  StcaWork sw{};
  sw.Ub = w.Ub;
  sw.Y = w.Y;
  sw.tile_prefix = w.prefix;
  sw.max_tiles = (int)std::max<int64_t>(1, (int64_t)a.B * ((a.k + 127) / 128));
  if ((s = stca_tc_attention(sa_args, sw, st)) != SA_OK) return s;
  SA_TIMED("tokenwise_finish_kernel", st,
           (tokenwise_finish_kernel<<<blocks_for(rows * a.d), 256, 0, st>>>(a.off_dev, a.k, a.d, a.eps, w.Y,
                                                                            a.H, a.mass, w.Hhat, rows)));
  // S = Hhat W_V (and its bf16 copy)
  Gemm g;
  g.M = (int)rows; g.N = a.d; g.K = a.d;
  g.A = w.Hhat; g.lda = a.d;
  g.B = a.W_V; g.ldb = a.d;
  g.C = a.S; g.ldc = a.d;
  g.C16 = (__nv_bfloat16*)a.S_bf16; g.ldc16 = a.d; g.tag = "gemm:S_proj";
  return gemm(g, st);
}

}  // namespace sa
