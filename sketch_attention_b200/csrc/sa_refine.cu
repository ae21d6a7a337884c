// Stacked Sketch Attention refinement (SequenceO1 Sec. 3.3, eqs. (12)-(16)):
// n_iter iterations of
//   X^ = A X_u (the tensor-core forward, per-user prototypes after the first)
//   Xbar = LN(X~ + X^),   X~ = LN(Xbar + FFN(Xbar)),  FFN = SwiGLU of width 2d
// The per-row LayerNorms and the SwiGLU gate are small k x d kernels here; the
// FFN's matrix products use the projection GEMM.
#include <algorithm>

#include "gemm.cuh"
#include "sa_internal.cuh"

namespace sa {

namespace {
// out[r, :] = LN(a[ra, :] + b[r, :]) * g + beta, one warp per row (D = 32 * V
// features, V per lane as float4s); ra = r, or r % a_rows when a holds a_rows
// rows shared by every user (the first iteration's prototypes).  Mean and
// biased variance over D.
template <int V>
__global__ void __launch_bounds__(256) residual_ln_kernel(const float* __restrict__ a, int a_rows,
                                                          const float* __restrict__ b,
                                                          const float* __restrict__ g,
                                                          const float* __restrict__ beta, float eps,
                                                          int64_t rows, float* __restrict__ out) {
  constexpr int D = 32 * V;
  const int64_t r = ((int64_t)blockIdx.x * 256 + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (r >= rows) return;
  const int64_t ra = a_rows > 0 ? r % a_rows : r;
  float v[V];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < V; i += 4) {
    const int c = lane * V + i;
    const float4 x = *(const float4*)(a + ra * D + c), y = *(const float4*)(b + r * D + c);
    v[i] = x.x + y.x; v[i + 1] = x.y + y.y; v[i + 2] = x.z + y.z; v[i + 3] = x.w + y.w;
    sum += (v[i] + v[i + 1]) + (v[i + 2] + v[i + 3]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mean = sum / (float)D;
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < V; ++i) sq += (v[i] - mean) * (v[i] - mean);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  const float rstd = rsqrtf(sq / (float)D + eps);
#pragma unroll
  for (int i = 0; i < V; i += 4) {
    const int c = lane * V + i;
    float4 o;
    o.x = (v[i] - mean) * rstd * (g ? g[c] : 1.f) + (beta ? beta[c] : 0.f);
    o.y = (v[i + 1] - mean) * rstd * (g ? g[c + 1] : 1.f) + (beta ? beta[c + 1] : 0.f);
    o.z = (v[i + 2] - mean) * rstd * (g ? g[c + 2] : 1.f) + (beta ? beta[c + 2] : 0.f);
    o.w = (v[i + 3] - mean) * rstd * (g ? g[c + 3] : 1.f) + (beta ? beta[c + 3] : 0.f);
    *(float4*)(out + r * D + c) = o;
  }
}

// U = SiLU(G1) * G3,  SiLU(x) = x / (1 + e^-x); n4 float4s
__global__ void __launch_bounds__(256) swiglu_kernel(const float4* __restrict__ G1,
                                                     const float4* __restrict__ G3, int64_t n4,
                                                     float4* __restrict__ U) {
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n4; i += (int64_t)gridDim.x * 256) {
    const float4 x = G1[i], y = G3[i];
    U[i] = make_float4(x.x / (1.f + expf(-x.x)) * y.x, x.y / (1.f + expf(-x.y)) * y.y,
                       x.z / (1.f + expf(-x.z)) * y.z, x.w / (1.f + expf(-x.w)) * y.w);
  }
}

unsigned blocks_for(int64_t n, int per_block) {
  return (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + per_block - 1) / per_block, 1 << 20));
}
}  // namespace

sa_status sa_residual_ln(const float* a, int a_rows, const float* b, const float* g, const float* beta, float eps,
                         int64_t rows, int d, float* out, cudaStream_t st) {
  if (rows <= 0) return SA_OK;
  if (d != 128) return fail(SA_ERR_UNSUPPORTED, "the LayerNorm kernels take d = 128");
  SA_TIMED("residual_ln_kernel", st,
           (residual_ln_kernel<4><<<blocks_for(rows * 32, 256), 256, 0, st>>>(a, a_rows, b, g, beta, eps, rows, out)));
  return SA_OK;
}

sa_status sa_swiglu(const float* G1, const float* G3, int64_t n, float* U, cudaStream_t st) {
  if (n <= 0) return SA_OK;
  SA_TIMED("swiglu_kernel", st,
           (swiglu_kernel<<<blocks_for(n / 4, 256), 256, 0, st>>>((const float4*)G1, (const float4*)G3,
                                                                 n / 4, (float4*)U)));
  return SA_OK;
}

size_t refine_layout(void* base, int B, int64_t n, int k, int d, SaFwdWork* w, RefineWork* r) {
  Carve c(base);
  SaFwdWork v;
  v.ch = make_chunking(n, sa_tc_num_chunks(k), 1);
  const size_t bkd = (size_t)B * k * d;
  v.T = c.take<float>((size_t)d * d);
  v.Pf = c.take<float>(bkd);                       // P' of every user (the first iteration uses k rows)
  v.Pb = c.take<__nv_bfloat16>(bkd);
  v.lse = c.take<float>((size_t)std::max<int64_t>(n, 1));
  v.Muser = c.take<float>((size_t)B * k);
  v.slotH = c.take<float>((size_t)std::max(v.ch.G, 1) * 2 * k * d);
  v.slotM = c.take<float>((size_t)std::max(v.ch.G, 1) * 2 * k);
  v.Hhat = c.take<float>(bkd);
  RefineWork q;
  q.Huser = c.take<float>(bkd);
  q.H = c.take<float>(bkd);
  q.mass = c.take<float>((size_t)B * k);
  q.Xbar = c.take<float>(bkd);
  q.G1 = c.take<float>(2 * bkd);
  q.G3 = c.take<float>(2 * bkd);
  q.U = c.take<float>(2 * bkd);
  q.F = c.take<float>(bkd);
  if (w) *w = v;
  if (r) *r = q;
  return c.bytes();
}

sa_status sa_refine_run(const void* X, sa_dtype x_dtype, const int64_t* off_dev, int B, int64_t n,
                        int k, int d, const float* P0, int n_iter, const sa_refine_layer* layers,
                        float ln_eps, float* sketch, const SaFwdWork& w, const RefineWork& r,
                        cudaStream_t st) {
  const int64_t rows = (int64_t)B * k;
  sa_status s;
  for (int it = 0; it < n_iter; ++it) {
    const sa_refine_layer& L = layers[it];
    const bool per_user = it > 0;
    const float* Xt = per_user ? sketch : P0;      // X~(it): shared [k, d], then [B, k, d]
    // eq. (12): P' = X~ W_Q W_K^T log2(e)/sqrt(d), one set per user after the first iteration
    if ((s = sa_fold(per_user ? (int)rows : k, d, Xt, L.W_Q, L.W_K, w.T, w.Pf, w.Pb, st)) != SA_OK)
      return s;
    // eqs. (13)-(14): X^ = A X_u (H; the mass and S projection are not used here)
    SaFwdArgs a{X, x_dtype, off_dev, B, n, k, d, Xt, L.W_Q, L.W_K, nullptr, 0.f,
                r.Huser, r.mass, r.H, nullptr, nullptr};
    a.p_user_rows = per_user ? k : 0;
    if (n > 0 && (s = sa_tc_forward(a, w, st)) != SA_OK) return s;
    if ((s = sa_reduce(a, w, st)) != SA_OK) return s;
    // eq. (15): Xbar = LN(X~ + X^)
    SA_TIMED("residual_ln_kernel", st,
             (residual_ln_kernel<4><<<blocks_for(rows * 32, 256), 256, 0, st>>>(
                 Xt, per_user ? 0 : k, r.H, L.ln1_g, L.ln1_b, ln_eps, rows, r.Xbar)));
    // eq. (16): FFN(Xbar) = (SiLU(Xbar W1) * (Xbar W3)) W2
    Gemm g1;
    g1.M = (int)rows; g1.N = 2 * d; g1.K = d;
    g1.A = r.Xbar; g1.lda = d; g1.B = L.W1; g1.ldb = 2 * d; g1.C = r.G1; g1.ldc = 2 * d;
    g1.tag = "gemm:refine_ffn";
    if ((s = gemm(g1, st)) != SA_OK) return s;
    Gemm g3 = g1;
    g3.B = L.W3; g3.C = r.G3;
    if ((s = gemm(g3, st)) != SA_OK) return s;
    if ((s = sa_swiglu(r.G1, r.G3, rows * 2 * d, r.U, st)) != SA_OK) return s;
    Gemm g2;
    g2.M = (int)rows; g2.N = d; g2.K = 2 * d;
    g2.A = r.U; g2.lda = 2 * d; g2.B = L.W2; g2.ldb = d; g2.C = r.F; g2.ldc = d;
    g2.tag = "gemm:refine_ffn";
    if ((s = gemm(g2, st)) != SA_OK) return s;
    // X~(it+1) = LN(Xbar + FFN), written over X~(it) (no longer read)
    SA_TIMED("residual_ln_kernel", st,
             (residual_ln_kernel<4><<<blocks_for(rows * 32, 256), 256, 0, st>>>(
                 r.Xbar, 0, r.F, L.ln2_g, L.ln2_b, ln_eps, rows, sketch)));
  }
  return SA_OK;
}

}  // namespace sa
