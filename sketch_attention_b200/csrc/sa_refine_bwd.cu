// Backward of the stacked Sketch Attention refinement (SequenceO1 Sec. 3.3,
// eqs. (12)-(16), trained end to end; the pages print no backward, this is the
// chain rule of the forward in sa_refine.cu).
//
// The forward is recomputed with what the backward reads kept per iteration:
// the iteration's prototypes X~ (the first iteration's P0 copied to every user),
// their folded bf16 form P' = X~ W_Q W_K^T log2(e)/sqrt(d), the per-token
// log2-sum-exp, X^ = A X, Xbar = LN(X~ + X^) and F = FFN(Xbar).  Then, from the
// last iteration to the first, with dX~ the gradient of the iteration's output:
//   dY2   = LN backward of (Xbar + F) given dX~            (+ the LN2 gain/bias sums)
//   dXbar = dY2 + FFN backward at Xbar given dY2           (+ dW1, dW3, dW2)
//   dY1   = LN backward of (X~ + X^) given dXbar           (+ the LN1 gain/bias sums)
//   dX~  <- dY1 (the residual) + dQ W_Q^T,  dX^ = dY1
// where the SA part is the backward of X^ = A X_u with the user's own
// prototypes: dA = dX^ . x, c = sum_j A dA, dZ = A (dA - c),
//   dX_u += A^T dX^ + ln2 dZ^T P'_u (the tensor-core dX kernel, P'_u the user's folded prototypes),
//   E_u = sum_t dZ_t^T x_t (the tensor-core E kernel),
//   dQ_u = E_u W_K / sqrt(d),  dW_Q += X~_u^T dQ_u,  dW_K += E_u^T (X~_u W_Q) / sqrt(d).
// The SA backward kernels run once per iteration for the whole batch with
// per-user prototypes (user u's folded P' rows) and keep E per user; dX
// accumulates over the iterations in fp32.  After the first iteration
// dP0 = sum_u dX~_u.
#include <algorithm>
#include <vector>

#include "sa_internal.cuh"
#include "stca_internal.cuh"

namespace sa {

namespace {
constexpr int kMaxIter = 8;
constexpr int LN_ROWS = 64;      // rows per block of the LayerNorm backward (8 warps x 8 rows)

struct RB {
  // per iteration
  float* Xin[kMaxIter];            // [B, k, d] prototypes entering the iteration
  __nv_bfloat16* Pb[kMaxIter];     // [B k, d]  their folded bf16 form
  float* lse[kMaxIter];            // [n]       per-token log2-sum-exp
  float* H[kMaxIter];              // [B, k, d] X^ = A X
  float* Xbar[kMaxIter];           // [B, k, d]
  float* F[kMaxIter];              // [B, k, d] FFN(Xbar)
  // forward scratch
  SaFwdWork fw;
  float *G1, *G3, *U;              // [B k, 2d]
  // backward scratch
  float *dXt, *dXt2, *dY2, *dXbar, *dY1;   // [B, k, d]
  float *Euser, *dQ, *Qall;                // [B, k, d]
  __nv_bfloat16 *dHb, *dHlo;               // [B k, d]
  float *cbuf;                             // [n]
  float *dmz, *dmc;                        // [B, k] zeros (no mass term), centred (zeros)
  float* slotE;                            // [G_E, 2, k, d] E of users spanning E chunks
  float* lnpart;                           // [LN blocks, 2, d]
  float* gsplit;                           // split-K partials of the weight-gradient GEMMs
  FfnBwdScratch fb;
};

size_t layout(void* base, int B, int64_t n, int k, int d, int n_iter, RB* out) {
  Carve c(base);
  RB v;
  const size_t bkd = (size_t)B * k * d, rows = (size_t)B * k;
  const size_t nn = (size_t)std::max<int64_t>(n, 1);
  for (int i = 0; i < n_iter; ++i) {
    v.Xin[i] = c.take<float>(bkd);
    v.Pb[i] = c.take<__nv_bfloat16>(bkd);
    v.lse[i] = c.take<float>(nn);
    v.H[i] = c.take<float>(bkd);
    v.Xbar[i] = c.take<float>(bkd);
    v.F[i] = c.take<float>(bkd);
  }
  v.fw.ch = make_chunking(n, sa_tc_num_chunks(k), 1);
  v.fw.T = c.take<float>((size_t)d * d);
  v.fw.Pf = c.take<float>(bkd);
  v.fw.Pb = nullptr;
  v.fw.lse = nullptr;
  v.fw.Muser = c.take<float>(rows);
  v.fw.slotH = c.take<float>((size_t)std::max(v.fw.ch.G, 1) * 2 * k * d);
  v.fw.slotM = c.take<float>((size_t)std::max(v.fw.ch.G, 1) * 2 * k);
  v.fw.Hhat = c.take<float>(bkd);
  v.G1 = c.take<float>(2 * bkd);
  v.G3 = c.take<float>(2 * bkd);
  v.U = c.take<float>(2 * bkd);
  v.dXt = c.take<float>(bkd);
  v.dXt2 = c.take<float>(bkd);
  v.dY2 = c.take<float>(bkd);
  v.dXbar = c.take<float>(bkd);
  v.dY1 = c.take<float>(bkd);
  v.Euser = c.take<float>(bkd);
  v.dQ = c.take<float>(bkd);
  v.Qall = c.take<float>(bkd);
  v.dHb = c.take<__nv_bfloat16>(bkd);
  v.dHlo = c.take<__nv_bfloat16>(bkd);
  v.cbuf = c.take<float>(nn);
  v.dmz = c.take<float>(rows);
  v.dmc = c.take<float>(rows);
  v.slotE = c.take<float>((size_t)std::max(sa_bwd_tc_e_chunks(k), 1) * 2 * k * d);
  v.lnpart = c.take<float>((rows + LN_ROWS - 1) / LN_ROWS * 2 * d);
  v.gsplit = c.take<float>((size_t)kMaxSplit * d * d);
  v.fb = ffn_bwd_scratch_carve(c, (int64_t)rows, d);
  if (out) *out = v;
  return c.bytes();
}

// out[u, j, :] = P0[j, :]
__global__ void broadcast_rows_kernel(const float* __restrict__ P0, int64_t kd, int B, float* __restrict__ out) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < kd * B; e += (int64_t)gridDim.x * blockDim.x)
    out[e] = P0[e % kd];
}

// out[e] = sum_u in[u * kd + e]
__global__ void sum_users_kernel(const float* __restrict__ in, int64_t kd, int B, float* __restrict__ out) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < kd; e += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int u = 0; u < B; ++u) s += in[(int64_t)u * kd + e];
    out[e] = s;
  }
}

// hi = bf16(x), lo = bf16(x - hi)
__global__ void split_bf16_kernel(const float* __restrict__ x, int64_t n, __nv_bfloat16* __restrict__ hi,
                                  __nv_bfloat16* __restrict__ lo) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const float v = x[e];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    hi[e] = h;
    lo[e] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

// LayerNorm backward over rows of d = 128: with y = a[r] + b[r], xh = (y - mean) rstd and
// z = xh g + beta, given dz: dy = rstd (dz g - mean(dz g) - xh mean(dz g xh)).  One warp per
// row, four features per lane; each block also writes its rows' sums of dz xh (-> dg) and of
// dz (-> dbeta) to part[block][2][d].
__global__ void __launch_bounds__(256) ln_backward_kernel(const float* __restrict__ a, const float* __restrict__ b,
                                                          const float* __restrict__ g, const float* __restrict__ dz,
                                                          float eps, int64_t rows, float* __restrict__ dy,
                                                          float* __restrict__ part) {
  constexpr int D = 128;
  __shared__ float sg[8][D], sb[8][D];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  float ag[4] = {0.f, 0.f, 0.f, 0.f}, ab[4] = {0.f, 0.f, 0.f, 0.f};
  float gv[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) gv[i] = g ? g[lane * 4 + i] : 1.f;
  for (int rr = 0; rr < LN_ROWS / 8; ++rr) {
    const int64_t r = (int64_t)blockIdx.x * LN_ROWS + rr * 8 + warp;
    if (r >= rows) break;
    const float4 x = *(const float4*)(a + r * D + lane * 4), y = *(const float4*)(b + r * D + lane * 4);
    const float v[4] = {x.x + y.x, x.y + y.y, x.z + y.z, x.w + y.w};
    float s = (v[0] + v[1]) + (v[2] + v[3]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / (float)D;
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) q += (v[i] - mean) * (v[i] - mean);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    const float rstd = rsqrtf(q / (float)D + eps);
    const float4 dzz = *(const float4*)(dz + r * D + lane * 4);
    const float dv[4] = {dzz.x, dzz.y, dzz.z, dzz.w};
    float xh[4], dg[4], m1 = 0.f, m2 = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xh[i] = (v[i] - mean) * rstd;
      dg[i] = dv[i] * gv[i];
      m1 += dg[i];
      m2 += dg[i] * xh[i];
      ag[i] += dv[i] * xh[i];
      ab[i] += dv[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      m1 += __shfl_xor_sync(0xffffffffu, m1, o);
      m2 += __shfl_xor_sync(0xffffffffu, m2, o);
    }
    m1 /= (float)D;
    m2 /= (float)D;
    float4 out;
    out.x = rstd * (dg[0] - m1 - xh[0] * m2);
    out.y = rstd * (dg[1] - m1 - xh[1] * m2);
    out.z = rstd * (dg[2] - m1 - xh[2] * m2);
    out.w = rstd * (dg[3] - m1 - xh[3] * m2);
    *(float4*)(dy + r * D + lane * 4) = out;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    sg[warp][lane * 4 + i] = ag[i];
    sb[warp][lane * 4 + i] = ab[i];
  }
  __syncthreads();
  if (threadIdx.x < D) {
    float s1 = 0.f, s2 = 0.f;
    for (int w = 0; w < 8; ++w) {
      s1 += sg[w][threadIdx.x];
      s2 += sb[w][threadIdx.x];
    }
    part[((int64_t)blockIdx.x * 2) * D + threadIdx.x] = s1;
    part[((int64_t)blockIdx.x * 2 + 1) * D + threadIdx.x] = s2;
  }
}

// dg[c] = sum_blocks part[blk][0][c], db[c] = sum_blocks part[blk][1][c] (either output nullable)
__global__ void ln_param_grads_kernel(const float* __restrict__ part, int blocks, int d, float* dg, float* db) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= 2 * d) return;
  const int which = c / d, col = c % d;
  float s = 0.f;
  for (int b = 0; b < blocks; ++b) s += part[((int64_t)b * 2 + which) * d + col];
  float* out = which == 0 ? dg : db;
  if (out) out[col] = s;
}

unsigned grid_for(int64_t n) { return (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 1 << 16)); }

sa_status ln_backward(const float* a, const float* b, const float* g, const float* dz, float eps, int64_t rows,
                      int d, float* dy, float* dgain, float* dbias, float* part, cudaStream_t st) {
  const int blocks = (int)((rows + LN_ROWS - 1) / LN_ROWS);
  if (blocks == 0) return SA_OK;
  SA_TIMED("ln_backward_kernel", st,
           (ln_backward_kernel<<<blocks, 256, 0, st>>>(a, b, g, dz, eps, rows, dy, part)));
  if (dgain || dbias)
    SA_TIMED("ln_param_grads_kernel", st,
             (ln_param_grads_kernel<<<(2 * d + 255) / 256, 256, 0, st>>>(part, blocks, d, dgain, dbias)));
  return SA_OK;
}

Gemm plain(int M, int N, int K, const float* A, int64_t lda, bool ta, const float* Bm, int64_t ldb, bool tb,
           float* C, int64_t ldc, const char* tag) {
  Gemm g;
  g.M = M; g.N = N; g.K = K;
  g.A = A; g.lda = lda; g.transA = ta;
  g.B = Bm; g.ldb = ldb; g.transB = tb;
  g.C = C; g.ldc = ldc; g.tag = tag;
  return g;
}
}  // namespace

size_t refine_bwd_layout(void* base, int B, int64_t n, int k, int d, int n_iter, void* views) {
  return layout(base, B, n, k, d, n_iter, (RB*)views);
}

sa_status sa_refine_backward_run(const void* X, const int64_t* off_host, const int64_t* off_dev, int B,
                                 int64_t n, int k, int d, const float* P0, int n_iter,
                                 const sa_refine_layer* layers, float ln_eps, const float* dsketch,
                                 float* dX, float* dP0, const sa_refine_layer_grad* grads, void* workspace,
                                 cudaStream_t st) {
  if (n_iter > kMaxIter) return fail(SA_ERR_UNSUPPORTED, "the refinement backward takes at most 8 iterations");
  RB v;
  layout(workspace, B, n, k, d, n_iter, &v);
  const int64_t rows = (int64_t)B * k, bkd = rows * d, kd = (int64_t)k * d;
  const float rs = 1.f / sqrtf((float)d);
  sa_status s;

  // ---------------------------------------------------------------- forward, kept per iteration
  SA_TIMED("broadcast_rows_kernel", st, (broadcast_rows_kernel<<<grid_for(bkd), 256, 0, st>>>(P0, kd, B, v.Xin[0])));
  for (int it = 0; it < n_iter; ++it) {
    const sa_refine_layer& L = layers[it];
    SaFwdWork w = v.fw;
    w.Pb = v.Pb[it];
    w.lse = v.lse[it];
    if ((s = sa_fold((int)rows, d, v.Xin[it], L.W_Q, L.W_K, w.T, w.Pf, w.Pb, st)) != SA_OK) return s;
    // (S: the forward's per-user H rows, mass: its masses; both scratch here)
    SaFwdArgs a{X, SA_BF16, off_dev, B, n, k, d, v.Xin[it], L.W_Q, L.W_K, nullptr, 0.f,
                v.G1, v.dQ, v.H[it], nullptr, nullptr};
    a.p_user_rows = k;
    if (n > 0 && (s = sa_tc_forward(a, w, st)) != SA_OK) return s;
    if ((s = sa_reduce(a, w, st)) != SA_OK) return s;
    if ((s = sa_residual_ln(v.Xin[it], 0, v.H[it], L.ln1_g, L.ln1_b, ln_eps, rows, d, v.Xbar[it], st)) != SA_OK)
      return s;
    Gemm g1 = plain((int)rows, 2 * d, d, v.Xbar[it], d, false, L.W1, 2 * d, false, v.G1, 2 * d, "gemm:refine_ffn");
    if ((s = gemm(g1, st)) != SA_OK) return s;
    Gemm g3 = g1;
    g3.B = L.W3; g3.C = v.G3;
    if ((s = gemm(g3, st)) != SA_OK) return s;
    if ((s = sa_swiglu(v.G1, v.G3, rows * 2 * d, v.U, st)) != SA_OK) return s;
    Gemm g2 = plain((int)rows, d, 2 * d, v.U, 2 * d, false, L.W2, d, false, v.F[it], d, "gemm:refine_ffn");
    if ((s = gemm(g2, st)) != SA_OK) return s;
    if (it + 1 < n_iter &&
        (s = sa_residual_ln(v.Xbar[it], 0, v.F[it], L.ln2_g, L.ln2_b, ln_eps, rows, d, v.Xin[it + 1], st)) != SA_OK)
      return s;
  }

  // ---------------------------------------------------------------- backward
  SA_CUDA(cudaMemsetAsync(v.dmz, 0, sizeof(float) * rows, st));
  SA_CUDA(cudaMemcpyAsync(v.dXt, dsketch, sizeof(float) * bkd, cudaMemcpyDeviceToDevice, st));
  for (int it = n_iter - 1; it >= 0; --it) {
    const sa_refine_layer& L = layers[it];
    const sa_refine_layer_grad& G = grads[it];
    // eq. (16): X~out = LN2(Xbar + F),  F = FFN(Xbar)
    if ((s = ln_backward(v.Xbar[it], v.F[it], L.ln2_g, v.dXt, ln_eps, rows, d, v.dY2, L.ln2_g ? G.dln2_g : nullptr,
                         L.ln2_b ? G.dln2_b : nullptr, v.lnpart, st)) != SA_OK)
      return s;
    if ((s = ffn_residual_backward_tc(v.Xbar[it], rows, d, L.W1, L.W3, L.W2, v.dY2, v.dXbar, G.dW1, G.dW3, G.dW2,
                                      v.fb, st)) != SA_OK)
      return s;
    // eq. (15): Xbar = LN1(X~ + X^)
    if ((s = ln_backward(v.Xin[it], v.H[it], L.ln1_g, v.dXbar, ln_eps, rows, d, v.dY1, L.ln1_g ? G.dln1_g : nullptr,
                         L.ln1_b ? G.dln1_b : nullptr, v.lnpart, st)) != SA_OK)
      return s;
    // eq. (14): X^ = A X_u with each user's own prototypes (one launch of each SA
    // backward kernel for the batch; E kept per user)
    SA_TIMED("split_bf16_kernel", st, (split_bf16_kernel<<<grid_for(bkd), 256, 0, st>>>(v.dY1, bkd, v.dHb, v.dHlo)));
    if (n == 0) {
      SA_CUDA(cudaMemsetAsync(v.Euser, 0, sizeof(float) * bkd, st));
    } else {
      SaBwdArgs ab{};
      ab.X = X;
      ab.x_dtype = SA_BF16;
      ab.off_dev = off_dev;
      ab.B = B;
      ab.n_total = n;
      ab.k = k;
      ab.d = d;
      ab.dX = nullptr;
      ab.dX32 = dX;
      ab.dX_acc = it < n_iter - 1;
      ab.per_user = true;
      SaBwdWork wb{};
      wb.ch = make_chunking(n, sa_bwd_tc_dx_chunks(), 1);
      wb.chE = make_chunking(n, sa_bwd_tc_e_chunks(k), 1);
      wb.Pb = v.Pb[it];
      wb.lse = v.lse[it];
      wb.cbuf = v.cbuf;
      wb.dHb = v.dHb;
      wb.dHlo = v.dHlo;
      wb.dm = v.dmz;
      wb.dmc = v.dmc;
      wb.Euser = v.Euser;
      wb.slotE = v.slotE;
      if ((s = sa_bwd_tc_run(ab, wb, st)) != SA_OK) return s;
    }
    // dQ = E W_K / sqrt(d);  dX~ = dY1 + dQ W_Q^T
    Gemm gq = plain((int)rows, d, d, v.Euser, d, false, L.W_K, d, false, v.dQ, d, "gemm:refine_grads");
    gq.alpha = rs;
    if ((s = gemm(gq, st)) != SA_OK) return s;
    Gemm gx = plain((int)rows, d, d, v.dQ, d, false, L.W_Q, d, true, v.dXt2, d, "gemm:refine_grads");
    gx.Cin = v.dY1; gx.ldcin = d;
    if ((s = gemm(gx, st)) != SA_OK) return s;
    // dW_Q = sum_u X~_u^T dQ_u;  dW_K = sum_u E_u^T (X~_u W_Q) / sqrt(d)
    Gemm gwq = plain(d, d, (int)rows, v.Xin[it], d, true, v.dQ, d, false, G.dW_Q, d, "gemm:refine_grads");
    gwq.split_k = gemm_split_for(d, d, (int)rows, kMaxSplit);
    gwq.split_ws = v.gsplit;
    if ((s = gemm(gwq, st)) != SA_OK) return s;
    Gemm gqa = plain((int)rows, d, d, v.Xin[it], d, false, L.W_Q, d, false, v.Qall, d, "gemm:refine_grads");
    if ((s = gemm(gqa, st)) != SA_OK) return s;
    Gemm gwk = plain(d, d, (int)rows, v.Euser, d, true, v.Qall, d, false, G.dW_K, d, "gemm:refine_grads");
    gwk.alpha = rs;
    gwk.split_k = gemm_split_for(d, d, (int)rows, kMaxSplit);
    gwk.split_ws = v.gsplit;
    if ((s = gemm(gwk, st)) != SA_OK) return s;
    std::swap(v.dXt, v.dXt2);
  }
  // the first iteration's prototypes are P0 for every user
  SA_TIMED("sum_users_kernel", st, (sum_users_kernel<<<grid_for(kd), 256, 0, st>>>(v.dXt, kd, B, dP0)));
  return SA_OK;
}

}  // namespace sa
