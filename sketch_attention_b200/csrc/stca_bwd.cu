// Backward of one STCA branch of full layers (SequenceO1 Sec. 2.3 eq. (4),
// Sec. 5.1 eqs. (24)-(27)): gradients of <dout, out> with respect to the
// queries, the key rows and every weight.
//
// fp32 throughout (bf16 inputs are widened once).  The forward is recomputed
// layer by layer, keeping each layer's query states, head projections,
// attention outputs and transformed key rows; the attention itself is
// evaluated per user with its score matrix materialised (R_u = C_u * heads
// rows by L_u keys) and recomputed in the backward:
//   S = U X^T (U = (q W_Q^h) W_K^h^T / sqrt(d_h)),  P = softmax_rows(S),  Y = P X
//   dP = dY X^T,  dS = P o (dP - rowsum(dY o Y)),  dU = dS X,
//   dX += dS^T U + P^T dY        (K = V = X)
// then the head projections, W_O and the two SwiGLU FFNs by their chain
// rules.  With bf16 inputs the six attention products per user and layer run
// on the tensor cores (tc_gemm.cu) with bf16 copies of U, X, dY, P and dS; with
// fp32 inputs, and for every other contraction, the fp32 projection GEMM.
// Users are processed in order on the stream, so the results are deterministic.
#include <algorithm>
#include <cmath>

#include "sa_internal.cuh"
#include "stca_internal.cuh"

namespace sa {

namespace {
template <class T>
__global__ void widen_kernel(const T* __restrict__ in, int64_t n, float* __restrict__ out) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x)
    out[e] = load_as_f32(in, e);
}

// Xg[j] = kv[kvb[u] + (j - kpre[u])] for the rows of user u (host loop over users)
template <class T>
__global__ void gather_rows_kernel(const T* __restrict__ kv, int64_t src0, int64_t n, int D,
                                   float* __restrict__ dst) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * D; e += (int64_t)gridDim.x * blockDim.x)
    dst[e] = load_as_f32(kv, src0 * D + e);
}

// dst[j] += src[j] over n * D values
__global__ void add_rows_kernel(const float* __restrict__ src, int64_t n, float* __restrict__ dst) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x)
    dst[e] += src[e];
}

// softmax of each row of S [rows, L] (row pitch ld) in place, and its bf16 split
// Pb + Plo (same pitch) when given; one block per row
__global__ void __launch_bounds__(256) softmax_rows_kernel(float* __restrict__ S, int64_t L, int64_t ld,
                                                          __nv_bfloat16* __restrict__ Pb,
                                                          __nv_bfloat16* __restrict__ Plo) {
  __shared__ float red[8];
  float* row = S + (int64_t)blockIdx.x * ld;
  const int lane = threadIdx.x % 32, w = threadIdx.x / 32;
  float m = -INFINITY;
  for (int64_t j = threadIdx.x; j < L; j += 256) m = fmaxf(m, row[j]);
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[w] = m;
  __syncthreads();
  m = red[0];
  for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i]);
  __syncthreads();
  float s = 0.f;
  for (int64_t j = threadIdx.x; j < L; j += 256) {
    const float e = expf(row[j] - m);
    row[j] = e;
    s += e;
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) red[w] = s;
  __syncthreads();
  s = 0.f;
  for (int i = 0; i < 8; ++i) s += red[i];
  const float inv = 1.f / s;
  for (int64_t j = threadIdx.x; j < L; j += 256) {
    const float v = row[j] * inv;
    row[j] = v;
    if (Pb) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      Pb[(int64_t)blockIdx.x * ld + j] = hi;
      Plo[(int64_t)blockIdx.x * ld + j] = __float2bfloat16_rn(v - __bfloat162float(hi));
    }
  }
}

// dS = P o (dP - sum_d dY[r, d] Y[r, d]) in place over dP (row pitch ld), and its bf16
// split dSb + dSlo (same pitch) when given; one block per row
__global__ void __launch_bounds__(256) softmax_bwd_kernel(const float* __restrict__ P, float* __restrict__ dP,
                                                          int64_t L, int64_t ld, const float* __restrict__ dY,
                                                          const float* __restrict__ Y, int D,
                                                          __nv_bfloat16* __restrict__ dSb,
                                                          __nv_bfloat16* __restrict__ dSlo) {
  __shared__ float red[8];
  const int64_t r = blockIdx.x;
  float v = 0.f;
  for (int d = threadIdx.x; d < D; d += 256) v += dY[r * D + d] * Y[r * D + d];
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = v;
  __syncthreads();
  float c = 0.f;
  for (int i = 0; i < 8; ++i) c += red[i];
  for (int64_t j = threadIdx.x; j < L; j += 256) {
    const float v = P[r * ld + j] * (dP[r * ld + j] - c);
    dP[r * ld + j] = v;
    if (dSb) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      dSb[r * ld + j] = hi;
      dSlo[r * ld + j] = __float2bfloat16_rn(v - __bfloat162float(hi));
    }
  }
}

// x = hi + lo with both in bf16 (hi the rounding of x, lo the rounding of the rest):
// products over hi and lo carry x to about 16 bits
__global__ void split_kernel(const float* __restrict__ in, int64_t n, __nv_bfloat16* __restrict__ hi,
                             __nv_bfloat16* __restrict__ lo) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const float x = in[e];
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi[e] = h;
    lo[e] = __float2bfloat16_rn(x - __bfloat162float(h));
  }
}

// dG1 = dU o G3 o SiLU'(G1), dG3 = dU o SiLU(G1); SiLU'(g) = s (1 + g (1 - s)), s = 1/(1+e^-g).
// The outputs may overwrite the inputs element by element (no __restrict__).
__global__ void swiglu_bwd_kernel(const float* G1, const float* G3, const float* dU, int64_t n, float* dG1,
                                  float* dG3) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const float g = G1[e], s = 1.f / (1.f + expf(-g));
    dG1[e] = dU[e] * G3[e] * s * (1.f + g * (1.f - s));
    dG3[e] = dU[e] * g * s;
  }
}

__device__ __forceinline__ void put_split(float v, __nv_bfloat16* hi, __nv_bfloat16* lo, int64_t e) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  hi[e] = h;
  lo[e] = __float2bfloat16_rn(v - __bfloat162float(h));
}

// U = SiLU(G1) * G3, written only as its hi + lo split
__global__ void swiglu_split_kernel(const float* __restrict__ G1, const float* __restrict__ G3, int64_t n,
                                    __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const float g = G1[e];
    put_split(g / (1.f + expf(-g)) * G3[e], hi, lo, e);
  }
}

// dG1 and dG3 as swiglu_bwd_kernel computes them, written only as hi + lo splits
__global__ void swiglu_bwd_split_kernel(const float* __restrict__ G1, const float* __restrict__ G3,
                                        const float* __restrict__ dU, int64_t n, __nv_bfloat16* __restrict__ d1_hi,
                                        __nv_bfloat16* __restrict__ d1_lo, __nv_bfloat16* __restrict__ d3_hi,
                                        __nv_bfloat16* __restrict__ d3_lo) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const float g = G1[e], s = 1.f / (1.f + expf(-g));
    put_split(dU[e] * G3[e] * s * (1.f + g * (1.f - s)), d1_hi, d1_lo, e);
    put_split(dU[e] * g * s, d3_hi, d3_lo, e);
  }
}

unsigned grid_for(int64_t n) { return (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 1 << 16)); }

bool has_hist(const stca_full_layer& L) { return L.hist_W1 != nullptr; }
bool has_query(const stca_full_layer& L) { return L.q_W1 != nullptr; }

// bf16 hi + lo scratch for the FFN products' operands on the tensor cores: x [rows, D],
// two [rows, 2D] slots and the three weights (2 D^2 each)
struct FfnScratch {
  __nv_bfloat16 *x_hi, *x_lo, *a_hi, *a_lo, *b_hi, *b_lo, *w_hi, *w_lo;
};

// The stream, the split-K partials and the split scratch shared by every GEMM of one
// call (they run in stream order); tcp: bf16 inputs, products on the tensor cores.
struct Ctx {
  cudaStream_t st;
  float* split;
  bool tcp;
  FfnScratch fs;
};

// GEMM with split-K when its output tiles alone leave most SMs idle (the weight
// gradients and the per-user P X, dS X products have small outputs and long K)
sa_status mm(Gemm g, const Ctx& cx) {
  if (g.M > 0 && g.N > 0) {
    const int64_t out = (int64_t)g.M * g.N * g.batch;
    int split = gemm_split_for(g.M, g.N * g.batch, g.K, kMaxSplit);
    split = (int)std::min<int64_t>(split, (int64_t)(kStcaBwdSplitFloats / (size_t)std::max<int64_t>(out, 1)));
    if (split > 1) {
      g.split_k = split;
      g.split_ws = cx.split;
    }
  }
  return gemm(g, cx.st);
}

// C = alpha A B (+ Cin) for plain row-major operands
Gemm plain(int M, int N, int K, const float* A, int64_t lda, bool ta, const float* B, int64_t ldb, bool tb,
           float* C, int64_t ldc, const char* tag) {
  Gemm g;
  g.M = M; g.N = N; g.K = K;
  g.A = A; g.lda = lda; g.transA = ta;
  g.B = B; g.ldb = ldb; g.transB = tb;
  g.C = C; g.ldc = ldc; g.tag = tag;
  return g;
}

struct Ffn {
  const float *W1, *W3, *W2;
  float *dW1, *dW3, *dW2;
};

// a bf16 split x = hi + lo of an fp32 operand
struct Split {
  const __nv_bfloat16 *hi, *lo;
  Split at(int64_t off) const { return {hi + off, lo + off}; }
};

// C[M, N] = A B (+ Cin) on the tensor cores over split operands (about 16 significant
// bits each): A K-major or (a_mn) M-major, B K-major or (b_mn) N-major
sa_status tc(int M, int N, int K, Split A, int64_t lda, bool a_mn, Split B, int64_t ldb, bool b_mn, float* C,
             int64_t ldc, const float* Cin, const Ctx& cx, const char* tag = "tc_gemm:stca_bwd_attn") {
  cudaStream_t st = cx.st;
  TcGemm g;
  g.part = cx.split; g.part_floats = kStcaBwdSplitFloats;
  g.M = M; g.N = N; g.K = K;
  g.A = A.hi; g.A_lo = A.lo; g.lda = lda; g.a_mn = a_mn;
  g.B = B.hi; g.B_lo = B.lo; g.ldb = ldb; g.b_mn = b_mn;
  g.C = C; g.ldc = ldc; g.Cin = Cin; g.ldcin = ldc;
  g.tag = tag;
  return tc_gemm(g, st);
}

// hi + lo split of n fp32 values into the given scratch
sa_status split_to(const float* x, int64_t n, __nv_bfloat16* hi, __nv_bfloat16* lo, Split* out, cudaStream_t st) {
  SA_TIMED("split_kernel", st, (split_kernel<<<grid_for(n), 256, 0, st>>>(x, n, hi, lo)));
  *out = {hi, lo};
  return SA_OK;
}

// the FFN's three weights split into the weight scratch: W1, W3 [D, 2D], W2 [2D, D]
sa_status split_weights(const Ffn& f, int D, Split w[3], const Ctx& cx) {
  const float* W[3] = {f.W1, f.W3, f.W2};
  const int64_t n = 2LL * D * D;
  sa_status s;
  for (int i = 0; i < 3; ++i)
    if ((s = split_to(W[i], n, cx.fs.w_hi + i * n, cx.fs.w_lo + i * n, &w[i], cx.st)) != SA_OK) return s;
  return SA_OK;
}

constexpr const char* kFfnTag = "tc_gemm:stca_bwd_ffn";

// y = x + FFN(x) over `rows` rows
sa_status ffn_fwd(const float* x, int64_t rows, int D, const Ffn& f, float* G1, float* G3, float* U, float* y,
                  const Ctx& cx) {
  cudaStream_t st = cx.st;
  if (rows == 0) return SA_OK;
  sa_status s;
  if (cx.tcp) {
    Split w[3], xs, us;
    const int R = (int)rows;
    if ((s = split_weights(f, D, w, cx)) != SA_OK) return s;
    if ((s = split_to(x, rows * D, cx.fs.x_hi, cx.fs.x_lo, &xs, st)) != SA_OK) return s;
    if ((s = tc(R, 2 * D, D, xs, D, false, w[0], 2 * D, true, G1, 2 * D, nullptr, cx, kFfnTag)) != SA_OK) return s;
    if ((s = tc(R, 2 * D, D, xs, D, false, w[1], 2 * D, true, G3, 2 * D, nullptr, cx, kFfnTag)) != SA_OK) return s;
    const int64_t n2 = rows * 2 * D;
    SA_TIMED("swiglu_split_kernel", st,
             (swiglu_split_kernel<<<grid_for(n2), 256, 0, st>>>(G1, G3, n2, cx.fs.a_hi, cx.fs.a_lo)));
    us = {cx.fs.a_hi, cx.fs.a_lo};
    return tc(R, D, 2 * D, us, 2 * D, false, w[2], D, true, y, D, x, cx, kFfnTag);
  }
  if ((s = mm(plain((int)rows, 2 * D, D, x, D, false, f.W1, 2 * D, false, G1, 2 * D, "gemm:stca_bwd_ffn"), cx)) != SA_OK) return s;
  if ((s = mm(plain((int)rows, 2 * D, D, x, D, false, f.W3, 2 * D, false, G3, 2 * D, "gemm:stca_bwd_ffn"), cx)) != SA_OK) return s;
  if ((s = sa_swiglu(G1, G3, rows * 2 * D, U, st)) != SA_OK) return s;
  Gemm g = plain((int)rows, D, 2 * D, U, 2 * D, false, f.W2, D, false, y, D, "gemm:stca_bwd_ffn");
  g.Cin = x; g.ldcin = D;
  return mm(g, cx);
}

// given dy (the gradient of y = x + FFN(x)), dx = dy + dG1 W1^T + dG3 W3^T and the
// weight gradients; dx may alias dy
sa_status ffn_bwd(const float* x, int64_t rows, int D, const Ffn& f, const float* dy, float* dx, float* G1,
                  float* G3, float* U, float* dU, const Ctx& cx) {
  cudaStream_t st = cx.st;
  sa_status s;
  if (rows == 0) {
    for (float* w : {f.dW1, f.dW3, f.dW2})
      SA_CUDA(cudaMemsetAsync(w, 0, sizeof(float) * 2 * D * D, st));
    return SA_OK;
  }
  if (cx.tcp) {
    Split w[3], xs, as, bs;
    const int R = (int)rows;
    const int64_t n1 = rows * D, n2 = rows * 2 * D;
    if ((s = split_weights(f, D, w, cx)) != SA_OK) return s;
    if ((s = split_to(x, n1, cx.fs.x_hi, cx.fs.x_lo, &xs, st)) != SA_OK) return s;
    if ((s = tc(R, 2 * D, D, xs, D, false, w[0], 2 * D, true, G1, 2 * D, nullptr, cx, kFfnTag)) != SA_OK) return s;
    if ((s = tc(R, 2 * D, D, xs, D, false, w[1], 2 * D, true, G3, 2 * D, nullptr, cx, kFfnTag)) != SA_OK) return s;
    // U (split only) = SiLU(G1) * G3;  dW2 = U^T dy (U read M-major);  dU = dy W2^T (W2 read K-major)
    SA_TIMED("swiglu_split_kernel", st,
             (swiglu_split_kernel<<<grid_for(n2), 256, 0, st>>>(G1, G3, n2, cx.fs.a_hi, cx.fs.a_lo)));
    as = {cx.fs.a_hi, cx.fs.a_lo};
    if ((s = split_to(dy, n1, cx.fs.b_hi, cx.fs.b_lo, &bs, st)) != SA_OK) return s;
    if ((s = tc(2 * D, D, R, as, 2 * D, true, bs, D, true, f.dW2, D, nullptr, cx, kFfnTag)) != SA_OK) return s;
    if ((s = tc(R, 2 * D, D, bs, D, false, w[2], D, false, dU, 2 * D, nullptr, cx, kFfnTag)) != SA_OK) return s;
    // dG1 (slot a) and dG3 (slot b), split only: dW1 = x^T dG1, dW3 = x^T dG3,
    // dx = dy + dG1 W1^T + dG3 W3^T
    SA_TIMED("swiglu_bwd_split_kernel", st,
             (swiglu_bwd_split_kernel<<<grid_for(n2), 256, 0, st>>>(G1, G3, dU, n2, cx.fs.a_hi, cx.fs.a_lo,
                                                                    cx.fs.b_hi, cx.fs.b_lo)));
    if ((s = tc(D, 2 * D, R, xs, D, true, as, 2 * D, true, f.dW1, 2 * D, nullptr, cx, kFfnTag)) != SA_OK) return s;
    if ((s = tc(D, 2 * D, R, xs, D, true, bs, 2 * D, true, f.dW3, 2 * D, nullptr, cx, kFfnTag)) != SA_OK) return s;
    if ((s = tc(R, D, 2 * D, as, 2 * D, false, w[0], 2 * D, false, dx, D, dy, cx, kFfnTag)) != SA_OK) return s;
    return tc(R, D, 2 * D, bs, 2 * D, false, w[1], 2 * D, false, dx, D, dx, cx, kFfnTag);
  }
  if ((s = mm(plain((int)rows, 2 * D, D, x, D, false, f.W1, 2 * D, false, G1, 2 * D, "gemm:stca_bwd_ffn"), cx)) != SA_OK) return s;
  if ((s = mm(plain((int)rows, 2 * D, D, x, D, false, f.W3, 2 * D, false, G3, 2 * D, "gemm:stca_bwd_ffn"), cx)) != SA_OK) return s;
  if ((s = sa_swiglu(G1, G3, rows * 2 * D, U, st)) != SA_OK) return s;
  // dW2 = U^T dy;  dU = dy W2^T
  if ((s = mm(plain(2 * D, D, (int)rows, U, 2 * D, true, dy, D, false, f.dW2, D, "gemm:stca_bwd_ffn"), cx)) != SA_OK) return s;
  if ((s = mm(plain((int)rows, 2 * D, D, dy, D, false, f.W2, D, true, dU, 2 * D, "gemm:stca_bwd_ffn"), cx)) != SA_OK) return s;
  // dG1 over U (no longer needed), dG3 over G1 (each element read before it is written)
  SA_TIMED("swiglu_bwd_kernel", st,
           (swiglu_bwd_kernel<<<grid_for(rows * 2 * D), 256, 0, st>>>(G1, G3, dU, rows * 2 * D, U, G1)));
  // now U = dG1, G1 = dG3
  if ((s = mm(plain(D, 2 * D, (int)rows, x, D, true, U, 2 * D, false, f.dW1, 2 * D, "gemm:stca_bwd_ffn"), cx)) != SA_OK) return s;
  if ((s = mm(plain(D, 2 * D, (int)rows, x, D, true, G1, 2 * D, false, f.dW3, 2 * D, "gemm:stca_bwd_ffn"), cx)) != SA_OK) return s;
  Gemm g1 = plain((int)rows, D, 2 * D, U, 2 * D, false, f.W1, 2 * D, true, dx, D, "gemm:stca_bwd_ffn");
  g1.Cin = dy; g1.ldcin = D;
  if ((s = mm(g1, cx)) != SA_OK) return s;
  Gemm g3 = plain((int)rows, D, 2 * D, G1, 2 * D, false, f.W3, 2 * D, true, dx, D, "gemm:stca_bwd_ffn");
  g3.Cin = dx; g3.ldcin = D;
  return mm(g3, cx);
}
}  // namespace

FfnBwdScratch ffn_bwd_scratch_carve(Carve& c, int64_t rows, int D) {
  FfnBwdScratch f;
  const size_t r = (size_t)std::max<int64_t>(rows, 1);
  f.G1 = c.take<float>(r * 2 * D);
  f.G3 = c.take<float>(r * 2 * D);
  f.U = c.take<float>(r * 2 * D);
  f.dU = c.take<float>(r * 2 * D);
  f.split = c.take<float>(kStcaBwdSplitFloats);
  f.x_hi = c.take<__nv_bfloat16>(r * D);
  f.x_lo = c.take<__nv_bfloat16>(r * D);
  f.a_hi = c.take<__nv_bfloat16>(r * 2 * D);
  f.a_lo = c.take<__nv_bfloat16>(r * 2 * D);
  f.b_hi = c.take<__nv_bfloat16>(r * 2 * D);
  f.b_lo = c.take<__nv_bfloat16>(r * 2 * D);
  f.w_hi = c.take<__nv_bfloat16>((size_t)6 * D * D);
  f.w_lo = c.take<__nv_bfloat16>((size_t)6 * D * D);
  return f;
}

sa_status ffn_residual_backward_tc(const float* x, int64_t rows, int D, const float* W1, const float* W3,
                                   const float* W2, const float* dy, float* dx, float* dW1, float* dW3, float* dW2,
                                   const FfnBwdScratch& f, cudaStream_t st) {
  Ctx cx;
  cx.st = st;
  cx.split = f.split;
  cx.tcp = true;
  cx.fs = {f.x_hi, f.x_lo, f.a_hi, f.a_lo, f.b_hi, f.b_lo, f.w_hi, f.w_lo};
  Ffn fn{W1, W3, W2, dW1, dW3, dW2};
  return ffn_bwd(x, rows, D, fn, dy, dx, f.G1, f.G3, f.U, f.dU, cx);
}

sa_status split_hi_lo(const float* x, int64_t n, __nv_bfloat16* hi, __nv_bfloat16* lo, cudaStream_t st) {
  if (n <= 0) return SA_OK;
  SA_TIMED("split_kernel", st, (split_kernel<<<grid_for(n), 256, 0, st>>>(x, n, hi, lo)));
  return SA_OK;
}

size_t stca_bwd_layout(void* base, const StcaBwdShape& sh, StcaBwdWork* w) {
  Carve c(base);
  StcaBwdWork v;
  const size_t C = (size_t)std::max<int64_t>(sh.C, 1), R = (size_t)std::max<int64_t>(sh.kv_total, 1);
  const size_t D = sh.D, HD = (size_t)sh.heads * sh.d_h, H = sh.heads, NL = sh.n_layers;
  v.qin = c.take<float>((NL + 1) * C * D);
  v.qmid = c.take<float>(NL * C * D);
  v.Qh = c.take<float>(NL * C * HD);
  v.U = c.take<float>(NL * C * H * D);
  v.Y = c.take<float>(NL * C * H * D);
  v.O = c.take<float>(NL * C * HD);
  v.Xk = c.take<float>((NL + 1) * R * D);
  const size_t wide = std::max(C, R) * 2 * D;
  v.G1 = c.take<float>(wide);
  v.G3 = c.take<float>(wide);
  v.Uf = c.take<float>(wide);
  v.dUf = c.take<float>(wide);
  const size_t sl = (size_t)std::max<int64_t>(sh.max_rows_x_keys, 1);
  v.S = c.take<float>(sl);
  v.dS = c.take<float>(sl);
  const bool tc = sh.dtype == SA_BF16;        // bf16 inputs: the attention products on the tensor cores
  v.Ub = c.take<__nv_bfloat16>(tc ? NL * C * H * D : 1);
  v.Ulo = c.take<__nv_bfloat16>(tc ? NL * C * H * D : 1);
  v.Xkb = c.take<__nv_bfloat16>(tc ? NL * R * D : 1);
  v.Xklo = c.take<__nv_bfloat16>(tc ? NL * R * D : 1);
  v.dYb = c.take<__nv_bfloat16>(tc ? C * H * D : 1);
  v.dYlo = c.take<__nv_bfloat16>(tc ? C * H * D : 1);
  v.Pb = c.take<__nv_bfloat16>(tc ? sl : 1);
  v.Plo = c.take<__nv_bfloat16>(tc ? sl : 1);
  v.dSb = c.take<__nv_bfloat16>(tc ? sl : 1);
  v.dSlo = c.take<__nv_bfloat16>(tc ? sl : 1);
  const size_t rows_max = std::max(C, R);
  for (__nv_bfloat16** p : {&v.fx_hi, &v.fx_lo}) *p = c.take<__nv_bfloat16>(tc ? rows_max * D : 1);
  for (__nv_bfloat16** p : {&v.fa_hi, &v.fa_lo, &v.fb_hi, &v.fb_lo}) *p = c.take<__nv_bfloat16>(tc ? rows_max * 2 * D : 1);
  for (__nv_bfloat16** p : {&v.fw_hi, &v.fw_lo}) *p = c.take<__nv_bfloat16>(tc ? 6 * D * D : 1);
  v.dq = c.take<float>(C * D);
  v.dqmid = c.take<float>(C * D);
  v.dO = c.take<float>(C * HD);
  v.dY = c.take<float>(C * H * D);
  v.dU = c.take<float>(C * H * D);
  v.dQh = c.take<float>(C * HD);
  v.dX = c.take<float>(R * D);
  v.gsplit = c.take<float>(kStcaBwdSplitFloats);
  if (w) *w = v;
  return c.bytes();
}

sa_status stca_backward_run(const StcaArgs& a, const StcaBwdHost& hst, const stca_full_layer* layers,
                            const stca_full_layer_grad* grads, const float* dout, float* dq_out, float* dkv,
                            const StcaBwdWork& w, cudaStream_t st) {
  const int B = a.B, D = a.D, H = a.heads, dh = a.d_h, HD = H * dh, NL = a.n_layers;
  const int64_t C = a.C_total, R = hst.kv_total;
  const size_t CD = (size_t)C * D, CHD = (size_t)C * HD, CHD2 = (size_t)C * H * D, RD = (size_t)R * D;
  const float inv_sqrt = 1.f / std::sqrt((float)dh);
  sa_status s;
  const bool tcp = a.dtype == SA_BF16;       // the attention and FFN products on the tensor cores
  const Ctx cx{st, w.gsplit, tcp, {w.fx_hi, w.fx_lo, w.fa_hi, w.fa_lo, w.fb_hi, w.fb_lo, w.fw_hi, w.fw_lo}};
  // ---------------------------------------------------------------- inputs, widened
  if (C > 0) {
    if (a.dtype == SA_BF16)
      SA_TIMED("widen_kernel", st, (widen_kernel<<<grid_for(CD), 256, 0, st>>>((const __nv_bfloat16*)a.q, CD, w.qin)));
    else
      SA_TIMED("widen_kernel", st, (widen_kernel<<<grid_for(CD), 256, 0, st>>>((const float*)a.q, CD, w.qin)));
  }
  for (int u = 0; u < B; ++u) {
    const int64_t n = hst.kv_end[u] - hst.kv_begin[u];
    if (n == 0) continue;
    float* dst = w.Xk + (size_t)hst.kpre[u] * D;
    if (a.dtype == SA_BF16)
      SA_TIMED("gather_rows_kernel", st, (gather_rows_kernel<<<grid_for(n * D), 256, 0, st>>>(
                                            (const __nv_bfloat16*)a.kv, hst.kv_begin[u], n, D, dst)));
    else
      SA_TIMED("gather_rows_kernel", st, (gather_rows_kernel<<<grid_for(n * D), 256, 0, st>>>(
                                            (const float*)a.kv, hst.kv_begin[u], n, D, dst)));
  }
  // Xs(0): the gathered key rows; Xs(l + 1): the rows after layer l's history FFN,
  // which are layer l's keys and values and the input of layer l + 1's FFN
  auto Xs = [&](int l) { return w.Xk + (size_t)l * RD; };
  // ---------------------------------------------------------------- forward recompute
  for (int l = 0; l < NL; ++l) {
    const stca_full_layer& L = layers[l];
    const float* qin = w.qin + (size_t)l * CD;
    float* qmid = w.qmid + (size_t)l * CD;
    float* Qh = w.Qh + (size_t)l * CHD;
    float* U = w.U + (size_t)l * CHD2;
    float* Y = w.Y + (size_t)l * CHD2;
    float* O = w.O + (size_t)l * CHD;
    if (has_hist(L)) {
      Ffn f{L.hist_W1, L.hist_W3, L.hist_W2, nullptr, nullptr, nullptr};
      if ((s = ffn_fwd(Xs(l), R, D, f, w.G1, w.G3, w.Uf, Xs(l + 1), cx)) != SA_OK) return s;
    } else if (R > 0) {
      SA_CUDA(cudaMemcpyAsync(Xs(l + 1), Xs(l), sizeof(float) * RD, cudaMemcpyDeviceToDevice, st));
    }
    const float* X = Xs(l + 1);
    const Split Xb{w.Xkb + (size_t)l * RD, w.Xklo + (size_t)l * RD};   // its bf16 split (tensor-core path)
    if (tcp && R > 0)
      SA_TIMED("split_kernel", st, (split_kernel<<<grid_for(RD), 256, 0, st>>>(X, RD, w.Xkb + (size_t)l * RD,
                                                                               w.Xklo + (size_t)l * RD)));
    if (C == 0) continue;
    // Qh[:, h] = q W_Q^h;  U[c*H + h] = Qh[:, h] W_K^h^T / sqrt(d_h)
    Gemm g1 = plain((int)C, dh, D, qin, D, false, L.attn.W_Q, dh, false, Qh, HD, "gemm:stca_bwd_proj");
    g1.batch = H; g1.sB = (int64_t)D * dh; g1.sC = dh;
    if ((s = mm(g1, cx)) != SA_OK) return s;
    Gemm g2 = plain((int)C, D, dh, Qh, HD, false, L.attn.W_K, dh, true, U, (int64_t)H * D, "gemm:stca_bwd_proj");
    g2.batch = H; g2.sA = dh; g2.sB = (int64_t)D * dh; g2.sC = D; g2.alpha = inv_sqrt;
    if ((s = mm(g2, cx)) != SA_OK) return s;
    const Split Ub{w.Ub + (size_t)l * CHD2, w.Ulo + (size_t)l * CHD2};
    if (tcp)
      SA_TIMED("split_kernel", st, (split_kernel<<<grid_for(CHD2), 256, 0, st>>>(U, CHD2, w.Ub + (size_t)l * CHD2,
                                                                                 w.Ulo + (size_t)l * CHD2)));
    // per user: S = U_u X_u^T, P = softmax, Y_u = P X_u
    for (int u = 0; u < B; ++u) {
      const int64_t r0 = hst.cand[u] * H, ru = (hst.cand[u + 1] - hst.cand[u]) * H;
      const int64_t lu = hst.kv_end[u] - hst.kv_begin[u];
      if (ru == 0) continue;
      float* Yu = Y + (size_t)r0 * D;
      if (lu == 0) {
        SA_CUDA(cudaMemsetAsync(Yu, 0, sizeof(float) * ru * D, st));
        continue;
      }
      const float* Xu = X + (size_t)hst.kpre[u] * D;
      const int64_t lp = score_pitch(lu);
      if (tcp) {
        const Split Xbu = Xb.at((int64_t)hst.kpre[u] * D), Ubu = Ub.at(r0 * D), Pb{w.Pb, w.Plo};
        if ((s = tc((int)ru, (int)lu, D, Ubu, D, false, Xbu, D, false, w.S, lp, nullptr, cx)) != SA_OK) return s;
        SA_TIMED("softmax_rows_kernel", st, (softmax_rows_kernel<<<(unsigned)ru, 256, 0, st>>>(w.S, lu, lp, w.Pb,
                                                                                                w.Plo)));
        if ((s = tc((int)ru, D, (int)lu, Pb, lp, false, Xbu, D, true, Yu, D, nullptr, cx)) != SA_OK) return s;
      } else {
        if ((s = mm(plain((int)ru, (int)lu, D, U + (size_t)r0 * D, D, false, Xu, D, true, w.S, lp, "gemm:stca_bwd_attn"), cx)) != SA_OK) return s;
        SA_TIMED("softmax_rows_kernel", st, (softmax_rows_kernel<<<(unsigned)ru, 256, 0, st>>>(w.S, lu, lp, nullptr, nullptr)));
        if ((s = mm(plain((int)ru, D, (int)lu, w.S, lp, false, Xu, D, false, Yu, D, "gemm:stca_bwd_attn"), cx)) != SA_OK) return s;
      }
    }
    // O[:, h] = Y_h W_V^h;  qmid = q + O W_O (or q + O)
    Gemm g3 = plain((int)C, dh, D, Y, (int64_t)H * D, false, L.attn.W_V, dh, false, O, HD, "gemm:stca_bwd_proj");
    g3.batch = H; g3.sA = D; g3.sB = (int64_t)D * dh; g3.sC = dh;
    if ((s = mm(g3, cx)) != SA_OK) return s;
    if (L.attn.W_O) {
      Gemm g4 = plain((int)C, D, HD, O, HD, false, L.attn.W_O, D, false, qmid, D, "gemm:stca_bwd_proj");
      g4.Cin = qin; g4.ldcin = D;
      if ((s = mm(g4, cx)) != SA_OK) return s;
    } else {
      SA_CUDA(cudaMemcpyAsync(qmid, qin, sizeof(float) * CD, cudaMemcpyDeviceToDevice, st));
      SA_TIMED("add_rows_kernel", st, (add_rows_kernel<<<grid_for(CD), 256, 0, st>>>(O, CD, qmid)));
    }
    float* qout = w.qin + (size_t)(l + 1) * CD;
    if (has_query(L)) {
      Ffn f{L.q_W1, L.q_W3, L.q_W2, nullptr, nullptr, nullptr};
      if ((s = ffn_fwd(qmid, C, D, f, w.G1, w.G3, w.Uf, qout, cx)) != SA_OK) return s;
    } else {
      SA_CUDA(cudaMemcpyAsync(qout, qmid, sizeof(float) * CD, cudaMemcpyDeviceToDevice, st));
    }
  }
  // ---------------------------------------------------------------- backward
  if (C > 0) SA_CUDA(cudaMemcpyAsync(w.dq, dout, sizeof(float) * CD, cudaMemcpyDeviceToDevice, st));
  if (R > 0) SA_CUDA(cudaMemsetAsync(w.dX, 0, sizeof(float) * RD, st));
  for (int l = NL - 1; l >= 0; --l) {
    const stca_full_layer& L = layers[l];
    const stca_full_layer_grad& Gd = grads[l];
    const float* qin = w.qin + (size_t)l * CD;
    const float* qmid = w.qmid + (size_t)l * CD;
    const float* Qh = w.Qh + (size_t)l * CHD;
    const float* U = w.U + (size_t)l * CHD2;
    const float* Y = w.Y + (size_t)l * CHD2;
    const float* O = w.O + (size_t)l * CHD;
    const float* X = Xs(l + 1);
    // query FFN: dqmid = dq + FFN_q backward
    if (has_query(L)) {
      Ffn f{L.q_W1, L.q_W3, L.q_W2, Gd.q_dW1, Gd.q_dW3, Gd.q_dW2};
      if ((s = ffn_bwd(qmid, C, D, f, w.dq, w.dqmid, w.G1, w.G3, w.Uf, w.dUf, cx)) != SA_OK) return s;
    } else if (C > 0) {
      SA_CUDA(cudaMemcpyAsync(w.dqmid, w.dq, sizeof(float) * CD, cudaMemcpyDeviceToDevice, st));
    }
    // W_O: dO = dqmid W_O^T, dW_O = O^T dqmid; the residual passes dqmid to q
    if (L.attn.W_O) {
      if ((s = mm(plain((int)C, HD, D, w.dqmid, D, false, L.attn.W_O, D, true, w.dO, HD, "gemm:stca_bwd_proj"), cx)) != SA_OK) return s;
      if (Gd.dW_O) {
        if (C > 0) {
          if ((s = mm(plain(HD, D, (int)C, O, HD, true, w.dqmid, D, false, Gd.dW_O, D, "gemm:stca_bwd_proj"), cx)) != SA_OK) return s;
        } else {
          SA_CUDA(cudaMemsetAsync(Gd.dW_O, 0, sizeof(float) * HD * D, st));
        }
      }
    } else if (C > 0) {
      SA_CUDA(cudaMemcpyAsync(w.dO, w.dqmid, sizeof(float) * CD, cudaMemcpyDeviceToDevice, st));
    }
    // dY_h = dO_h W_V^h^T;  dW_V^h = Y_h^T dO_h
    Gemm gy = plain((int)C, D, dh, w.dO, HD, false, L.attn.W_V, dh, true, w.dY, (int64_t)H * D, "gemm:stca_bwd_proj");
    gy.batch = H; gy.sA = dh; gy.sB = (int64_t)D * dh; gy.sC = D;
    if ((s = mm(gy, cx)) != SA_OK) return s;
    if (tcp && C > 0)
      SA_TIMED("split_kernel", st, (split_kernel<<<grid_for(CHD2), 256, 0, st>>>(w.dY, CHD2, w.dYb, w.dYlo)));
    if (C > 0) {
      Gemm gv = plain(D, dh, (int)C, Y, (int64_t)H * D, true, w.dO, HD, false, Gd.dW_V, dh, "gemm:stca_bwd_proj");
      gv.batch = H; gv.sA = D; gv.sB = dh; gv.sC = (int64_t)D * dh;
      if ((s = mm(gv, cx)) != SA_OK) return s;
    } else {
      SA_CUDA(cudaMemsetAsync(Gd.dW_V, 0, sizeof(float) * H * D * dh, st));
    }
    // attention, per user
    for (int u = 0; u < B; ++u) {
      const int64_t r0 = hst.cand[u] * H, ru = (hst.cand[u + 1] - hst.cand[u]) * H;
      const int64_t lu = hst.kv_end[u] - hst.kv_begin[u];
      if (ru == 0) continue;
      float* dUu = w.dU + (size_t)r0 * D;
      if (lu == 0) {
        SA_CUDA(cudaMemsetAsync(dUu, 0, sizeof(float) * ru * D, st));
        continue;
      }
      const float* Xu = X + (size_t)hst.kpre[u] * D;
      const float* Uu = U + (size_t)r0 * D;
      const float* dYu = w.dY + (size_t)r0 * D;
      float* dXu = w.dX + (size_t)hst.kpre[u] * D;
      const int64_t lp = score_pitch(lu);
      if (tcp) {
        const Split Xbu{w.Xkb + (size_t)l * RD + (size_t)hst.kpre[u] * D,
                        w.Xklo + (size_t)l * RD + (size_t)hst.kpre[u] * D};
        const Split Ubu{w.Ub + (size_t)l * CHD2 + (size_t)r0 * D, w.Ulo + (size_t)l * CHD2 + (size_t)r0 * D};
        const Split dYbu{w.dYb + (size_t)r0 * D, w.dYlo + (size_t)r0 * D};
        const Split Pb{w.Pb, w.Plo}, dSb{w.dSb, w.dSlo};
        if ((s = tc((int)ru, (int)lu, D, Ubu, D, false, Xbu, D, false, w.S, lp, nullptr, cx)) != SA_OK) return s;
        SA_TIMED("softmax_rows_kernel", st, (softmax_rows_kernel<<<(unsigned)ru, 256, 0, st>>>(w.S, lu, lp, w.Pb,
                                                                                                w.Plo)));
        // dP = dY X^T, then dS = P o (dP - <dY, Y>)
        if ((s = tc((int)ru, (int)lu, D, dYbu, D, false, Xbu, D, false, w.dS, lp, nullptr, cx)) != SA_OK) return s;
        SA_TIMED("softmax_bwd_kernel", st, (softmax_bwd_kernel<<<(unsigned)ru, 256, 0, st>>>(
                                               w.S, w.dS, lu, lp, dYu, Y + (size_t)r0 * D, D, w.dSb, w.dSlo)));
        // dU = dS X;  dX += dS^T U + P^T dY  (the transposed score matrices are M-major operands)
        if ((s = tc((int)ru, D, (int)lu, dSb, lp, false, Xbu, D, true, dUu, D, nullptr, cx)) != SA_OK) return s;
        if ((s = tc((int)lu, D, (int)ru, dSb, lp, true, Ubu, D, true, dXu, D, dXu, cx)) != SA_OK) return s;
        if ((s = tc((int)lu, D, (int)ru, Pb, lp, true, dYbu, D, true, dXu, D, dXu, cx)) != SA_OK) return s;
        continue;
      }
      if ((s = mm(plain((int)ru, (int)lu, D, Uu, D, false, Xu, D, true, w.S, lp, "gemm:stca_bwd_attn"), cx)) != SA_OK) return s;
      SA_TIMED("softmax_rows_kernel", st, (softmax_rows_kernel<<<(unsigned)ru, 256, 0, st>>>(w.S, lu, lp, nullptr, nullptr)));
      if ((s = mm(plain((int)ru, (int)lu, D, dYu, D, false, Xu, D, true, w.dS, lp, "gemm:stca_bwd_attn"), cx)) != SA_OK) return s;
      SA_TIMED("softmax_bwd_kernel", st, (softmax_bwd_kernel<<<(unsigned)ru, 256, 0, st>>>(
                                             w.S, w.dS, lu, lp, dYu, Y + (size_t)r0 * D, D, nullptr, nullptr)));
      if ((s = mm(plain((int)ru, D, (int)lu, w.dS, lp, false, Xu, D, false, dUu, D, "gemm:stca_bwd_attn"), cx)) != SA_OK) return s;
      Gemm gk = plain((int)lu, D, (int)ru, w.dS, lp, true, Uu, D, false, dXu, D, "gemm:stca_bwd_attn");
      gk.Cin = dXu; gk.ldcin = D;
      if ((s = mm(gk, cx)) != SA_OK) return s;
      Gemm gvv = plain((int)lu, D, (int)ru, w.S, lp, true, dYu, D, false, dXu, D, "gemm:stca_bwd_attn");
      gvv.Cin = dXu; gvv.ldcin = D;
      if ((s = mm(gvv, cx)) != SA_OK) return s;
    }
    // dQh_h = dU_h W_K^h / sqrt(d_h);  dW_K^h = dU_h^T Qh_h / sqrt(d_h)
    Gemm gq = plain((int)C, dh, D, w.dU, (int64_t)H * D, false, L.attn.W_K, dh, false, w.dQh, HD, "gemm:stca_bwd_proj");
    gq.batch = H; gq.sA = D; gq.sB = (int64_t)D * dh; gq.sC = dh; gq.alpha = inv_sqrt;
    if ((s = mm(gq, cx)) != SA_OK) return s;
    if (C > 0) {
      Gemm gk = plain(D, dh, (int)C, w.dU, (int64_t)H * D, true, Qh, HD, false, Gd.dW_K, dh, "gemm:stca_bwd_proj");
      gk.batch = H; gk.sA = D; gk.sB = dh; gk.sC = (int64_t)D * dh; gk.alpha = inv_sqrt;
      if ((s = mm(gk, cx)) != SA_OK) return s;
      // dW_Q^h = q^T dQh_h
      Gemm gw = plain(D, dh, (int)C, qin, D, true, w.dQh, HD, false, Gd.dW_Q, dh, "gemm:stca_bwd_proj");
      gw.batch = H; gw.sB = dh; gw.sC = (int64_t)D * dh;
      if ((s = mm(gw, cx)) != SA_OK) return s;
      // dq = dqmid + sum_h dQh_h W_Q^h^T
      for (int h = 0; h < H; ++h) {
        Gemm gd = plain((int)C, D, dh, w.dQh + h * dh, HD, false, L.attn.W_Q + (size_t)h * D * dh, dh, true, w.dq, D,
                        "gemm:stca_bwd_proj");
        gd.Cin = h == 0 ? w.dqmid : w.dq; gd.ldcin = D;
        if ((s = mm(gd, cx)) != SA_OK) return s;
      }
    } else {
      SA_CUDA(cudaMemsetAsync(Gd.dW_K, 0, sizeof(float) * H * D * dh, st));
      SA_CUDA(cudaMemsetAsync(Gd.dW_Q, 0, sizeof(float) * H * D * dh, st));
    }
    // history FFN: the gradient reaches the layer's input rows
    if (has_hist(L)) {
      Ffn f{L.hist_W1, L.hist_W3, L.hist_W2, Gd.hist_dW1, Gd.hist_dW3, Gd.hist_dW2};
      if ((s = ffn_bwd(Xs(l), R, D, f, w.dX, w.dX, w.G1, w.G3, w.Uf, w.dUf, cx)) != SA_OK) return s;
    }
  }
  // ---------------------------------------------------------------- outputs
  if (dq_out && C > 0) SA_CUDA(cudaMemcpyAsync(dq_out, w.dq, sizeof(float) * CD, cudaMemcpyDeviceToDevice, st));
  if (dkv) {
    if (a.kv_rows > 0) SA_CUDA(cudaMemsetAsync(dkv, 0, sizeof(float) * a.kv_rows * D, st));
    for (int u = 0; u < B; ++u) {
      const int64_t n = (hst.kv_end[u] - hst.kv_begin[u]) * D;
      if (n == 0) continue;
      SA_TIMED("add_rows_kernel", st, (add_rows_kernel<<<grid_for(n), 256, 0, st>>>(
                                         w.dX + (size_t)hst.kpre[u] * D, n, dkv + (size_t)hst.kv_begin[u] * D)));
    }
  }
  return SA_OK;
}

}  // namespace sa
