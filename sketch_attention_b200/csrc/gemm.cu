// Tiled SIMT fp32 GEMM: 64 x 64 output tile per CTA, 16-deep k slices staged
// through shared memory, 4 x 4 outputs per thread.  Arbitrary sizes, strides,
// transposes and batch; used only for the small projection GEMMs.
#include <algorithm>

#include "gemm.cuh"

namespace sa {

namespace {
constexpr int TM = 64, TN = 64, TK = 16;

__global__ void __launch_bounds__(256) gemm_kernel(Gemm g) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int b = blockIdx.z / g.split_k, sk = blockIdx.z % g.split_k;
  const int kper = ((g.K + g.split_k - 1) / g.split_k + TK - 1) / TK * TK;
  const int kbeg = sk * kper, kend = min(g.K, kbeg + kper);
  const float* A = g.A + (int64_t)b * g.sA;
  const float* Bm = g.B + (int64_t)b * g.sB;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = kbeg; k0 < kend; k0 += TK) {
    // 64 x 16 of A and 16 x 64 of B, 4 elements of each per thread.
    for (int e = threadIdx.x; e < TM * TK; e += 256) {
      int mm, kk;
      if (g.transA) { mm = e % TM; kk = e / TM; } else { kk = e % TK; mm = e / TK; }
      int m = m0 + mm, k = k0 + kk;
      float v = 0.f;
      if (m < g.M && k < kend) v = g.transA ? A[(int64_t)k * g.lda + m] : A[(int64_t)m * g.lda + k];
      As[kk][mm] = v;
    }
    for (int e = threadIdx.x; e < TN * TK; e += 256) {
      int nn, kk;
      if (g.transB) { kk = e % TK; nn = e / TK; } else { nn = e % TN; kk = e / TN; }
      int n = n0 + nn, k = k0 + kk;
      float v = 0.f;
      if (n < g.N && k < kend) v = g.transB ? Bm[(int64_t)n * g.ldb + k] : Bm[(int64_t)k * g.ldb + n];
      Bs[kk][nn] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bb[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }
  if (g.split_k > 1) {
    float* part = g.split_ws + (int64_t)blockIdx.z * g.M * g.N;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = m0 + ty + 16 * i;
      if (m >= g.M) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + tx + 16 * j;
        if (n < g.N) part[(int64_t)m * g.N + n] = acc[i][j];
      }
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int m = m0 + ty + 16 * i;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int n = n0 + tx + 16 * j;
      if (n >= g.N) continue;
      float v = g.alpha * acc[i][j];
      if (g.bias) v += g.bias[n];
      if (g.Cin) v += g.Cin[(int64_t)b * g.sCin + (int64_t)m * g.ldcin + n];
      if (g.C) g.C[(int64_t)b * g.sC + (int64_t)m * g.ldc + n] = v;
      if (g.C16) g.C16[(int64_t)b * g.sC16 + (int64_t)m * g.ldc16 + n] = __float2bfloat16_rn(v);
    }
  }
}
// Adds the split_k partial slices of each output in order, then the epilogue.
__global__ void gemm_split_reduce_kernel(Gemm g) {
  const int64_t mn = (int64_t)g.M * g.N;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < mn * g.batch;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int b = (int)(e / mn);
    const int64_t r = e % mn;
    const int m = (int)(r / g.N), n = (int)(r % g.N);
    float v = 0.f;
    for (int s = 0; s < g.split_k; ++s) v += g.split_ws[((int64_t)b * g.split_k + s) * mn + r];
    v *= g.alpha;
    if (g.bias) v += g.bias[n];
    if (g.Cin) v += g.Cin[(int64_t)b * g.sCin + (int64_t)m * g.ldcin + n];
    if (g.C) g.C[(int64_t)b * g.sC + (int64_t)m * g.ldc + n] = v;
    if (g.C16) g.C16[(int64_t)b * g.sC16 + (int64_t)m * g.ldc16 + n] = __float2bfloat16_rn(v);
  }
}
}  // namespace

int gemm_split_for(int M, int N, int K, int max_split) {
  const int tiles = ((M + TM - 1) / TM) * ((N + TN - 1) / TN);
  int s = std::min((K + 511) / 512, std::max(1, 296 / std::max(tiles, 1)));
  return std::max(1, std::min(s, max_split));
}

sa_status gemm(const Gemm& g0, cudaStream_t stream) {
  if (g0.M <= 0 || g0.N <= 0 || g0.batch <= 0) return SA_OK;
  Gemm g = g0;
  if (g.split_k < 1 || !g.split_ws) g.split_k = 1;
  dim3 grid((g.N + TN - 1) / TN, (g.M + TM - 1) / TM, g.batch * g.split_k);
  SA_TIMED(g.tag ? g.tag : "gemm_kernel", stream, (gemm_kernel<<<grid, 256, 0, stream>>>(g)));
  if (g.split_k > 1) {
    const int64_t n = (int64_t)g.M * g.N * g.batch;
    SA_TIMED("gemm_split_reduce_kernel", stream,
             (gemm_split_reduce_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, 4096), 256, 0,
                                         stream>>>(g)));
  }
  return SA_OK;
}

}  // namespace sa
