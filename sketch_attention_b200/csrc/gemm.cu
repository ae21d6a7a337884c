// Tiled SIMT fp32 GEMM: a BM x BN output tile per CTA (BN = 32 when N <= 32,
// else 64; BM = 64 when 128-row tiles would leave the SMs short of CTAs, else
// 128), 8 x 4 outputs per thread read from shared memory as float4.  The
// 16-deep k slices stream through NS shared-memory stages with asynchronous
// element copies (zero-filled past the edges), NS - 1 slices ahead of the
// multiply, so global latency is paid about once per CTA rather than once per
// slice.  Arbitrary sizes, strides, transposes and batch; used only for the
// small projection GEMMs.
#include <algorithm>

#include "gemm.cuh"

namespace sa {

namespace {
constexpr int BK = 16, RM = 8, RN = 4, NS = 3;

__device__ __forceinline__ void cp_async4(float* dst, const float* src, bool pred) {
  // 4-byte asynchronous copy; with pred false nothing is read and zero is written
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(pred ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// the 16-bit copy of an output: bf16, or fp16 with |v| > 65504 flagged on the device
__device__ __forceinline__ void store16(const Gemm& g, int64_t i, float v) {
  if (g.c16_half) {
    if (!(fabsf(v) <= 65504.f) && g.err) atomicOr(g.err, DEV_ERR_RANGE);
    reinterpret_cast<__half*>(g.C16)[i] = __float2half_rn(v);
  } else {
    g.C16[i] = __float2bfloat16_rn(v);
  }
}

template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// TA / TB: A stored [K, M] / B stored [N, K] (compile-time, so each variant's
// unrolled copy loops stay small in the instruction cache)
template <int BM, int BN, bool TA, bool TB>
__global__ void __launch_bounds__((BM / RM) * (BN / RN), 2) gemm_kernel(Gemm g) {
  constexpr int NT = (BM / RM) * (BN / RN);
  constexpr int LA = BM * BK / NT, LB = BK * BN / NT;     // elements copied per thread per slice
  __shared__ __align__(16) float As[NS][BK][BM + 4];
  __shared__ __align__(16) float Bs[NS][BK][BN + 4];
  const int b = blockIdx.z / g.split_k, sk = blockIdx.z % g.split_k;
  const int kper = ((g.K + g.split_k - 1) / g.split_k + BK - 1) / BK * BK;
  const int kbeg = sk * kper, kend = min(g.K, kbeg + kper);
  const int nsl = kend > kbeg ? (kend - kbeg + BK - 1) / BK : 0;
  const float* A = g.A + (int64_t)b * g.sA;
  const float* Bm = g.B + (int64_t)b * g.sB;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int tx = threadIdx.x % (BN / RN), ty = threadIdx.x / (BN / RN);
  float acc[RM][RN] = {};
  // element e = threadIdx.x + NT * l of a slice; the operand's contiguous index
  // runs fastest across threads (coalesced global reads)
  auto issue = [&](int sl) {
    if (sl < nsl) {
      const int k0 = kbeg + sl * BK, st = sl % NS;
#pragma unroll
      for (int l = 0; l < LA; ++l) {
        const int e = threadIdx.x + NT * l;
        int mm, kk;
        if (TA) { mm = e % BM; kk = e / BM; } else { kk = e % BK; mm = e / BK; }
        const int m = m0 + mm, k = k0 + kk;
        const bool ok = m < g.M && k < kend;
        cp_async4(&As[st][kk][mm], ok ? (TA ? A + (int64_t)k * g.lda + m : A + (int64_t)m * g.lda + k) : A, ok);
      }
#pragma unroll
      for (int l = 0; l < LB; ++l) {
        const int e = threadIdx.x + NT * l;
        int nn, kk;
        if (TB) { kk = e % BK; nn = e / BK; } else { nn = e % BN; kk = e / BN; }
        const int n = n0 + nn, k = k0 + kk;
        const bool ok = n < g.N && k < kend;
        cp_async4(&Bs[st][kk][nn], ok ? (TB ? Bm + (int64_t)n * g.ldb + k : Bm + (int64_t)k * g.ldb + n) : Bm, ok);
      }
    }
    cp_async_commit();   // one group per slice index, empty past the end
  };
#pragma unroll
  for (int sl = 0; sl < NS - 1; ++sl) issue(sl);
  for (int sl = 0; sl < nsl; ++sl) {
    cp_async_wait<NS - 2>();   // slice sl has landed (this thread's copies)
    __syncthreads();           // ... everyone's; and stage (sl - 1) % NS is no longer read
    issue(sl + NS - 1);
    const int st = sl % NS;
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      const float4 a0 = *(const float4*)&As[st][kk][ty * RM];
      const float4 a1 = *(const float4*)&As[st][kk][ty * RM + 4];
      const float4 b0 = *(const float4*)&Bs[st][kk][tx * RN];
      const float av[RM] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[RN] = {b0.x, b0.y, b0.z, b0.w};
#pragma unroll
      for (int i = 0; i < RM; ++i)
#pragma unroll
        for (int j = 0; j < RN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
  }
  cp_async_wait<0>();
  if (g.split_k > 1) {
    float* part = g.split_ws + (int64_t)blockIdx.z * g.M * g.N;
#pragma unroll
    for (int i = 0; i < RM; ++i) {
      const int m = m0 + ty * RM + i;
      if (m >= g.M) continue;
#pragma unroll
      for (int j = 0; j < RN; ++j) {
        const int n = n0 + tx * RN + j;
        if (n < g.N) part[(int64_t)m * g.N + n] = acc[i][j];
      }
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < RM; ++i) {
    const int m = m0 + ty * RM + i;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < RN; ++j) {
      const int n = n0 + tx * RN + j;
      if (n >= g.N) continue;
      float v = g.alpha * acc[i][j];
      if (g.bias) v += g.bias[n];
      if (g.Cin) v += g.Cin[(int64_t)b * g.sCin + (int64_t)m * g.ldcin + n];
      if (g.C) g.C[(int64_t)b * g.sC + (int64_t)m * g.ldc + n] = v;
      if (g.C16) store16(g, (int64_t)b * g.sC16 + (int64_t)m * g.ldc16 + n, v);
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
    if (g.C16) store16(g, (int64_t)b * g.sC16 + (int64_t)m * g.ldc16 + n, v);
  }
}
}  // namespace

int gemm_split_for(int M, int N, int K, int max_split) {
  // enough CTAs for about three per SM, and at least four 16-deep k slices per CTA
  const int bn = N <= 32 ? 32 : 64;
  const int tiles = std::max(1, ((M + 127) / 128) * ((N + bn - 1) / bn));
  const int target = 3 * device_info().sm_count;
  int s = std::min((K + 63) / 64, (target + tiles - 1) / tiles);
  return std::max(1, std::min(s, max_split));
}

sa_status gemm(const Gemm& g0, cudaStream_t stream) {
  if (g0.M <= 0 || g0.N <= 0 || g0.batch <= 0) return SA_OK;
  Gemm g = g0;
  if (g.split_k < 1 || !g.split_ws) g.split_k = 1;
  const char* tag = g.tag ? g.tag : "gemm_kernel";
  const int bn = g.N <= 32 ? 32 : 64;
  const int64_t ctas128 = (int64_t)((g.N + bn - 1) / bn) * ((g.M + 127) / 128) * g.batch * g.split_k;
  const bool small = ctas128 < 2 * device_info().sm_count;
  const int bm = small ? 64 : 128;
  if ((g.M + bm - 1) / bm > 65535 || (int64_t)g.batch * g.split_k > 65535)
    return fail(SA_ERR_UNSUPPORTED, std::string(tag) + ": more than 65535 row tiles or batches");
  dim3 grid((g.N + bn - 1) / bn, (g.M + bm - 1) / bm, g.batch * g.split_k);
  const int nt = (bm / RM) * (bn / RN);
  const int variant = (bm == 64 ? 0 : 4) + (bn == 32 ? 0 : 2) + 0;   // tile shape
  switch (variant + (g.transA ? 8 : 0) + (g.transB ? 1 : 0)) {
#define SA_GEMM_CASE(V, BM_, BN_, TA_, TB_)                                               \
  case V:                                                                                  \
    SA_TIMED(tag, stream, (gemm_kernel<BM_, BN_, TA_, TB_><<<grid, nt, 0, stream>>>(g))); \
    break;
    SA_GEMM_CASE(0, 64, 32, false, false)
    SA_GEMM_CASE(1, 64, 32, false, true)
    SA_GEMM_CASE(2, 64, 64, false, false)
    SA_GEMM_CASE(3, 64, 64, false, true)
    SA_GEMM_CASE(4, 128, 32, false, false)
    SA_GEMM_CASE(5, 128, 32, false, true)
    SA_GEMM_CASE(6, 128, 64, false, false)
    SA_GEMM_CASE(7, 128, 64, false, true)
    SA_GEMM_CASE(8, 64, 32, true, false)
    SA_GEMM_CASE(9, 64, 32, true, true)
    SA_GEMM_CASE(10, 64, 64, true, false)
    SA_GEMM_CASE(11, 64, 64, true, true)
    SA_GEMM_CASE(12, 128, 32, true, false)
    SA_GEMM_CASE(13, 128, 32, true, true)
    SA_GEMM_CASE(14, 128, 64, true, false)
    SA_GEMM_CASE(15, 128, 64, true, true)
#undef SA_GEMM_CASE
    default: break;
  }
  if (g.split_k > 1) {
    const int64_t n = (int64_t)g.M * g.N * g.batch;
    SA_TIMED("gemm_split_reduce_kernel", stream,
             (gemm_split_reduce_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, 4096), 256, 0,
                                         stream>>>(g)));
  }
  return SA_OK;
}

}  // namespace sa
