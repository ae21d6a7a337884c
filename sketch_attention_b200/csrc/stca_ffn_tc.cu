// History-side SwiGLU FFN of the full STCA layer on the sm_100a tensor cores
// (SequenceO1 Sec. 5.1, eq. (27)): for every bf16 key row x (D = 128)
//   x <- x + (SiLU(x W1) * (x W3)) W2,   W1, W3 [128, 256], W2 [256, 128]
// in place, with the 256-wide inner activations never leaving the SM.
//
// Persistent: one CTA per SM keeps both weight layers resident in shared
// memory (bf16, 192 KB) and walks 128-row tiles.  A tile's inner width is
// done in four quarters of 64:
//   G_q  = X [W1_q | W3_q]     M=128 rows, N=128, K=128   (SS, fp32 in TMEM)
//   U_q  = SiLU(G1_q) * G3_q   registers -> bf16 pairs in TMEM
//   F   += U_q W2_q            M=128, N=128, K=64          (A from TMEM)
// and x + F goes back to the row as bf16.  G and U are double-buffered, so
// the tensor pipe computes G_{q+1} while the epilogue warps turn G_q into U_q.
// SiLU(g) g3 = (g/2) g3 (1 + tanh(g/2)): one MUFU operation per element.
//
// Warp roles (10 warps): 0 TMA, 1 MMA issue + TMEM owner, 2-9 two warpgroups
// of epilogue (warpgroup h takes inner columns 32h..32h+31 of each quarter
// and output columns 64h..64h+63).
#include <algorithm>
#include <cstring>
#include <mutex>

#include "stca_internal.cuh"
#include "tc_ptx.cuh"

namespace sa {

namespace {
using namespace tc;

constexpr int DD = 128, TM = 128, THREADS = 320;
constexpr uint32_t W13_BYTES = 4 * 128 * DD * 2;   // [512 rows][128] bf16, two 64-column atoms
constexpr uint32_t W2_BYTES = DD * 2 * DD * 2;     // [128 rows][256] bf16, four 64-column atoms
constexpr uint32_t X_BYTES = TM * DD * 2;          // one row tile, two atoms
constexpr uint32_t OFF_W13 = 0, OFF_W2 = OFF_W13 + W13_BYTES, OFF_X = OFF_W2 + W2_BYTES;
constexpr uint32_t OFF_BAR = OFF_X + X_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
// TMEM columns: G double buffer, U double buffer (bf16 pairs), F accumulator
constexpr uint32_t TM_G = 0, TM_U = 256, TM_F = 384, TM_COLS = 512;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

struct Bars {
  uint64_t w_full, x_full, x_empty, g_full[2], g_empty[2], u_full[2], u_empty[2], f_full, f_empty,
      mma_done;
  uint32_t tmem_base;
  int abort;
};

struct Params {
  __nv_bfloat16* X;
  int64_t rows;
  int ntiles;
  int* err;
};

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(THREADS, 1)
    stca_hist_ffn_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                            const __grid_constant__ CUtensorMap tmW13,
                            const __grid_constant__ CUtensorMap tmW2, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Bars* bars = (Bars*)(smem + OFF_BAR);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(&bars->w_full, 1);
    mbar_init(&bars->x_full, 1);
    mbar_init(&bars->x_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->g_full[b], 1);
      mbar_init(&bars->g_empty[b], 256);
      mbar_init(&bars->u_full[b], 256);
      mbar_init(&bars->u_empty[b], 1);
    }
    mbar_init(&bars->f_full, 1);
    mbar_init(&bars->f_empty, 256);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmW13);
    prefetch_tensormap(&tmW2);
    mbar_arrive_expect_tx(&bars->w_full, W13_BYTES + W2_BYTES);
    for (int a = 0; a < 2; ++a)
      for (int r = 0; r < 2; ++r)
        tma_load_2d(smem + OFF_W13 + a * (W13_BYTES / 2) + r * (W13_BYTES / 4), &tmW13, &bars->w_full,
                    64 * a, 256 * r);
    for (int a = 0; a < 4; ++a)
      tma_load_2d(smem + OFF_W2 + a * (W2_BYTES / 4), &tmW2, &bars->w_full, 64 * a, 0);
    int i = 0, issued = 0;
    for (int t = blockIdx.x; t < p.ntiles; t += gridDim.x, ++i) {
      if (i > 0 && !mbar_wait(&bars->x_empty, (i - 1) & 1, abort, p.err)) break;
      mbar_arrive_expect_tx(&bars->x_full, X_BYTES);
      tma_load_2d(smem + OFF_X, &tmX, &bars->x_full, 0, t * TM);
      tma_load_2d(smem + OFF_X + X_BYTES / 2, &tmX, &bars->x_full, 64, t * TM);
      issued = i + 1;
      // the next tile waits for this one's logits; start its trip to L2 now
      const int tn = t + (int)gridDim.x;
      if (tn < p.ntiles) {
        tma_prefetch_l2_2d(&tmX, 0, tn * TM);
        tma_prefetch_l2_2d(&tmX, 64, tn * TM);
      }
    }
    if (*abort) {
      mbar_wait_bounded(&bars->w_full, 0);
      if (issued > 0) mbar_wait_bounded(&bars->x_full, (issued - 1) & 1);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    const uint32_t id = idesc_bf16(128, 128, false, false);
    const uint32_t xa = smem_u32(smem + OFF_X), w13 = smem_u32(smem + OFF_W13),
                   w2 = smem_u32(smem + OFF_W2);
    bool ok = mbar_wait(&bars->w_full, 0, abort, p.err);
    int i = 0;
    // G_q = X [W1_q | W3_q]; the quarter's rows of W13t start at 128 q
    auto gemm1 = [&](int q) -> bool {
      const int b = q & 1, n = 2 * i + (q >> 1);
      if (n >= 1 && !mbar_wait(&bars->g_empty[b], (n - 1) & 1, abort, p.err)) return false;
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_ss(tmem + TM_G + 128 * b,
               smem_desc(xa + (ks >> 2) * (X_BYTES / 2) + (ks & 3) * 32, 16, 1024, SWZ_128B),
               smem_desc(w13 + (ks >> 2) * (W13_BYTES / 2) + q * 16384 + (ks & 3) * 32, 16, 1024, SWZ_128B),
               id, ks > 0 ? 1u : 0u);
      mma_commit(&bars->g_full[b]);
      return true;
    };
    // F += U_q W2_q; atom q of W2t holds inner columns 64q..64q+63
    auto gemm2 = [&](int q) -> bool {
      const int b = q & 1, n = 2 * i + (q >> 1);
      if (!mbar_wait(&bars->u_full[b], n & 1, abort, p.err)) return false;
      if (q == 0 && i >= 1 && !mbar_wait(&bars->f_empty, (i - 1) & 1, abort, p.err)) return false;
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_ts(tmem + TM_F, tmem + TM_U + 32 * b + 8 * ks,
               smem_desc(w2 + q * (W2_BYTES / 4) + ks * 32, 16, 1024, SWZ_128B), id,
               (q > 0 || ks > 0) ? 1u : 0u);
      mma_commit(&bars->u_empty[b]);
      if (q == 3) mma_commit(&bars->f_full);
      return true;
    };
    for (int t = blockIdx.x; ok && t < p.ntiles; t += gridDim.x, ++i) {
      if (!mbar_wait(&bars->x_full, i & 1, abort, p.err)) break;
      tc_fence_after();
      ok = gemm1(0) && gemm1(1) && gemm2(0) && gemm1(2) && gemm2(1) && gemm1(3);
      if (!ok) break;
      mma_commit(&bars->x_empty);      // X is read by the first-layer MMAs only
      ok = gemm2(2) && gemm2(3);
    }
    mma_commit(&bars->mma_done);
    mbar_wait_bounded(&bars->mma_done, 0);
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue
    const int q4 = warp % 4, h = (warp - 2) / 4;
    const int row = q4 * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    const float2 half2 = make_float2(0.5f, 0.5f);
    int i = 0;
    for (int t = blockIdx.x; t < p.ntiles; t += gridDim.x, ++i) {
      bool ok = true;
      for (int q = 0; q < 4; ++q) {
        const int b = q & 1, n = 2 * i + (q >> 1);
        if (!mbar_wait(&bars->g_full[b], n & 1, abort, p.err)) { ok = false; break; }
        tc_fence_after();
        float g1[32], g3[32];
        tmem_ld32(tmem + lane_addr + TM_G + 128 * b + 32 * h, g1);
        tmem_ld32(tmem + lane_addr + TM_G + 128 * b + 64 + 32 * h, g3);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->g_empty[b]);
        uint32_t u[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float2 hx = __fmul2_rn(make_float2(g1[2 * j], g1[2 * j + 1]), half2);
          const float2 th = make_float2(tanh_approx(hx.x), tanh_approx(hx.y));
          const float2 hg = __fmul2_rn(hx, make_float2(g3[2 * j], g3[2 * j + 1]));
          const float2 uu = __ffma2_rn(hg, th, hg);
          u[j] = pack_bf16x2(uu.x, uu.y);
        }
        // U buffer b was last read by the second-layer MMAs of use n-1
        if (n >= 1 && !mbar_wait(&bars->u_empty[b], (n - 1) & 1, abort, p.err)) { ok = false; break; }
        tc_fence_after();
        tmem_st16(tmem + lane_addr + TM_U + 32 * b + 16 * h, u);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->u_full[b]);
      }
      if (!ok || !mbar_wait(&bars->f_full, i & 1, abort, p.err)) break;
      tc_fence_after();
      float f[64];
      tmem_ld32(tmem + lane_addr + TM_F + 64 * h, f);
      tmem_ld32(tmem + lane_addr + TM_F + 64 * h + 32, f + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars->f_empty);
      const int64_t grow = (int64_t)t * TM + row;
      if (grow < p.rows) {
        uint4* px = (uint4*)(p.X + grow * DD + 64 * h);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint4 x = px[v];
          uint32_t* xw = (uint32_t*)&x;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 xb = *(__nv_bfloat162*)&xw[e];
            const float2 xf = __bfloat1622float2(xb);
            xw[e] = pack_bf16x2(xf.x + f[8 * v + 2 * e], xf.y + f[8 * v + 2 * e + 1]);
          }
          px[v] = x;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

// W13t[128 q + r][k] = W1[k][64 q + r] (r < 64), W3[k][64 q + r - 64] (r >= 64);
// W2t[n][j] = W2[j][n]
__global__ void ffn_weights_bf16_kernel(const float* __restrict__ W1, const float* __restrict__ W3,
                                        const float* __restrict__ W2, __nv_bfloat16* __restrict__ W13t,
                                        __nv_bfloat16* __restrict__ W2t) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < 4 * 128 * DD) {
    const int r = e / DD, k = e % DD;
    const int q = r / 128, rr = r % 128;
    const float* src = rr < 64 ? W1 : W3;
    W13t[e] = __float2bfloat16_rn(src[k * 2 * DD + 64 * q + (rr & 63)]);
  } else if (e < 4 * 128 * DD + DD * 2 * DD) {
    const int f = e - 4 * 128 * DD;
    const int n = f / (2 * DD), j = f % (2 * DD);
    W2t[f] = __float2bfloat16_rn(W2[j * DD + n]);
  }
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* q = nullptr;
    cudaDriverEntryPointQueryResult r;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      fn = (EncodeFn)q;
  });
  return fn;
}

// bf16 matrix [outer][inner], boxes of 64 x box_outer, 128-byte swizzle
sa_status make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  EncodeFn enc = encode_fn();
  if (!enc) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return SA_OK;
}
}  // namespace

sa_status stca_ffn_weights_bf16(const float* W1, const float* W3, const float* W2, __nv_bfloat16* W13t,
                                __nv_bfloat16* W2t, cudaStream_t st) {
  constexpr int n = 4 * 128 * DD + DD * 2 * DD;
  SA_TIMED("ffn_weights_bf16_kernel", st,
           (ffn_weights_bf16_kernel<<<(n + 255) / 256, 256, 0, st>>>(W1, W3, W2, W13t, W2t)));
  return SA_OK;
}

sa_status stca_hist_ffn_tc(__nv_bfloat16* X, int64_t rows, const __nv_bfloat16* W13t,
                           const __nv_bfloat16* W2t, cudaStream_t st) {
  if (rows <= 0) return SA_OK;
  if (rows >= (1LL << 31) - TM) return fail(SA_ERR_UNSUPPORTED, "history rows must be < 2^31 - 128");
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(stca_hist_ffn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  });
  CUtensorMap tmX, tmW13, tmW2;
  sa_status s;
  if ((s = make_map(&tmX, X, DD, (uint64_t)rows, TM)) != SA_OK) return s;
  if ((s = make_map(&tmW13, W13t, DD, 4 * 128, 256)) != SA_OK) return s;
  if ((s = make_map(&tmW2, W2t, 2 * DD, DD, 128)) != SA_OK) return s;
  const int ntiles = (int)((rows + TM - 1) / TM);
  const int grid = std::min(ntiles, device_info().sm_count);
  Params p{X, rows, ntiles, device_status_word()};
  SA_TIMED("stca_hist_ffn_tc_kernel", st,
           (stca_hist_ffn_tc_kernel<<<grid, THREADS, SMEM_BYTES, st>>>(tmX, tmW13, tmW2, p)));
  return SA_OK;
}

}  // namespace sa
