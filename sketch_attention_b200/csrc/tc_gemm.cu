// bf16 GEMM on the sm_100a tensor cores for the STCA projections and the STCA
// backward's attention and SwiGLU FFN products: C[M, N] = alpha A B (+ Cin), fp32
// accumulation, fp32 and/or 16-bit output.
// An operand may come as a split pair x = hi + lo (both bf16, lo the rounding of
// x - hi): the K loop then runs again over hi x lo and lo x hi into the same
// accumulator (lo x lo, below 2^-16 of the product, is dropped), which carries
// fp32 operands to about 16 significant bits on the bf16 tensor cores.
//
// A is [M, K], stored K-major (A[m lda + k]) or M-major (A[k lda + m]); B is
// [K, N], stored K-major (B[n ldb + k]) or N-major (B[k ldb + n]).  One CTA per
// 128 x 128 output tile: TMA brings 64-deep K slices of both operands into a
// three-stage ring (128-byte swizzle; a K-major operand is one 64 x 128 box, an
// MN-major one two 64 x 64 boxes), one thread issues the MMAs (M = 128,
// N = 128, K = 16) into a TMEM accumulator, and four warps write the tile through
// shared memory (row-contiguous stores).  Two CTAs share an SM, so one CTA's
// epilogue overlaps the other's loads and MMAs.
// Edges are zero-filled by the TMA and masked in the epilogue.  A deep K over few
// output tiles is split across CTAs (grid z): each writes its raw partial tile to a
// workspace slice and a second kernel adds the slices in order (deterministic).
#include <algorithm>
#include <mutex>

#include "stca_internal.cuh"
#include "tc_ptx.cuh"
#include "tma_map.cuh"

namespace sa {

namespace {
using namespace tc;

constexpr int TM = 128, TN = 128, TK = 64, NST = 3, THREADS = 192;
constexpr uint32_t OP_BYTES = TM * TK * 2;                 // 16 KB per operand per stage
constexpr uint32_t STAGE = 2 * OP_BYTES;
constexpr uint32_t OFF_BAR = NST * STAGE;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 128 + 1024;
constexpr uint32_t TM_COLS = 128;
// two CTAs per SM (2 x ~99.5 KB of shared memory, 2 x 128 TMEM columns): one CTA's
// epilogue overlaps the other's loads and MMAs, which matters for the short-K products
static_assert(2 * (SMEM_BYTES + 1024) <= 228 * 1024, "two CTAs per SM");

struct Bars {
  uint64_t full[NST], empty[NST], done;
  uint32_t tmem_base;
  int abort;
};

struct Params {
  int M, N, K;
  int ph_alo, ph_blo;     // the K-loop pass that reads A's (B's) lo part; -1: none
  float* C;
  int64_t ldc;
  const float* Cin;
  int64_t ldcin;
  float alpha;
  int kt_per;             // K slices (of TK) per split; the split index is blockIdx.z
  float* part;            // split > 1: raw partial tiles, [split][M][N]
  int* err;
  __nv_bfloat16* C16;     // optional 16-bit output (bf16, or fp16 when c16_half)
  int64_t ldc16;
  int c16_half;
  __nv_bfloat16* Chi;     // optional hi + lo bf16 split of the output: hi = bf16(c), lo = bf16(c - hi)
  __nv_bfloat16* Clo;
  int64_t ldcs;
};

// the 16-bit copy of an output element; an fp16 value beyond its range is flagged
__device__ __forceinline__ void store_split(const Params& p, int64_t m, int n, float v) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(v);
  p.Chi[m * p.ldcs + n] = hi;
  p.Clo[m * p.ldcs + n] = __float2bfloat16_rn(v - __bfloat162float(hi));
}
__device__ __forceinline__ void store_c16(const Params& p, int64_t m, int n, float v) {
  if (p.c16_half) {
    if (!(fabsf(v) <= 65504.f)) atomicOr(p.err, DEV_ERR_RANGE);
    reinterpret_cast<__half*>(p.C16)[m * p.ldc16 + n] = __float2half_rn(v);
  } else {
    p.C16[m * p.ldc16 + n] = __float2bfloat16_rn(v);
  }
}

// the smem descriptor of K-step ks (16 deep) of a 64-deep operand slice
__device__ __forceinline__ uint64_t op_desc(uint32_t base, int ks, bool mn) {
  return mn ? smem_desc(base + ks * 2048, OP_BYTES / 2, 1024, SWZ_128B)   // two 64-wide MN atoms
            : smem_desc(base + ks * 32, 16, 1024, SWZ_128B);              // 128 rows, K along the row
}

// CIN: the launch adds Cin in its epilogue (no split K)
template <bool AMN, bool BMN, bool CIN>
__global__ void __launch_bounds__(THREADS, 2)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAl,
                   const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmBl, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Bars* bars = (Bars*)(smem + OFF_BAR);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  const int kt0 = blockIdx.z * p.kt_per;
  const int nk = min(p.kt_per, (p.K + TK - 1) / TK - kt0);        // >= 1 (the host sizes the split)
  const int nit = nk * (1 + (p.ph_alo >= 0) + (p.ph_blo >= 0));   // K slices over all passes

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) { mbar_init(&bars->full[s], 1); mbar_init(&bars->empty[s], 1); }
    mbar_init(&bars->done, 1);
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
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (p.ph_alo >= 0) prefetch_tensormap(&tmAl);
    if (p.ph_blo >= 0) prefetch_tensormap(&tmBl);
    int issued = 0;
    for (int it = 0; it < nit; ++it) {
      const int s = it % NST, ph = it / nk, k0 = (kt0 + it % nk) * TK;
      const CUtensorMap* ma = ph == p.ph_alo ? &tmAl : &tmA;
      const CUtensorMap* mb = ph == p.ph_blo ? &tmBl : &tmB;
      if (it >= NST && !mbar_wait(&bars->empty[s], ((it / NST) - 1) & 1, abort, p.err)) break;
      mbar_arrive_expect_tx(&bars->full[s], STAGE);
      uint8_t* a = smem + s * STAGE;
      uint8_t* b = a + OP_BYTES;
      if (AMN) {
        tma_load_2d(a, ma, &bars->full[s], m0, k0);
        tma_load_2d(a + OP_BYTES / 2, ma, &bars->full[s], m0 + 64, k0);
      } else {
        tma_load_2d(a, ma, &bars->full[s], k0, m0);
      }
      if (BMN) {
        tma_load_2d(b, mb, &bars->full[s], n0, k0);
        tma_load_2d(b + OP_BYTES / 2, mb, &bars->full[s], n0 + 64, k0);
      } else {
        tma_load_2d(b, mb, &bars->full[s], k0, n0);
      }
      issued = it + 1;
    }
    if (*abort)
      for (int it = std::max(0, issued - NST); it < issued; ++it)
        mbar_wait_bounded(&bars->full[it % NST], (it / NST) & 1);
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    const uint32_t id = idesc_bf16(128, 128, AMN, BMN);
    for (int it = 0; it < nit; ++it) {
      const int s = it % NST;
      if (!mbar_wait(&bars->full[s], (it / NST) & 1, abort, p.err)) break;
      tc_fence_after();
      const uint32_t a = smem_u32(smem + s * STAGE), b = a + OP_BYTES;
#pragma unroll
      for (int ks = 0; ks < TK / 16; ++ks)
        mma_ss(tmem, op_desc(a, ks, AMN), op_desc(b, ks, BMN), id, (it > 0 || ks > 0) ? 1u : 0u);
      mma_commit(&bars->empty[s]);
    }
    mma_commit(&bars->done);
    mbar_wait_bounded(&bars->done, 0);
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue
    // warp q owns TMEM lanes (tile rows) 32q..32q+31; each 32 x 32 block goes from
    // TMEM (a row per thread) through a padded shared-memory block (the operand ring is
    // idle once every MMA has completed) so that each store writes 128 contiguous bytes
    // of one row
    // The added input Cin of a block is loaded as 32 independent row loads before the
    // block's stores (the first block's while the MMAs still run), so its latency is paid
    // once per block rather than once per row.  Cin may alias C: each element is read
    // and then written by the same thread.
    const int q = warp % 4;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    float* blk = (float*)smem + q * (32 * 33);
    float cv[CIN ? 32 : 1];
    auto load_cin = [&](int c) {
      const int n = n0 + 32 * c + lane;
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        const int m = m0 + q * 32 + r;
        cv[r] = (m < p.M && n < p.N) ? p.Cin[(int64_t)m * p.ldcin + n] : 0.f;
      }
    };
    if constexpr (CIN) load_cin(0);
    if (mbar_wait(&bars->done, 0, abort, p.err)) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < TN / 32; ++c) {
        float v[32];
        tmem_ld32(tmem + lane_addr + 32 * c, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) blk[lane * 33 + i] = v[i];
        __syncwarp();
        const int n = n0 + 32 * c + lane;
        if constexpr (CIN) {
#pragma unroll
          for (int r = 0; r < 32; ++r) {
            const int m = m0 + q * 32 + r;
            if (m < p.M && n < p.N) {
              const float v = p.alpha * blk[r * 33 + lane] + cv[r];
              if (p.C) p.C[(int64_t)m * p.ldc + n] = v;
              if (p.C16) store_c16(p, m, n, v);
              if (p.Chi) store_split(p, m, n, v);
            }
          }
        } else {
#pragma unroll 4
          for (int r = 0; r < 32; ++r) {
            const int m = m0 + q * 32 + r;
            if (m < p.M && n < p.N) {
              float x = blk[r * 33 + lane];
              if (p.part) {
                p.part[((int64_t)blockIdx.z * p.M + m) * p.N + n] = x;
              } else {
                if (p.C) p.C[(int64_t)m * p.ldc + n] = p.alpha * x;
                if (p.C16) store_c16(p, m, n, p.alpha * x);
                if (p.Chi) store_split(p, m, n, p.alpha * x);
              }
            }
          }
        }
        __syncwarp();
        if constexpr (CIN) {
          if (c + 1 < TN / 32) load_cin(c + 1);
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

// C = alpha sum_z part[z] (+ Cin), the slices added in order
__global__ void tc_gemm_reduce_kernel(const float* __restrict__ part, int splits, Params p) {
  const int64_t mn = (int64_t)p.M * p.N;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < mn; e += (int64_t)gridDim.x * blockDim.x) {
    float v = 0.f;
    for (int z = 0; z < splits; ++z) v += part[z * mn + e];
    const int64_t m = e / p.N;
    const int n = (int)(e % p.N);
    v *= p.alpha;
    if (p.Cin) v += p.Cin[m * p.ldcin + n];
    if (p.C) p.C[m * p.ldc + n] = v;
    if (p.C16) store_c16(p, m, n, v);
    if (p.Chi) store_split(p, m, n, v);
  }
}

template <bool AMN, bool BMN, bool CIN>
void set_limit() {
  static unsigned long long done = 0;
  static std::mutex mu;
  set_smem_limit_once((const void*)tc_gemm_kernel<AMN, BMN, CIN>, SMEM_BYTES, &done, mu);
}

template <bool AMN, bool BMN, bool CIN>
sa_status launch(const char* tag, dim3 grid, cudaStream_t st, const CUtensorMap& tmA, const CUtensorMap& tmAl,
                 const CUtensorMap& tmB, const CUtensorMap& tmBl, const Params& p) {
  set_limit<AMN, BMN, CIN>();
  SA_TIMED(tag, st, (tc_gemm_kernel<AMN, BMN, CIN><<<grid, THREADS, SMEM_BYTES, st>>>(tmA, tmAl, tmB, tmBl, p)));
  return SA_OK;
}

template <bool AMN, bool BMN>
sa_status launch(bool cin, const char* tag, dim3 grid, cudaStream_t st, const CUtensorMap& tmA,
                 const CUtensorMap& tmAl, const CUtensorMap& tmB, const CUtensorMap& tmBl, const Params& p) {
  return cin ? launch<AMN, BMN, true>(tag, grid, st, tmA, tmAl, tmB, tmBl, p)
             : launch<AMN, BMN, false>(tag, grid, st, tmA, tmAl, tmB, tmBl, p);
}
}  // namespace

sa_status tc_gemm(const TcGemm& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0) return SA_OK;
  if (g.K <= 0) return fail(SA_ERR_INVALID_ARG, "tc_gemm: K must be positive");
  if (g.lda % 8 || g.ldb % 8) return fail(SA_ERR_INVALID_ARG, "tc_gemm: leading dimensions must be multiples of 8");
  if ((g.M + TM - 1) / TM > 65535) return fail(SA_ERR_UNSUPPORTED, "tc_gemm: too many row tiles");
  CUtensorMap tmA, tmAl, tmB, tmBl;
  // A: K-major [M rows of lda] or M-major [K rows of lda]; B: K-major [N rows] or N-major [K rows]
  // (the extents are the matrix's, the pitch its leading dimension, so a tail reads as zero)
  auto map_a = [&](CUtensorMap* m, const __nv_bfloat16* x) {
    return g.a_mn ? tma_map_bf16(m, x, (uint64_t)g.M, (uint64_t)g.K, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B, g.lda)
                  : tma_map_bf16(m, x, (uint64_t)g.K, (uint64_t)g.M, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B, g.lda);
  };
  auto map_b = [&](CUtensorMap* m, const __nv_bfloat16* x) {
    return g.b_mn ? tma_map_bf16(m, x, (uint64_t)g.N, (uint64_t)g.K, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B, g.ldb)
                  : tma_map_bf16(m, x, (uint64_t)g.K, (uint64_t)g.N, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B, g.ldb);
  };
  sa_status s;
  if ((s = map_a(&tmA, g.A)) != SA_OK || (s = map_b(&tmB, g.B)) != SA_OK) return s;
  tmAl = tmA;
  tmBl = tmB;
  if (g.A_lo && (s = map_a(&tmAl, g.A_lo)) != SA_OK) return s;
  if (g.B_lo && (s = map_b(&tmBl, g.B_lo)) != SA_OK) return s;
  // passes: hi x hi, then hi x lo (B split), then lo x hi (A split)
  const int ph_blo = g.B_lo ? 1 : -1;
  const int ph_alo = g.A_lo ? (g.B_lo ? 2 : 1) : -1;
  // split K while the output tiles fill less than the SMs, keeping >= 8 K slices a split
  const int tiles = ((g.N + TN - 1) / TN) * ((g.M + TM - 1) / TM), nk = (g.K + TK - 1) / TK;
  const int kSMs = device_info().sm_count;
  int split = 1;
  if (g.part && tiles < kSMs) {
    split = std::min({(kSMs + tiles - 1) / tiles, std::max(1, nk / std::max(1, g.min_split_slices)), 64});
    split = (int)std::min<int64_t>(split, (int64_t)(g.part_floats / ((size_t)g.M * g.N)));
    split = std::max(split, 1);
  }
  const int kt_per = (nk + split - 1) / split;
  split = (nk + kt_per - 1) / kt_per;            // every split gets >= 1 slice
  if (!g.C && !g.C16) return fail(SA_ERR_INVALID_ARG, "tc_gemm: no output");
  Params p{g.M, g.N, g.K, ph_alo, ph_blo, g.C, g.ldc, g.Cin, g.ldcin, g.alpha, kt_per,
           split > 1 ? g.part : nullptr, device_status_word(), g.C16, g.ldc16, g.c16_half ? 1 : 0,
           g.Chi, g.Clo, g.ldcs};
  dim3 grid((g.N + TN - 1) / TN, (g.M + TM - 1) / TM, split);
  const char* tag = g.tag ? g.tag : "tc_gemm_kernel";
  const bool cin = split == 1 && g.Cin != nullptr;
  if ((s = g.a_mn ? (g.b_mn ? launch<true, true>(cin, tag, grid, st, tmA, tmAl, tmB, tmBl, p)
                            : launch<true, false>(cin, tag, grid, st, tmA, tmAl, tmB, tmBl, p))
                  : (g.b_mn ? launch<false, true>(cin, tag, grid, st, tmA, tmAl, tmB, tmBl, p)
                            : launch<false, false>(cin, tag, grid, st, tmA, tmAl, tmB, tmBl, p))) != SA_OK)
    return s;
  if (split > 1) {
    const int64_t mn = (int64_t)g.M * g.N;
    const unsigned blocks = (unsigned)std::min<int64_t>((mn + 255) / 256, 4 * kSMs);
    Params pr = p;
    pr.part = nullptr;
    SA_TIMED("tc_gemm_reduce_kernel", st, (tc_gemm_reduce_kernel<<<blocks, 256, 0, st>>>(g.part, split, pr)));
  }
  return SA_OK;
}

}  // namespace sa
