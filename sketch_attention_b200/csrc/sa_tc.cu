// Tensor-core Sketch Attention forward for sm_100a (SequenceO1 Sec. 3.1,
// eqs. (6)-(9); the fused streaming operator of Sec. 4.4, re-designed for
// tcgen05, TMEM and TMA).
//
// Two kernels, neither of which ever writes the k x n assignment matrix:
//
//   sa_lse_tc_kernel  token-parallel, one CTA per token chunk.  Per 128-token
//     tile (moved into TMEM, the MMA's A operand) it streams P' in chunks of 128
//     prototypes: Z_c = X_t P'_c^T
//     (M=128 tokens, N=128, K=d) into TMEM; four warpgroups (32 prototypes of
//     each chunk each, one thread per token) keep an online maximum and sum of
//     2^z, and at the end of the tile combine their quarters into the token's
//     log2-sum-exp over all k prototypes.
//
//   sa_agg_tc_kernel  prototype-slice-parallel, one CTA per (128-prototype
//     slice, token chunk), transposed so the prototypes are the TMEM lanes:
//     per tile Z = P'_slice X_t^T into one of three TMEM buffers; two
//     warpgroups (64 tokens each, one thread per prototype) turn Z into
//     probabilities p = 2^(z - lse), sum them into the prototype's mass, and
//     write them back over Z as bf16 pairs, the TMEM A operand of
//     H_slice += p X_t   (M=128 prototypes, N=d, K=128 tokens)
//     which accumulates in TMEM.  At the end of a user's piece of the chunk H
//     and the mass go to HBM.
//
// The logits are computed twice (once per kernel); in exchange no CTA waits
// for another, every SM takes part, and a probability tile is written once,
// already normalised.
#include <algorithm>
#include <mutex>

#include "exp2_poly.cuh"
#include "sa_internal.cuh"
#include "tc_ptx.cuh"
#include "tma_map.cuh"

// Pairs (bit i: pair i of each group of 8 pairs) whose exponentials the lse and
// the aggregation kernel evaluate on the FMA pipe instead of the MUFU.
#ifndef SA_LSE_POLY
#define SA_LSE_POLY 0x02
#endif
#ifndef SA_AGG_POLY
#define SA_AGG_POLY 0x02
#endif

namespace sa {

namespace {
using namespace tc;

constexpr int TILE = 128;            // tokens per tile = prototypes per chunk or slice
constexpr int DD = 128;              // d
constexpr float kLn2f = 0.69314718055994530942f;
constexpr float kLog2ef = 1.44269504088896340736f;

// Iterates the tiles of chunk g: f(tile_index, piece, user, tile_begin,
// piece_end, first_tile_of_piece, last_tile_of_piece); stops if f returns false.
template <class F>
__device__ __forceinline__ void for_each_tile(const int64_t* off, int B, const Chunking& ch, int g,
                                              F&& f) {
  const int64_t cb = (int64_t)g * ch.T, ce = min(cb + ch.T, ch.n_total);
  int t = 0, piece = 0;
  for (int u = user_of_token(off, B, cb); u < B && off[u] < ce; ++u) {
    const int64_t pb = max(off[u], cb), pe = min(off[u + 1], ce);
    if (pb >= pe) continue;
    for (int64_t tb = pb; tb < pe; tb += TILE, ++t)
      if (!f(t, piece, u, tb, pe, tb == pb, tb + TILE >= pe)) return;
    ++piece;
  }
}

// 2^e for a pair: on the FMA pipe (fitted cubic) or the MUFU
template <bool POLY>
__device__ __forceinline__ float2 exp2_pair(float2 e) {
  if (POLY) return exp2_poly2(e);
  return make_float2(ex2(e.x), ex2(e.y));
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// ============================================================== lse kernel
constexpr int L_NXS = 2, L_NPS = 4;                 // X stages, P' chunk stages
constexpr uint32_t T_BYTES = TILE * DD * 2;         // [128 x 128] bf16: 2 SW128 halves of 16 KB
constexpr uint32_t L_OFF_X = 0;
constexpr uint32_t L_OFF_P = L_OFF_X + L_NXS * T_BYTES;
constexpr uint32_t L_OFF_XCH = L_OFF_P + L_NPS * T_BYTES;   // [3][2][128]: warpgroups 1-3's max and sum
constexpr uint32_t L_OFF_BAR = L_OFF_XCH + 6 * TILE * 4;
constexpr uint32_t L_SMEM = L_OFF_BAR + 256 + 1024;
constexpr int L_THREADS = 704;   // warp 0 TMA, 1 MMA + TMEM owner, 2-17 four softmax warpgroups,
                                 // 18-21 X tiles from shared memory into TMEM
// TMEM columns: two [128 x 128] fp32 logits buffers, two X tiles (bf16 pairs: the
// MMA's A operand, so the logits MMAs read only P' from shared memory)
constexpr uint32_t L_TM_Z = 0, L_TM_X = 256, L_TM_COLS = 512;

struct LBars {
  uint64_t x_full[L_NXS], x_empty[L_NXS], c_full[L_NPS], c_empty[L_NPS];
  uint64_t z_full[2], z_empty[2], xt_full[2], xt_empty[2], cx_full, cx_empty, mma_done;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(LBars) <= 256, "barrier block");

struct LParams {
  const int64_t* off;
  int B;
  Chunking ch;
  int k;
  float* lse_a;        // [n] required output: the log2-sum-exp times a_scale
  float a_scale;       // 1 (log2 units) or ln 2 (natural units)
  float* lse_b;        // [n] optional natural-log copy
  int p_user_rows;     // rows of P' per user (k: per-user prototypes), 0: one shared P'
  int* err;
};

__global__ void __launch_bounds__(L_THREADS, 1)
    sa_lse_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP,
                     LParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  LBars* bars = (LBars*)(smem + L_OFF_BAR);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = blockIdx.x;
  if (g >= p.ch.G) return;
  const int nch = p.k / TILE;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L_NXS; ++s) { mbar_init(&bars->x_full[s], 1); mbar_init(&bars->x_empty[s], 128); }
    for (int s = 0; s < L_NPS; ++s) { mbar_init(&bars->c_full[s], 1); mbar_init(&bars->c_empty[s], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->z_full[b], 1);
      mbar_init(&bars->z_empty[b], 512);
      mbar_init(&bars->xt_full[b], 128);
      mbar_init(&bars->xt_empty[b], 1);
    }
    mbar_init(&bars->cx_full, 384);
    mbar_init(&bars->cx_empty, 128);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, L_TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmP);
    int cc = 0, issued_t = 0, issued_c = 0;
    for_each_tile(p.off, p.B, p.ch, g, [&](int t, int, int u, int64_t tb, int64_t, bool, bool) {
      const int s = t % L_NXS;
      const int prow0 = u * p.p_user_rows;
      if (t >= L_NXS && !mbar_wait(&bars->x_empty[s], ((t / L_NXS) - 1) & 1, abort, p.err)) return false;
      mbar_arrive_expect_tx(&bars->x_full[s], T_BYTES);
      uint8_t* xd = smem + L_OFF_X + s * T_BYTES;
      tma_load_2d(xd, &tmX, &bars->x_full[s], 0, (int)tb);
      tma_load_2d(xd + T_BYTES / 2, &tmX, &bars->x_full[s], 64, (int)tb);
      issued_t = t + 1;
      for (int c = 0; c < nch; ++c, ++cc) {
        const int cs = cc % L_NPS;
        if (cc >= L_NPS && !mbar_wait(&bars->c_empty[cs], ((cc / L_NPS) - 1) & 1, abort, p.err)) return false;
        mbar_arrive_expect_tx(&bars->c_full[cs], T_BYTES);
        uint8_t* pd = smem + L_OFF_P + cs * T_BYTES;
        tma_load_2d(pd, &tmP, &bars->c_full[cs], 0, prow0 + c * TILE);
        tma_load_2d(pd + T_BYTES / 2, &tmP, &bars->c_full[cs], 64, prow0 + c * TILE);
        issued_c = cc + 1;
      }
      return true;
    });
    if (*abort) {
      for (int t = std::max(0, issued_t - L_NXS); t < issued_t; ++t)
        mbar_wait_bounded(&bars->x_full[t % L_NXS], (t / L_NXS) & 1);
      for (int c = std::max(0, issued_c - L_NPS); c < issued_c; ++c)
        mbar_wait_bounded(&bars->c_full[c % L_NPS], (c / L_NPS) & 1);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ logits MMAs
    // Z_c = X_t P'_c^T with X_t from TMEM (A) and P'_c from shared memory (B)
    const uint32_t id = idesc_bf16(128, 128, false, false);
    int ai = 0;
    for_each_tile(p.off, p.B, p.ch, g, [&](int t, int, int, int64_t, int64_t, bool, bool) {
      const int xb = t & 1;
      if (!mbar_wait(&bars->xt_full[xb], (t >> 1) & 1, abort, p.err)) return false;
      for (int c = 0; c < nch; ++c) {
        const int a = ai + c, cs = a % L_NPS, b = a & 1;
        if (!mbar_wait(&bars->c_full[cs], (a / L_NPS) & 1, abort, p.err)) return false;
        if (a >= 2 && !mbar_wait(&bars->z_empty[b], ((a >> 1) - 1) & 1, abort, p.err)) return false;
        tc_fence_after();
        const uint32_t pa = smem_u32(smem + L_OFF_P + cs * T_BYTES);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts(tmem + L_TM_Z + 128 * b, tmem + L_TM_X + 64 * xb + 8 * ks,
                 smem_desc(pa + (ks >> 2) * (T_BYTES / 2) + (ks & 3) * 32, 16, 1024, SWZ_128B), id,
                 ks > 0 ? 1u : 0u);
        mma_commit(&bars->z_full[b]);
        mma_commit(&bars->c_empty[cs]);                     // P' is read by this MMA only
      }
      mma_commit(&bars->xt_empty[xb]);                      // X in TMEM is read by these MMAs only
      ai += nch;
      return true;
    });
    mma_commit(&bars->mma_done);
    mbar_wait_bounded(&bars->mma_done, 0);
  } else if (warp >= 2 && warp <= 17) {
    // ------------------------------------------------------------ four threads per token
    // warpgroup h reads columns 32h..32h+31 of each chunk's logits
    const int q = warp % 4, h = (warp - 2) / 4;
    const int row = q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    float* xch = (float*)(smem + L_OFF_XCH);
    int ai = 0;
    for_each_tile(p.off, p.B, p.ch, g, [&](int t, int, int, int64_t tb, int64_t pe, bool, bool) {
      float m = -__builtin_huge_valf();
      float2 s2 = make_float2(0.f, 0.f);
      for (int c = 0; c < nch; ++c) {
        const int a = ai + c, b = a & 1;
        if (!mbar_wait(&bars->z_full[b], (a >> 1) & 1, abort, p.err)) return false;
        tc_fence_after();
        float z[32];
        tmem_ld32(tmem + lane_addr + L_TM_Z + 128 * b + 32 * h, z);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->z_empty[b]);
        float mz = max3f(z[0], z[1], z[2]);
#pragma unroll
        for (int j = 3; j + 1 < 32; j += 2) mz = max3f(mz, z[j], z[j + 1]);
        const float mn = fmaxf(m, fmaxf(mz, z[31]));
        const float sc = ex2(m - mn);                      // 0 on the first chunk
        s2 = __fmul2_rn(s2, make_float2(sc, sc));
        m = mn;
        const float2 nm = make_float2(-mn, -mn);
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 e = __fadd2_rn(make_float2(z[j], z[j + 1]), nm);
          const float2 v = ((SA_LSE_POLY >> ((j / 2) & 7)) & 1) ? exp2_pair<true>(e) : exp2_pair<false>(e);
          s2 = __fadd2_rn(s2, v);
        }
      }
      ai += nch;
      const float s = s2.x + s2.y;
      if (h > 0) {
        // hand the quarter-row statistics to warpgroup 0 (the slot is free once it read the last ones)
        if (t > 0 && !mbar_wait(&bars->cx_empty, (t - 1) & 1, abort, p.err)) return false;
        xch[(h - 1) * 2 * TILE + row] = m;
        xch[(h - 1) * 2 * TILE + TILE + row] = s;
        mbar_arrive(&bars->cx_full);
        return true;
      }
      if (!mbar_wait(&bars->cx_full, t & 1, abort, p.err)) return false;
      float mm[3], ss[3];
#pragma unroll
      for (int w = 0; w < 3; ++w) { mm[w] = xch[w * 2 * TILE + row]; ss[w] = xch[w * 2 * TILE + TILE + row]; }
      mbar_arrive(&bars->cx_empty);
      const float M = fmaxf(fmaxf(m, mm[0]), fmaxf(mm[1], mm[2]));
      const float l2 = M + lg2(s * ex2(m - M) + ss[0] * ex2(mm[0] - M) + ss[1] * ex2(mm[1] - M) + ss[2] * ex2(mm[2] - M));
      if (tb + row < pe) {
        p.lse_a[tb + row] = l2 * p.a_scale;
        if (p.lse_b) p.lse_b[tb + row] = l2 * kLn2f;
      }
      return true;
    });
  } else if (warp >= 18) {
    // ------------------------------------------------------------ X tile into TMEM
    // Each thread moves its token's row (16 pieces of 16 bytes; piece 8a + c of the
    // row sits in 128-byte-swizzled half a at chunk c ^ (row % 8)) into TMEM as bf16
    // pairs, the A operand of the tile's logits MMAs.
    const int q = warp % 4;
    const int row = q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    for_each_tile(p.off, p.B, p.ch, g, [&](int t, int, int, int64_t, int64_t, bool, bool) {
      const int s = t % L_NXS, xb = t & 1;
      if (!mbar_wait(&bars->x_full[s], (t / L_NXS) & 1, abort, p.err)) return false;
      if (t >= 2 && !mbar_wait(&bars->xt_empty[xb], ((t >> 1) - 1) & 1, abort, p.err)) return false;
      const uint32_t base = smem_u32(smem + L_OFF_X + s * T_BYTES) + row * 128;
      uint32_t v[64];
#pragma unroll
      for (int pc = 0; pc < 16; ++pc) {
        const uint32_t addr = base + (pc >> 3) * (T_BYTES / 2) + (((pc & 7) ^ (row & 7)) << 4);
        asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(v[4 * pc]), "=r"(v[4 * pc + 1]), "=r"(v[4 * pc + 2]), "=r"(v[4 * pc + 3])
                     : "r"(addr));
      }
      mbar_arrive(&bars->x_empty[s]);
      tc_fence_after();
      tmem_st32(tmem + lane_addr + L_TM_X + 64 * xb, v);
      tmem_st32(tmem + lane_addr + L_TM_X + 64 * xb + 32, v + 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->xt_full[xb]);
      return true;
    });
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L_TM_COLS);
  }
}

// ============================================================== aggregation kernel
// Transposed: the prototypes of the slice are the MMA rows (TMEM lanes), the
// tokens the columns, so the probabilities are written where the logits were
// and feed the aggregation MMA from TMEM:
//   Z_t = P'_slice X_t^T   (M=128 prototypes, N=128 tokens, K=d; both operands in shared memory)
//   p   = 2^(Z_t - lse)     fp32 -> bf16 pairs over the first half of the warpgroup's own
//                           Z columns (each warpgroup owns 64 tokens); the fp32 values
//                           are summed in registers into the prototype's mass
//   H  += p X_t            (M=128 prototypes, N=d, K=128 tokens; p from TMEM, X MN-major)
// A tile's logits -> probabilities -> aggregation chain crosses three mbarrier
// hand-offs, so three logits buffers are kept in flight; that takes every TMEM
// column (3 x 128 + H 128), which is why P' is a shared-memory operand here and
// the mass is not an extra block of MMA columns.
#ifndef SA_AGG_NS
#define SA_AGG_NS 4
#endif
constexpr int A_NS = SA_AGG_NS;                       // X stages (a tile is held until its aggregation)
constexpr int A_NZ = 3;                               // logits/probability buffers
constexpr uint32_t X_BOX = TILE * 32;                 // one [128 x 16] bf16 SW32 box = 4 KB
constexpr uint32_t X_STAGE = 8 * X_BOX;               // 32 KB
constexpr uint32_t A_OFF_PQ = 0;                      // P' slice: 2 x [128 x 64] SW128 = 32 KB
constexpr uint32_t A_OFF_X = T_BYTES;
constexpr uint32_t A_OFF_LSE = A_OFF_X + A_NS * X_STAGE;   // [A_NS][128] fp32: -lse of the stage's tokens
constexpr uint32_t A_OFF_M = A_OFF_LSE + A_NS * TILE * 4;  // [2 slots][2 warpgroups][128] partial masses
constexpr uint32_t A_OFF_BAR = A_OFF_M + 2 * 2 * TILE * 4;
constexpr uint32_t A_SMEM = A_OFF_BAR + 256 + 1024;
constexpr int A_THREADS = 480;   // warp 0 TMA + lse tiles, 1 logits MMAs + TMEM owner, 2 aggregation
                                 // MMAs, 3-6 H drain, 7-10 and 11-14 two softmax warpgroups
constexpr uint32_t A_TM_Z = 0, A_TM_H = 384, A_TM_COLS = 512;
static_assert(A_SMEM <= 232448, "shared memory per CTA");

struct ABars {
  uint64_t x_full[A_NS], x_empty[A_NS], z_full[A_NZ], p_full[A_NZ], z_free[A_NZ];
  uint64_t h_full, h_empty, pq_full, pq_empty, m_full[2], m_empty[2], mma_done[2];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(ABars) <= 256, "barrier block");

struct AParams {
  const int64_t* off;
  int B;
  Chunking ch;
  int k;
  const float* lse;    // [n] per-token log-sum-exp, times in_scale in log2 units
  float in_scale;
  float* Huser;        // [B, k, d] users that lie inside one chunk
  float* Muser;        // [B, k]
  float* slotH;        // [G, 2, k, d] pieces at chunk boundaries
  float* slotM;        // [G, 2, k]
  int p_user_rows;     // rows of P' per user (k: per-user prototypes), 0: one shared P'
  int* err;
};

__global__ void __launch_bounds__(A_THREADS, 1)
    sa_agg_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP,
                     AParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  ABars* bars = (ABars*)(smem + A_OFF_BAR);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int slices = p.k / TILE;
  const int sl = blockIdx.x % slices, g = blockIdx.x / slices;
  if (g >= p.ch.G) return;
  const bool per_user = p.p_user_rows > 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < A_NS; ++s) { mbar_init(&bars->x_full[s], 1); mbar_init(&bars->x_empty[s], 1); }
    for (int b = 0; b < A_NZ; ++b) {
      mbar_init(&bars->z_full[b], 1);
      mbar_init(&bars->p_full[b], 256);
      mbar_init(&bars->z_free[b], 1);
    }
    for (int b = 0; b < 2; ++b) { mbar_init(&bars->m_full[b], 256); mbar_init(&bars->m_empty[b], 128); }
    mbar_init(&bars->h_full, 1);
    mbar_init(&bars->h_empty, 128);
    mbar_init(&bars->pq_full, 1);
    mbar_init(&bars->pq_empty, 1);
    mbar_init(&bars->mma_done[0], 1);
    mbar_init(&bars->mma_done[1], 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, A_TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int64_t n_total = p.off[p.B];

  if (warp == 0) {
    // ------------------------------------------------------------ P' slices, X tiles, -lse tiles
    // The warp copies the tile's per-token -lse (-inf past the piece: p = 0) into the
    // stage's slot before lane 0 arrives on x_full; the values are loaded a tile ahead.
    // Lane 0 takes every wait and tells the warp (a uniform decision: no lane may be
    // left behind at the __syncwarp below).
    if (lane == 0) {
      prefetch_tensormap(&tmX);
      prefetch_tensormap(&tmP);
    }
    int issued = 0, pq_issued = 0;
    float cur[4], nxt[4];
    for_each_tile(p.off, p.B, p.ch, g, [&](int t, int piece, int u, int64_t tb, int64_t pe, bool first, bool) {
      const int s = t % A_NS;
      bool ok = true;
      if (first && (piece == 0 || per_user)) {
        // the P' slice: once, or at every user's first tile when the prototypes are per user
        if (lane == 0) {
          if (piece > 0) ok = mbar_wait(&bars->pq_empty, (piece - 1) & 1, abort, p.err);
          if (ok) {
            mbar_arrive_expect_tx(&bars->pq_full, T_BYTES);
            const int prow = u * p.p_user_rows + sl * TILE;
            tma_load_2d(smem + A_OFF_PQ, &tmP, &bars->pq_full, 0, prow);
            tma_load_2d(smem + A_OFF_PQ + T_BYTES / 2, &tmP, &bars->pq_full, 64, prow);
            pq_issued = piece + 1;
          }
        }
        if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) return false;
      }
      if (t == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int64_t tok = tb + 32 * i + lane;
          cur[i] = tok < n_total ? p.lse[tok] : 0.f;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) cur[i] = nxt[i];
      }
      const int64_t nb = tb + TILE < pe ? tb + TILE : pe;   // the next tile's first token
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t tok = nb + 32 * i + lane;
        if (tok < n_total) nxt[i] = p.lse[tok];
      }
      if (t >= A_NS && lane == 0) ok = mbar_wait(&bars->x_empty[s], ((t / A_NS) - 1) & 1, abort, p.err);
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) return false;
      float* ls = (float*)(smem + A_OFF_LSE) + s * TILE;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t tok = tb + 32 * i + lane;
        ls[32 * i + lane] = tok < pe ? -cur[i] * p.in_scale : -__builtin_huge_valf();
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars->x_full[s], X_STAGE);
        uint8_t* dst = smem + A_OFF_X + s * X_STAGE;
        for (int bx = 0; bx < 8; ++bx) tma_load_2d(dst + bx * X_BOX, &tmX, &bars->x_full[s], 16 * bx, (int)tb);
      }
      issued = t + 1;
      return true;
    });
    if (*abort && lane == 0) {
      if (pq_issued > 0) mbar_wait_bounded(&bars->pq_full, (pq_issued - 1) & 1);
      for (int t = std::max(0, issued - A_NS); t < issued; ++t)
        mbar_wait_bounded(&bars->x_full[t % A_NS], (t / A_NS) & 1);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ logits MMAs
    const uint32_t id1 = idesc_bf16(128, 128, false, false);
    const uint64_t dp = smem_desc(smem_u32(smem + A_OFF_PQ), 16, 1024, SWZ_128B);
    for_each_tile(p.off, p.B, p.ch, g, [&](int t, int piece, int, int64_t, int64_t, bool first, bool last) {
      const int s = t % A_NS, b = t % A_NZ;
      if (first && (piece == 0 || per_user) &&
          !mbar_wait(&bars->pq_full, (per_user ? piece : 0) & 1, abort, p.err))
        return false;
      if (!mbar_wait(&bars->x_full[s], (t / A_NS) & 1, abort, p.err)) return false;
      // buffer b was last read (as probabilities) by the aggregation of tile t - A_NZ
      if (t >= A_NZ && !mbar_wait(&bars->z_free[b], ((t / A_NZ) - 1) & 1, abort, p.err)) return false;
      tc_fence_after();
      const uint64_t dx = smem_desc(smem_u32(smem + A_OFF_X + s * X_STAGE), 16, 256, SWZ_32B);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_ss(tmem + A_TM_Z + 128 * b, dp + (uint64_t)((((ks >> 2) * (T_BYTES / 2)) + (ks & 3) * 32) >> 4),
               dx + (uint64_t)((ks * X_BOX) >> 4), id1, ks > 0 ? 1u : 0u);
      mma_commit(&bars->z_full[b]);
      if (last && per_user) mma_commit(&bars->pq_empty);   // this user's P' slice is done
      return true;
    });
    mma_commit(&bars->mma_done[0]);
    mbar_wait_bounded(&bars->mma_done[0], 0);
  } else if (warp == 2 && lane == 0) {
    // ------------------------------------------------------------ aggregation MMAs
    const uint32_t id2 = idesc_bf16(128, DD, false, true);
    for_each_tile(p.off, p.B, p.ch, g, [&](int t, int piece, int, int64_t, int64_t, bool first, bool last) {
      const int s = t % A_NS, b = t % A_NZ;
      if (first && piece > 0 && !mbar_wait(&bars->h_empty, (piece - 1) & 1, abort, p.err)) return false;
      if (!mbar_wait(&bars->p_full[b], (t / A_NZ) & 1, abort, p.err)) return false;
      tc_fence_after();
      const uint64_t dx = smem_desc(smem_u32(smem + A_OFF_X + s * X_STAGE), X_BOX, 256, SWZ_32B);
      // tokens 16 ks .. 16 ks + 15: warpgroup ks / 4 wrote their pairs at its column base
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_ts(tmem + A_TM_H, tmem + A_TM_Z + 128 * b + 64 * (ks >> 2) + 8 * (ks & 3),
               dx + (uint64_t)((ks * 512) >> 4), id2, (first && ks == 0) ? 0u : 1u);
      mma_commit(&bars->x_empty[s]);
      mma_commit(&bars->z_free[b]);
      if (last) mma_commit(&bars->h_full);
      return true;
    });
    mma_commit(&bars->mma_done[1]);
    mbar_wait_bounded(&bars->mma_done[1], 0);
  } else if (warp >= 3 && warp <= 6) {
    // ------------------------------------------------------------ H and the mass out of the SM
    const int q = warp % 4;
    const int row = q * 32 + lane;                     // prototype of the slice = TMEM lane
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const int64_t cb = (int64_t)g * p.ch.T, ce = min(cb + p.ch.T, p.ch.n_total);
    const float* msl = (const float*)(smem + A_OFF_M);
    for_each_tile(p.off, p.B, p.ch, g, [&](int, int piece, int u, int64_t, int64_t, bool, bool last) {
      if (!last) return true;
      if (!mbar_wait(&bars->h_full, piece & 1, abort, p.err)) return false;
      tc_fence_after();
      const int dest = piece_dest(p.off[u], p.off[u + 1], cb, ce);
      const int j = sl * TILE + row;
      float* Hrow;
      float* mrow;
      if (dest == DEST_USER) {
        Hrow = p.Huser + ((int64_t)u * p.k + j) * DD;
        mrow = p.Muser + (int64_t)u * p.k + j;
      } else {
        Hrow = p.slotH + (((int64_t)g * 2 + dest) * p.k + j) * DD;
        mrow = p.slotM + ((int64_t)g * 2 + dest) * p.k + j;
      }
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        float hv[16];
        tmem_ld16(tmem + lane_addr + A_TM_H + 16 * c, hv);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          *(float4*)(Hrow + 16 * c + i) = make_float4(hv[i], hv[i + 1], hv[i + 2], hv[i + 3]);
      }
      tc_fence_before();
      mbar_arrive(&bars->h_empty);
      // the piece's mass: the two softmax warpgroups' sums of this prototype's probabilities
      const int slot = piece & 1;
      if (!mbar_wait(&bars->m_full[slot], (piece >> 1) & 1, abort, p.err)) return false;
      *mrow = msl[(slot * 2 + 0) * TILE + row] + msl[(slot * 2 + 1) * TILE + row];
      mbar_arrive(&bars->m_empty[slot]);
      return true;
    });
  } else if (warp >= 7) {
    // ------------------------------------------------------------ probabilities
    // warpgroup h owns tokens 64h..64h+63 of each tile (TMEM columns of the buffer);
    // each thread one prototype (TMEM lane)
    const int q = warp % 4, h = (warp - 7) / 4;
    const int row = q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    float* msl = (float*)(smem + A_OFF_M);
    float2 msum = make_float2(0.f, 0.f);
    for_each_tile(p.off, p.B, p.ch, g, [&](int t, int piece, int, int64_t, int64_t, bool, bool last) {
      const int s = t % A_NS, b = t % A_NZ;
      // the stage's -lse values were written before its x_full arrival
      if (!mbar_wait(&bars->x_full[s], (t / A_NS) & 1, abort, p.err)) return false;
      if (!mbar_wait(&bars->z_full[b], (t / A_NZ) & 1, abort, p.err)) return false;
      tc_fence_after();
      const uint32_t zc = tmem + lane_addr + A_TM_Z + 128 * b + 64 * h;
      const float4* nl = (const float4*)((const float*)(smem + A_OFF_LSE) + s * TILE + 64 * h);
      // two passes of 32 tokens; pass c writes its 16 pairs over Z columns the
      // warpgroup has already read (columns 16c..16c+15 of its 64)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float z[32];
        tmem_ld32(zc + 32 * c, z);
        tmem_wait_ld();
        uint32_t o[16];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 l = nl[8 * c + j / 4];
          const float2 e0 = __fadd2_rn(make_float2(z[j], z[j + 1]), make_float2(l.x, l.y));
          const float2 e1 = __fadd2_rn(make_float2(z[j + 2], z[j + 3]), make_float2(l.z, l.w));
          const float2 v0 = ((SA_AGG_POLY >> ((j / 2) & 7)) & 1) ? exp2_pair<true>(e0) : exp2_pair<false>(e0);
          const float2 v1 = ((SA_AGG_POLY >> ((j / 2 + 1) & 7)) & 1) ? exp2_pair<true>(e1) : exp2_pair<false>(e1);
          msum = __fadd2_rn(msum, __fadd2_rn(v0, v1));
          o[j / 2] = pack_bf16x2(v0.x, v0.y);
          o[j / 2 + 1] = pack_bf16x2(v1.x, v1.y);
        }
        tmem_st16(zc + 16 * c, o);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[b]);
      if (last) {
        // hand this warpgroup's part of the prototype's mass to the drain (slot piece % 2,
        // free once the drain of piece - 2 has read it)
        const int slot = piece & 1;
        if (piece >= 2 && !mbar_wait(&bars->m_empty[slot], ((piece >> 1) - 1) & 1, abort, p.err)) return false;
        msl[(slot * 2 + h) * TILE + row] = msum.x + msum.y;
        mbar_arrive(&bars->m_full[slot]);
        msum = make_float2(0.f, 0.f);
      }
      return true;
    });
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, A_TM_COLS);
  }
}

// ============================================================== host side

// [outer, 128] bf16 rows; boxes of box_inner x 128 rows
sa_status make_map(CUtensorMap* map, const void* base, uint64_t outer, uint32_t box_inner,
                   CUtensorMapSwizzle swz) {
  return tma_map_bf16(map, base, DD, outer, box_inner, TILE, swz);
}

std::mutex g_mu;
bool g_attr_set[64] = {};

void set_attributes() {
  const int dev = device_info().device & 63;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_attr_set[dev]) return;
  cudaFuncSetAttribute(sa_lse_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L_SMEM);
  cudaFuncSetAttribute(sa_agg_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, A_SMEM);
  g_attr_set[dev] = true;
}
}  // namespace

bool sa_tc_supported(sa_dtype x_dtype, int k, int d) {
  return x_dtype == SA_BF16 && d == DD && k % TILE == 0 && k >= TILE && k <= 4096;
}

// token chunks of the aggregation kernel: one CTA per (slice, chunk), about one wave
int sa_tc_num_chunks(int k) { return std::max(1, device_info().sm_count / (k / TILE)); }

sa_status sa_tc_forward(const SaFwdArgs& a, const SaFwdWork& w, cudaStream_t st) {
  if (a.n_total >= (1LL << 31)) return fail(SA_ERR_UNSUPPORTED, "n_total must be < 2^31");
  // the per-token log-sum-exp goes to the workspace (log2 units) or, when the
  // workspace has none, to the caller's natural-log output
  float* lse_a = w.lse;
  float a_scale = 1.f, in_scale = 1.f;
  float* lse_b = a.lse_out;
  if (!lse_a) {
    if (!a.lse_out) return fail(SA_ERR_INVALID_ARG, "the forward needs an lse buffer");
    lse_a = a.lse_out;
    lse_b = nullptr;
    a_scale = kLn2f;
    in_scale = kLog2ef;
  }
  CUtensorMap tmX128, tmX32, tmP;
  sa_status s;
  if ((s = make_map(&tmX128, a.X, (uint64_t)a.n_total, 64, CU_TENSOR_MAP_SWIZZLE_128B)) != SA_OK) return s;
  if ((s = make_map(&tmX32, a.X, (uint64_t)a.n_total, 16, CU_TENSOR_MAP_SWIZZLE_32B)) != SA_OK) return s;
  const uint64_t p_rows = (uint64_t)a.k * (a.p_user_rows > 0 ? (uint64_t)a.B : 1);
  if ((s = make_map(&tmP, w.Pb, p_rows, 64, CU_TENSOR_MAP_SWIZZLE_128B)) != SA_OK) return s;
  set_attributes();
  const Chunking ch1 = make_chunking(a.n_total, device_info().sm_count, 1);
  LParams lp{a.off_dev, a.B, ch1, a.k, lse_a, a_scale, lse_b, a.p_user_rows, device_status_word()};
  SA_TIMED("sa_lse_tc_kernel", st, (sa_lse_tc_kernel<<<ch1.G, L_THREADS, L_SMEM, st>>>(tmX128, tmP, lp)));
  AParams ap{a.off_dev, a.B, w.ch, a.k, lse_a, in_scale, a.S, w.Muser, w.slotH, w.slotM, a.p_user_rows,
             device_status_word()};
  SA_TIMED("sa_agg_tc_kernel", st,
           (sa_agg_tc_kernel<<<(a.k / TILE) * w.ch.G, A_THREADS, A_SMEM, st>>>(tmX32, tmP, ap)));
  return SA_OK;
}

}  // namespace sa
