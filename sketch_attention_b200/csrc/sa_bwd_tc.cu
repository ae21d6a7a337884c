// Tensor-core Sketch Attention backward for sm_100a: the chain rule of the SA
// forward (SequenceO1 Sec. 3.1, eqs. (6)-(9); the pages call SA fully
// differentiable and print no backward).
//
// With A = 2^{z - lse} (z = P' x in base-2 units, lse saved by the forward),
// dA_tj = dH_j . x_t + dm_j, c_t = sum_j A_tj dA_tj and dZ = A o (dA - c):
//   dX_t = sum_j A_tj dH_j + ln2 sum_j dZ_tj P'_j
//        = Q_t - ln2 c_t V_t,   Q = A dH + ln2 (A o dA) P',  V = A P'
//   E    = sum_t dZ_t^T x_t   (weight gradients follow from E by small GEMMs)
// dm is centred per user (dZ and dX do not change when a constant is added to
// dA); this keeps ln2 (A o dA) P' - ln2 c V free of a large common term.
//
// Two kernels:
//   sa_bwd_dx_tc_kernel  token-parallel: one CTA per token chunk, all k per
//     tile in chunks of 64 prototypes.  Per chunk: [Z|G] = X [P'_c;dH_c]^T
//     (M=128 tokens, N=128), then A and ln2 A o dA as bf16 into TMEM, and
//     V += A P'_c,  Q += A dH_c + (ln2 A o dA) P'_c  (the two terms of Q share
//     one accumulator by concatenating their K; A is the TMEM operand, so the
//     aggregation MMAs read only P'_c and dH_c from shared memory).  Q also
//     takes A times the bf16 residual of dH (dH = dH_hi + dH_lo), so only A's
//     rounding is left in it.  c_t accumulates in registers; at the end of
//     the tile dX = Q - ln2 c V, so c is not needed beforehand.
//   sa_bwd_e_tc_kernel   prototype-slice-parallel: one CTA per (128-prototype
//     slice, token chunk).  Per tile: [Z|G] (N=256), dZ (bf16, SMEM), then
//     E_slice += dZ^T X (M=128 prototypes, N=128) in TMEM.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "sa_internal.cuh"
#include "exp2_poly.cuh"
#include "tc_ptx.cuh"
#include "tma_map.cuh"

// Pairs (of the 4 in a group of 8 prototypes) whose exponentials the E kernel
// evaluates on the FMA pipe instead of the MUFU.
#ifndef SA_E_POLY_PAIRS
#define SA_E_POLY_PAIRS 0x0
#endif

namespace sa {

namespace {
using namespace tc;

constexpr int TILE = 128, DD = 128;
constexpr float kLn2f = 0.69314718055994530942f;

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

// ============================================================== dX kernel
constexpr int KC = 64;                       // prototypes per chunk
constexpr int DX_NXS = 1, DX_NCS = 4;        // X stages (only the logits MMAs read X), chunk stages
constexpr uint32_t XT_BYTES = 32768;         // [128 tokens x 128] bf16: 2 SW128 halves of 16 KB
constexpr uint32_t CH_BYTES = 49152;         // [P' h0 | dH h0 | P' h1 | dH h1 | dHlo h0 | dHlo h1], 8 KB each
constexpr uint32_t DX_OFF_X = 0;
constexpr uint32_t DX_OFF_CH = DX_OFF_X + DX_NXS * XT_BYTES;
constexpr uint32_t DX_OFF_DM = DX_OFF_CH + DX_NCS * CH_BYTES;
constexpr uint32_t DX_OFF_CP = DX_OFF_DM + DX_NCS * KC * 4;      // [128] partial c of warpgroup 1
constexpr uint32_t DX_OFF_BAR = DX_OFF_CP + TILE * 4;
constexpr uint32_t DX_SMEM = DX_OFF_BAR + 256 + 1024;
constexpr int DX_THREADS = 352;              // warp 0 TMA, 1 logits MMAs, 2-9 two threads per
                                             // token, 10 aggregation MMAs
// TMEM columns: [Z|G] of the current chunk; V = A P'; Q = A dH + (ln2 A o dA) P';
// two buffers of the chunk's A and ln2 A o dA as bf16 pairs (the TMEM operand
// of the aggregation MMAs: 32 columns each).
constexpr uint32_t DX_TM_ZG = 0, DX_TM_V = 128, DX_TM_Q = 256, DX_TM_AA = 384;

struct DxBars {
  // avq_done[s]: the aggregation MMAs of the chunk in stage s completed, so
  // both its shared-memory stage and its TMEM A buffer are free again
  uint64_t x_full[DX_NXS], x_empty[DX_NXS], c_full[DX_NCS], avq_done[DX_NCS];
  uint64_t zg_full, zg_empty, aa_full[2], acc_full, cx_full, cx_empty, mma_done[2];
  uint32_t tmem_base;
  int abort;
};

struct DxParams {
  const int64_t* off;
  int B;
  Chunking ch;
  int k;
  const float* lse2;     // [n] per-token log2-sum-exp
  const float* dmc;      // [B, k] centred dm
  __nv_bfloat16* dX;     // [n, d] (unless dX32)
  float* cout;           // [n]
  int* err;
  float* dX32;           // optional [n, d] fp32 output instead of dX, added to when acc32
  int acc32;
  int p_user_rows;       // rows of P' per user (k: per-user prototypes), 0: one shared P'
};

// 384: caps registers at 168, as three warps share two of the SM's sub-partitions
__global__ void __launch_bounds__(384, 1)
    sa_bwd_dx_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP,
                        const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmL,
                        DxParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  DxBars* bars = (DxBars*)(smem + DX_OFF_BAR);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = blockIdx.x;
  if (g >= p.ch.G) return;
  const int nch = p.k / KC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < DX_NXS; ++s) { mbar_init(&bars->x_full[s], 1); mbar_init(&bars->x_empty[s], 1); }
    for (int s = 0; s < DX_NCS; ++s) { mbar_init(&bars->c_full[s], 1); mbar_init(&bars->avq_done[s], 1); }
    mbar_init(&bars->zg_full, 1);
    mbar_init(&bars->zg_empty, 256);
    for (int b = 0; b < 2; ++b) mbar_init(&bars->aa_full[b], 256);
    mbar_init(&bars->cx_full, 128);
    mbar_init(&bars->cx_empty, 128);
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->mma_done[0], 1);
    mbar_init(&bars->mma_done[1], 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
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
    prefetch_tensormap(&tmH);
    prefetch_tensormap(&tmL);
    int cc = 0, issued_t = 0, issued_c = 0;
    const int64_t n_total = p.off[p.B];
    for_each_tile(p.off, p.B, p.ch, g, [&](int t, int, int u, int64_t tb, int64_t pe, bool, bool) {
      // the next X tile (in this user, else the next user's first rows) to L2
      const int64_t nx = tb + TILE < pe ? tb + TILE : pe;
      if (nx < n_total) {
        tma_prefetch_l2_2d(&tmX, 0, (int)nx);
        tma_prefetch_l2_2d(&tmX, 64, (int)nx);
      }
      auto load_x = [&]() -> bool {
        const int s = t % DX_NXS;
        if (t >= DX_NXS && !mbar_wait(&bars->x_empty[s], ((t / DX_NXS) - 1) & 1, abort, p.err)) return false;
        mbar_arrive_expect_tx(&bars->x_full[s], XT_BYTES);
        uint8_t* xd = smem + DX_OFF_X + s * XT_BYTES;
        tma_load_2d(xd, &tmX, &bars->x_full[s], 0, (int)tb);
        tma_load_2d(xd + XT_BYTES / 2, &tmX, &bars->x_full[s], 64, (int)tb);
        issued_t = t + 1;
        return true;
      };
      // Stages free up in the order the previous tile's MMAs complete: chunks
      // nch-4 and nch-3 before the tile's X (its last logits MMA), the rest
      // after; so this tile's first two chunks are loaded before its X.
      const int x_at = std::min(2, nch);
      for (int c = 0; c < nch; ++c, ++cc) {
        if (c == x_at && !load_x()) return false;
        const int cs = cc % DX_NCS;
        if (cc >= DX_NCS && !mbar_wait(&bars->avq_done[cs], ((cc / DX_NCS) - 1) & 1, abort, p.err)) return false;
        mbar_arrive_expect_tx(&bars->c_full[cs], CH_BYTES + KC * 4);
        uint8_t* cd = smem + DX_OFF_CH + cs * CH_BYTES;
        const int hrow = (int)((int64_t)u * p.k + c * KC);
        const int prow = (int)((int64_t)u * p.p_user_rows + c * KC);
        tma_load_2d(cd, &tmP, &bars->c_full[cs], 0, prow);
        tma_load_2d(cd + 8192, &tmH, &bars->c_full[cs], 0, hrow);
        tma_load_2d(cd + 16384, &tmP, &bars->c_full[cs], 64, prow);
        tma_load_2d(cd + 24576, &tmH, &bars->c_full[cs], 64, hrow);
        tma_load_2d(cd + 32768, &tmL, &bars->c_full[cs], 0, hrow);
        tma_load_2d(cd + 40960, &tmL, &bars->c_full[cs], 64, hrow);
        bulk_load(smem + DX_OFF_DM + cs * KC * 4, p.dmc + (int64_t)u * p.k + c * KC, KC * 4, &bars->c_full[cs]);
        issued_c = cc + 1;
      }
      if (x_at == nch && !load_x()) return false;
      return true;
    });
    if (*abort) {
      for (int t = std::max(0, issued_t - DX_NXS); t < issued_t; ++t)
        mbar_wait_bounded(&bars->x_full[t % DX_NXS], (t / DX_NXS) & 1);
      for (int c = std::max(0, issued_c - DX_NCS); c < issued_c; ++c)
        mbar_wait_bounded(&bars->c_full[c % DX_NCS], (c / DX_NCS) & 1);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ logits MMA issuer
    const uint32_t id_zg = idesc_bf16(128, 128, false, false);
    int ai = 0;   // global chunk index
    for_each_tile(p.off, p.B, p.ch, g, [&](int t, int, int, int64_t, int64_t, bool, bool) {
      const int s = t % DX_NXS;
      if (!mbar_wait(&bars->x_full[s], (t / DX_NXS) & 1, abort, p.err)) return false;
      const uint32_t xa = smem_u32(smem + DX_OFF_X + s * XT_BYTES);
      for (int c = 0; c < nch; ++c) {
        const int a = ai + c, cs = a % DX_NCS;
        if (!mbar_wait(&bars->c_full[cs], (a / DX_NCS) & 1, abort, p.err)) return false;
        if (a > 0 && !mbar_wait(&bars->zg_empty, (a - 1) & 1, abort, p.err)) return false;
        tc_fence_after();
        const uint32_t cb = smem_u32(smem + DX_OFF_CH + cs * CH_BYTES);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss(tmem + DX_TM_ZG, smem_desc(xa + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, SWZ_128B),
                 smem_desc(cb + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, SWZ_128B), id_zg,
                 ks > 0 ? 1u : 0u);
        mma_commit(&bars->zg_full);
        if (c == nch - 1) mma_commit(&bars->x_empty[s]);   // X is read by the logits MMAs only
      }
      ai += nch;
      return true;
    });
    mma_commit(&bars->mma_done[0]);
    mbar_wait_bounded(&bars->mma_done[0], 0);
  } else if (warp == 10 && lane == 0) {
    // ------------------------------------------------------------ aggregation MMA issuer
    // A thread of its own, so its waits overlap the logits thread's issue and
    // the other way round.  The two threads' MMAs share no TMEM columns.
    const uint32_t id_acc = idesc_bf16(128, 128, false, true);   // A from TMEM, B MN-major
    int ai = 0;
    for_each_tile(p.off, p.B, p.ch, g, [&](int, int, int, int64_t, int64_t, bool, bool) {
      for (int c = 0; c < nch; ++c) {
        const int a = ai + c, cs = a % DX_NCS, b = a & 1;
        // aa_full also implies that the epilogue of the previous tile has read V and
        // Q: every thread finishes that epilogue before it writes this tile's A
        if (!mbar_wait(&bars->c_full[cs], (a / DX_NCS) & 1, abort, p.err)) return false;
        if (!mbar_wait(&bars->aa_full[b], (a >> 1) & 1, abort, p.err)) return false;
        tc_fence_after();
        const uint32_t ta = tmem + DX_TM_AA + 64 * b;    // A in columns 0-31, ln2 A o dA in 32-63
        const uint32_t cb = smem_u32(smem + DX_OFF_CH + cs * CH_BYTES);
        // V += A P'_c;  Q += A dH_c (hi and lo parts) + (ln2 A o dA) P'_c
#pragma unroll
        for (int ks = 0; ks < KC / 16; ++ks) {
          const uint32_t acc = (c == 0 && ks == 0) ? 0u : 1u;
          const uint64_t bP = smem_desc(cb + ks * 2048, 16384, 1024, SWZ_128B);
          mma_ts(tmem + DX_TM_V, ta + ks * 8, bP, id_acc, acc);
          mma_ts(tmem + DX_TM_Q, ta + ks * 8, smem_desc(cb + 8192 + ks * 2048, 16384, 1024, SWZ_128B),
                 id_acc, acc);
          // the bf16 residual of dH, so dH enters Q to ~16 bits
          mma_ts(tmem + DX_TM_Q, ta + ks * 8, smem_desc(cb + 32768 + ks * 2048, 8192, 1024, SWZ_128B),
                 id_acc, 1u);
          mma_ts(tmem + DX_TM_Q, ta + 32 + ks * 8, bP, id_acc, 1u);
        }
        mma_commit(&bars->avq_done[cs]);
        if (c == nch - 1) mma_commit(&bars->acc_full);
      }
      ai += nch;
      return true;
    });
    mma_commit(&bars->mma_done[1]);
    mbar_wait_bounded(&bars->mma_done[1], 0);
  } else if (warp >= 2 && warp <= 9) {
    // ------------------------------------------------------------ two threads per token
    // Warpgroup h (warps 2-5: h = 0, 6-9: h = 1) owns prototypes 32h..32h+31 of every
    // chunk; its partial c_t is handed to warpgroup 0, which writes dX and c.
    const int q = warp % 4, h = (warp - 2) / 4;
    const int row = q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    float* cpart = (float*)(smem + DX_OFF_CP);
    int ai = 0;
    for_each_tile(p.off, p.B, p.ch, g, [&](int t, int, int, int64_t tb, int64_t pe, bool, bool) {
      const bool valid = tb + row < pe;
      // a padding row gets lse = +inf, so its A = 2^(z - inf) = 0 without a select
      const float l2 = valid ? p.lse2[tb + row] : __builtin_huge_valf();
      const float2 nl2 = make_float2(-l2, -l2), ln2v = make_float2(kLn2f, kLn2f);
      float2 c2 = make_float2(0.f, 0.f);   // partial c_t (even / odd prototypes)
      for (int c = 0; c < nch; ++c) {
        const int a = ai + c, cs = a % DX_NCS, b = a & 1;
        if (!mbar_wait(&bars->zg_full, a & 1, abort, p.err)) return false;
        tc_fence_after();
        float z[32], gv[32];
        tmem_ld32(tmem + lane_addr + DX_TM_ZG + 32 * h, z);
        tmem_ld32(tmem + lane_addr + DX_TM_ZG + 64 + 32 * h, gv);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->zg_empty);
        if (!mbar_wait(&bars->c_full[cs], (a / DX_NCS) & 1, abort, p.err)) return false;
        const float4* dm4 = (const float4*)(smem + DX_OFF_DM + cs * KC * 4) + 8 * h;
        uint32_t pa[16], pd[16];   // A and ln2 A o dA, bf16 pairs (even prototype low)
        // two prototypes per instruction (packed fp32x2 add / mul / fma)
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const float4 d0 = dm4[2 * q8], d1 = dm4[2 * q8 + 1];
          const float2 dmp[4] = {make_float2(d0.x, d0.y), make_float2(d0.z, d0.w),
                                 make_float2(d1.x, d1.y), make_float2(d1.z, d1.w)};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int j = q8 * 8 + 2 * i;
            const float2 e = __fadd2_rn(make_float2(z[j], z[j + 1]), nl2);
            const float2 A = make_float2(ex2(e.x), ex2(e.y));
            const float2 dA = __fadd2_rn(make_float2(gv[j], gv[j + 1]), dmp[i]);
            c2 = __ffma2_rn(A, dA, c2);
            const float2 ad = __fmul2_rn(__fmul2_rn(A, dA), ln2v);
            pa[4 * q8 + i] = pack_bf16x2(A.x, A.y);
            pd[4 * q8 + i] = pack_bf16x2(ad.x, ad.y);
          }
        }
        // TMEM A buffer b was last read by the aggregation MMAs of chunk a-2
        if (a >= 2 && !mbar_wait(&bars->avq_done[(a - 2) % DX_NCS], ((a - 2) / DX_NCS) & 1, abort, p.err))
          return false;
        tc_fence_after();
        tmem_st16(tmem + lane_addr + DX_TM_AA + 64 * b + 16 * h, pa);
        tmem_st16(tmem + lane_addr + DX_TM_AA + 64 * b + 32 + 16 * h, pd);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->aa_full[b]);
      }
      ai += nch;
      float cacc = c2.x + c2.y;
      if (h == 1) {
        // hand the partial c to warpgroup 0 (the slot is free once it has read the last one)
        if (t > 0 && !mbar_wait(&bars->cx_empty, (t - 1) & 1, abort, p.err)) return false;
        cpart[row] = cacc;
        mbar_arrive(&bars->cx_full);
        return true;
      }
      if (!mbar_wait(&bars->cx_full, t & 1, abort, p.err)) return false;
      cacc += cpart[row];
      mbar_arrive(&bars->cx_empty);
      // dX_t = Q - ln2 c_t V
      if (!mbar_wait(&bars->acc_full, t & 1, abort, p.err)) return false;
      tc_fence_after();
      const float lc = kLn2f * cacc;
#pragma unroll
      for (int qb = 0; qb < 4; ++qb) {
        float v[32], qv[32];
        tmem_ld32(tmem + lane_addr + DX_TM_V + 32 * qb, v);
        tmem_ld32(tmem + lane_addr + DX_TM_Q + 32 * qb, qv);
        tmem_wait_ld();
        if (valid && p.dX32) {
          float4* dst = (float4*)(p.dX32 + (tb + row) * DD + 32 * qb);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float4 o = make_float4(fmaf(-lc, v[4 * i], qv[4 * i]), fmaf(-lc, v[4 * i + 1], qv[4 * i + 1]),
                                   fmaf(-lc, v[4 * i + 2], qv[4 * i + 2]), fmaf(-lc, v[4 * i + 3], qv[4 * i + 3]));
            if (p.acc32) {
              const float4 a0 = dst[i];
              o.x += a0.x; o.y += a0.y; o.z += a0.z; o.w += a0.w;
            }
            dst[i] = o;
          }
        } else if (valid) {
          uint32_t o[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            o[i / 2] = pack_bf16x2(fmaf(-lc, v[i], qv[i]), fmaf(-lc, v[i + 1], qv[i + 1]));
          uint4* dst = (uint4*)(p.dX + (tb + row) * DD + 32 * qb);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        }
      }
      if (valid) p.cout[tb + row] = cacc;
      return true;
    });
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================== E kernel
// X tiles in flight (each is held from its load until the E MMA of its tile) and dZ buffers
#ifndef SA_E_NXS
#define SA_E_NXS 3
#endif
#ifndef SA_E_NDZ
#define SA_E_NDZ 2
#endif
constexpr int E_NXS = SA_E_NXS, E_NDZ = SA_E_NDZ;
constexpr uint32_t E_OFF_PH = 0;              // [P' h0 | dH h0 | P' h1 | dH h1], 16 KB each
constexpr uint32_t E_OFF_X = 65536;
constexpr uint32_t E_OFF_DZ = E_OFF_X + E_NXS * XT_BYTES;   // E_NDZ x [128 protos x 128 tokens] MN-major
constexpr uint32_t E_OFF_DM = E_OFF_DZ + E_NDZ * 32768;
constexpr uint32_t E_OFF_BAR = E_OFF_DM + TILE * 4;
constexpr uint32_t E_SMEM = E_OFF_BAR + 256 + 1024;
// warp 0 TMA, 1 MMA, then E_NWG warpgroups, group h computing dZ for the
// prototypes E_PW h .. E_PW h + E_PW-1 of the slice (so each reads its share of [Z|G]
// at once and the next tile's logits MMA overlaps all of the dZ work)
#ifndef SA_E_NWG
#define SA_E_NWG 2
#endif
constexpr int E_NWG = SA_E_NWG, E_PW = TILE / E_NWG;
static_assert(E_NWG == 2 || E_NWG == 4, "two or four dZ warpgroups");
constexpr int E_THREADS = 64 + 128 * E_NWG;
constexpr int E_BOUND = E_NWG == 2 ? 384 : E_THREADS;   // 384 with two: caps registers at 168
constexpr uint32_t E_TM_ZG = 0, E_TM_E = 256;

struct EBars {
  uint64_t p_full, h_full, h_empty, x_full[E_NXS], x_empty[E_NXS];
  uint64_t zg_full, zg_empty, dz_full[E_NDZ], dz_empty[E_NDZ], e_full, e_empty, mma_done;
  uint32_t tmem_base;
  int abort;
};

struct EParams {
  const int64_t* off;
  int B;
  Chunking ch;
  int k;
  const float* lse2;
  const float* cin;      // [n] c_t with the centred dm
  const float* dmc;      // [B, k]
  float* Epart;          // [G, k, d]
  int* err;
  // per-user prototypes: P' slice reloaded with each user's dH slice, and E written at
  // the end of every user's piece (to the user's rows, or a slot of the chunk when the
  // user spans chunks) instead of once per chunk
  int per_user;
  float* Euser;          // [B, k, d]
  float* slotE;          // [G, 2, k, d]
};

// PU: per-user prototypes and per-user E (EParams::per_user)
template <bool PU>
__global__ void __launch_bounds__(E_BOUND, 1)
    sa_bwd_e_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP,
                       const __grid_constant__ CUtensorMap tmH, EParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  EBars* bars = (EBars*)(smem + E_OFF_BAR);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int slices = p.k / TILE;
  const int sl = blockIdx.x % slices, g = blockIdx.x / slices;
  if (g >= p.ch.G) return;

  if (threadIdx.x == 0) {
    mbar_init(&bars->p_full, 1);
    mbar_init(&bars->h_full, 1);
    constexpr int NT = 128 * E_NWG;          // dZ threads
    mbar_init(&bars->h_empty, 1 + NT);       // the last zg of a piece, and the threads done with its dm
    for (int s = 0; s < E_NXS; ++s) { mbar_init(&bars->x_full[s], 1); mbar_init(&bars->x_empty[s], 1); }
    mbar_init(&bars->zg_full, 1);
    mbar_init(&bars->zg_empty, NT);
    for (int b = 0; b < E_NDZ; ++b) { mbar_init(&bars->dz_full[b], NT); mbar_init(&bars->dz_empty[b], 1); }
    mbar_init(&bars->e_full, 1);
    mbar_init(&bars->e_empty, NT);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmP);
    prefetch_tensormap(&tmH);
    if (!PU) {
      mbar_arrive_expect_tx(&bars->p_full, 32768);
      tma_load_2d(smem + E_OFF_PH, &tmP, &bars->p_full, 0, sl * TILE);
      tma_load_2d(smem + E_OFF_PH + 32768, &tmP, &bars->p_full, 64, sl * TILE);
    }
    int issued_t = 0, issued_h = 0;
    for_each_tile(p.off, p.B, p.ch, g, [&](int t, int piece, int u, int64_t tb, int64_t, bool first, bool) {
      if (first) {
        if (piece > 0 && !mbar_wait(&bars->h_empty, (piece - 1) & 1, abort, p.err)) return false;
        mbar_arrive_expect_tx(&bars->h_full, (PU ? 65536 : 32768) + TILE * 4);
        const int hrow = (int)((int64_t)u * p.k + sl * TILE);
        if (PU) {
          // this user's P' slice (the first two 16 KB blocks of the pair layout)
          tma_load_2d(smem + E_OFF_PH, &tmP, &bars->h_full, 0, hrow);
          tma_load_2d(smem + E_OFF_PH + 32768, &tmP, &bars->h_full, 64, hrow);
        }
        tma_load_2d(smem + E_OFF_PH + 16384, &tmH, &bars->h_full, 0, hrow);
        tma_load_2d(smem + E_OFF_PH + 49152, &tmH, &bars->h_full, 64, hrow);
        bulk_load(smem + E_OFF_DM, p.dmc + (int64_t)u * p.k + sl * TILE, TILE * 4, &bars->h_full);
        issued_h = piece + 1;
      }
      const int s = t % E_NXS;
      if (t >= E_NXS && !mbar_wait(&bars->x_empty[s], ((t / E_NXS) - 1) & 1, abort, p.err)) return false;
      mbar_arrive_expect_tx(&bars->x_full[s], XT_BYTES);
      uint8_t* xd = smem + E_OFF_X + s * XT_BYTES;
      tma_load_2d(xd, &tmX, &bars->x_full[s], 0, (int)tb);
      tma_load_2d(xd + XT_BYTES / 2, &tmX, &bars->x_full[s], 64, (int)tb);
      issued_t = t + 1;
      return true;
    });
    if (*abort) {
      if (!PU) mbar_wait_bounded(&bars->p_full, 0);
      if (issued_h > 0) mbar_wait_bounded(&bars->h_full, (issued_h - 1) & 1);
      for (int t = std::max(0, issued_t - E_NXS); t < issued_t; ++t)
        mbar_wait_bounded(&bars->x_full[t % E_NXS], (t / E_NXS) & 1);
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t id_zg = idesc_bf16(128, 256, false, false);
    const uint32_t id_e = idesc_bf16(128, 128, true, true);
    const uint32_t ph = smem_u32(smem + E_OFF_PH);
    int prev_t = -1, prev_s = 0, prev_piece = 0;
    bool prev_first = false, prev_last = false;
    auto emma = [&](int t, int s, int piece, bool first, bool last) -> bool {
      const int b = t % E_NDZ;
      // per user: E starts afresh at each piece, once the previous piece's E is drained
      if (PU && first && piece > 0 && !mbar_wait(&bars->e_empty, (piece - 1) & 1, abort, p.err))
        return false;
      if (!mbar_wait(&bars->dz_full[b], (t / E_NDZ) & 1, abort, p.err)) return false;
      tc_fence_after();
      const uint32_t dz = smem_u32(smem + E_OFF_DZ + b * 32768);
      const uint32_t xa = smem_u32(smem + E_OFF_X + s * XT_BYTES);
      const bool fresh = PU ? first : t == 0;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_ss(tmem + E_TM_E, smem_desc(dz + ks * 2048, 16384, 1024, SWZ_128B),
               smem_desc(xa + ks * 2048, 16384, 1024, SWZ_128B), id_e, (!fresh || ks > 0) ? 1u : 0u);
      mma_commit(&bars->dz_empty[b]);
      mma_commit(&bars->x_empty[s]);
      if (PU && last) mma_commit(&bars->e_full);
      return true;
    };
    bool ok = PU || mbar_wait(&bars->p_full, 0, abort, p.err);
    if (ok) {
      for_each_tile(p.off, p.B, p.ch, g, [&](int t, int piece, int, int64_t, int64_t, bool first, bool last) {
        const int s = t % E_NXS;
        if (first && !mbar_wait(&bars->h_full, piece & 1, abort, p.err)) return false;
        if (!mbar_wait(&bars->x_full[s], (t / E_NXS) & 1, abort, p.err)) return false;
        if (t > 0 && !mbar_wait(&bars->zg_empty, (t - 1) & 1, abort, p.err)) return false;
        tc_fence_after();
        const uint32_t xa = smem_u32(smem + E_OFF_X + s * XT_BYTES);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss(tmem + E_TM_ZG, smem_desc(xa + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, SWZ_128B),
                 smem_desc(ph + (ks >> 2) * 32768 + (ks & 3) * 32, 16, 1024, SWZ_128B), id_zg,
                 ks > 0 ? 1u : 0u);
        mma_commit(&bars->zg_full);
        if (last) mma_commit(&bars->h_empty);
        if (prev_t >= 0 && !emma(prev_t, prev_s, prev_piece, prev_first, prev_last)) return false;
        prev_t = t;
        prev_s = s;
        prev_piece = piece;
        prev_first = first;
        prev_last = last;
        return true;
      });
      if (prev_t >= 0 && !*abort && emma(prev_t, prev_s, prev_piece, prev_first, prev_last) && !PU)
        mma_commit(&bars->e_full);
    }
    mma_commit(&bars->mma_done);
    mbar_wait_bounded(&bars->mma_done, 0);
  } else if (warp >= 2) {
    const int q = warp % 4, h = (warp - 2) / 4;
    const int row = q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    bool ok = true;
    const int64_t n_total = p.off[p.B];
    float l2_next = 0.f, ct_next = 0.f;   // this row's lse and c for the next tile, loaded a tile ahead
    const int64_t cb = (int64_t)g * p.ch.T, ce = min(cb + p.ch.T, p.ch.n_total);
    // this thread's E_PW columns of the prototype's row of E, into dst
    auto write_e = [&](float* dst) {
      tc_fence_after();
#pragma unroll
      for (int c = E_PW / 32 * h; c < E_PW / 32 * (h + 1); ++c) {
        float v[32];
        tmem_ld32(tmem + lane_addr + E_TM_E + 32 * c, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *(float4*)(dst + 32 * c + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      }
    };
    for_each_tile(p.off, p.B, p.ch, g, [&](int t, int piece, int u, int64_t tb, int64_t pe, bool first, bool last) {
      const bool valid = tb + row < pe;
      float l2r = l2_next, ctr = ct_next;
      if (t == 0 && valid) { l2r = p.lse2[tb + row]; ctr = p.cin[tb + row]; }
      // the next tile starts 128 rows on, or at the end of this piece (rows of
      // other users are loaded harmlessly; each tile checks its own validity)
      const int64_t nb = tb + TILE < pe ? tb + TILE : pe;
      if (nb + row < n_total) { l2_next = p.lse2[nb + row]; ct_next = p.cin[nb + row]; }
      // a padding row gets lse = +inf, so its A = 2^(z - inf) = 0 without a select
      const float l2 = valid ? l2r : __builtin_huge_valf();
      const float ct = valid ? ctr : 0.f;
      const float2 nl2 = make_float2(-l2, -l2), nct = make_float2(-ct, -ct);
      if (first && !mbar_wait(&bars->h_full, piece & 1, abort, p.err)) return ok = false;
      if (!mbar_wait(&bars->zg_full, t & 1, abort, p.err)) return ok = false;
      tc_fence_after();
      const int b = t % E_NDZ;
      const uint32_t dz = smem_u32(smem + E_OFF_DZ + b * 32768) + row * 128;
      const float4* dm4 = (const float4*)(smem + E_OFF_DM);
      {
        float z[E_PW], gv[E_PW];
#pragma unroll
        for (int c = 0; c < E_PW / 32; ++c) {
          tmem_ld32(tmem + lane_addr + E_TM_ZG + E_PW * h + 32 * c, z + 32 * c);
          tmem_ld32(tmem + lane_addr + E_TM_ZG + 128 + E_PW * h + 32 * c, gv + 32 * c);
        }
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->zg_empty);
        if (t >= E_NDZ && !mbar_wait(&bars->dz_empty[b], ((t / E_NDZ) - 1) & 1, abort, p.err)) return ok = false;
        // two prototypes per instruction (packed fp32x2 add / mul)
#pragma unroll
        for (int c8 = 0; c8 < E_PW / 8; ++c8) {
          const int p0 = E_PW * h + 8 * c8;   // the first of these eight prototypes in the slice
          const float4 d0 = dm4[p0 / 4], d1 = dm4[p0 / 4 + 1];
          const float2 dmp[4] = {make_float2(d0.x, d0.y), make_float2(d0.z, d0.w),
                                 make_float2(d1.x, d1.y), make_float2(d1.z, d1.w)};
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int j = c8 * 8 + 2 * i;
            const float2 e = __fadd2_rn(make_float2(z[j], z[j + 1]), nl2);
            const float2 A = ((SA_E_POLY_PAIRS >> i) & 1) ? exp2_poly2(e) : make_float2(ex2(e.x), ex2(e.y));
            const float2 dA = __fadd2_rn(make_float2(gv[j], gv[j + 1]), dmp[i]);
            const float2 dzv = __fmul2_rn(A, __fadd2_rn(dA, nct));
            o[i] = pack_bf16x2(dzv.x, dzv.y);
          }
          // MN-major SW128 A operand of E += dZ^T X: M-block p0/64, token row `row`
          st_shared_v4(dz + (p0 / 64) * 16384 + ((((p0 % 64) / 8) ^ (row & 7)) << 4), o[0], o[1], o[2], o[3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars->dz_full[b]);
      if (last) mbar_arrive(&bars->h_empty);   // this piece's dm is no longer read
      if (PU && last) {
        // the user's E over this piece: to the user's rows, or to a slot of the chunk when
        // the user spans chunks (added up by e_user_reduce_kernel); then E may start afresh
        if (!mbar_wait(&bars->e_full, piece & 1, abort, p.err)) return ok = false;
        const int dest = piece_dest(p.off[u], p.off[u + 1], cb, ce);
        const int j = sl * TILE + row;
        write_e(dest == DEST_USER ? p.Euser + ((int64_t)u * p.k + j) * DD
                                  : p.slotE + (((int64_t)g * 2 + dest) * p.k + j) * DD);
        tc_fence_before();
        mbar_arrive(&bars->e_empty);
      }
      return true;
    });
    if (ok && !PU && mbar_wait(&bars->e_full, 0, abort, p.err))
      write_e(p.Epart + ((int64_t)g * p.k + sl * TILE + row) * DD);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================== host side

sa_status map_rows(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows) {
  return tma_map_bf16(map, base, DD, rows, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Per-user E of users that span E chunks: E_u = its first chunk's slot 1 + the middle
// chunks' slot 0 + its last chunk's slot 0, added in that order; users inside one chunk
// were written by the E kernel, users without tokens get zeros.
__global__ void e_user_reduce_kernel(const int64_t* __restrict__ off, Chunking ch, int k,
                                     const float* __restrict__ slotE, float* __restrict__ Euser) {
  const int u = blockIdx.y;
  const int64_t ub = off[u], ue = off[u + 1];
  const int64_t kd = (int64_t)k * DD;
  float* dst = Euser + (int64_t)u * kd;
  if (ue <= ub) {
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < kd; e += (int64_t)gridDim.x * blockDim.x)
      dst[e] = 0.f;
    return;
  }
  const int64_t gf = ub / ch.T, gl = (ue - 1) / ch.T;
  if (gf == gl) return;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < kd; e += (int64_t)gridDim.x * blockDim.x) {
    float v = slotE[((int64_t)gf * 2 + 1) * kd + e];
    for (int64_t g = gf + 1; g <= gl; ++g) v += slotE[((int64_t)g * 2 + 0) * kd + e];
    dst[e] = v;
  }
}

// dmc[u, j] = dm[u, j] - mean_j dm[u, :]
__global__ void center_rows_kernel(const float* __restrict__ dm, int k, float* __restrict__ dmc) {
  __shared__ float part[256];
  const int u = blockIdx.x;
  float s = 0.f;
  for (int j = threadIdx.x; j < k; j += 256) s += dm[(int64_t)u * k + j];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  const float mean = part[0] / (float)k;
  for (int j = threadIdx.x; j < k; j += 256) dmc[(int64_t)u * k + j] = dm[(int64_t)u * k + j] - mean;
}
}  // namespace

bool sa_bwd_tc_supported(sa_dtype x_dtype, int k, int d) {
  return x_dtype == SA_BF16 && d == DD && k % TILE == 0 && k >= TILE && k <= 4096;
}

int sa_bwd_tc_dx_chunks() { return device_info().sm_count; }
int sa_bwd_tc_e_chunks(int k) { return std::max(1, device_info().sm_count / (k / TILE)); }

sa_status sa_bwd_tc_run(const SaBwdArgs& a, const SaBwdWork& w, cudaStream_t st) {
  static unsigned long long done_dx = 0, done_e = 0, done_e_pu = 0;
  static std::mutex mu;
  set_smem_limit_once((const void*)sa_bwd_dx_tc_kernel, DX_SMEM, &done_dx, mu);
  set_smem_limit_once((const void*)sa_bwd_e_tc_kernel<false>, E_SMEM, &done_e, mu);
  set_smem_limit_once((const void*)sa_bwd_e_tc_kernel<true>, E_SMEM, &done_e_pu, mu);
  if (a.n_total >= (1LL << 31) || (int64_t)a.B * a.k >= (1LL << 31))
    return fail(SA_ERR_UNSUPPORTED, "row counts must be < 2^31");
  SA_TIMED("center_rows_kernel", st, (center_rows_kernel<<<a.B, 256, 0, st>>>(w.dm, a.k, w.dmc)));
  CUtensorMap tmX, tmP64, tmH64, tmP128, tmH128;
  sa_status s;
  // per-user prototypes: P' has B k rows, user u's at u k
  const uint64_t p_rows = a.per_user ? (uint64_t)a.B * a.k : (uint64_t)a.k;
  if (a.per_user && (!w.Euser || !w.slotE)) return fail(SA_ERR_INVALID_ARG, "per-user backward: no E outputs");
  if ((s = map_rows(&tmX, a.X, (uint64_t)a.n_total, 128)) != SA_OK) return s;
  if ((s = map_rows(&tmP64, w.Pb, p_rows, 64)) != SA_OK) return s;
  if ((s = map_rows(&tmH64, w.dHb, (uint64_t)a.B * a.k, 64)) != SA_OK) return s;
  CUtensorMap tmL64;
  if ((s = map_rows(&tmL64, w.dHlo, (uint64_t)a.B * a.k, 64)) != SA_OK) return s;
  if ((s = map_rows(&tmP128, w.Pb, p_rows, 128)) != SA_OK) return s;
  if ((s = map_rows(&tmH128, w.dHb, (uint64_t)a.B * a.k, 128)) != SA_OK) return s;
  DxParams dp{a.off_dev, a.B, w.ch, a.k, w.lse, w.dmc, (__nv_bfloat16*)a.dX, w.cbuf, device_status_word(),
              a.dX32, a.dX_acc ? 1 : 0, a.per_user ? a.k : 0};
  SA_TIMED("sa_bwd_dx_tc_kernel", st,
           (sa_bwd_dx_tc_kernel<<<w.ch.G, DX_THREADS, DX_SMEM, st>>>(tmX, tmP64, tmH64, tmL64, dp)));
  EParams ep{a.off_dev, a.B, w.chE, a.k, w.lse, w.cbuf, w.dmc, w.Epart, device_status_word(),
             a.per_user ? 1 : 0, w.Euser, w.slotE};
  if (a.per_user)
    SA_TIMED("sa_bwd_e_tc_kernel", st,
             (sa_bwd_e_tc_kernel<true><<<w.chE.G * (a.k / TILE), E_THREADS, E_SMEM, st>>>(tmX, tmP128, tmH128, ep)));
  else
    SA_TIMED("sa_bwd_e_tc_kernel", st,
             (sa_bwd_e_tc_kernel<false><<<w.chE.G * (a.k / TILE), E_THREADS, E_SMEM, st>>>(tmX, tmP128, tmH128, ep)));
  if (a.per_user)
    SA_TIMED("e_user_reduce_kernel", st,
             (e_user_reduce_kernel<<<dim3(64, a.B), 256, 0, st>>>(a.off_dev, w.chE, a.k, w.slotE, w.Euser)));
  return SA_OK;
}

}  // namespace sa
