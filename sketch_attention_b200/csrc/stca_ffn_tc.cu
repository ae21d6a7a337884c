// History-side SwiGLU FFN of the full STCA layer on the sm_100a tensor cores
// (SequenceO1 Sec. 5.1, eq. (27)): for every fp16 key row x (D = 128)
//   x <- x + (SiLU(x W1) * (x W3)) W2,   W1, W3 [128, 256], W2 [256, 128]
// in place, with the 256-wide inner activations never leaving the SM.
//
// Every operand is fp16 (11 significant bits), not bf16 (8): the weights, the
// inner activations and the stored rows are computed or converted values, and
// bf16 roundings of all three put the layer's output about 3.6e-3 (mean
// relative) from the exact one, fp16 roundings about 8 times less.  The rows of
// this path stay far inside the fp16 range; a stored row value above 65504 sets
// the range bit of the device status word.
//
// Persistent: one CTA per SM keeps W1|W3 resident in shared memory (fp16,
// 128 KB), streams W2 a quarter at a time from L2, and walks 128-row tiles
// with two X buffers.  A tile's inner width is
// done in four quarters of 64:
//   G_q  = X [W1_q | W3_q]     M=128 rows, N=128, K=128   (X from TMEM, fp32 in TMEM)
//   U_q  = SiLU(G1_q) * G3_q   registers -> fp16 pairs in TMEM
//   F   += U_q W2_q            M=128, N=128, K=64          (A from TMEM)
// and x + F goes back to the row as fp16.  G and U are double-buffered, so
// the tensor pipe computes G_{q+1} while the epilogue warps turn G_q into U_q.
// SiLU(g) g3 = (g/2) g3 (1 + tanh(g/2)): one MUFU operation per element.
//
// Shared memory bandwidth: an N=128 MMA with both operands in shared memory
// reads 128 bytes per clock, all that an SM's shared memory delivers, so the
// X tile is moved into TMEM once per tile and every MMA reads only its B
// operand from shared memory.
//
// The same kernel builds the events' input rows with the action-side SwiGLU
// fusion of Sec. 3.6 / App. D, eq. (20): x = e + FFN([e; a]) for e = item
// embedding, a = action embedding.  The action part of the first layer,
// a [W1_a | W3_a], takes one of n_actions values, so it is a per-action bias of
// G (precomputed, kept in shared memory in place of the X tiles); the rows are
// gathered from the item table by id instead of read by TMA, and the result
// goes to a separate bf16 output.
//
// Warp roles (16 warps): 0 TMA of W1|W3 and the X tiles, 1 first-layer MMA
// issue + TMEM owner, 2-9 two warpgroups of SiLU gating (warpgroup h takes the
// quarters of parity h), 10-13 X into TMEM and the residual add and
// write-back, 14 TMA of the W2 quarters, 15 second-layer MMA issue.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "stca_internal.cuh"
#include "tc_ptx.cuh"
#include "tma_map.cuh"

namespace sa {

namespace {
using namespace tc;

constexpr int DD = 128, TM = 128, THREADS = 512;
constexpr uint32_t W13_BYTES = 4 * 128 * DD * 2;   // [512 rows][128] fp16, two 64-column atoms
constexpr uint32_t W2Q_BYTES = DD * 64 * 2;        // one quarter of W2t: [128 rows][64] fp16
constexpr uint32_t X_BYTES = TM * DD * 2;          // one row tile, two atoms
// W1|W3 stay resident; X tiles and W2 quarters (re-read from L2) are double-buffered
constexpr uint32_t OFF_W13 = 0, OFF_X = OFF_W13 + W13_BYTES, OFF_W2 = OFF_X + 2 * X_BYTES;
constexpr uint32_t OFF_BAR = OFF_W2 + 2 * W2Q_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
// TMEM columns: G double buffer, U double buffer (bf16 pairs), the X tile as the
// first layer's A operand (fp16 pairs), F accumulator
constexpr uint32_t TM_G = 0, TM_U = 256, TM_X = 320, TM_F = 384, TM_COLS = 512;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

struct Bars {
  uint64_t w_full, x_full[2], x_empty[2], w2_full[2], w2_empty[2], xt_full, xt_empty, g_full[2],
      g_empty[2], u_full[2], u_empty[2], f_full, f_empty, mma_done[2];
  uint32_t tmem_base;
  int abort;
};

struct Params {
  __half* X;           // rows transformed in place (history FFN)
  int64_t rows;
  int ntiles;
  int* err;
  // event rows (eq. (20)): Xout[i] = bf16(item[ids[i]] + FFN([item[ids[i]]; action[acts[i]]]))
  const __nv_bfloat16* item;
  int64_t vocab;
  const int32_t* ids;
  const uint8_t* acts;
  int n_actions;
  const float* cb;     // [n_actions][512]: per quarter q, a W1_a[:, 64q..] then a W3_a[:, 64q..]
  __nv_bfloat16* Xout;
};
constexpr int kMaxActions = 16;
constexpr int CB_STRIDE = 516;   // floats per action in shared memory (4 banks apart per action)
static_assert(kMaxActions * CB_STRIDE * 4 <= 2 * X_BYTES, "bias table fits the X stages");

// SiLU(g1) g3 for a pair of elements: (g1/2) g3 (1 + tanh(g1/2)), one MUFU tanh per
// element (tanh.approx: relative error about 2^-11, the size of the fp16 rounding of U).
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t silu_mul_f16x2(float a0, float a1, float b0, float b1) {
  const float2 hx = __fmul2_rn(make_float2(a0, a1), make_float2(0.5f, 0.5f));
  const float2 th = make_float2(tanh_approx(hx.x), tanh_approx(hx.y));
  const float2 hg = __fmul2_rn(hx, make_float2(b0, b1));
  const float2 u = __ffma2_rn(hg, th, hg);
  return pack_f16x2(u.x, u.y);
}

// EV: event rows of eq. (20) (gathered inputs, per-action bias, bf16 output);
// else the history FFN of eq. (27), in place on fp16 rows
template <bool EV>
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
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->x_full[b], 1);
      mbar_init(&bars->x_empty[b], 128);
      mbar_init(&bars->w2_full[b], 1);
      mbar_init(&bars->w2_empty[b], 1);
      mbar_init(&bars->g_full[b], 1);
      mbar_init(&bars->g_empty[b], 128);
      mbar_init(&bars->u_full[b], 128);
      mbar_init(&bars->u_empty[b], 1);
    }
    mbar_init(&bars->xt_full, 128);
    mbar_init(&bars->xt_empty, 1);
    mbar_init(&bars->f_full, 1);
    mbar_init(&bars->f_empty, 128);
    mbar_init(&bars->mma_done[0], 1);
    mbar_init(&bars->mma_done[1], 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (EV) {
    // the per-action bias of G (the X stages are free: rows are gathered, not loaded)
    float* cbs = (float*)(smem + OFF_X);
    for (int e = threadIdx.x; e < p.n_actions * 512; e += THREADS)
      cbs[(e / 512) * CB_STRIDE + e % 512] = p.cb[e];
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
    // ---------------------------------------------------------------- TMA: W1|W3, X tiles
    if (!EV) prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmW13);
    mbar_arrive_expect_tx(&bars->w_full, W13_BYTES);
    for (int a = 0; a < 2; ++a)
      for (int r = 0; r < 2; ++r)
        tma_load_2d(smem + OFF_W13 + a * (W13_BYTES / 2) + r * (W13_BYTES / 4), &tmW13, &bars->w_full,
                    64 * a, 256 * r);
    int i = 0, issued = 0;
    for (int t = blockIdx.x; !EV && t < p.ntiles; t += gridDim.x, ++i) {
      const int s = i & 1;
      if (i >= 2 && !mbar_wait(&bars->x_empty[s], ((i >> 1) - 1) & 1, abort, p.err)) break;
      mbar_arrive_expect_tx(&bars->x_full[s], X_BYTES);
      tma_load_2d(smem + OFF_X + s * X_BYTES, &tmX, &bars->x_full[s], 0, t * TM);
      tma_load_2d(smem + OFF_X + s * X_BYTES + X_BYTES / 2, &tmX, &bars->x_full[s], 64, t * TM);
      issued = i + 1;
      // the tile after next: start its trip to L2
      const int tn = t + 2 * (int)gridDim.x;
      if (tn < p.ntiles) {
        tma_prefetch_l2_2d(&tmX, 0, tn * TM);
        tma_prefetch_l2_2d(&tmX, 64, tn * TM);
      }
    }
    if (*abort) {
      mbar_wait_bounded(&bars->w_full, 0);
      for (int j = std::max(0, issued - 2); j < issued; ++j)
        mbar_wait_bounded(&bars->x_full[j & 1], (j >> 1) & 1);
    }
  } else if (warp == 14 && lane == 0) {
    // ---------------------------------------------------------------- TMA: W2 quarters
    prefetch_tensormap(&tmW2);
    int i = 0, issued = 0;
    for (int t = blockIdx.x; t < p.ntiles; t += gridDim.x, ++i) {
      bool ok = true;
      for (int q = 0; q < 4; ++q) {
        const int b = q & 1, n = 2 * i + (q >> 1);
        if (n >= 1 && !mbar_wait(&bars->w2_empty[b], (n - 1) & 1, abort, p.err)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars->w2_full[b], W2Q_BYTES);
        tma_load_2d(smem + OFF_W2 + b * W2Q_BYTES, &tmW2, &bars->w2_full[b], 64 * q, 0);
        issued = n + 1;
      }
      if (!ok) break;
    }
    if (*abort)
      for (int n = std::max(0, issued - 2); n < issued; ++n)
        mbar_wait_bounded(&bars->w2_full[n & 1], (n >> 1) & 1);
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- first-layer MMAs
    // G_q = X [W1_q | W3_q]; the quarter's rows of W13t start at 128 q.  A thread of
    // its own, so a G buffer is refilled as soon as its gating warpgroup has read it,
    // whatever the second-layer MMAs are waiting for.
    const uint32_t id = idesc_f16(128, 128, false, false);
    const uint32_t w13 = smem_u32(smem + OFF_W13);
    bool ok = mbar_wait(&bars->w_full, 0, abort, p.err);
    int i = 0;
    for (int t = blockIdx.x; ok && t < p.ntiles; t += gridDim.x, ++i) {
      if (!mbar_wait(&bars->xt_full, i & 1, abort, p.err)) break;
      for (int q = 0; ok && q < 4; ++q) {
        const int b = q & 1, n = 2 * i + (q >> 1);
        if (n >= 1 && !mbar_wait(&bars->g_empty[b], (n - 1) & 1, abort, p.err)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts(tmem + TM_G + 128 * b, tmem + TM_X + 8 * ks,
                 smem_desc(w13 + (ks >> 2) * (W13_BYTES / 2) + q * 16384 + (ks & 3) * 32, 16, 1024, SWZ_128B),
                 id, ks > 0 ? 1u : 0u);
        mma_commit(&bars->g_full[b]);
      }
      if (ok) mma_commit(&bars->xt_empty);     // X in TMEM is read by these MMAs only
    }
    mma_commit(&bars->mma_done[0]);
    mbar_wait_bounded(&bars->mma_done[0], 0);
  } else if (warp == 15 && lane == 0) {
    // ---------------------------------------------------------------- second-layer MMAs
    // F += U_q W2_q; W2 slot q % 2 holds W2t's inner columns 64q..64q+63
    const uint32_t id = idesc_f16(128, 128, false, false);
    const uint32_t w2 = smem_u32(smem + OFF_W2);
    bool ok = true;
    int i = 0;
    for (int t = blockIdx.x; ok && t < p.ntiles; t += gridDim.x, ++i) {
      for (int q = 0; q < 4; ++q) {
        const int b = q & 1, n = 2 * i + (q >> 1);
        if (!mbar_wait(&bars->u_full[b], n & 1, abort, p.err) ||
            !mbar_wait(&bars->w2_full[b], n & 1, abort, p.err) ||
            (q == 0 && i >= 1 && !mbar_wait(&bars->f_empty, (i - 1) & 1, abort, p.err))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_ts(tmem + TM_F, tmem + TM_U + 32 * b + 8 * ks,
                 smem_desc(w2 + b * W2Q_BYTES + ks * 32, 16, 1024, SWZ_128B), id, (q > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bars->u_empty[b]);
        mma_commit(&bars->w2_empty[b]);
        if (q == 3) mma_commit(&bars->f_full);
      }
    }
    mma_commit(&bars->mma_done[1]);
    mbar_wait_bounded(&bars->mma_done[1], 0);
  } else if (warp >= 2 && warp < 10) {
    // ---------------------------------------------------------------- SiLU gate
    // Warpgroup h = 0, 1 takes the quarters q with q % 2 == h (G and U buffer
    // h), so two quarters are in flight: one warpgroup waits on TMEM while the
    // other computes.  Each thread owns one row; 32 inner columns per pass.
    const int q4 = warp % 4, h = (warp - 2) / 4;
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    int i = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < p.ntiles; t += gridDim.x, ++i) {
      // eq. (20): this row's action bias (a row past the end or with a bad type takes action 0;
      // its output is dropped or zeroed by the write-back warps)
      const float* cbr = nullptr;
      if (EV) {
        const int64_t grow = (int64_t)t * TM + q4 * 32 + lane;
        const int a = grow < p.rows ? (int)p.acts[grow] : 0;
        cbr = (const float*)(smem + OFF_X) + (a < p.n_actions ? a : 0) * CB_STRIDE;
      }
      for (int q = h; q < 4; q += 2) {
        const int n = 2 * i + (q >> 1);
        if (!mbar_wait(&bars->g_full[h], n & 1, abort, p.err)) { ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < 2; ++c) {
          float g1[32], g3[32];
          tmem_ld32(tmem + lane_addr + TM_G + 128 * h + 32 * c, g1);
          tmem_ld32(tmem + lane_addr + TM_G + 128 * h + 64 + 32 * c, g3);
          tmem_wait_ld();
          if (c == 1) {
            tc_fence_before();
            mbar_arrive(&bars->g_empty[h]);
          }
          if (EV) {
            const float4* b1 = (const float4*)(cbr + 128 * q + 32 * c);
            const float4* b3 = (const float4*)(cbr + 128 * q + 64 + 32 * c);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 x1 = b1[j], x3 = b3[j];
              g1[4 * j] += x1.x; g1[4 * j + 1] += x1.y; g1[4 * j + 2] += x1.z; g1[4 * j + 3] += x1.w;
              g3[4 * j] += x3.x; g3[4 * j + 1] += x3.y; g3[4 * j + 2] += x3.z; g3[4 * j + 3] += x3.w;
            }
          }
          uint32_t u[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) u[j] = silu_mul_f16x2(g1[2 * j], g1[2 * j + 1], g3[2 * j], g3[2 * j + 1]);
          // U buffer h was last read by the second-layer MMAs of use n-1
          if (c == 0 && n >= 1 && !mbar_wait(&bars->u_empty[h], (n - 1) & 1, abort, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          tmem_st16(tmem + lane_addr + TM_U + 32 * h + 16 * c, u);
        }
        if (!ok) break;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->u_full[h]);
      }
    }
  } else if (warp >= 10 && warp < 14) {
    // ---------------------------------------------------------------- X to TMEM, x + F
    // Each thread owns one row.  It moves the row of the next tile from shared
    // memory (swizzled) into TMEM as the first layer's A operand, so the MMAs
    // read only W1|W3 from shared memory, then writes x + F of this tile.
    const int q4 = warp % 4;
    const int row = q4 * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    // tile j's row: 16 pieces of 16 bytes (8 bf16), piece 8a + c at atom a, chunk c ^ (row % 8)
    float vmax = 0.f;                   // largest |x + F| (or, for events, |e|) seen by this thread
    // EV: each row's table index runs ahead of the tiles: the raw id and type of tile
    // i + 2 are loaded while tile i is finished, validated (-1: past the end, an id
    // outside the table or a bad type) and the item row prefetched to L2 one tile later,
    // then gathered into TMEM when tile i + 1 is staged; the write-back gathers it again
    // (from L2) to add F.
    auto ev_raw = [&](int j, int32_t& id, int& act) {
      const int64_t grow = (int64_t)(blockIdx.x + (int64_t)j * gridDim.x) * TM + row;
      id = -1;
      act = 0;
      if (grow < p.rows) {
        id = p.ids[grow];
        act = p.acts[grow];
      }
    };
    auto ev_valid = [&](int32_t id, int act) -> int64_t {
      return (id >= 0 && (int64_t)id < p.vocab && act < p.n_actions) ? (int64_t)id : -1;
    };
    auto ev_prefetch = [&](int64_t id) {
      if (id >= 0) {
        const char* a = (const char*)(p.item + id * DD);
        asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
        asm volatile("prefetch.global.L2 [%0];" ::"l"(a + 128));
      }
    };
    auto stage_x = [&](int j, int64_t id) -> bool {
      const int s = j & 1;
      uint32_t v[64];
      if (EV) {
        if (j >= 1 && !mbar_wait(&bars->xt_empty, (j - 1) & 1, abort, p.err)) return false;
        uint4 e[16];
        const uint4* src = (const uint4*)(p.item + (id >= 0 ? id : 0) * DD);
#pragma unroll
        for (int c = 0; c < 16; ++c) e[c] = id >= 0 ? src[c] : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint32_t w[4] = {e[c].x, e[c].y, e[c].z, e[c].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            // bf16 -> fp32 exactly (the bf16 bits are the high half), then to fp16
            const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xFFFF0000u);
            vmax = fmaxf(vmax, fmaxf(fabsf(lo), fabsf(hi)));
            v[4 * c + k] = pack_f16x2(lo, hi);
          }
        }
      } else {
        if (!mbar_wait(&bars->x_full[s], (j >> 1) & 1, abort, p.err)) return false;
        if (j >= 1 && !mbar_wait(&bars->xt_empty, (j - 1) & 1, abort, p.err)) return false;
        const uint32_t base = smem_u32(smem + OFF_X + s * X_BYTES) + row * 128;
#pragma unroll
        for (int pc = 0; pc < 16; ++pc) {
          const uint32_t addr = base + (pc >> 3) * (X_BYTES / 2) + (((pc & 7) ^ (row & 7)) << 4);
          asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                       : "=r"(v[4 * pc]), "=r"(v[4 * pc + 1]), "=r"(v[4 * pc + 2]), "=r"(v[4 * pc + 3])
                       : "r"(addr));
        }
        mbar_arrive(&bars->x_empty[s]);
      }
      tc_fence_after();
      tmem_st32(tmem + lane_addr + TM_X, v);
      tmem_st32(tmem + lane_addr + TM_X + 32, v + 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->xt_full);
      return true;
    };
    int i = 0;
    int64_t id0 = -1, id1 = -1;            // tiles i and i + 1 (validated)
    int32_t raw2 = -1;                     // tile i + 2 (loaded, not yet validated)
    int act2 = 0;
    if (EV) {
      int32_t r;
      int a;
      ev_raw(0, r, a);
      id0 = ev_valid(r, a);
      ev_raw(1, r, a);
      id1 = ev_valid(r, a);
      ev_prefetch(id1);
      ev_raw(2, raw2, act2);
    }
    bool ok = blockIdx.x < p.ntiles && stage_x(0, id0);
    for (int t = blockIdx.x; ok && t < p.ntiles; t += gridDim.x, ++i) {
      int64_t id2 = -1;
      if (EV) {
        id2 = ev_valid(raw2, act2);
        ev_prefetch(id2);
        ev_raw(i + 3, raw2, act2);
      }
      // the next tile's X goes in as soon as this tile's first-layer MMAs are done
      if (t + (int)gridDim.x < p.ntiles && !stage_x(i + 1, id1)) break;
      const int64_t grow = (int64_t)t * TM + row;
      const bool valid = grow < p.rows;
      uint32_t xr[64];                  // the row as fp16 pairs (events: the bf16 item row)
      const bool ev_ok = !EV || id0 >= 0;
      if (EV) {
        if (valid && !ev_ok && p.err) atomicOr(p.err, DEV_ERR_INDEX);
        // the item row again (in L2: it was staged a tile ago)
        const uint4* px = (const uint4*)(p.item + (ev_ok ? id0 : 0) * DD);
#pragma unroll
        for (int v = 0; v < 16; ++v) {
          const uint4 x = (valid && ev_ok) ? px[v] : make_uint4(0, 0, 0, 0);
          xr[4 * v] = x.x; xr[4 * v + 1] = x.y; xr[4 * v + 2] = x.z; xr[4 * v + 3] = x.w;
        }
        id0 = id1;
        id1 = id2;
      } else {
        const uint4* px = (const uint4*)(p.X + (valid ? grow : 0) * DD);
#pragma unroll
        for (int v = 0; v < 16; ++v) {
          const uint4 x = valid ? px[v] : make_uint4(0, 0, 0, 0);
          xr[4 * v] = x.x; xr[4 * v + 1] = x.y; xr[4 * v + 2] = x.z; xr[4 * v + 3] = x.w;
        }
      }
      if (!mbar_wait(&bars->f_full, i & 1, abort, p.err)) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float f[16];
        tmem_ld16(tmem + lane_addr + TM_F + 16 * c, f);
        tmem_wait_ld16(f);
        if (c == 7) {
          tc_fence_before();
          mbar_arrive(&bars->f_empty);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (EV) {
            // x = e + F, rounded once to bf16; a bad id or type gives a zero row
            const uint32_t w = xr[8 * c + e];
            const float y0 = __uint_as_float(w << 16) + f[2 * e];
            const float y1 = __uint_as_float(w & 0xFFFF0000u) + f[2 * e + 1];
            xr[8 * c + e] = ev_ok ? pack_bf16x2(y0, y1) : 0u;
          } else {
            __half2 hx;
            memcpy(&hx, &xr[8 * c + e], 4);
            const float2 x = __half22float2(hx);
            const float y0 = x.x + f[2 * e], y1 = x.y + f[2 * e + 1];
            vmax = fmaxf(vmax, fmaxf(fabsf(y0), fabsf(y1)));
            xr[8 * c + e] = pack_f16x2(y0, y1);
          }
        }
      }
      if (valid) {
        uint4* po = EV ? (uint4*)(p.Xout + grow * DD) : (uint4*)(p.X + grow * DD);
#pragma unroll
        for (int v = 0; v < 16; ++v)
          po[v] = make_uint4(xr[4 * v], xr[4 * v + 1], xr[4 * v + 2], xr[4 * v + 3]);
      }
    }
    // NaN fails the comparison too
    if (!(vmax <= 65504.f) && p.err) atomicOr(p.err, DEV_ERR_RANGE);
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
__global__ void ffn_weights_f16_kernel(const float* __restrict__ W1, const float* __restrict__ W3,
                                       const float* __restrict__ W2, __half* __restrict__ W13t,
                                       __half* __restrict__ W2t, int* __restrict__ err) {
  float v = 0.f;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < 4 * 128 * DD) {
    const int r = e / DD, k = e % DD;
    const int q = r / 128, rr = r % 128;
    const float* src = rr < 64 ? W1 : W3;
    v = src[k * 2 * DD + 64 * q + (rr & 63)];
    W13t[e] = __float2half_rn(v);
  } else if (e < 4 * 128 * DD + DD * 2 * DD) {
    const int f = e - 4 * 128 * DD;
    const int n = f / (2 * DD), j = f % (2 * DD);
    v = W2[j * DD + n];
    W2t[f] = __float2half_rn(v);
  }
  if (!(fabsf(v) <= 65504.f) && err) atomicOr(err, DEV_ERR_RANGE);
}


// fp16 matrix [outer][inner], boxes of 64 x box_outer, 128-byte swizzle
sa_status make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  return tma_map_2byte(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, base, inner, outer, 64, box_outer,
                       CU_TENSOR_MAP_SWIZZLE_128B);
}
}  // namespace

sa_status stca_ffn_weights_f16(const float* W1, const float* W3, const float* W2, __half* W13t, __half* W2t,
                               cudaStream_t st) {
  constexpr int n = 4 * 128 * DD + DD * 2 * DD;
  SA_TIMED("ffn_weights_f16_kernel", st,
           (ffn_weights_f16_kernel<<<(n + 255) / 256, 256, 0, st>>>(W1, W3, W2, W13t, W2t,
                                                                     device_status_word())));
  return SA_OK;
}

namespace {
std::mutex g_mu;
unsigned long long g_done[2] = {0, 0};

sa_status ffn_launch(bool ev, const Params& p0, const void* x_map_base, const __half* W13t, const __half* W2t,
                     cudaStream_t st) {
  if (ev) set_smem_limit_once((const void*)stca_hist_ffn_tc_kernel<true>, SMEM_BYTES, &g_done[1], g_mu);
  else set_smem_limit_once((const void*)stca_hist_ffn_tc_kernel<false>, SMEM_BYTES, &g_done[0], g_mu);
  CUtensorMap tmX, tmW13, tmW2;
  sa_status s;
  if ((s = make_map(&tmW13, W13t, DD, 4 * 128, 256)) != SA_OK) return s;
  if ((s = make_map(&tmW2, W2t, 2 * DD, DD, 128)) != SA_OK) return s;
  if (ev) tmX = tmW13;                  // not read: event rows are gathered by id
  else if ((s = make_map(&tmX, x_map_base, DD, (uint64_t)p0.rows, TM)) != SA_OK) return s;
  Params p = p0;
  p.ntiles = (int)((p.rows + TM - 1) / TM);
  p.err = device_status_word();
  const int grid = std::min(p.ntiles, device_info().sm_count);
  if (ev)
    SA_TIMED("events_ffn_tc_kernel", st,
             (stca_hist_ffn_tc_kernel<true><<<grid, THREADS, SMEM_BYTES, st>>>(tmX, tmW13, tmW2, p)));
  else
    SA_TIMED("stca_hist_ffn_tc_kernel", st,
             (stca_hist_ffn_tc_kernel<false><<<grid, THREADS, SMEM_BYTES, st>>>(tmX, tmW13, tmW2, p)));
  return SA_OK;
}

// cb[a][128 q + c] = (action[a] W1[D:, :])[64 q + c] for c < 64, (action[a] W3[D:, :])[64 q + c - 64] else
__global__ void __launch_bounds__(512) action_bias_kernel(const __nv_bfloat16* __restrict__ action,
                                                          const float* __restrict__ W1,
                                                          const float* __restrict__ W3, float* __restrict__ cb) {
  const int a = blockIdx.x, e = threadIdx.x;
  const int q = e / 128, c = e % 128;
  const float* W = (c < 64 ? W1 : W3) + (int64_t)DD * 2 * DD + 64 * q + (c & 63);
  float acc = 0.f;
  for (int k = 0; k < DD; ++k) acc = fmaf(__bfloat162float(action[(int64_t)a * DD + k]), W[(int64_t)k * 2 * DD], acc);
  cb[a * 512 + e] = acc;
}
}  // namespace

sa_status stca_hist_ffn_tc(__half* X, int64_t rows, const __half* W13t, const __half* W2t, cudaStream_t st) {
  if (rows <= 0) return SA_OK;
  if (rows >= (1LL << 31) - TM) return fail(SA_ERR_UNSUPPORTED, "history rows must be < 2^31 - 128");
  Params p{};
  p.X = X;
  p.rows = rows;
  return ffn_launch(false, p, X, W13t, W2t, st);
}

size_t events_ffn_layout(void* base, int n_actions, EventsFfnWork* w) {
  Carve c(base);
  EventsFfnWork v;
  v.W13t = c.take<__half>((size_t)4 * DD * DD);
  v.W2t = c.take<__half>((size_t)2 * DD * DD);
  v.cb = c.take<float>((size_t)std::max(n_actions, 1) * 512);
  if (w) *w = v;
  return c.bytes();
}

sa_status events_ffn_run(const __nv_bfloat16* item, int64_t vocab, const __nv_bfloat16* action, int n_actions,
                         const int32_t* ids, const uint8_t* acts, int64_t n, const float* W1, const float* W3,
                         const float* W2, __nv_bfloat16* X, const EventsFfnWork& w, cudaStream_t st) {
  if (n <= 0) return SA_OK;
  if (n >= (1LL << 31) - TM) return fail(SA_ERR_UNSUPPORTED, "events must be < 2^31 - 128");
  if (n_actions < 1 || n_actions > kMaxActions)
    return fail(SA_ERR_UNSUPPORTED, "the fused event rows take 1..16 action types");
  sa_status s;
  if ((s = stca_ffn_weights_f16(W1, W3, W2, w.W13t, w.W2t, st)) != SA_OK) return s;
  SA_TIMED("action_bias_kernel", st, (action_bias_kernel<<<n_actions, 512, 0, st>>>(action, W1, W3, w.cb)));
  Params p{};
  p.rows = n;
  p.item = item;
  p.vocab = vocab;
  p.ids = ids;
  p.acts = acts;
  p.n_actions = n_actions;
  p.cb = w.cb;
  p.Xout = X;
  return ffn_launch(true, p, nullptr, w.W13t, w.W2t, st);
}

}  // namespace sa
