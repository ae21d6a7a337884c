// Tensor-core STCA attention for sm_100a (SequenceO1 Sec. 2.3 eq. (4) in the
// single-query reordering of Sec. 5.1 eq. (24)).
//
// One CTA per tile of 128 query rows of one user; a row is a (candidate,
// head) pair whose query vector u_h = (q W_Q^h) W_K^h^T * log2(e)/sqrt(d_h) was
// produced by the projection GEMM (bf16, D = 128 wide).  Keys and values are
// the same raw history rows x_i, so one SMEM tile per block of 128 keys
// serves both contractions:
//   S = U X_blk^T    (M=128 rows, N=128 keys, K=128; X tile K-major)
//   O += P X_blk     (M=128 rows, N=128, K=128 keys; P from TMEM, X tile MN-major)
// The softmax over keys is online: each thread owns one query row (one TMEM
// lane); the running maximum is only raised when a block's maximum exceeds it
// by more than 8 (base-2 units), so O in TMEM is rarely rescaled.
//
// Warp roles (8 warps): 0 TMA, 1 MMA issue + TMEM owner, 2-3 idle,
// 4-7 softmax and the final normalisation.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "exp2_poly.cuh"
#include "stca_internal.cuh"
#include "tc_ptx.cuh"
#include "tma_map.cuh"

namespace sa {

namespace {
using namespace tc;

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

#ifndef STCA_NSK
#define STCA_NSK 3                   // key/value tile stages
#endif
#ifndef STCA_POLY_MASK
#define STCA_POLY_MASK 0x22          // key pairs (of each eight) whose exponential runs on the FMA pipe
#endif
constexpr int TQ = 128, TKB = 128, DD = 128, NSK = STCA_NSK, THREADS = 256;
constexpr uint32_t TILE_BYTES = TQ * DD * 2;                       // 32 KB
constexpr uint32_t OFF_Q = 0, OFF_KV = TILE_BYTES, OFF_BAR = OFF_KV + NSK * TILE_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_P0 = 256, TM_P1 = 320, TM_O = 384, TM_COLS = 512;
constexpr float kRescale = 8.f;      // raise the running max only past this margin

struct Bars {
  uint64_t q_full, kv_full[NSK], kv_empty[NSK], s_full[2], p_full[2], pv_done[2], o_done;
  uint32_t tmem_base;
  int abort;
};

struct Params {
  const int* prefix;
  const int64_t* cand;
  const int64_t* kvb;
  const int64_t* kve;
  int B, heads;
  float* Y;              // fp32 output, or (Y NULL) hi + lo bf16 splits of it
  __nv_bfloat16* Yhi;
  __nv_bfloat16* Ylo;
  int* err;
};

// F16: the query and key operands are fp16 (and so are the probabilities), else bf16
template <bool F16>
__global__ void __launch_bounds__(THREADS, 1)
    stca_attn_tc_kernel(const __grid_constant__ CUtensorMap tmU,
                        const __grid_constant__ CUtensorMap tmK, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Bars* bars = (Bars*)(smem + OFF_BAR);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tile = blockIdx.x;
  if (tile >= p.prefix[p.B]) return;
  int lo = 0, hi = p.B - 1;                 // user: largest u with prefix[u] <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  const int u = lo;
  const int64_t rend = p.cand[u + 1] * p.heads;
  const int64_t r0 = p.cand[u] * p.heads + (int64_t)(tile - p.prefix[u]) * TQ;
  const int64_t kb = p.kvb[u], ke = p.kve[u];
  const int nblk = (int)((ke - kb + TKB - 1) / TKB);
  if (nblk == 0) {
    // no keys: the attention output is zero
    for (int e = threadIdx.x; e < TQ * DD; e += THREADS) {
      const int64_t row = r0 + e / DD;
      if (row < rend) {
        if (p.Y) {
          p.Y[row * DD + e % DD] = 0.f;
        } else {
          p.Yhi[row * DD + e % DD] = __float2bfloat16_rn(0.f);
          p.Ylo[row * DD + e % DD] = __float2bfloat16_rn(0.f);
        }
      }
    }
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < NSK; ++s) { mbar_init(&bars->kv_full[s], 1); mbar_init(&bars->kv_empty[s], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->p_full[b], 128);
      mbar_init(&bars->pv_done[b], 1);
    }
    mbar_init(&bars->o_done, 1);
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
    prefetch_tensormap(&tmU);
    prefetch_tensormap(&tmK);
    mbar_arrive_expect_tx(&bars->q_full, TILE_BYTES);
    tma_load_2d(smem + OFF_Q, &tmU, &bars->q_full, 0, (int)r0);
    tma_load_2d(smem + OFF_Q + TILE_BYTES / 2, &tmU, &bars->q_full, 64, (int)r0);
    int issued = 0;
    for (int j = 0; j < nblk; ++j) {
      const int s = j % NSK;
      if (j >= NSK && !mbar_wait(&bars->kv_empty[s], ((j / NSK) - 1) & 1, abort, p.err)) break;
      mbar_arrive_expect_tx(&bars->kv_full[s], TILE_BYTES);
      uint8_t* dst = smem + OFF_KV + s * TILE_BYTES;
      const int row = (int)(kb + (int64_t)j * TKB);
      tma_load_2d(dst, &tmK, &bars->kv_full[s], 0, row);
      tma_load_2d(dst + TILE_BYTES / 2, &tmK, &bars->kv_full[s], 64, row);
      issued = j + 1;
    }
    if (*abort) {
      mbar_wait_bounded(&bars->q_full, 0);
      for (int j = std::max(0, issued - NSK); j < issued; ++j)
        mbar_wait_bounded(&bars->kv_full[j % NSK], (j / NSK) & 1);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    const uint32_t idS = F16 ? idesc_f16(128, 128, false, false) : idesc_bf16(128, 128, false, false);
    const uint32_t idO = F16 ? idesc_f16(128, 128, false, true) : idesc_bf16(128, 128, false, true);
    const uint32_t qa = smem_u32(smem + OFF_Q);
    auto pv = [&](int j) -> bool {
      const int b = j & 1, s = j % NSK;
      if (!mbar_wait(&bars->p_full[b], (j >> 1) & 1, abort, p.err)) return false;
      tc_fence_after();
      const uint32_t va = smem_u32(smem + OFF_KV + s * TILE_BYTES);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_ts(tmem + TM_O, tmem + (b ? TM_P1 : TM_P0) + ks * 8,
               smem_desc(va + ks * 2048, 16384, 1024, SWZ_128B), idO, (j > 0 || ks > 0) ? 1u : 0u);
      mma_commit(&bars->kv_empty[s]);
      mma_commit(&bars->pv_done[b]);
      return true;
    };
    bool ok = mbar_wait(&bars->q_full, 0, abort, p.err);
    for (int j = 0; ok && j < nblk; ++j) {
      const int s = j % NSK, b = j & 1;
      if (!mbar_wait(&bars->kv_full[s], (j / NSK) & 1, abort, p.err)) { ok = false; break; }
      tc_fence_after();
      const uint32_t ka = smem_u32(smem + OFF_KV + s * TILE_BYTES);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_ss(tmem + (b ? TM_S1 : TM_S0),
               smem_desc(qa + (ks >> 2) * (TILE_BYTES / 2) + (ks & 3) * 32, 16, 1024, SWZ_128B),
               smem_desc(ka + (ks >> 2) * (TILE_BYTES / 2) + (ks & 3) * 32, 16, 1024, SWZ_128B),
               idS, ks > 0 ? 1u : 0u);
      mma_commit(&bars->s_full[b]);
      if (j > 0 && !pv(j - 1)) { ok = false; break; }
    }
    if (ok) pv(nblk - 1);
    mma_commit(&bars->o_done);
    mbar_wait_bounded(&bars->o_done, 0);
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax
    const int q = warp % 4;
    const int row = q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    float m = -__builtin_huge_valf(), l = 0.f;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      const int b = j & 1;
      if (!mbar_wait(&bars->s_full[b], (j >> 1) & 1, abort, p.err)) { ok = false; break; }
      tc_fence_after();
      float sv[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_addr + (b ? TM_S1 : TM_S0) + 32 * c, sv + 32 * c);
      tmem_wait_ld();
      const int64_t kbase = kb + (int64_t)j * TKB;
      if (kbase + TKB > ke) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (kbase + i >= ke) sv[i] = -__builtin_huge_valf();
      }
      // block maximum: eight independent chains of three-input maxima
      float bm;
      {
        float c[8];
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) {
          const float* w = sv + 16 * q8;
          float m3 = max3f(w[0], w[1], w[2]);
#pragma unroll
          for (int j = 3; j + 1 < 16; j += 2) m3 = max3f(m3, w[j], w[j + 1]);
          c[q8] = fmaxf(m3, w[15]);
        }
        bm = fmaxf(max3f(c[0], c[1], c[2]), max3f(c[3], c[4], max3f(c[5], c[6], c[7])));
      }
      const bool raise = bm > m + kRescale;
      if (__any_sync(0xffffffffu, raise)) {
        const float mn = fmaxf(m, bm);
        const float corr = ex2(m - mn);        // 0 on the first block, 1 if this row keeps m
        m = mn;
        l *= corr;
        if (j > 0) {
          // O holds blocks < j: wait for the last of them, then rescale in place
          if (!mbar_wait(&bars->pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort, p.err)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(tmem + lane_addr + TM_O + 32 * c, o);
            tmem_wait_ld();
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(o[i] * corr);
            tmem_st32(tmem + lane_addr + TM_O + 32 * c, w);
          }
          tmem_wait_st();
        }
      }
      // P buffer b was last read by PV(j-2)
      if (j >= 2 && !mbar_wait(&bars->pv_done[b], ((j >> 1) - 1) & 1, abort, p.err)) { ok = false; break; }
      uint32_t pw[64];
      float2 lsa[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      const float2 nm = make_float2(-m, -m);
#pragma unroll
      for (int i = 0; i < 128; i += 2) {
        // the pairs STCA_POLY_MASK selects on the FMA pipe (fitted cubic), the rest on the MUFU
        const float2 e = __fadd2_rn(make_float2(sv[i], sv[i + 1]), nm);
        float2 v;
        if ((STCA_POLY_MASK >> ((i / 2) % 8)) & 1) {
          v = exp2_poly2(e);                 // clamps at 2^-125: a masked key (-inf) must give 0
          v.x = e.x < -125.f ? 0.f : v.x;
          v.y = e.y < -125.f ? 0.f : v.y;
        } else {
          v = make_float2(ex2(e.x), ex2(e.y));
        }
        lsa[(i / 2) & 3] = __fadd2_rn(lsa[(i / 2) & 3], v);   // four independent sums
        pw[i / 2] = F16 ? pack_f16x2(v.x, v.y) : pack_bf16x2(v.x, v.y);
      }
      const float2 ls2 = __fadd2_rn(__fadd2_rn(lsa[0], lsa[1]), __fadd2_rn(lsa[2], lsa[3]));
      const float ls = ls2.x + ls2.y;
      l += ls;
      tmem_st32(tmem + lane_addr + (b ? TM_P1 : TM_P0), pw);
      tmem_st32(tmem + lane_addr + (b ? TM_P1 : TM_P0) + 32, pw + 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[b]);
    }
    if (ok && mbar_wait(&bars->o_done, 0, abort, p.err)) {
      tc_fence_after();
      const int64_t grow = r0 + row;
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32(tmem + lane_addr + TM_O + 32 * c, o);
        tmem_wait_ld();
        if (grow < rend && p.Y) {
          float* dst = p.Y + grow * DD + 32 * c;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *(float4*)(dst + i) = make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
        } else if (grow < rend) {
          // the output projection's operand: y = hi + lo, hi = bf16(y), lo = bf16(y - hi)
          uint32_t hi[16], lo[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float y0 = o[i] * inv, y1 = o[i + 1] * inv;
            hi[i / 2] = pack_bf16x2(y0, y1);
            lo[i / 2] = pack_bf16x2(y0 - __uint_as_float(hi[i / 2] << 16), y1 - __uint_as_float(hi[i / 2] & 0xFFFF0000u));
          }
          uint4* dh = (uint4*)(p.Yhi + grow * DD + 32 * c);
          uint4* dl = (uint4*)(p.Ylo + grow * DD + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            dh[i] = make_uint4(hi[4 * i], hi[4 * i + 1], hi[4 * i + 2], hi[4 * i + 3]);
            dl[i] = make_uint4(lo[4 * i], lo[4 * i + 1], lo[4 * i + 2], lo[4 * i + 3]);
          }
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


// ============================================================== host side
sa_status make_map(CUtensorMap* map, const void* base, uint64_t rows, bool f16) {
  return tma_map_2byte(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, DD,
                       rows, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
}
}  // namespace

bool stca_tc_supported(sa_dtype dtype, int D) { return dtype == SA_BF16 && D == DD; }

sa_status stca_tc_attention(const StcaArgs& a, const StcaWork& w, cudaStream_t st, bool split_y) {
  static unsigned long long done = 0, done16 = 0;
  static std::mutex mu;
  set_smem_limit_once((const void*)stca_attn_tc_kernel<false>, SMEM_BYTES, &done, mu);
  set_smem_limit_once((const void*)stca_attn_tc_kernel<true>, SMEM_BYTES, &done16, mu);
  if (a.kv_rows >= (1LL << 31) || a.C_total * a.heads >= (1LL << 31))
    return fail(SA_ERR_UNSUPPORTED, "row counts must be < 2^31");
  CUtensorMap tmU, tmK;
  sa_status s = make_map(&tmU, w.Ub, (uint64_t)(a.C_total * a.heads), a.kv_f16);
  if (s != SA_OK) return s;
  if (a.kv_rows > 0) {
    s = make_map(&tmK, a.kv, (uint64_t)a.kv_rows, a.kv_f16);
    if (s != SA_OK) return s;
  } else {
    memset(&tmK, 0, sizeof(tmK));     // never read: every key range is empty
  }
  Params p{w.tile_prefix, a.cand_dev, a.kvb_dev, a.kve_dev, a.B, a.heads, split_y ? nullptr : w.Y,
           split_y ? w.Yhi : nullptr, split_y ? w.Ylo : nullptr, device_status_word()};
  if (a.kv_f16)
    SA_TIMED("stca_attn_tc_kernel", st,
             (stca_attn_tc_kernel<true><<<w.max_tiles, THREADS, SMEM_BYTES, st>>>(tmU, tmK, p)));
  else
    SA_TIMED("stca_attn_tc_kernel", st,
             (stca_attn_tc_kernel<false><<<w.max_tiles, THREADS, SMEM_BYTES, st>>>(tmU, tmK, p)));
  return SA_OK;
}

}  // namespace sa
