// Tensor-core Sketch Attention forward for sm_100a (SequenceO1 Sec. 3.1,
// eqs. (6)-(9); the fused streaming operator of Sec. 4.4, re-designed for
// tcgen05, TMEM and TMA).
//
// Work split.  The token stream is cut into G chunks, one per cluster of
// C = k/128 CTAs.  CTA r of a cluster owns prototypes [128 r, 128 r + 128):
// its slice of P' (bf16, SMEM-resident) and its accumulator
// H_slice = [A_slice X | A_slice 1] (128 x 144 fp32 in TMEM; the last 16
// columns hold the mass).  Every CTA of the cluster streams the same 128-token
// tiles of X through SMEM with TMA (no multicast: each CTA issues its own
// loads, the copies after the first come from L2).  An X tile stays in SMEM
// from its load until its aggregation MMA, so the number of stages bounds the
// tiles in flight; the shared-memory budget goes to four stages.
//
// Per tile (t = 128 tokens of one user):
//   MMA1   Z^T[t, j] = X_t . P'_j              (M=128 tokens, N=128 prototypes, K=d)
//   softmax over all k prototypes of each token: each CTA reduces its 128
//          logits in registers (one TMEM lane = one token = one thread) to a
//          log2-sum-exp, sends it to every CTA of the cluster (DSMEM bulk
//          copies), and rescales its exponentials by 2^{m - lse_total}
//   MMA2   H_slice[j, :] += sum_t p[t, j] [x_t | 1]   (M=128 prototypes, N=144, K=128 tokens)
// so the k x n assignment matrix never leaves the SM.
//
// Warp roles (11 warps): 0 TMA, 1 logits MMAs + TMEM owner, 2 aggregation
// MMAs, 3-6 softmax of even tiles (and the H drain at the end of a piece),
// 7-10 softmax of odd tiles.  A warp reads TMEM lanes 32 (warp % 4) .. +31, so
// each group of four consecutive warps covers all 128 lanes.
#include <algorithm>
#include <mutex>

#include "sa_internal.cuh"
#include "tc_ptx.cuh"

namespace sa {

namespace {
using namespace tc;

constexpr int TILE = 128;            // tokens per tile = prototypes per CTA
constexpr int DD = 128;              // d
constexpr int NS = 4;                // X pipeline stages (tiles in flight)
constexpr int MAXC = 8;              // cluster size limit (k <= 1024)
constexpr int N2 = DD + 16;          // MMA2 N: d columns + 16 mass columns
constexpr int THREADS = 352;

// shared-memory layout (offsets from a 1024-aligned base)
constexpr uint32_t X_BOX = TILE * 32;                  // one [128 x 16] bf16 SW32 box = 4 KB
constexpr uint32_t X_STAGE = 9 * X_BOX;                // 8 boxes of X + 1 box of ones = 36 KB
constexpr uint32_t OFF_PQ = 0;                         // P' slice: 2 x [128 x 64] SW128 = 32 KB
constexpr uint32_t OFF_X = 32768;
constexpr uint32_t OFF_P = OFF_X + NS * X_STAGE;       // one 32 KB probability tile
constexpr uint32_t OFF_XCHG = OFF_P + 32768;           // [4 slots][MAXC][128] fp32
constexpr uint32_t OFF_BAR = OFF_XCHG + 4 * MAXC * TILE * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;  // + barriers + alignment slack

// TMEM columns
constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_H = 256, TM_COLS = 512;

struct Bars {
  uint64_t x_full[NS], x_empty[NS];
  uint64_t s_full[2], s_empty[2], p_full, p_empty;
  uint64_t h_full, h_empty, pq_full, mma_done;
  uint64_t xchg[4];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

struct Params {
  const int64_t* off;
  int B;
  Chunking ch;
  int k;
  float* Huser;
  float* Muser;
  float* slotH;
  float* slotM;
  float* lse;          // optional per-token ln-sum-exp output
  int* err;
};

// Iterates the tiles of chunk g: calls f(tile_index, user, tile_begin,
// piece_begin, piece_end, first_tile_of_piece, last_tile_of_piece) in order;
// stops early if f returns false.
template <class F>
__device__ __forceinline__ void for_each_tile(const Params& p, int g, F&& f) {
  const int64_t cb = (int64_t)g * p.ch.T, ce = min(cb + p.ch.T, p.ch.n_total);
  int t = 0;
  for (int u = user_of_token(p.off, p.B, cb); u < p.B && p.off[u] < ce; ++u) {
    const int64_t pb = max(p.off[u], cb), pe = min(p.off[u + 1], ce);
    for (int64_t tb = pb; tb < pe; tb += TILE, ++t)
      if (!f(t, u, tb, pb, pe, tb == pb, tb + TILE >= pe)) return;
  }
}

__global__ void __launch_bounds__(THREADS, 1)
    sa_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                     const __grid_constant__ CUtensorMap tmP, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Bars* bars = (Bars*)(smem + OFF_BAR);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank(), C = cluster_size();
  const int g = (int)cluster_id_x();
  const bool chunk_ok = g < p.ch.G;

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) { mbar_init(&bars->x_full[s], 1); mbar_init(&bars->x_empty[s], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_empty[b], 128);
    }
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->p_empty, 1);
    mbar_init(&bars->h_full, 1);
    mbar_init(&bars->h_empty, 128);
    mbar_init(&bars->pq_full, 1);
    mbar_init(&bars->mma_done, 2);        // both MMA-issuing threads
    for (int s = 0; s < 4; ++s) mbar_init(&bars->xchg[s], 1);
    bars->abort = 0;
    fence_mbar_init();
    // arm the exchange slots for their first use (tiles 0..3)
    for (int s = 0; s < 4; ++s) mbar_arrive_expect_tx(&bars->xchg[s], (C - 1) * TILE * 4);
  }
  // constant ones block of every stage (MMA2 columns d..d+15 -> prototype mass)
  for (int i = threadIdx.x; i < NS * (int)X_BOX / 4; i += THREADS) {
    const int s = i / (X_BOX / 4), w = i % (X_BOX / 4);
    ((uint32_t*)(smem + OFF_X + s * X_STAGE + 8 * X_BOX))[w] = 0x3F803F80u;   // bf16 1.0 pairs
  }
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();          // peers' barriers are initialised before any exchange
  const uint32_t tmem = bars->tmem_base;

  if (chunk_ok) {
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      prefetch_tensormap(&tmX);
      prefetch_tensormap(&tmP);
      mbar_arrive_expect_tx(&bars->pq_full, 2 * 16384);
      tma_load_2d(smem + OFF_PQ, &tmP, &bars->pq_full, 0, (int)(rank * TILE));
      tma_load_2d(smem + OFF_PQ + 16384, &tmP, &bars->pq_full, 64, (int)(rank * TILE));
      int issued = 0;
      for_each_tile(p, g, [&](int t, int, int64_t tb, int64_t, int64_t, bool, bool) {
        const int s = t % NS;
        if (t >= NS && !mbar_wait(&bars->x_empty[s], ((t / NS) - 1) & 1, abort, p.err)) return false;
        mbar_arrive_expect_tx(&bars->x_full[s], 8 * X_BOX);
        uint8_t* dst = smem + OFF_X + s * X_STAGE;
        for (int b = 0; b < 8; ++b) tma_load_2d(dst + b * X_BOX, &tmX, &bars->x_full[s], 16 * b, (int)tb);
        issued = t + 1;
        return true;
      });
      if (*abort) {
        // let the loads still in flight land before the CTA can exit
        mbar_wait_bounded(&bars->pq_full, 0);
        for (int t = std::max(0, issued - NS); t < issued; ++t)
          mbar_wait_bounded(&bars->x_full[t % NS], (t / NS) & 1);
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------ logits MMAs
      // MMA1 of a tile is issued as soon as its X tile has landed and the
      // logits buffer it reuses has been read by the softmax warps.
      const uint32_t id1 = idesc_bf16(128, 128, false, false);
      const uint32_t pq = smem_u32(smem + OFF_PQ);
      if (mbar_wait(&bars->pq_full, 0, abort, p.err)) {
        for_each_tile(p, g, [&](int t, int, int64_t, int64_t, int64_t, bool, bool) {
          const int s = t % NS, b = t & 1;
          if (!mbar_wait(&bars->x_full[s], (t / NS) & 1, abort, p.err)) return false;
          if (t >= 2 && !mbar_wait(&bars->s_empty[b], ((t >> 1) - 1) & 1, abort, p.err)) return false;
          tc_fence_after();
          const uint32_t xa = smem_u32(smem + OFF_X + s * X_STAGE);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t da = smem_desc(xa + ks * X_BOX, 16, 256, SWZ_32B);
            const uint64_t db = smem_desc(pq + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, SWZ_128B);
            mma_ss(tmem + (b ? TM_S1 : TM_S0), da, db, id1, ks > 0 ? 1u : 0u);
          }
          mma_commit(&bars->s_full[b]);
          return true;
        });
      }
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(&bars->mma_done);
      mbar_wait_bounded(&bars->mma_done, 0);
    } else if (warp == 2 && lane == 0) {
      // ------------------------------------------------------------ aggregation MMAs
      // A second issuing thread, so MMA2 of a tile starts the moment its
      // probabilities are written, independent of the logits of later tiles
      // (the two streams touch disjoint TMEM and SMEM).
      const uint32_t id2 = idesc_bf16(128, N2, true, true);
      int piece = -1;
      for_each_tile(p, g, [&](int t, int, int64_t, int64_t, int64_t, bool first, bool last) {
        const int s = t % NS;
        if (first) ++piece;
        if (first && piece > 0 && !mbar_wait(&bars->h_empty, (piece - 1) & 1, abort, p.err)) return false;
        if (!mbar_wait(&bars->p_full, t & 1, abort, p.err)) return false;
        tc_fence_after();
        const uint32_t pa = smem_u32(smem + OFF_P);
        const uint32_t xa = smem_u32(smem + OFF_X + s * X_STAGE);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t da = smem_desc(pa + ks * 2048, 16384, 1024, SWZ_128B);
          const uint64_t db = smem_desc(xa + ks * 512, X_BOX, 256, SWZ_32B);
          mma_ss(tmem + TM_H, da, db, id2, (first && ks == 0) ? 0u : 1u);
        }
        mma_commit(&bars->p_empty);
        mma_commit(&bars->x_empty[s]);
        if (last) mma_commit(&bars->h_full);
        return true;
      });
      mma_commit(&bars->mma_done);
      mbar_wait_bounded(&bars->mma_done, 0);
    } else if (warp >= 3) {
      // ------------------------------------------------------------ softmax groups
      const int wg = (warp - 3) / 4;            // 0: even tiles, 1: odd tiles
      const int q = warp % 4;                   // TMEM lane quarter
      const int row = q * 32 + lane;            // token within the tile / prototype lane
      const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
      const float* xchg = (const float*)(smem + OFF_XCHG);
      int piece = -1;
      for_each_tile(p, g, [&](int t, int u, int64_t tb, int64_t pb, int64_t pe, bool first, bool last) {
        if (first) ++piece;
        if ((t & 1) == wg) {
          const int b = t & 1;
          const bool valid = tb + row < pe;
          // logits of this token over the CTA's 128 prototypes (base-2 units)
          if (!mbar_wait(&bars->s_full[b], (t >> 1) & 1, abort, p.err)) return false;
          tc_fence_after();
          // Eight chunks of 16 logits, each exponentiated against the running
          // maximum at that point (mc[c]) and scaled by 2^8, kept as fp16 pairs
          // (11-bit mantissa, normal range down to 2^-22 of the chunk maximum).
          // The load of chunk c+1 is in flight while chunk c is processed; the
          // logits buffer is released as soon as the last chunk has landed.
          const uint32_t sbuf = tmem + lane_addr + (b ? TM_S1 : TM_S0);
          uint32_t ep[64];
          float mc[8];
          float m = -__builtin_huge_valf();
          float2 s2 = make_float2(0.f, 0.f);   // running sum, as two partial sums
          float zbuf[2][16];
          tmem_ld16(sbuf, zbuf[0]);
          tmem_wait_ld16(zbuf[0]);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float* z = zbuf[c & 1];
            if (c < 7) tmem_ld16(sbuf + 16 * (c + 1), zbuf[(c + 1) & 1]);
            float cm = z[0];
#pragma unroll
            for (int j = 1; j < 16; ++j) cm = fmaxf(cm, z[j]);
            const float mn = fmaxf(m, cm);
            const float sc = ex2(m - mn);
            s2 = __fmul2_rn(s2, make_float2(sc, sc));
            m = mn;
            mc[c] = mn;
            const float2 off = make_float2(8.f - mn, 8.f - mn);
            // two logits per instruction (packed fp32x2 add)
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const float2 zz = __fadd2_rn(make_float2(z[j], z[j + 1]), off);
              const float2 e = make_float2(ex2(zz.x), ex2(zz.y));
              s2 = __fadd2_rn(s2, e);
              ep[8 * c + j / 2] = pack_f16x2(e.x, e.y);
            }
            if (c < 7) tmem_wait_ld16(zbuf[(c + 1) & 1]);
            if (c == 6) {
              tc_fence_before();
              mbar_arrive(&bars->s_empty[b]);
            }
          }
          const float l = valid ? m + lg2(s2.x + s2.y) - 8.f : -__builtin_huge_valf();
          // this CTA's log2-sum-exp of every token goes into its own row of the
          // exchange slot, and from there to the same row in every other CTA
          const int slot = t & 3;
          float* own = (float*)(smem + OFF_XCHG) + (slot * MAXC + rank) * TILE;
          own[row] = l;
          fence_proxy_async_smem();
          named_bar_sync(1 + wg, 128);
          if (row == 0) {
            const uint32_t src = smem_u32(own);
            const uint32_t bar = smem_u32(&bars->xchg[slot]);
            for (uint32_t c = 0; c < C; ++c)
              if (c != rank) bulk_copy_to_peer(map_to_rank(src, c), src, TILE * 4, map_to_rank(bar, c));
          }
          if (!mbar_wait(&bars->xchg[slot], (t >> 2) & 1, abort, p.err)) return false;
          float rc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          if (valid) {
            float L = -__builtin_huge_valf();
            for (uint32_t c = 0; c < C; ++c) L = fmaxf(L, xchg[(slot * MAXC + c) * TILE + row]);
            float z = 0.f;
            for (uint32_t c = 0; c < C; ++c) z += ex2(xchg[(slot * MAXC + c) * TILE + row] - L);
            const float lt = L + lg2(z);
            if (p.lse && rank == 0) p.lse[tb + row] = lt * 0.69314718055994530942f;
#pragma unroll
            for (int c = 0; c < 8; ++c) rc[c] = ex2(mc[c] - 8.f - lt);
          }
          named_bar_sync(1 + wg, 128);      // every thread has read the slot
          if (row == 0) mbar_arrive_expect_tx(&bars->xchg[slot], (C - 1) * TILE * 4);   // re-arm for t+4
          // probabilities p[t, j] = e_j r as bf16 into the MN-major SW128 A tile of MMA2
          if (t >= 1 && !mbar_wait(&bars->p_empty, (t - 1) & 1, abort, p.err)) return false;
          const uint32_t pa = smem_u32(smem + OFF_P) + row * 128;
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) {           // 16-byte chunks of 8 prototypes
            const float2 r = make_float2(rc[cc >> 1], rc[cc >> 1]);
            const uint32_t* e4 = ep + 4 * cc;
            const float2 a0 = __fmul2_rn(unpack_f16x2(e4[0]), r), a1 = __fmul2_rn(unpack_f16x2(e4[1]), r);
            const float2 a2 = __fmul2_rn(unpack_f16x2(e4[2]), r), a3 = __fmul2_rn(unpack_f16x2(e4[3]), r);
            st_shared_v4(pa + (cc >> 3) * 16384 + (((cc & 7) ^ (row & 7)) << 4),
                         pack_bf16x2(a0.x, a0.y), pack_bf16x2(a1.x, a1.y),
                         pack_bf16x2(a2.x, a2.y), pack_bf16x2(a3.x, a3.y));
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&bars->p_full);
        }
        if (last && wg == 0) {
          // ------------------------------------------------------ drain H of the piece
          if (!mbar_wait(&bars->h_full, piece & 1, abort, p.err)) return false;
          tc_fence_after();
          const int64_t ub = p.off[u], ue = p.off[u + 1];
          const int64_t cb = (int64_t)g * p.ch.T, ce = min(cb + p.ch.T, p.ch.n_total);
          const int dest = piece_dest(ub, ue, cb, ce);
          const int j = (int)rank * TILE + row;
          float* Hrow;
          float* mrow;
          if (dest == DEST_USER) {
            Hrow = p.Huser + ((int64_t)u * p.k + j) * DD;
            mrow = p.Muser + (int64_t)u * p.k + j;
          } else {
            Hrow = p.slotH + (((int64_t)g * 2 + dest) * p.k + j) * DD;
            mrow = p.slotM + ((int64_t)g * 2 + dest) * p.k + j;
          }
          float hv[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            tmem_ld32(tmem + lane_addr + TM_H + 32 * c, hv);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *(float4*)(Hrow + 32 * c + i) = make_float4(hv[i], hv[i + 1], hv[i + 2], hv[i + 3]);
          }
          const float mass = tmem_ld1(tmem + lane_addr + TM_H + DD);
          tmem_wait_ld();
          *mrow = mass;
          tc_fence_before();
          mbar_arrive(&bars->h_empty);
        }
        return true;
      });
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
  cluster_sync();          // no peer copies may target this CTA after it exits
}

struct Cached {
  bool init = false;
  int clusters[MAXC + 1] = {};
};
std::mutex g_mu;
Cached g_cache[64];

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeFn)p;
  });
  return fn;
}

sa_status make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                   uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeFn enc = encode_fn();
  if (!enc) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return SA_OK;
}

int clusters_for(int C) {
  const DeviceInfo& di = device_info();
  std::lock_guard<std::mutex> lock(g_mu);
  Cached& c = g_cache[di.device & 63];
  if (!c.init) {
    cudaFuncSetAttribute(sa_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    cudaFuncSetAttribute(sa_fwd_tc_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    for (int cs = 1; cs <= MAXC; ++cs) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = cs;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(cs * (di.sm_count / cs), 1, 1);
      cfg.blockDim = dim3(THREADS, 1, 1);
      cfg.dynamicSmemBytes = SMEM_BYTES;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, sa_fwd_tc_kernel, &cfg) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = std::max(1, di.sm_count / cs);
      }
      c.clusters[cs] = n;
    }
    c.init = true;
  }
  return c.clusters[C];
}
}  // namespace

bool sa_tc_supported(sa_dtype x_dtype, int k, int d) {
  return x_dtype == SA_BF16 && d == DD && k % TILE == 0 && k / TILE >= 1 && k / TILE <= MAXC;
}

int sa_tc_num_chunks(int k) { return clusters_for(k / TILE); }

sa_status sa_tc_forward(const SaFwdArgs& a, const SaFwdWork& w, cudaStream_t st) {
  const int C = a.k / TILE;
  if (a.n_total >= (1LL << 31)) return fail(SA_ERR_UNSUPPORTED, "n_total must be < 2^31");
  CUtensorMap tmX, tmP;
  sa_status s = make_map(&tmX, a.X, DD, (uint64_t)a.n_total, 16, TILE, CU_TENSOR_MAP_SWIZZLE_32B);
  if (s != SA_OK) return s;
  s = make_map(&tmP, w.Pb, DD, (uint64_t)a.k, 64, TILE, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != SA_OK) return s;
  Params p{a.off_dev, a.B, w.ch, a.k, a.S, w.Muser, w.slotH, w.slotM, a.lse_out,
           device_status_word()};
  clusters_for(C);   // sets the kernel attributes once per device
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = C;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(C * w.ch.G, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cudaError_t le = cudaSuccess;
  SA_TIMED("sa_fwd_tc_kernel", st, (le = cudaLaunchKernelEx(&cfg, sa_fwd_tc_kernel, tmX, tmP, p)));
  if (le != cudaSuccess) return cuda_fail(le, "sa_fwd_tc_kernel launch");
  return SA_OK;
}

}  // namespace sa
