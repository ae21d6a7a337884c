// Full STCA layers (SequenceO1 Sec. 5.1, eqs. (26)-(28)): the single-query
// attention layer of stca.cu plus two SwiGLU FFNs of inner width 2D,
//   history side, before the attention:  x <- x + (SiLU(x W1) * (x W3)) W2
//   query side, after the W_O residual:  q <- q + (SiLU(q W1) * (q W3)) W2
// The history transform does not depend on the target, so it runs once per
// key row (the amortisation the pages' eq. (33) counts for grouped requests)
// on a private copy of each user's key range, which then serves as the
// layer's keys and values.  bf16 keys: the copy is fp16 (the rows it holds after
// a transform are computed values, kept to 11 significant bits rather than
// bf16's 8), transformed by the fused tensor-core FFN of stca_ffn_tc.cu, and
// every layer's attention reads it with fp16 operands; fp32 keys and the (small)
// query side: the projection GEMM.
#include <algorithm>
#include <cstring>

#include "sa_internal.cuh"
#include "stca_internal.cuh"

namespace sa {

namespace {
// kpre[u] = sum_{v<u} (kve[v] - kvb[v])
__global__ void range_prefix_kernel(const int64_t* __restrict__ kvb, const int64_t* __restrict__ kve,
                                    int B, int64_t* __restrict__ kpre) {
  if (blockIdx.x != 0 || threadIdx.x != 0) return;
  int64_t acc = 0;
  kpre[0] = 0;
  for (int u = 0; u < B; ++u) {
    acc += kve[u] - kvb[u];
    kpre[u + 1] = acc;
  }
}

// Hk[kpre[u] + j] = kv[kvb[u] + j]: 16-byte pieces, a thread per piece.
__global__ void gather_ranges_kernel(const uint4* __restrict__ kv, const int64_t* __restrict__ kvb,
                                     const int64_t* __restrict__ kpre, int B, int pieces_per_row,
                                     int64_t total_pieces, uint4* __restrict__ Hk) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total_pieces;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / pieces_per_row;
    const int c = (int)(e % pieces_per_row);
    int lo = 0, hi = B - 1;                // user: largest u with kpre[u] <= r
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (kpre[mid] <= r) lo = mid; else hi = mid - 1;
    }
    Hk[e] = kv[(kvb[lo] + (r - kpre[lo])) * pieces_per_row + c];
  }
}

// Hk[kpre[u] + j] = fp16(kv[kvb[u] + j]) for bf16 rows: 8 elements (16 bytes) per thread;
// a value above the fp16 range sets the range bit of the device status word.
__global__ void gather_ranges_f16_kernel(const uint4* __restrict__ kv, const int64_t* __restrict__ kvb,
                                         const int64_t* __restrict__ kpre, int B, int pieces_per_row,
                                         int64_t total_pieces, uint4* __restrict__ Hk, int* __restrict__ err) {
  float vmax = 0.f;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total_pieces;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / pieces_per_row;
    const int c = (int)(e % pieces_per_row);
    int lo = 0, hi = B - 1;                // user: largest u with kpre[u] <= r
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (kpre[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const uint4 x = kv[(kvb[lo] + (r - kpre[lo])) * pieces_per_row + c];
    const uint32_t in[4] = {x.x, x.y, x.z, x.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32
      const float a = __uint_as_float(in[i] << 16), b = __uint_as_float(in[i] & 0xFFFF0000u);
      vmax = fmaxf(vmax, fmaxf(fabsf(a), fabsf(b)));
      const __half2 h = __floats2half2_rn(a, b);
      memcpy(&out[i], &h, 4);
    }
    Hk[e] = make_uint4(out[0], out[1], out[2], out[3]);
  }
  if (!(vmax <= 65504.f) && err) atomicOr(err, DEV_ERR_RANGE);
}

unsigned grid_for(int64_t n) { return (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 1 << 16)); }

bool has_hist(const stca_full_layer& L) { return L.hist_W1 != nullptr; }
bool has_query(const stca_full_layer& L) { return L.q_W1 != nullptr; }

// X <- X + (SiLU(X W1) * (X W3)) W2 over `rows` fp32 rows of width D (GEMMs).
sa_status ffn_residual_gemm(float* X, int64_t rows, int D, const float* W1, const float* W3,
                            const float* W2, float* G1, float* G3, float* U, const char* tag,
                            cudaStream_t st) {
  if (rows == 0) return SA_OK;
  if (rows >= (1LL << 31)) return fail(SA_ERR_UNSUPPORTED, "FFN rows must be < 2^31");
  Gemm g1;
  g1.M = (int)rows; g1.N = 2 * D; g1.K = D;
  g1.A = X; g1.lda = D; g1.B = W1; g1.ldb = 2 * D; g1.C = G1; g1.ldc = 2 * D; g1.tag = tag;
  sa_status s;
  if ((s = gemm(g1, st)) != SA_OK) return s;
  Gemm g3 = g1;
  g3.B = W3; g3.C = G3;
  if ((s = gemm(g3, st)) != SA_OK) return s;
  if ((s = sa_swiglu(G1, G3, rows * 2 * D, U, st)) != SA_OK) return s;
  Gemm g2;
  g2.M = (int)rows; g2.N = D; g2.K = 2 * D;
  g2.A = U; g2.lda = 2 * D; g2.B = W2; g2.ldb = D;
  g2.C = X; g2.ldc = D; g2.Cin = X; g2.ldcin = D; g2.tag = tag;
  return gemm(g2, st);
}
}  // namespace

size_t stca_full_layout(void* base, int B, int64_t C, int64_t kv_total, int D, int heads, int d_h,
                        sa_dtype dtype, StcaFullWork* w) {
  Carve c(base);
  StcaFullWork v;
  // the attention part: the same carve as the plain branch
  const size_t rows = (size_t)std::max<int64_t>(C, 1);
  v.attn = stca_attn_carve(c, B, C, D, heads, d_h);
  const size_t kt = (size_t)std::max<int64_t>(kv_total, 1);
  v.Hk = c.take<uint8_t>(kt * D * (dtype == SA_BF16 ? 2 : 4));
  v.kpre = c.take<int64_t>((size_t)B + 1);
  const size_t grows = std::max<size_t>(rows, dtype == SA_F32 ? kt : 1);
  v.G1 = c.take<float>(grows * 2 * D);
  v.G3 = c.take<float>(grows * 2 * D);
  v.U = c.take<float>(grows * 2 * D);
  v.W13t = c.take<__half>((size_t)4 * D * D);
  v.W2t = c.take<__half>((size_t)2 * D * D);
  if (w) *w = v;
  return c.bytes();
}

sa_status stca_full_run(const StcaArgs& a0, const stca_full_layer* layers, int64_t kv_total,
                        const StcaFullWork& w, cudaStream_t st) {
  StcaArgs a = a0;
  sa_status s;
  if ((s = stca_begin(a, w.attn, st)) != SA_OK) return s;
  bool any_hist = false;
  for (int l = 0; l < a.n_layers; ++l) any_hist |= has_hist(layers[l]);
  const int esz = a.dtype == SA_BF16 ? 2 : 4;
  if (any_hist) {
    // a private copy of every user's key range: Hk rows [kpre[u], kpre[u+1])
    SA_TIMED("range_prefix_kernel", st,
             (range_prefix_kernel<<<1, 1, 0, st>>>(a.kvb_dev, a.kve_dev, a.B, w.kpre)));
    const int ppr = a.D * esz / 16;
    const int64_t pieces = kv_total * ppr;
    if (pieces > 0) {
      if (a.dtype == SA_BF16)
        SA_TIMED("gather_ranges_f16_kernel", st,
                 (gather_ranges_f16_kernel<<<grid_for(pieces), 256, 0, st>>>(
                     (const uint4*)a.kv, a.kvb_dev, w.kpre, a.B, ppr, pieces, (uint4*)w.Hk,
                     device_status_word())));
      else
        SA_TIMED("gather_ranges_kernel", st,
                 (gather_ranges_kernel<<<grid_for(pieces), 256, 0, st>>>(
                     (const uint4*)a.kv, a.kvb_dev, w.kpre, a.B, ppr, pieces, (uint4*)w.Hk)));
    }
    if (a.dtype == SA_BF16) {
      // every layer attends over the fp16 copy (a layer without a history FFN reads the
      // rows it was given, converted exactly within the fp16 range)
      a.kv = w.Hk;
      a.kv_rows = kv_total;
      a.kvb_dev = w.kpre;
      a.kve_dev = w.kpre + 1;
      a.kv_f16 = true;
    }
  }
  bool split_ready = true;
  for (int l = 0; l < a.n_layers; ++l) {
    const stca_full_layer& L = layers[l];
    if (has_hist(L)) {
      // eq. (27): the layer's keys and values become x + FFN_h(x)
      if (a.dtype == SA_BF16) {
        if ((s = stca_ffn_weights_f16(L.hist_W1, L.hist_W3, L.hist_W2, w.W13t, w.W2t, st)) != SA_OK)
          return s;
        if ((s = stca_hist_ffn_tc((__half*)w.Hk, kv_total, w.W13t, w.W2t, st)) != SA_OK) return s;
      } else {
        if ((s = ffn_residual_gemm((float*)w.Hk, kv_total, a.D, L.hist_W1, L.hist_W3, L.hist_W2, w.G1,
                                   w.G3, w.U, "gemm:stca_hist_ffn", st)) != SA_OK)
          return s;
      }
      a.kv = w.Hk;
      a.kv_rows = kv_total;
      a.kvb_dev = w.kpre;
      a.kve_dev = w.kpre + 1;
    }
    // q's split is ready from stca_begin for the first layer, and from the previous
    // layer's output projection when that layer has no query FFN (which changes q)
    const bool split_out = !has_query(L) && l + 1 < a.n_layers;
    if ((s = stca_attend_layer(a, L.attn, w.attn, st, split_ready, split_out)) != SA_OK) return s;
    split_ready = split_out;
    // eq. (26): q <- q + FFN_q(q)
    if (has_query(L) &&
        (s = ffn_residual_gemm(a.out, a.C_total, a.D, L.q_W1, L.q_W3, L.q_W2, w.G1, w.G3, w.U,
                               "gemm:stca_q_ffn", st)) != SA_OK)
      return s;
  }
  return SA_OK;
}

}  // namespace sa
