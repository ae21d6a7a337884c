// STCA forward (SequenceO1 Sec. 2.3 eq. (4) in the reordering of Sec. 5.1
// eq. (24)) and the linear fusion of the two branches (Sec. 3.4).
//
// Per layer:  Qh = q W_Q^h;  U_h = Qh W_K^h^T * log2(e)/sqrt(d_h)  (GEMMs)
//             Y_h = softmax_i(U_h . x_i) x  over the user's keys  (attention)
//             O_h = Y_h W_V^h;  q <- q + concat_h(O_h) W_O          (GEMMs)
// Query rows of the attention are (candidate, head) pairs, so the history is
// read once per tile of 32 (CUDA cores) or 128 (tensor cores) rows.
#include <algorithm>

#include "stca_internal.cuh"

namespace sa {

namespace {
constexpr float kInf = __builtin_huge_valf();

template <class T>
__global__ void to_f32_kernel(const T* __restrict__ in, int64_t n, float* __restrict__ out) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x)
    out[e] = load_as_f32(in, e);
}

__global__ void add_kernel(float* __restrict__ y, const float* __restrict__ x, int64_t n) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x)
    y[e] += x[e];
}

// prefix[u] = number of query tiles of users < u; a user has
// ceil(C_u * heads / tq) tiles.
__global__ void tile_prefix_kernel(const int64_t* __restrict__ cand, int B, int heads, int tq,
                                   int* __restrict__ prefix) {
  if (blockIdx.x != 0 || threadIdx.x != 0) return;
  int acc = 0;
  prefix[0] = 0;
  for (int u = 0; u < B; ++u) {
    const int64_t rows = (cand[u + 1] - cand[u]) * heads;
    acc += (int)((rows + tq - 1) / tq);
    prefix[u + 1] = acc;
  }
}

// CUDA-core flash attention over K = V = x rows, D = 128.
template <class KT>
__global__ void __launch_bounds__(256) stca_attn_simt_kernel(
    const float* __restrict__ U, const KT* __restrict__ kv, const int64_t* __restrict__ cand,
    const int64_t* __restrict__ kvb, const int64_t* __restrict__ kve,
    const int* __restrict__ prefix, int B, int heads, float* __restrict__ Y) {
  constexpr int D = 128, TQ = 32, TK = 32, CPT = D / 8;
  __shared__ float Qs[TQ][D + 1];
  __shared__ float Ks[TK][D + 1];
  __shared__ float Pt[TQ][TK + 1];
  const int tile = blockIdx.x;
  if (tile >= prefix[B]) return;
  int lo = 0, hi = B - 1;                     // user: largest u with prefix[u] <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  const int u = lo;
  const int64_t rbeg = cand[u] * heads, rend = cand[u + 1] * heads;
  const int64_t r0 = rbeg + (int64_t)(tile - prefix[u]) * TQ;
  const int tid = threadIdx.x;
  for (int e = tid; e < TQ * D; e += 256) {
    const int rr = e / D, c = e % D;
    Qs[rr][c] = (r0 + rr < rend) ? U[(r0 + rr) * D + c] : 0.f;
  }
  const int r = tid / 8, sub = tid % 8;
  float acc[CPT];
#pragma unroll
  for (int i = 0; i < CPT; ++i) acc[i] = 0.f;
  float m = -kInf, l = 0.f;
  const int64_t kb = kvb[u], ke = kve[u];
  for (int64_t k0 = kb; k0 < ke; k0 += TK) {
    __syncthreads();
    for (int e = tid; e < TK * D; e += 256) {
      const int ii = e / D, c = e % D;
      Ks[ii][c] = (k0 + ii < ke) ? load_as_f32(kv, (k0 + ii) * D + c) : 0.f;
    }
    __syncthreads();
    float s[TK / 8];
    float smax = -kInf;
#pragma unroll
    for (int j = 0; j < TK / 8; ++j) {
      const int ii = sub + 8 * j;
      float v = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) v = fmaf(Qs[r][c], Ks[ii][c], v);
      s[j] = (k0 + ii < ke) ? v : -kInf;
      smax = fmaxf(smax, s[j]);
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
    const float mnew = fmaxf(m, smax);
    const float corr = exp2f(m - mnew);
    float psum = 0.f;
#pragma unroll
    for (int j = 0; j < TK / 8; ++j) {
      const float p = exp2f(s[j] - mnew);
      Pt[r][sub + 8 * j] = p;
      psum += p;
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    l = l * corr + psum;
    m = mnew;
    __syncwarp();
    __syncthreads();
#pragma unroll
    for (int i = 0; i < CPT; ++i) acc[i] *= corr;
#pragma unroll 4
    for (int ii = 0; ii < TK; ++ii) {
      const float p = Pt[r][ii];
#pragma unroll
      for (int i = 0; i < CPT; ++i) acc[i] = fmaf(p, Ks[ii][sub + 8 * i], acc[i]);
    }
  }
  const int64_t row = r0 + r;
  if (row < rend) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int i = 0; i < CPT; ++i) Y[row * D + sub + 8 * i] = acc[i] * inv;
  }
}

unsigned grid_for(int64_t n) { return (unsigned)std::min<int64_t>((n + 255) / 256, 8192); }
}  // namespace

sa_status stca_begin(const StcaArgs& a, const StcaWork& w, cudaStream_t st) {
  const int64_t C = a.C_total;
  const int64_t nq = C * a.D;
  if (nq > 0) {
    if (a.dtype == SA_BF16)
      SA_TIMED("to_f32_kernel", st,
               (to_f32_kernel<<<grid_for(nq), 256, 0, st>>>((const __nv_bfloat16*)a.q, nq, a.out)));
    else
      SA_TIMED("to_f32_kernel", st,
               (to_f32_kernel<<<grid_for(nq), 256, 0, st>>>((const float*)a.q, nq, a.out)));
  }
  if (C == 0) return SA_OK;
  const int tq = stca_tc_supported(a.dtype, a.D) ? 128 : 32;
  SA_TIMED("tile_prefix_kernel", st,
           (tile_prefix_kernel<<<1, 1, 0, st>>>(a.cand_dev, a.B, a.heads, tq, w.tile_prefix)));
  return SA_OK;
}

sa_status stca_attend_layer(const StcaArgs& a, const stca_layer& L, const StcaWork& w, cudaStream_t st) {
  const int D = a.D, H = a.heads, dh = a.d_h, HD = a.heads * a.d_h;
  const int64_t C = a.C_total;
  const int64_t nq = C * D;
  if (C == 0) return SA_OK;
  const bool tc = stca_tc_supported(a.dtype, D);
  sa_status s;
  {
    // Qh[:, h] = q W_Q^h
    Gemm g1;
    g1.M = (int)C; g1.N = dh; g1.K = D;
    g1.A = a.out; g1.lda = D; g1.sA = 0;
    g1.B = L.W_Q; g1.ldb = dh; g1.sB = (int64_t)D * dh;
    g1.C = w.Qh; g1.ldc = HD; g1.sC = dh; g1.tag = "gemm:stca_Qh";
    g1.batch = H;
    if ((s = gemm(g1, st)) != SA_OK) return s;
    // U[c, h, :] = Qh[:, h] W_K^h^T * log2(e)/sqrt(d_h)
    Gemm g2;
    g2.M = (int)C; g2.N = D; g2.K = dh;
    g2.A = w.Qh; g2.lda = HD; g2.sA = dh;
    g2.B = L.W_K; g2.ldb = dh; g2.transB = true; g2.sB = (int64_t)D * dh;
    if (tc) {
      g2.C16 = w.Ub; g2.ldc16 = (int64_t)H * D; g2.sC16 = D;
      g2.c16_half = a.kv_f16; g2.err = device_status_word();
    }
    else { g2.C = w.U; g2.ldc = (int64_t)H * D; g2.sC = D; }
    g2.alpha = 1.4426950408889634f / sqrtf((float)dh); g2.tag = "gemm:stca_U";
    g2.batch = H;
    if ((s = gemm(g2, st)) != SA_OK) return s;
    // Y = attention over the user's keys
    if (tc) {
      if ((s = stca_tc_attention(a, w, st)) != SA_OK) return s;
    } else {
      if (a.dtype == SA_BF16)
        SA_TIMED("stca_attn_simt_kernel", st,
                 (stca_attn_simt_kernel<__nv_bfloat16><<<w.max_tiles, 256, 0, st>>>(
                     w.U, (const __nv_bfloat16*)a.kv, a.cand_dev, a.kvb_dev, a.kve_dev,
                     w.tile_prefix, a.B, H, w.Y)));
      else
        SA_TIMED("stca_attn_simt_kernel", st,
                 (stca_attn_simt_kernel<float><<<w.max_tiles, 256, 0, st>>>(
                     w.U, (const float*)a.kv, a.cand_dev, a.kvb_dev, a.kve_dev, w.tile_prefix,
                     a.B, H, w.Y)));
    }
    // O[:, h] = Y[:, h, :] W_V^h
    Gemm g3;
    g3.M = (int)C; g3.N = dh; g3.K = D;
    g3.A = w.Y; g3.lda = (int64_t)H * D; g3.sA = D;
    g3.B = L.W_V; g3.ldb = dh; g3.sB = (int64_t)D * dh;
    g3.C = w.O; g3.ldc = HD; g3.sC = dh; g3.tag = "gemm:stca_O";
    g3.batch = H;
    if ((s = gemm(g3, st)) != SA_OK) return s;
    // q <- q + O W_O  (or q + O)
    if (L.W_O) {
      Gemm g4;
      g4.M = (int)C; g4.N = D; g4.K = HD;
      g4.A = w.O; g4.lda = HD;
      g4.B = L.W_O; g4.ldb = D;
      g4.C = a.out; g4.ldc = D;
      g4.Cin = a.out; g4.ldcin = D; g4.tag = "gemm:stca_WO";
      if ((s = gemm(g4, st)) != SA_OK) return s;
    } else {
      SA_TIMED("add_kernel", st, (add_kernel<<<grid_for(nq), 256, 0, st>>>(a.out, w.O, nq)));
    }
  }
  return SA_OK;
}

sa_status stca_run(const StcaArgs& a, const StcaWork& w, cudaStream_t st) {
  sa_status s = stca_begin(a, w, st);
  for (int l = 0; s == SA_OK && l < a.n_layers; ++l) s = stca_attend_layer(a, a.layers[l], w, st);
  return s;
}

sa_status stca_fuse_run(const float* z_r, const float* z_u, const float* W_F, const float* b_F,
                        int64_t C, int D, float* out, cudaStream_t st) {
  if (C == 0) return SA_OK;
  Gemm g1;
  g1.M = (int)C; g1.N = D; g1.K = D;
  g1.A = z_r; g1.lda = D; g1.B = W_F; g1.ldb = D; g1.C = out; g1.ldc = D; g1.bias = b_F; g1.tag = "gemm:fuse";
  sa_status s = gemm(g1, st);
  if (s != SA_OK) return s;
  Gemm g2;
  g2.M = (int)C; g2.N = D; g2.K = D;
  g2.A = z_u; g2.lda = D; g2.B = W_F + (int64_t)D * D; g2.ldb = D;
  g2.C = out; g2.ldc = D; g2.Cin = out; g2.ldcin = D; g2.tag = "gemm:fuse";
  return gemm(g2, st);
}

}  // namespace sa
