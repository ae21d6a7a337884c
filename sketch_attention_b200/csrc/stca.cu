// STCA forward (SequenceO1 Sec. 2.3 eq. (4) in the reordering of Sec. 5.1
// eq. (24)) and the linear fusion of the two branches (Sec. 3.4).
//
// Per layer:  Qh = q W_Q^h;  U_h = Qh W_K^h^T * log2(e)/sqrt(d_h)  (GEMMs)
//             Y_h = softmax_i(U_h . x_i) x  over the user's keys  (attention)
//             O_h = Y_h W_V^h;  q <- q + concat_h(O_h) W_O          (GEMMs)
// With bf16 inputs the projections run on the tensor cores with the heads' weights
// folded (two GEMMs per layer, see stca_attend_layer); fp32 inputs keep the CUDA-core
// GEMMs and attention.
// Query rows of the attention are (candidate, head) pairs, so the history is
// read once per tile of 32 (CUDA cores) or 128 (tensor cores) rows.
#include <algorithm>

#include "stca_internal.cuh"

namespace sa {

namespace {
constexpr float kInf = __builtin_huge_valf();


__global__ void add_kernel(float* __restrict__ y, const float* __restrict__ x, int64_t n) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x)
    y[e] += x[e];
}

// The start of an STCA call: q -> out (fp32) and, when qhi is given, q's hi + lo
// bf16 split; block 0 also writes prefix[u] = the number of query tiles of users < u (a
// user has ceil(C_u * heads / tq) tiles): per-user counts in parallel, then a scan over
// shared memory, 256 users at a time.
template <class T>
__global__ void __launch_bounds__(256) stca_begin_kernel(const T* __restrict__ q, int64_t n, float* __restrict__ out,
                                                         __nv_bfloat16* __restrict__ qhi, __nv_bfloat16* __restrict__ qlo,
                                                         const int64_t* __restrict__ cand, int B, int heads, int tq,
                                                         int* __restrict__ prefix) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const float v = load_as_f32(q, e);
    out[e] = v;
    if (qhi) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      qhi[e] = hi;
      qlo[e] = __float2bfloat16_rn(v - __bfloat162float(hi));
    }
  }
  if (blockIdx.x != 0 || !prefix) return;
  __shared__ int cnt[256];
  int base = 0;
  if (threadIdx.x == 0) prefix[0] = 0;
  for (int u0 = 0; u0 < B; u0 += 256) {
    const int u = u0 + threadIdx.x;
    cnt[threadIdx.x] = u < B ? (int)(((cand[u + 1] - cand[u]) * heads + tq - 1) / tq) : 0;
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int i = 0; i < 256 && u0 + i < B; ++i) {
        base += cnt[i];
        prefix[u0 + i + 1] = base;
      }
    }
    __syncthreads();
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

// The heads' folded weights of one layer as hi + lo bf16 splits:
//   M[k][h D + n] = sum_j W_Q^h[k][j] W_K^h[n][j] * scale        ([D, heads D])
//   N[h D + k][n] = sum_j W_V^h[k][j] W_O[h d_h + j][n]          ([heads D, D]; with W_O NULL
//                   (the identity) N[h D + k][n] = W_V^h[k][n - h d_h] inside head h's columns)
// One block per (head, matrix, 16 rows of k); the contraction over j runs in slices of 32
// staged in shared memory (the block's rows of W_Q^h or W_V^h, and W_K^h transposed or head
// h's rows of W_O); D = 128, each thread 8 outputs.
__global__ void __launch_bounds__(256) fold_heads_kernel(const float* __restrict__ W_Q, const float* __restrict__ W_K,
                                                         const float* __restrict__ W_V, const float* __restrict__ W_O,
                                                         int heads, int d_h, float scale,
                                                         __nv_bfloat16* __restrict__ Mhi, __nv_bfloat16* __restrict__ Mlo,
                                                         __nv_bfloat16* __restrict__ Nhi, __nv_bfloat16* __restrict__ Nlo) {
  constexpr int D = 128, KR = 16, JS = 32;
  __shared__ float a[KR][JS + 1];       // a[r][j]: W_Q^h (or W_V^h) row k0 + r, slice columns
  __shared__ float bt[JS][D + 1];       // bt[j][n]: W_K^h[n][j] (or W_O[h d_h + j][n])
  const int h = blockIdx.x, which = blockIdx.y, k0 = blockIdx.z * KR;
  const bool isM = which == 0;
  const float* Arows = (isM ? W_Q : W_V) + (int64_t)h * D * d_h;
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = 0.f;
  if (isM || W_O) {
    for (int j0 = 0; j0 < d_h; j0 += JS) {
      const int js = min(JS, d_h - j0);
      __syncthreads();
      for (int e = threadIdx.x; e < KR * JS; e += 256) {
        const int r = e / JS, j = e % JS;
        a[r][j] = j < js ? Arows[(int64_t)(k0 + r) * d_h + j0 + j] : 0.f;
      }
      for (int e = threadIdx.x; e < JS * D; e += 256) {
        const int j = e / D, n = e % D;
        float x = 0.f;
        if (j < js) x = isM ? W_K[((int64_t)h * D + n) * d_h + j0 + j] : W_O[((int64_t)h * d_h + j0 + j) * D + n];
        bt[j][n] = x;
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = threadIdx.x + 256 * i, r = e / D, n = e % D;
        for (int j = 0; j < js; ++j) v[i] = fmaf(a[r][j], bt[j][n], v[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = threadIdx.x + 256 * i, r = e / D, n = e % D, k = k0 + r;
    float x = v[i];
    if (isM) {
      x *= scale;
    } else if (!W_O) {
      x = (n >= h * d_h && n < (h + 1) * d_h) ? Arows[(int64_t)k * d_h + (n - h * d_h)] : 0.f;
    }
    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
    const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
    if (isM) {
      const int64_t o = (int64_t)k * heads * D + h * D + n;
      Mhi[o] = hi;
      Mlo[o] = lo;
    } else {
      const int64_t o = ((int64_t)h * D + k) * D + n;
      Nhi[o] = hi;
      Nlo[o] = lo;
    }
  }
}
}  // namespace

StcaWork stca_attn_carve(Carve& c, int B, int64_t C, int D, int heads, int d_h) {
  StcaWork v;
  const size_t rows = (size_t)std::max<int64_t>(C, 1);
  const size_t HD = (size_t)heads * D;
  v.Qh = c.take<float>(rows * heads * d_h);
  v.U = c.take<float>(rows * HD);
  v.Ub = c.take<__nv_bfloat16>(rows * HD);
  v.Y = c.take<float>(rows * HD);
  v.O = c.take<float>(rows * heads * d_h);
  v.tile_prefix = c.take<int>((size_t)B + 1);
  v.max_tiles = 0;
  v.Mhi = c.take<__nv_bfloat16>((size_t)D * HD);
  v.Mlo = c.take<__nv_bfloat16>((size_t)D * HD);
  v.Nhi = c.take<__nv_bfloat16>(HD * D);
  v.Nlo = c.take<__nv_bfloat16>(HD * D);
  v.qhi = c.take<__nv_bfloat16>(rows * D);
  v.qlo = c.take<__nv_bfloat16>(rows * D);
  v.Yhi = c.take<__nv_bfloat16>(rows * HD);
  v.Ylo = c.take<__nv_bfloat16>(rows * HD);
  v.part_floats = 4 * rows * D;
  v.part = c.take<float>(v.part_floats);
  return v;
}

sa_status stca_begin(const StcaArgs& a, const StcaWork& w, cudaStream_t st) {
  const int64_t C = a.C_total;
  const int64_t nq = C * a.D;
  if (nq == 0) return SA_OK;
  const bool tc = stca_tc_supported(a.dtype, a.D);
  const int tq = tc ? 128 : 32;
  __nv_bfloat16* qhi = tc ? w.qhi : nullptr;
  __nv_bfloat16* qlo = tc ? w.qlo : nullptr;
  if (a.dtype == SA_BF16)
    SA_TIMED("stca_begin_kernel", st,
             (stca_begin_kernel<<<grid_for(nq), 256, 0, st>>>((const __nv_bfloat16*)a.q, nq, a.out, qhi, qlo,
                                                              a.cand_dev, a.B, a.heads, tq, w.tile_prefix)));
  else
    SA_TIMED("stca_begin_kernel", st,
             (stca_begin_kernel<<<grid_for(nq), 256, 0, st>>>((const float*)a.q, nq, a.out, qhi, qlo, a.cand_dev,
                                                              a.B, a.heads, tq, w.tile_prefix)));
  return SA_OK;
}

// The tensor-core path (bf16 inputs, D = 128): the heads' projections folded into two
// weight matrices per layer, so each layer is two GEMMs on the tensor cores over hi + lo
// bf16 splits of their fp32 operands (about 16 significant bits, see tc_gemm):
//   U = q M,   M = [W_Q^h W_K^h^T log2(e)/sqrt(d_h)]_h   [D, heads D]   (16-bit output: the
//              attention's query operand, one row of D per (candidate, head))
//   q <- q + Y N,   N = [W_V^h W_O^h]_h                 [heads D, D]   (Y: the attention's
//              output, [C, heads D])
// (the associativity of eqs. (24)-(26): (q W_Q^h) W_K^h^T = q (W_Q^h W_K^h^T) and
// sum_h (Y_h W_V^h) W_O^h = Y N).
sa_status tc_projections_prepare(const StcaArgs& a, const stca_layer& L, const StcaWork& w, cudaStream_t st) {
  const int D = a.D, H = a.heads, dh = a.d_h;
  if (D != 128) return fail(SA_ERR_UNSUPPORTED, "the tensor-core projections take D = 128");
  SA_TIMED("fold_heads_kernel", st,
           (fold_heads_kernel<<<dim3(H, 2, D / 16), 256, 0, st>>>(L.W_Q, L.W_K, L.W_V, L.W_O, H, dh,
                                                                  1.4426950408889634f / sqrtf((float)dh), w.Mhi,
                                                                  w.Mlo, w.Nhi, w.Nlo)));
  return SA_OK;
}

sa_status stca_attend_layer(const StcaArgs& a, const stca_layer& L, const StcaWork& w, cudaStream_t st,
                            bool q_split, bool split_out) {
  const int D = a.D, H = a.heads, dh = a.d_h, HD = a.heads * a.d_h;
  const int64_t C = a.C_total;
  const int64_t nq = C * D;
  if (C == 0) return SA_OK;
  const bool tc = stca_tc_supported(a.dtype, D);
  sa_status s;
  if (tc) {
    if ((s = tc_projections_prepare(a, L, w, st)) != SA_OK) return s;
    if (!q_split && (s = split_hi_lo(a.out, nq, w.qhi, w.qlo, st)) != SA_OK) return s;
    TcGemm gu;                                // U = q M -> the attention's 16-bit queries
    gu.M = (int)C; gu.N = H * D; gu.K = D;
    gu.A = w.qhi; gu.A_lo = w.qlo; gu.lda = D;
    gu.B = w.Mhi; gu.B_lo = w.Mlo; gu.ldb = (int64_t)H * D; gu.b_mn = true;
    gu.C16 = w.Ub; gu.ldc16 = (int64_t)H * D; gu.c16_half = a.kv_f16;
    gu.tag = "tc_gemm:stca_U";
    if ((s = tc_gemm(gu, st)) != SA_OK) return s;
    if ((s = stca_tc_attention(a, w, st, true)) != SA_OK) return s;
    TcGemm go;                                // q <- q + Y N
    go.M = (int)C; go.N = D; go.K = H * D;
    go.A = w.Yhi; go.A_lo = w.Ylo; go.lda = (int64_t)H * D;
    go.B = w.Nhi; go.B_lo = w.Nlo; go.ldb = D; go.b_mn = true;
    go.C = a.out; go.ldc = D; go.Cin = a.out; go.ldcin = D;
    if (split_out) { go.Chi = w.qhi; go.Clo = w.qlo; go.ldcs = D; }   // the next layer's q split
    go.tag = "tc_gemm:stca_O";
    return tc_gemm(go, st);
  }
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
    g2.C = w.U; g2.ldc = (int64_t)H * D; g2.sC = D;
    g2.alpha = 1.4426950408889634f / sqrtf((float)dh); g2.tag = "gemm:stca_U";
    g2.batch = H;
    if ((s = gemm(g2, st)) != SA_OK) return s;
    // Y = attention over the user's keys (CUDA cores)
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
  // stca_begin split q; each output projection splits the q it writes for the next layer
  for (int l = 0; s == SA_OK && l < a.n_layers; ++l)
    s = stca_attend_layer(a, a.layers[l], w, st, true, l + 1 < a.n_layers);
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
