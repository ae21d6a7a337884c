// Sketch Attention on the CUDA cores (fp32 FMA): the fp32 path, and the path
// for shapes the tensor-core kernel does not take.  Also holds the pieces
// every SA path shares: prototype folding, the split-n reduction with the
// normalisation, and the backward kernels.
//
// Paper: SequenceO1, Sec. 3.1 eqs. (6)-(9) (forward); the backward is the
// chain rule of that forward.
//
// Units: the folded prototypes P' = P W_Q W_K^T * log2(e)/sqrt(d) give
// logits in base-2 units, z = P' x = Z log2(e), so every exponential is an
// exp2.  Per-token statistics ("lse") are log2(sum_j 2^z_j).
#include <algorithm>

#include "sa_internal.cuh"
#include "stca_internal.cuh"

namespace sa {

namespace {
constexpr float kInf = __builtin_huge_valf();
constexpr float kLn2 = 0.69314718055994530942f;

template <int D, class XT>
__device__ __forceinline__ void load_row_f32(float* dst, const XT* src, int64_t row, bool valid) {
#pragma unroll 4
  for (int c = 0; c < D; ++c) dst[c] = valid ? load_as_f32(src, row * D + c) : 0.f;
}

// ---------------------------------------------------------------- pass 1
// lse[t] = log2 sum_j 2^{z_jt} over all k prototypes, one thread per token.
template <class XT, int D>
__global__ void __launch_bounds__(128) sa_lse_kernel(const XT* __restrict__ X, int64_t n_total,
                                                     const float* __restrict__ Pf, int k,
                                                     float* __restrict__ lse,
                                                     float* __restrict__ lse_nat) {
  __shared__ float Ps[32][D];
  const int64_t t = (int64_t)blockIdx.x * 128 + threadIdx.x;
  const bool valid = t < n_total;
  float x[D];
  load_row_f32<D>(x, X, valid ? t : 0, valid);
  float m = -kInf, s = 0.f;
  for (int j0 = 0; j0 < k; j0 += 32) {
    const int nj = min(32, k - j0);
    __syncthreads();
    for (int e = threadIdx.x; e < nj * D; e += 128) Ps[e / D][e % D] = Pf[(int64_t)j0 * D + e];
    __syncthreads();
    for (int jj = 0; jj < nj; ++jj) {
      float z = 0.f;
#pragma unroll
      for (int c = 0; c < D; ++c) z = fmaf(Ps[jj][c], x[c], z);
      if (z > m) { s = s * exp2f(m - z) + 1.f; m = z; }
      else s += exp2f(z - m);
    }
  }
  if (valid) {
    const float l2 = m + log2f(s);
    lse[t] = l2;
    if (lse_nat) lse_nat[t] = l2 * kLn2;
  }
}

// lse2[t] = lse[t] * log2(e): a caller-provided natural-log lse in base-2 units.
__global__ void lse_to_log2_kernel(const float* __restrict__ lse, int64_t n,
                                   float* __restrict__ lse2) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x)
    lse2[e] = lse[e] * 1.4426950408889634f;
}

// ---------------------------------------------------------------- pass 2
// One CTA = (block of KB prototypes, chunk g).  For each piece of the chunk:
//   H_j += sum_t 2^{z_jt - lse_t} x_t,   m_j += sum_t 2^{z_jt - lse_t}.
template <class XT, int D>
__global__ void __launch_bounds__(256) sa_agg_kernel(
    const XT* __restrict__ X, const int64_t* __restrict__ off, int B, Chunking ch,
    const float* __restrict__ Pf, int k, const float* __restrict__ lse,
    float* __restrict__ Huser, float* __restrict__ Muser, float* __restrict__ slotH,
    float* __restrict__ slotM) {
  constexpr int KB = 32, TT = 32, CPT = D / 8;
  __shared__ float Ps[KB][D + 1];
  __shared__ float Xs[TT][D + 1];
  __shared__ float Pt[KB][TT + 1];
  __shared__ float Ls[TT];
  const int tid = threadIdx.x;
  const int j0 = blockIdx.x * KB;
  const int nj = min(KB, k - j0);
  const int g = blockIdx.y;
  const int64_t cb = (int64_t)g * ch.T, ce = min(cb + ch.T, ch.n_total);
  for (int e = tid; e < KB * D; e += 256) {
    const int jj = e / D, c = e % D;
    Ps[jj][c] = jj < nj ? Pf[(int64_t)(j0 + jj) * D + c] : 0.f;
  }
  const int ja = tid / 8;           // accumulation row
  const int ca = tid % 8;           // accumulation columns ca + 8 i
  for (int u = user_of_token(off, B, cb); u < B && off[u] < ce; ++u) {
    const int64_t pb = max(off[u], cb), pe = min(off[u + 1], ce);
    if (pb >= pe) continue;
    float acc[CPT];
#pragma unroll
    for (int i = 0; i < CPT; ++i) acc[i] = 0.f;
    float macc = 0.f;
    for (int64_t t0 = pb; t0 < pe; t0 += TT) {
      __syncthreads();
      for (int e = tid; e < TT * D; e += 256) {
        const int tt = e / D, c = e % D;
        const int64_t t = t0 + tt;
        Xs[tt][c] = t < pe ? load_as_f32(X, t * D + c) : 0.f;
      }
      if (tid < TT) Ls[tid] = (t0 + tid < pe) ? lse[t0 + tid] : kInf;
      __syncthreads();
      {
        const int tt = tid % TT;
#pragma unroll
        for (int r = 0; r < KB / 8; ++r) {
          const int jj = tid / TT + 8 * r;
          float z = 0.f;
#pragma unroll 8
          for (int c = 0; c < D; ++c) z = fmaf(Ps[jj][c], Xs[tt][c], z);
          Pt[jj][tt] = jj < nj ? exp2f(z - Ls[tt]) : 0.f;
        }
      }
      __syncthreads();
#pragma unroll 4
      for (int tt = 0; tt < TT; ++tt) {
        const float p = Pt[ja][tt];
        macc += p;
#pragma unroll
        for (int i = 0; i < CPT; ++i) acc[i] = fmaf(p, Xs[tt][ca + 8 * i], acc[i]);
      }
    }
    if (ja < nj) {
      const int dest = piece_dest(off[u], off[u + 1], cb, ce);
      float* Hrow;
      float* mrow;
      if (dest == DEST_USER) {
        Hrow = Huser + ((int64_t)u * k + j0 + ja) * D;
        mrow = Muser + (int64_t)u * k + j0 + ja;
      } else {
        Hrow = slotH + (((int64_t)g * 2 + dest) * k + j0 + ja) * D;
        mrow = slotM + ((int64_t)g * 2 + dest) * k + j0 + ja;
      }
#pragma unroll
      for (int i = 0; i < CPT; ++i) Hrow[ca + 8 * i] = acc[i];
      if (ca == 0) *mrow = macc;
    }
  }
}

// ---------------------------------------------------------------- split-n reduce
// Assemble H_u and m_u of every user from the per-user rows and the chunk
// slots (fixed order, so the result is deterministic), write mass and the
// optional H, and Hh = H/(m+eps) (zero where m+eps == 0) for the value GEMM.
__global__ void __launch_bounds__(256) sa_reduce_kernel(
    const int64_t* __restrict__ off, int B, Chunking ch, int k, int D, float eps,
    const float* __restrict__ Huser, const float* __restrict__ Muser,
    const float* __restrict__ slotH, const float* __restrict__ slotM,
    float* __restrict__ Hout, float* __restrict__ mass_out, float* __restrict__ Hhat,
    __nv_bfloat16* __restrict__ Hhi, __nv_bfloat16* __restrict__ Hlo) {
  constexpr int RB = 8;
  __shared__ float inv[RB];
  const int u = blockIdx.y;
  const int j0 = blockIdx.x * RB;
  const int64_t ub = off[u], ue = off[u + 1];
  const bool empty = ue <= ub;
  const int64_t gf = empty ? 0 : ub / ch.T, gl = empty ? 0 : (ue - 1) / ch.T;
  if (threadIdx.x < RB) {
    const int j = j0 + threadIdx.x;
    if (j < k) {
      float m = 0.f;
      if (!empty) {
        if (gf == gl) m = Muser[(int64_t)u * k + j];
        else {
          m = slotM[((int64_t)gf * 2 + 1) * k + j];
          for (int64_t g = gf + 1; g < gl; ++g) m += slotM[((int64_t)g * 2 + 0) * k + j];
          m += slotM[((int64_t)gl * 2 + 0) * k + j];
        }
      }
      mass_out[(int64_t)u * k + j] = m;
      const float den = m + eps;
      inv[threadIdx.x] = den > 0.f ? 1.f / den : 0.f;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < RB * D; e += 256) {
    const int jj = e / D, c = e % D, j = j0 + jj;
    if (j >= k) continue;
    float h = 0.f;
    if (!empty) {
      if (gf == gl) h = Huser[((int64_t)u * k + j) * D + c];
      else {
        h = slotH[(((int64_t)gf * 2 + 1) * k + j) * D + c];
        for (int64_t g = gf + 1; g < gl; ++g) h += slotH[(((int64_t)g * 2 + 0) * k + j) * D + c];
        h += slotH[(((int64_t)gl * 2 + 0) * k + j) * D + c];
      }
    }
    const int64_t o = ((int64_t)u * k + j) * D + c;
    if (Hout) Hout[o] = h;
    const float hh = h * inv[jj];
    Hhat[o] = hh;
    if (Hhi) {
      // the output projection's split operand: hh = hi + lo
      const __nv_bfloat16 hi = __float2bfloat16_rn(hh);
      Hhi[o] = hi;
      Hlo[o] = __float2bfloat16_rn(hh - __bfloat162float(hi));
    }
  }
}

// ---------------------------------------------------------------- backward
// Per row (u, j): Hh = H/(m+eps), dH = dHh/(m+eps), dm = -(dHh . Hh)/(m+eps) + dmass.
__global__ void __launch_bounds__(256) sa_bwd_prologue_kernel(
    int rows, int D, float eps, const float* __restrict__ H, const float* __restrict__ mass,
    const float* __restrict__ dHh, const float* __restrict__ dmass, float* __restrict__ Hhat,
    float* __restrict__ dH, __nv_bfloat16* __restrict__ dHb, __nv_bfloat16* __restrict__ dHlo,
    float* __restrict__ dm, __nv_bfloat16* __restrict__ Hhi, __nv_bfloat16* __restrict__ Hlo) {
  const int warp = (blockIdx.x * 256 + threadIdx.x) / 32, lane = threadIdx.x % 32;
  if (warp >= rows) return;
  const float den = mass[warp] + eps;
  const float inv = den > 0.f ? 1.f / den : 0.f;
  float dot = 0.f;
  for (int c = lane; c < D; c += 32) {
    const int64_t o = (int64_t)warp * D + c;
    const float hh = H[o] * inv;
    Hhat[o] = hh;
    if (Hhi) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(hh);
      Hhi[o] = hi;
      Hlo[o] = __float2bfloat16_rn(hh - __bfloat162float(hi));
    }
    dH[o] = dHh[o] * inv;
    if (dHb) {
      const float v = dHh[o] * inv;
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      dHb[o] = hi;
      dHlo[o] = __float2bfloat16_rn(v - __bfloat162float(hi));
    }
    dot = fmaf(dHh[o], hh, dot);
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, s);
  if (lane == 0) dm[warp] = -dot * inv + (dmass ? dmass[warp] : 0.f);
}

// Per token t of user u: c_t = sum_j A_jt (dH_j . x_t + dm_j), then
// dX_t = sum_j A_jt dH_j + sum_j dZ_jt p'_j (natural units), dZ = A (dA - c).
template <class XT, int D>
__global__ void __launch_bounds__(256) sa_bwd_token_kernel(
    const XT* __restrict__ X, const int64_t* __restrict__ off, int B, Chunking ch,
    const float* __restrict__ Pf, int k, const float* __restrict__ lse,
    const float* __restrict__ dH, const float* __restrict__ dm, float* __restrict__ cbuf,
    XT* __restrict__ dX) {
  constexpr int TT = 32, KB = 16, CPT = D / 8;
  __shared__ float Xs[TT][D + 1];
  __shared__ float Ps[KB][D + 1];
  __shared__ float Gs[KB][D + 1];
  __shared__ float As[KB][TT + 1];
  __shared__ float Zs[KB][TT + 1];
  __shared__ float dms[KB];
  __shared__ float Ls[TT], Cs[TT];
  __shared__ float cpart[8][TT];
  const int tid = threadIdx.x;
  const int g = blockIdx.x;
  const int64_t cb = (int64_t)g * ch.T, ce = min(cb + ch.T, ch.n_total);
  const int tt1 = tid % TT, jg = tid / TT;       // pass-1 mapping
  const int tt2 = tid / 8, c2 = tid % 8;         // pass-2 mapping
  for (int u = user_of_token(off, B, cb); u < B && off[u] < ce; ++u) {
    const int64_t pb = max(off[u], cb), pe = min(off[u + 1], ce);
    if (pb >= pe) continue;
    const float* dHu = dH + (int64_t)u * k * D;
    const float* dmu = dm + (int64_t)u * k;
    for (int64_t t0 = pb; t0 < pe; t0 += TT) {
      __syncthreads();
      for (int e = tid; e < TT * D; e += 256) {
        const int tt = e / D, c = e % D;
        const int64_t t = t0 + tt;
        Xs[tt][c] = t < pe ? load_as_f32(X, t * D + c) : 0.f;
      }
      if (tid < TT) Ls[tid] = (t0 + tid < pe) ? lse[t0 + tid] : kInf;
      float cacc = 0.f;
      for (int j0 = 0; j0 < k; j0 += KB) {
        const int nj = min(KB, k - j0);
        __syncthreads();
        for (int e = tid; e < KB * D; e += 256) {
          const int jj = e / D, c = e % D;
          Ps[jj][c] = jj < nj ? Pf[(int64_t)(j0 + jj) * D + c] : 0.f;
          Gs[jj][c] = jj < nj ? dHu[(int64_t)(j0 + jj) * D + c] : 0.f;
        }
        if (tid < KB) dms[tid] = tid < nj ? dmu[j0 + tid] : 0.f;
        __syncthreads();
#pragma unroll
        for (int r = 0; r < KB / 8; ++r) {
          const int jj = jg + 8 * r;
          if (jj >= nj) continue;
          float z = 0.f, gd = 0.f;
#pragma unroll 8
          for (int c = 0; c < D; ++c) {
            z = fmaf(Ps[jj][c], Xs[tt1][c], z);
            gd = fmaf(Gs[jj][c], Xs[tt1][c], gd);
          }
          const float a = exp2f(z - Ls[tt1]);
          cacc = fmaf(a, gd + dms[jj], cacc);
        }
      }
      cpart[jg][tt1] = cacc;
      __syncthreads();
      if (tid < TT) {
        float c = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) c += cpart[q][tid];
        Cs[tid] = c;
      }
      float acc[CPT];
#pragma unroll
      for (int i = 0; i < CPT; ++i) acc[i] = 0.f;
      for (int j0 = 0; j0 < k; j0 += KB) {
        const int nj = min(KB, k - j0);
        __syncthreads();
        for (int e = tid; e < KB * D; e += 256) {
          const int jj = e / D, c = e % D;
          Ps[jj][c] = jj < nj ? Pf[(int64_t)(j0 + jj) * D + c] : 0.f;
          Gs[jj][c] = jj < nj ? dHu[(int64_t)(j0 + jj) * D + c] : 0.f;
        }
        if (tid < KB) dms[tid] = tid < nj ? dmu[j0 + tid] : 0.f;
        __syncthreads();
#pragma unroll
        for (int r = 0; r < KB / 8; ++r) {
          const int jj = jg + 8 * r;
          float a = 0.f, dz = 0.f;
          if (jj < nj) {
            float z = 0.f, gd = 0.f;
#pragma unroll 8
            for (int c = 0; c < D; ++c) {
              z = fmaf(Ps[jj][c], Xs[tt1][c], z);
              gd = fmaf(Gs[jj][c], Xs[tt1][c], gd);
            }
            a = exp2f(z - Ls[tt1]);
            dz = a * (gd + dms[jj] - Cs[tt1]);
          }
          As[jj][tt1] = a;
          Zs[jj][tt1] = dz * kLn2;     // p' in log2 units -> natural units
        }
        __syncthreads();
#pragma unroll 4
        for (int jj = 0; jj < KB; ++jj) {
          const float a = As[jj][tt2], dz = Zs[jj][tt2];
#pragma unroll
          for (int i = 0; i < CPT; ++i)
            acc[i] = fmaf(a, Gs[jj][c2 + 8 * i], fmaf(dz, Ps[jj][c2 + 8 * i], acc[i]));
        }
      }
      const int64_t t = t0 + tt2;
      if (t < pe) {
#pragma unroll
        for (int i = 0; i < CPT; ++i) store_from_f32(dX, t * D + c2 + 8 * i, acc[i]);
      }
      if (tid < TT && t0 + tid < pe) cbuf[t0 + tid] = Cs[tid];
    }
  }
}

// E_part[g] = sum over the chunk's tokens of dZ_jt x_t (all users together).
template <class XT, int D>
__global__ void __launch_bounds__(256) sa_bwd_E_kernel(
    const XT* __restrict__ X, const int64_t* __restrict__ off, int B, Chunking ch,
    const float* __restrict__ Pf, int k, const float* __restrict__ lse,
    const float* __restrict__ dH, const float* __restrict__ dm, const float* __restrict__ cbuf,
    float* __restrict__ Epart) {
  constexpr int KB = 16, TT = 32, CPT = D / 16;
  __shared__ float Ps[KB][D + 1];
  __shared__ float Gs[KB][D + 1];
  __shared__ float Xs[TT][D + 1];
  __shared__ float Pt[KB][TT + 1];
  __shared__ float dms[KB];
  __shared__ float Ls[TT], Cs[TT];
  const int tid = threadIdx.x;
  const int j0 = blockIdx.x * KB;
  const int nj = min(KB, k - j0);
  const int g = blockIdx.y;
  const int64_t cb = (int64_t)g * ch.T, ce = min(cb + ch.T, ch.n_total);
  for (int e = tid; e < KB * D; e += 256) {
    const int jj = e / D, c = e % D;
    Ps[jj][c] = jj < nj ? Pf[(int64_t)(j0 + jj) * D + c] : 0.f;
  }
  const int ja = tid / 16, ca = tid % 16;
  float acc[CPT];
#pragma unroll
  for (int i = 0; i < CPT; ++i) acc[i] = 0.f;
  for (int u = user_of_token(off, B, cb); u < B && off[u] < ce; ++u) {
    const int64_t pb = max(off[u], cb), pe = min(off[u + 1], ce);
    if (pb >= pe) continue;
    __syncthreads();
    for (int e = tid; e < KB * D; e += 256) {
      const int jj = e / D, c = e % D;
      Gs[jj][c] = jj < nj ? dH[((int64_t)u * k + j0 + jj) * D + c] : 0.f;
    }
    if (tid < KB) dms[tid] = tid < nj ? dm[(int64_t)u * k + j0 + tid] : 0.f;
    for (int64_t t0 = pb; t0 < pe; t0 += TT) {
      __syncthreads();
      for (int e = tid; e < TT * D; e += 256) {
        const int tt = e / D, c = e % D;
        const int64_t t = t0 + tt;
        Xs[tt][c] = t < pe ? load_as_f32(X, t * D + c) : 0.f;
      }
      if (tid < TT) {
        const bool v = t0 + tid < pe;
        Ls[tid] = v ? lse[t0 + tid] : kInf;
        Cs[tid] = v ? cbuf[t0 + tid] : 0.f;
      }
      __syncthreads();
      {
        const int tt = tid % TT;
#pragma unroll
        for (int r = 0; r < KB / 8; ++r) {
          const int jj = tid / TT + 8 * r;
          float z = 0.f, gd = 0.f;
#pragma unroll 8
          for (int c = 0; c < D; ++c) {
            z = fmaf(Ps[jj][c], Xs[tt][c], z);
            gd = fmaf(Gs[jj][c], Xs[tt][c], gd);
          }
          const float a = exp2f(z - Ls[tt]);
          Pt[jj][tt] = jj < nj ? a * (gd + dms[jj] - Cs[tt]) : 0.f;
        }
      }
      __syncthreads();
#pragma unroll 4
      for (int tt = 0; tt < TT; ++tt) {
        const float p = Pt[ja][tt];
#pragma unroll
        for (int i = 0; i < CPT; ++i) acc[i] = fmaf(p, Xs[tt][ca + 16 * i], acc[i]);
      }
    }
  }
  if (ja < nj) {
#pragma unroll
    for (int i = 0; i < CPT; ++i) Epart[((int64_t)g * k + j0 + ja) * D + ca + 16 * i] = acc[i];
  }
}

// out[e] = sum_g part[g][e], fixed order.
__global__ void sum_slices_kernel(const float* __restrict__ part, int G, int64_t n,
                                  float* __restrict__ out) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int g = 0; g < G; ++g) s += part[(int64_t)g * n + e];
    out[e] = s;
  }
}

template <class XT, int D>
sa_status launch_simt_forward(const SaFwdArgs& a, const SaFwdWork& w, cudaStream_t st) {
  const int64_t N = a.n_total;
  if (N > 0) {
    SA_TIMED("sa_lse_kernel", st,
             (sa_lse_kernel<XT, D><<<(unsigned)((N + 127) / 128), 128, 0, st>>>(
                 (const XT*)a.X, N, w.Pf, a.k, w.lse, a.lse_out)));
    dim3 grid((a.k + 31) / 32, w.ch.G);
    SA_TIMED("sa_agg_kernel", st,
             (sa_agg_kernel<XT, D><<<grid, 256, 0, st>>>((const XT*)a.X, a.off_dev, a.B, w.ch,
                                                        w.Pf, a.k, w.lse, a.S, w.Muser, w.slotH,
                                                        w.slotM)));
  }
  return SA_OK;
}

template <class XT, int D>
sa_status launch_simt_backward(const SaBwdArgs& a, const SaBwdWork& w, cudaStream_t st) {
  SA_TIMED("sa_bwd_token_kernel", st,
           (sa_bwd_token_kernel<XT, D><<<w.ch.G, 256, 0, st>>>(
               (const XT*)a.X, a.off_dev, a.B, w.ch, w.Pf, a.k, w.lse, w.dH, w.dm, w.cbuf,
               (XT*)a.dX)));
  dim3 grid((a.k + 15) / 16, w.chE.G);
  SA_TIMED("sa_bwd_E_kernel", st,
           (sa_bwd_E_kernel<XT, D><<<grid, 256, 0, st>>>((const XT*)a.X, a.off_dev, a.B, w.chE,
                                                        w.Pf, a.k, w.lse, w.dH, w.dm, w.cbuf,
                                                        w.Epart)));
  return SA_OK;
}

// lse (base 2) of every token: converted from the caller's saved lse, or recomputed.
template <class XT, int D>
sa_status backward_lse(const SaBwdArgs& a, const SaBwdWork& w, cudaStream_t st) {
  const int64_t N = a.n_total;
  if (a.lse_in) {
    SA_TIMED("lse_to_log2_kernel", st,
             (lse_to_log2_kernel<<<(unsigned)std::min<int64_t>((N + 255) / 256, 8192), 256, 0, st>>>(
                 a.lse_in, N, w.lse)));
  } else {
    SA_TIMED("sa_lse_kernel", st,
             (sa_lse_kernel<XT, D><<<(unsigned)((N + 127) / 128), 128, 0, st>>>(
                 (const XT*)a.X, N, w.Pf, a.k, w.lse, nullptr)));
  }
  return SA_OK;
}
}  // namespace

// ---------------------------------------------------------------- host entry points
sa_status sa_fold(int k, int d, const float* P, const float* W_Q, const float* W_K, float* T,
                  float* Pf, __nv_bfloat16* Pb, cudaStream_t st) {
  // T = W_Q W_K^T;  P' = P T * log2(e)/sqrt(d)
  Gemm g1;
  g1.M = d; g1.N = d; g1.K = d;
  g1.A = W_Q; g1.lda = d;
  g1.B = W_K; g1.ldb = d; g1.transB = true;
  g1.C = T; g1.ldc = d; g1.tag = "gemm:fold";
  sa_status s = gemm(g1, st);
  if (s != SA_OK) return s;
  Gemm g2;
  g2.M = k; g2.N = d; g2.K = d;
  g2.A = P; g2.lda = d;
  g2.B = T; g2.ldb = d;
  g2.C = Pf; g2.ldc = d; g2.tag = "gemm:fold";
  g2.C16 = Pb; g2.ldc16 = d;
  g2.alpha = 1.4426950408889634f / sqrtf((float)d);
  return gemm(g2, st);
}

sa_status sa_simt_forward(const SaFwdArgs& a, const SaFwdWork& w, cudaStream_t st) {
  const bool bf = a.x_dtype == SA_BF16;
  if (a.d == 64) return bf ? launch_simt_forward<__nv_bfloat16, 64>(a, w, st)
                           : launch_simt_forward<float, 64>(a, w, st);
  return bf ? launch_simt_forward<__nv_bfloat16, 128>(a, w, st)
            : launch_simt_forward<float, 128>(a, w, st);
}

sa_status sa_reduce(const SaFwdArgs& a, const SaFwdWork& w, cudaStream_t st) {
  dim3 grid((a.k + 7) / 8, a.B);
  SA_TIMED("sa_reduce_kernel", st,
           (sa_reduce_kernel<<<grid, 256, 0, st>>>(a.off_dev, a.B, w.ch, a.k, a.d, a.eps, a.S,
                                                   w.Muser, w.slotH, w.slotM, a.H, a.mass,
                                                   w.Hhat, w.Vhi ? w.Hhi : nullptr,
                                                   w.Vhi ? w.Hlo : nullptr)));
  return SA_OK;
}

sa_status sa_reduce_and_project(const SaFwdArgs& a, const SaFwdWork& w, cudaStream_t st) {
  sa_status s = sa_reduce(a, w, st);
  if (s != SA_OK) return s;
  if (w.Hhi && w.Vhi) {
    // S = Hh W_V on the tensor cores over hi + lo splits of both (three passes, about 16
    // significant bits), with its bf16 copy
    if ((s = split_hi_lo(a.W_V, (int64_t)a.d * a.d, w.Vhi, w.Vlo, st)) != SA_OK) return s;
    TcGemm t;
    t.M = a.B * a.k; t.N = a.d; t.K = a.d;
    t.A = w.Hhi; t.A_lo = w.Hlo; t.lda = a.d;
    t.B = w.Vhi; t.B_lo = w.Vlo; t.ldb = a.d; t.b_mn = true;
    t.C = a.S; t.ldc = a.d;
    t.C16 = (__nv_bfloat16*)a.S_bf16; t.ldc16 = a.d;
    t.tag = "tc_gemm:S_proj";
    return tc_gemm(t, st);
  }
  // S = Hh W_V (and its bf16 copy)
  Gemm g;
  g.M = a.B * a.k; g.N = a.d; g.K = a.d;
  g.A = w.Hhat; g.lda = a.d;
  g.B = a.W_V; g.ldb = a.d;
  g.C = a.S; g.ldc = a.d;
  g.C16 = (__nv_bfloat16*)a.S_bf16; g.ldc16 = a.d; g.tag = "gemm:S_proj";
  return gemm(g, st);
}

sa_status sa_backward_run(const SaBwdArgs& a, const SaBwdWork& w, bool tc, cudaStream_t st) {
  const int rows = a.B * a.k;
  const int D = a.d;
  // the two W_V products on the tensor cores over hi + lo splits (three passes, about 16
  // significant bits) when the workspace has the split buffers, else fp32 GEMMs
  const bool tcp = tc && w.dShi && w.Hhi && w.Vhi;
  sa_status s;
  // dHh = dS W_V^T
  if (tcp) {
    if ((s = split_hi_lo(a.dS, (int64_t)rows * D, w.dShi, w.dSlo, st)) != SA_OK) return s;
    if ((s = split_hi_lo(a.W_V, (int64_t)D * D, w.Vhi, w.Vlo, st)) != SA_OK) return s;
    TcGemm t;
    t.M = rows; t.N = D; t.K = D;
    t.A = w.dShi; t.A_lo = w.dSlo; t.lda = D;
    t.B = w.Vhi; t.B_lo = w.Vlo; t.ldb = D;      // B[n][k] = W_V[n][k]: K-major
    t.C = w.dHh; t.ldc = D; t.tag = "tc_gemm:dHh";
    if ((s = tc_gemm(t, st)) != SA_OK) return s;
  } else {
    Gemm g;
    g.M = rows; g.N = D; g.K = D;
    g.A = a.dS; g.lda = D;
    g.B = a.W_V; g.ldb = D; g.transB = true;
    g.C = w.dHh; g.ldc = D; g.tag = "gemm:dHh";
    if ((s = gemm(g, st)) != SA_OK) return s;
  }
  SA_TIMED("sa_bwd_prologue_kernel", st,
           (sa_bwd_prologue_kernel<<<(rows * 32 + 255) / 256, 256, 0, st>>>(
               rows, D, a.eps, a.H, a.mass, w.dHh, a.dmass, w.Hhat, w.dH, tc ? w.dHb : nullptr,
               tc ? w.dHlo : nullptr, w.dm, tcp ? w.Hhi : nullptr, tcp ? w.Hlo : nullptr)));
  // dW_V = sum_u Hh_u^T dS_u
  if (tcp) {
    TcGemm t;
    t.M = D; t.N = D; t.K = rows;
    t.A = w.Hhi; t.A_lo = w.Hlo; t.lda = D; t.a_mn = true;      // A[k][m] = Hhat[k][m]
    t.B = w.dShi; t.B_lo = w.dSlo; t.ldb = D; t.b_mn = true;    // B[k][n] = dS[k][n]
    t.C = a.dW_V; t.ldc = D;
    if (a.accumulate) { t.Cin = a.dW_V; t.ldcin = D; }
    t.part = w.gsplit; t.part_floats = (size_t)kMaxSplit * D * D;
    t.tag = "tc_gemm:dW_V";
    if ((s = tc_gemm(t, st)) != SA_OK) return s;
  } else {
    Gemm gv;
    gv.M = D; gv.N = D; gv.K = rows;
    gv.A = w.Hhat; gv.lda = D; gv.transA = true;
    gv.B = a.dS; gv.ldb = D;
    gv.C = a.dW_V; gv.ldc = D;
    if (a.accumulate) { gv.Cin = a.dW_V; gv.ldcin = D; }
    gv.tag = "gemm:dW_V";
    gv.split_k = gemm_split_for(D, D, rows, kMaxSplit);
    gv.split_ws = w.gsplit;
    if ((s = gemm(gv, st)) != SA_OK) return s;
  }
  if (a.n_total > 0) {
    const bool bf = a.x_dtype == SA_BF16;
    if (D == 64) s = bf ? backward_lse<__nv_bfloat16, 64>(a, w, st) : backward_lse<float, 64>(a, w, st);
    else s = bf ? backward_lse<__nv_bfloat16, 128>(a, w, st) : backward_lse<float, 128>(a, w, st);
    if (s != SA_OK) return s;
    if (tc) s = sa_bwd_tc_run(a, w, st);
    else if (D == 64) s = bf ? launch_simt_backward<__nv_bfloat16, 64>(a, w, st)
                             : launch_simt_backward<float, 64>(a, w, st);
    else s = bf ? launch_simt_backward<__nv_bfloat16, 128>(a, w, st)
                : launch_simt_backward<float, 128>(a, w, st);
    if (s != SA_OK) return s;
  }
  return sa_bwd_weight_grads(a, w, st);
}

sa_status sa_sum_slices(const float* part, int G, int64_t n, float* out, cudaStream_t st) {
  if (n <= 0) return SA_OK;
  if (G <= 0) {
    SA_CUDA(cudaMemsetAsync(out, 0, n * sizeof(float), st));
    return SA_OK;
  }
  SA_TIMED("sum_slices_kernel", st,
           (sum_slices_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, 4096), 256, 0, st>>>(part, G, n, out)));
  return SA_OK;
}

sa_status sa_bwd_weight_grads(const SaBwdArgs& a, const SaBwdWork& w, cudaStream_t st) {
  const int D = a.d, k = a.k;
  const int64_t n = (int64_t)k * D;
  if (a.n_total > 0 && w.chE.G > 0) {
    SA_TIMED("sum_slices_kernel", st,
             (sum_slices_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, 4096), 256, 0,
                                  st>>>(w.Epart, w.chE.G, n, w.E)));
  } else {
    SA_CUDA(cudaMemsetAsync(w.E, 0, n * sizeof(float), st));
  }
  const float rs = 1.f / sqrtf((float)D);
  sa_status s;
  // dQ = E W_K / sqrt(d)
  Gemm g1;
  g1.M = k; g1.N = D; g1.K = D;
  g1.A = w.E; g1.lda = D; g1.B = a.W_K; g1.ldb = D; g1.C = w.dQ; g1.ldc = D; g1.alpha = rs; g1.tag = "gemm:E_grads";
  if ((s = gemm(g1, st)) != SA_OK) return s;
  // dP = dQ W_Q^T
  Gemm g2;
  g2.M = k; g2.N = D; g2.K = D;
  g2.A = w.dQ; g2.lda = D; g2.B = a.W_Q; g2.ldb = D; g2.transB = true; g2.C = a.dP; g2.ldc = D;
  if (a.accumulate) { g2.Cin = a.dP; g2.ldcin = D; } g2.tag = "gemm:E_grads";
  if ((s = gemm(g2, st)) != SA_OK) return s;
  // dW_Q = P^T dQ
  Gemm g3;
  g3.M = D; g3.N = D; g3.K = k;
  g3.A = a.P; g3.lda = D; g3.transA = true; g3.B = w.dQ; g3.ldb = D; g3.C = a.dW_Q; g3.ldc = D;
  if (a.accumulate) { g3.Cin = a.dW_Q; g3.ldcin = D; } g3.tag = "gemm:E_grads";
  g3.split_k = gemm_split_for(D, D, k, kMaxSplit);
  g3.split_ws = w.gsplit;
  if ((s = gemm(g3, st)) != SA_OK) return s;
  // Q = P W_Q;  dW_K = E^T Q / sqrt(d)
  Gemm g4;
  g4.M = k; g4.N = D; g4.K = D;
  g4.A = a.P; g4.lda = D; g4.B = a.W_Q; g4.ldb = D; g4.C = w.Q; g4.ldc = D; g4.tag = "gemm:E_grads";
  if ((s = gemm(g4, st)) != SA_OK) return s;
  Gemm g5;
  g5.M = D; g5.N = D; g5.K = k;
  g5.A = w.E; g5.lda = D; g5.transA = true; g5.B = w.Q; g5.ldb = D; g5.C = a.dW_K; g5.ldc = D;
  if (a.accumulate) { g5.Cin = a.dW_K; g5.ldcin = D; } g5.tag = "gemm:E_grads";
  g5.alpha = rs;
  g5.split_k = gemm_split_for(D, D, k, kMaxSplit);
  g5.split_ws = w.gsplit;
  return gemm(g5, st);
}

}  // namespace sa
