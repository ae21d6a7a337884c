// Internal interfaces of the STCA kernels.
#pragma once
#include "common.cuh"
#include "gemm.cuh"

namespace sa {

struct StcaArgs {
  const void* q; sa_dtype dtype;
  const int64_t* cand_dev; int B; int64_t C_total;
  const void* kv; int64_t kv_rows;
  const int64_t* kvb_dev; const int64_t* kve_dev;
  int D, heads, d_h, n_layers;
  const stca_layer* layers;   // host array
  float* out;
  int64_t max_rows_per_user;  // max over users of C_u * heads (host-computed)
  // bf16 dtype only: kv rows (and the attention's query operand) are fp16 rather than
  // bf16 (the full layer's transformed key rows, computed values kept to 11 bits)
  bool kv_f16 = false;
};

struct StcaWork {
  float* Qh;           // [C, heads*d_h]
  float* U;            // [C*heads, D]   fp32 (CUDA-core attention)
  __nv_bfloat16* Ub;   // [C*heads, D]   bf16 or, with kv_f16, fp16 (tensor-core attention)
  float* Y;            // [C*heads, D]
  float* O;            // [C, heads*d_h]
  int* tile_prefix;    // [B+1]
  int max_tiles;       // upper bound on the number of query tiles
  // tensor-core projections (bf16 inputs): the heads' folded weights
  //   M = [W_Q^h W_K^h^T log2(e)/sqrt(d_h)]_h  [D, heads*D]  and  N = [W_V^h W_O^h]_h  [heads*D, D]
  // and hi + lo bf16 splits of them, of the query state q [C, D] and of Y [C, heads*D]
  __nv_bfloat16 *Mhi, *Mlo, *Nhi, *Nlo, *qhi, *qlo, *Yhi, *Ylo;
  float* part;         // split-K partials of the output projection
  size_t part_floats;
};

// Carves the attention part of an STCA workspace (B users, C candidates) from c.
StcaWork stca_attn_carve(Carve& c, int B, int64_t C, int D, int heads, int d_h);

sa_status stca_run(const StcaArgs& a, const StcaWork& w, cudaStream_t st);
// The two halves of stca_run: q -> out (fp32) and the query-tile prefix, then
// one attention layer (projections, attention over a.kv, W_O, residual).
// With bf16 inputs stca_begin also writes q's hi + lo split (w.qhi, w.qlo); a layer reads
// that split when q_split is true (else it splits q itself) and, with split_out, has its
// output projection write the split of the new q for the next layer.
sa_status stca_begin(const StcaArgs& a, const StcaWork& w, cudaStream_t st);
sa_status stca_attend_layer(const StcaArgs& a, const stca_layer& L, const StcaWork& w, cudaStream_t st,
                            bool q_split = false, bool split_out = false);

// Full STCA layers (history- and query-side SwiGLU FFNs).
struct StcaFullWork {
  StcaWork attn;
  void* Hk;                 // [kv_total, D] key rows (fp32 inputs: fp32; bf16 inputs: fp16), transformed in place
  int64_t* kpre;            // [B+1] start of each user's rows in Hk
  float* G1; float* G3; float* U;   // [max(C, rows of an fp32 history FFN), 2D] fp32
  __half* W13t;             // [4 * 128, D] fp16: the tensor-core FFN's first-layer weights
  __half* W2t;              // [D, 2D] fp16: its second-layer weights (transposed)
};
size_t stca_full_layout(void* base, int B, int64_t C, int64_t kv_total, int D, int heads, int d_h,
                        sa_dtype dtype, StcaFullWork* w);
sa_status stca_full_run(const StcaArgs& a, const stca_full_layer* layers, int64_t kv_total,
                        const StcaFullWork& w, cudaStream_t st);

// bf16 tensor-core GEMM: C[M, N] = alpha A B (+ Cin), fp32 out.  A is K-major
// (A[m lda + k]) or, with a_mn, M-major (A[k lda + m]); B is K-major (B[n ldb + k])
// or, with b_mn, N-major (B[k ldb + n]).  lda, ldb multiples of 8; A, B 16-byte aligned.
struct TcGemm {
  int M = 0, N = 0, K = 0;
  const __nv_bfloat16* A = nullptr; int64_t lda = 0; bool a_mn = false;
  const __nv_bfloat16* B = nullptr; int64_t ldb = 0; bool b_mn = false;
  const __nv_bfloat16* A_lo = nullptr;     // optional lo parts of split operands (same layout)
  const __nv_bfloat16* B_lo = nullptr;
  float* part = nullptr;                   // optional split-K workspace of part_floats floats
  size_t part_floats = 0;
  float* C = nullptr; int64_t ldc = 0;   // fp32 output (may be NULL when C16 is given)
  const float* Cin = nullptr; int64_t ldcin = 0;
  float alpha = 1.f;
  // optional 16-bit copy of the output: bf16, or (c16_half) fp16 with |v| > 65504 flagged
  // in the device status word
  __nv_bfloat16* C16 = nullptr; int64_t ldc16 = 0; bool c16_half = false;
  // optional hi + lo bf16 split of the output (the operand of a following split GEMM)
  __nv_bfloat16* Chi = nullptr; __nv_bfloat16* Clo = nullptr; int64_t ldcs = 0;
  const char* tag = nullptr;
  int min_split_slices = 8;   // split K only while every split keeps this many 64-deep K slices
};
sa_status tc_gemm(const TcGemm& g, cudaStream_t st);
// Backward of y = x + (SiLU(x W1) * (x W3)) W2 (inner width 2D) over `rows` fp32 rows on the
// tensor cores with hi + lo split operands: dx = dy + the FFN's input gradient (dx may alias
// dy), dW1, dW3 [D, 2D] and dW2 [2D, D] overwritten.
struct FfnBwdScratch {
  float *G1, *G3, *U, *dU, *split;
  __nv_bfloat16 *x_hi, *x_lo, *a_hi, *a_lo, *b_hi, *b_lo, *w_hi, *w_lo;
};
FfnBwdScratch ffn_bwd_scratch_carve(Carve& c, int64_t rows, int D);
sa_status ffn_residual_backward_tc(const float* x, int64_t rows, int D, const float* W1, const float* W3,
                                   const float* W2, const float* dy, float* dx, float* dW1, float* dW3, float* dW2,
                                   const FfnBwdScratch& f, cudaStream_t st);
// x = hi + lo: hi = bf16(x), lo = bf16(x - hi), for n fp32 values
sa_status split_hi_lo(const float* x, int64_t n, __nv_bfloat16* hi, __nv_bfloat16* lo, cudaStream_t st);

// Backward of a branch of full layers (fp32, GEMM-based).
struct StcaBwdShape {
  int64_t C, kv_total, max_rows_x_keys;   // max over users of C_u * heads * pitch(kv_end - kv_begin)
  int D, heads, d_h, n_layers;
  sa_dtype dtype;
};
// row pitch of a user's score matrix: its key count rounded up to 8 (16-byte rows in bf16)
inline int64_t score_pitch(int64_t keys) { return (keys + 7) / 8 * 8; }
struct StcaBwdHost {                      // host copies of the offsets, read while issuing
  const int64_t* cand;                    // [B+1]
  const int64_t* kv_begin;                // [B]
  const int64_t* kv_end;                  // [B]
  const int64_t* kpre;                    // [B+1] start of each user's rows among the gathered rows
  int64_t kv_total;
};
struct StcaBwdWork {
  float *qin, *qmid, *Qh, *U, *Y, *O;     // per layer (qin: n_layers + 1 states)
  float* Xk;                              // [n_layers + 1, kv_total, D] key-row states
  float *G1, *G3, *Uf, *dUf;              // [max(C, kv_total), 2D]
  float *S, *dS;                          // one user's score matrix and its gradient
  float *dq, *dqmid, *dO, *dY, *dU, *dQh, *dX;
  float* gsplit;                          // split-K partials of the GEMMs with small outputs
  // bf16 operands of the tensor-core attention products (bf16 inputs only)
  __nv_bfloat16 *Ub, *Ulo, *Xkb, *Xklo, *dYb, *dYlo, *Pb, *Plo, *dSb, *dSlo;
  __nv_bfloat16 *fx_hi, *fx_lo, *fa_hi, *fa_lo, *fb_hi, *fb_lo, *fw_hi, *fw_lo;   // FFN operand splits
};
constexpr size_t kStcaBwdSplitFloats = (size_t)16 << 20;
size_t stca_bwd_layout(void* base, const StcaBwdShape& sh, StcaBwdWork* w);
sa_status stca_backward_run(const StcaArgs& a, const StcaBwdHost& hst, const stca_full_layer* layers,
                            const stca_full_layer_grad* grads, const float* dout, float* dq_out, float* dkv,
                            const StcaBwdWork& w, cudaStream_t st);

// x <- x + (SiLU(x W1) * (x W3)) W2 for rows of fp16 x, D = 128, in place, on
// the tensor cores; W13t / W2t (fp16) as prepared by stca_ffn_weights_f16.
sa_status stca_ffn_weights_f16(const float* W1, const float* W3, const float* W2, __half* W13t, __half* W2t,
                               cudaStream_t st);
sa_status stca_hist_ffn_tc(__half* X, int64_t rows, const __half* W13t, const __half* W2t, cudaStream_t st);

// Event rows with the action-side SwiGLU fusion (eq. (20)), d = 128, inner width 256:
// X[i] = bf16(e + (SiLU(z W1) * (z W3)) W2), e = item[ids[i]], z = [e; action[acts[i]]];
// W1, W3 [2d, 2d], W2 [2d, d] fp32.  Workspace: the fp16 weights and the per-action bias.
struct EventsFfnWork {
  __half* W13t;
  __half* W2t;
  float* cb;   // [n_actions, 512]
};
size_t events_ffn_layout(void* base, int n_actions, EventsFfnWork* w);
sa_status events_ffn_run(const __nv_bfloat16* item, int64_t vocab, const __nv_bfloat16* action, int n_actions,
                         const int32_t* ids, const uint8_t* acts, int64_t n, const float* W1, const float* W3,
                         const float* W2, __nv_bfloat16* X, const EventsFfnWork& w, cudaStream_t st);

bool stca_tc_supported(sa_dtype dtype, int D);
// Y = attention over each user's keys into w.Y (fp32), or (split_y) into w.Yhi / w.Ylo
sa_status stca_tc_attention(const StcaArgs& a, const StcaWork& w, cudaStream_t st, bool split_y = false);

}  // namespace sa
