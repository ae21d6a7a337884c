/*
 * sketch_attn.h -- C ABI of the Sketch Attention (SA) / STCA library for one
 * NVIDIA B200 (sm_100a).
 *
 * The operations are those of the SequenceO1 paper ("SequenceO1: End-to-End
 * Ultra-Long (100K) Sequence Modeling in Recommendation with Low-Rank
 * Caching"); each entry point cites the section and equation it computes.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Row-major arrays, row-vector convention (x W).
 *  - Pointers named *_host are host memory and are read during the call only;
 *    every other pointer is device memory owned by the caller.  The library
 *    allocates nothing: scratch memory is the caller's `workspace`, whose size
 *    the matching *_workspace() query returns for the current device.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Outputs are fully overwritten, never accumulated into.
 *  - Ragged users: user u owns rows [offsets[u], offsets[u+1]) of X;
 *    offsets[0] = 0, offsets non-decreasing, offsets[B] = total rows.  Both a
 *    host copy (validated, used for sizes) and a device copy (read by the
 *    kernels) are passed; they must hold the same values.
 *  - Errors are status codes.  Nothing is thrown across the ABI, nothing
 *    aborts, and no kernel traps.  sa_last_error() returns a message for the
 *    calling thread's last failing call.  Device pointers must be 16-byte
 *    aligned.
 *  - Numbers: weights and outputs are fp32.  X, STCA queries and keys are
 *    fp32 (SA_F32) or bf16 (SA_BF16).  bf16 paths multiply bf16 operands on
 *    the tensor cores with fp32 accumulation; fp32 paths use fp32 FMA.
 */
#ifndef SKETCH_ATTN_H
#define SKETCH_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,   /* bad pointer, size, offsets or alignment     */
  SA_ERR_UNSUPPORTED = 2,   /* valid but outside the supported shapes      */
  SA_ERR_CUDA = 3,          /* a CUDA runtime call failed                  */
  SA_ERR_TIMEOUT = 4,       /* a device-side wait gave up (see poll below) */
  SA_ERR_WORKSPACE = 5      /* workspace NULL or smaller than the query    */
} sa_status;

typedef enum { SA_F32 = 0, SA_BF16 = 1 } sa_dtype;

/* cudaStream_t without including the CUDA headers. */
typedef struct CUstream_st* sa_stream_t;

/* Library version (major*10000 + minor*100 + patch). */
int sa_version(void);

/* Message describing the calling thread's last non-OK status. */
const char* sa_last_error(void);

/*
 * Synchronises `stream`, then reads and clears the library's device error
 * word.  Returns SA_ERR_TIMEOUT if a kernel's bounded wait expired since the
 * last poll, SA_ERR_CUDA on a CUDA error, else SA_OK.
 */
sa_status sa_poll_device_status(sa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Sketch Attention forward                                                  */
/* ------------------------------------------------------------------------ */
/*
 * Bytes of workspace sa_forward needs for these sizes on the current device.
 */
size_t sa_forward_workspace(int B, int64_t n_total, int k, int d, sa_dtype x_dtype);

/*
 * sa_forward -- the sketch of every user (paper Sec. 3.1, eqs. (6)-(9)).
 *
 * Per user u with history X_u (n_u x d):
 *   Z   = (P W_Q)(X_u W_K)^T / sqrt(d)                    eq. (6), k x n_u
 *   A   = softmax over the k prototypes of each column    eqs. (7)-(8)
 *   H_u = A X_u                                           eq. (9)
 *   m_u = row sums of A (mass of each prototype)
 *   S_u = diag(1/(m_u + eps)) H_u W_V
 * The value projection W_V and the division by (m + eps) are this library's
 * reading; with W_V = I and eps = 0 the pages' sketch is H = S diag(m).
 * The k x n_u matrices Z and A are never written to memory.
 *
 * X        [n_total, d] x_dtype; n_total = offsets_host[B].
 * P        [k, d] fp32 prototypes; W_Q, W_K, W_V [d, d] fp32.
 * S        [B, k, d] fp32 out.   mass [B, k] fp32 out.
 * H        [B, k, d] fp32 out, optional (NULL): the unnormalised A X, which
 *          sa_backward needs.
 * S_bf16   [B, k, d] bf16 out, optional (NULL): S rounded to bf16 (for STCA).
 * lse      [n_total] fp32 out, optional (NULL): each token's log-sum-exp over
 *          the k prototypes, ln sum_j exp Z_ji (sa_backward reuses it).
 * A user with n_u = 0 gets S = 0, mass = 0, H = 0.
 * Supported: 1 <= k <= 4096, d in {64, 128}, B >= 1, eps >= 0.
 */
sa_status sa_forward(const void* X, sa_dtype x_dtype,
                     const int64_t* offsets_host, const int64_t* offsets_dev, int B,
                     int k, int d,
                     const float* P, const float* W_Q, const float* W_K, const float* W_V,
                     float eps,
                     float* S, float* mass, float* H, void* S_bf16, float* lse,
                     void* workspace, size_t ws_bytes, sa_stream_t stream);

/*
 * sa_forward_noalloc -- sa_forward for callers that cannot allocate device
 * memory (code running inside a memory pool it does not own, plugins whose
 * host forbids device allocations, work recorded once and replayed).  The
 * paper has no counterpart: this is an interface variant of sa_forward, with
 * the same inputs, outputs and results up to rounding, and no workspace.
 * Scratch lives in a fixed 8 MiB device array inside the library, held by
 * every GPU that loads it until the process exits.  The call allocates
 * nothing.
 * Limits: x_dtype = SA_BF16, d = 128, k a multiple of 128 up to 512,
 * 1 <= B <= 8; anything else returns SA_ERR_UNSUPPORTED before any GPU work.
 * With lse = NULL the per-token log-sum-exp also takes scratch (4 bytes per
 * token), which bounds n_total; pass lse to lift that bound.
 * Calls share the array: calls that overlap on the GPU (other streams, other
 * host threads) race and must be serialised.  No scratch word needs to start
 * at zero.  The first call on each device looks up the array's address, with
 * that device current; make it before any stream capture.
 */
sa_status sa_forward_noalloc(const void* X, sa_dtype x_dtype,
                             const int64_t* offsets_host, const int64_t* offsets_dev, int B,
                             int k, int d,
                             const float* P, const float* W_Q, const float* W_K,
                             const float* W_V, float eps,
                             float* S, float* mass, float* H, void* S_bf16, float* lse,
                             sa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Sketch Attention backward                                                 */
/* ------------------------------------------------------------------------ */
size_t sa_backward_workspace(int B, int64_t n_total, int k, int d, sa_dtype x_dtype);

/*
 * sa_backward -- gradients of L = sum_u <dS_u, S_u> + <dmass_u, m_u> through
 * sa_forward (the pages call SA fully differentiable, Sec. 3.1, and print no
 * backward; these are the chain-rule derivatives of the forward above):
 *   Hh = H/(m+eps); dW_V = sum_u Hh^T dS; dHh = dS W_V^T
 *   dH = dHh/(m+eps); dm = -(dHh . Hh)/(m+eps) + dmass
 *   dA_ji = dH_j . x_i + dm_j;  c_i = sum_j A_ji dA_ji;  dZ = A o (dA - c)
 *   dX_i = sum_j A_ji dH_j + sum_j dZ_ji p'_j,  p'_j = row j of P W_Q W_K^T / sqrt(d)
 *   E = sum_u dZ_u X_u;  dP = E W_K W_Q^T/sqrt(d);  dW_Q = P^T E W_K/sqrt(d);
 *   dW_K = E^T P W_Q/sqrt(d)
 *
 * Inputs as sa_forward, plus H and mass from sa_forward, dS [B,k,d] fp32,
 * dmass [B,k] fp32 (NULL = zero) and lse [n_total] from sa_forward (NULL = the
 * backward recomputes it).
 * dX [n_total, d] x_dtype out; dP [k,d], dW_Q, dW_K, dW_V [d,d] fp32 out
 * (sums over the batch).
 */
sa_status sa_backward(const void* X, sa_dtype x_dtype,
                      const int64_t* offsets_host, const int64_t* offsets_dev, int B,
                      int k, int d,
                      const float* P, const float* W_Q, const float* W_K, const float* W_V,
                      float eps,
                      const float* H, const float* mass, const float* dS, const float* dmass,
                      const float* lse, void* dX, float* dP, float* dW_Q, float* dW_K, float* dW_V,
                      void* workspace, size_t ws_bytes, sa_stream_t stream);

/*
 * sa_backward_accumulate -- sa_backward that adds the weight gradients into
 * dP, dW_Q, dW_K and dW_V instead of overwriting them (dX is written as in
 * sa_backward).  The weights are shared by all users, so their gradients over
 * a batch are the sum over any split of its users into groups: call it once
 * per group (e.g. to overlap the next group's host-to-device copy with this
 * group's work) after zeroing or a first sa_backward.  Same arguments, layouts
 * and errors as sa_backward; no counterpart in the paper (an interface form).
 */
sa_status sa_backward_accumulate(const void* X, sa_dtype x_dtype, const int64_t* offsets_host,
                                 const int64_t* offsets_dev, int B, int k, int d, const float* P,
                                 const float* W_Q, const float* W_K, const float* W_V, float eps,
                                 const float* H, const float* mass, const float* dS,
                                 const float* dmass, const float* lse, void* dX, float* dP,
                                 float* dW_Q, float* dW_K, float* dW_V, void* workspace,
                                 size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Token-wise normalisation variant                                          */
/* ------------------------------------------------------------------------ */

size_t sa_forward_tokenwise_workspace(int B, int64_t n_total, int k, int d, sa_dtype x_dtype);

/*
 * sa_forward_tokenwise -- the "vanilla attention" baseline the paper compares
 * SA with (Sec. 7.1, Table 1; Sec. 2's latent-query, token-wise softmax): the
 * affinities of eq. (6), normalised over each prototype's tokens instead of
 * over each token's prototypes:
 *   A_{j,i} = exp S_{j,i} / sum_{i' of user u} exp S_{j,i'},  H = A X_u,
 *   m_j = sum_i A_{j,i} (1 for a user with events, 0 without),
 *   S = diag(1/(m+eps)) H W_V  (the same output step as sa_forward).
 * Arguments, layouts and ownership as sa_forward (no lse output).  bf16 X and
 * d = 128 only (else SA_ERR_UNSUPPORTED); any k >= 1.  Asynchronous on stream.
 */
sa_status sa_forward_tokenwise(const void* X, sa_dtype x_dtype, const int64_t* offsets_host,
                               const int64_t* offsets_dev, int B, int k, int d, const float* P,
                               const float* W_Q, const float* W_K, const float* W_V, float eps,
                               float* S, float* mass, float* H, void* S_bf16, void* workspace,
                               size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Stacked refinement                                                        */
/* ------------------------------------------------------------------------ */

/* One refinement iteration's parameters (device pointers, fp32, row-major). */
typedef struct {
  const float* W_Q;     /* [d, d]  eq. (12) */
  const float* W_K;     /* [d, d]  eq. (12) */
  const float* ln1_g;   /* [d] gain of the LN of eq. (15), or NULL for ones */
  const float* ln1_b;   /* [d] bias of that LN, or NULL for zeros */
  const float* W1;      /* [d, 2d] SwiGLU FFN of eq. (16): the SiLU-gated branch */
  const float* W3;      /* [d, 2d] the linear branch */
  const float* W2;      /* [2d, d] the output projection */
  const float* ln2_g;   /* [d] gain of the LN of eq. (16), or NULL for ones */
  const float* ln2_b;   /* [d] bias of that LN, or NULL for zeros */
} sa_refine_layer;

size_t sa_refine_workspace(int B, int64_t n_total, int k, int d, sa_dtype x_dtype);

/*
 * sa_refine_forward -- stacked SA refinement (paper Sec. 3.3, eqs. (12)-(16)),
 * n_iter iterations starting from the shared prototypes X~(0) = P0 [k, d]:
 *   A     = softmax over prototypes of (X~ W_Q)(X_u W_K)^T / sqrt(d)   (12)-(13)
 *   X^    = A X_u                     (14, the sum over the user's events)
 *   Xbar  = LN(X~ + X^)               (15)
 *   X~    = LN(Xbar + FFN(Xbar)),  FFN(y) = (SiLU(y W1) * (y W3)) W2   (16)
 * From the second iteration on the prototypes X~ are per user.  LN normalises
 * each row over d (mean, biased variance, ln_eps), then applies gain and bias.
 * Output: sketch [B, k, d] fp32 = X~(n_iter).  X, offsets as in sa_forward;
 * layers: host array of n_iter structs.  Tensor-core path only: x_dtype =
 * SA_BF16, d = 128, k a multiple of 128 (else SA_ERR_UNSUPPORTED).  The
 * caller owns every buffer; asynchronous on `stream`.
 */
sa_status sa_refine_forward(const void* X, sa_dtype x_dtype, const int64_t* offsets_host,
                            const int64_t* offsets_dev, int B, int k, int d, const float* P0,
                            int n_iter, const sa_refine_layer* layers, float ln_eps,
                            float* sketch, void* workspace, size_t ws_bytes,
                            sa_stream_t stream);

/* Gradients of one refinement iteration's parameters (fp32 device buffers shaped as
 * the parameters; written, not accumulated; sums over the users).  A gradient whose
 * parameter is NULL in the layer is not written (its pointer may be NULL). */
typedef struct {
  float* dW_Q;
  float* dW_K;
  float* dln1_g;
  float* dln1_b;
  float* dW1;
  float* dW3;
  float* dW2;
  float* dln2_g;
  float* dln2_b;
} sa_refine_layer_grad;

size_t sa_refine_backward_workspace(int B, int64_t n_total, int k, int d, int n_iter, sa_dtype x_dtype);

/*
 * sa_refine_backward -- the backward of sa_refine_forward (paper Sec. 3.3, eqs.
 * (12)-(16), trained end to end): given dsketch [B, k, d] fp32, the gradient of
 * the returned sketch, writes
 *   dX   [n_total, d] fp32: the gradient with respect to the events' rows;
 *   dP0  [k, d] fp32: the gradient with respect to the shared prototypes;
 *   grads[i]: the gradients of iteration i's parameters.
 * Inputs as sa_refine_forward (bf16 X, d = 128, k a multiple of 128 up to 4096,
 * n_iter <= 8).  The forward is recomputed with its intermediates kept in the
 * workspace.  Per iteration, from the last: the LayerNorm and SwiGLU backward
 * (the FFN products on the tensor cores over hi + lo bf16 splits), then the SA
 * backward of X^ = A X_u with every user's own prototypes (the tensor-core
 * kernels of sa_backward, run user by user, dX accumulated in fp32): dA = dX^ . x,
 * c = sum_j A dA, dZ = A (dA - c), dX += A dX^ + dZ (X~ W_Q W_K^T)/sqrt(d),
 * E_u = dZ^T X_u, dX~ += E_u W_K W_Q^T / sqrt(d), and the W_Q, W_K gradients
 * summed over users.  Workspace: sa_refine_backward_workspace bytes, 16-byte
 * aligned, caller owned.  Asynchronous on `stream`.
 */
sa_status sa_refine_backward(const void* X, sa_dtype x_dtype, const int64_t* offsets_host,
                             const int64_t* offsets_dev, int B, int k, int d, const float* P0,
                             int n_iter, const sa_refine_layer* layers, float ln_eps,
                             const float* dsketch, float* dX, float* dP0,
                             const sa_refine_layer_grad* grads, void* workspace, size_t ws_bytes,
                             sa_stream_t stream);

/*
 * sa_gather_events -- the events' input rows on the device: for i < n
 *   X[i] = item_table[item_ids[i]] + action_table[action_ids[i]]
 * (an item embedding plus the embedding of the feedback type, the workloads'
 * events; paper Sec. 3.6, the plain sum next to eq. (20)'s fused rows of
 * sa_gather_events_fused), so that a step ships 5 bytes of ids per event
 * instead of its row.
 * item_table [vocab, d] and action_table [n_actions, d] bf16, 16-byte aligned;
 * item_ids int32 [n] (4-byte aligned), action_ids uint8 [n]; X [n, d] bf16 out.
 * The sum is formed in fp32 and rounded to nearest even.  d a multiple of 8.
 * An id outside its table gives a zero row and makes the next
 * sa_poll_device_status return SA_ERR_INVALID_ARG (no out-of-bounds read).
 */
sa_status sa_gather_events(const void* item_table, int64_t vocab, const void* action_table,
                           int n_actions, const int32_t* item_ids, const uint8_t* action_ids,
                           int64_t n, int d, void* X, sa_stream_t stream);

size_t sa_gather_events_fused_workspace(int n_actions, int d, int d_ff);

/*
 * sa_gather_events_fused -- the events' input rows with the action-side SwiGLU
 * fusion (paper Sec. 3.6 / App. D, eq. (20)): for i < n, with
 * e = item_table[item_ids[i]], a = action_table[action_ids[i]] and z = [e ; a],
 *   X[i] = e + (SiLU(z W1) * (z W3)) W2
 * W1, W3 [2d, d_ff] and W2 [d_ff, d] fp32 row-major device arrays (no biases);
 * the FFN maps the 2d-wide concatenation back to width d for the residual.
 * d = 128, d_ff = 256 and 1..16 action types (else SA_ERR_UNSUPPORTED).
 * Tables bf16, ids as in sa_gather_events, X [n, d] bf16 out (rounded once to
 * nearest even).  The tensor-core products take fp16 operands (the weights,
 * e and the inner activations), fp32 accumulation; the action half of the
 * first layer is computed once per action type into the workspace.
 * Workspace: sa_gather_events_fused_workspace bytes, 16-byte aligned, caller
 * owned.  An id or action type outside its table gives a zero row and makes
 * the next sa_poll_device_status return SA_ERR_INVALID_ARG.
 */
sa_status sa_gather_events_fused(const void* item_table, int64_t vocab, const void* action_table,
                                 int n_actions, const int32_t* item_ids, const uint8_t* action_ids,
                                 int64_t n, int d, const float* W1, const float* W3, const float* W2,
                                 int d_ff, void* X, void* workspace, size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* STCA: stacked target-to-history single-query cross attention             */
/* ------------------------------------------------------------------------ */
/* Weights of one STCA layer (device pointers). */
typedef struct {
  const float* W_Q;   /* [heads, D, d_h] */
  const float* W_K;   /* [heads, D, d_h] */
  const float* W_V;   /* [heads, D, d_h] */
  const float* W_O;   /* [heads*d_h, D], or NULL for the identity (needs heads*d_h == D) */
} stca_layer;

size_t stca_forward_workspace(int B, int64_t C_total, int D, int heads, int d_h, sa_dtype dtype);

/*
 * stca_forward -- one STCA branch over a batch of users (paper Sec. 2.3
 * eq. (4), evaluated in the single-query reordering of Sec. 5.1 eq. (24)).
 * For every candidate query q of user u and every layer:
 *   for each head h:  u_h = (q W_Q^h) W_K^h^T
 *                     alpha = softmax_i(u_h . x_i / sqrt(d_h)),  i in [kv_begin[u], kv_end[u])
 *                     o_h = (sum_i alpha_i x_i) W_V^h
 *   q <- q + concat_h(o_h) W_O
 * Keys and values are the raw history rows x_i.  An empty key range gives
 * o = 0.  The recent branch passes the last L_r events of each history
 * (eq. 3); the sketch branch passes the sketches (eq. 19).
 *
 * q       [C_total, D] dtype: candidate targets, user u owns rows
 *         [cand_offsets[u], cand_offsets[u+1]).
 * kv      [kv_rows, D] dtype; 0 <= kv_begin[u] <= kv_end[u] <= kv_rows.
 * layers  host array of n_layers weight sets (device pointers inside).
 * out     [C_total, D] fp32: the query after the last layer.
 * Supported: D == 128, heads*d_h <= 4096, n_layers >= 1.
 */
sa_status stca_forward(const void* q, sa_dtype dtype,
                       const int64_t* cand_offsets_host, const int64_t* cand_offsets_dev, int B,
                       const void* kv, int64_t kv_rows,
                       const int64_t* kv_begin_host, const int64_t* kv_end_host,
                       const int64_t* kv_begin_dev, const int64_t* kv_end_dev,
                       int D, int heads, int d_h, int n_layers, const stca_layer* layers,
                       float* out, void* workspace, size_t ws_bytes, sa_stream_t stream);

/*
 * The full STCA layer (paper Sec. 5.1, eqs. (26)-(28)): the attention layer
 * above plus two SwiGLU FFNs of inner width 2D (no biases, SiLU(x) =
 * x / (1 + e^-x) on the first branch), each with a residual add:
 *   history side (eq. (27)), before the layer's attention, on every key row:
 *       x <- x + (SiLU(x hist_W1) * (x hist_W3)) hist_W2
 *     the transformed rows are this layer's keys and values and the input of
 *     the next layer's history FFN (the transform is target-independent, so
 *     it runs once per key row, not once per candidate);
 *   query side (eq. (26)), after the W_O residual:
 *       q <- q + (SiLU(q q_W1) * (q q_W3)) q_W2
 * hist_W1, hist_W3, q_W1, q_W3 [D, 2D]; hist_W2, q_W2 [2D, D]; fp32 device
 * pointers.  Each FFN is either fully given or fully NULL (absent).
 */
typedef struct {
  stca_layer attn;
  const float* hist_W1;
  const float* hist_W3;
  const float* hist_W2;
  const float* q_W1;
  const float* q_W3;
  const float* q_W2;
} stca_full_layer;

/* kv_total = sum over users of kv_end[u] - kv_begin[u] (the key rows the
 * history FFNs transform; a range shared by two users counts twice). */
size_t stca_forward_full_workspace(int B, int64_t C_total, int64_t kv_total, int D, int heads,
                                   int d_h, sa_dtype dtype);

/*
 * stca_forward_full -- one STCA branch of full layers.  Arguments as in
 * stca_forward; layers is a host array of n_layers stca_full_layer.  The
 * key rows are copied into the workspace (each user's range, in user order)
 * before the first history FFN, so kv is only read.  With dtype SA_BF16 the
 * transformed rows are kept in bf16 (they are the attention's keys) and the
 * history FFN runs on the tensor cores with bf16 weights and fp32
 * accumulation; with SA_F32 everything is fp32.  The query FFN is fp32.
 * Errors: as stca_forward, and SA_ERR_INVALID_ARG for a partly given FFN.
 */
sa_status stca_forward_full(const void* q, sa_dtype dtype,
                            const int64_t* cand_offsets_host, const int64_t* cand_offsets_dev,
                            int B, const void* kv, int64_t kv_rows,
                            const int64_t* kv_begin_host, const int64_t* kv_end_host,
                            const int64_t* kv_begin_dev, const int64_t* kv_end_dev,
                            int D, int heads, int d_h, int n_layers,
                            const stca_full_layer* layers, float* out, void* workspace,
                            size_t ws_bytes, sa_stream_t stream);

/* Gradients of one full STCA layer's weights (fp32 device buffers, shaped as the
 * weights; written, not accumulated).  dW_O is ignored when the layer's W_O is NULL,
 * and an absent FFN's gradients are ignored. */
typedef struct {
  float* dW_Q;
  float* dW_K;
  float* dW_V;
  float* dW_O;
  float* hist_dW1;
  float* hist_dW3;
  float* hist_dW2;
  float* q_dW1;
  float* q_dW3;
  float* q_dW2;
} stca_full_layer_grad;

/* Workspace of stca_backward_full; the host offsets are those of the call. */
size_t stca_backward_full_workspace(int B, const int64_t* cand_offsets_host,
                                    const int64_t* kv_begin_host, const int64_t* kv_end_host,
                                    int D, int heads, int d_h, int n_layers, sa_dtype dtype);

/*
 * stca_backward_full -- the backward of stca_forward_full: given dout [C_total, D]
 * fp32, the gradient of the branch output, writes
 *   dq   [C_total, D] fp32 (or NULL): the gradient with respect to q;
 *   dkv  [kv_rows, D] fp32 (or NULL): the gradient with respect to kv (a row in no
 *        user's range gets 0; a row in several ranges sums their gradients);
 *   grads[l]: every weight gradient of layer l.
 * Inputs as stca_forward_full.  The layers are recomputed in fp32 (bf16 inputs are
 * widened, not rounded further) and each user's attention is evaluated with its
 * C_u*heads x L_u score matrix in the workspace, so the workspace grows with the
 * largest user.  With SA_BF16 inputs the attention products run on the tensor
 * cores with each fp32 operand split into two bf16 parts (hi + lo, about 16
 * significant bits; three MMA passes per product), with SA_F32 inputs on fp32
 * CUDA cores.  Deterministic: users are processed in order and split-K partial
 * sums are added in a fixed order.
 * Errors: as stca_forward_full, and SA_ERR_INVALID_ARG for a NULL gradient buffer
 * of a weight that is present.
 */
sa_status stca_backward_full(const void* q, sa_dtype dtype,
                             const int64_t* cand_offsets_host, const int64_t* cand_offsets_dev,
                             int B, const void* kv, int64_t kv_rows,
                             const int64_t* kv_begin_host, const int64_t* kv_end_host,
                             const int64_t* kv_begin_dev, const int64_t* kv_end_dev,
                             int D, int heads, int d_h, int n_layers,
                             const stca_full_layer* layers, const float* dout, float* dq,
                             float* dkv, const stca_full_layer_grad* grads, void* workspace,
                             size_t ws_bytes, sa_stream_t stream);

/*
 * stca_fuse -- linear fusion of the two branches (paper Sec. 3.4 leaves the
 * fusion to a light MLP or gate; this library applies one linear layer):
 *   out = [z_r ; z_u] W_F + b_F
 * z_r, z_u [C, D] fp32; W_F [2D, D] fp32; b_F [D] fp32 or NULL; out [C, D].
 */
sa_status stca_fuse(const float* z_r, const float* z_u, const float* W_F, const float* b_F,
                    int64_t C, int D, float* out, sa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Measurement support (not part of the method)                              */
/* ------------------------------------------------------------------------ */
/*
 * Exponentials per second on the current GPU (all SMs, synchronous): mode 0 with
 * every 2^x on the MUFU (ex2.approx), mode 1 with the SA forward kernels' mix
 * (one pair in eight by a cubic on the FMA pipe).  The co-roofline of the
 * forward: each of its two kernels evaluates k exponentials per token.
 */
sa_status sa_measure_exp2_rate(int mode, double* per_second, sa_stream_t stream);

/*
 * Self-test of the device-side failure path (no fault): launches one thread that
 * waits on an mbarrier nothing arrives at, with the bounded wait every kernel of
 * the library uses, for about budget_cycles SM clocks (1 .. 4e9).  On expiry the
 * wait sets the device error word and the kernel returns, so the next
 * sa_poll_device_status returns SA_ERR_TIMEOUT and the context stays usable.
 */
sa_status sa_selftest_bounded_wait(long long budget_cycles, sa_stream_t stream);

/* Number of kernels this library has launched in this process. */
long long sa_launch_count(void);

/*
 * enable = 1 clears the kernel timers and starts recording a CUDA event pair
 * on the launch stream around each launch of the library's kernels; 0 stops.
 * Costs one event record per launch boundary; results are read below.
 */
sa_status sa_profile(int enable);

/*
 * Per-kernel device time since sa_profile(1), summed from the event pairs
 * (synchronises on them).  Fills entry i (0-based) and returns 1, or returns
 * 0 when i is past the last kernel.  `name` receives at most name_len bytes.
 */
int sa_profile_read(int i, char* name, int name_len, double* total_ms, long long* launches);

#ifdef __cplusplus
}
#endif

#endif /* SKETCH_ATTN_H */
