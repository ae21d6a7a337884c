"""Plain, slow fp64 CPU oracle for Sketch Attention (SA) and STCA.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this package.  The product path (the
C-ABI library and its Python binding) never calls it, and it shares no code
with the CUDA kernels: it reads plain arrays and writes plain arrays.

Citations name the SequenceO1 paper ("SequenceO1: End-to-End Ultra-Long
(100K) Sequence Modeling in Recommendation with Low-Rank Caching"), as given
by its reading-note page (equations (1)-(36)) and its arXiv HTML text, by
section and equation number.

Readings where the pages leave a step open (each is an explicit choice):
* SA value projection and per-prototype normalisation: the pages aggregate
  raw X (eq. 9).  Here S = diag(1/(m+eps)) (A X) W_V with m_j = sum_i A_ji;
  H = A X (the pages' X-tilde) is returned as well.  A prototype whose
  m_j + eps is zero (eps = 0 and no mass) gets S_j = 0.
* Softmax stabiliser: the per-token maximum over prototypes is subtracted
  (Sec. 4.4 asks FlashSA for a numerically stable softmax); the result is unchanged.
* STCA layer body: attention, optional output projection W_O, residual add
  to the query (eq. 4 plus the W_O term of eq. 26), no LayerNorm.  The full
  layer of eqs. (26)-(28) adds two optional SwiGLU FFNs of inner width 2D
  (no biases, SiLU on the first branch), each with a residual add:
  - on the history, before the layer's attention: X <- X + FFN_h(X), a
    per-row, target-independent transform (eq. (27)); the transformed rows
    are the keys and values of this layer and the input of the next layer's
    history FFN;
  - on the query, after the W_O residual: q <- q + FFN_q(q) (eq. (26)).
* STCA over an empty key range: the attention output is zero.
* Fusion: a linear map [z_r; z_u] W_F + b_F (Sec. 3.4 leaves the fusion open).
* Stacked refinement (Sec. 3.3): X^ = A X exactly as eq. (14) writes it (the
  sum over the user's events, no mass normalisation); LN is a row LayerNorm
  over d with biased variance, eps and an optional gain and bias; the FFN is
  SwiGLU with inner width 2d and no biases (eq. (23) counts 6 T w w_f FLOPs
  with w_f = 2w), SiLU on the first branch.  A user without events gets
  X^ = 0.

Parity pins (tests/test_oracle_*.py): per-token column sums, total mass,
permutation invariance, k = 1 mean, uniform assignment at zero logits,
identical tokens, a two-prototype closed form that fixes the 1/sqrt(d) scale
and the operand order, central finite differences for every gradient, STCA at
L = 1, identical keys, torch SDPA in fp64, the eq. (24) reordering, and the
analytic FLOP numbers the pages print; for the full STCA layer, torch's SiLU
and SDPA in fp64, key-permutation invariance, the layer chaining of the
history FFN and the reordering with both FFNs.  No function here is "parity
unpinned".
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "sa_forward", "sa_user", "sa_backward", "stca_branch", "stca_branch_reordered",
    "stca_fuse", "assignment", "token_lse", "layer_norm", "swiglu_ffn", "sa_refine_user",
    "sa_refine", "tokenwise_user", "sa_forward_tokenwise", "stca_branch_grads", "event_rows",
]


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def assignment(Xu, P, W_Q, W_K) -> np.ndarray:
    """A in R^{k x n}: prototype-wise softmax of the affinities.

    Affinities S = (P W_Q)(X W_K)^T / sqrt(d)            -- Sec. 3.1, eq. (6)
    A_{j,i} = exp S_{j,i} / sum_j' exp S_{j',i}           -- eqs. (7)-(8)
    so each token's column of A sums to one over the k prototypes.
    """
    Xu, P, W_Q, W_K = _f64(Xu), _f64(P), _f64(W_Q), _f64(W_K)
    d = P.shape[1]
    Q = P @ W_Q                       # k x d
    K = Xu @ W_K                      # n x d
    Z = (Q @ K.T) / math.sqrt(d)      # k x n, eq. (6)
    Zc = Z - Z.max(axis=0, keepdims=True)
    E = np.exp(Zc)
    return E / E.sum(axis=0, keepdims=True)   # softmax over prototypes, eq. (8)


def token_lse(Xu, P, W_Q, W_K) -> np.ndarray:
    """Each token's log-sum-exp over the prototypes, ln sum_j exp S_{j,i}: the
    normaliser of the prototype-wise softmax (eqs. (6)-(8))."""
    Xu, P, W_Q, W_K = _f64(Xu), _f64(P), _f64(W_Q), _f64(W_K)
    d = P.shape[1]
    Z = ((P @ W_Q) @ (Xu @ W_K).T) / math.sqrt(d)
    zmax = Z.max(axis=0)
    return zmax + np.log(np.exp(Z - zmax[None, :]).sum(axis=0))


def sa_user(Xu, P, W_Q, W_K, W_V, eps: float):
    """One user's sketch.  Returns (S, m, H) with
    H = A X (eq. 9), m_j = sum_i A_{j,i}, S = diag(1/(m+eps)) H W_V."""
    Xu = _f64(Xu)
    k, d = np.shape(P)
    if Xu.shape[0] == 0:
        return np.zeros((k, d)), np.zeros(k), np.zeros((k, d))
    A = assignment(Xu, P, W_Q, W_K)
    m = A.sum(axis=1)
    H = A @ Xu                                  # eq. (9)
    denom = (m + eps)[:, None]
    Hh = np.divide(H, denom, out=np.zeros_like(H), where=denom > 0)   # empty prototype -> 0
    S = Hh @ _f64(W_V)
    return S, m, H


def sa_forward(X, offsets: Sequence[int], P, W_Q, W_K, W_V, eps: float):
    """Sketches of a ragged batch: users own rows [offsets[u], offsets[u+1]).

    Returns S [B,k,d], mass [B,k], H [B,k,d] in fp64.
    """
    offsets = np.asarray(offsets, np.int64)
    B = len(offsets) - 1
    k, d = np.shape(P)
    S = np.zeros((B, k, d))
    mass = np.zeros((B, k))
    H = np.zeros((B, k, d))
    for u in range(B):
        S[u], mass[u], H[u] = sa_user(X[offsets[u]:offsets[u + 1]], P, W_Q, W_K, W_V, eps)
    return S, mass, H


def sa_backward(X, offsets, P, W_Q, W_K, W_V, eps: float, dS, dmass=None):
    """Gradients of sum_u <dS_u, S_u> + <dmass_u, m_u> with respect to
    X, P, W_Q, W_K, W_V (weights are shared, so their gradients sum over users).

    The pages state that SA is differentiable end to end (Sec. 3.1) but print
    no backward; these are the chain-rule derivatives of the forward above,
    written out step by step:
        Hh = H/(m+eps),  dW_V += Hh^T G,  dHh = G W_V^T
        dH_j = dHh_j/(m_j+eps),  dm_j = -(dHh_j . H_j)/(m_j+eps)^2 + dmass_j
        dA_ji = dH_j . x_i + dm_j,  c_i = sum_j A_ji dA_ji
        dZ_ji = A_ji (dA_ji - c_i)
        dQ = dZ K/sqrt(d),  dK = dZ^T Q/sqrt(d)
        dX = A^T dH + dK W_K^T,  dP += dQ W_Q^T,  dW_Q += P^T dQ,  dW_K += X^T dK
    """
    X = _f64(X)
    P, W_Q, W_K, W_V = _f64(P), _f64(W_Q), _f64(W_K), _f64(W_V)
    offsets = np.asarray(offsets, np.int64)
    B = len(offsets) - 1
    k, d = P.shape
    dX = np.zeros_like(X)
    dP = np.zeros_like(P)
    dW_Q = np.zeros_like(W_Q)
    dW_K = np.zeros_like(W_K)
    dW_V = np.zeros_like(W_V)
    Q = P @ W_Q
    for u in range(B):
        lo, hi = int(offsets[u]), int(offsets[u + 1])
        if hi == lo:
            continue
        Xu = X[lo:hi]
        G = _f64(dS[u])
        A = assignment(Xu, P, W_Q, W_K)
        m = A.sum(axis=1)
        H = A @ Xu
        Hh = H / (m + eps)[:, None]
        dW_V += Hh.T @ G
        dHh = G @ W_V.T
        dH = dHh / (m + eps)[:, None]
        dm = -np.sum(dHh * H, axis=1) / (m + eps) ** 2
        if dmass is not None:
            dm = dm + _f64(dmass[u])
        dA = dH @ Xu.T + dm[:, None]               # k x n
        c = np.sum(A * dA, axis=0, keepdims=True)  # 1 x n
        dZ = A * (dA - c)
        K = Xu @ W_K
        dQ = dZ @ K / math.sqrt(d)
        dK = dZ.T @ Q / math.sqrt(d)
        dX[lo:hi] = A.T @ dH + dK @ W_K.T
        dP += dQ @ W_Q.T
        dW_Q += P.T @ dQ
        dW_K += Xu.T @ dK
    return dX, dP, dW_Q, dW_K, dW_V


# --------------------------------------------------------------------------
# STCA
# --------------------------------------------------------------------------
def _softmax_rows(s: np.ndarray) -> np.ndarray:
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=1, keepdims=True)


def _history_ffn(Xu, lay) -> np.ndarray:
    """X + FFN_h(X) when the layer has a history FFN (eq. (27)), else X."""
    if getattr(lay, "hist_W1", None) is None:
        return Xu
    return Xu + swiglu_ffn(Xu, lay.hist_W1, lay.hist_W3, lay.hist_W2)


def _query_ffn(qu, lay) -> np.ndarray:
    """q + FFN_q(q) when the layer has a query FFN (eq. (26)), else q."""
    if getattr(lay, "q_W1", None) is None:
        return qu
    return qu + swiglu_ffn(qu, lay.q_W1, lay.q_W3, lay.q_W2)


def stca_branch(q, cand_offsets, kv, kv_begin, kv_end, layers, heads: int, d_h: int):
    """Stacked target-to-history single-query cross attention, direct form.

    One layer (Sec. 2.3, eq. (4)), per head h:
        alpha = softmax((q W_Q^h)(X W_K^h)^T / sqrt(d_h))   over the L keys
        o_h   = alpha (X W_V^h)
    then q <- q + concat_h(o_h) W_O (W_O = identity when absent).
    Candidates of user u are rows [cand_offsets[u], cand_offsets[u+1]) of q;
    their keys/values are rows [kv_begin[u], kv_end[u]) of kv.
    ``layers`` is a list of objects with W_Q, W_K, W_V ([heads, D, d_h]) and
    W_O ([heads*d_h, D] or None), and optionally the full layer's FFNs
    (eqs. (26)-(27)): hist_W1, hist_W3 [D, 2D], hist_W2 [2D, D] applied to
    the history before the attention, q_W1, q_W3, q_W2 applied to the query
    after the W_O residual (None = absent).
    """
    out = _f64(q).copy()
    kv = _f64(kv)
    cand_offsets = np.asarray(cand_offsets, np.int64)
    for u in range(len(cand_offsets) - 1):
        c0, c1 = int(cand_offsets[u]), int(cand_offsets[u + 1])
        if c1 == c0:
            continue
        Xu = kv[int(kv_begin[u]):int(kv_end[u])]
        qu = out[c0:c1]
        for lay in layers:
            Xu = _history_ffn(Xu, lay)
            o = np.zeros((c1 - c0, heads * d_h))
            if Xu.shape[0] > 0:
                for h in range(heads):
                    Wq, Wk, Wv = _f64(lay.W_Q[h]), _f64(lay.W_K[h]), _f64(lay.W_V[h])
                    scores = (qu @ Wq) @ (Xu @ Wk).T / math.sqrt(d_h)
                    alpha = _softmax_rows(scores)
                    o[:, h * d_h:(h + 1) * d_h] = alpha @ (Xu @ Wv)
            qu = qu + (o if lay.W_O is None else o @ _f64(lay.W_O))
            qu = _query_ffn(qu, lay)
        out[c0:c1] = qu
    return out


def stca_branch_reordered(q, cand_offsets, kv, kv_begin, kv_end, layers, heads: int, d_h: int):
    """The same layers in the single-query reordering of Sec. 5.1, eq. (24):
        u = (q W_Q^h) W_K^h^T,  alpha = softmax(u X^T / sqrt(d_h)),  o = (alpha X) W_V^h.
    Keys and values are the raw history rows.  Used only as a cross-check of
    ``stca_branch``."""
    out = _f64(q).copy()
    kv = _f64(kv)
    cand_offsets = np.asarray(cand_offsets, np.int64)
    for u in range(len(cand_offsets) - 1):
        c0, c1 = int(cand_offsets[u]), int(cand_offsets[u + 1])
        if c1 == c0:
            continue
        Xu = kv[int(kv_begin[u]):int(kv_end[u])]
        qu = out[c0:c1]
        for lay in layers:
            Xu = _history_ffn(Xu, lay)
            o = np.zeros((c1 - c0, heads * d_h))
            if Xu.shape[0] > 0:
                for h in range(heads):
                    Wq, Wk, Wv = _f64(lay.W_Q[h]), _f64(lay.W_K[h]), _f64(lay.W_V[h])
                    uvec = (qu @ Wq) @ Wk.T
                    alpha = _softmax_rows(uvec @ Xu.T / math.sqrt(d_h))
                    o[:, h * d_h:(h + 1) * d_h] = (alpha @ Xu) @ Wv
            qu = qu + (o if lay.W_O is None else o @ _f64(lay.W_O))
            qu = _query_ffn(qu, lay)
        out[c0:c1] = qu
    return out


STCA_WEIGHTS = ("W_Q", "W_K", "W_V", "W_O", "hist_W1", "hist_W3", "hist_W2", "q_W1", "q_W3", "q_W2")


def stca_branch_grads(q, cand_offsets, kv, kv_begin, kv_end, layers, heads: int, d_h: int, dout):
    """Gradients of sum(dout * stca_branch(...)) with respect to q, kv and every weight of
    every layer, by reverse-mode differentiation (torch autograd, fp64, CPU) of the same
    definition as ``stca_branch`` written with torch operations: per user, the layer's
    history FFN (if any), the attention of eq. (4) per head, W_O and the residual, the
    query FFN (if any).  A key row shared by several users' ranges collects the gradient
    of every use.  Returns {"dq": [C, D], "dkv": [rows, D], "layers": [{name: grad}]}
    with None for an absent weight."""
    import torch

    t = lambda a: torch.tensor(_f64(a), dtype=torch.float64)
    qv = t(q).requires_grad_(True)
    kvv = t(kv).requires_grad_(True)
    W = []
    for lay in layers:
        W.append({k: (t(getattr(lay, k)).requires_grad_(True) if getattr(lay, k, None) is not None else None)
                  for k in STCA_WEIGHTS})

    def ffn(x, W1, W3, W2):
        a = x @ W1
        return ((a / (1.0 + torch.exp(-a))) * (x @ W3)) @ W2

    cand_offsets = np.asarray(cand_offsets, np.int64)
    outs = []
    for u in range(len(cand_offsets) - 1):
        c0, c1 = int(cand_offsets[u]), int(cand_offsets[u + 1])
        if c1 == c0:
            continue
        Xu = kvv[int(kv_begin[u]):int(kv_end[u])]
        qu = qv[c0:c1]
        for w in W:
            if w["hist_W1"] is not None:
                Xu = Xu + ffn(Xu, w["hist_W1"], w["hist_W3"], w["hist_W2"])
            if Xu.shape[0] > 0:
                o = []
                for h in range(heads):
                    s = (qu @ w["W_Q"][h]) @ (Xu @ w["W_K"][h]).T / math.sqrt(d_h)
                    o.append(torch.softmax(s, dim=1) @ (Xu @ w["W_V"][h]))
                o = torch.cat(o, dim=1)
            else:
                o = torch.zeros(c1 - c0, heads * d_h, dtype=torch.float64)
            qu = qu + (o if w["W_O"] is None else o @ w["W_O"])
            if w["q_W1"] is not None:
                qu = qu + ffn(qu, w["q_W1"], w["q_W3"], w["q_W2"])
        outs.append((c0, c1, qu))
    total = sum((o * t(dout)[c0:c1]).sum() for c0, c1, o in outs) if outs else qv.sum() * 0.0
    leaves = [qv, kvv] + [v for w in W for v in w.values() if v is not None]
    grads = torch.autograd.grad(total, leaves, allow_unused=True)
    g = iter(grads)
    res = {"dq": next(g), "dkv": next(g), "layers": []}
    for w in W:
        res["layers"].append({k: (next(g) if v is not None else None) for k, v in w.items()})
    zero = lambda x, like: torch.zeros_like(like) if x is None else x
    res["dq"] = zero(res["dq"], qv).numpy()
    res["dkv"] = zero(res["dkv"], kvv).numpy()
    for li, w in enumerate(W):
        for k, v in w.items():
            if v is not None:
                res["layers"][li][k] = zero(res["layers"][li][k], v).numpy()
    return res


def event_rows(item_table, action_table, item_ids, action_ids) -> np.ndarray:
    """Event embeddings x_i = item_table[id_i] + action_table[a_i] (the workloads'
    events: an item embedding plus the embedding of the feedback type, the plain
    sum that eq. (20)'s fusion adds a SwiGLU term to), exact in fp64."""
    return _f64(item_table)[np.asarray(item_ids, np.int64)] + _f64(action_table)[np.asarray(action_ids, np.int64)]


def event_rows_fused(item_table, action_table, item_ids, action_ids, W1, W3, W2) -> np.ndarray:
    """Action-side SwiGLU fusion (Sec. 3.6 / App. D, eq. (20)):
        x_i = e_i + FFN_SwiGLU([e_i ; a_i]),   e_i = item_table[id_i], a_i = action_table[type_i]
    with FFN_SwiGLU(z) = (SiLU(z W1) * (z W3)) W2 on the concatenated 2d-wide
    feature, mapped back to the item embedding's width d so the residual add is
    defined; W1, W3 [2d, w_f], W2 [w_f, d] (the workloads take w_f = 2d, eq. (23)'s
    inner width for an FFN of width d), no biases."""
    e = _f64(item_table)[np.asarray(item_ids, np.int64)]
    a = _f64(action_table)[np.asarray(action_ids, np.int64)]
    return e + swiglu_ffn(np.concatenate([e, a], axis=1), W1, W3, W2)


def stca_fuse(z_r, z_u, W_F, b_F=None):
    """Linear fusion of the two branches: [z_r ; z_u] W_F + b_F (Sec. 3.4)."""
    z = np.concatenate([_f64(z_r), _f64(z_u)], axis=1)
    out = z @ _f64(W_F)
    if b_F is not None:
        out = out + _f64(b_F)[None, :]
    return out


# --------------------------------------------------------------------------
# Stacked refinement
# --------------------------------------------------------------------------
def layer_norm(Y, g=None, b=None, eps: float = 1e-5) -> np.ndarray:
    """LN over the last axis (Sec. 3.3, eqs. (15)-(16)): (y - mean) / sqrt(var + eps),
    biased variance, then times the gain g and plus the bias b when given."""
    Y = _f64(Y)
    mu = Y.mean(axis=-1, keepdims=True)
    var = ((Y - mu) ** 2).mean(axis=-1, keepdims=True)
    out = (Y - mu) / np.sqrt(var + eps)
    if g is not None:
        out = out * _f64(g)
    if b is not None:
        out = out + _f64(b)
    return out


def swiglu_ffn(Y, W1, W3, W2) -> np.ndarray:
    """The FFN of eq. (16): (SiLU(Y W1) * (Y W3)) W2 with SiLU(x) = x / (1 + e^-x);
    W1, W3 [d, 2d], W2 [2d, d] (the SwiGLU of eq. (23) with inner width 2d)."""
    Y = _f64(Y)
    a = Y @ _f64(W1)
    return ((a / (1.0 + np.exp(-a))) * (Y @ _f64(W3))) @ _f64(W2)


def sa_refine_user(Xu, P0, layers, ln_eps: float = 1e-5) -> np.ndarray:
    """One user's stacked refinement (Sec. 3.3), starting from X~(0) = P0 [k, d];
    per iteration, with that iteration's weights:
        S  = (X~ W_Q)(X W_K)^T / sqrt(d),  A = softmax over prototypes   (12)-(13)
        X^ = A X                                                        (14)
        Xbar = LN(X~ + X^)                                              (15)
        X~ = LN(Xbar + FFN(Xbar))                                       (16)
    ``layers``: dicts with W_Q, W_K, W1, W3, W2 and optional ln1_g, ln1_b, ln2_g,
    ln2_b.  Returns X~ after the last iteration."""
    Xu = _f64(Xu)
    Xt = _f64(P0)
    for L in layers:
        if Xu.shape[0] == 0:
            Xhat = np.zeros_like(Xt)
        else:
            Xhat = assignment(Xu, Xt, L["W_Q"], L["W_K"]) @ Xu
        Xbar = layer_norm(Xt + Xhat, L.get("ln1_g"), L.get("ln1_b"), ln_eps)
        Xt = layer_norm(Xbar + swiglu_ffn(Xbar, L["W1"], L["W3"], L["W2"]), L.get("ln2_g"),
                        L.get("ln2_b"), ln_eps)
    return Xt


REFINE_WEIGHTS = ("W_Q", "W_K", "W1", "W3", "W2", "ln1_g", "ln1_b", "ln2_g", "ln2_b")


def sa_refine_grads(X, offsets: Sequence[int], P0, layers, dout, ln_eps: float = 1e-5):
    """Gradients of sum(dout * sa_refine(...)) with respect to X, P0 and every weight of
    every iteration, by reverse-mode differentiation (torch autograd, fp64, CPU) of the
    same definition as ``sa_refine_user`` written with torch operations: per user and
    iteration, S = (X~ W_Q)(X W_K)^T / sqrt(d), the softmax over prototypes, X^ = A X,
    Xbar = LN(X~ + X^), X~ = LN(Xbar + FFN(Xbar)) (eqs. (12)-(16)).  The weights are
    shared by the users, so their gradients are sums over users.  Returns
    {"dX": [n, d], "dP0": [k, d], "layers": [{name: grad or None}]}."""
    import torch

    t = lambda a: torch.tensor(_f64(a), dtype=torch.float64)
    Xv = t(X).requires_grad_(True)
    P0v = t(P0).requires_grad_(True)
    W = [{k: (t(L[k]).requires_grad_(True) if L.get(k) is not None else None) for k in REFINE_WEIGHTS}
         for L in layers]

    def ln(y, g, b):
        mu = y.mean(dim=-1, keepdim=True)
        var = ((y - mu) ** 2).mean(dim=-1, keepdim=True)
        out = (y - mu) / torch.sqrt(var + ln_eps)
        if g is not None:
            out = out * g
        if b is not None:
            out = out + b
        return out

    d = Xv.shape[1]
    offsets = np.asarray(offsets, np.int64)
    total = P0v.sum() * 0.0
    dt = t(dout)
    for u in range(len(offsets) - 1):
        Xu = Xv[int(offsets[u]):int(offsets[u + 1])]
        Xt = P0v
        for w in W:
            if Xu.shape[0] > 0:
                S = (Xt @ w["W_Q"]) @ (Xu @ w["W_K"]).T / math.sqrt(d)
                Xhat = torch.softmax(S, dim=0) @ Xu
            else:
                Xhat = torch.zeros_like(Xt)
            Xbar = ln(Xt + Xhat, w["ln1_g"], w["ln1_b"])
            a = Xbar @ w["W1"]
            Xt = ln(Xbar + ((a / (1.0 + torch.exp(-a))) * (Xbar @ w["W3"])) @ w["W2"], w["ln2_g"], w["ln2_b"])
        total = total + (Xt * dt[u]).sum()
    leaves = [Xv, P0v] + [v for w in W for v in w.values() if v is not None]
    grads = torch.autograd.grad(total, leaves, allow_unused=True)
    g = iter(grads)
    z = lambda v, r: (torch.zeros_like(v) if r is None else r).numpy()
    res = {"dX": z(Xv, next(g)), "dP0": z(P0v, next(g)), "layers": []}
    for w in W:
        res["layers"].append({k: (z(v, next(g)) if v is not None else None) for k, v in w.items()})
    return res


def sa_refine(X, offsets: Sequence[int], P0, layers, ln_eps: float = 1e-5) -> np.ndarray:
    """Refined sketches of a ragged batch: [B, k, d] fp64."""
    offsets = np.asarray(offsets, np.int64)
    B = len(offsets) - 1
    k, d = np.shape(P0)
    out = np.zeros((B, k, d))
    for u in range(B):
        out[u] = sa_refine_user(X[offsets[u]:offsets[u + 1]], P0, layers, ln_eps)
    return out


# --------------------------------------------------------------------------
# Token-wise normalisation variant (the vanilla-attention baseline)
# --------------------------------------------------------------------------
def tokenwise_user(Xu, P, W_Q, W_K, W_V, eps: float):
    """The affinities of eq. (6) normalised over the user's tokens instead of the
    prototypes (Sec. 7.1, Table 1; Sec. 2's latent-query, token-wise softmax):
        A_{j,i} = exp S_{j,i} / sum_i' exp S_{j,i'},  H = A X,  m_j = sum_i A_{j,i}
    and the output step of sa_user, S = diag(1/(m+eps)) H W_V.  Returns (S, m, H);
    a user without events gets zeros."""
    Xu = _f64(Xu)
    k, d = np.shape(P)
    if Xu.shape[0] == 0:
        return np.zeros((k, d)), np.zeros(k), np.zeros((k, d))
    Z = ((_f64(P) @ _f64(W_Q)) @ (Xu @ _f64(W_K)).T) / math.sqrt(d)   # k x n, eq. (6)
    Zc = Z - Z.max(axis=1, keepdims=True)
    E = np.exp(Zc)
    A = E / E.sum(axis=1, keepdims=True)          # softmax over tokens (rows sum to 1)
    m = A.sum(axis=1)
    H = A @ Xu
    denom = (m + eps)[:, None]
    Hh = np.divide(H, denom, out=np.zeros_like(H), where=denom > 0)
    return Hh @ _f64(W_V), m, H


def sa_forward_tokenwise(X, offsets: Sequence[int], P, W_Q, W_K, W_V, eps: float):
    """Token-wise variant over a ragged batch: S [B,k,d], mass [B,k], H [B,k,d]."""
    offsets = np.asarray(offsets, np.int64)
    B = len(offsets) - 1
    k, d = np.shape(P)
    S, mass, H = np.zeros((B, k, d)), np.zeros((B, k)), np.zeros((B, k, d))
    for u in range(B):
        S[u], mass[u], H[u] = tokenwise_user(X[offsets[u]:offsets[u + 1]], P, W_Q, W_K, W_V, eps)
    return S, mass, H
