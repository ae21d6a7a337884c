"""Seeded synthetic inputs for Sketch Attention (SA) and STCA.

This module is shared by the tests, the benchmark and the smoke check.  It
draws random numbers and lays them out; it holds none of the method's
arithmetic (no logits, softmax, aggregation or attention), so the CPU oracle
and the CUDA path can both consume its arrays without sharing any code.

Workload shapes follow what the SequenceO1 pages fix: histories truncated at
n_max = 100K events (Sec. 2.1), a mean length of 85K under that truncation
(Fig. 1(c) discussion), k = 1K prototypes and d = 128 (Table 2 discussion),
a recent suffix of L_r = 10K (eq. 3), and events that combine an item and an
action type (eq. 1, App. D).  The pages' own data is private; these synthetic
inputs stand in for it.

Conventions
-----------
* One numpy PCG64 generator per problem; config c uses seed 1000 + c.
* ``N(0, s)`` with s = 0.02 means standard deviation 0.02 (embedding tables);
  ``N(0, 1/d)`` means variance 1/d (weights).
* bf16 tensors are produced by round-to-nearest-even from fp32 and carried as
  raw uint16 bit patterns; ``bf16_to_f64`` widens them exactly.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

L_RECENT = 10_000          # recent-suffix length L_r (eq. 3)
N_MAX = 100_000            # history truncation n_max (Sec. 2.1)
N_ACTIONS = 8              # action types per event


# --------------------------------------------------------------------------
# bf16 plumbing
# --------------------------------------------------------------------------
def bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    assert np.isfinite(a).all()
    u = a.view(np.uint32)
    # finite values: the sum stays below 2^32
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_to_f32(bits).astype(np.float64)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Values of ``a`` rounded to the nearest bf16, returned as fp32."""
    return bf16_to_f32(bf16_bits(a))


# --------------------------------------------------------------------------
# samplers
# --------------------------------------------------------------------------
def rng_for(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def gauss(rng, shape, std: float) -> np.ndarray:
    a = rng.standard_normal(shape, dtype=np.float32)
    a *= np.float32(std)
    return a


class ZipfSampler:
    """p(r) proportional to r^-s over ranks r = 1..V, by inverse-CDF sampling.

    Item ids are a seeded permutation of the ranks, so popular items are not
    the small ids.
    """

    def __init__(self, rng, vocab: int, s: float = 1.1):
        w = np.arange(1, vocab + 1, dtype=np.float64) ** (-s)
        self.cdf = np.cumsum(w)
        self.cdf /= self.cdf[-1]
        self.perm = rng.permutation(vocab).astype(np.int64)

    def sample(self, rng, n: int) -> np.ndarray:
        u = rng.random(n)
        r = np.searchsorted(self.cdf, u, side="right")
        r = np.minimum(r, len(self.cdf) - 1)
        return self.perm[r]


@dataclasses.dataclass
class EventTables:
    """Item and action-type embedding tables (std 0.02 each)."""
    item: np.ndarray          # [vocab, d] fp32
    action: np.ndarray        # [N_ACTIONS, d] fp32
    zipf: ZipfSampler

    @staticmethod
    def make(rng, d: int, vocab: int) -> "EventTables":
        item = gauss(rng, (vocab, d), 0.02)
        action = gauss(rng, (N_ACTIONS, d), 0.02)
        return EventTables(item, action, ZipfSampler(rng, vocab))

    def events(self, rng, n: int, with_ids: bool = False):
        """n event embeddings item[id] + action[a], fp32 (not yet rounded); with
        ``with_ids`` also the item ids (int32) and action types (uint8) drawn."""
        ids = self.zipf.sample(rng, n)
        acts = rng.integers(0, N_ACTIONS, n)
        rows = self.item[ids] + self.action[acts]
        if with_ids:
            return rows, ids.astype(np.int32), acts.astype(np.uint8)
        return rows

    def targets(self, rng, n: int) -> np.ndarray:
        return self.item[self.zipf.sample(rng, n)].copy()


# --------------------------------------------------------------------------
# SA problems
# --------------------------------------------------------------------------
@dataclasses.dataclass
class SAProblem:
    name: str
    dtype: str                # "f32" or "bf16"
    offsets: np.ndarray       # int64 [B+1]
    X: np.ndarray             # f32 [N, d] values, or uint16 bf16 bits [N, d]
    P: np.ndarray             # f32 [k, d]
    W_Q: np.ndarray           # f32 [d, d]
    W_K: np.ndarray
    W_V: np.ndarray
    eps: float = 1e-6
    dS: Optional[np.ndarray] = None   # f32 [B, k, d] upstream gradient
    item_ids: Optional[np.ndarray] = None     # int32 [N] the events' item ids (when kept)
    action_ids: Optional[np.ndarray] = None   # uint8 [N] their action types

    @property
    def B(self) -> int:
        return len(self.offsets) - 1

    @property
    def k(self) -> int:
        return self.P.shape[0]

    @property
    def d(self) -> int:
        return self.P.shape[1]

    @property
    def n_total(self) -> int:
        return int(self.offsets[-1])

    def x_f64(self, lo: int = 0, hi: Optional[int] = None) -> np.ndarray:
        """Rows [lo, hi) of X as exact fp64."""
        rows = self.X[lo:hi]
        if self.dtype == "bf16":
            return bf16_to_f64(rows)
        return rows.astype(np.float64)

    def subset(self, users: Sequence[int]) -> "SAProblem":
        """The same weights restricted to some users (rows re-packed)."""
        pieces, offs = [], [0]
        for u in users:
            lo, hi = int(self.offsets[u]), int(self.offsets[u + 1])
            pieces.append(self.X[lo:hi])
            offs.append(offs[-1] + hi - lo)
        X = np.concatenate(pieces, axis=0) if pieces else self.X[:0]
        dS = None if self.dS is None else self.dS[list(users)]
        return dataclasses.replace(self, name=self.name + f"[users={list(users)}]",
                                   offsets=np.asarray(offs, np.int64), X=X, dS=dS)


def _weights(rng, k: int, d: int, p_scale: float = 1.0):
    std = 1.0 / math.sqrt(d)           # variance 1/d
    P = gauss(rng, (k, d), std * p_scale)
    W_Q = gauss(rng, (d, d), std)
    W_K = gauss(rng, (d, d), std)
    W_V = gauss(rng, (d, d), std)
    return P.astype(np.float32), W_Q, W_K, W_V


def _pack(dtype: str, rows: np.ndarray) -> np.ndarray:
    return bf16_bits(rows) if dtype == "bf16" else np.ascontiguousarray(rows, np.float32)


def make_sa_problem(lengths: Sequence[int], k: int, d: int, dtype: str, seed: int,
                    x_kind: str = "gauss", p_scale: float = 1.0, vocab: int = 4096,
                    with_grad: bool = False, name: str = "custom",
                    tables: Optional[EventTables] = None) -> SAProblem:
    """A generic SA problem.

    x_kind: "gauss" draws X ~ N(0, std 1/sqrt(d)); "events" draws item+action
    embeddings (std 0.02 tables, Zipf(1.1) item ids over ``vocab`` items).
    p_scale multiplies the prototypes (large values give sharp assignments).
    """
    rng = rng_for(seed)
    lengths = [int(n) for n in lengths]
    offsets = np.zeros(len(lengths) + 1, np.int64)
    offsets[1:] = np.cumsum(lengths)
    P, W_Q, W_K, W_V = _weights(rng, k, d, p_scale)
    if x_kind == "events" and tables is None:
        tables = EventTables.make(rng, d, vocab)
    chunks = []
    for n in lengths:
        if x_kind == "gauss":
            rows = gauss(rng, (n, d), 1.0 / math.sqrt(d))
        elif x_kind == "events":
            rows = tables.events(rng, n)
        else:
            raise ValueError(x_kind)
        chunks.append(_pack(dtype, rows))
    if chunks:
        X = np.concatenate(chunks, axis=0)
    else:
        X = _pack(dtype, np.zeros((0, d), np.float32))
    dS = gauss(rng, (len(lengths), k, d), 1.0) if with_grad else None
    return SAProblem(name, dtype, offsets, X, P, W_Q, W_K, W_V, 1e-6, dS)


def lengths_uniform(rng, B: int, lo: int, hi: int):
    return rng.integers(lo, hi + 1, B).tolist()


def lengths_lognormal(rng, B: int, mu: float = 11.40186, sigma: float = 0.3,
                      lo: int = 10_000, hi: int = N_MAX):
    """Lognormal lengths clipped to [lo, hi]; mu, sigma give a clipped mean near 85K."""
    n = np.exp(rng.normal(mu, sigma, B))
    return np.clip(np.round(n), lo, hi).astype(np.int64).tolist()


# The five benchmark workloads.  Config 1 is the small fp32 case; 2, 3, 5 are
# SA at production shapes; 4 is STCA on cached sketches.
SA_WORKLOADS = {
    1: "sa_fwd f32 B=1 n=4096 d=64 k=64",
    2: "sa_fwd bf16 B=8 n~U[20K,100K] d=128 k=512",
    3: "sa_fwd bf16 B=32 n=100K d=128 k=1024",
    5: "sa_fwd+sa_bwd bf16 B=64 n~lognormal(mean 85K) d=128 k=1024",
}


def sa_workload(cfg: int, vocab: int = 1_000_000, users: Optional[int] = None,
                with_tables: bool = False, keep_ids: bool = False):
    """SA inputs for workload ``cfg`` (1, 2, 3 or 5).

    ``users`` truncates the batch to its first users (same random stream for
    the lengths and weights, so the first users match the full batch's).
    ``keep_ids`` also records each event's item id and action type (the same
    draws, so X is unchanged).
    """
    rng = rng_for(1000 + cfg)
    if cfg == 1:
        lengths, k, d, dtype, kind = [4096], 64, 64, "f32", "gauss"
    elif cfg == 2:
        lengths, k, d, dtype, kind = lengths_uniform(rng, 8, 20_000, 100_000), 512, 128, "bf16", "events"
    elif cfg == 3:
        lengths, k, d, dtype, kind = [N_MAX] * 32, 1024, 128, "bf16", "events"
    elif cfg == 5:
        lengths, k, d, dtype, kind = lengths_lognormal(rng, 64), 1024, 128, "bf16", "events"
    else:
        raise ValueError(f"no SA workload {cfg}")
    if users is not None:
        lengths = lengths[:users]
    P, W_Q, W_K, W_V = _weights(rng, k, d)
    tables = EventTables.make(rng, d, vocab) if kind == "events" else None
    offsets = np.zeros(len(lengths) + 1, np.int64)
    offsets[1:] = np.cumsum(lengths)
    X = np.empty((int(offsets[-1]), d), np.uint16 if dtype == "bf16" else np.float32)
    keep = keep_ids and kind == "events"
    item_ids = np.empty(int(offsets[-1]), np.int32) if keep else None
    action_ids = np.empty(int(offsets[-1]), np.uint8) if keep else None
    for u, n in enumerate(lengths):
        if kind == "gauss":
            rows = gauss(rng, (n, d), 1.0 / math.sqrt(d))
        elif keep:
            rows, item_ids[offsets[u]:offsets[u + 1]], action_ids[offsets[u]:offsets[u + 1]] = \
                tables.events(rng, n, with_ids=True)
        else:
            rows = tables.events(rng, n)
        X[offsets[u]:offsets[u + 1]] = _pack(dtype, rows)
    dS = gauss(rng, (len(lengths), k, d), 1.0) if cfg == 5 else None
    prob = SAProblem(SA_WORKLOADS[cfg], dtype, offsets, X, P, W_Q, W_K, W_V, 1e-6, dS, item_ids, action_ids)
    if with_tables:
        return prob, tables, rng
    return prob


# --------------------------------------------------------------------------
# STCA problems
# --------------------------------------------------------------------------
@dataclasses.dataclass
class STCALayer:
    W_Q: np.ndarray      # f32 [heads, D, d_h]
    W_K: np.ndarray      # f32 [heads, D, d_h]
    W_V: np.ndarray      # f32 [heads, D, d_h]
    W_O: Optional[np.ndarray]   # f32 [heads*d_h, D] or None (identity)
    # the full layer's SwiGLU FFNs (None = absent): history side, then query side
    hist_W1: Optional[np.ndarray] = None   # f32 [D, 2D]
    hist_W3: Optional[np.ndarray] = None   # f32 [D, 2D]
    hist_W2: Optional[np.ndarray] = None   # f32 [2D, D]
    q_W1: Optional[np.ndarray] = None      # f32 [D, 2D]
    q_W3: Optional[np.ndarray] = None      # f32 [D, 2D]
    q_W2: Optional[np.ndarray] = None      # f32 [2D, D]


@dataclasses.dataclass
class STCABranch:
    """One STCA branch: per-user queries against a per-user key/value range."""
    q: np.ndarray               # [C_total, D]   f32 values or bf16 bits
    cand_offsets: np.ndarray    # int64 [B+1]
    kv: np.ndarray              # [rows, D]      f32 values or bf16 bits
    kv_begin: np.ndarray        # int64 [B]
    kv_end: np.ndarray          # int64 [B]


@dataclasses.dataclass
class STCAProblem:
    name: str
    dtype: str
    heads: int
    d_h: int
    recent: STCABranch           # z_r branch (eq. 17)
    sketch: STCABranch           # z_u branch (eq. 19)
    layers_r: list               # STCALayer per layer, recent branch
    layers_u: list               # STCALayer per layer, sketch branch
    W_F: np.ndarray              # f32 [2D, D]
    b_F: np.ndarray              # f32 [D]

    @property
    def D(self) -> int:
        return self.W_F.shape[1]

    def widen(self, a: np.ndarray) -> np.ndarray:
        return bf16_to_f64(a) if self.dtype == "bf16" else a.astype(np.float64)


def stca_layers(rng, n_layers: int, D: int, heads: int, d_h: int, with_wo: bool = True):
    std = 1.0 / math.sqrt(D)
    out = []
    for _ in range(n_layers):
        W_Q = gauss(rng, (heads, D, d_h), std)
        W_K = gauss(rng, (heads, D, d_h), std)
        W_V = gauss(rng, (heads, D, d_h), std)
        W_O = gauss(rng, (heads * d_h, D), std) if with_wo else None
        out.append(STCALayer(W_Q, W_K, W_V, W_O))
    return out


def event_problem(n: int, vocab: int, d: int, seed: int, n_actions: int = N_ACTIONS):
    """Seeded inputs of the event-embedding gather: bf16 item and action tables
    (bits, std 0.02 like the workloads' tables), Zipf(1.1) item ids (int32) and
    uniform action types (uint8) for n events."""
    rng = rng_for(seed)
    item = bf16_bits(gauss(rng, (vocab, d), 0.02))
    action = bf16_bits(gauss(rng, (n_actions, d), 0.02))
    ids = ZipfSampler(rng, vocab).sample(rng, n).astype(np.int32)
    acts = rng.integers(0, n_actions, n).astype(np.uint8)
    return item, action, ids, acts


def event_ffn_weights(rng, d: int, d_ff: int = None, scale: float = 1.0):
    """Weights of the action-side SwiGLU fusion of the event rows: W1, W3 [2d, d_ff]
    with std scale/sqrt(2d) and W2 [d_ff, d] with std 1/sqrt(d_ff) (variance 1 over
    the fan-in; d_ff = 2d by default), fp32."""
    d_ff = 2 * d if d_ff is None else d_ff
    return (gauss(rng, (2 * d, d_ff), scale / math.sqrt(2 * d)), gauss(rng, (2 * d, d_ff), scale / math.sqrt(2 * d)),
            gauss(rng, (d_ff, d), 1.0 / math.sqrt(d_ff)))


def add_stca_ffns(rng, layers, D: int, hist: bool = True, query: bool = True):
    """Give each STCA layer the full layer's SwiGLU FFNs: W1, W3 [D, 2D] with
    std 1/sqrt(D) and W2 [2D, D] with std 1/sqrt(2D), history side and/or
    query side.  Returns the same list."""
    for lay in layers:
        if hist:
            lay.hist_W1 = gauss(rng, (D, 2 * D), 1.0 / math.sqrt(D))
            lay.hist_W3 = gauss(rng, (D, 2 * D), 1.0 / math.sqrt(D))
            lay.hist_W2 = gauss(rng, (2 * D, D), 1.0 / math.sqrt(2 * D))
        if query:
            lay.q_W1 = gauss(rng, (D, 2 * D), 1.0 / math.sqrt(D))
            lay.q_W3 = gauss(rng, (D, 2 * D), 1.0 / math.sqrt(D))
            lay.q_W2 = gauss(rng, (2 * D, D), 1.0 / math.sqrt(2 * D))
    return layers


def refine_layers(rng, n_iter: int, d: int, affine: bool = True):
    """Weights of the stacked refinement, one dict per iteration: W_Q, W_K [d, d]
    and the SwiGLU FFN W1, W3 [d, 2d] (std 1/sqrt(d)), W2 [2d, d] (std 1/sqrt(2d));
    with ``affine`` the LN gains ~ 1 + 0.1 N(0, 1) and biases ~ 0.1 N(0, 1)."""
    out = []
    for _ in range(n_iter):
        L = {"W_Q": gauss(rng, (d, d), 1.0 / math.sqrt(d)),
             "W_K": gauss(rng, (d, d), 1.0 / math.sqrt(d)),
             "W1": gauss(rng, (d, 2 * d), 1.0 / math.sqrt(d)),
             "W3": gauss(rng, (d, 2 * d), 1.0 / math.sqrt(d)),
             "W2": gauss(rng, (2 * d, d), 1.0 / math.sqrt(2 * d))}
        for key in ("ln1", "ln2"):
            if affine:
                L[key + "_g"] = (1.0 + gauss(rng, (d,), 0.1)).astype(np.float32)
                L[key + "_b"] = gauss(rng, (d,), 0.1)
            else:
                L[key + "_g"] = L[key + "_b"] = None
        out.append(L)
    return out


def suffix_ranges(offsets: np.ndarray, L_r: int = L_RECENT):
    """The recent suffix X_r of each user as a [begin, end) row range (eq. 3);
    a user shorter than L_r contributes its whole history."""
    off = np.asarray(offsets, np.int64)
    end = off[1:].copy()
    begin = np.maximum(off[:-1], end - L_r)
    return begin, end


def make_stca_problem(B: int, cands: Sequence[int], kv_recent: Sequence[int], k: int, D: int,
                      heads: int, d_h: int, n_layers: int, dtype: str, seed: int,
                      vocab: int = 4096, with_wo: bool = True, name: str = "custom") -> STCAProblem:
    """A generic STCA problem: per user ``cands[u]`` targets, a recent history of
    ``kv_recent[u]`` events and a k x D sketch with N(0,1) rows."""
    rng = rng_for(seed)
    tables = EventTables.make(rng, D, vocab)
    layers_r = stca_layers(rng, n_layers, D, heads, d_h, with_wo)
    layers_u = stca_layers(rng, n_layers, D, heads, d_h, with_wo)
    W_F = gauss(rng, (2 * D, D), 1.0 / math.sqrt(2 * D))
    b_F = np.zeros(D, np.float32)
    cand_off = np.zeros(B + 1, np.int64)
    cand_off[1:] = np.cumsum(cands)
    q = _pack(dtype, tables.targets(rng, int(cand_off[-1])))
    hist_off = np.zeros(B + 1, np.int64)
    hist_off[1:] = np.cumsum(kv_recent)
    hist = np.concatenate([_pack(dtype, tables.events(rng, int(n))) for n in kv_recent], axis=0) \
        if B else _pack(dtype, np.zeros((0, D), np.float32))
    rb, re = suffix_ranges(hist_off)
    sketch = _pack(dtype, gauss(rng, (B * k, D), 1.0))
    sb = np.arange(B, dtype=np.int64) * k
    recent = STCABranch(q, cand_off, hist, rb, re)
    sk = STCABranch(q, cand_off, sketch, sb, sb + k)
    return STCAProblem(name, dtype, heads, d_h, recent, sk, layers_r, layers_u, W_F, b_F)


STCA_WORKLOAD_4 = "stca_fwd bf16 B=16 C=512/user L_r=10K k=1024 D=128 h=4 d_h=32 layers=2"


def stca_workload(vocab: int = 1_000_000, users: int = 16, cands: int = 512) -> STCAProblem:
    """STCA on cached sketches: 16 users, k=1024 x 128 sketches, 10K suffixes,
    512 candidates per user, 2 layers x 4 heads x d_h 32, bf16."""
    return make_stca_problem(users, [cands] * users, [L_RECENT] * users, 1024, 128, 4, 32, 2,
                             "bf16", 1004, vocab=vocab, name=STCA_WORKLOAD_4)


@dataclasses.dataclass
class TrainStep:
    """The end-to-end step: SA forward and backward over the batch, then STCA on
    the sketches and on each user's last L_r events against its candidates,
    then the linear fusion."""
    sa: SAProblem
    cand_offsets: np.ndarray     # int64 [B+1]
    q: np.ndarray                # bf16 bits [C_total, d] candidate targets
    recent_begin: np.ndarray     # int64 [B] rows of sa.X
    recent_end: np.ndarray
    heads: int
    d_h: int
    layers_r: list
    layers_u: list
    W_F: np.ndarray
    b_F: np.ndarray
    item_table: Optional[np.ndarray] = None     # bf16 bits [vocab, d]: the events' item embeddings
    action_table: Optional[np.ndarray] = None   # bf16 bits [N_ACTIONS, d]


TRAIN_STEP_WORKLOAD = ("train step bf16 B=64 n~lognormal(mean 85K) d=128 k=1024: sa_fwd+sa_bwd, "
                       "then STCA (2 layers x 4 heads x d_h 32) on sketches and 10K suffixes, "
                       "256 candidates/user, fuse")


def train_step_workload(vocab: int = 1_000_000, users: Optional[int] = None,
                        cands: int = 256) -> TrainStep:
    sa, tables, rng = sa_workload(5, vocab=vocab, users=users, with_tables=True, keep_ids=True)
    D, heads, d_h = sa.d, 4, 32
    layers_r = stca_layers(rng, 2, D, heads, d_h)
    layers_u = stca_layers(rng, 2, D, heads, d_h)
    W_F = gauss(rng, (2 * D, D), 1.0 / math.sqrt(2 * D))
    b_F = np.zeros(D, np.float32)
    cand_off = np.arange(sa.B + 1, dtype=np.int64) * cands
    q = bf16_bits(tables.targets(rng, int(cand_off[-1])))
    rb, re = suffix_ranges(sa.offsets)
    return TrainStep(sa, cand_off, q, rb, re, heads, d_h, layers_r, layers_u, W_F, b_F,
                     bf16_bits(tables.item), bf16_bits(tables.action))
