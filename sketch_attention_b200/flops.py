"""Analytic GEMM-FLOP model of SequenceO1 (App. G of the paper, eqs. (23)-(36)).

Counting rule of the pages: FLOPs(U V) = 2 m r p for U in R^{m x r},
V in R^{r x p}; softmax exponentials, LayerNorm, bias and activations are not
counted.  These numbers are analytic context for the benchmark, not a
hardware target.
"""
from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class Hyper:
    """Hyper-parameters of the pages' FLOP instantiation (Sec. 5.4)."""
    d: int = 128          # SA width
    N_sa: int = 2         # stacked SA iterations
    L_s: int = 1024       # sketch length (number of prototypes)
    h: int = 16           # STCA heads
    d_h: int = 64         # STCA head width
    D: int = 1024         # STCA model width
    N_stca: int = 4       # STCA layers


def swiglu(T: int, w: int, w_f: int) -> float:
    """eq. (23): 6 T w w_f."""
    return 6.0 * T * w * w_f


def stca_layer(L: int, hp: Hyper) -> float:
    """eq. (26): 4 L D h + 20 D^2 per target and layer."""
    return 4.0 * L * hp.D * hp.h + 20.0 * hp.D ** 2


def stca(L: int, hp: Hyper) -> float:
    """eq. (28): N_stca (12 L D^2 + 4 L D h + 20 D^2), the history FFN of eq. (27) included."""
    return hp.N_stca * (12.0 * L * hp.D ** 2 + stca_layer(L, hp))


def sa_layer(L: int, hp: Hyper) -> float:
    """eq. (29): 2 L d^2 + 14 L_s d^2 + 4 L_s L d."""
    return 2.0 * L * hp.d ** 2 + 14.0 * hp.L_s * hp.d ** 2 + 4.0 * hp.L_s * L * hp.d


def sa(L: int, hp: Hyper) -> float:
    """eq. (30): N_sa iterations of eq. (29)."""
    return hp.N_sa * sa_layer(L, hp)


def adapt(hp: Hyper) -> float:
    """Sketch adapter W_A: 2 L_s d D (Sec. 5.3)."""
    return 2.0 * hp.L_s * hp.d * hp.D


def hit(hp: Hyper) -> float:
    """eq. (31), cache hit: adapter + STCA over the sketch."""
    return adapt(hp) + stca(hp.L_s, hp)


def expected(L: int, p_hit: float, hp: Hyper) -> float:
    """eq. (32): hit cost plus the miss-weighted SA cost."""
    return hit(hp) + (1.0 - p_hit) * sa(L, hp)


def stca_mrlb(L: int, R: int, hp: Hyper) -> float:
    """eq. (33): direct STCA when only the history FFN is amortised over R targets."""
    return 12.0 * hp.N_stca * L * hp.D ** 2 / R + hp.N_stca * stca_layer(L, hp)


def seqo1_mrlb(L: int, R: int, p_hit: float, hp: Hyper) -> float:
    """eq. (34): SequenceO1 with SA, adapter and sketch-side FFN amortised over R."""
    return (hp.N_stca * (4.0 * hp.L_s * hp.D * hp.h + 20.0 * hp.D ** 2)
            + (adapt(hp) + 12.0 * hp.N_stca * hp.L_s * hp.D ** 2 + (1.0 - p_hit) * sa(L, hp)) / R)


def headline(L: int = 100_000, hp: Hyper = Hyper()) -> dict:
    """The pages' three FLOP ratios (Sec. 5.4), in GFLOPs per target."""
    direct = stca(L, hp)
    seq = expected(L, 0.5, hp)
    tr_stca, tr_seq = stca_mrlb(L, 40, hp), seqo1_mrlb(L, 40, 0.5, hp)
    in_stca, in_seq = stca_mrlb(L, 300, hp), seqo1_mrlb(L, 300, 0.6, hp)
    g = 1e9
    return {
        "direct_stca_gflops": direct / g,
        "seqo1_expected_gflops": seq / g,
        "no_mrlb_ratio": direct / seq,
        "train_stca_gflops": tr_stca / g,
        "train_seqo1_gflops": tr_seq / g,
        "train_ratio": tr_stca / tr_seq,
        "infer_stca_gflops": in_stca / g,
        "infer_seqo1_gflops": in_seq / g,
        "infer_ratio": in_stca / in_seq,
        "sa_gflops_per_user": sa(L, hp) / g,
    }


# Per-token work of this library's SA kernels (not a page formula): the two
# contractions logits = P' X^T and H += A X are 2 k d flops each per token; the
# softmax takes k exponentials per token.
def sa_fwd_flops_per_token(k: int, d: int) -> float:
    return 4.0 * k * d


def sa_bwd_flops_per_token(k: int, d: int) -> float:
    # recompute logits (2kd), dH.x (2kd), dX = [A|dZ][dH;P'] (4kd), E += dZ^T X (2kd)
    return 10.0 * k * d


def stca_attn_flops_per_candidate(L: int, D: int, heads: int, layers: int) -> float:
    """eq. (25)'s length term 4 L D h per layer (scores + weighted sum over D-wide keys)."""
    return 4.0 * L * D * heads * layers
