"""The analytic FLOP model reproduces the figures the pages print
(tests/golden/flop_model.txt, Sec. 5.4 of the paper's reading note)."""
import os

from sketch_attention_b200 import flops

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "flop_model.txt")


def _golden():
    rows = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, value, prec = line.split()[:3]
            rows[key] = (float(value), float(prec))
    return rows


def test_printed_figures():
    got = flops.headline(100_000)
    rows = _golden()
    assert len(rows) == 9
    for key, (value, prec) in rows.items():
        assert abs(got[key] - value) <= prec, (key, got[key], value)


def test_sa_dominant_term():
    """eq. (29): at L = 100K the 4 L_s L d term dominates the SA cost."""
    hp = flops.Hyper()
    dom = 4.0 * hp.L_s * 100_000 * hp.d
    assert 0.9 < dom / flops.sa_layer(100_000, hp) < 1.0
    assert flops.sa_fwd_flops_per_token(1024, 128) == 524288.0
