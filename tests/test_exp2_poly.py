"""The FMA-pipe exponential used for part of the softmax exponentials: its
coefficients are reproducible from the generator, and the routine's fp32
arithmetic (restated step by step by the generator) meets its error bound."""
import os

import numpy as np

from sketch_attention_b200.csrc import gen_exp2_poly as gen

HEADER = os.path.join(os.path.dirname(gen.__file__), "exp2_poly.cuh")


def test_header_is_generated_from_the_fit():
    with open(HEADER) as fh:
        assert fh.read() == gen.header(gen.fit())


def test_error_bound_over_the_softmax_range():
    c = gen.fit()
    assert gen.max_rel_error(c) < 1e-4


def test_special_values():
    c = gen.fit()
    x = np.array([0.0, 1.0, -1.0, 8.0, 0.5, -0.5, -20.25], np.float32)
    y = gen.exp2_fp32(x, c).astype(np.float64)
    np.testing.assert_allclose(y, np.exp2(x.astype(np.float64)), rtol=1e-4)
    # far below the range: clamped to about 2^-125, still a positive normal number
    lo = gen.exp2_fp32(np.array([-200.0, -np.inf], np.float32), c)
    assert np.all(lo > 0) and np.all(lo < 2.0 ** -124) and np.all(np.isfinite(lo))


def test_monotone_across_integer_boundaries():
    c = gen.fit()
    x = np.concatenate([np.arange(-30, 9, dtype=np.float32) + d for d in (-1e-3, 0.0, 1e-3, 0.4999, 0.5001)])
    x.sort()
    y = gen.exp2_fp32(x, c)
    assert np.all(np.diff(y.astype(np.float64)) >= 0)
