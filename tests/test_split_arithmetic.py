"""The error model behind the STCA backward's tensor-core products (no GPU).

With bf16 inputs the backward splits every fp32 operand x into hi = bf16(x) and
lo = bf16(x - hi) and forms A B as Ah Bh + Ah Bl + Al Bh (lo x lo dropped).  These
tests check, in exact fp64 arithmetic on the rounded parts, the two worst-case
bounds the GPU tests' tolerance for that path is derived from.  bf16 keeps 8
significant bits, so round to nearest is within 2^-8 |x|; the split keeps x to
within 2^-8 of that, 2^-16 |x|; and each product entry is within 3 x 2^-16 of
sum_k |a_ik| |b_kj| (the two operands' split errors and the dropped lo x lo, each
at most 2^-16 |a| |b| per term).  A single bf16 rounding of each operand (the
scheme the split replaced) exceeds that bound, which the last test shows."""
import numpy as np

from sa_inputs import round_bf16, rng_for


def _split(x32):
    hi = round_bf16(x32)
    lo = round_bf16((x32.astype(np.float64) - hi.astype(np.float64)).astype(np.float32))
    return hi.astype(np.float64), lo.astype(np.float64)


def _normal_f32(rng, shape, scale=1.0):
    # values well inside the normal bf16 range, so no subnormal rounding enters
    return (rng.standard_normal(shape) * scale).astype(np.float32)


def test_split_keeps_sixteen_bits():
    rng = rng_for(9001)
    for scale in (1e-3, 1.0, 37.0):
        x = _normal_f32(rng, (4096,), scale)
        hi, lo = _split(x)
        x64 = x.astype(np.float64)
        # hi alone: relative rounding <= 2^-8; hi + lo: <= 2^-8 of that
        assert np.all(np.abs(x64 - hi) <= 2.0 ** -8 * np.abs(x64))
        assert np.all(np.abs(x64 - hi - lo) <= 2.0 ** -16 * np.abs(x64))


def test_zero_and_exact_values_split_exactly():
    x = np.array([0.0, 1.0, -2.5, 0.15625, 3.0 * 2.0 ** -10], np.float32)   # all bf16-exact
    hi, lo = _split(x)
    np.testing.assert_array_equal(hi, x.astype(np.float64))
    np.testing.assert_array_equal(lo, 0.0)


def _three_pass(A, B):
    Ah, Al = _split(A)
    Bh, Bl = _split(B)
    return Ah @ Bh + Ah @ Bl + Al @ Bh


def test_three_pass_product_bound():
    """Shapes of the backward's products: a short K (D = 128) and a long one (keys)."""
    rng = rng_for(9002)
    for M, K, N in ((64, 128, 96), (32, 2048, 40)):
        A = _normal_f32(rng, (M, K))
        B = _normal_f32(rng, (K, N), 0.05)
        exact = A.astype(np.float64) @ B.astype(np.float64)
        bound = 3 * 2.0 ** -16 * (np.abs(A.astype(np.float64)) @ np.abs(B.astype(np.float64)))
        err = np.abs(_three_pass(A, B) - exact)
        assert np.all(err <= bound), float(np.max(err / bound))


def test_plain_bf16_operands_miss_the_bound():
    rng = rng_for(9003)
    A = _normal_f32(rng, (64, 512))
    B = _normal_f32(rng, (512, 64))
    exact = A.astype(np.float64) @ B.astype(np.float64)
    bound = 3 * 2.0 ** -16 * (np.abs(A.astype(np.float64)) @ np.abs(B.astype(np.float64)))
    plain = round_bf16(A).astype(np.float64) @ round_bf16(B).astype(np.float64)
    assert np.max(np.abs(plain - exact) / bound) > 2.0
