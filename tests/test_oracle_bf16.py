"""Pins for oracle.bf16: round-to-nearest-even to bfloat16 (the IEEE rule)."""
import numpy as np

from oracle.bf16 import rnd, rnd32


def _bits_rne_from_f32(x32):
    """Independent RNE on float32 bit patterns: keep the top 16 bits."""
    b = x32.view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def test_hand_values():
    # ties go to even, values above a tie go up, pi -> 3.140625
    assert rnd([1.0 + 2.0 ** -8])[0] == 1.0
    assert rnd([1.0 + 3 * 2.0 ** -8])[0] == 1.0 + 2.0 ** -6
    assert rnd([1.0 + 3 * 2.0 ** -9])[0] == 1.0 + 2.0 ** -7
    assert rnd([np.pi])[0] == 3.140625
    assert rnd([-np.pi])[0] == -3.140625
    assert rnd([65504.0])[0] == 65536.0
    assert np.isinf(rnd([1e39])[0])
    assert rnd([0.0])[0] == 0.0 and np.signbit(rnd([-0.0])[0])


def test_single_rounding_from_float64():
    # just above a tie in float64 but exactly a tie after a float32 rounding
    x = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert rnd32([x])[0] == 1.0 + 2.0 ** -8
    assert rnd([x])[0] == 1.0 + 2.0 ** -7


def test_matches_bit_rule_on_float32_inputs():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(200000) * 10.0 ** rng.uniform(-30, 30, 200000)).astype(np.float32)
    x = x[np.isfinite(x)]
    np.testing.assert_array_equal(rnd(x.astype(np.float64)), _bits_rne_from_f32(x))


def test_subnormals():
    q = 2.0 ** -133        # bfloat16 subnormal spacing
    assert rnd([2.5 * q])[0] == 2 * q
    assert rnd([3.5 * q])[0] == 4 * q
    assert rnd([0.4 * q])[0] == 0.0


def test_idempotent_and_nonfinite():
    rng = np.random.default_rng(2)
    x = rnd(rng.standard_normal(1000))
    np.testing.assert_array_equal(rnd(x), x)
    out = rnd([np.nan, np.inf, -np.inf])
    assert np.isnan(out[0]) and out[1] == np.inf and out[2] == -np.inf
