"""The stressed-score bound of the GPU tests adds half a bf16 ulp of the oracle value;
pin that helper against the spacing of adjacent bf16 bit patterns (CPU only)."""
import numpy as np

from gpu_util import half_ulp_bf16
from oracle import ws_oracle as orc


def test_half_ulp_matches_bf16_spacing():
    rng = np.random.default_rng(5)
    # positive normal bf16 patterns (exponent field 1..254), and their negatives
    bits = rng.integers(0x0080, 0x7F7F, size=4000, dtype=np.int64).astype(np.uint16)
    x = orc.bf16_to_f64(bits)
    nxt = orc.bf16_to_f64((bits.astype(np.int64) + 1).astype(np.uint16))
    # the next pattern up is one ulp of x's binade away (also from a binade's top value)
    spacing = nxt - x
    np.testing.assert_array_equal(half_ulp_bf16(x), spacing / 2)
    np.testing.assert_array_equal(half_ulp_bf16(-x), spacing / 2)
    assert half_ulp_bf16(np.array([0.0]))[0] == 0.0
    # the values quoted beside the stressed bound
    assert half_ulp_bf16(np.array([4.2116]))[0] == 2.0 ** -6
    assert half_ulp_bf16(np.array([1.0]))[0] == 2.0 ** -8
