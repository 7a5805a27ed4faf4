"""The test-side tolerance for the requantisation of h (tests/parity.py): which E4M3 codes and
block exponents count as correct when the kernel decides on an fp32 h.  CPU only."""
import numpy as np

from oracle import formats as F
from oracle import moe as M
from parity import AMBIG_REL, h_decision_range


def _range(h):
    hq, hexp = M.quantize_blocks(h)
    return h_decision_range(h, hq, hexp)


def test_values_off_boundaries_have_one_answer():
    rng = np.random.default_rng(0)
    h = rng.standard_normal((8, 256))
    lo, hi, own = _range(h)
    amb = lo != hi
    assert amb.mean() < 1e-2                       # a boundary within 2^-16 relative is rare
    assert np.array_equal(lo[~amb], own[~amb]) and np.array_equal(hi[~amb], own[~amb])
    assert np.all((lo <= own) & (own <= hi))


def test_value_on_a_rounding_midpoint_admits_both_neighbours():
    # block amax 448 -> exponent 0; 1.0625 lies halfway between the E4M3 values 1.0 and 1.125
    h = np.zeros((1, 128))
    h[0, 0] = 448.0
    h[0, 1] = 1.0625
    lo, hi, own = _range(h)
    assert own[0, 1] == 1.0                        # ties to the even code
    assert lo[0, 1] == 1.0 and hi[0, 1] == 1.125
    assert lo[0, 0] == hi[0, 0] == 448.0           # the block maximum is representable
    assert np.count_nonzero(lo != hi) == 1


def test_block_amax_on_the_scale_boundary_admits_both_exponents():
    # amax = 448 * 2^3 exactly: exponent 3; a hair above needs exponent 4.  E4M3 keeps its
    # relative resolution under the doubling except in the subnormal range (spacing 2^-9 of
    # the scaled value), where 1.25 * 2^-9 * 2^3 rounds to 2^-6 at exponent 3 but to 2^-5 at 4
    h = np.zeros((1, 128))
    h[0, 0] = 448.0 * 8
    h[0, 1] = 8 * 1.25 * 2.0 ** -9
    lo, hi, own = _range(h)
    p3 = own[0, 1]
    alt = np.ldexp(F.decode_e4m3(F.encode_e4m3(np.ldexp(h[0, 1], -4))), 4)
    assert p3 != alt
    assert lo[0, 1] == min(p3, alt) and hi[0, 1] == max(p3, alt)
    assert AMBIG_REL < 1e-4
