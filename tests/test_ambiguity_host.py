"""The allowance helpers the GPU parity tests use (tests/ambiguity.py) on
hand-built blocks, on the CPU: an element gets an allowance only when a
value inside its error band could round to another E4M3 code, or its block's
amax could select another scale, and the allowance is exactly the change of
the dequantised value."""
import numpy as np

from . import ambiguity as amb


def _block(vals):
    v = np.zeros((1, 32))
    v[0, :len(vals)] = vals
    return v


def test_no_band_no_allowance():
    rng = np.random.default_rng(0)
    v = rng.standard_normal((4, 64))
    assert np.all(amb.code_ambiguity(v, np.zeros_like(v)) == 0.0)


def test_rounding_tie_inside_the_band():
    # block amax 384 (an E4M3 value) -> scale 2^0; 3.125 is the midpoint of the codes 3.0 and 3.25
    v = _block([384.0, 3.125, 3.0625])
    band = np.full_like(v, 1e-6)
    D = amb.code_ambiguity(v, band)
    assert D[0, 1] == 0.25          # 3.125 may come out as 3.0 or 3.25
    assert D[0, 2] == 0.0           # 3.0625 rounds to 3.0 from anywhere in its band
    assert D[0, 0] == 0.0


def test_scale_boundary_inside_the_band():
    # amax exactly 448 = largest E4M3 at scale 2^0; a larger amax selects 2^1,
    # where 13 * 2^-9 is a tie between subnormal codes and decodes to 12 * 2^-9
    v = _block([448.0, 13 * 2.0 ** -9])
    band = np.zeros_like(v)
    band[0, 0] = 1e-9
    D = amb.code_ambiguity(v, band)
    assert D[0, 1] == 2.0 ** -9
    far = _block([440.0, 13 * 2.0 ** -9])
    assert np.all(amb.code_ambiguity(far, band) == 0.0)


def test_bf16_alternatives_bracket_the_value():
    a = np.array([1.0, 1.0 + 2.0 ** -8, 3.0])        # 1 + 2^-8 is a bf16 tie (between 1 and 1 + 2^-7)
    lo, hi = amb.bf16_alternatives(a, np.full(3, 1e-12))
    assert lo[0] == hi[0] == 1.0 and lo[2] == hi[2] == 3.0
    assert lo[1] == 1.0 and hi[1] == 1.0 + 2.0 ** -7


def test_within_subtracts_the_allowance():
    ref = np.array([1.0, -1.0, 1.0, -1.0])
    gpu = ref + np.array([0.125, 0.0, 0.0, 0.0])
    assert amb.within(gpu, ref, 0.0, np.zeros(4), bf16_out=False) == 0.125
    assert amb.within(gpu, ref, 0.0, np.array([0.125, 0, 0, 0]), bf16_out=False) == 0.0
    # bf16 outputs also allow half a bf16 ulp of the reference (2^-8 |ref|)
    assert amb.within(ref + 2.0 ** -8, ref, 0.0, np.zeros(4)) == 0.0
