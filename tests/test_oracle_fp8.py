"""Pins for the oracle's E4M3 encoder (CPU)."""
import numpy as np
import torch

from oracle import fp8


def test_every_finite_code_round_trips():
    codes = np.arange(256, dtype=np.uint8)
    vals = fp8.decode(codes)
    finite = ~np.isnan(vals)
    assert finite.sum() == 254
    back = fp8.encode(vals[finite].astype(np.float32))
    # +0 and -0 are distinct codes and both survive
    assert np.array_equal(back, codes[finite])
    assert vals[0x7E] == 448.0 and vals[0xFE] == -448.0 and vals[0x01] == 2.0 ** -9


def test_matches_torch_cast_inside_the_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200000) * s for s in (1e-3, 0.05, 1.0, 30.0, 200.0)])
    x = x[np.abs(x) <= 440].astype(np.float32)
    ours = fp8.encode(x)
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, lib)


def test_ties_round_to_even_and_overflow_saturates():
    x = np.array([2.0 ** -10, 3 * 2.0 ** -10, 1.0 + 1 / 16, 1.0 + 3 / 16, 449.0, 463.9, 464.0,
                  1e6, -1e6, 0.0, -0.0], np.float32)
    got = fp8.encode(x)
    want = [0x00, 0x02, 0x38, 0x3A, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x00, 0x80]
    assert got.tolist() == want
    assert fp8.encode(np.array([np.nan], np.float32))[0] == 0x7F


# ---------------------------------------------------------------- the scale step
# The pool value is e4m3(fp32(x) / fp32(scale)) (zigzag.py, materialize_full_kv
# hands layer.k_scale / layer.v_scale to set_kv_buffer; the division is read as
# rounded once in fp32).  The expected codes below are fixed by arithmetic, not
# by calling the encoder:
#   * 1.125 / 0.375 = 3 exactly, and 3.0 = 1.5 * 2^1 is code 0.1000.100 = 0x44;
#   * 125 / 0.25 = 500 > 448: finite overflow saturates to 0x7E (0xFE negative);
#   * pairs whose exact quotient lies within half an fp32 ulp of an E4M3 tie
#     (1.0625 between 1.0 = 0x38 and 1.125 = 0x39; 1.1875 between 1.125 = 0x39
#     and 1.25 = 0x3A).  Rounded in fp32 the quotient IS the tie, which goes to
#     the even mantissa (0x38, 0x3A); an encoder fed the exact or fp64 quotient
#     rounds the other way (0x39 both times).
from fractions import Fraction

import pytest

TIE_ABOVE = (0.50390625, 0.4742646813392639, Fraction(17, 16), 0x38)   # quotient just above 1.0625
TIE_BELOW = (0.5, 0.42105263471603394, Fraction(19, 16), 0x3A)         # quotient just below 1.1875


def _check_scale_pins(scale_encode):
    assert scale_encode(np.array([1.125], np.float32), 0.375)[0] == 0x44
    assert scale_encode(np.array([-1.125], np.float32), 0.375)[0] == 0xC4
    assert scale_encode(np.array([125.0, -125.0], np.float32), 0.25).tolist() == [0x7E, 0xFE]
    assert scale_encode(np.array([np.nan], np.float32), 0.25)[0] == 0x7F
    for x, s, tie, code in (TIE_ABOVE, TIE_BELOW):
        assert scale_encode(np.array([x], np.float32), s)[0] == code


def test_tie_fixtures_sit_within_half_an_fp32_ulp_of_the_tie():
    """The fixtures really are the cases described (exact rational arithmetic)."""
    half_ulp = Fraction(1, 2 ** 24)           # fp32 spacing in [1, 2) is 2^-23
    for x, s, tie, _ in (TIE_ABOVE, TIE_BELOW):
        assert float(np.float32(x)) == x and float(np.float32(s)) == s
        assert float(torch.tensor(x).to(torch.bfloat16).float()) == x   # x is a bf16 value
        gap = Fraction(x) / Fraction(s) - tie
        assert gap != 0 and abs(gap) < half_ulp
    assert (Fraction(TIE_ABOVE[0]) / Fraction(TIE_ABOVE[1])) > TIE_ABOVE[2]
    assert (Fraction(TIE_BELOW[0]) / Fraction(TIE_BELOW[1])) < TIE_BELOW[2]


def test_scale_encode_divides_once_in_fp32():
    _check_scale_pins(fp8.scale_encode)


@pytest.mark.parametrize("mistake", ["multiply", "fp64-divide", "scale-as-bf16"])
def test_planted_scale_mistakes_are_caught(mistake):
    def wrong(x, scale):
        x = np.asarray(x, np.float32)
        if mistake == "multiply":
            return fp8.encode(x * np.float32(scale))
        if mistake == "fp64-divide":
            return fp8.encode(x.astype(np.float64) / float(scale))
        s16 = float(torch.tensor(scale).to(torch.bfloat16).float())
        return fp8.encode((x / np.float32(s16)).astype(np.float32))
    with pytest.raises(AssertionError):
        _check_scale_pins(wrong)
