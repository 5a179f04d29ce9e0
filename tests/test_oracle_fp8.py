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
