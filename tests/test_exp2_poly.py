"""Pins for the FMA-pipe 2^x the attention kernel uses for part of its
exponentials (CPU, numpy float32 emulation of the same steps)."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "zigzag_context_causal_b200", "csrc")


def _header_coeffs():
    text = open(os.path.join(CSRC, "exp2_poly.h")).read()
    return [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f", text).group(1))) for i in range(4)]


def _generator():
    spec = importlib.util.spec_from_file_location("gen", os.path.join(CSRC, "gen_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _emulate(x, c):
    """The kernel's steps in float32: clamp, round via 1.5*2^23, Horner, exponent add."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = (x - r).astype(np.float32)
    p = ((c[3] * f + c[2]).astype(np.float32) * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = p.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << 23) & 0xFFFFFFFF)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_header_matches_generator():
    gen = _generator()
    want = [np.float32(v) for v in gen.coefficients()]
    assert _header_coeffs() == want
    assert gen.max_rel_error(gen.coefficients()) < 1.1e-4


def test_polynomial_exp2_error_bound_over_softmax_range():
    c = _header_coeffs()
    x = np.linspace(-120.0, 8.0, 400001, dtype=np.float32)
    got = _emulate(x, c).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 2e-4           # far below bf16's 2^-9 relative rounding of P
    assert _emulate(np.zeros(1, np.float32), c)[0] == np.float32(c[0])


def test_masked_entries_vanish():
    c = _header_coeffs()
    out = _emulate(np.array([-np.inf, -1e30, -126.0, -200.0], np.float32), c)
    assert np.all(np.isfinite(out)) and np.all(out >= 0) and np.all(out < 1e-37)
