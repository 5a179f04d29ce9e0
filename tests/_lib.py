"""Locate (and if needed build) libzz for the tests."""
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "zigzag_context_causal_b200", "libzz.so")


def ensure_built():
    if not os.path.exists(LIB):
        from zigzag_context_causal_b200.build import build
        build()
    import zigzag_context_causal_b200 as zz
    return zz
