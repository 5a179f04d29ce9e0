"""Locate (and if needed build) libzz for the tests."""
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "zigzag_context_causal_b200", "libzz.so")


def ensure_built():
    if not os.path.exists(LIB):
        import importlib.util
        spec = importlib.util.spec_from_file_location(
            "zz_build", os.path.join(ROOT, "zigzag_context_causal_b200", "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build()
    import zigzag_context_causal_b200 as zz
    return zz
