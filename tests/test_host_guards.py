"""Host-side guards (CPU only).

* The Python package has no fallback: without libzz.so next to it, importing
  it raises ImportError.
* No product module imports the oracle (it is test infrastructure).
* bench.py reports ncu traffic only while the kernel source it was taken from
  is unchanged (the recorded hash must match).
"""
import importlib.util
import json
import os
import re
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "zigzag_context_causal_b200")


def test_package_refuses_to_import_without_its_library(tmp_path):
    dst = tmp_path / "zigzag_context_causal_b200"
    dst.mkdir()
    shutil.copy(os.path.join(PKG, "__init__.py"), dst / "__init__.py")
    spec = importlib.util.spec_from_file_location("zz_nolib", dst / "__init__.py",
                                                  submodule_search_locations=[str(dst)])
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError, match="libzz.so not found"):
        spec.loader.exec_module(mod)


def test_product_code_does_not_import_the_oracle():
    pattern = re.compile(r"^\s*(from|import)\s+oracle\b", re.M)
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith(".py"):
                with open(os.path.join(dirpath, f)) as fh:
                    assert not pattern.search(fh.read()), f"{f} imports the oracle"


def test_traffic_is_reported_only_for_the_recorded_source(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    try:
        import bench
    finally:
        sys.path.remove(ROOT)
    prof = tmp_path / "profiles"
    prof.mkdir()
    csrc = tmp_path / "zigzag_context_causal_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.KERNEL_SOURCES["rerange_standalone"]:
        shutil.copy(os.path.join(PKG, "csrc", name), csrc / name)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    good = bench.kernel_source_hash("rerange_standalone")
    entry = {"kernel": "rerange_standalone", "dram_bytes_per_launch": 123, "source_sha256": good}
    (prof / "traffic.json").write_text(json.dumps({"rerange_standalone": entry}))
    assert bench.load_traffic("rerange_standalone") == 123
    assert bench.load_traffic("attn_long") is None                      # no entry
    with open(csrc / "rerange.cu", "a") as fh:                            # the kernel changes
        fh.write("\n// edited\n")
    assert bench.load_traffic("rerange_standalone") is None
