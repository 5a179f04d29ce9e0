"""Plain CPU oracle for zigzag context-parallel prefill.  TEST INFRASTRUCTURE.

This package is the slow, obviously-correct statement of what the CUDA path
computes.  It is used only by ``tests/``, by ``__graft_entry__.smoke()`` and by
``bench.py``'s CPU-baseline leg; the product path (the ``libzz`` C ABI and its
Python binding) never imports, links or executes it, and shares no code with it.

Sources, by page title and section:
  * "sgl-project--sglang/python/sglang/srt/layers/cp/zigzag.py" — module
    docstring (block assignment and rerange order), ``can_apply``,
    ``build_metadata``, ``shard_hidden_states``, ``gather_kv_cache``,
    ``run_attention``, ``materialize_full_kv``, ``_all_gather_reorganized``;
  * "PR #34485 完整报告" (diffusion AITer backend takes grouped-query K/V),
    implementation section item 1 — the ``num_heads % num_kv_heads == 0`` rule.

Modules:
  ``plan``      — the metadata lists, for every rank (integer arithmetic).
  ``rerange``   — shard, padded all-gather, trim + reverse split/cat, pool write.
  ``attention`` — fp64 causal attention per zigzag half, unsharded reference,
                  and a scalar brute force for tiny inputs.

Every function here is pinned by ``tests/test_oracle_*.py`` to facts the pages
or the mathematics fix (worked example, asserts, closed forms, identity and
union properties, brute force); none is marked "parity unpinned".
"""
from . import plan, rerange, attention  # noqa: F401
