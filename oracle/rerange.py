"""Row movement of zigzag CP, restated with numpy.  TEST INFRASTRUCTURE.

Follows "sgl-project--sglang/python/sglang/srt/layers/cp/zigzag.py":
``shard_hidden_states`` (split by ``split_list``, concatenate in
``zigzag_index`` order), ``_all_gather_reorganized`` (zero-pad every rank to
``max_rank_len``, all-gather in rank order, trim each rank back to its own
token count), ``gather_kv_cache`` (split the trimmed buffer by
``reverse_split_len``, concatenate in ``cp_reverse_index`` order) and
``materialize_full_kv`` (write the result into the pool at ``out_cache_loc``).

Every function moves whole rows and never looks at their values, so any dtype
works; bf16 data is handled as its 16-bit patterns, which makes every
comparison byte-exact.
"""
from __future__ import annotations

import numpy as np

from .plan import Plan


def _split(x: np.ndarray, sizes) -> list:
    out, at = [], 0
    for n in sizes:
        out.append(x[at:at + n])
        at += n
    assert at == x.shape[0], "split sizes must cover the rows exactly"
    return out


def shard(x_natural: np.ndarray, plan: Plan, rank: int) -> np.ndarray:
    """Rows of rank ``rank`` in rank-local order: its prev block of every
    sequence, then its next block of every sequence (``shard_hidden_states``)."""
    chunks = _split(x_natural, plan.split_list)
    return np.concatenate([chunks[i] for i in plan.zigzag_index[rank]], axis=0)


def all_gather_padded(locals_: list, plan: Plan) -> np.ndarray:
    """What ``all_gather_into_tensor`` delivers: every rank's rows zero-padded
    to ``max_rank_len`` and stacked in rank order, ``[c*M, ...]``."""
    M = plan.M
    parts = []
    for x in locals_:
        pad = np.zeros((M - x.shape[0],) + x.shape[1:], dtype=x.dtype)
        parts.append(np.concatenate([x, pad], axis=0))
    return np.concatenate(parts, axis=0)


def trim(gathered: np.ndarray, plan: Plan) -> np.ndarray:
    """Drop the padding: rank r keeps its first ``per_rank_actual_token[r]`` rows."""
    M = plan.M
    return np.concatenate(
        [gathered[r * M: r * M + n] for r, n in enumerate(plan.per_rank_actual_token)], axis=0)


def gather_kv(gathered: np.ndarray, plan: Plan) -> np.ndarray:
    """Rank-ordered padded buffer -> natural token order (``gather_kv_cache``)."""
    chunks = _split(trim(gathered, plan), plan.reverse_split_len)
    return np.concatenate([chunks[i] for i in plan.cp_reverse_index], axis=0)


def write_pool(pool: np.ndarray, out_cache_loc: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """``set_kv_buffer`` with unit scales: ``pool[out_cache_loc[t]] = rows[t]``."""
    pool = pool.copy()
    pool[np.asarray(out_cache_loc, dtype=np.int64)] = rows
    return pool


def rerange_to_pool(gathered: np.ndarray, plan: Plan, pool: np.ndarray,
                    out_cache_loc: np.ndarray) -> np.ndarray:
    """``materialize_full_kv`` for one tensor: gather, rerange, write the pool."""
    return write_pool(pool, out_cache_loc, gather_kv(gathered, plan))


def ranked_layout(x_natural: np.ndarray, plan: Plan) -> np.ndarray:
    """All ranks' local rows, padded to ``M`` and stacked: ``[c*M, ...]``.

    For Q this is the virtual-rank layout that one launch over all ranks
    reads; for K and V it is the all-gathered buffer."""
    return all_gather_padded([shard(x_natural, plan, r) for r in range(plan.cp_size)], plan)
