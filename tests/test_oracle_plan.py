"""Pins for the oracle's metadata and row movement (CPU only).

Every expected value here comes from the zigzag page itself (its c=4 example,
its asserts), from a case worked by hand (tests/golden), or from a property
that must hold for any correct implementation (shard then rerange is the
identity; the causal work per rank is equal for equal blocks).
"""
import json
import os
import random

import numpy as np
import pytest

from oracle import plan as P
from oracle import rerange as R

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _random_cases(n, seed, cps=(1, 2, 3, 4, 5, 8), max_bs=5, max_len=200):
    rng = random.Random(seed)
    for _ in range(n):
        c = rng.choice(cps)
        bs = rng.randint(1, max_bs)
        lens = [rng.randint(2 * c, max_len) for _ in range(bs)]
        yield c, lens


def test_worked_example_c4_assignment_and_order():
    g = _load("zigzag_c4_example.json")
    c = g["cp_size"]
    L = 8 * 5                                      # any multiple of 2c: equal blocks
    p = P.build_metadata(c, L, extend_lens=[L])
    # bs = 1: chunk number == block number
    assert p.zigzag_index == g["rank_blocks"]
    # Gathered buffer = rank 0's blocks, rank 1's blocks, ...
    gathered_blocks = [b for r in range(c) for b in p.zigzag_index[r]]
    assert gathered_blocks == g["gathered_block_order"]
    # The rerange picks, for natural block b, its position in the gathered order.
    expect_rev = [g["gathered_block_order"].index(b) for b in g["reranged_block_order"]]
    assert p.cp_reverse_index == expect_rev == [0, 2, 4, 6, 7, 5, 3, 1]
    # And moving real rows reproduces the page's picture.
    block_of_token = np.repeat(np.arange(2 * c), L // (2 * c))
    gathered = R.ranked_layout(block_of_token, p)
    trimmed = R.trim(gathered, p)
    seen = [int(trimmed[i]) for i in range(0, L, L // (2 * c))]
    assert seen == g["gathered_block_order"]
    assert R.gather_kv(gathered, p).tolist() == block_of_token.tolist()


def test_uneven_case_worked_by_hand():
    g = _load("uneven_c2_lens_10_9.json")
    p = P.build_metadata(g["cp_size"], sum(g["extend_lens"]), extend_lens=g["extend_lens"])
    for key in ("split_list", "zigzag_index", "cp_reverse_index", "reverse_split_len",
                "per_rank_actual_token", "max_rank_len", "kv_len_prev", "kv_len_next",
                "q_len_prev", "q_len_next", "cu_seqlens_q_prev", "cu_seqlens_q_next"):
        assert getattr(p, key) == g[key], key


@pytest.mark.parametrize("seed", range(4))
def test_page_asserts_hold_on_random_batches(seed):
    for c, lens in _random_cases(60, seed):
        p = P.build_metadata(c, sum(lens), extend_lens=lens)
        P.check_invariants(p)
        nblk = 2 * c
        assert all(len(z) == 2 * len(lens) for z in p.zigzag_index)
        # blocks differ by at most one token and the longer ones come first
        for blk, L in zip(p.blocks, lens):
            assert sum(blk) == L and max(blk) - min(blk) <= 1
            assert blk == sorted(blk, reverse=True)
        # every chunk is owned by exactly one rank
        owned = sorted(i for z in p.zigzag_index for i in z)
        assert owned == list(range(len(lens) * nblk))
        assert sum(p.reverse_split_len) == sum(lens)


@pytest.mark.parametrize("seed", range(4))
def test_shard_then_rerange_is_identity(seed):
    """rerange . split == identity, on token ids, over random uneven batches."""
    for c, lens in _random_cases(60, 100 + seed):
        p = P.build_metadata(c, sum(lens), extend_lens=lens)
        ids = np.arange(sum(lens), dtype=np.int64)
        gathered = R.ranked_layout(ids, p)
        assert gathered.shape[0] == c * p.M
        assert R.gather_kv(gathered, p).tolist() == ids.tolist()
        # padding rows are zero and sit at the end of each rank
        for r, n in enumerate(p.per_rank_actual_token):
            assert not gathered[r * p.M + n:(r + 1) * p.M].any()


def test_pool_write_places_every_token():
    c, lens = 3, [50, 37]
    p = P.build_metadata(c, sum(lens), extend_lens=lens)
    rows = np.arange(sum(lens) * 2, dtype=np.int16).reshape(-1, 2)
    loc = np.random.default_rng(0).permutation(200)[: sum(lens)]
    pool = np.full((200, 2), -7, dtype=np.int16)
    out = R.rerange_to_pool(R.ranked_layout(rows, p), p, pool, loc)
    assert (out[loc] == rows).all()
    untouched = np.setdiff1d(np.arange(200), loc)
    assert (out[untouched] == -7).all()


@pytest.mark.parametrize("c", [2, 3, 4, 8])
def test_closed_forms(c):
    L = 2 * c * 7 + 3
    p = P.build_metadata(c, L, extend_lens=[L])
    b = p.blocks[0]
    assert p.kv_len_next[0][0] == L                   # rank 0's next block is the last one
    assert p.kv_len_prev[0][0] == b[0]
    assert p.kv_len_next[c - 1][0] - p.kv_len_prev[c - 1][0] == b[c]
    for r in range(c):
        assert p.kv_len_prev[r][0] == sum(b[: r + 1])
        assert p.kv_len_next[r][0] == L - sum(b[2 * c - r:])
        assert p.q_len_prev[r][0] + p.q_len_next[r][0] == p.per_rank_actual_token[r]


@pytest.mark.parametrize("c,B", [(2, 5), (4, 16), (8, 3)])
def test_equal_blocks_give_equal_causal_work(c, B):
    """With equal blocks of size B every rank sees B^2(2c-1) + B(B+1) pairs."""
    from oracle.attention import causal_pairs
    L = 2 * c * B
    p = P.build_metadata(c, L, extend_lens=[L])
    for r in range(c):
        pairs = (causal_pairs(p.q_len_prev[r][0], p.kv_len_prev[r][0])
                 + causal_pairs(p.q_len_next[r][0], p.kv_len_next[r][0]))
        assert pairs == B * B * (2 * c - 1) + B * (B + 1)


def test_pad_fold_in_and_prefix():
    # pad goes to the last sequence (and to seqs_len[-1] when the lists match)
    p = P.build_metadata(2, 30, seqs_len=[12, 15], extend_lens=[10, 15])
    assert p.extend_lens == [10, 20]
    assert p.prefix == [2, 0]
    assert sum(p.split_list) == 30
    assert p.kv_len_next[0] == [12, 20]
    assert p.kv_len_prev[1][0] == 2 + sum(p.blocks[0][:2])
    # seqs_len shorter than extend -> prefix clamps at 0
    p = P.build_metadata(2, 20, seqs_len=[5, 5], extend_lens=[10, 10])
    assert p.prefix == [0, 0]
    # seqs_len of another length -> no prefix
    p = P.build_metadata(2, 20, seqs_len=[30], extend_lens=[10, 10])
    assert p.prefix == [0, 0]
    # no extend list: one sequence of num_tokens
    p = P.build_metadata(2, 9)
    assert p.extend_lens == [9] and p.blocks == [[3, 2, 2, 2]]


def test_can_apply():
    assert not P.can_apply(1, 100, [100])
    assert not P.can_apply(4, 7, None)
    assert P.can_apply(4, 8, None)
    assert not P.can_apply(4, 100, [50, 7, 43])
    assert P.can_apply(4, 100, [50, 8, 42])
