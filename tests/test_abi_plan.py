"""C-ABI library on the CPU: exported symbols, planner parity with the oracle,
and the error contract.  No compute kernel is launched here."""
import ctypes
import random

import numpy as np
import pytest

from oracle import plan as P
from oracle import rerange as R
from tests._lib import ensure_built

zz = ensure_built()


def test_every_header_function_is_exported():
    names = zz.header_functions()
    assert len(names) >= 11
    lib = ctypes.CDLL(zz.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def _cases(n, seed):
    rng = random.Random(seed)
    for _ in range(n):
        c = rng.choice([2, 3, 4, 5, 8])
        bs = rng.randint(1, 6)
        lens = [rng.randint(2 * c, 300) for _ in range(bs)]
        yield c, lens


FIELDS = ["extend_lens", "prefix", "split_list", "cp_reverse_index", "reverse_split_len",
          "per_rank_actual_token", "max_rank_len"]
RANK_FIELDS = {"zigzag_index": "zigzag_index", "kv_len_prev": "kv_len_prev",
               "kv_len_next": "kv_len_next", "q_len_prev": "q_len_prev", "q_len_next": "q_len_next",
               "cu_seqlens_q_prev": "cu_seqlens_q_prev", "cu_seqlens_q_next": "cu_seqlens_q_next"}


@pytest.mark.parametrize("seed", range(3))
def test_planner_matches_oracle_bit_exact(seed):
    for c, lens in _cases(40, seed):
        ref = P.build_metadata(c, sum(lens), extend_lens=lens)
        plan = zz.Plan(c, extend_lens=lens)
        assert plan.M == ref.M
        for f in FIELDS:
            want = getattr(ref, "prefix" if f == "prefix" else f)
            assert plan.get(f) == list(want), f
        for f, attr in RANK_FIELDS.items():
            assert plan.get_all_ranks(f) == getattr(ref, attr), f
        # natural token -> ranked row map equals the oracle's shard + padded gather
        ids = np.arange(sum(lens))
        ranked = R.ranked_layout(ids + 1, ref)          # 0 marks padding
        src_row = np.array(plan.get("src_row"))
        assert (ranked[src_row] == ids + 1).all()
        # ranked row -> natural token (the push form's table) is the same layout, -1 on padding
        rank_tok = np.array(plan.get("rank_tok"))
        assert (rank_tok + 1 == ranked).all()
        for r in range(c):
            info = plan.info(r)
            assert info.total_q_prev == ref.total_q_prev[r]
            assert info.total_q_next == ref.total_q_next[r]
            assert info.max_seqlen_q_prev == ref.max_seqlen_q_prev[r]
            assert info.max_seqlen_q_next == ref.max_seqlen_q_next[r]


def test_planner_pad_fold_in_and_prefix_match_oracle():
    for c, ext, seqs, n in [(2, [10, 15], [12, 15], 30), (3, [40, 22], [50, 30], 70),
                            (4, [64], None, 70), (2, [9, 9], [5, 5], 18)]:
        ref = P.build_metadata(c, n, seqs_len=seqs, extend_lens=ext)
        plan = zz.Plan(c, extend_lens=ext, seq_lens=seqs, num_tokens=n)
        assert plan.get("extend_lens") == ref.extend_lens
        assert plan.get("prefix") == ref.prefix
        assert plan.get_all_ranks("kv_len_prev") == ref.kv_len_prev
        assert plan.get_all_ranks("kv_len_next") == ref.kv_len_next


def test_worked_uneven_example_through_the_abi():
    plan = zz.Plan(2, extend_lens=[10, 9])
    assert plan.get("split_list") == [3, 3, 2, 2, 3, 2, 2, 2]
    assert plan.get_all_ranks("zigzag_index") == [[0, 4, 3, 7], [1, 5, 2, 6]]
    assert plan.get("cp_reverse_index") == [0, 4, 6, 2, 1, 5, 7, 3]
    assert plan.get("kv_len_prev", 1) == [6, 5] and plan.get("kv_len_next", 1) == [8, 7]


@pytest.mark.parametrize("c,n,lens", [(1, 100, [100]), (4, 7, None), (4, 100, [50, 7, 43])])
def test_not_applicable(c, n, lens):
    with pytest.raises(zz.ZZError) as e:
        zz.Plan(c, extend_lens=lens, num_tokens=n)
    assert e.value.status == zz.ZZ_ERR_NOT_APPLICABLE


def test_invalid_plan_arguments():
    with pytest.raises(zz.ZZError) as e:
        zz.Plan(2, extend_lens=[10, 10], num_tokens=15)      # num_tokens < sum
    assert e.value.status == zz.ZZ_ERR_INVALID_ARG
    with pytest.raises(zz.ZZError) as e:
        zz.Plan(2, extend_lens=[10, -4], num_tokens=15)
    assert e.value.status == zz.ZZ_ERR_INVALID_ARG


def test_head_ratio_contract_needs_no_gpu():
    """num_heads % num_kv_heads != 0 is rejected before any device work."""
    plan = zz.Plan(2, extend_lens=[64])
    fake = ctypes.c_void_p(1 << 20)
    for h_q, h_kv, want in [(32, 5, zz.ZZ_ERR_INVALID_ARG)]:
        st = zz.raw_call("zz_attn_prefill", plan.handle, 0, 2, fake, fake, fake, 1024, fake, 8, 16,
                         fake, None, h_q, h_kv, 128, ctypes.c_float(0.0), zz.ZZ_BF16, None)
        assert st == want
        assert "multiple of num_kv_heads" in zz.last_error()


def test_workspace_layout_is_256_aligned_and_covers_tables():
    plan = zz.Plan(8, extend_lens=[131072])
    nbytes = plan.workspace_bytes()
    assert nbytes % 256 == 0
    assert nbytes >= 4 * 131072
