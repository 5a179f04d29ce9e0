"""Planted mistakes in the oracle must be caught by the pins (CPU only).

Each case perturbs one step of the oracle the way a plausible bug would
(an off-by-one mask, a transposed head mapping, a wrong rerange index, a
dropped term in a kv length) and checks that the corresponding pin rejects it.
"""
import numpy as np
import pytest

from oracle import attention as A
from oracle import plan as P
from oracle import rerange as R


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_off_by_one_mask_is_caught_by_brute_force(monkeypatch):
    lq, kv_len, d = 4, 9, 3
    q, k, v = _rand((lq, 1, d), 0), _rand((kv_len, 1, d), 1), _rand((kv_len, 1, d), 2)
    good = A.brute_force(q, k, v, kv_len, 0.5)
    real = A.attention_rows

    def shifted(q_rows, rows, k_, v_, kv_len_, lq_, scale, causal=True):   # sees one key too few
        return real(q_rows, rows, k_, v_, kv_len_ - 1, lq_, scale, causal)
    monkeypatch.setattr(A, "attention_rows", shifted)
    bad, _ = A.attention_half(q, k, v, kv_len, 0.5)
    assert np.abs(bad - good).max() > 1e-3


def test_modulo_head_mapping_is_caught_by_gqa_pin():
    lq, kv_len, h_kv, g, d = 5, 8, 2, 3, 4
    q = _rand((lq, h_kv * g, d), 3)
    k, v = _rand((kv_len, h_kv, d), 4), _rand((kv_len, h_kv, d), 5)
    # h % h_kv instead of h // g, written as an explicit head repeat
    wrong_k = k[:, [h % h_kv for h in range(h_kv * g)]]
    wrong_v = v[:, [h % h_kv for h in range(h_kv * g)]]
    o_wrong, _ = A.attention_half(q, wrong_k, wrong_v, kv_len, 0.5)
    o_right, _ = A.attention_half(q, np.repeat(k, g, 1), np.repeat(v, g, 1), kv_len, 0.5)
    assert np.abs(o_wrong - o_right).max() > 1e-3


def test_swapped_reverse_index_is_caught_by_identity_pin():
    p = P.build_metadata(3, 41, extend_lens=[41])
    ids = np.arange(41)
    p.cp_reverse_index[3], p.cp_reverse_index[4] = p.cp_reverse_index[4], p.cp_reverse_index[3]
    assert R.gather_kv(R.ranked_layout(ids, p), p).tolist() != ids.tolist()


def test_dropped_own_block_in_kv_len_is_caught_by_closed_form():
    c, L = 4, 2 * 4 * 7 + 3
    p = P.build_metadata(c, L, extend_lens=[L])
    b = p.blocks[0]
    wrong = [sum(b[:r]) for r in range(c)]                 # forgets block r itself
    assert any(w != p.kv_len_prev[r][0] for r, w in enumerate(wrong))
    assert wrong[0] != b[0]


def test_top_left_mask_is_caught_by_union_pin():
    """Aligning the mask top-left (row i sees keys 0..i) breaks the union pin."""
    c, L, d = 2, 24, 4
    p = P.build_metadata(c, L, extend_lens=[L])
    q, k, v = _rand((L, 1, d), 6), _rand((L, 1, d), 7), _rand((L, 1, d), 8)
    ref, _ = A.full_causal(q, k, v, 0.5)
    r = 1
    ql = R.shard(q, p, r)
    lq = p.q_len_next[r][0]
    top_left = A.brute_force(ql[p.total_q_prev[r]:], k, v, lq, 0.5)   # kv_len := Lq
    rows = [i for i, t in enumerate(R.shard(np.arange(L), p, r)) if i >= p.total_q_prev[r]]
    tokens = R.shard(np.arange(L), p, r)[rows]
    assert np.abs(top_left - ref[tokens]).max() > 1e-3


def test_dropped_prefix_in_kv_len_is_caught_by_prefix_union_pin():
    """kv lengths that forget the cached prefix shift every row's key window."""
    c, ext, pre, d = 2, [23, 17], [5, 9], 8
    full = [e + q for e, q in zip(ext, pre)]
    p = P.build_metadata(c, sum(ext), seqs_len=full, extend_lens=ext)
    q_all = [_rand((n, 2, d), 70 + s) for s, n in enumerate(full)]
    k_all = [_rand((n, 1, d), 80 + s) for s, n in enumerate(full)]
    v_all = [_rand((n, 1, d), 90 + s) for s, n in enumerate(full)]
    q_ext = np.concatenate([q_all[s][pre[s]:] for s in range(2)])
    for kv in (p.kv_len_prev, p.kv_len_next):        # the planted mistake
        for r in range(c):
            kv[r] = [kv[r][s] - pre[s] for s in range(2)]
    per_rank = [A.run_rank(p, r, R.shard(q_ext, p, r), k_all, v_all, 0.5)[0] for r in range(c)]
    o_tok = R.gather_kv(R.all_gather_padded(per_rank, p), p)
    ref = np.concatenate([A.full_causal(q_all[s], k_all[s], v_all[s], 0.5)[0][pre[s]:] for s in range(2)])
    assert np.abs(o_tok - ref).max() > 1e-3
