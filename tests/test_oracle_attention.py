"""Pins for the oracle's fp64 attention (CPU only).

  * brute force: a scalar math.exp/math.fsum loop on tiny inputs;
  * union: every rank's prev/next outputs, moved back to token order, equal
    plain causal attention over the whole sequence;
  * single-key rows: the first query of block 0 sees one key, so o = v0;
  * GQA reduces to MHA with each K/V head repeated G times;
  * log-sum-exp against scipy's logsumexp;
  * outputs are convex combinations of V rows.
"""
import numpy as np
import pytest
from scipy.special import logsumexp

from oracle import attention as A
from oracle import plan as P
from oracle import rerange as R


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_brute_force_matches_numpy_path():
    lq, kv_len, h_q, h_kv, d = 5, 13, 4, 2, 6
    q = _rand((lq, h_q, d), 1)
    k = _rand((kv_len, h_kv, d), 2)
    v = _rand((kv_len, h_kv, d), 3)
    o, _ = A.attention_half(q, k, v, kv_len, 0.37)
    ob = A.brute_force(q, k, v, kv_len, 0.37)
    assert np.abs(o - ob).max() < 1e-13


def test_brute_force_on_a_zigzag_rank():
    c, lens, h_q, h_kv, d = 2, [11, 9], 2, 1, 4
    p = P.build_metadata(c, sum(lens), extend_lens=lens)
    q = _rand((sum(lens), h_q, d), 4)
    k = _rand((sum(lens), h_kv, d), 5)
    v = _rand((sum(lens), h_kv, d), 6)
    starts = np.cumsum([0] + lens)
    ks = [k[starts[s]:starts[s + 1]] for s in range(2)]
    vs = [v[starts[s]:starts[s + 1]] for s in range(2)]
    for r in range(c):
        o, _ = A.run_rank(p, r, R.shard(q, p, r), ks, vs, 0.5)
        # rebuild the same rows by brute force, half by half
        ql = R.shard(q, p, r)
        rows = []
        for kv_len, cu, base in ((p.kv_len_prev[r], p.cu_seqlens_q_prev[r], 0),
                                 (p.kv_len_next[r], p.cu_seqlens_q_next[r], p.total_q_prev[r])):
            for s in range(2):
                rows.append(A.brute_force(ql[base + cu[s]: base + cu[s + 1]], ks[s], vs[s],
                                          kv_len[s], 0.5))
        assert np.abs(o - np.concatenate(rows)).max() < 1e-13


@pytest.mark.parametrize("c,lens,h_q,h_kv", [(2, [64], 4, 4), (3, [37, 50], 4, 2),
                                             (4, [71, 40, 33], 8, 1)])
def test_union_of_halves_equals_unsharded(c, lens, h_q, h_kv):
    d = 8
    p = P.build_metadata(c, sum(lens), extend_lens=lens)
    q = _rand((sum(lens), h_q, d), 7)
    k = _rand((sum(lens), h_kv, d), 8)
    v = _rand((sum(lens), h_kv, d), 9)
    starts = np.cumsum([0] + lens)
    ks = [k[starts[s]:starts[s + 1]] for s in range(len(lens))]
    vs = [v[starts[s]:starts[s + 1]] for s in range(len(lens))]
    scale = d ** -0.5
    per_rank = [A.run_rank(p, r, R.shard(q, p, r), ks, vs, scale) for r in range(c)]
    o_ranked = R.all_gather_padded([o for o, _ in per_rank], p)
    lse_ranked = R.all_gather_padded([l for _, l in per_rank], p)
    o_tok = R.gather_kv(o_ranked, p)
    lse_tok = R.gather_kv(lse_ranked, p)
    ref_o = np.concatenate([A.full_causal(q[starts[s]:starts[s + 1]], ks[s], vs[s], scale)[0]
                            for s in range(len(lens))])
    ref_l = np.concatenate([A.full_causal(q[starts[s]:starts[s + 1]], ks[s], vs[s], scale)[1]
                            for s in range(len(lens))])
    assert np.abs(o_tok - ref_o).max() < 1e-12
    assert np.abs(lse_tok - ref_l).max() < 1e-12


def test_first_query_of_block0_returns_v0_exactly():
    c, L = 4, 64
    p = P.build_metadata(c, L, extend_lens=[L])
    q = _rand((L, 2, 8), 10) * 30.0
    k = _rand((L, 2, 8), 11)
    v = _rand((L, 2, 8), 12)
    o, lse = A.run_rank(p, 0, R.shard(q, p, 0), [k], [v], 1.0)
    assert (o[0] == v[0]).all()                       # rank 0 prev half row 0: one key
    s0 = np.einsum("hd,hd->h", q[0], k[0])
    assert np.abs(lse[0] - s0).max() < 1e-12


def test_gqa_equals_mha_with_repeated_heads():
    lq, kv_len, h_kv, g, d = 9, 20, 2, 4, 8
    q = _rand((lq, h_kv * g, d), 13)
    k = _rand((kv_len, h_kv, d), 14)
    v = _rand((kv_len, h_kv, d), 15)
    o_gqa, _ = A.attention_half(q, k, v, kv_len, 0.3)
    o_mha, _ = A.attention_half(q, np.repeat(k, g, axis=1), np.repeat(v, g, axis=1), kv_len, 0.3)
    assert np.abs(o_gqa - o_mha).max() < 1e-14
    with pytest.raises(ValueError, match="multiple of num_kv_heads"):
        A.attention_half(_rand((3, 32, 4), 0), _rand((3, 5, 4), 1), _rand((3, 5, 4), 2), 3, 1.0)


def test_lse_and_convexity():
    lq, kv_len, d = 6, 15, 5
    q = _rand((lq, 1, d), 16)
    k = _rand((kv_len, 1, d), 17)
    v = _rand((kv_len, 1, d), 18)
    o, lse = A.attention_half(q, k, v, kv_len, 0.7)
    for i in range(lq):
        last = kv_len - lq + i
        s = 0.7 * (k[: last + 1, 0] @ q[i, 0])
        assert abs(lse[i, 0] - logsumexp(s)) < 1e-12
        vis = v[: last + 1, 0]
        assert (o[i, 0] <= vis.max(0) + 1e-12).all() and (o[i, 0] >= vis.min(0) - 1e-12).all()


def test_sampled_rows_equal_full_half():
    lq, kv_len, d = 40, 100, 8
    q = _rand((lq, 2, d), 19)
    k = _rand((kv_len, 1, d), 20)
    v = _rand((kv_len, 1, d), 21)
    o, l = A.attention_half(q, k, v, kv_len, 0.2, row_chunk=7)
    rows = np.array([0, 13, 39])
    o2, l2 = A.attention_rows(q[rows], rows, k, v, kv_len, lq, 0.2)
    assert np.abs(o[rows] - o2).max() < 1e-14 and np.abs(l[rows] - l2).max() < 1e-14


def test_flop_count_closed_form():
    c, B, h_q, d = 4, 16, 8, 64
    L = 2 * c * B
    p = P.build_metadata(c, L, extend_lens=[L])
    assert A.plan_flops(p, h_q, d) == 4 * d * h_q * (L * (L + 1) // 2)


def test_noncausal_brute_force_and_library_softmax():
    from scipy.special import softmax
    lq, kv_len, h_q, h_kv, d = 6, 17, 4, 2, 5
    q = _rand((lq, h_q, d), 30)
    k = _rand((kv_len, h_kv, d), 31)
    v = _rand((kv_len, h_kv, d), 32)
    o, _ = A.attention_half(q, k, v, kv_len, 0.4, causal=False)
    assert np.abs(o - A.brute_force(q, k, v, kv_len, 0.4, causal=False)).max() < 1e-13
    for h in range(h_q):
        p = softmax(0.4 * q[:, h] @ k[:, h // 2].T, axis=1)
        assert np.abs(o[:, h] - p @ v[:, h // 2]).max() < 1e-13


def test_noncausal_union_equals_full_noncausal_attention():
    c, lens, h_q, h_kv, d = 3, [40, 29], 4, 1, 8
    p = P.build_metadata(c, sum(lens), extend_lens=lens)
    q, k, v = _rand((sum(lens), h_q, d), 33), _rand((sum(lens), h_kv, d), 34), _rand((sum(lens), h_kv, d), 35)
    starts = np.cumsum([0] + lens)
    ks = [k[starts[s]:starts[s + 1]] for s in range(2)]
    vs = [v[starts[s]:starts[s + 1]] for s in range(2)]
    per_rank = [A.run_rank(p, r, R.shard(q, p, r), ks, vs, 0.3, causal=False)[0] for r in range(c)]
    o_tok = R.gather_kv(R.all_gather_padded(per_rank, p), p)
    ref = np.concatenate([A.attention_half(q[starts[s]:starts[s + 1]], ks[s], vs[s], lens[s], 0.3,
                                           causal=False)[0] for s in range(2)])
    assert np.abs(o_tok - ref).max() < 1e-12


def test_union_with_cached_prefix_equals_tail_of_full_attention():
    """With a cached prefix, every extend token at position prefix + t sees keys
    0 .. prefix + t: the ranks' halves, back in token order, equal the extend
    rows of plain causal attention over the whole sequence (prefix included)."""
    c, ext, pre, h_q, h_kv, d = 2, [23, 17], [5, 9], 4, 2, 8
    full = [e + q for e, q in zip(ext, pre)]
    p = P.build_metadata(c, sum(ext), seqs_len=full, extend_lens=ext)
    assert p.prefix == pre
    q_all = [_rand((n, h_q, d), 40 + s) for s, n in enumerate(full)]
    k_all = [_rand((n, h_kv, d), 50 + s) for s, n in enumerate(full)]
    v_all = [_rand((n, h_kv, d), 60 + s) for s, n in enumerate(full)]
    q_ext = np.concatenate([q_all[s][pre[s]:] for s in range(2)])
    scale = d ** -0.5
    per_rank = [A.run_rank(p, r, R.shard(q_ext, p, r), k_all, v_all, scale) for r in range(c)]
    o_tok = R.gather_kv(R.all_gather_padded([o for o, _ in per_rank], p), p)
    l_tok = R.gather_kv(R.all_gather_padded([l for _, l in per_rank], p), p)
    ref = [A.full_causal(q_all[s], k_all[s], v_all[s], scale) for s in range(2)]
    ref_o = np.concatenate([ref[s][0][pre[s]:] for s in range(2)])
    ref_l = np.concatenate([ref[s][1][pre[s]:] for s in range(2)])
    assert np.abs(o_tok - ref_o).max() < 1e-12
    assert np.abs(l_tok - ref_l).max() < 1e-12
