"""Causal attention of the two zigzag halves, in fp64.  TEST INFRASTRUCTURE.

Follows "sgl-project--sglang/python/sglang/srt/layers/cp/zigzag.py",
``run_attention``: rank-local Q is cut at ``total_q_prev_tokens``; each half is
attention of its queries (``cu_seqlens_q``) against the first ``kv_len`` keys of
the sequence's full K/V, and the two results are concatenated.  The causal
mask is not printed on the page; the reading used here (and by the CUDA path)
is bottom-right alignment — query row ``i`` of a half with ``Lq`` rows sits at
position ``kv_len - Lq + i`` and sees keys ``0 .. kv_len - Lq + i``.  Softmax
scale defaults to ``D**-0.5`` ("PR #34485 完整报告", unit test section).
Grouped K/V: query head ``h`` reads K/V head ``h // (H_q / H_kv)``; ``H_q`` must
be a multiple of ``H_kv`` ("PR #34485 完整报告", implementation item 1).

All arithmetic is fp64 on the exact input values (bf16 inputs are widened
without rounding).  ``brute_force`` restates the same definition with scalar
Python loops (``math.exp``/``math.fsum``) and shares no code with the numpy
path.
"""
from __future__ import annotations

import math

import numpy as np

from .plan import Plan


def check_heads(h_q: int, h_kv: int) -> int:
    if h_kv <= 0 or h_q % h_kv != 0:
        raise ValueError(
            f"num_heads ({h_q}) must be a multiple of num_kv_heads ({h_kv})")
    return h_q // h_kv


def _as64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor (bf16 has no numpy dtype)
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def attention_rows(q_rows, rows, k, v, kv_len: int, lq: int, scale: float, causal: bool = True):
    """Output and log-sum-exp of selected query rows of one half.

    ``q_rows``: ``[n, H_q, D]`` the queries of half-local rows ``rows``;
    ``k``, ``v``: ``[>= kv_len, H_kv, D]`` the sequence's keys and values in
    natural order.  Returns ``o [n, H_q, D]`` and ``lse [n, H_q]`` (natural log).
    With ``causal=False`` every row sees all ``kv_len`` keys (the local-Q /
    global-KV attention of an AllGather-KV layout, "Compose Ulysses with
    AllGather-KV as a 2D SP topology": non-causal only).
    """
    q_rows, k, v = _as64(q_rows), _as64(k)[:kv_len], _as64(v)[:kv_len]
    n, h_q, d = q_rows.shape
    g = check_heads(h_q, k.shape[1])
    rows = np.asarray(rows, dtype=np.int64)
    last_key = kv_len - lq + rows if causal else np.full(rows.shape, kv_len - 1)  # inclusive
    keys = np.arange(kv_len)
    visible = keys[None, :] <= last_key[:, None]            # [n, kv_len]
    o = np.empty((n, h_q, d))
    lse = np.empty((n, h_q))
    for h in range(h_q):
        kh, vh = k[:, h // g, :], v[:, h // g, :]
        s = (q_rows[:, h, :] @ kh.T) * scale
        s = np.where(visible, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        z = p.sum(axis=1, keepdims=True)
        o[:, h, :] = (p @ vh) / z
        lse[:, h] = (m + np.log(z))[:, 0]
    return o, lse


def attention_half(q_half, k, v, kv_len: int, scale: float, row_chunk: int = 512, causal: bool = True):
    """All rows of one half (``Lq = q_half.shape[0]``), in row chunks."""
    lq = q_half.shape[0]
    outs, lses = [], []
    for a in range(0, lq, row_chunk):
        rows = np.arange(a, min(a + row_chunk, lq))
        o, l = attention_rows(q_half[a:a + row_chunk], rows, k, v, kv_len, lq, scale, causal)
        outs.append(o)
        lses.append(l)
    return np.concatenate(outs, 0), np.concatenate(lses, 0)


def run_rank(plan: Plan, rank: int, q_local, k_seqs, v_seqs, scale: float, causal: bool = True):
    """One rank's ``run_attention``: prev half then next half, concatenated.

    ``q_local``: ``[per_rank_actual_token[rank], H_q, D]`` rank-local queries;
    ``k_seqs[s]``/``v_seqs[s]``: full keys/values of sequence ``s`` (prefix
    included) in natural order.  Returns ``o`` and ``lse`` in rank-local order.
    Non-causal: every half sees the whole sequence (prefix + extend keys).
    """
    q_local = _as64(q_local)
    split = plan.total_q_prev[rank]
    halves = [(q_local[:split], plan.cu_seqlens_q_prev[rank], plan.kv_len_prev[rank]),
              (q_local[split:], plan.cu_seqlens_q_next[rank], plan.kv_len_next[rank])]
    outs, lses = [], []
    for q_h, cu, kv_len in halves:
        for s in range(plan.bs):
            kv = kv_len[s] if causal else plan.prefix[s] + plan.extend_lens[s]
            o, l = attention_half(q_h[cu[s]:cu[s + 1]], k_seqs[s], v_seqs[s], kv, scale, causal=causal)
            outs.append(o)
            lses.append(l)
    return np.concatenate(outs, 0), np.concatenate(lses, 0)


def full_causal(q_seq, k_seq, v_seq, scale: float):
    """Unsharded causal attention over one whole sequence (bottom-right when
    K/V hold a prefix longer than the queries)."""
    return attention_half(q_seq, k_seq, v_seq, _as64(k_seq).shape[0], scale)


def brute_force(q_half, k, v, kv_len: int, scale: float, causal: bool = True):
    """Scalar restatement for tiny inputs: ``sum_j e^{s_j} v_j / sum_j e^{s_j}``
    over the visible keys, with ``math.exp`` and ``math.fsum``."""
    q_half, k, v = _as64(q_half).tolist(), _as64(k).tolist(), _as64(v).tolist()
    lq, h_q, d = len(q_half), len(q_half[0]), len(q_half[0][0])
    g = h_q // len(k[0])
    out = [[[0.0] * d for _ in range(h_q)] for _ in range(lq)]
    for i in range(lq):
        last = kv_len - lq + i if causal else kv_len - 1
        for h in range(h_q):
            kvh = h // g
            sc = [scale * math.fsum(q_half[i][h][t] * k[j][kvh][t] for t in range(d))
                  for j in range(last + 1)]
            top = max(sc)
            w = [math.exp(x - top) for x in sc]
            z = math.fsum(w)
            for t in range(d):
                out[i][h][t] = math.fsum(w[j] * v[j][kvh][t] for j in range(last + 1)) / z
    return np.array(out)


def causal_pairs(lq: int, kv_len: int) -> int:
    """Visible (query, key) pairs of one half: ``Lq*(kv_len-Lq) + Lq*(Lq+1)/2``."""
    return lq * (kv_len - lq) + lq * (lq + 1) // 2


def plan_flops(plan: Plan, h_q: int, d: int) -> int:
    """Causal attention FLOPs of all ranks: ``4 * D * H_q`` per visible pair
    (``2*D`` for Q.K plus ``2*D`` for P.V)."""
    pairs = 0
    for r in range(plan.cp_size):
        for s in range(plan.bs):
            pairs += causal_pairs(plan.q_len_prev[r][s], plan.kv_len_prev[r][s])
            pairs += causal_pairs(plan.q_len_next[r][s], plan.kv_len_next[r][s])
    return 4 * d * h_q * pairs
