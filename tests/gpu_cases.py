"""Shared builders for the GPU parity tests.

A case draws natural-order Q/K/V with ``synth``, runs the product path on the
GPU through the C ABI (shard -> rerange into the paged pool -> attention), and
lets the oracle compute the expected rows from the same natural-order inputs.
Oracle values never come from the GPU.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

import synth
from oracle import attention as OA
from oracle import plan as OP
from oracle import rerange as OR
from tests._lib import ensure_built

zz = ensure_built()

BF16_MAX_ABS, BF16_MEAN_ABS = 2e-2, 2e-3
FP32_MAX_ABS = 1e-4


@dataclass
class Case:
    cp: int
    lens: list
    h_q: int
    h_kv: int
    d: int
    dtype: str = "bf16"
    page_size: int = 16
    seed: int = 0
    scale: float = 0.5           # value scale of the N(0,1) draws
    page_seed: int | None = 1
    prefix: list | None = None   # cached-prefix tokens per sequence (already in the pool)
    causal: bool = True
    k_ramp: float = 0.0          # > 0: key magnitudes grow along each sequence (synth.key_ramp)


class Run:
    """Everything one case needs on both sides."""

    def __init__(self, case: Case, device: str = "cuda", gen_device: str | None = None):
        self.case = c = case
        self.dev = device
        prefix = c.prefix or [0] * len(c.lens)
        full = [p + L for p, L in zip(prefix, c.lens)]
        self.ref_plan = OP.build_metadata(c.cp, sum(c.lens), seqs_len=full if c.prefix else None,
                                          extend_lens=c.lens)
        self.plan = zz.Plan(c.cp, extend_lens=c.lens, seq_lens=full if c.prefix else None)
        self.plan.upload()
        T = sum(c.lens)
        gdev = gen_device or ("cpu" if T * c.h_q * c.d < 2**27 else device)
        # natural-order inputs: prefix tokens first, then the extend tokens, per sequence
        self.q, k_all, v_all = synth.qkv(sum(full), c.h_q, c.h_kv, c.d, c.seed, c.scale, c.dtype, gdev)
        if c.k_ramp:
            k_all = synth.key_ramp(k_all, full, c.k_ramp)
        starts = np.cumsum([0] + full)
        ext_rows = np.concatenate([np.arange(starts[s] + prefix[s], starts[s + 1]) for s in range(len(full))])
        ext_idx = torch.from_numpy(ext_rows).to(gdev)
        self.q = self.q.index_select(0, ext_idx).contiguous()
        self.k_seqs = [k_all[starts[s]:starts[s + 1]] for s in range(len(full))]
        self.v_seqs = [v_all[starts[s]:starts[s + 1]] for s in range(len(full))]
        k_ext = k_all.index_select(0, ext_idx).contiguous()
        v_ext = v_all.index_select(0, ext_idx).contiguous()
        self.pool = synth.paged_pool(full, c.page_size, c.page_seed, spare_pages=3)
        # GPU side
        dt = self.q.dtype
        M, cp = self.plan.M, c.cp
        self.q_dev = self.q.to(device)
        self.q_ranked = torch.zeros(cp * M, c.h_q, c.d, dtype=dt, device=device)
        zz.shard_rows(self.plan, self.q_dev, self.q_ranked)
        self.k_gath = torch.zeros(cp * M, c.h_kv, c.d, dtype=dt, device=device)
        self.v_gath = torch.zeros_like(self.k_gath)
        zz.shard_rows(self.plan, k_ext.to(device), self.k_gath)
        zz.shard_rows(self.plan, v_ext.to(device), self.v_gath)
        slots = self.pool.num_slots
        self.k_pool = torch.zeros(slots, c.h_kv, c.d, dtype=dt, device=device)
        self.v_pool = torch.zeros_like(self.k_pool)
        loc_all = torch.from_numpy(self.pool.out_cache_loc)
        ext_loc = loc_all[torch.from_numpy(ext_rows)].to(device)
        if c.prefix:   # cached prefix K/V are already in the pool
            pre_rows = torch.from_numpy(np.setdiff1d(np.arange(sum(full)), ext_rows))
            pl = loc_all[pre_rows].to(device)
            self.k_pool[pl] = k_all[pre_rows.to(gdev)].to(device)
            self.v_pool[pl] = v_all[pre_rows.to(gdev)].to(device)
        self.ext_loc = ext_loc.contiguous()
        zz.rerange_kv_to_pool(self.plan, self.k_gath, self.v_gath, self.k_pool, self.v_pool, self.ext_loc)
        self.page_table = torch.from_numpy(self.pool.page_table).to(device)
        self.out = torch.full_like(self.q_ranked, float("nan"))
        self.lse = torch.full((cp * M, c.h_q), float("nan"), dtype=torch.float32, device=device)
        self.softmax_scale = 1.0 / math.sqrt(c.d)

    def attend(self, rank_begin=0, rank_count=None):
        zz.attn_prefill(self.plan, self.q_ranked, self.k_pool, self.v_pool, self.page_table,
                        self.case.page_size, self.out, self.lse, softmax_scale=self.softmax_scale,
                        rank_begin=rank_begin, rank_count=rank_count, causal=self.case.causal)
        torch.cuda.synchronize()

    # ---------------- oracle side
    def expected_rank(self, r):
        """Oracle outputs of rank r, rank-local order (full)."""
        ql = OR.shard(self.q.float().cpu().numpy() if self.q.dtype == torch.float32
                      else self.q.cpu().double().numpy(), self.ref_plan, r)
        ks = [k.cpu().double().numpy() for k in self.k_seqs]
        vs = [v.cpu().double().numpy() for v in self.v_seqs]
        return OA.run_rank(self.ref_plan, r, ql, ks, vs, self.softmax_scale, causal=self.case.causal)

    def sampled_rows(self, per_half: int, rng_seed: int = 0):
        """[(rank, local_row, half, seq, row_in_half)] — first, last and random rows of every half."""
        p = self.ref_plan
        rng = np.random.default_rng(rng_seed)
        out = []
        for r in range(p.cp_size):
            for h, (cu, base) in enumerate(((p.cu_seqlens_q_prev[r], 0),
                                            (p.cu_seqlens_q_next[r], p.total_q_prev[r]))):
                for s in range(p.bs):
                    lq = cu[s + 1] - cu[s]
                    rows = {0, lq - 1} | set(rng.integers(0, lq, per_half).tolist())
                    for j in sorted(rows):
                        out.append((r, base + cu[s] + j, h, s, j))
        return out

    def tile_rows(self, rng_seed: int = 0, tile: int = 128):
        """One row from EVERY ``tile``-row query tile of every half (at an offset
        that changes from tile to tile, so both 128-row sub-tiles of a CTA, every
        work item and every position inside a tile get exercised), plus the
        first and last row of each half."""
        p = self.ref_plan
        rng = np.random.default_rng(rng_seed)
        out = []
        for r in range(p.cp_size):
            for h, (cu, base) in enumerate(((p.cu_seqlens_q_prev[r], 0),
                                            (p.cu_seqlens_q_next[r], p.total_q_prev[r]))):
                for s in range(p.bs):
                    lq = cu[s + 1] - cu[s]
                    rows = {0, lq - 1}
                    for t0 in range(0, lq, tile):
                        rows.add(t0 + int(rng.integers(0, min(tile, lq - t0))))
                    for j in sorted(rows):
                        out.append((r, base + cu[s] + j, h, s, j))
        return out

    def expected_rows(self, samples):
        """Oracle o, lse for sampled rows, one oracle call per (rank, half,
        sequence) so that each half's keys are read once."""
        p = self.ref_plan
        ks = [k.double().cpu().numpy() for k in self.k_seqs]
        vs = [v.double().cpu().numpy() for v in self.v_seqs]
        starts = np.cumsum([0] + self.case.lens)
        groups = {}
        for i, (r, lrow, h, s, j) in enumerate(samples):
            groups.setdefault((r, h, s), []).append((i, j))
        res = [None] * len(samples)
        for (r, h, s), members in groups.items():
            kv_len = (p.kv_len_prev if h == 0 else p.kv_len_next)[r][s]
            lq = (p.q_len_prev if h == 0 else p.q_len_next)[r][s]
            blk = r if h == 0 else 2 * p.cp_size - 1 - r
            first_tok = starts[s] + sum(p.blocks[s][:blk])             # natural token of row 0
            js = np.array([j for _, j in members])
            idx = torch.from_numpy(first_tok + js).to(self.q.device)
            qrows = self.q[idx].double().cpu().numpy()
            o, l = OA.attention_rows(qrows, js, ks[s], vs[s], kv_len, lq, self.softmax_scale)
            for n, (i, _) in enumerate(members):
                res[i] = (o[n], l[n])
        return res

    def padding_rows(self):
        """Rows of the [c*M] layout that belong to no half (never to be written)."""
        p = self.ref_plan
        return np.concatenate([np.arange(r * p.M + n, (r + 1) * p.M)
                               for r, n in enumerate(p.per_rank_actual_token)]).astype(np.int64)


def assert_close(got: np.ndarray, want: np.ndarray, dtype: str, what: str = ""):
    err = np.abs(got.astype(np.float64) - want)
    mx, mean = float(err.max()), float(err.mean())
    if dtype == "fp32":
        assert mx <= FP32_MAX_ABS, f"{what}: max-abs {mx:.3e} > {FP32_MAX_ABS}"
    else:
        assert mx <= BF16_MAX_ABS, f"{what}: max-abs {mx:.3e} > {BF16_MAX_ABS}"
        assert mean <= BF16_MEAN_ABS, f"{what}: mean-abs {mean:.3e} > {BF16_MEAN_ABS}"
    return mx, mean
