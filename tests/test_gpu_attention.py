"""Attention parity with the fp64 oracle (GPU), through the C ABI.

Small cases are compared on every valid output row; the full-size
configurations on one row of EVERY 128-row query tile of every half of every
rank (at an offset that varies from tile to tile) plus each half's first and
last row, so every work item and both query sub-tiles of each CTA are checked.
Rows of the [c*M] layout that belong to no half must stay unwritten (NaN).
Tolerances: bf16 max-abs 2e-2 and mean-abs 2e-3, fp32 max-abs 1e-4.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import rerange as OR
from tests.gpu_cases import Case, Run, assert_close, zz

pytestmark = pytest.mark.gpu


def _check_full(run: Run):
    run.attend()
    p = run.ref_plan
    out = run.out.float().cpu().numpy()
    lse = run.lse.cpu().numpy()
    for r in range(p.cp_size):
        o_ref, l_ref = run.expected_rank(r)
        n = p.per_rank_actual_token[r]
        got = out[r * p.M: r * p.M + n]
        assert np.isfinite(got).all()
        assert_close(got, o_ref, run.case.dtype, f"rank {r} out")
        assert np.abs(lse[r * p.M: r * p.M + n] - l_ref).max() < 2e-3, f"rank {r} lse"
    _check_padding_untouched(run)


def _check_padding_untouched(run: Run):
    pad = torch.from_numpy(run.padding_rows()).to(run.out.device)
    if pad.numel():
        assert torch.isnan(run.out.index_select(0, pad).float()).all(), "a padding row was written"
        assert torch.isnan(run.lse.index_select(0, pad)).all(), "a padding row's lse was written"


SMALL = [
    Case(2, [256], 4, 4, 64, dtype="fp32", page_size=256, scale=1.0, page_seed=None),  # fp32, unpaged
    Case(2, [300, 517], 8, 2, 128, page_size=16),          # GQA 4, ragged blocks and tails
    Case(3, [700], 4, 4, 128, page_size=64),               # MHA: row-tile pairs
    Case(2, [333], 6, 2, 128, page_size=32),               # odd group (3)
    Case(2, [600, 129], 8, 1, 128, page_size=16),          # MQA
    Case(2, [400], 4, 2, 64, page_size=32),                # bf16 head_dim 64
    Case(2, [1000], 4, 2, 128, page_size=256),             # page larger than a K/V tile
    Case(4, [1100, 600], 4, 2, 128, page_size=8),          # page 8
    Case(2, [260, 300], 4, 2, 128, page_size=16, prefix=[100, 37]),   # cached prefix
    Case(2, [96], 2, 1, 128, page_size=16),                # every half shorter than one tile
    Case(2, [48], 2, 2, 64, dtype="fp32", page_size=16),   # fp32 paged
    Case(3, [500, 129], 4, 4, 64, page_size=64),           # bf16 head_dim 64, MHA row-tile pairs
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"c{c.cp}-L{c.lens}-{c.h_q}/{c.h_kv}-d{c.d}-{c.dtype}-ps{c.page_size}")
def test_small_cases_every_row(case):
    _check_full(Run(case))


# Key magnitudes that grow along the sequence: later tiles' scores exceed the
# first tile's maximum by far more than the kernel's range for a kept tile, so
# the kernel must redo tiles (new maximum, O and l rescaled) several times per
# row, in every kernel and mode.
REDO = [
    Case(4, [1500, 700], 8, 2, 128, page_size=16, k_ramp=4.0),                   # CTA pairs, heads
    Case(2, [2100], 4, 4, 128, page_size=64, k_ramp=4.0),                        # CTA pairs, row tiles
    Case(2, [1300], 4, 2, 64, page_size=32, k_ramp=4.0),                         # single CTA, head_dim 64
    Case(2, [900], 4, 2, 128, page_size=16, k_ramp=8.0, causal=False),           # non-causal
    Case(2, [700, 300], 4, 2, 128, page_size=16, prefix=[300, 64], k_ramp=8.0),  # cached prefix
]


def _max_growth_log2(run: Run) -> float:
    """Largest rise of a 128-key tile's score maximum (log2 units) over the first
    tile's, for the last query row of sequence 0, head 0."""
    c = run.case
    k = run.k_seqs[0][:, 0].double().cpu().numpy()
    q = run.q[c.lens[0] - 1, 0].double().cpu().numpy()
    s = (k @ q) * run.softmax_scale / np.log(2.0)
    tiles = [s[i:i + 128].max() for i in range(0, len(s), 128)]
    return float(max(tiles) - tiles[0])


@pytest.mark.parametrize("case", REDO, ids=["pair-heads", "pair-rows", "single-d64", "noncausal", "prefix"])
def test_growing_scores_redo_tiles_every_row(case):
    run = Run(case)
    assert _max_growth_log2(run) > 24.0      # a row sum of at least 2^24 > 2^16: redone
    _check_full(run)


def test_c4_L4096_gqa8_every_row():
    _check_full(Run(Case(4, [4096], 32, 4, 128, page_size=16)))


def test_single_rank_launches_match_full_launch():
    run = Run(Case(4, [1500, 700], 8, 2, 128, page_size=16))
    run.attend()
    full = run.out.clone()
    p = run.ref_plan
    for r in range(p.cp_size):
        run.out.fill_(float("nan"))
        q_r = run.q_ranked[r * p.M:(r + 1) * p.M]
        out_r = torch.full_like(q_r, float("nan"))
        zz.attn_prefill(run.plan, q_r, run.k_pool, run.v_pool, run.page_table, 16, out_r,
                        softmax_scale=run.softmax_scale, rank_begin=r, rank_count=1)
        torch.cuda.synchronize()
        n = p.per_rank_actual_token[r]
        assert torch.equal(out_r[:n], full[r * p.M: r * p.M + n])


def test_concurrent_launches_sharing_a_plan_are_bit_identical():
    """Launches on two streams that share one plan and its workspace, running at
    the same time, each give exactly the output of a launch run alone: the
    persistent kernel hands out work units per launch (no shared counter), and
    every unit is computed once in a fixed order.  Several waves of units, so
    units are handed out while the other launch is running."""
    run = Run(Case(4, [4096], 32, 4, 128, page_size=16))
    p = run.ref_plan
    q_sets = [run.q_ranked, (run.q_ranked * -0.75).contiguous()]
    ref = []
    for q in q_sets:
        o = torch.full_like(q, float("nan"))
        zz.attn_prefill(run.plan, q, run.k_pool, run.v_pool, run.page_table, 16, o,
                        softmax_scale=run.softmax_scale)
        torch.cuda.synchronize()
        ref.append(o)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [[torch.full_like(q_sets[i], float("nan")) for _ in range(4)] for i in range(2)]
    torch.cuda.synchronize()
    for k in range(4):
        for i in range(2):
            zz.attn_prefill(run.plan, q_sets[i], run.k_pool, run.v_pool, run.page_table, 16, outs[i][k],
                            softmax_scale=run.softmax_scale, stream=streams[i])
    torch.cuda.synchronize()
    valid = torch.cat([torch.arange(r * p.M, r * p.M + p.per_rank_actual_token[r]) for r in range(p.cp_size)])
    valid = valid.to(run.out.device)
    for i in range(2):
        assert torch.isfinite(ref[i].index_select(0, valid).float()).all()
        for k in range(4):
            assert torch.equal(outs[i][k].index_select(0, valid), ref[i].index_select(0, valid)), (i, k)
    assert run.plan.device_status() == 0


def test_union_in_token_order_equals_unsharded_attention():
    """Outputs of all ranks, moved back to token order, equal plain causal attention."""
    from oracle import attention as OA
    run = Run(Case(4, [2000], 8, 2, 128, page_size=16))
    run.attend()
    p = run.ref_plan
    o_tok = OR.gather_kv(run.out.float().cpu().numpy(), p)
    ref, _ = OA.full_causal(run.q.double().cpu().numpy(), run.k_seqs[0].double().cpu().numpy(),
                            run.v_seqs[0].double().cpu().numpy(), run.softmax_scale)
    assert_close(o_tok, ref, "bf16", "union")


def _check_sampled(run: Run, per_half: int | None = None):
    """per_half=None: one row of every query tile; else first/last + random rows."""
    run.attend()
    samples = run.tile_rows() if per_half is None else run.sampled_rows(per_half)
    want = run.expected_rows(samples)
    p = run.ref_plan
    idx = torch.tensor([r * p.M + lrow for (r, lrow, *_rest) in samples], device=run.out.device)
    got = run.out.index_select(0, idx).float().cpu().numpy()
    ref = np.stack([w[0] for w in want])
    assert np.isfinite(got).all()
    assert_close(got, ref, "bf16", f"{len(samples)} sampled rows")
    gl = run.lse.index_select(0, idx).cpu().numpy()
    assert np.abs(gl - np.stack([w[1] for w in want])).max() < 2e-3
    _check_padding_untouched(run)


def test_varlen_batch_c4_every_tile():
    lens = synth.varlen_lengths(8, 1000, 8192, seed=0)
    _check_sampled(Run(Case(4, lens, 32, 4, 128, page_size=16)))


@pytest.mark.parametrize("cp", [2, 4, 8])
@pytest.mark.parametrize("h_q,h_kv", [(32, 32), (32, 8), (32, 1)], ids=["mha", "gqa4", "mqa"])
def test_L32768_head_ratio_sweep_every_tile(h_q, h_kv, cp):
    _check_sampled(Run(Case(cp, [32768], h_q, h_kv, 128, page_size=16)))


def test_long_context_c8_L131072_every_tile():
    _check_sampled(Run(Case(8, [131072], 64, 8, 128, page_size=64)))


def _random_cases(n: int, seed: int = 2024):
    """Seeded random small configurations: cp size, batch and ragged lengths,
    GQA group (odd groups and MHA included), head_dim, page size, cached
    prefix, causal or not, and growing scores; sized so that the oracle checks
    every output row in about a second each."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        cp = int(rng.choice([2, 3, 4, 8]))
        bs = int(rng.integers(1, 4))
        lens = [int(x) for x in rng.integers(2 * cp, 900 // bs + 2 * cp, bs)]
        h_kv = int(rng.choice([1, 2, 4]))
        group = int(rng.choice([1, 2, 3, 4, 8]))
        h_q = h_kv * group
        if h_q > 16:
            h_kv, h_q = 1, group
        d = int(rng.choice([64, 128]))
        ps = int(rng.choice([8, 16, 32, 64, 128, 256]))
        prefix = [int(x) for x in rng.integers(0, 300, bs)] if rng.random() < 0.3 else None
        causal = bool(rng.random() < 0.8)
        ramp = 4.0 if rng.random() < 0.2 else 0.0
        out.append(Case(cp, lens, h_q, h_kv, d, page_size=ps, prefix=prefix, causal=causal, k_ramp=ramp,
                        seed=int(rng.integers(0, 1000))))
    return out


RANDOM = _random_cases(32)


@pytest.mark.parametrize("case", RANDOM, ids=lambda c: f"c{c.cp}-L{c.lens}-{c.h_q}/{c.h_kv}-d{c.d}-ps{c.page_size}"
                         f"{'-pre' if c.prefix else ''}{'' if c.causal else '-nc'}{'-ramp' if c.k_ramp else ''}")
def test_random_small_configs_every_row(case):
    _check_full(Run(case))
