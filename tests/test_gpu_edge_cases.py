"""Edge cases and the error contract on the GPU."""
import numpy as np
import pytest
import torch

from tests.gpu_cases import Case, Run, assert_close, zz

pytestmark = pytest.mark.gpu


def _check_full(run):
    run.attend()
    p = run.ref_plan
    out = run.out.float().cpu().numpy()
    for r in range(p.cp_size):
        o_ref, _ = run.expected_rank(r)
        n = p.per_rank_actual_token[r]
        assert np.isfinite(out[r * p.M: r * p.M + n]).all()
        assert_close(out[r * p.M: r * p.M + n], o_ref, run.case.dtype, f"rank {r}")
    assert run.plan.device_status() == 0


@pytest.mark.parametrize("case", [
    Case(2, [4], 2, 1, 128, page_size=16),                     # every block is one token
    Case(4, [8, 9, 15, 16, 17], 4, 2, 128, page_size=8),       # minimal and near-minimal lengths
    Case(2, [5] * 40, 2, 2, 64, page_size=16),                 # many short sequences
    Case(8, [257, 1000, 129], 6, 3, 128, page_size=32),        # odd group 3, c=8
    Case(3, [129, 130], 2, 2, 128, page_size=128),             # tiles that end one row past a tile
], ids=["blocks-of-one", "minimal", "bs40", "c8-g3", "ps128-ragged"])
def test_edge_case_parity(case):
    _check_full(Run(case))


def test_unsupported_shapes_are_refused():
    run = Run(Case(2, [64], 2, 2, 128, page_size=16))
    with pytest.raises(zz.ZZError) as e:
        zz.attn_prefill(run.plan, run.q_ranked, run.k_pool, run.v_pool, run.page_table, 24, run.out)
    assert e.value.status == zz.ZZ_ERR_UNSUPPORTED
    q96 = torch.zeros(run.q_ranked.shape[0], 2, 96, dtype=torch.bfloat16, device="cuda")
    kv96 = torch.zeros(run.k_pool.shape[0], 2, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(zz.ZZError) as e:
        zz.attn_prefill(run.plan, q96, kv96, kv96, run.page_table, 16, q96)
    assert e.value.status == zz.ZZ_ERR_UNSUPPORTED
    with pytest.raises(zz.ZZError) as e:        # page table too short for the kv lengths
        zz.attn_prefill(run.plan, run.q_ranked, run.k_pool, run.v_pool, run.page_table[:, :1], 16,
                        run.out)
    assert e.value.status == zz.ZZ_ERR_INVALID_ARG


def test_bounded_wait_gives_up_and_context_stays_usable():
    status = torch.zeros(2, dtype=torch.int64, device="cuda")
    zz.debug_wait_timeout(50_000_000, status)               # 50 ms on a barrier nobody arrives at
    torch.cuda.synchronize()
    flag, ns = status.tolist()
    assert flag == 1
    assert 40_000_000 <= ns < 2_000_000_000
    # the context still runs real work afterwards
    _check_full(Run(Case(2, [200], 4, 2, 128, page_size=16)))


def test_launch_after_a_timeout_aborts_at_entry():
    """While the plan's status word carries a timeout from an earlier launch,
    an attention launch (the persistent CTA-pair kernel here: several waves of
    work units) gives up at entry in every cluster: it asks for no further
    units, writes nothing and returns; after the status is read and cleared,
    the same launch is exact again."""
    run = Run(Case(4, [4096], 32, 4, 128, page_size=16))
    ws = run.plan.workspace
    status_off = ws.numel() - 256                      # the status word closes the workspace
    ws[status_off:status_off + 4].copy_(torch.tensor([4, 0, 0, 0], dtype=torch.uint8))
    with pytest.raises(zz.ZZError, match="outside the pool"):
        run.plan.device_status()                       # the offset is the status word's
    ws[status_off:status_off + 4].copy_(torch.tensor([1, 0, 0, 0], dtype=torch.uint8))
    run.out.fill_(float("nan"))
    run.attend()
    assert torch.isnan(run.out.float()).all(), "an aborted launch wrote output"
    assert run.plan.device_status() == 1               # timeout bit, read and cleared
    _check_full(run)


@pytest.mark.parametrize("case", [
    Case(2, [300, 517], 8, 2, 128, page_size=16, causal=False),
    Case(3, [700], 4, 4, 128, page_size=64, causal=False),              # row-pair mode
    Case(2, [260, 300], 4, 2, 128, page_size=16, prefix=[100, 37], causal=False),
    Case(2, [256], 4, 4, 64, dtype="fp32", page_size=256, scale=1.0, page_seed=None, causal=False),
    Case(2, [333, 200], 4, 2, 64, page_size=32, causal=False),          # bf16 head_dim 64
], ids=["gqa", "mha", "prefix", "fp32", "d64"])
def test_noncausal_local_q_global_kv(case):
    _check_full(Run(case))


@pytest.mark.parametrize("dtype,d,ps,bad", [("bf16", 128, 16, 10**6), ("bf16", 128, 64, -1),
                                           ("fp32", 64, 256, 2**28)],
                         ids=["bf16-past-end", "bf16-negative", "fp32-past-end"])
def test_page_outside_pool_is_reported_and_contained(dtype, d, ps, bad):
    """A page-table entry outside the pool is never dereferenced: its keys read as
    zeros, the status word reports it, other sequences stay exact, and the
    context keeps working."""
    run = Run(Case(2, [300, 212], 4, 2, d, dtype=dtype, page_size=ps, scale=0.5))
    run.page_table[0, 1] = bad                       # sequence 0, second page
    run.attend()
    with pytest.raises(zz.ZZError, match="outside the pool") as e:
        run.plan.device_status()
    assert e.value.status == zz.ZZ_ERR_INVALID_ARG
    assert run.plan.device_status() == 0             # the read cleared it
    p = run.ref_plan
    out = run.out.float().cpu().numpy()
    for r in range(p.cp_size):
        o_ref, _ = run.expected_rank(r)
        tp = p.total_q_prev[r]
        for lo, hi in ((p.cu_seqlens_q_prev[r][1], p.cu_seqlens_q_prev[r][2]),
                       (tp + p.cu_seqlens_q_next[r][1], tp + p.cu_seqlens_q_next[r][2])):
            assert_close(out[r * p.M + lo: r * p.M + hi], o_ref[lo:hi], dtype, f"rank {r} seq 1")
    _check_full(Run(Case(2, [200], 4, 2, 128, page_size=16)))
