"""The allocation-free attention entry point (GPU).

zz_attn_prefill_noalloc is for callers that cannot give the library device
memory of their own: a host runtime whose device memory all belongs to its own
arena and that offers plug-ins no allocation call, or a process that must keep
its device footprint fixed after start-up.  Instead of a caller-allocated
workspace it keeps the plan's tables in a 1 MiB array inside the library.

Checked here through the C ABI: two calls in a row give exactly the bytes of
the workspace-based zz_attn_prefill (same kernel, same tables), for all ranks
and for a subset of ranks; a page-table entry outside the pool is reported
through zz_plan_device_status; a plan too large for the array is refused
before any work is enqueued.
"""
import ctypes

import pytest
import torch

from tests.gpu_cases import Case, Run, zz

pytestmark = pytest.mark.gpu


def _call_noalloc(run: Run, out: torch.Tensor, lse: torch.Tensor, rank_begin: int = 0,
                  rank_count: int | None = None, plan=None, q=None) -> int:
    c = run.case
    plan = plan or run.plan
    q = run.q_ranked if q is None else q
    rank_count = plan.cp_size if rank_count is None else rank_count
    return zz.raw_call(
        "zz_attn_prefill_noalloc", plan.handle, rank_begin, rank_count, q.data_ptr(),
        run.k_pool.data_ptr(), run.v_pool.data_ptr(), run.k_pool.shape[0], run.page_table.data_ptr(),
        run.page_table.shape[1], c.page_size, out.data_ptr(), lse.data_ptr(), c.h_q, c.h_kv, c.d,
        ctypes.c_float(run.softmax_scale), zz.ZZ_BF16, torch.cuda.current_stream().cuda_stream)


CASES = [Case(4, [1500, 700], 8, 2, 128, page_size=16),     # GQA 4: head-pair work items
         Case(3, [900], 4, 4, 128, page_size=64)]           # MHA: row-tile-pair work items


@pytest.mark.parametrize("case", CASES, ids=["gqa4-varlen", "mha"])
def test_noalloc_equals_workspace_entry_point_on_two_calls(case):
    run = Run(case)
    run.attend()                                   # workspace-based entry point
    for _ in range(2):
        out = torch.full_like(run.out, float("nan"))
        lse = torch.full_like(run.lse, float("nan"))
        assert _call_noalloc(run, out, lse) == zz.ZZ_OK, zz.last_error()
        torch.cuda.synchronize()
        # identical bytes, padding rows (NaN, never written) included
        assert torch.equal(out.view(torch.int16), run.out.view(torch.int16))
        assert torch.equal(lse.view(torch.int32), run.lse.view(torch.int32))
    assert run.plan.device_status() == 0


@pytest.mark.parametrize("case", CASES, ids=["gqa4-varlen", "mha"])
def test_noalloc_rank_subset_equals_workspace_entry_point(case):
    """A per-rank caller's launch: ranks [1, c) of the plan, Q/O holding only those ranks."""
    run = Run(case)
    M, cp = run.plan.M, run.plan.cp_size
    rb, rc = 1, cp - 1
    q_sub = run.q_ranked[rb * M:(rb + rc) * M].contiguous()
    want = torch.full_like(q_sub, float("nan"))
    want_lse = torch.full((rc * M, case.h_q), float("nan"), dtype=torch.float32, device="cuda")
    zz.attn_prefill(run.plan, q_sub, run.k_pool, run.v_pool, run.page_table, case.page_size, want,
                    want_lse, softmax_scale=run.softmax_scale, rank_begin=rb, rank_count=rc)
    for _ in range(2):
        out = torch.full_like(want, float("nan"))
        lse = torch.full_like(want_lse, float("nan"))
        assert _call_noalloc(run, out, lse, rb, rc, q=q_sub) == zz.ZZ_OK, zz.last_error()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), want.view(torch.int16))
        assert torch.equal(lse.view(torch.int32), want_lse.view(torch.int32))


def test_noalloc_reports_a_page_outside_the_pool():
    run = Run(Case(2, [300, 212], 4, 2, 128, page_size=16))
    run.attend()
    assert run.plan.device_status() == 0
    run.page_table[0, 1] = 10 ** 6                  # sequence 0, second page: far past the pool
    out = torch.full_like(run.out, float("nan"))
    lse = torch.full_like(run.lse, float("nan"))
    # a plan that was never uploaded: its status lives only in the static array
    fresh = zz.Plan(run.case.cp, extend_lens=run.case.lens)
    for plan in (fresh, run.plan):
        assert _call_noalloc(run, out, lse, plan=plan) == zz.ZZ_OK, zz.last_error()
        with pytest.raises(zz.ZZError, match="outside the pool") as e:
            plan.device_status()
        assert e.value.status == zz.ZZ_ERR_INVALID_ARG
        assert plan.device_status() == 0            # the read cleared it
    # the next call starts from a clear status word and a good table
    run.page_table[0, 1] = torch.from_numpy(run.pool.page_table)[0, 1].item()
    assert _call_noalloc(run, out, lse, plan=fresh) == zz.ZZ_OK, zz.last_error()
    assert fresh.device_status() == 0


def test_noalloc_refuses_tables_larger_than_its_scratch():
    plan = zz.Plan(8, extend_lens=[16] * 4096)      # 65536 halves: 2 MiB of half table
    fake = 1 << 20                                   # never dereferenced: refused first
    st = zz.raw_call("zz_attn_prefill_noalloc", plan.handle, 0, 8, fake, fake, fake, 1 << 16, fake,
                     1, 16, fake, None, 8, 8, 128, ctypes.c_float(0.0), zz.ZZ_BF16, None)
    assert st == zz.ZZ_ERR_INVALID_ARG
    assert "static scratch" in zz.last_error()
    with pytest.raises(zz.ZZError):                  # nothing ran, so nothing to report
        plan.device_status()
