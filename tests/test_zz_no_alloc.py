"""The allocation-free attention entry point (GPU).

zz_attn_prefill_noalloc serves callers that cannot allocate device memory for
the plan's tables themselves (for example code running while a CUDA graph is
captured, or a runtime whose device memory belongs to its own arena).  It keeps
those tables in a 1 MiB array inside the library instead.  Here it is called
through the C ABI twice in a row and each result is compared with the
workspace-based zz_attn_prefill on the same inputs; a plan too large for the
array must be refused before any work is enqueued.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests.gpu_cases import BF16_MAX_ABS, BF16_MEAN_ABS, Case, Run, zz

pytestmark = pytest.mark.gpu


def _call_noalloc(run: Run, out: torch.Tensor, lse: torch.Tensor) -> int:
    c = run.case
    return zz.raw_call(
        "zz_attn_prefill_noalloc", run.plan.handle, 0, run.plan.cp_size, run.q_ranked.data_ptr(),
        run.k_pool.data_ptr(), run.v_pool.data_ptr(), run.k_pool.shape[0], run.page_table.data_ptr(),
        run.page_table.shape[1], c.page_size, out.data_ptr(), lse.data_ptr(), c.h_q, c.h_kv, c.d,
        ctypes.c_float(run.softmax_scale), zz.ZZ_BF16, torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("case", [Case(4, [1500, 700], 8, 2, 128, page_size=16),
                                  Case(3, [900], 4, 4, 128, page_size=64)],
                         ids=["gqa4-varlen", "mha"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(case):
    run = Run(case)
    run.attend()                                   # workspace-based entry point
    ref = run.out.float().cpu().numpy()
    ref_lse = run.lse.cpu().numpy()
    p = run.ref_plan
    valid = np.concatenate([np.arange(r * p.M, r * p.M + n)
                            for r, n in enumerate(p.per_rank_actual_token)])
    for _ in range(2):
        out = torch.full_like(run.out, float("nan"))
        lse = torch.full_like(run.lse, float("nan"))
        assert _call_noalloc(run, out, lse) == zz.ZZ_OK, zz.last_error()
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()[valid]
        err = np.abs(got - ref[valid])
        assert np.isfinite(got).all()
        assert err.max() <= BF16_MAX_ABS and err.mean() <= BF16_MEAN_ABS
        assert np.abs(lse.cpu().numpy()[valid] - ref_lse[valid]).max() < 2e-3


def test_noalloc_refuses_tables_larger_than_its_scratch():
    plan = zz.Plan(8, extend_lens=[16] * 4096)      # 65536 halves: 2 MiB of half table
    fake = 1 << 20
    st = zz.raw_call("zz_attn_prefill_noalloc", plan.handle, 0, 8, fake, fake, fake, 1 << 16, fake,
                     1, 16, fake, None, 8, 8, 128, ctypes.c_float(0.0), zz.ZZ_BF16, None)
    assert st == zz.ZZ_ERR_INVALID_ARG
    assert "static scratch" in zz.last_error()
