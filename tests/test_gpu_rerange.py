"""Bit-exact parity of the shard and rerange kernels with the oracle (GPU)."""
import numpy as np
import pytest
import torch

import synth
from oracle import plan as OP
from oracle import rerange as OR
from tests._lib import ensure_built

zz = ensure_built()
pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    return (t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)).numpy()


CASES = [
    # cp, lens, h_kv, d, dtype, page_size
    (2, [256], 4, 64, "fp32", 256),                       # small fp32, one page
    (4, [4096], 4, 128, "bf16", 16),                      # c=4, L=4096, ps 16
    (4, synth.varlen_lengths(8, 1000, 8192, seed=0), 4, 128, "bf16", 16),  # varlen x8
    (3, [37, 1, 2049, 300], 1, 128, "bf16", 64) ,          # ragged, short sequence, MQA
    (2, [32768], 8, 128, "bf16", 16),                     # the standalone rerange shape
    (4, [32768], 8, 128, "bf16", 16),
    (8, [32768], 8, 128, "bf16", 16),
    (2, [3000, 77], 32, 128, "bf16", 16),                 # 8 KB rows, ragged ends of the CTA ranges
]


@pytest.mark.parametrize("cp,lens,h_kv,d,dtype,ps", CASES)
def test_rerange_bit_exact_and_untouched_slots(cp, lens, h_kv, d, dtype, ps):
    lens = [max(L, 2 * cp) for L in lens]
    ref = OP.build_metadata(cp, sum(lens), extend_lens=lens)
    plan = zz.Plan(cp, extend_lens=lens)
    plan.upload()
    T = sum(lens)
    _, k, v = synth.qkv(T, 1, h_kv, d, seed=3, scale=0.5, dtype=dtype, device="cpu")
    pool = synth.paged_pool(lens, ps, seed=5, spare_pages=2)
    # gathered buffers as the all-gather delivers them (built by the oracle)
    kb, vb = _bits(k), _bits(v)
    kg = OR.ranked_layout(kb, ref)
    vg = OR.ranked_layout(vb, ref)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    view = torch.int16 if dtype == "bf16" else torch.int32
    kg_d = torch.from_numpy(kg).view(tdt).cuda()
    vg_d = torch.from_numpy(vg).view(tdt).cuda()
    sentinel = np.full((pool.num_slots, h_kv, d), 0x7A5A if dtype == "bf16" else 0x3F7A5A5A,
                       dtype=kb.dtype)
    kp = torch.from_numpy(sentinel.copy()).view(tdt).cuda()
    vp = torch.from_numpy(sentinel.copy()).view(tdt).cuda()
    loc = torch.from_numpy(pool.out_cache_loc).cuda()
    zz.rerange_kv_to_pool(plan, kg_d, vg_d, kp, vp, loc)
    torch.cuda.synchronize()
    want_k = OR.rerange_to_pool(kg, ref, sentinel, pool.out_cache_loc)
    want_v = OR.rerange_to_pool(vg, ref, sentinel, pool.out_cache_loc)
    assert np.array_equal(_bits(kp), want_k)
    assert np.array_equal(_bits(vp), want_v)


@pytest.mark.parametrize("cp,lens", [(2, [10, 9]), (4, [4096]), (3, [37, 8, 2049, 300]),
                                     (8, [131072])])
def test_shard_rows_bit_exact(cp, lens):
    ref = OP.build_metadata(cp, sum(lens), extend_lens=lens)
    plan = zz.Plan(cp, extend_lens=lens)
    plan.upload()
    T = sum(lens)
    x = torch.arange(T * 8, dtype=torch.int32).reshape(T, 8)
    dst = torch.full((cp * plan.M, 8), -1, dtype=torch.int32, device="cuda")
    zz.shard_rows(plan, x.cuda(), dst)
    torch.cuda.synchronize()
    want = OR.ranked_layout(x.numpy(), ref)
    got = dst.cpu().numpy()
    for r, n in enumerate(ref.per_rank_actual_token):
        rows = slice(r * ref.M, r * ref.M + n)
        assert np.array_equal(got[rows], want[rows])
        assert (got[r * ref.M + n:(r + 1) * ref.M] == -1).all()   # padding untouched


@pytest.mark.parametrize("h_kv,d", [(1, 64), (8, 128)], ids=["vector-copy", "bulk-copy"])
def test_rerange_k_only_and_out_of_range_slots_skipped(h_kv, d):
    cp, lens = 2, [64]
    plan = zz.Plan(cp, extend_lens=lens)
    plan.upload()
    ref = OP.build_metadata(cp, 64, extend_lens=lens)
    kg = torch.randn(cp * plan.M, h_kv, d).to(torch.bfloat16).cuda()
    kp = torch.zeros(64, h_kv, d, dtype=torch.bfloat16, device="cuda")
    loc = torch.arange(64, dtype=torch.int64)
    loc[5] = 1000                                    # out of range: must be skipped
    loc[6] = -3
    zz.rerange_kv_to_pool(plan, kg, None, kp, None, loc.cuda())
    torch.cuda.synchronize()
    nat = OR.gather_kv(kg.cpu().view(torch.int16).numpy(), ref)
    got = kp.cpu().view(torch.int16).numpy()
    keep = [t for t in range(64) if t not in (5, 6)]
    assert np.array_equal(got[keep], nat[keep])
    assert (got[5] == 0).all() and (got[6] == 0).all()
    assert plan.device_status() == 0


@pytest.mark.parametrize("cp,lens,width,dtype", [(4, [37, 50, 8], 16, torch.int32),
                                                 (3, [300, 129], 1, torch.int32),   # 4-byte rows
                                                 (2, [64, 90], 3, torch.int32),     # 12-byte rows
                                                 (8, [4096], 2, torch.int64)])
def test_gather_and_take_back_bit_exact(cp, lens, width, dtype):
    ref = OP.build_metadata(cp, sum(lens), extend_lens=lens)
    plan = zz.Plan(cp, extend_lens=lens)
    plan.upload()
    T = sum(lens)
    x = (torch.arange(T * width, dtype=torch.int64).reshape(T, width) * 7 + 3).to(dtype)
    xr = x if width > 1 else x.reshape(T)
    ranked = torch.full((cp * plan.M,) + tuple(xr.shape[1:]), -1, dtype=dtype, device="cuda")
    zz.shard_rows(plan, xr.cuda(), ranked)
    want_ranked = OR.ranked_layout(xr.numpy(), ref)
    got = ranked.cpu().numpy()
    for r, n in enumerate(ref.per_rank_actual_token):
        assert np.array_equal(got[r * ref.M: r * ref.M + n], want_ranked[r * ref.M: r * ref.M + n])
    back = torch.full_like(xr.cuda(), -1)
    zz.gather_rows(plan, ranked, back)          # gather_hidden_states
    torch.cuda.synchronize()
    assert np.array_equal(back.cpu().numpy(), OR.gather_kv(want_ranked, ref))
    for r in range(cp):
        mine = torch.full((ref.per_rank_actual_token[r],) + tuple(xr.shape[1:]), -1, dtype=dtype,
                          device="cuda")
        zz.take_back_rows(plan, r, xr.cuda(), mine)
        torch.cuda.synchronize()
        assert np.array_equal(mine.cpu().numpy(), OR.shard(xr.numpy(), ref, r))
    with pytest.raises(zz.ZZError):
        zz.take_back_rows(plan, cp, xr.cuda(), back)


@pytest.mark.parametrize("cp,lens,h_kv,d,ks,vs", [(4, [4096], 4, 128, 0.37, 2.5),
                                                  (3, [37, 1000, 129], 1, 64, 1e-3, 7.0),   # saturating K
                                                  (8, [32768], 8, 128, 0.05, 0.05)])
def test_rerange_fp8_pool_bit_exact(cp, lens, h_kv, d, ks, vs):
    from oracle import fp8
    ref = OP.build_metadata(cp, sum(lens), extend_lens=lens)
    plan = zz.Plan(cp, extend_lens=lens)
    plan.upload()
    T = sum(lens)
    _, k, v = synth.qkv(T, 1, h_kv, d, seed=9, scale=0.5, dtype="bf16", device="cpu")
    pool = synth.paged_pool(lens, 16, seed=2, spare_pages=1)
    kg = OR.ranked_layout(k.float().numpy(), ref)
    vg = OR.ranked_layout(v.float().numpy(), ref)
    kg_d = torch.from_numpy(kg).to(torch.bfloat16).cuda()   # exact: values are bf16 already
    vg_d = torch.from_numpy(vg).to(torch.bfloat16).cuda()
    kp = torch.full((pool.num_slots, h_kv, d), 0x55, dtype=torch.uint8, device="cuda")
    vp = torch.full_like(kp, 0x55)
    zz.rerange_kv_to_pool_fp8(plan, kg_d, vg_d, kp, vp, torch.from_numpy(pool.out_cache_loc).cuda(), ks, vs)
    torch.cuda.synchronize()
    base = np.full((pool.num_slots, h_kv, d), 0x55, np.uint8)
    want_k = base.copy()
    want_k[pool.out_cache_loc] = fp8.scale_encode(OR.gather_kv(kg, ref), ks)
    want_v = base.copy()
    want_v[pool.out_cache_loc] = fp8.scale_encode(OR.gather_kv(vg, ref), vs)
    assert np.array_equal(kp.cpu().numpy(), want_k)
    assert np.array_equal(vp.cpu().numpy(), want_v)
