"""Push-form all-gather + rerange (zz_rerange_push_kv) against the oracle (GPU).

On one GPU every destination pool is a tensor on this device: virtual rank r's
push writes its rows into all destination pools, and once every rank has
pushed, each pool must equal the oracle's all-gather + rerange + pool write bit
for bit, with every slot outside the tokens untouched.  A two-process test maps
the other process's pool through the IPC helpers (both processes on this GPU,
no kernel waits on another) and checks the same.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import synth
from oracle import plan as OP
from oracle import rerange as OR
from tests._lib import ensure_built

zz = ensure_built()
pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    return (t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)).numpy()


def _setup(cp, lens, h_kv, d, dtype, ps, seed=3):
    ref = OP.build_metadata(cp, sum(lens), extend_lens=lens)
    plan = zz.Plan(cp, extend_lens=lens)
    plan.upload()
    _, k, v = synth.qkv(sum(lens), 1, h_kv, d, seed=seed, scale=0.5, dtype=dtype, device="cpu")
    pool = synth.paged_pool(lens, ps, seed=5, spare_pages=2)
    kb, vb = _bits(k), _bits(v)
    kg, vg = OR.ranked_layout(kb, ref), OR.ranked_layout(vb, ref)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    sentinel = np.full((pool.num_slots, h_kv, d), 0x7A5A if dtype == "bf16" else 0x3F7A5A5A, dtype=kb.dtype)
    return ref, plan, pool, kg, vg, tdt, sentinel


CASES = [
    # cp, lens, h_kv, d, dtype, page_size, destinations
    (2, [300, 212], 2, 128, "bf16", 16, 2),
    (4, [517, 263, 1000], 1, 64, "fp32", 32, 4),
    (3, [97], 4, 128, "bf16", 8, 3),
    (4, synth.varlen_lengths(8, 1000, 8192, seed=0), 4, 128, "bf16", 16, 4),
    (8, [32768], 8, 128, "bf16", 64, 8),
    (4, [4096], 4, 128, "bf16", 16, 1),     # one destination: the plain rerange
    (2, [64], 2, 64, "bf16", 16, 16),       # ZZ_MAX_PUSH_DST destinations
]


@pytest.mark.parametrize("cp,lens,h_kv,d,dtype,ps,n_dst", CASES)
def test_push_every_rank_fills_every_pool(cp, lens, h_kv, d, dtype, ps, n_dst):
    ref, plan, pool, kg, vg, tdt, sentinel = _setup(cp, lens, h_kv, d, dtype, ps)
    M = plan.M
    kg_d = torch.from_numpy(kg).view(tdt).cuda()
    vg_d = torch.from_numpy(vg).view(tdt).cuda()
    kps = [torch.from_numpy(sentinel.copy()).view(tdt).cuda() for _ in range(n_dst)]
    vps = [torch.from_numpy(sentinel.copy()).view(tdt).cuda() for _ in range(n_dst)]
    loc = torch.from_numpy(pool.out_cache_loc).cuda()
    for r in range(cp):
        zz.rerange_push_kv(plan, r, kg_d[r * M:(r + 1) * M], vg_d[r * M:(r + 1) * M], kps, vps,
                           [loc] * n_dst, pool.num_slots)
    torch.cuda.synchronize()
    want_k = OR.rerange_to_pool(kg, ref, sentinel, pool.out_cache_loc)
    want_v = OR.rerange_to_pool(vg, ref, sentinel, pool.out_cache_loc)
    for j in range(n_dst):
        assert np.array_equal(_bits(kps[j]), want_k), f"K pool {j}"
        assert np.array_equal(_bits(vps[j]), want_v), f"V pool {j}"


def test_push_per_destination_maps_k_only_and_skipped_slots():
    """Each destination has its own slot map; slots outside the pool are skipped."""
    cp, lens, h_kv, d = 3, [40, 71], 2, 64
    ref, plan, pool, kg, vg, tdt, sentinel = _setup(cp, lens, h_kv, d, "bf16", 8)
    M, T = plan.M, sum(lens)
    loc_a = pool.out_cache_loc.copy()
    rng = np.random.default_rng(11)
    loc_b = rng.permutation(pool.num_slots)[:T].astype(np.int64)      # another allocator state
    loc_b[::7] = -1
    loc_b[3::11] = pool.num_slots + 5                                    # out of range: skipped
    kg_d = torch.from_numpy(kg).view(tdt).cuda()
    kps = [torch.from_numpy(sentinel.copy()).view(tdt).cuda() for _ in range(2)]
    locs = [torch.from_numpy(loc_a).cuda(), torch.from_numpy(loc_b).cuda()]
    for r in range(cp):
        zz.rerange_push_kv(plan, r, kg_d[r * M:(r + 1) * M], None, kps, None, locs, pool.num_slots)
    torch.cuda.synchronize()
    rows = OR.gather_kv(kg, ref)
    assert np.array_equal(_bits(kps[0]), OR.write_pool(sentinel, loc_a, rows))
    keep = (loc_b >= 0) & (loc_b < pool.num_slots)
    assert np.array_equal(_bits(kps[1]), OR.write_pool(sentinel, loc_b[keep], rows[keep]))


def test_push_argument_errors():
    cp, lens = 2, [64]
    plan = zz.Plan(cp, extend_lens=lens)
    plan.upload()
    M = plan.M
    k = torch.zeros(M, 2, 64, dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros(256, 2, 64, dtype=torch.bfloat16, device="cuda")
    loc = torch.arange(64, dtype=torch.int64, device="cuda")
    for bad_rank in (-1, cp):
        with pytest.raises(zz.ZZError, match="rank out of range"):
            zz.rerange_push_kv(plan, bad_rank, k, None, [pool], None, [loc], 256)
    with pytest.raises(zz.ZZError, match="n_dst"):
        zz.rerange_push_kv(plan, 0, k, None, [pool] * 17, None, [loc] * 17, 256)
    with pytest.raises(zz.ZZError, match="both be set"):
        zz.rerange_push_kv(plan, 0, k, k, [pool], None, [loc], 256)
    with pytest.raises(zz.ZZError, match="16-byte aligned"):
        zz.rerange_push_kv(plan, 0, k, None, [pool.data_ptr() + 8], None, [loc], 256)
    with pytest.raises(zz.ZZError, match="NULL destination"):
        zz.rerange_push_kv(plan, 0, k, None, [0], None, [loc], 256)
    st = zz.raw_call("zz_rerange_push_kv", plan.handle, 0, k.data_ptr(), None, None, None, None, 1,
                     256, 2, 64, zz.ZZ_BF16, None)
    assert st == zz.ZZ_ERR_INVALID_ARG


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ipc_worker(rank, world, port, out_q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    mapped = []
    try:
        import bench
        from tests._lib import ensure_built as eb
        zzw = eb()
        torch.cuda.set_device(0)
        cp, lens, h_kv, d, ps = 2 * world, [300, 517], 2, 128, 16
        ref = OP.build_metadata(cp, sum(lens), extend_lens=lens)
        plan = zzw.Plan(cp, extend_lens=lens)
        plan.upload()
        M = plan.M
        _, k, v = synth.qkv(sum(lens), 1, h_kv, d, seed=3, scale=0.5, dtype="bf16", device="cpu")
        kg, vg = OR.ranked_layout(_bits(k), ref), OR.ranked_layout(_bits(v), ref)
        pool = synth.paged_pool(lens, ps, seed=5, spare_pages=2)
        sentinel = np.full((pool.num_slots, h_kv, d), 0x7A5A, dtype=np.int16)
        kp = torch.from_numpy(sentinel.copy()).view(torch.bfloat16).cuda()
        vp = torch.from_numpy(sentinel.copy()).view(torch.bfloat16).cuda()
        loc = torch.from_numpy(pool.out_cache_loc).cuda()
        r0, r_per = bench.rank_range(cp, world, rank)
        k_local = torch.from_numpy(kg[r0 * M:(r0 + r_per) * M]).view(torch.bfloat16).cuda()
        v_local = torch.from_numpy(vg[r0 * M:(r0 + r_per) * M]).view(torch.bfloat16).cuda()
        dsts, mapped = bench.exchange_pools(dist, zzw.ipc_export, zzw.PeerBuffer, [kp, vp], rank, world)
        bench.push_all_local(zzw, plan, r0, r_per, M, k_local, v_local, dsts, loc, pool.num_slots)
        torch.cuda.synchronize()
        dist.barrier()                      # every process's pushes have completed
        want_k = OR.rerange_to_pool(kg, ref, sentinel, pool.out_cache_loc)
        want_v = OR.rerange_to_pool(vg, ref, sentinel, pool.out_cache_loc)
        ok = bool(np.array_equal(_bits(kp), want_k) and np.array_equal(_bits(vp), want_v))
        dist.barrier()                      # nobody reads a peer pool any more
        for m in mapped:
            m.close()
        mapped = []
        dist.barrier()
        out_q.put((rank, ok, ""))
    except Exception as e:  # report, never hang the parent
        out_q.put((rank, False, repr(e)))
    finally:
        for m in mapped:
            m.close()
        dist.destroy_process_group()


def test_push_into_peer_pool_over_ipc_two_processes():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    for rank, ok, err in sorted(res):
        assert ok, f"process {rank}: {err or 'pool differs from the oracle'}"
