"""Multi-process (gloo, world size 2, CPU) check of the N>1 host logic.

Each process owns c/N virtual ranks, builds its rank-local K shard from the
C planner's token -> row map, and the shards are all-gathered with the same
helper bench.py uses.  The gathered buffer must equal the oracle's padded
rank-ordered layout, and the oracle's rerange of it must give natural order.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, cp, lens, out_q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        from oracle import plan as OP
        from oracle import rerange as OR
        from tests._lib import ensure_built
        zz = ensure_built()
        plan = zz.Plan(cp, extend_lens=lens)
        M, T = plan.M, plan.total_tokens
        r0, r_per = bench.rank_range(cp, world, rank)
        k_nat = torch.arange(T * 3, dtype=torch.int32).reshape(T, 3) + 1
        src_row = np.array(plan.get("src_row"))
        local = torch.zeros(r_per * M, 3, dtype=torch.int32)
        mine = (src_row >= r0 * M) & (src_row < (r0 + r_per) * M)
        local[torch.from_numpy(src_row[mine] - r0 * M)] = k_nat[torch.from_numpy(np.nonzero(mine)[0])]
        gathered = torch.zeros(cp * M, 3, dtype=torch.int32)
        bench.all_gather_rows(dist, gathered, local)
        ref = OP.build_metadata(cp, T, extend_lens=lens)
        want = OR.ranked_layout(k_nat.numpy(), ref)
        ok_layout = bool(np.array_equal(gathered.numpy(), want))
        ok_nat = bool(np.array_equal(OR.gather_kv(gathered.numpy(), ref), k_nat.numpy()))
        out_q.put((rank, r0, r_per, ok_layout, ok_nat))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cp,lens", [(4, [37, 50]), (8, [300]), (2, [17, 9, 33])])
def test_two_process_allgather_layout_matches_oracle(cp, lens):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, cp, lens, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    owned = sorted(r for _, r0, n, _, _ in results for r in range(r0, r0 + n))
    assert owned == list(range(cp))                  # every virtual rank exactly once
    assert all(ok for *_, ok, _ in results), "gathered buffer differs from the oracle layout"
    assert all(ok for *_, ok in results), "rerange of the gathered buffer is not natural order"


def test_rank_range_rejects_uneven_split():
    import bench
    with pytest.raises(ValueError):
        bench.rank_range(6, 4, 0)


class _FakeMap:
    def __init__(self, handle, offset, log):
        self.ptr = 1_000_000 * int(handle.decode().split(":")[1]) + offset
        self.handle = handle
        self.closed = False
        log.append(handle)

    def close(self):
        self.closed = True


def _exchange_worker(rank, world, port, out_q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        # K and V of one rank share an allocation ("alloc:<rank>"), at offsets 0 and 4096
        pools = ["K", "V"]
        export = lambda t: (f"alloc:{rank + 1}".encode(), 0 if t == "K" else 4096)  # noqa: E731
        log = []
        dsts, mapped = bench.exchange_pools(dist, export, lambda h, o: _FakeMap(h, o, log), pools,
                                            rank, world)
        out_q.put((rank, dsts, [m.handle for m in mapped], log))
    finally:
        dist.destroy_process_group()


def test_exchange_pools_orders_destinations_by_rank():
    """Destination j of the push is rank j's pool; this rank's own tensors stay
    tensors; one mapping per peer allocation, shared by K and V."""
    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_exchange_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
    for rank, dsts, mapped, log in res:
        for j in range(world):
            if j == rank:
                assert dsts[0][j] == "K" and dsts[1][j] == "V"
            else:
                assert dsts[0][j] == 1_000_000 * (j + 1)
                assert dsts[1][j] == 1_000_000 * (j + 1) + 4096
        assert sorted(mapped) == sorted(f"alloc:{j + 1}".encode() for j in range(world) if j != rank)
        assert len(log) == world - 1
