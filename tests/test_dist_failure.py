"""Multi-process host logic on the CPU (gloo): ordering of the push exchange,
and what the surviving ranks see when a rank fails or leaves between steps.

* Push form: each rank writes its rows into every rank's pool, so a rank's
  next push can overwrite a pool that another rank's attention is still
  reading.  ``bench.kv_exchange`` fences on both sides of the push; pools in
  shared memory and a deliberately slow reader show that the fence before the
  push is what keeps the reader's data intact (without it the test sees the
  overwrite).
* Failure: a rank exits, raises, or stops between steps.  The survivors'
  heartbeat (``bench.heartbeat``, a bounded wait on the process group's store)
  names the missing rank within its timeout, before any collective of the
  step is launched.  A collective that a peer never joins is bounded by the
  process group's timeout and raises instead of hanging.
No GPU is involved: failures are made on the host.
"""
import os
import socket
import time

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _put_and_exit(q, item, code):
    """Queue ``item`` and leave at once.  ``put`` only hands the item to a feeder
    thread; close + join_thread flush it to the pipe before os._exit, which
    would otherwise drop it."""
    q.put(item)
    q.close()
    q.join_thread()
    os._exit(code)


def _init(rank, world, port, timeout_s=60):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=timeout_s))


# ---------------------------------------------------------------- push ordering
ROWS = 64


def _push_worker(rank, world, port, pools, steps, with_war_fence, out_q):
    _init(rank, world, port)
    try:
        import bench
        fence_t = torch.zeros(1)
        errors = 0

        def fence():
            dist.all_reduce(fence_t)

        for i in range(steps):
            value = float(i + 1)

            def push():    # this rank's rows into every rank's pool
                for j in range(world):
                    pools[j][rank * ROWS:(rank + 1) * ROWS] = value

            if with_war_fence:
                bench.kv_exchange(world, True, fence, push, None, None)
            else:          # the same exchange without the fence before the push
                push()
                fence()
            # "attention": read this rank's pool; rank 0 reads slowly, so a peer
            # that pushes step i+1 too early overwrites what it is still reading
            for _ in range(5):
                if not bool((pools[rank] == value).all()):
                    errors += 1
                time.sleep(0.05 if rank == 0 else 0.0)
        out_q.put((rank, errors))
    finally:
        dist.destroy_process_group()


def _run_push(with_war_fence, world=2, steps=4):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    pools = [torch.zeros(world * ROWS).share_memory_() for _ in range(world)]
    procs = [ctx.Process(target=_push_worker, args=(r, world, port, pools, steps, with_war_fence, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    return res


def test_push_exchange_fences_before_and_after_the_push():
    res = _run_push(with_war_fence=True)
    assert all(e == 0 for e in res.values()), f"a pool changed while it was read: {res}"


def test_without_the_fence_before_the_push_the_reader_sees_an_overwrite():
    """The planted race: it must be visible, or the test above proves nothing."""
    res = _run_push(with_war_fence=False)
    assert res[0] > 0


def test_kv_exchange_order_on_one_rank_and_in_the_gather_form():
    import bench
    log = []
    bench.kv_exchange(2, True, lambda: log.append("fence"), lambda: log.append("push"), None, None)
    assert log == ["fence", "push", "fence"]
    log.clear()
    bench.kv_exchange(1, True, None, lambda: log.append("push"), None, None)
    assert log == ["push"]
    log.clear()
    bench.kv_exchange(2, False, None, None, lambda: log.append("gather"), lambda: log.append("rerange"))
    assert log == ["gather", "rerange"]
    log.clear()
    bench.kv_exchange(1, False, None, None, lambda: log.append("gather"), lambda: log.append("rerange"))
    assert log == ["rerange"]


# ---------------------------------------------------------------- failures
HB_TIMEOUT = 3.0


def _fail_worker(rank, world, port, mode, out_q):
    _init(rank, world, port, timeout_s=4)
    import bench
    store = dist.distributed_c10d._get_default_store()
    t = torch.ones(1)
    try:
        for step in range(3):
            if rank == world - 1 and step == 1:      # the failing rank, between steps 0 and 1
                if mode == "exit":
                    os._exit(0)                      # leaves without a word
                if mode == "raise":
                    raise RuntimeError("host-side failure injected between steps")
                if mode == "stall":
                    time.sleep(3 * HB_TIMEOUT)       # alive, but never reaches step 1
                    out_q.put((rank, "stalled", 0.0))
                    return
            t0 = time.monotonic()
            try:
                bench.heartbeat(store, f"step{step}", rank, world, HB_TIMEOUT)
            except bench.RankFailure as e:
                out_q.put((rank, str(e), time.monotonic() - t0))
                return
            dist.all_reduce(t)                       # the step's collective
        out_q.put((rank, "completed", 0.0))
    except RuntimeError as e:
        if "injected" in str(e):
            _put_and_exit(out_q, (rank, "raised", 0.0), 1)
        raise


@pytest.mark.parametrize("mode", ["exit", "raise", "stall"])
def test_survivors_report_a_rank_that_left_between_steps(mode):
    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_fail_worker, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    survivors = {}
    deadline = time.monotonic() + 120
    while len(survivors) < world - 1 and time.monotonic() < deadline:
        rank, msg, waited = q.get(timeout=120)
        if rank != world - 1:
            survivors[rank] = (msg, waited)
    for p in procs:
        p.join(timeout=30)
        if p.is_alive():
            p.kill()
    assert sorted(survivors) == list(range(world - 1))
    for rank, (msg, waited) in survivors.items():
        assert f"ranks [{world - 1}] did not reach step1" in msg, msg
        assert HB_TIMEOUT * 0.9 <= waited < HB_TIMEOUT + 5.0      # bounded, not a hang


def _collective_worker(rank, world, port, out_q):
    _init(rank, world, port, timeout_s=3)
    t = torch.ones(1)
    if rank == 1:
        time.sleep(6)                                # never joins the collective in time
        _put_and_exit(out_q, (rank, "slept", 0.0), 0)
    t0 = time.monotonic()
    try:
        dist.all_reduce(t)
        item = (rank, "returned", time.monotonic() - t0)
    except Exception as e:  # gloo raises on the process-group timeout
        item = (rank, type(e).__name__, time.monotonic() - t0)
    _put_and_exit(out_q, item, 0)


def test_a_collective_nobody_joins_ends_with_an_error_within_the_group_timeout():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_collective_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    while 0 not in got:
        rank, what, waited = q.get(timeout=60)
        got[rank] = (what, waited)
    for p in procs:
        p.join(timeout=30)
        if p.is_alive():
            p.kill()
    what, waited = got[0]
    assert what != "returned"
    assert waited < 3 + 5.0


def test_gather_buffers_are_plain_tensors_without_nccl():
    import bench
    k, v, reg = bench.gather_buffers(dist, torch, "cpu", (8, 2, 4), torch.float32, world=1)
    assert reg["kind"] == "plain" and k.shape == v.shape == (8, 2, 4)
    bench.release_gather_buffers(reg)               # nothing registered: a no-op
