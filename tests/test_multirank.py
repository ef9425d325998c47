"""Multi-rank plumbing of bench.py on CPU (gloo, two ranks on 127.0.0.1).

The layer has no data-path collective: every rank runs its own layer
(heads and layers are independent problems), so the only collectives are
the max over ranks of the timed region and the sum of the work the ranks
did.  These are checked here with two gloo ranks, and a rank that fails
before a collective must make the other rank's collective end with an
error within the process-group timeout instead of hanging.
"""
import datetime
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank: int, world: int, port: int):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))


def _reduce_worker(rank: int, world: int, port: int, q):
    _env(rank, world, port)
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    r, w, local = bench.dist_env()
    mx = bench.reduce_max(10.0 + rank, w)        # per-rank device time -> max
    sm = bench.reduce_sum(1.5 * (rank + 1), w)   # per-rank work -> sum
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, r, w, local, mx, sm))


def _failing_worker(rank: int, world: int, port: int, q):
    _env(rank, world, port)
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        q.put((rank, "left"))
        q.close()
        q.join_thread()            # the message is out before the process goes
        os._exit(3)                # leaves between steps, before the timing reduction
    try:
        bench.reduce_max(1.0, world)
        q.put((rank, "no error"))
    except Exception as e:         # the collective must fail, not hang
        q.put((rank, type(e).__name__))
    q.close()
    q.join_thread()
    os._exit(0)


def _run(target, world: int, timeout: float):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = []
    for _ in range(world):
        out.append(q.get(timeout=timeout))
    for p in procs:
        p.join(timeout=timeout)
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not exit")
    return sorted(out), [p.exitcode for p in procs]


def test_two_rank_max_and_sum():
    results, codes = _run(_reduce_worker, 2, 120)
    assert codes == [0, 0]
    for rank, r, w, local, mx, sm in results:
        assert (r, w, local) == (rank, 2, rank)
        assert mx == 11.0
        assert sm == 4.5


def test_rank_that_leaves_fails_the_collective():
    results, codes = _run(_failing_worker, 2, 120)
    assert codes == [0, 3]
    assert results[1] == (1, "left")
    assert results[0][0] == 0 and results[0][1] != "no error"
