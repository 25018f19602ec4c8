"""The bench's multi-rank host logic on two CPU ranks (gloo over 127.0.0.1): the max-over-ranks
timing, the barrier, per-rank input seeds (weak scaling) and the whole-job value; and a rank
that never joins: the other rank's collective ends with an error after the process group's
short timeout instead of waiting for good.  No GPU is involved."""
import datetime
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def _rank_main(rank, world, port, q):
    try:
        dist = _init(rank, world, port, 60)
        import bench
        ms = bench.max_over_ranks(1.5 + rank, world)  # rank 1 is the slower one
        bench.barrier(world)
        seeds = [bench.rank_set_seed(1002, rank, i) for i in range(6)]
        q.put((rank, ms, seeds, bench.weak_scaling_value(world, 1000, ms)))
        dist.destroy_process_group()
    except Exception as e:  # reported to the test, not swallowed
        q.put((rank, "error", repr(e), None))


def _absent_peer_main(rank, world, port, q):
    try:
        dist = _init(rank, world, port, 3)
        import bench
        if rank == 1:
            q.put((rank, "left", None))
            return  # leaves between steps, without taking part in the next collective
        try:
            bench.max_over_ranks(1.0, world)
            q.put((rank, "returned", None))
        except Exception as e:
            q.put((rank, "raised", type(e).__name__))
    except Exception as e:
        q.put((rank, "setup-error", repr(e)))


def _run(target, world=2):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    return sorted(out, key=lambda x: x[0])


@pytest.mark.timeout(240)
def test_two_ranks_max_over_ranks_and_weak_scaling():
    out = _run(_rank_main)
    assert all(o[1] != "error" for o in out), out
    assert [o[1] for o in out] == [2.5, 2.5]                  # both ranks see the slowest time
    assert not set(out[0][2]) & set(out[1][2])                # each rank its own input sets
    assert out[0][3] == out[1][3] == 2 * 1000 / 2.5e-3        # all ranks' elements / max time


@pytest.mark.timeout(240)
def test_absent_rank_ends_the_collective_with_an_error():
    out = _run(_absent_peer_main)
    assert out[1][1] == "left"
    assert out[0][1] == "raised", out
