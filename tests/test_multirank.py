"""The multi-rank host logic of bench.py on two gloo ranks (CPU).

Under torchrun every rank runs its own batch of the workload (weak scaling, no data-path
collective): each rank reads its rank from the environment, draws its inputs from its own
seed, and the job's time is the slowest rank's, reduced with an all-reduce MAX.  The value
is then the tokens of all ranks over that time."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, port: int, q) -> None:
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import bench
    from long_context_sparse_softmax_b200 import workloads as wl
    r, w, local = bench.dist_env()
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=datetime.timedelta(seconds=60))
    try:
        # the slowest rank's time wins
        t = bench.max_over_ranks(10.0 + 5.0 * r, "cpu", w)
        # each rank's own inputs: same shapes, its own seed
        spec = wl.shrink(bench.rank_spec(wl.CSA_DECODE, r), name="multirank", seq_lens=(512, 700), k=64)
        inp = wl.make_decode(spec, "cpu")
        sums = [None] * w
        dist.all_gather_object(sums, (spec.seed, float(inp["q_raw"].float().sum()), tuple(inp["q_raw"].shape)))
        q.put((r, w, local, t, sums))
    except Exception as e:  # report instead of hanging the other rank's queue read
        q.put((r, "error", repr(e)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    try:
        res = sorted([q.get(timeout=180) for _ in range(WORLD)], key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    for item in res:
        assert item[1] != "error", item
    for r, (rank, w, local, t, sums) in enumerate(res):
        assert (rank, w, local) == (r, WORLD, r)
        assert t == 15.0  # max of 10 and 15
        seeds = [s[0] for s in sums]
        assert seeds == [1, 1001]  # rank 0 keeps the workload's seed
        assert sums[0][2] == sums[1][2]  # same shapes
        assert sums[0][1] != sums[1][1]  # different inputs
    assert all(p.exitcode == 0 for p in procs)


def test_weak_throughput_counts_every_rank():
    import bench
    # 2 ranks x 32 query tokens x 10 steps in 15 ms
    assert bench.weak_throughput(2, 32, 10, 15.0) == pytest.approx(2 * 32 * 10 / 0.015)
    assert bench.max_over_ranks(3.5, "cpu", 1) == 3.5
    assert bench.dist_env() == (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                                int(os.environ.get("LOCAL_RANK", "0")))
