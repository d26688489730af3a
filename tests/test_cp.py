"""Context-parallel CSA prefill (long_context_sparse_softmax_b200.cp).

CPU: the partition of a sequence into block-aligned rank ranges, and the two moves between
ranks - the W - 1 row halo from the previous rank and the all-gather of every rank's
entry rows - on two and three gloo ranks, checked row by row.
GPU: two and three ranks stepped in one process on one device (no kernel waits for
another rank's); the outputs of every query are bit-identical to the single-device
prefill of the same sequence, which the other GPU tests check against the oracle."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_sparse_softmax_b200 import cp


@pytest.mark.parametrize("L,m,world", [(4096, 4, 2), (4099, 4, 3), (65536, 4, 8), (1 << 20, 128, 8), (1000, 4, 4)])
def test_partition_is_block_aligned_and_covers_the_sequence(L, m, world):
    ranges, nb = cp.partition(L, m, world)
    assert ranges[0][0] == 0 and ranges[-1][1] == L
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0
    for r, (t0, t1) in enumerate(ranges):
        assert t0 % m == 0
        assert t0 // m == min(r * nb, L // m)      # rank r's first block
        # every complete block of the range is one of rank r's nb blocks
        assert t1 // m - t0 // m <= nb
    assert sum(t1 // m - t0 // m for t0, t1 in ranges) == L // m
    assert cp.halo_range(0, 128) == (0, 0) and cp.halo_range(1000, 128) == (873, 1000)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, L, m, W):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        comm = cp.DistComm()
        ranges, nb = cp.partition(L, m, world)
        t0, t1 = ranges[rank]
        # raw rows labelled with their position
        x = torch.arange(t0, t1, dtype=torch.int64)[:, None].repeat(1, 3)
        h0, _ = cp.halo_range(t0, W)
        halo = comm.halo(x[max(0, x.shape[0] - (W - 1)):], t0 - h0)
        # entry rows labelled with their global index; padding rows stay -1
        full = torch.full((world * nb, 2), -1, dtype=torch.int64)
        for j in range(t0 // m, t1 // m):
            full[j] = torch.tensor([j, 7 * j])
        comm.all_gather_rows(full, nb)
        q.put((rank, halo[:, 0].tolist(), list(range(h0, t0)), full.tolist()))
    except Exception as e:
        q.put((rank, "error", repr(e), None))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,L", [(2, 4096 + 3), (3, 3000)])
def test_halo_and_all_gather_on_gloo_ranks(world, L):
    m, W = 4, 128
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, L, m, W)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = sorted([q.get(timeout=180) for _ in range(world)], key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    n_c = L // m
    for rank, halo, want, full in res:
        assert halo != "error", want
        assert halo == want  # the previous rank's last W - 1 positions, in order
        for j, row in enumerate(full):
            assert row == ([j, 7 * j] if j < n_c else [-1, -1])
    assert all(p.exitcode == 0 for p in procs)


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 3])
def test_cp_prefill_ranks_on_one_gpu_match_single_device_prefill(world):
    from long_context_sparse_softmax_b200 import runner
    from long_context_sparse_softmax_b200 import workloads as wl
    L = 3000
    s = wl.shrink(wl.CSA_PREFILL, name=f"cp_{world}", seed=60 + world, seq_lens=(L,), H=64, k=128, q_first=0, n_q=L)
    inp = wl.make_prefill(s, "cuda")
    ref = runner.Prefill(inp, "cuda")
    ref.step()
    ranges, _ = cp.partition(L, s.m, world)
    ranks = [cp.CpPrefillRank(s, L, r, world, cp.local_inputs(inp, t0, t1), "cuda") for r, (t0, t1) in enumerate(ranges)]
    cp.run_local(ranks)
    torch.cuda.synchronize()
    assert ref.read_status() == 0 and all(int(r.status.item()) == 0 for r in ranks)
    out = torch.cat([r.out.view(-1, s.H, s.Dv) for r in ranks])
    idx = torch.cat([r.idx for r in ranks])
    assert torch.equal(idx, ref.idx)
    assert torch.equal(out, ref.out.view(-1, s.H, s.Dv))
    assert torch.equal(torch.cat([r.lse for r in ranks]), ref.lse)
