"""The multi-GPU path of bench.py is replicas only (sequences are
independent; no collective on the data path): every rank runs its own
decoder and the job's time is the slowest rank's.  These tests run that
host logic as two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=2)
    try:
        # rank 0 is slower in the first value, rank 1 in the second
        got = bench.max_over_ranks([10.0 - rank, 1.0 + rank], "cpu", 2)
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res[0] == res[1] == [10.0, 2.0]


def test_single_rank_is_identity():
    assert bench.max_over_ranks([3.5, 7.0], "cpu", 1) == [3.5, 7.0]


@pytest.mark.parametrize("ws", [1, 2, 8])
def test_replica_throughput_is_weak_scaling(ws):
    # 64 tokens per rank per step at 2 ms (slowest rank): ws * 32000 tokens/s
    assert bench.replica_throughput(64, 2.0, ws) == pytest.approx(32000.0 * ws)
