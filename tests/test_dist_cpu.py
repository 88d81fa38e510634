"""Host logic of the multi-GPU bench path on CPU: two gloo ranks run the same replica
bookkeeping bench.py uses under torchrun (max-over-ranks timing, whole-job
aggregation, workload selection), with no GPU and no data-path collective."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        r, w, local = bench.dist_env()
        t_max = bench.reduce_max(0.5 + rank)            # rank 1 is the slow one
        L = bench.workloads_by_name()[bench.DEFAULT_WORKLOAD]
        value = bench.aggregate(bench.gemm_flops(L), t_max, w)
        q.put((r, w, local, t_max, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    flops = 2.0 * 4096 * 14336 * 4096
    for r, (rank, w, local, t_max, value) in enumerate(res):
        assert rank == r and w == world and local == r
        assert t_max == 1.5                               # max over ranks, same on every rank
        assert value == pytest.approx(flops * world / 1.5 / 1e12)


def test_single_process_defaults(monkeypatch):
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (0, 1, 0)
    assert bench.reduce_max(2.5) == 2.5
    args = bench.parse_args([])
    assert args.gpus == 1 and args.impl == "ours" and args.workload == bench.DEFAULT_WORKLOAD
