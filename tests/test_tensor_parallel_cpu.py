"""Host logic of the tensor-parallel layers on CPU: two or three gloo ranks cut the weight
(columns, or K on MX-block boundaries), run each rank's share with the oracle as the
per-rank operations, and join the results with the module's own all-gather /
all-reduce. The joined y must equal the oracle's unsharded layer (exactly for the
column cut; within fp32 summation for the K cut), and a K shard's codes, scales and
1/s must be the unsharded ones' columns bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from mxfp4_w4a4_post_b200.tensor_parallel import split_k, split_range


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_split_range_partitions():
    for n in range(0, 70):
        for world in range(1, 6):
            for align in (1, 3, 32):
                pieces = [split_range(n, world, r, align) for r in range(world)]
                assert pieces[0][0] == 0 and pieces[-1][1] == n
                for (lo, hi), (lo2, _) in zip(pieces, pieces[1:]):
                    assert lo <= hi == lo2                      # contiguous, disjoint
                units = [-(-(hi - lo) // align) for lo, hi in pieces]
                assert max(units) - min(units) <= 1             # balanced in whole units
                for lo, hi in pieces:
                    assert (lo % align == 0 or lo == n) and (hi % align == 0 or hi == n)
                    assert units == sorted(units, reverse=True)


def test_split_k_whole_blocks():
    assert [split_k(96, 2, r) for r in range(2)] == [(0, 64), (64, 96)]
    assert [split_k(32, 2, r) for r in range(2)] == [(0, 32), (32, 32)]
    with pytest.raises(ValueError):
        split_k(48, 2, 0)
    with pytest.raises(ValueError):
        split_range(10, 2, 2)


class OracleOps:
    """Per-rank operations computed by the oracle (CPU, fp64 GEMM)."""

    def prepare(self, W, s):
        import oracle
        Wn = W.contiguous().view(_torch().int16).numpy().view(np.uint16)
        return oracle.prepare_weight(Wn, s.contiguous().numpy())

    def linear(self, x, w, out_dtype):
        import oracle
        codes, scales, inv = w
        xn = x.contiguous().view(_torch().int16).numpy().view(np.uint16)
        ac, as_ = oracle.quant_rows(xn, inv)
        y = oracle.gemm_fp64(ac, as_, codes, scales, xn.shape[1])
        return _torch().from_numpy(y).to(out_dtype)

    def linear_gather(self, x, w, dests):
        y = self.linear(x, w, dests[0].dtype)
        for d in dests:
            d.copy_(y)
        return dests


def _torch():
    import torch
    return torch


def _bf16(a):
    return _torch().from_numpy(np.ascontiguousarray(a).view(np.int16)).view(_torch().bfloat16)


def _worker(rank, world, port, shape, q):
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    from mxfp4_w4a4_post_b200 import workloads as wl
    from mxfp4_w4a4_post_b200.tensor_parallel import ColumnParallelW4A4, RowParallelW4A4
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        M, N, K = shape
        L = wl.with_shape(wl.tiny_layer(), M=M, N=N, K=K)
        x, W, s = _bf16(wl.draw_x(L)), _bf16(wl.draw_W(L)), torch.from_numpy(wl.draw_s(L))
        ops = OracleOps()
        col = ColumnParallelW4A4.from_full(W, s, ops=ops)
        yc = col.forward(x, out_dtype=torch.float32).numpy()
        yc_local = col.forward(x, out_dtype=torch.float32, gather=False).numpy()
        row = RowParallelW4A4.from_full(W, s, ops=ops)
        yr = row.forward(x, out_dtype=torch.float32).numpy()
        yr_presliced = row.forward(x[:, row.k0:row.k1].contiguous(), out_dtype=torch.float32).numpy()
        q.put((rank, (col.n0, col.n1), (row.k0, row.k1), yc, yc_local, yr, yr_presliced, row.weight))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,shape", [(2, (5, 70, 160)), (2, (3, 1, 32)), (2, (130, 64, 96)),
                                         (3, (7, 70, 160)), (3, (4, 2, 64))])
def test_multi_rank_column_and_row_parallel(world, shape):
    import oracle
    from mxfp4_w4a4_post_b200 import workloads as wl
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, shape, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    M, N, K = shape
    L = wl.with_shape(wl.tiny_layer(), M=M, N=N, K=K)
    x, W, s = wl.draw_x(L), wl.draw_W(L), wl.draw_s(L)
    wc, ws, winv = oracle.prepare_weight(W, s)
    ac, as_ = oracle.quant_rows(x, winv)
    y_ref = oracle.gemm_fp64(ac, as_, wc, ws, K)
    for rank, (n0, n1), (k0, k1), yc, yc_local, yr, yr_pre, wrow in res:
        assert (n0, n1) == split_range(N, world, rank) and (k0, k1) == split_k(K, world, rank)
        # column cut: every output element is the same dot product as unsharded
        assert np.array_equal(yc, y_ref.astype(np.float32))
        assert np.array_equal(yc_local, y_ref[:, n0:n1].astype(np.float32))
        # K cut: fp32 partial sums of exact fp64 partial products
        scale = np.sqrt(np.mean(y_ref ** 2)) + 1e-30
        assert np.max(np.abs(yr - y_ref)) <= 1e-6 * scale
        assert np.array_equal(yr, yr_pre)
        if k1 > k0:
            c, sc, inv = wrow
            assert np.array_equal(c, wc[:, k0 // 2:k1 // 2])
            assert np.array_equal(sc, ws[:, k0 // 32:k1 // 32])
            assert np.array_equal(inv.view(np.uint32), winv[k0:k1].view(np.uint32))
        else:
            assert wrow is None
    # every rank holds the same joined result
    for r in res[1:]:
        assert np.array_equal(res[0][3], r[3]) and np.array_equal(res[0][5], r[5])


def test_gathered_column_cut_host_logic():
    """forward_into: each rank's shard writes its columns into every full-width output;
    two shards emulated in one process, three outputs, joined without a collective."""
    import torch
    import oracle
    from mxfp4_w4a4_post_b200 import workloads as wl
    from mxfp4_w4a4_post_b200.tensor_parallel import ColumnParallelW4A4
    M, N, K = 6, 70, 96
    L = wl.with_shape(wl.tiny_layer(), M=M, N=N, K=K)
    x, W, s = _bf16(wl.draw_x(L)), _bf16(wl.draw_W(L)), torch.from_numpy(wl.draw_s(L))
    ops = OracleOps()
    ys = [torch.full((M, N), float("nan")) for _ in range(3)]
    for rank in range(2):
        n0, n1 = split_range(N, 2, rank)
        shard = ColumnParallelW4A4(N, K, n0, n1, ops.prepare(W[n0:n1], s), None, ops)
        shard.forward_into(x, ys)
    wc, ws, winv = oracle.prepare_weight(wl.draw_W(L), wl.draw_s(L))
    ac, as_ = oracle.quant_rows(wl.draw_x(L), winv)
    ref = oracle.gemm_fp64(ac, as_, wc, ws, K).astype(np.float32)
    for y in ys:
        assert np.array_equal(y.numpy(), ref)
