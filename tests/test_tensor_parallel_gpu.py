"""Tensor-parallel layers on one B200. (1) Shard exactness of the CUDA path: a K shard
cut on 32-element boundaries, prepared on its own, gives the unsharded prepared
weight's codes, scales and 1/s for those columns bit for bit, and a row shard its rows.
(2) The shards' layers, run one after another on the one GPU, joined on the host,
match the oracle's unsharded layer. (3) The module's own path with its NCCL collective
in a one-rank process group."""
import socket

import numpy as np
import pytest

import oracle
from helpers import assert_bf16_matches_f32, assert_gemm_close, bf16_dev, f32_dev, host
from mxfp4_w4a4_post_b200 import workloads as wl
from mxfp4_w4a4_post_b200.tensor_parallel import split_k, split_range

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mq():
    import mxfp4_w4a4_post_b200 as m
    from mxfp4_w4a4_post_b200 import build
    build.build()
    return m


def rowmajor_scales(atoms, rows, K):
    return oracle.unswizzle_scales(host(atoms), rows, K)


def layer(M, N, K):
    L = wl.with_shape(wl.tiny_layer(), M=M, N=N, K=K)
    return L, wl.draw_x(L), wl.draw_W(L), wl.draw_s(L)


@pytest.mark.parametrize("world", [2, 3, 4])
def test_shards_are_exact(mq, world):
    M, N, K = 64, 300, 800
    L, x, W, s = layer(M, N, K)
    Wd, sd = bf16_dev(W), f32_dev(s)
    full = mq.prepare_weight(Wd, sd)
    fc, fs, fi = host(full.codes), rowmajor_scales(full.scales, N, K), host(full.inv_s)
    for r in range(world):
        k0, k1 = split_k(K, world, r)
        sh = mq.prepare_weight(Wd[:, k0:k1], sd[k0:k1].contiguous())
        assert np.array_equal(host(sh.codes), fc[:, k0 // 2:k1 // 2]), (world, r)
        assert np.array_equal(rowmajor_scales(sh.scales, N, k1 - k0), fs[:, k0 // 32:k1 // 32]), (world, r)
        assert np.array_equal(host(sh.inv_s).view(np.uint32), fi[k0:k1].view(np.uint32))
        n0, n1 = split_range(N, world, r)
        shn = mq.prepare_weight(Wd[n0:n1], sd)
        assert np.array_equal(host(shn.codes), fc[n0:n1])
        assert np.array_equal(rowmajor_scales(shn.scales, n1 - n0, K), fs[n0:n1])


@pytest.mark.parametrize("M,N,K", [(16, 256, 4096), (200, 520, 1024)])
def test_shard_layers_joined_on_host(mq, M, N, K):
    import torch
    world = 4
    L, x, W, s = layer(M, N, K)
    xd, Wd, sd = bf16_dev(x), bf16_dev(W), f32_dev(s)
    wc, ws, winv = oracle.prepare_weight(W, s)
    ac, as_ = oracle.quant_rows(x, winv)
    y_ref = oracle.gemm_fp64(ac, as_, wc, ws, K)
    cols = []
    for r in range(world):
        n0, n1 = split_range(N, world, r)
        cols.append(mq.linear(xd, mq.prepare_weight(Wd[n0:n1], sd), out_dtype=torch.float32))
    y_col = host(torch.cat(cols, dim=1))
    assert_gemm_close(y_col, y_ref, "column shards joined")
    y_row = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    for r in range(world):
        k0, k1 = split_k(K, world, r)
        w = mq.prepare_weight(Wd[:, k0:k1], sd[k0:k1].contiguous())
        y_row += mq.linear(xd[:, k0:k1], w, out_dtype=torch.float32)
    assert_gemm_close(host(y_row), y_ref, "K shards summed")
    assert mq.device_error() == 0


def test_module_with_nccl_one_rank(mq):
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    from mxfp4_w4a4_post_b200.tensor_parallel import ColumnParallelW4A4, RowParallelW4A4
    s_ = socket.socket()
    s_.bind(("127.0.0.1", 0))
    port = s_.getsockname()[1]
    s_.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        M, N, K = 40, 384, 512
        L, x, W, s = layer(M, N, K)
        xd, Wd, sd = bf16_dev(x), bf16_dev(W), f32_dev(s)
        wc, ws, winv = oracle.prepare_weight(W, s)
        ac, as_ = oracle.quant_rows(x, winv)
        y_ref = oracle.gemm_fp64(ac, as_, wc, ws, K)
        col = ColumnParallelW4A4.from_full(Wd, sd)
        assert (col.n0, col.n1) == (0, N)
        assert_gemm_close(host(col.forward(xd, out_dtype=torch.float32)), y_ref, "column-parallel, NCCL")
        row = RowParallelW4A4.from_full(Wd, sd)
        assert (row.k0, row.k1) == (0, K)
        assert_gemm_close(host(row.forward(xd, out_dtype=torch.float32)), y_ref, "row-parallel, NCCL")
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert mq.device_error() == 0


# (M, N, K, shards): prefill tiles, decode (swapped) tiles, and a shape for which the
# ordinary layer runs on the stream-K schedule (the gathered output never does)
GATHER_CASES = [(200, 520, 1024, 2), (5, 300, 512, 3), (16, 256, 16384, 2), (8, 40000, 512, 2)]


@pytest.mark.parametrize("M,N,K,shards", GATHER_CASES)
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_gathered_column_cut(mq, M, N, K, shards, dt):
    """Every shard writes its columns straight into two full-width outputs (local
    buffers standing in for two ranks' y; no rank waits on another): both equal the
    oracle's unsharded layer, and their pad columns and the guard bytes around them
    are untouched."""
    import torch
    from mxfp4_w4a4_post_b200.tensor_parallel import ColumnParallelW4A4
    dtype = torch.float32 if dt == "f32" else torch.bfloat16
    L, x, W, s = layer(M, N, K)
    xd, Wd, sd = bf16_dev(x), bf16_dev(W), f32_dev(s)
    ld, guard = N + 8, 4096
    esz = 4 if dt == "f32" else 2
    raws = [torch.full((2 * guard + M * ld * esz,), 0xA5, dtype=torch.uint8, device="cuda") for _ in range(2)]
    ys = [r[guard:guard + M * ld * esz].view(dtype).view(M, ld)[:, :N] for r in raws]
    shard_out = []
    for r in range(shards):
        n0, n1 = split_range(N, shards, r)
        w = mq.prepare_weight(Wd[n0:n1], sd)
        ColumnParallelW4A4(N, K, n0, n1, w).forward_into(xd, ys)
        shard_out.append((n0, n1, w))
    torch.cuda.synchronize()
    for raw in raws:
        b = host(raw)
        assert (b[:guard] == 0xA5).all() and (b[-guard:] == 0xA5).all(), "guard bytes changed"
        full = b[guard:-guard].view(np.uint16 if esz == 2 else np.uint32).reshape(M, ld)
        assert (full[:, N:].view(np.uint8) == 0xA5).all(), "pad columns changed"
    y0, y1 = host(ys[0].float()), host(ys[1].float())
    assert np.array_equal(y0, y1)
    wc, ws, winv = oracle.prepare_weight(W, s)
    ac, as_ = oracle.quant_rows(x, winv)
    ref = oracle.gemm_fp64(ac, as_, wc, ws, K)
    if dt == "f32":
        assert_gemm_close(y0, ref, f"gathered column cut {M}x{N}x{K}")
    # each shard's columns equal the ordinary layer's output for that shard whenever
    # that one computes every tile over its whole K range on one CTA or a CTA pair (same
    # K order per tile, same MMAs, another store path): no stream-K workspace, and no K
    # split over a cluster, which these shapes (K <= 1024 at prefill rows, or decode
    # rows) never get
    for n0, n1, w in shard_out:
        y_lin = mq.linear(xd, w, out_dtype=dtype)
        if mq.gemm_workspace_bytes(M, n1 - n0, K, dtype) == 0:
            assert torch.equal(ys[0][:, n0:n1], y_lin), (n0, n1)
        else:
            y32 = mq.linear(xd, w, out_dtype=torch.float32)
            if dt == "f32":
                assert_gemm_close(host(ys[0][:, n0:n1]), host(y32).astype(np.float64), "stream-K shard")
            else:
                assert_bf16_matches_f32(ys[0][:, n0:n1], y32, "stream-K shard")
    assert mq.device_error() == 0
