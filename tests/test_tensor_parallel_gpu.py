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
from helpers import assert_gemm_close, bf16_dev, f32_dev, host
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
