"""Layers that share one input (q/k/v projections, gate/up projections) through
macaq_multi_linear_w4a4: one quantiser launch transforms x once per weight, with that
weight's own 1/s, and one GEMM launch covers every weight's tiles. Every output is
compared with the oracle's layer for its own weight; the activation codes and scales
each weight's transform leaves in the workspace are compared bit for bit."""
import numpy as np
import pytest

import oracle
from helpers import (assert_bf16_matches_f32, assert_codes_equal, assert_gemm_close, assert_scales_equal,
                     bf16_dev, f32_dev, host, oracle_on_all_cores)
from mxfp4_w4a4_post_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mq():
    import mxfp4_w4a4_post_b200 as m
    from mxfp4_w4a4_post_b200 import build
    build.build()
    return m


def check_layers(mq, M, K, Ns, dt="f32", pad=0, seed=0):
    import torch
    base = wl.with_shape(wl.tiny_layer(), M=M, N=Ns[0], K=K, seed=seed)
    x = wl.draw_x(base)
    xd = bf16_dev(x)
    layers = [wl.with_shape(base, N=N, seed=seed + 1 + g) for g, N in enumerate(Ns)]
    Ws = [wl.draw_W(L) for L in layers]
    ss = [wl.draw_s(L) for L in layers]
    pws = [mq.prepare_weight(bf16_dev(W), f32_dev(s)) for W, s in zip(Ws, ss)]
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    bigs = [torch.full((M, N + pad), float("nan"), dtype=tdt, device="cuda") for N in Ns]
    ys = [b[:, :N] for b, N in zip(bigs, Ns)]
    ws = torch.full((mq.lib().macaq_multi_linear_workspace_bytes(M, K, len(Ns)),), 0xFF, dtype=torch.uint8,
                    device="cuda")
    mq.multi_linear(xd, pws, ys=ys, workspace=ws)
    torch.cuda.synchronize()
    rows_pad = (M + 127) // 128 * 128
    off_scales = (len(Ns) * rows_pad * (K // 2) + 255) // 256 * 256
    sb = rows_pad * ((K // 32 + 7) // 8 * 8)
    for g, (W, s, pw, y, big, N) in enumerate(zip(Ws, ss, pws, ys, bigs, Ns)):
        with oracle_on_all_cores():
            rwc, rws, rinv = oracle.prepare_weight(W, s)
            rac, ras = oracle.quant_rows(x, rinv)
            ref = oracle.gemm_fp64(rac, ras, rwc, rws, K)
        codes = host(ws[g * rows_pad * (K // 2):g * rows_pad * (K // 2) + M * (K // 2)]).reshape(M, K // 2)
        assert_codes_equal(codes, rac, f"layer {g} activation codes")
        assert_scales_equal(host(ws[off_scales + g * sb:off_scales + (g + 1) * sb]), ras, K, f"layer {g} scales")
        if dt == "f32":
            assert_gemm_close(host(y), ref, f"layer {g} ({M}x{N}x{K})")
        else:
            y32 = mq.linear(xd, pw, out_dtype=torch.float32)
            assert_gemm_close(host(y32), ref, f"layer {g} single ({M}x{N}x{K})")
            assert_bf16_matches_f32(y, y32, f"layer {g} bf16")
        if pad:
            assert torch.isnan(big[:, N:]).all().item(), f"layer {g}: padding columns written"
    assert mq.device_error() == 0


@pytest.mark.parametrize("M,K,Ns,dt,pad", [
    (40, 1024, (520, 136, 64), "f32", 0),
    (300, 768, (384, 200), "bf16", 8),
    (129, 512, (1000,), "f32", 4),
    (256, 1024, (1024, 128, 128), "bf16", 0),
    (256, 12288, (256, 128), "f32", 4),     # few tiles, long K: each tile's K range split over 4 CTAs
])
def test_shared_input_layers(mq, M, K, Ns, dt, pad):
    check_layers(mq, M, K, Ns, dt, pad)


def test_qwen3_32b_qkv_and_gate_up_b256(mq):
    """The decoder-layer shapes at 256 rows: q/k/v (8192/1024/1024 x 5120) and gate/up
    (2 x 25600 x 5120), each set in one launch pair."""
    check_layers(mq, 256, 5120, (8192, 1024, 1024), "f32", 0, seed=3)
    check_layers(mq, 256, 5120, (25600, 25600), "bf16", 0, seed=5)


def test_workspace_reuse_two_calls(mq):
    """Two calls through one workspace with different inputs: the second sees nothing
    of the first (tables and activation codes are rewritten by every call)."""
    check_layers(mq, 64, 512, (256, 96), "f32", 0, seed=7)
    check_layers(mq, 64, 512, (256, 96), "f32", 0, seed=8)
