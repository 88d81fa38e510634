"""End-to-end parity of the MACaQ W4A4 layer (prepare -> quantise -> FP4 GEMM) through
the C ABI on the seeded workloads, from the tiny layer to the full-size prefill,
decode and decoder-layer shapes. Codes and scales are compared in full, bit for bit;
GEMM outputs on all rows (small shapes) or on sampled rows (large shapes) against
the oracle's fp64 sum of decoded products. The sampled rows cover every 128-row M
tile of the launch and, in each, all four 32-row groups of the scale atom."""
import numpy as np
import pytest

import oracle
from helpers import (assert_bf16_matches_f32, assert_codes_equal, assert_gemm_close, assert_scales_equal,
                     bf16_dev, f32_dev, host, oracle_on_all_cores, tile_covering_rows)
from mxfp4_w4a4_post_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mq():
    import mxfp4_w4a4_post_b200 as m
    from mxfp4_w4a4_post_b200 import build
    build.build()
    return m


def run_layer(mq, layer, sample_rows=None, check_bf16=True):
    import torch
    x, W, s = wl.draw_x(layer), wl.draw_W(layer), wl.draw_s(layer)
    M, N, K = layer.M, layer.N, layer.K
    xd, Wd, sd = bf16_dev(x), bf16_dev(W), f32_dev(s)
    pw = mq.prepare_weight(Wd, sd)
    y32 = mq.linear(xd, pw, out_dtype=torch.float32)
    a_codes, a_scales = mq.quant_act(xd, pw.inv_s)
    torch.cuda.synchronize()
    del Wd

    # weight preparation and activation quantisation: bit-exact in full
    with oracle_on_all_cores():
        rwc, rws, rinv = oracle.prepare_weight(W, s)
        rac, ras = oracle.quant_rows(x, rinv)
    assert np.array_equal(host(pw.inv_s).view(np.uint32), rinv.view(np.uint32)), "inv_s"
    assert_codes_equal(host(pw.codes), rwc, f"{layer.name} W codes")
    assert_scales_equal(host(pw.scales), rws, K, f"{layer.name} W scales")
    assert_codes_equal(host(a_codes), rac, f"{layer.name} x codes")
    assert_scales_equal(host(a_scales), ras, K, f"{layer.name} x scales")

    # the GEMM output against the oracle's fp64 reference: every row, or seeded rows
    # that reach every M tile and every 32-row group of the scale atom
    rows = np.arange(M) if sample_rows is None or M <= sample_rows else tile_covering_rows(M, sample_rows)
    with oracle_on_all_cores():
        ref = oracle.gemm_fp64(rac, ras, rwc, rws, K, rows=rows)
    fro, mx = assert_gemm_close(host(y32)[rows], ref, layer.name)
    if check_bf16:
        y16 = mq.linear(xd, pw, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert_bf16_matches_f32(y16, y32, layer.name)
    return fro, mx


def test_tiny_layer(mq):
    run_layer(mq, wl.tiny_layer())


def test_tiny_layer_reference_values(mq):
    """The tiny layer's fp32 output equals the oracle's fp64 product to fp32 rounding:
    every 32-block partial sum is exact in fp32, so only the cross-block adds round."""
    import torch
    L = wl.tiny_layer()
    x, W, s = wl.draw_x(L), wl.draw_W(L), wl.draw_s(L)
    pw = mq.prepare_weight(bf16_dev(W), f32_dev(s))
    y = host(mq.linear(bf16_dev(x), pw, out_dtype=torch.float32)).astype(np.float64)
    rwc, rws, rinv = oracle.prepare_weight(W, s)
    rac, ras = oracle.quant_rows(x, rinv)
    ref = oracle.gemm_fp64(rac, ras, rwc, rws, L.K)
    # any fp32 summation of the 8 exact block sums errs by at most 7 u sum|a w|
    absprod = np.abs(oracle.dequant_rows(rac, ras, L.K)) @ np.abs(oracle.dequant_rows(rwc, rws, L.K)).T
    assert np.all(np.abs(y - ref) <= 8 * 2.0 ** -24 * absprod)


def test_quality_sanity_against_unquantised(mq):
    """Not a parity pin: on the outlier-heavy tiny layer the W4A4 output stays close to
    the unquantised x W^T (the layer is a faithful approximation)."""
    import torch
    L = wl.with_shape(wl.tiny_layer(), M=64, N=256, K=512)
    x, W, s = wl.draw_x(L), wl.draw_W(L), wl.draw_s(L)
    pw = mq.prepare_weight(bf16_dev(W), f32_dev(s))
    y = host(mq.linear(bf16_dev(x), pw, out_dtype=torch.float32)).astype(np.float64)
    exact = wl.bf16_bits_to_f32(x).astype(np.float64) @ wl.bf16_bits_to_f32(W).astype(np.float64).T
    rel = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    assert rel < 0.25, rel


@pytest.mark.parametrize("batch", [1, 8, 16, 64])
def test_qwen3_32b_up_decode(mq, batch):
    run_layer(mq, wl.qwen3_32b_up_decode(batch))


def test_qwen3_32b_up_decode_t3_variant(mq):
    run_layer(mq, wl.qwen3_32b_up_decode_t3(16))


def test_llama3_8b_gate_up_prefill(mq):
    run_layer(mq, wl.llama3_8b_gate_up_prefill(), sample_rows=256)


def test_qwen3_32b_down_prefill(mq):
    run_layer(mq, wl.qwen3_32b_down_prefill(), sample_rows=256, check_bf16=False)


@pytest.mark.parametrize("idx", range(7))
def test_qwen3_32b_decoder_layer_b256(mq, idx):
    run_layer(mq, wl.qwen3_32b_layer_decode(256)[idx])


def test_ragged_layer(mq):
    run_layer(mq, wl.with_shape(wl.llama3_8b_gate_up_prefill(), M=333, N=1111, K=1056))


def test_strided_activations(mq):
    """x with a row stride larger than K (a view into a wider buffer)."""
    import torch
    L = wl.with_shape(wl.tiny_layer(), M=40, N=256, K=512)
    x, W, s = wl.draw_x(L), wl.draw_W(L), wl.draw_s(L)
    wide = np.zeros((40, 520), np.uint16)
    wide[:, :512] = x
    xd = bf16_dev(wide)[:, :512]
    pw = mq.prepare_weight(bf16_dev(W), f32_dev(s))
    y = host(mq.linear(xd, pw, out_dtype=torch.float32))
    rwc, rws, rinv = oracle.prepare_weight(W, s)
    rac, ras = oracle.quant_rows(x, rinv)
    assert_gemm_close(y, oracle.gemm_fp64(rac, ras, rwc, rws, 512), "strided x")


def test_device_error_word_is_clear(mq):
    assert mq.device_error() == 0


# (M, N, K): decode shapes for the fused transform (one launch; the GEMM kernel makes
# the MXFP4 activations in shared memory; also on the stream-K schedule), a K whose block
# count needs scale padding and a partial last K tile, shapes beyond the default row
# limit of the fused path, and two above what the kernel takes (the call then runs the
# two-launch path).
FUSED_CASES = [(1, 25600, 5120), (2, 19000, 4096), (1, 300, 800), (2, 1000, 96), (1, 700, 4128),
               (16, 25600, 5120), (32, 4096, 5120), (7, 300, 800), (64, 4096, 5120), (128, 1024, 768)]


@pytest.mark.parametrize("M,N,K", FUSED_CASES)
def test_fused_transform(mq, M, N, K):
    """macaq_linear_w4a4 with fused = 2 (one launch wherever the kernel takes the shape) and
    fused = 1 (one launch where it is faster): y is bit-identical to the two-launch layer
    (fused = 0: the quantiser kernel, then the GEMM with the same tile plan), for fp32 and
    bf16 output, on two inputs in a row through one workspace, and within the GEMM
    tolerance of the oracle."""
    import torch
    L = wl.with_shape(wl.tiny_layer(), M=M, N=N, K=K)
    W, s = wl.draw_W(L), wl.draw_s(L)
    pw = mq.prepare_weight(bf16_dev(W), f32_dev(s))
    rwc, rws, rinv = oracle.prepare_weight(W, s)
    need = mq.linear_workspace_bytes(M, N, K, torch.float32)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")
    for seed in (21, 22):
        x = wl.draw_x(wl.with_shape(L, seed=seed))
        xd = bf16_dev(x)
        y = mq.linear(xd, pw, out_dtype=torch.float32, workspace=ws, fused="always")
        y_two = mq.linear(xd, pw, out_dtype=torch.float32, fused=False)
        y_auto = mq.linear(xd, pw, out_dtype=torch.float32, fused=True)
        y16 = mq.linear(xd, pw, out_dtype=torch.bfloat16, workspace=ws, fused="always")
        y16_two = mq.linear(xd, pw, out_dtype=torch.bfloat16, fused=False)
        torch.cuda.synchronize()
        assert np.array_equal(host(y).view(np.uint32), host(y_two).view(np.uint32)), f"fused {M}x{N}x{K} fp32"
        assert np.array_equal(host(y_auto).view(np.uint32), host(y_two).view(np.uint32)), f"fused=1 {M}x{N}x{K}"
        assert torch.equal(y16.view(torch.int16), y16_two.view(torch.int16)), f"fused {M}x{N}x{K} bf16"
        rac, ras = oracle.quant_rows(x, rinv)
        assert_gemm_close(host(y), oracle.gemm_fp64(rac, ras, rwc, rws, K), f"fused {M}x{N}x{K} seed {seed}")
    assert mq.device_error() == 0


def test_fused_transform_strided(mq):
    """The fused transform reads x through its row stride (a view into a wider buffer)."""
    import torch
    M, N, K = 9, 640, 1024
    L = wl.with_shape(wl.tiny_layer(), M=M, N=N, K=K)
    x, W, s = wl.draw_x(L), wl.draw_W(L), wl.draw_s(L)
    wide = np.zeros((M, K + 24), np.uint16)
    wide[:, :K] = x
    xd = bf16_dev(wide)[:, :K]
    pw = mq.prepare_weight(bf16_dev(W), f32_dev(s))
    y = mq.linear(xd, pw, out_dtype=torch.float32, fused="always")
    y_two = mq.linear(bf16_dev(x), pw, out_dtype=torch.float32, fused=False)
    torch.cuda.synchronize()
    assert np.array_equal(host(y).view(np.uint32), host(y_two).view(np.uint32))
