"""Parity of Flip-Refinement (offline refinement of weight codes) with the oracle: the
full fp64 Gram matrix of transformed calibration rows, and the refined codes and move
counts of every row, bit for bit; on the Llama-3-8B gate/up weight (14336 x 4096) on
sampled rows."""
import numpy as np
import pytest

import oracle
from helpers import assert_codes_equal, assert_gemm_close, bf16_dev, f32_dev, host
from mxfp4_w4a4_post_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mq():
    import mxfp4_w4a4_post_b200 as m
    from mxfp4_w4a4_post_b200 import build
    build.build()
    return m


def calib(L, T, seed=101):
    return wl.draw_x(wl.with_shape(L, M=T, seed=seed))


@pytest.mark.parametrize("T,K", [(1, 32), (200, 256), (129, 640)])
def test_hessian_full_bit_exact(mq, T, K):
    L = wl.with_shape(wl.tiny_layer(), M=T, N=32, K=K)
    x, s = calib(L, T), wl.draw_s(L)
    H = host(mq.hessian_full(bf16_dev(x), f32_dev(s)))
    ref = oracle.hessian_full(x, (np.float32(1.0) / s).astype(np.float32))
    assert np.array_equal(H.view(np.uint64), ref.view(np.uint64)), np.argwhere(H != ref)[:5]


@pytest.mark.parametrize("N,K,hess", [(48, 256, False), (70, 512, True), (9, 1024, False)])
def test_flip_refine_bit_exact(mq, N, K, hess):
    """Starting from round-to-nearest (or from the Hessian exponent search), every row's
    refined codes and its number of moves equal the oracle's."""
    import torch
    L = wl.with_shape(wl.tiny_layer(), M=256, N=N, K=K)
    W, s, x = wl.draw_W(L), wl.draw_s(L), calib(L, 256)
    xd, Wd, sd = bf16_dev(x), bf16_dev(W), f32_dev(s)
    H = mq.hessian_full(xd, sd)
    if hess:
        Hb = mq.hessian_blocks(xd, sd)
        pw = mq.prepare_weight_hessian(Wd, sd, Hb)
    else:
        pw = mq.prepare_weight(Wd, sd)
    torch.cuda.synchronize()
    c0 = host(pw.codes).copy()
    sc_rm = oracle.unswizzle_scales(host(pw.scales), N, K)
    moves = host(mq.flip_refine(Wd, sd, H, pw))
    torch.cuda.synchronize()
    rc, rmoves = oracle.flip_refine(W, s, host(H), c0, sc_rm, 1 << 20)
    assert np.array_equal(moves, rmoves), (moves[:8], rmoves[:8])
    assert moves.sum() > 0
    assert_codes_equal(host(pw.codes), rc, f"flip codes {N}x{K}")


def test_flip_refine_round_cap(mq):
    import torch
    L = wl.with_shape(wl.tiny_layer(), M=128, N=16, K=256)
    W, s, x = wl.draw_W(L), wl.draw_s(L), calib(L, 128)
    Wd, sd = bf16_dev(W), f32_dev(s)
    H = mq.hessian_full(bf16_dev(x), sd)
    pw = mq.prepare_weight(Wd, sd)
    torch.cuda.synchronize()
    c0 = host(pw.codes).copy()
    sc_rm = oracle.unswizzle_scales(host(pw.scales), 16, 256)
    moves = host(mq.flip_refine(Wd, sd, H, pw, max_rounds=3))
    rc, rmoves = oracle.flip_refine(W, s, host(H), c0, sc_rm, 3)
    assert np.array_equal(moves, rmoves) and (moves <= 3).all()
    assert_codes_equal(host(pw.codes), rc, "flip codes, 3 rounds")


def test_flip_refine_llama3_8b_gate_up(mq):
    """Full-size weight (14336 x 4096, 512 calibration rows) on the GPU; the oracle
    refines 4 sampled rows with the same H and compares codes and move counts."""
    import torch
    L = wl.llama3_8b_gate_up_prefill()
    W, s = wl.draw_W(L), wl.draw_s(L)
    x = calib(L, 512)
    xd, Wd, sd = bf16_dev(x), bf16_dev(W), f32_dev(s)
    H = mq.hessian_full(xd, sd)
    pw = mq.prepare_weight(Wd, sd)
    torch.cuda.synchronize()
    c0 = host(pw.codes).copy()
    moves = host(mq.flip_refine(Wd, sd, H, pw, max_rounds=256))
    torch.cuda.synchronize()
    Hh = host(H)
    rows = np.array([0, 1234, 9001, L.N - 1])
    sc_rm = oracle.unswizzle_scales(host(pw.scales), L.N, L.K)[rows]
    rc, rmoves = oracle.flip_refine(W[rows], s, Hh, c0[rows], sc_rm, 256)
    assert np.array_equal(moves[rows], rmoves), (moves[rows], rmoves)
    assert_codes_equal(host(pw.codes)[rows], rc, "gate/up flip codes (sampled rows)")
    assert mq.device_error() == 0


def test_flip_refined_weights_through_the_layer(mq):
    """Refined weight bytes go through the unchanged GEMM, and the layer's output error
    against the unquantised product, on the calibration rows, does not grow."""
    import torch
    L = wl.with_shape(wl.tiny_layer(), M=256, N=256, K=512)
    W, s, x = wl.draw_W(L), wl.draw_s(L), calib(L, 256)
    xd, Wd, sd = bf16_dev(x), bf16_dev(W), f32_dev(s)
    H = mq.hessian_full(xd, sd)
    pw0 = mq.prepare_weight(Wd, sd)
    pw = mq.prepare_weight(Wd, sd)
    mq.flip_refine(Wd, sd, H, pw)
    y0 = host(mq.linear(xd, pw0, out_dtype=torch.float32)).astype(np.float64)
    y1 = host(mq.linear(xd, pw, out_dtype=torch.float32)).astype(np.float64)
    torch.cuda.synchronize()
    rc, rs, rinv = oracle.prepare_weight(W, s)
    ac, as_ = oracle.quant_rows(x, rinv)
    wc = host(pw.codes)
    assert_gemm_close(y1, oracle.gemm_fp64(ac, as_, wc, rs, L.K), "flip-refined layer")
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    Wf = (W.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    y = xf @ Wf.T
    assert np.linalg.norm(y1 - y) <= np.linalg.norm(y0 - y)
    assert mq.device_error() == 0
