"""Parity of the Hessian exponent search (offline weight preparation) with the oracle:
the fp64 Gram blocks of transformed calibration rows and the codes / scales chosen per
weight block are compared bit for bit, on small shapes in full and on the Llama-3-8B
gate/up weight (14336 x 4096) on sampled rows."""
import numpy as np
import pytest

import oracle
from helpers import assert_codes_equal, assert_gemm_close, assert_scales_equal, bf16_dev, f32_dev, host
from mxfp4_w4a4_post_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mq():
    import mxfp4_w4a4_post_b200 as m
    from mxfp4_w4a4_post_b200 import build
    build.build()
    return m


def calib(L, T, seed=101):
    """Calibration activations with the workload's own distribution, another seed."""
    return wl.draw_x(wl.with_shape(L, M=T, seed=seed))


@pytest.mark.parametrize("T,K", [(1, 64), (300, 256), (129, 800)])
def test_hessian_blocks_bit_exact(mq, T, K):
    L = wl.with_shape(wl.tiny_layer(), M=T, N=32, K=K)
    x, s = calib(L, T), wl.draw_s(L)
    H = host(mq.hessian_blocks(bf16_dev(x), f32_dev(s)))
    ref = oracle.hessian_blocks(x, (np.float32(1.0) / s).astype(np.float32))
    assert np.array_equal(H.view(np.uint64), ref.view(np.uint64)), np.argwhere(H != ref)[:5]


@pytest.mark.parametrize("N,K", [(300, 256), (130, 800), (7, 32)])
def test_prepare_weight_hessian_bit_exact(mq, N, K):
    L = wl.with_shape(wl.tiny_layer(), M=64, N=N, K=K)
    W, s, x = wl.draw_W(L), wl.draw_s(L), calib(L, 64)
    Hd = mq.hessian_blocks(bf16_dev(x), f32_dev(s))
    pw = mq.prepare_weight_hessian(bf16_dev(W), f32_dev(s), Hd)
    import torch
    torch.cuda.synchronize()
    rc, rs, rinv = oracle.prepare_weight_hessian(W, s, host(Hd))
    assert np.array_equal(host(pw.inv_s).view(np.uint32), rinv.view(np.uint32))
    assert_codes_equal(host(pw.codes), rc, f"hessian codes {N}x{K}")
    assert_scales_equal(host(pw.scales), rs, K, f"hessian scales {N}x{K}")
    # the search moved some exponents away from the floor rule
    _, s0, _ = oracle.prepare_weight(W, s)
    assert (rs != s0).any()


def test_prepare_weight_hessian_llama3_8b_gate_up(mq):
    """Full-size weight on the GPU; the oracle checks 24 sampled rows (rows are
    independent) and the scale padding of the whole buffer stays zero."""
    import torch
    L = wl.llama3_8b_gate_up_prefill()
    W, s = wl.draw_W(L), wl.draw_s(L)
    x = calib(L, 512)
    Hd = mq.hessian_blocks(bf16_dev(x), f32_dev(s))
    H = host(Hd)
    assert np.array_equal(H.view(np.uint64),
                          oracle.hessian_blocks(x, (np.float32(1.0) / s).astype(np.float32)).view(np.uint64))
    pw = mq.prepare_weight_hessian(bf16_dev(W), f32_dev(s), Hd)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.random.default_rng(3).choice(L.N, 22, replace=False), [0, L.N - 1]]))
    rc, rs, _ = oracle.prepare_weight_hessian(W[rows], s, H)
    codes = host(pw.codes)
    assert_codes_equal(codes[rows], rc, "gate/up hessian codes (sampled rows)")
    atoms = host(pw.scales)
    for i, r in enumerate(rows):
        for b in range(L.K // 32):
            assert atoms[oracle.scale_offset(int(r), b, L.K)] == rs[i, b], (r, b)


def test_hessian_weights_through_the_layer(mq):
    """The searched weight bytes go through the unchanged GEMM: y matches the oracle's
    fp64 product of the same codes."""
    import torch
    L = wl.with_shape(wl.tiny_layer(), M=48, N=384, K=512)
    W, s, x = wl.draw_W(L), wl.draw_s(L), wl.draw_x(L)
    Hd = mq.hessian_blocks(bf16_dev(calib(L, 256)), f32_dev(s))
    pw = mq.prepare_weight_hessian(bf16_dev(W), f32_dev(s), Hd)
    y = mq.linear(bf16_dev(x), pw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rc, rs, rinv = oracle.prepare_weight_hessian(W, s, host(Hd))
    ac, as_ = oracle.quant_rows(x, rinv)
    assert_gemm_close(host(y), oracle.gemm_fp64(ac, as_, rc, rs, L.K), "hessian layer")
    assert mq.device_error() == 0
