"""Parity of the activation transform and the weight preparation: the CUDA kernel's
E2M1 codes and E8M0 scales must equal the oracle's bit for bit."""
import math

import numpy as np
import pytest

import oracle
from helpers import (C32, assert_codes_equal, assert_scales_equal, bf16_dev, f32_dev, host)
from mxfp4_w4a4_post_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mq():
    import mxfp4_w4a4_post_b200 as m
    from mxfp4_w4a4_post_b200 import build
    build.build()
    return m


def run_quant(mq, x_u16, mult, ld=None):
    """Quantise through the C ABI; optional row stride ld > K (padded rows)."""
    import torch
    rows, K = x_u16.shape
    if ld is not None and ld != K:
        padded = np.zeros((rows, ld), np.uint16)
        padded[:, :K] = x_u16
        xd = bf16_dev(padded)[:, :K]
    else:
        xd = bf16_dev(x_u16)
    codes, scales = mq.quant_act(xd, f32_dev(mult))
    torch.cuda.synchronize()
    return host(codes), host(scales)


def check_quant(mq, x_u16, mult, what, ld=None):
    codes, scales = run_quant(mq, x_u16, mult, ld)
    rc, rs = oracle.quant_rows(x_u16, mult)
    K = x_u16.shape[1]
    assert_codes_equal(codes, rc, what + " codes")
    assert_scales_equal(scales, rs, K, what + " scales")


def test_tiny_layer_activations(mq):
    L = wl.tiny_layer()
    x, s = wl.draw_x(L), wl.draw_s(L)
    check_quant(mq, x, np.float32(1.0) / s, "tiny x")


def test_tiny_layer_weight_preparation(mq):
    import torch
    L = wl.tiny_layer()
    W, s = wl.draw_W(L), wl.draw_s(L)
    pw = mq.prepare_weight(bf16_dev(W), f32_dev(s))
    torch.cuda.synchronize()
    rc, rs, rinv = oracle.prepare_weight(W, s)
    assert_codes_equal(host(pw.codes), rc, "tiny W codes")
    assert_scales_equal(host(pw.scales), rs, L.K, "tiny W scales")
    assert np.array_equal(host(pw.inv_s).view(np.uint32), rinv.view(np.uint32))


@pytest.mark.parametrize("rows,K,ld", [(1, 32, None), (5, 96, None), (127, 256, None), (128, 288, None),
                                       (129, 800, 808), (300, 4096, None), (7, 25600, 25608),
                                       (2, 64, 72)])
def test_ragged_shapes(mq, rows, K, ld):
    L = wl.with_shape(wl.llama3_8b_gate_up_prefill(), M=rows, K=K)
    x = wl.draw_x(L)
    s = wl.draw_s(L)
    check_quant(mq, x, np.float32(1.0) / s, f"rows={rows} K={K} ld={ld}", ld=ld)


def _bits_bf16(a):
    return (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_special_values(mq):
    """Zero blocks, negative zeros, bf16 subnormals, huge values, powers of two and
    one-hot blocks, all against the oracle."""
    K = 32 * 12
    rows = []
    rows.append(np.zeros(K, np.float32))
    rows.append(-np.zeros(K, np.float32))
    sub = np.full(K, 1e-39, np.float32)                       # bf16 subnormals
    sub[::3] = -2e-40
    rows.append(sub)
    big = np.linspace(-1e35, 1e35, K).astype(np.float32)
    rows.append(big)
    p2 = (2.0 ** np.arange(-20, -20 + K) % 64).astype(np.float32)
    rows.append(p2)
    oh = np.zeros(K, np.float32)
    oh[::32] = 3.0
    oh[40] = -7.0
    rows.append(oh)
    mixed = np.zeros(K, np.float32)
    mixed[:32] = -0.0
    mixed[32:64] = 1e-30
    mixed[64] = 1e30
    mixed[96:128] = np.float32(2.0 ** -130)
    rows.append(mixed)
    x = _bits_bf16(np.stack(rows))
    rng = np.random.default_rng(0)
    for mult in (np.ones(K, np.float32), np.exp(rng.normal(0, 0.5, K)).astype(np.float32)):
        check_quant(mq, x, mult, "special values")


def _neighbours(v, n):
    out = [np.float32(v)]
    lo = hi = np.float32(v)
    for _ in range(n):
        lo = np.nextafter(lo, np.float32(-np.inf))
        hi = np.nextafter(hi, np.float32(np.inf))
        out += [lo, hi]
    return out


def _tie_block(q_tie, e):
    """Multipliers u of a 32-element block (with x = 1) whose transform puts one value
    exactly on the E2M1 rounding midpoint q_tie * 2^e. With u = (D, 0, B, B, ..., B)
    the butterfly's odd-position chain only sees the pair differences (D, 0, 0, ...),
    so t_1 = D exactly, while the even chain sums to about D + 30 B and sets the block
    exponent. D is an fp32 with fl(c D) = q_tie 2^e. Returns None when no fp32 D
    reaches that value (then the midpoint can never occur)."""
    if q_tie < 0:
        u = _tie_block(-q_tie, e)            # the butterfly is odd: -u gives -v exactly
        return None if u is None else -u
    target = np.float32(q_tie * 2.0 ** e)
    Ds = [D for D in _neighbours(target / C32, 16) if np.float32(D * C32) == target]
    for D in Ds:
        for bf in (1.0, 0.5, 0.25):
            u = np.full(32, np.float32(bf * 2.0 ** e), np.float32)
            u[0], u[1] = D, 0.0
            v = oracle.fwht32(u)
            ee = oracle.e8m0_exponent(np.float32(np.abs(v).max()))
            q = v.astype(np.float64) * 2.0 ** -ee
            if ee == e and np.any(q == q_tie):
                return u
    return None


def test_rounding_ties_after_the_transform(mq):
    """Transformed values that land exactly on E2M1 rounding midpoints (0.25, 1.25, 1.75,
    2.5, 3.5, 5 times 2^e, both signs, several e): ties go to the even code. The
    midpoint 0.75 (mantissa 1.1b) is unreachable: no fp32 t has fl(c t) = 1.5 * 2^k."""
    ties = [0.25, 1.25, 1.75, 2.5, 3.5, 5.0]
    blocks = []
    for t in ties:
        for sgn in (1.0, -1.0):
            for e in (-100, -3, 0, 7, 90):
                u = _tie_block(sgn * t, e)
                assert u is not None, (t, sgn, e)
                blocks.append(u)
    assert _tie_block(0.75, 0) is None
    nb = len(blocks)
    K = 32 * nb
    x = np.ones((1, K), np.float32)
    mult = np.concatenate(blocks).astype(np.float32)
    xb = _bits_bf16(x)
    check_quant(mq, xb, mult, "tie blocks")
    # the same blocks, negated activations and rows repeated into a second 128-row slab
    x2 = np.tile(np.concatenate([x, -x]), (70, 1))
    check_quant(mq, _bits_bf16(x2), mult, "tie blocks, 140 rows")


def test_random_blocks_many_magnitudes(mq):
    rng = np.random.default_rng(2)
    rows, K = 64, 32 * 64
    mag = 2.0 ** rng.integers(-60, 60, size=(rows, K // 32)).repeat(32, axis=1)
    x = (rng.standard_t(2, size=(rows, K)) * mag).astype(np.float32)
    x[rng.random((rows, K)) < 0.1] = 0.0
    check_quant(mq, _bits_bf16(x), np.exp(rng.normal(0, 1.0, K)).astype(np.float32), "random magnitudes")
