"""Failure detection on the GPU without a fault: the GEMM kernel's bounded wait routines
are run by a self-test kernel against waits that cannot succeed (an mbarrier nothing
arrives at) with a short limit. Each wait must give up after the limit, record its code
and raise the CTA abort flag; a second wait in the same CTA must leave on that flag;
waits that can succeed must succeed; and a group of warps whose member gave up must
agree to leave together at its named barrier instead of holding the others there.
Afterwards the context must still run the layer correctly."""
import numpy as np
import pytest

import oracle
from helpers import assert_codes_equal, assert_gemm_close, assert_scales_equal, bf16_dev, f32_dev, host
from mxfp4_w4a4_post_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ERR_TIMEOUT_PRODUCER = 1
ERR_TIMEOUT_SET = 5


@pytest.fixture(scope="module")
def mq():
    import mxfp4_w4a4_post_b200 as m
    from mxfp4_w4a4_post_b200 import build
    build.build()
    return m


@pytest.mark.parametrize("limit_us", [1000, 20000])
def test_bounded_waits_give_up(mq, limit_us):
    r = mq.selftest_wait_timeout(limit_us)
    limit_ns = limit_us * 1000
    # mbarrier wait that nothing completes: gives up after the limit with its own code
    assert r["bar_timeout_ok"] == 0
    assert r["bar_err"] == ERR_TIMEOUT_PRODUCER
    assert limit_ns <= r["bar_timeout_ns"] < limit_ns + 500_000_000
    # the second wait (2 s limit) left on the abort flag, long before its own limit
    assert r["bar_abort_ok"] == 0
    assert r["bar_abort_ns"] < 1_000_000_000
    # a barrier that completes is seen completing
    assert r["bar_done_ok"] == 1
    # a warp group whose member gave up agrees to leave; the member's wait took the
    # limit and recorded its code, the others' own waits completed, and none was held
    assert r["set_agreed_ok"] == 0
    assert r["set_err"] == ERR_TIMEOUT_SET
    assert limit_ns <= r["set_timeout_ns"] < limit_ns + 500_000_000
    assert r["set_member_ok"] == 1
    # the layer's own error word is untouched
    assert mq.device_error() == 0


def test_context_usable_after_timeouts(mq):
    import torch
    mq.selftest_wait_timeout(500)
    L = wl.with_shape(wl.tiny_layer(), M=200, N=256, K=512)
    x, W, s = wl.draw_x(L), wl.draw_W(L), wl.draw_s(L)
    w = mq.prepare_weight(bf16_dev(W), f32_dev(s))
    codes, scales = mq.quant_act(bf16_dev(x), w.inv_s)
    y = mq.linear(bf16_dev(x), w, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rc, rs = oracle.quant_rows(x, (np.float32(1.0) / s).astype(np.float32))
    assert_codes_equal(host(codes), rc, "codes after self-test")
    assert_scales_equal(host(scales), rs, L.K, "scales after self-test")
    wc, ws, _ = oracle.prepare_weight(W, s)
    assert_gemm_close(host(y), oracle.gemm_fp64(rc, rs, wc, ws, L.K), "layer after self-test")
    assert mq.device_error() == 0
