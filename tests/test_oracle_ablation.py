"""Sanity check, not a parity pin: the ablation paragraph of the openai-hub.com MACaQ
article orders the steps (round-to-nearest MXFP4, then the block rotation, then the
per-channel scale) by falling error. On activations with outlier channels the oracle's
layer must show the same order against the exact x W^T:

    plain MXFP4 (no scale, no rotation)  >  rotation only (s = 1)  >  rotation + scale.

The pages calibrate s and print no rule for it; this test calibrates it as
s_k = sqrt(max_t |x_tk| / max_n |W_nk|) (balancing the two operands' channel ranges), and
the plain baseline quantises x and W block by block with the oracle's own E8M0 exponent
and E2M1 encoder. The seeded workloads' random s is not calibrated, so it is not used
here."""
import numpy as np
import pytest

import oracle
from mxfp4_w4a4_post_b200 import workloads as wl


def plain_mxfp4(a):
    """fp32 rows -> MXFP4 round to nearest (shared exponent per 32, E2M1) -> fp64 values."""
    R, K = a.shape
    blocks = a.reshape(R, K // 32, 32).astype(np.float32)
    e = oracle.e8m0_exponent(np.abs(blocks).max(axis=2).reshape(-1)).reshape(R, K // 32)
    q = (blocks * np.ldexp(np.float32(1.0), -e)[:, :, None].astype(np.float32)).astype(np.float32)
    codes = oracle.e2m1_encode(q.reshape(-1))
    table = np.array([oracle.e2m1_decode(c) for c in range(16)])
    return (table[codes].reshape(q.shape) * np.ldexp(1.0, e)[:, :, None]).reshape(R, K)


def layer(x, W, s, K):
    wc, ws, inv = oracle.prepare_weight(W, s.astype(np.float32))
    ac, as_ = oracle.quant_rows(x, inv)
    return oracle.gemm_fp64(ac, as_, wc, ws, K)


@pytest.mark.parametrize("L", [wl.with_shape(wl.tiny_layer(), M=64, N=256, K=512),
                               wl.with_shape(wl.llama3_8b_gate_up_prefill(), M=64, N=256, K=1024)],
                         ids=["normal_x_two_outlier_channels", "student_t_x_outlier_channels"])
def test_error_falls_with_each_step(L):
    x, W = wl.draw_x(L), wl.draw_W(L)
    xf = wl.bf16_bits_to_f32(x).astype(np.float64)
    Wf = wl.bf16_bits_to_f32(W).astype(np.float64)
    exact = xf @ Wf.T

    def err(y):
        return np.linalg.norm(y - exact) / np.linalg.norm(exact)

    e_plain = err(plain_mxfp4(xf.astype(np.float32)) @ plain_mxfp4(Wf.astype(np.float32)).T)
    e_rot = err(layer(x, W, np.ones(L.K), L.K))
    s_cal = np.clip(np.sqrt(np.abs(xf).max(axis=0) / np.maximum(np.abs(Wf).max(axis=0), 1e-30)), 1e-3, 1e3)
    e_cal = err(layer(x, W, s_cal, L.K))
    assert e_rot < 0.95 * e_plain, (e_plain, e_rot)
    assert e_cal < 0.8 * e_rot, (e_rot, e_cal)
