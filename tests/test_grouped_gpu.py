"""Parity of the grouped (mixture-of-experts) layer with the oracle applied group by
group: every expert's activation codes and scales (read from the padded workspace) bit
for bit, and every expert's output rows within the GEMM tolerance. Synthetic routing:
token counts per expert from a seeded skewed draw, tokens already sorted by expert."""
import numpy as np
import pytest

import oracle
from helpers import (assert_bf16_matches_f32, assert_codes_equal, assert_gemm_close, assert_scales_equal, bf16_dev,
                     f32_dev, host)
from mxfp4_w4a4_post_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mq():
    import mxfp4_w4a4_post_b200 as m
    from mxfp4_w4a4_post_b200 import build
    build.build()
    return m


def experts(G, N, K, seed0=300):
    """Per expert: its weight and channel scale (own seed, so its own transform)."""
    out = []
    for g in range(G):
        L = wl.with_shape(wl.tiny_layer(), M=1, N=N, K=K, seed=seed0 + g)
        out.append((wl.draw_W(L), wl.draw_s(L)))
    return out


def run_grouped(mq, sizes, N, K, out="f32", check_codes=True):
    import torch
    G = len(sizes)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    M = int(offsets[-1])
    x = wl.draw_x(wl.with_shape(wl.tiny_layer(), M=M, N=N, K=K, seed=77))
    ex = experts(G, N, K)
    pws = [mq.prepare_weight(bf16_dev(W), f32_dev(s)) for W, s in ex]
    need = mq.lib().macaq_grouped_linear_workspace_bytes((__import__("ctypes").c_int64 * (G + 1))(*offsets), G, K)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")
    dt = torch.float32 if out == "f32" else torch.bfloat16
    y = host(mq.grouped_linear(bf16_dev(x), list(offsets), pws, out_dtype=dt, workspace=ws).float())
    torch.cuda.synchronize()
    kb_pad = (K // 32 + 7) // 8 * 8
    cb = -(-max(sum(-(-m // 128) * 128 for m in sizes), 128) * (K // 2) // 256) * 256
    wsh = host(ws)
    row_p = 0
    for g, (W, s) in enumerate(ex):
        m = sizes[g]
        if m:
            rwc, rws, rinv = oracle.prepare_weight(W, s)
            xg = x[offsets[g]:offsets[g + 1]]
            ac, as_ = oracle.quant_rows(xg, rinv)
            if check_codes:
                codes = wsh[row_p * (K // 2):(row_p + m) * (K // 2)].reshape(m, K // 2)
                assert_codes_equal(codes, ac, f"expert {g} codes")
                pad = -(-m // 128) * 128
                atoms = wsh[cb + row_p * kb_pad: cb + (row_p + pad) * kb_pad]
                assert_scales_equal(atoms, as_, K, f"expert {g} scales")
            rows = np.arange(m) if m <= 64 else np.unique(np.concatenate(
                [np.random.default_rng(g).choice(m, 48, replace=False), [0, m - 1]]))
            ref = oracle.gemm_fp64(ac, as_, rwc, rws, K, rows=rows)
            yg = y[offsets[g]:offsets[g + 1]][rows]
            if out == "f32":
                assert_gemm_close(yg, ref, f"expert {g}")
            else:
                rel = np.linalg.norm(yg - ref) / max(np.linalg.norm(ref), 1e-30)
                assert rel < 4e-3, (g, rel)
        row_p += -(-m // 128) * 128
    assert mq.device_error() == 0
    return y


@pytest.mark.parametrize("sizes,N,K", [([3, 0, 130, 128, 257], 320, 512), ([5, 0, 0], 128, 256),
                                      ([1, 1, 1, 1], 200, 1024), ([300], 448, 768)])
def test_grouped_ragged(mq, sizes, N, K):
    run_grouped(mq, sizes, N, K)


def test_grouped_routed_tokens(mq):
    """1024 tokens over 8 experts with a skewed routing (seeded), bf16 output."""
    rng = np.random.default_rng(5)
    p = 1.0 / np.arange(1, 9) ** 1.2
    counts = np.bincount(rng.choice(8, 1024, p=p / p.sum()), minlength=8).tolist()
    run_grouped(mq, counts, 1024, 2048, out="bf16", check_codes=False)


def test_grouped_matches_per_expert_calls(mq):
    """The grouped launch and eight separate layer calls agree to fp32 accumulation
    order (the separate calls may take other tile shapes for small groups)."""
    import torch
    sizes = [40, 0, 200, 7, 129, 64, 1, 300]
    N, K = 384, 512
    offsets = np.concatenate([[0], np.cumsum(sizes)])
    x = wl.draw_x(wl.with_shape(wl.tiny_layer(), M=int(offsets[-1]), N=N, K=K, seed=78))
    xd = bf16_dev(x)
    pws = [mq.prepare_weight(bf16_dev(W), f32_dev(s)) for W, s in experts(len(sizes), N, K)]
    y = host(mq.grouped_linear(xd, list(offsets), pws, out_dtype=torch.float32))
    for g, m in enumerate(sizes):
        if m:
            yg = host(mq.linear(xd[offsets[g]:offsets[g + 1]], pws[g], out_dtype=torch.float32)).astype(np.float64)
            d = np.linalg.norm(y[offsets[g]:offsets[g + 1]] - yg) / max(np.linalg.norm(yg), 1e-30)
            assert d < 1e-5, (g, d)
