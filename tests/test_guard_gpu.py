"""Out-of-bounds writes (in place of a memory checker): every output buffer, and every
workspace, sits inside a larger allocation whose guard regions before and after it are
filled with 0xA5; a strided y also has pad columns between its rows. After each call the
guards and pad columns must still hold 0xA5. Small shapes: single blocks, ragged row
counts and widths, the stream-K schedule, the fused transform, grouped experts."""
import numpy as np
import pytest

import oracle
from helpers import assert_bf16_matches_f32, assert_gemm_close, bf16_dev, f32_dev, host
from mxfp4_w4a4_post_b200 import workloads as wl

pytestmark = pytest.mark.gpu

GUARD = 4096
FILL = 0xA5


@pytest.fixture(scope="module")
def mq():
    import mxfp4_w4a4_post_b200 as m
    from mxfp4_w4a4_post_b200 import build
    build.build()
    return m


class Guarded:
    """A byte buffer of `nbytes` with GUARD bytes of FILL on both sides (base 4 KB aligned)."""

    def __init__(self, nbytes):
        import torch
        self.nbytes = int(nbytes)
        self.raw = torch.full((GUARD + self.nbytes + GUARD,), FILL, dtype=torch.uint8, device="cuda")
        self.body = self.raw[GUARD:GUARD + self.nbytes]

    def as_(self, dtype, shape):
        return self.body.view(dtype).view(shape)

    def check(self, what):
        import torch
        torch.cuda.synchronize()
        r = host(self.raw)
        for name, part in (("before", r[:GUARD]), ("after", r[GUARD + self.nbytes:])):
            bad = np.flatnonzero(part != FILL)
            assert bad.size == 0, f"{what}: {bad.size} guard bytes {name} the buffer changed (first {bad[:4]})"


def strided_y(M, N, ld, dtype):
    """y [M, N] with row stride ld >= N inside a guarded buffer; returns (guard, y, full)."""
    import torch
    esz = torch.tensor([], dtype=dtype).element_size()
    g = Guarded(M * ld * esz)
    full = g.as_(dtype, (M, ld))
    return g, full[:, :N], full


def check_pad_columns(full, N, what):
    import torch
    torch.cuda.synchronize()
    pad = host(full[:, N:].contiguous().view(torch.uint8))
    assert (pad == FILL).all(), f"{what}: pad columns between rows changed"


@pytest.mark.parametrize("M,K", [(1, 32), (3, 96), (130, 800)])
def test_quant_act_guards(mq, M, K):
    import torch
    L = wl.with_shape(wl.tiny_layer(), M=M, N=32, K=K)
    x, s = wl.draw_x(L), wl.draw_s(L)
    gc, gs = Guarded(mq.codes_bytes(M, K)), Guarded(mq.scales_bytes(M, K))
    inv = f32_dev((np.float32(1.0) / s).astype(np.float32))
    mq.quant_act(bf16_dev(x), inv, codes=gc.as_(torch.uint8, (M, K // 2)), scales=gs.body)
    gc.check("quant codes")
    gs.check("quant scales")


@pytest.mark.parametrize("N,K", [(7, 32), (300, 256)])
def test_prepare_weight_guards(mq, N, K):
    import torch
    L = wl.with_shape(wl.tiny_layer(), M=4, N=N, K=K)
    W, s = wl.draw_W(L), wl.draw_s(L)
    gc, gs, gi = Guarded(mq.codes_bytes(N, K)), Guarded(mq.scales_bytes(N, K)), Guarded(4 * K)
    out = mq.PreparedWeight(gc.as_(torch.uint8, (N, K // 2)), gs.body, gi.as_(torch.float32, (K,)), N, K)
    mq.prepare_weight(bf16_dev(W), f32_dev(s), out=out)
    for g, what in ((gc, "weight codes"), (gs, "weight scales"), (gi, "inv_s")):
        g.check(what)


# (M, N, K, out dtype, row stride of y): ragged rows and widths, narrow and wide tiles,
# deep K over few tiles, and a stream-K case whose partial tiles and counters live in the
# workspace
GEMM_CASES = [
    (1, 16, 64, "f32", 20),
    (5, 200, 512, "bf16", 208),
    (200, 384, 512, "bf16", 392),
    (130, 136, 256, "f32", 140),
    (16, 256, 16384, "bf16", 264),
    (8, 19100, 768, "f32", 19104),
    (700, 4200, 256, "bf16", 4216),          # CTA pairs, ragged second CTA and weight half
    (300, 700, 12288, "bf16", 712),          # K split over clusters of four CTAs
]


@pytest.mark.parametrize("M,N,K,dt,ld", GEMM_CASES)
@pytest.mark.parametrize("fused", [False, "always"])
def test_linear_guards(mq, M, N, K, dt, ld, fused):
    import torch
    dtype = torch.float32 if dt == "f32" else torch.bfloat16
    L = wl.with_shape(wl.tiny_layer(), M=M, N=N, K=K)
    x, W, s = wl.draw_x(L), wl.draw_W(L), wl.draw_s(L)
    w = mq.prepare_weight(bf16_dev(W), f32_dev(s))
    gy, y, full = strided_y(M, N, ld, dtype)
    gw = Guarded(mq.linear_workspace_bytes(M, N, K, dtype))
    mq.linear(bf16_dev(x), w, y=y, workspace=gw.body, fused=fused)
    gy.check("y")
    gw.check("linear workspace")
    check_pad_columns(full, N, "y")
    y32 = y
    if dtype == torch.bfloat16:
        # bf16 output: within one bf16 ulp of the fp32 output of the same product
        y32 = mq.linear(bf16_dev(x), w, out_dtype=torch.float32, fused=fused)
        assert_bf16_matches_f32(y, y32, f"guarded linear {M}x{N}x{K}")
    rc, rs = oracle.quant_rows(x, (np.float32(1.0) / s).astype(np.float32))
    wc, ws, _ = oracle.prepare_weight(W, s)
    assert_gemm_close(host(y32), oracle.gemm_fp64(rc, rs, wc, ws, K), f"guarded linear {M}x{N}x{K}")
    assert mq.device_error() == 0


def test_hessian_guards(mq):
    import torch
    L = wl.with_shape(wl.tiny_layer(), M=40, N=70, K=96)
    x, W, s = wl.draw_x(L), wl.draw_W(L), wl.draw_s(L)
    K, N = L.K, L.N
    gh = Guarded(8 * K * 32)
    H = gh.as_(torch.float64, (K // 32, 32, 32))
    mq.hessian_blocks(bf16_dev(x), f32_dev(s), H=H)
    gh.check("hessian blocks")
    gc, gs, gi = Guarded(mq.codes_bytes(N, K)), Guarded(mq.scales_bytes(N, K)), Guarded(4 * K)
    out = mq.PreparedWeight(gc.as_(torch.uint8, (N, K // 2)), gs.body, gi.as_(torch.float32, (K,)), N, K)
    mq.prepare_weight_hessian(bf16_dev(W), f32_dev(s), H, out=out)
    for g, what in ((gc, "hessian codes"), (gs, "hessian scales"), (gi, "hessian inv_s")):
        g.check(what)
    gf = Guarded(8 * K * K)
    Hf = gf.as_(torch.float64, (K, K))
    mq.hessian_full(bf16_dev(x), f32_dev(s), H=Hf)
    gf.check("full hessian")
    w = mq.prepare_weight(bf16_dev(W), f32_dev(s))
    gws = Guarded(mq.lib().macaq_flip_workspace_bytes(N, K))
    mq.flip_refine(bf16_dev(W), f32_dev(s), Hf, w, max_rounds=64, workspace=gws.body)
    gws.check("flip workspace")


def test_grouped_guards(mq):
    import torch
    K, N = 256, 136
    offsets = [0, 3, 3, 140, 141]
    M = offsets[-1]
    L = wl.with_shape(wl.tiny_layer(), M=M, N=N, K=K)
    x = wl.draw_x(L)
    weights = []
    for g in range(len(offsets) - 1):
        Lg = wl.with_shape(L, seed=L.seed + 17 * (g + 1))
        weights.append(mq.prepare_weight(bf16_dev(wl.draw_W(Lg)), f32_dev(wl.draw_s(Lg))))
    gy, y, full = strided_y(M, N, N + 8, torch.bfloat16)
    offs = (mq.ctypes.c_int64 * len(offsets))(*offsets)
    gw = Guarded(mq.lib().macaq_grouped_linear_workspace_bytes(offs, len(weights), K))
    mq.grouped_linear(bf16_dev(x), offsets, weights, y=y, workspace=gw.body)
    gy.check("grouped y")
    gw.check("grouped workspace")
    check_pad_columns(full, N, "grouped y")
    assert mq.device_error() == 0
