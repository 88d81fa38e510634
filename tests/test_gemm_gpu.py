"""Parity of the block-scaled FP4 GEMM (tcgen05 kind::mxf4) with the oracle's fp64 sum
of decoded products. One-hot operands pin the nibble order and the scale layout;
random codes and scales cover every tile path (swapped decode tiles of width 16..128,
prefill tiles of width 128/192, 256 x 192 tiles of CTA pairs, tiles whose K range is
split over a cluster of 2..4 CTAs that finish them as a reduce-scatter of partial
slices, the stream-K schedule whose shared tiles are finished by their last
contributor, ragged M/N/K) and every output path (TMA tensor stores of staged boxes,
direct stores, transposed stores)."""
import numpy as np
import pytest

import oracle
from helpers import (assert_bf16_matches_f32, assert_gemm_close, host, random_mxfp4, u8_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mq():
    import mxfp4_w4a4_post_b200 as m
    from mxfp4_w4a4_post_b200 import build
    build.build()
    return m


def gpu_gemm(mq, a_codes, a_scales_rm, w_codes, w_scales_rm, K, out="f32"):
    """Run the CUDA GEMM on row-major oracle-format operands (scales swizzled into the
    tensor-core layout by the oracle's own layout function)."""
    import torch
    M, N = a_codes.shape[0], w_codes.shape[0]
    a_c = u8_dev(a_codes)
    a_s = u8_dev(oracle.swizzle_scales(a_scales_rm, K))
    w = mq.PreparedWeight(u8_dev(w_codes), u8_dev(oracle.swizzle_scales(w_scales_rm, K)),
                          torch.ones(K, dtype=torch.float32, device="cuda"), N, K)
    dt = torch.float32 if out == "f32" else torch.bfloat16
    y = mq.gemm_mxfp4(a_c, a_s, M, w, out_dtype=dt)
    torch.cuda.synchronize()
    return y


def one_hot_operands(M, N, K, picks):
    """picks: list of (m, n, k, code_a, code_w, ea, ew). Each pick puts one code in row m
    of A and row n of W at column k, with the given block exponents."""
    a = np.zeros((M, K), np.uint8)
    w = np.zeros((N, K), np.uint8)
    sa = np.full((M, K // 32), 127, np.uint8)
    sw = np.full((N, K // 32), 127, np.uint8)
    for m, n, k, ca, cw, ea, ew in picks:
        a[m, k] = ca
        w[n, k] = cw
        sa[m, k // 32] = 127 + ea
        sw[n, k // 32] = 127 + ew
    pack = lambda c: (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    return pack(a), sa, pack(w), sw


# the last two shapes run on CTA pairs (rows 128..255 of each 256-row tile, and weight
# rows 96..191 of each 192-row tile, in the second CTA of the pair) and with each tile's K
# range split over a cluster of four CTAs (every product lands in one CTA's partial tile)
@pytest.mark.parametrize("M,N,K", [(16, 128, 256), (300, 448, 512), (200, 130, 768), (700, 4200, 768),
                                   (130, 300, 12288)])
def test_one_hot_layout(mq, M, N, K):
    rng = np.random.default_rng(M + N + K)
    picks, used_k, used_m, used_n = [], set(), set(), set()
    cand_k = [k for k in range(K) if k % 2 == 0 or k % 7 == 1]
    while len(picks) < min(M, N, 24):
        m, n, k = int(rng.integers(M)), int(rng.integers(N)), int(rng.choice(cand_k))
        if m in used_m or n in used_n or k // 32 in used_k:
            continue
        used_m.add(m), used_n.add(n), used_k.add(k // 32)
        picks.append((m, n, k, int(rng.integers(1, 16)), int(rng.integers(1, 16)),
                      int(rng.integers(-6, 7)), int(rng.integers(-6, 7))))
        if len(used_k) == K // 32:
            break
    a, sa, w, sw = one_hot_operands(M, N, K, picks)
    y = host(gpu_gemm(mq, a, sa, w, sw, K)).astype(np.float64)
    expect = oracle.gemm_fp64(a, sa, w, sw, K)
    for m, n, k, ca, cw, ea, ew in picks:
        v = oracle.e2m1_decode(ca) * oracle.e2m1_decode(cw) * 2.0 ** (ea + ew)
        assert expect[m, n] == v
    assert np.array_equal(y, expect), np.argwhere(y != expect)[:5]


# (M, N, K): swapped decode tiles (M <= 128), prefill tiles (M > 128), ragged tails
SHAPES = [
    (1, 128, 256), (3, 300, 512), (16, 1000, 1024), (17, 256, 5120), (32, 2000, 2048),
    (64, 640, 4096), (100, 384, 1280), (128, 512, 768),
    (129, 224, 256), (256, 1024, 5120), (300, 700, 800), (512, 2240, 2048), (1000, 130, 1536),
    # CTA pairs: a 256-row tile whose second CTA has no rows (M % 256 = 44) or 8 of 128
    # rows in the first, and a last weight tile whose second half is empty (N % 192 = 88)
    # or partly filled (N % 192 = 168)
    (300, 7000, 768), (520, 4200, 768),
    # each tile's K range split over a cluster of 4 CTAs (tiles 128 and 192 wide), 3 and 2
    (300, 700, 12288), (640, 1000, 12288), (1024, 1000, 8192), (1536, 1000, 12288),
]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_random_operands(mq, M, N, K):
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    a, sa = random_mxfp4(rng, M, K)
    w, sw = random_mxfp4(rng, N, K)
    y = host(gpu_gemm(mq, a, sa, w, sw, K))
    rows = np.arange(M) if M <= 256 else np.unique(np.concatenate([rng.choice(M, 48, replace=False), [0, M - 1]]))
    ref = oracle.gemm_fp64(a, sa, w, sw, K, rows=rows)
    assert_gemm_close(y[rows], ref, f"gemm {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(8, 384, 1024), (300, 700, 800)])
def test_bf16_output(mq, M, N, K):
    rng = np.random.default_rng(5)
    a, sa = random_mxfp4(rng, M, K)
    w, sw = random_mxfp4(rng, N, K)
    y32 = gpu_gemm(mq, a, sa, w, sw, K, out="f32")
    y16 = gpu_gemm(mq, a, sa, w, sw, K, out="bf16")
    assert_bf16_matches_f32(y16, y32, f"bf16 {M}x{N}x{K}")


def test_extreme_scales(mq):
    """Scale bytes near both ends of the range the quantiser emits (0 and 252), and
    block sums that cancel exactly."""
    rng = np.random.default_rng(6)
    M, N, K = 64, 256, 512
    a, sa = random_mxfp4(rng, M, K, 0, 5)
    w, sw = random_mxfp4(rng, N, K, 240, 252)
    y = host(gpu_gemm(mq, a, sa, w, sw, K))
    assert_gemm_close(y, oracle.gemm_fp64(a, sa, w, sw, K), "extreme scales")


# (M, N, K, dtype, extra columns of row padding): rows whose byte length is a multiple of
# 16 go through the staged TMA-store epilogue (boxes clipped at ragged M and N edges) or
# vector stores, others through scalar stores; padding columns of a strided output stay
# untouched.
OUTPUT_CASES = [
    (300, 200, 512, "bf16", 0), (300, 200, 512, "f32", 0), (257, 333, 256, "bf16", 0),
    (300, 200, 512, "bf16", 24), (300, 200, 512, "f32", 12), (640, 1000, 768, "bf16", 0),
    (16, 256, 25600, "bf16", 8), (64, 640, 12288, "f32", 3),     # deep K over few tiles
    (1, 25600, 5120, "bf16", 8), (16, 19000, 5376, "f32", 4),    # stream-K: shared tiles
    (700, 4200, 256, "bf16", 0), (300, 7000, 768, "f32", 4),     # CTA pairs
    (1000, 6100, 768, "bf16", 8),                                # CTA pairs, unaligned rows
    (300, 700, 512, "bf16", 12),    # aligned row stride, rows not 16-byte multiples: no tensor store
]


@pytest.mark.parametrize("M,N,K,dt,pad", OUTPUT_CASES)
def test_output_paths(mq, M, N, K, dt, pad):
    import torch
    rng = np.random.default_rng(M + 3 * N + K + pad)
    a, sa = random_mxfp4(rng, M, K)
    w, sw = random_mxfp4(rng, N, K)
    y32 = host(gpu_gemm(mq, a, sa, w, sw, K, out="f32"))
    rows = np.unique(np.concatenate([rng.choice(M, min(M, 40), replace=False), [0, M - 1]]))
    assert_gemm_close(y32[rows], oracle.gemm_fp64(a, sa, w, sw, K, rows=rows), f"f32 {M}x{N}x{K}")
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    big = torch.full((M, N + pad), float("nan"), dtype=tdt, device="cuda")
    y = big[:, :N]
    pw = mq.PreparedWeight(u8_dev(w), u8_dev(oracle.swizzle_scales(sw, K)),
                           torch.ones(K, dtype=torch.float32, device="cuda"), N, K)
    mq.gemm_mxfp4(u8_dev(a), u8_dev(oracle.swizzle_scales(sa, K)), M, pw, y=y)
    torch.cuda.synchronize()
    if pad:
        assert torch.isnan(big[:, N:]).all().item(), "padding columns were written"
    if dt == "bf16":
        assert_bf16_matches_f32(y, torch.from_numpy(y32).cuda(), f"bf16 {M}x{N}x{K} pad {pad}")
    else:
        # the same call again: bit for bit (a shared tile's partials are added in a fixed
        # order, whichever contributor arrives last)
        assert np.array_equal(host(y).view(np.uint32), y32.view(np.uint32)), f"f32 {M}x{N}x{K} pad {pad}"


@pytest.mark.parametrize("M,N,K", [(1, 25600, 5120), (32, 19200, 1024), (24, 25600, 512), (16, 20000, 4096),
                                   (5, 19000, 5376)])
def test_stream_k_workspace_reuse(mq, M, N, K):
    """Decode shapes on the stream-K schedule (each tile of the last, partial round of
    output tiles split in two K halves taken by two CTAs; a shared tile is finished by the
    later of the two from the partial tiles in the workspace), odd K-tile counts
    included: two calls with different activations share one workspace that starts
    filled with 0xFF bytes; both must match the oracle."""
    import torch
    rng = np.random.default_rng(M + N + K)
    need = mq.gemm_workspace_bytes(M, N, K, torch.float32)
    assert need > 0, "shape expected to run on the stream-K schedule"
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")
    w, sw = random_mxfp4(rng, N, K)
    pw = mq.PreparedWeight(u8_dev(w), u8_dev(oracle.swizzle_scales(sw, K)),
                           torch.ones(K, dtype=torch.float32, device="cuda"), N, K)
    for call in range(2):
        a, sa = random_mxfp4(rng, M, K)
        y = mq.gemm_mxfp4(u8_dev(a), u8_dev(oracle.swizzle_scales(sa, K)), M, pw,
                          out_dtype=torch.float32, workspace=ws)
        torch.cuda.synchronize()
        rows = np.arange(M) if M <= 64 else np.unique(np.concatenate([rng.choice(M, 40, replace=False), [0, M - 1]]))
        assert_gemm_close(host(y)[rows], oracle.gemm_fp64(a, sa, w, sw, K, rows=rows), f"stream-K call {call}")
    assert mq.device_error() == 0
