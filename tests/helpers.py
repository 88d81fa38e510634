"""Shared helpers of the GPU parity tests: moving the seeded inputs to the device and
comparing the CUDA path with the oracle."""
import math

import numpy as np

import oracle

C32 = np.float32(1.0 / math.sqrt(32.0))


def bf16_dev(u16):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(u16, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def f32_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def u8_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8).reshape(-1)).cuda()


def host(t):
    return t.detach().cpu().numpy()


def assert_codes_equal(gpu_codes, ref_codes, what):
    g = np.asarray(gpu_codes, dtype=np.uint8).reshape(ref_codes.shape)
    if not np.array_equal(g, ref_codes):
        bad = np.argwhere(g != ref_codes)
        r, c = bad[0]
        raise AssertionError(f"{what}: {len(bad)} code bytes differ; first at row {r} byte {c}: "
                             f"gpu {g[r, c]:#04x} oracle {ref_codes[r, c]:#04x}")


def assert_scales_equal(gpu_atoms, ref_rowmajor, K, what):
    """Compare the whole padded atom buffer (padding must be zero) and, for a readable
    message, the row-major view."""
    g = np.asarray(gpu_atoms, dtype=np.uint8).reshape(-1)
    ref_atoms = oracle.swizzle_scales(ref_rowmajor, K)
    if not np.array_equal(g[:ref_atoms.size], ref_atoms):
        rows = ref_rowmajor.shape[0]
        g_rm = oracle.unswizzle_scales(g, rows, K)
        bad = np.argwhere(g_rm != ref_rowmajor)
        if len(bad):
            r, j = bad[0]
            raise AssertionError(f"{what}: {len(bad)} scale bytes differ; first at row {r} block {j}: "
                                 f"gpu {g_rm[r, j]} oracle {ref_rowmajor[r, j]}")
        raise AssertionError(f"{what}: padding bytes of the scale layout are not zero")


def gemm_error(y, ref):
    """(relative Frobenius error, max-abs error / rms(ref))."""
    y = np.asarray(y, dtype=np.float64)
    d = y - ref
    fro = np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300)
    rms = math.sqrt(float(np.mean(ref * ref))) if ref.size else 0.0
    mx = float(np.abs(d).max()) / max(rms, 1e-300) if d.size else 0.0
    return fro, mx


# Tolerance of the W4A4 GEMM against the fp64 sum of decoded products.
REL_FRO_TOL = 1e-3
MAX_ABS_TOL = 1e-2


def assert_gemm_close(y, ref, what):
    fro, mx = gemm_error(y, ref)
    assert fro <= REL_FRO_TOL and mx <= MAX_ABS_TOL, f"{what}: rel_fro={fro:.3e} max_abs/rms={mx:.3e}"
    return fro, mx


def assert_bf16_matches_f32(y_bf16, y_f32, what):
    """bf16 output within one bf16 ulp of the fp32 output of the same product."""
    import torch
    yb = y_bf16.float().cpu().numpy().astype(np.float64)
    yf = y_f32.cpu().numpy().astype(np.float64)
    ulp = np.abs(yf) * 2.0 ** -7 + 1e-38
    bad = np.abs(yb - yf) > ulp
    assert not bad.any(), f"{what}: {int(bad.sum())} bf16 outputs more than 1 ulp from fp32"


def random_mxfp4(rng, rows, K, scale_lo=117, scale_hi=137):
    """Random codes (every nibble value) and row-major scales."""
    codes = rng.integers(0, 256, size=(rows, K // 2)).astype(np.uint8)
    scales = rng.integers(scale_lo, scale_hi + 1, size=(rows, K // 32)).astype(np.uint8)
    return codes, scales
