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


def tile_covering_rows(M, n_rows=256, seed=0):
    """Seeded output rows for a GEMM parity check that touch every 128-row M tile and, in
    each, every 32-row group of the scale atom (rows r with (r // 32) % 4 = 0..3): the
    same number of random rows from each 32-row group (at least one, enough for
    n_rows in all), plus rows 0 and M - 1, topped up to min(M, n_rows) rows when short
    groups hold fewer. Sorted, unique."""
    rng = np.random.default_rng(seed)
    groups = [(g0, min(g0 + 32, M)) for g0 in range(0, M, 32)]
    per = max(1, -(-n_rows // len(groups)))
    rows = [0, M - 1]
    for g0, g1 in groups:
        k = min(per, g1 - g0)
        rows.extend((g0 + rng.choice(g1 - g0, k, replace=False)).tolist())
    rows = np.unique(np.asarray(rows, dtype=np.int64))
    short = min(M, n_rows) - rows.size
    if short > 0:          # short groups at the end: top up from the rows not taken
        rest = np.setdiff1d(np.arange(M, dtype=np.int64), rows)
        rows = np.unique(np.concatenate([rows, rng.choice(rest, short, replace=False)]))
    return rows


class oracle_on_all_cores:
    """Run the oracle's OpenMP build (bit-identical to the serial one, checked by
    test_oracle_openmp) inside the block, to keep large parity references to seconds."""

    def __enter__(self):
        oracle.set_openmp(True)
        return self

    def __exit__(self, *exc):
        oracle.set_openmp(False)
        return False
