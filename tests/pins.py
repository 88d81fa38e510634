"""Pins of the CPU oracle to things other than itself.

Each pin checks one oracle function against a closed form, a library routine
(scipy's Hadamard matrix, numpy's matmul and ldexp, IEEE division), brute force, or a
value the pages print. The oracle tests run every pin; the mutation tests compile
broken copies of the oracle and require that some pin fails for each.
"""
import math
import os
from fractions import Fraction

import numpy as np
import scipy.linalg

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

H32 = scipy.linalg.hadamard(32).astype(np.int64)          # Sylvester order, library routine
C32 = np.float32(1.0 / math.sqrt(32.0))                    # nearest fp32 to 2^-2.5


def golden_e2m1():
    vals = {}
    with open(os.path.join(GOLDEN, "e2m1_values.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                c, v = line.split()
                vals[int(c)] = float(v)
    return vals


def golden_storage_bits():
    with open(os.path.join(GOLDEN, "storage_bits.txt")) as f:
        return float([ln for ln in f if ln.strip() and not ln.startswith("#")][0])


# ----------------------------------------------------------- brute force -----

def bf_e2m1_encode(q: np.float32) -> int:
    """Nearest E2M1 magnitude by exhaustive search, ties to the even mantissa bit
    (the code whose lowest bit is 0); the sign bit copies the sign of q."""
    table = golden_e2m1()
    mags = [Fraction(table[c]) for c in range(8)]
    a = abs(Fraction(float(q)))                      # exact rational distances
    best = None
    for idx, m in enumerate(mags):
        d = abs(m - a)
        key = (d, idx & 1)           # distance first, then prefer even mantissa
        if best is None or key < best[0]:
            best = (key, idx)
    sign = 8 if math.copysign(1.0, float(q)) < 0 else 0
    return sign | best[1]


def bf_e8m0(amax: float) -> int:
    """e = clamp(floor(log2 amax) - 2, -127, 127) from math.frexp (exact)."""
    if amax == 0.0:
        return -127
    _, ex = math.frexp(amax)      # amax = m * 2^ex, m in [0.5, 1)
    return max(min(ex - 1 - 2, 127), -127)


def blockdiag_H(K):
    Hb = np.zeros((K, K), np.float64)
    for b in range(K // 32):
        Hb[32 * b:32 * b + 32, 32 * b:32 * b + 32] = H32
    return Hb


def pack_nibbles(codes_2d):
    lo = codes_2d[:, 0::2].astype(np.uint8)
    hi = codes_2d[:, 1::2].astype(np.uint8)
    return lo | (hi << 4)


# ------------------------------------------------------------------ pins -----

def pin_hadamard_matches_scipy():
    got = np.array([[oracle.hadamard_entry(i, j) for j in range(32)] for i in range(32)])
    assert np.array_equal(got, H32), "H32 entries differ from scipy.linalg.hadamard(32)"


def pin_hadamard_orthogonal():
    H = np.array([[oracle.hadamard_entry(i, j) for j in range(32)] for i in range(32)], np.int64)
    assert np.array_equal(H @ H.T, 32 * np.eye(32, dtype=np.int64))
    assert np.array_equal(H, H.T)


def pin_normalisation_constant():
    assert C32.view(np.uint32) == 0x3E3504F3
    exact = 2.0 ** -2.5
    for nb in (np.nextafter(C32, np.float32(1)), np.nextafter(C32, np.float32(0))):
        assert abs(float(C32) - exact) < abs(float(nb) - exact)


def pin_fwht_integer_exact():
    rng = np.random.default_rng(1)
    for _ in range(200):
        v = rng.integers(-1000, 1001, size=32)
        expect = (np.float32(H32 @ v) * C32).astype(np.float32)
        got = oracle.fwht32(v.astype(np.float32))
        assert np.array_equal(got.view(np.uint32), expect.view(np.uint32)), (v, got, expect)


def pin_fwht_float_bound():
    rng = np.random.default_rng(2)
    u = 2.0 ** -24
    for _ in range(200):
        v = (rng.standard_normal(32) * rng.choice([1e-3, 1.0, 1e3])).astype(np.float32)
        exact = (H32 @ v.astype(np.float64)) / math.sqrt(32.0)
        got = oracle.fwht32(v).astype(np.float64)
        bound = 8 * u * np.abs(v.astype(np.float64)).sum() / math.sqrt(32.0)
        assert np.all(np.abs(got - exact) <= bound), np.abs(got - exact).max() / bound


def pin_identity_exact():
    """x W^T == (x D^-1 H)(H D W^T) / 32 exactly, for small integers and s = 2^k."""
    rng = np.random.default_rng(3)
    M, N, K = 5, 7, 96
    x = rng.integers(-8, 9, size=(M, K)).astype(np.float64)
    W = rng.integers(-8, 9, size=(N, K)).astype(np.float64)
    s = 2.0 ** rng.integers(-3, 4, size=K)
    lhs = x @ W.T
    xa = oracle.transform_rows_f64(x, 1.0 / s, 1.0)
    wa = oracle.transform_rows_f64(W, s, 1.0)
    rhs = (xa @ wa.T) / 32.0
    assert np.array_equal(lhs, rhs)
    # the same transform written with the dense block matrix from scipy
    assert np.array_equal(xa, (x / s) @ blockdiag_H(K))


def pin_identity_random():
    rng = np.random.default_rng(4)
    M, N, K = 6, 9, 128
    x = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K))
    s = np.exp(rng.normal(0, 0.5, K))
    lhs = x @ W.T
    rhs = oracle.transform_rows_f64(x, 1.0 / s, math.sqrt(32)) @ \
        oracle.transform_rows_f64(W, s, math.sqrt(32)).T
    assert np.linalg.norm(lhs - rhs) <= 1e-12 * np.linalg.norm(lhs)


def pin_e2m1_decode():
    table = golden_e2m1()
    for c in range(16):
        got = oracle.e2m1_decode(c)
        assert got == table[c] and math.copysign(1, got) == math.copysign(1, table[c]), c


def _encode_sweep_points():
    table = golden_e2m1()
    mags = sorted(set(abs(table[c]) for c in range(8)))
    ties = [(a + b) / 2 for a, b in zip(mags[:-1], mags[1:])]
    pts = [np.float32(t) for t in ties + mags + [7.0, 8.0, 100.0, 1e30]]
    extra = []
    for p in pts:
        extra += [np.nextafter(p, np.float32(0)), np.nextafter(p, np.float32(np.inf))]
    pts = np.array(pts + extra + [1e-30, 1.4e-45, 0.0], np.float32)
    pts = np.concatenate([pts, -pts, np.linspace(-10, 10, 20001, dtype=np.float32)])
    return pts


def pin_e2m1_encode_bruteforce():
    pts = _encode_sweep_points()
    got = oracle.e2m1_encode(pts)
    for q, g in zip(pts, got):
        assert g == bf_e2m1_encode(q), (float(q), int(g), bf_e2m1_encode(q))


def pin_e8m0_closed_form():
    rng = np.random.default_rng(5)
    vals = [0.0, 1.4e-45, 1e-40, 1.1754942e-38, 1.17549435e-38, 3.4e38]
    for k in range(-149, 128):
        p = np.float32(2.0 ** k)
        vals += [p, np.nextafter(p, np.float32(0)), np.nextafter(p, np.float32(np.inf))]
    vals += list(np.abs(rng.standard_normal(2000)).astype(np.float32) *
                 np.float32(2.0) ** rng.integers(-140, 120, 2000).astype(np.float32))
    a = np.array(vals, np.float32)
    a = a[np.isfinite(a)]
    got = oracle.e8m0_exponent(a)
    for x, g in zip(a, got):
        assert g == bf_e8m0(float(x)), (float(x), int(g), bf_e8m0(float(x)))
        if g > -127:
            r = float(x) * 2.0 ** (-int(g))
            assert 4.0 <= r < 8.0


def _exact_rows(rng, rows, K):
    """Rows whose transform is exact in fp32: small-integer bf16 inputs and
    power-of-two multipliers."""
    xi = rng.integers(-64, 65, size=(rows, K)).astype(np.float32)
    xi[rng.random((rows, K)) < 0.2] = 0.0
    xi[0, :32] = 0.0                                   # an all-zero block
    xi[1, 32:64] = 0.0
    xi[1, 40] = 64.0                                   # a one-hot block
    mult = (2.0 ** rng.integers(-3, 4, size=K)).astype(np.float32)
    xb = (xi.view(np.uint32) >> 16).astype(np.uint16)  # small integers are exact in bf16
    return xi, xb, mult


def pin_quant_rows_exact_inputs():
    rng = np.random.default_rng(6)
    rows, K = 9, 192
    xi, xb, mult = _exact_rows(rng, rows, K)
    codes, scales = oracle.quant_rows(xb, mult)
    u = xi.astype(np.float64) * mult                   # exact
    for r in range(rows):
        exp_codes = np.zeros(K, np.uint8)
        for b in range(K // 32):
            t = H32 @ u[r, 32 * b:32 * b + 32]          # exact integer-ish sums
            v = (np.float32(t) * C32).astype(np.float32)
            e = bf_e8m0(float(np.abs(v).max()))
            assert scales[r, b] == e + 127, (r, b, scales[r, b], e)
            q = (v.astype(np.float64) * 2.0 ** (-e)).astype(np.float32)
            exp_codes[32 * b:32 * b + 32] = [bf_e2m1_encode(qq) for qq in q]
        assert np.array_equal(codes[r], pack_nibbles(exp_codes[None, :])[0]), r


def pin_quant_rows_error_bound():
    rng = np.random.default_rng(7)
    rows, K = 8, 256
    x = rng.standard_t(3, size=(rows, K)).astype(np.float32)
    x[:, 5] *= 40
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)   # truncation is fine for a bound test
    mult = np.exp(rng.normal(0, 0.5, K)).astype(np.float32)
    codes, scales = oracle.quant_rows(xb, mult)
    deq = oracle.dequant_rows(codes, scales, K)
    xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    v = (xf * mult.astype(np.float64)) @ blockdiag_H(K) / math.sqrt(32)
    for r in range(rows):
        for b in range(K // 32):
            vb = v[r, 32 * b:32 * b + 32]
            db = deq[r, 32 * b:32 * b + 32]
            e = int(scales[r, b]) - 127
            amax = np.abs(vb).max()
            rel = 1e-5                                  # fp32 transform error vs fp64
            if abs(math.log2(amax) - round(math.log2(amax))) > 1e-5:
                assert e == math.floor(math.log2(amax)) - 2, (r, b)
            step = 2.0 ** e
            for vv, dd in zip(vb, db):
                a = abs(vv) / step
                half = 0.25 if a < 2 else (0.5 if a < 4 else 1.0)
                lim = max(half, a - 6.0) * step + rel * amax
                assert abs(dd - vv) <= lim, (r, b, vv, dd, lim)


def pin_prepare_weight():
    rng = np.random.default_rng(8)
    N, K = 11, 128
    _, Wb, _ = _exact_rows(rng, N, K)
    s = np.exp(rng.normal(0, 0.5, K)).astype(np.float32)
    codes, scales, inv_s = oracle.prepare_weight(Wb, s)
    assert np.array_equal(inv_s.view(np.uint32), (np.float32(1.0) / s).view(np.uint32))
    c2, s2 = oracle.quant_rows(Wb, s)
    assert np.array_equal(codes, c2) and np.array_equal(scales, s2)


def pin_scale_layout():
    K = 32 * 13                                     # 13 blocks -> padded to 16
    assert oracle.scale_blocks_padded(K) == 16 and oracle.scale_rows_padded(130) == 256
    assert oracle.scale_rows_padded(128) == 128 and oracle.scale_blocks_padded(256) == 8
    # hand-derived offsets of the 128 x 4 atom: row r%32 -> 16 B, (r/32)%4 -> 4 B, j%4 -> 1 B
    cases = {(0, 0): 0, (1, 0): 16, (31, 0): 496, (32, 0): 4, (96, 0): 12, (0, 1): 1,
             (0, 3): 3, (0, 4): 512, (33, 5): 512 + 16 + 4 + 1, (128, 0): 4 * 512,
             (200, 9): (1 * 4 + 2) * 512 + (200 % 32) * 16 + 2 * 4 + 1}
    for (r, j), off in cases.items():
        assert oracle.scale_offset(r, j, K) == off, (r, j)
    rows = 130
    rng = np.random.default_rng(9)
    rm = rng.integers(1, 255, size=(rows, K // 32)).astype(np.uint8)
    atom = oracle.swizzle_scales(rm, K)
    assert atom.size == 256 * 16
    assert np.array_equal(oracle.unswizzle_scales(atom, rows, K), rm)
    assert int((atom != 0).sum()) == rm.size         # every padding byte is zero


def pin_dequant():
    table = golden_e2m1()
    rng = np.random.default_rng(10)
    rows, K = 3, 64
    codes = rng.integers(0, 256, size=(rows, K // 2)).astype(np.uint8)
    scales = rng.integers(100, 150, size=(rows, K // 32)).astype(np.uint8)
    got = oracle.dequant_rows(codes, scales, K)
    nib = np.empty((rows, K), np.int64)
    nib[:, 0::2] = codes & 0xF
    nib[:, 1::2] = codes >> 4
    dec = np.vectorize(lambda c: table[int(c)])(nib)
    expect = np.ldexp(dec, np.repeat(scales.astype(np.int64) - 127, 32, axis=1))
    assert np.array_equal(got, expect)


def pin_gemm():
    rng = np.random.default_rng(11)
    M, N, K = 6, 10, 128
    ac = rng.integers(0, 256, size=(M, K // 2)).astype(np.uint8)
    as_ = rng.integers(117, 137, size=(M, K // 32)).astype(np.uint8)
    wc = rng.integers(0, 256, size=(N, K // 2)).astype(np.uint8)
    ws = rng.integers(117, 137, size=(N, K // 32)).astype(np.uint8)
    y = oracle.gemm_fp64(ac, as_, wc, ws, K)
    ref = oracle.dequant_rows(ac, as_, K) @ oracle.dequant_rows(wc, ws, K).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-300)
    rows = np.array([4, 0, 5], np.int64)
    assert np.array_equal(oracle.gemm_fp64(ac, as_, wc, ws, K, rows=rows), y[rows])
    # one-hot: a single code 1.5 (0x3) at k=37 in row 2 against weight code 3.0 (0x5)
    a1 = np.zeros_like(ac)
    a1[2, 37 // 2] = 0x3 << 4                           # odd k -> high nibble
    w1 = np.zeros_like(wc)
    w1[7, 37 // 2] = 0x5 << 4
    sa = np.full_like(as_, 127)
    sa[2, 1] = 127 + 2
    sw = np.full_like(ws, 127)
    sw[7, 1] = 127 - 3
    y1 = oracle.gemm_fp64(a1, sa, w1, sw, K)
    expect = np.zeros((M, N))
    expect[2, 7] = 1.5 * 4 * 3.0 * 0.125
    assert np.array_equal(y1, expect)


def pin_storage():
    K = 4096
    bits = (K // 2 + K // 32) * 8 / K
    assert bits == golden_storage_bits()


# ------------------------------------------------ Hessian exponent search -----

def _np_block_codes(v, e):
    """Codes of v * 2^-e by the brute-force encoder, and their values dec * 2^e."""
    q = (v.astype(np.float64) * 2.0 ** (-e)).astype(np.float32)
    codes = np.array([bf_e2m1_encode(qq) for qq in q], np.uint8)
    table = golden_e2m1()
    vals = np.array([(-1.0 if c & 8 else 1.0) * table[c & 7] for c in codes]) * 2.0 ** e
    return codes, vals


def _np_search(v, H):
    """Independent restatement of the search: errors in fp64 by numpy, candidates in the
    order e0, e0 + 1, e0 - 1, a later one kept only when strictly better."""
    e0 = bf_e8m0(float(np.abs(v).max()))
    best = None
    for e in (e0, e0 + 1, e0 - 1):
        if not -127 <= e <= 127:
            continue
        codes, vals = _np_block_codes(v, e)
        d = v.astype(np.float64) - vals
        err = float(d @ H @ d)
        if best is None or err < best[0] * (1 - 1e-12) - 1e-300:
            best = (err, e, codes)
    return best


def _random_psd(rng, n=32):
    A = rng.standard_normal((n, 2 * n))
    return A @ A.T / (2 * n)


def pin_transform_block():
    rng = np.random.default_rng(20)
    xi, xb, mult = _exact_rows(rng, 3, 96)
    for r in range(3):
        for b in range(3):
            t = H32 @ (xi[r, 32 * b:32 * b + 32].astype(np.float64) * mult[32 * b:32 * b + 32])   # exact
            v = (np.float32(t) * C32).astype(np.float32)
            assert np.array_equal(oracle.transform_block(xb[r], mult, b), v), (r, b)


def pin_hessian_blocks():
    rng = np.random.default_rng(21)
    T, K = 12, 128
    x = rng.standard_t(3, size=(T, K)).astype(np.float32)
    x[:, 9] *= 30
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    inv_s = (np.float32(1.0) / np.exp(rng.normal(0, 0.5, K)).astype(np.float32)).astype(np.float32)
    H = oracle.hessian_blocks(xb, inv_s)
    for b in range(K // 32):
        V = np.stack([oracle.transform_block(xb[t], inv_s, b) for t in range(T)]).astype(np.float64)
        ref = V.T @ V                                  # library matmul
        assert np.allclose(H[b], ref, rtol=1e-13, atol=1e-300), b
        assert np.array_equal(H[b], H[b].T), b          # same products both ways
    # small integers: every sum is exact
    xi, xb2, mult = _exact_rows(rng, 5, 64)
    H2 = oracle.hessian_blocks(xb2, mult)
    for b in range(2):
        V = np.stack([oracle.transform_block(xb2[t], mult, b) for t in range(5)]).astype(np.float64)
        assert np.array_equal(H2[b], V.T @ V), b


def pin_block_error():
    rng = np.random.default_rng(22)
    d = rng.integers(-9, 10, 32).astype(np.float64)
    A = rng.integers(-5, 6, (32, 32))
    H = (A + A.T).astype(np.float64)
    assert oracle.block_error(d, H) == float(d @ H @ d)            # integers: exact
    d = rng.standard_normal(32)
    H = _random_psd(rng)
    assert math.isclose(oracle.block_error(d, H), float(d @ H @ d), rel_tol=1e-12)


def pin_block_error_at():
    rng = np.random.default_rng(23)
    for trial in range(20):
        v = (rng.standard_t(3, 32) * 2.0 ** rng.integers(-6, 7)).astype(np.float32)
        H = _random_psd(rng)
        e0 = bf_e8m0(float(np.abs(v).max()))
        for e in (e0 - 1, e0, e0 + 1):
            err, codes = oracle.block_error_at(v, e, H)
            ref_codes, vals = _np_block_codes(v, e)
            assert np.array_equal(codes, pack_nibbles(ref_codes[None, :])[0]), (trial, e)
            d = v.astype(np.float64) - vals
            assert math.isclose(err, float(d @ H @ d), rel_tol=1e-11, abs_tol=1e-300), (trial, e)


def pin_search_block():
    rng = np.random.default_rng(24)
    picked = {0: 0, 1: 0, -1: 0}
    for trial in range(300):
        v = (rng.standard_t(3, 32) * 2.0 ** rng.integers(-8, 8)).astype(np.float32)
        if trial % 3 == 0:
            v[rng.integers(32)] *= 12                  # an outlier
        H = np.eye(32) if trial % 2 == 0 else _random_psd(rng)
        codes, scale = oracle.search_block(v, H)
        e0 = bf_e8m0(float(np.abs(v).max()))
        err_ref, e_ref, codes_ref = _np_search(v, H)
        assert scale == e_ref + 127, (trial, scale - 127, e_ref)
        assert np.array_equal(codes, pack_nibbles(codes_ref[None, :])[0]), trial
        err_e0 = _np_search(v, np.zeros((32, 32)))[0]
        picked[e_ref - e0] += 1
        # never worse than the floor rule under the same H
        _, vals0 = _np_block_codes(v, e0)
        d0 = v.astype(np.float64) - vals0
        assert err_ref <= float(d0 @ H @ d0) * (1 + 1e-12), trial
        assert err_e0 == 0.0
    assert picked[0] > 0 and picked[1] > 0, picked
    # H = 0: every candidate ties, the floor rule stays
    v = (rng.standard_normal(32) * 5).astype(np.float32)
    codes, scale = oracle.search_block(v, np.zeros((32, 32)))
    assert scale == bf_e8m0(float(np.abs(v).max())) + 127
    # planted: an outlier whose coordinate H ignores makes e0 - 1 the best choice (it
    # clips the outlier at no cost and halves the step for the rest)
    v = np.full(32, 0.37, np.float32) * np.where(np.arange(32) % 2 == 0, 1, -1).astype(np.float32)
    v[0] = np.float32(7.9)
    Hd = np.eye(32)
    Hd[0, 0] = 0.0
    codes, scale = oracle.search_block(v, Hd)
    assert scale - 127 == bf_e8m0(7.9) - 1, scale - 127
    # planted: values just under 8 * 2^e0 saturate to 6 at e0; e0 + 1 is better under H = I
    v = np.full(32, 7.75, np.float32)
    codes, scale = oracle.search_block(v, np.eye(32))
    assert scale - 127 == bf_e8m0(7.75) + 1, scale - 127


def pin_prepare_weight_hessian():
    rng = np.random.default_rng(25)
    N, K = 7, 96
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    Wb = (W.view(np.uint32) >> 16).astype(np.uint16)
    s = np.exp(rng.normal(0, 0.5, K)).astype(np.float32)
    # H = 0: the floor rule everywhere, i.e. plain prepare_weight
    c0, s0, inv0 = oracle.prepare_weight_hessian(Wb, s, np.zeros((K // 32, 32, 32)))
    c1, s1, inv1 = oracle.prepare_weight(Wb, s)
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1) and np.array_equal(inv0, inv1)
    # general H: every block is the numpy search of its transformed block
    H = np.stack([_random_psd(rng) for _ in range(K // 32)])
    c2, s2, _ = oracle.prepare_weight_hessian(Wb, s, H)
    for n in range(N):
        for b in range(K // 32):
            v = oracle.transform_block(Wb[n], s, b)
            _, e, codes = _np_search(v, H[b])
            assert s2[n, b] == e + 127, (n, b)
            assert np.array_equal(c2[n, 16 * b:16 * b + 16], pack_nibbles(codes[None, :])[0]), (n, b)


# ------------------------------------------------------------ Flip-Refinement ---

FLIP_GRID = np.array([-6, -4, -3, -2, -1.5, -1, -0.5, 0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _decode_row(codes_row, scales_row, K):
    """Dequantised row from the golden E2M1 table and the E8M0 bytes."""
    table = golden_e2m1()
    nib = np.empty(K, np.uint8)
    nib[0::2] = codes_row & 0xF
    nib[1::2] = codes_row >> 4
    vals = np.array([(-1.0 if c & 8 else 1.0) * table[c & 7] for c in nib])
    return vals * 2.0 ** (np.repeat(scales_row.astype(np.int64), 32) - 127)


def _local_gains(wv, H, codes_row, scales_row):
    """Every adjacent move's change of e^T H e, by numpy (grid positions from values)."""
    K = wv.size
    what = _decode_row(codes_row, scales_row, K)
    step = 2.0 ** (np.repeat(scales_row.astype(np.int64), 32) - 127)
    e = wv.astype(np.float64) - what
    g = H @ e
    gains = []
    for k in range(K):
        pos = int(np.argmin(np.abs(FLIP_GRID - what[k] / step[k])))
        for d in (-1, 1):
            if 0 <= pos + d <= 14:
                delta = (FLIP_GRID[pos + d] - FLIP_GRID[pos]) * step[k]
                gains.append(delta * delta * H[k, k] - 2 * delta * g[k])
    return np.array(gains), float(e @ H @ e)


def pin_hessian_full():
    rng = np.random.default_rng(30)
    T, K = 9, 96
    x = rng.standard_t(3, size=(T, K)).astype(np.float32)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    inv_s = np.exp(rng.normal(0, 0.5, K)).astype(np.float32)
    H = oracle.hessian_full(xb, inv_s)
    V = np.concatenate([np.stack([oracle.transform_block(xb[t], inv_s, b) for b in range(K // 32)]).reshape(-1)[None]
                        for t in range(T)]).astype(np.float64)
    assert np.allclose(H, V.T @ V, rtol=1e-13, atol=1e-300)
    assert np.array_equal(H, H.T)
    Hb = oracle.hessian_blocks(xb, inv_s)
    for b in range(K // 32):                          # same products, same order
        assert np.array_equal(H[32 * b:32 * b + 32, 32 * b:32 * b + 32], Hb[b]), b
    _, xb2, mult = _exact_rows(rng, 4, 64)
    H2 = oracle.hessian_full(xb2, mult)
    V2 = np.concatenate([np.stack([oracle.transform_block(xb2[t], mult, b) for b in range(2)]).reshape(-1)[None]
                         for t in range(4)]).astype(np.float64)
    assert np.array_equal(H2, V2.T @ V2)


def pin_flip_refine_special_cases():
    rng = np.random.default_rng(31)
    N, K = 5, 64
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    Wb = (W.view(np.uint32) >> 16).astype(np.uint16)
    s = np.exp(rng.normal(0, 0.5, K)).astype(np.float32)
    c, sc, _ = oracle.prepare_weight(Wb, s)
    # diagonal H: coordinates are independent and round-to-nearest is already optimal
    Hd = np.diag(rng.uniform(0.1, 3.0, K))
    c1, m1 = oracle.flip_refine(Wb, s, Hd, c, sc, 1000)
    assert (m1 == 0).all() and np.array_equal(c1, c)
    # H = 0: no move lowers the error strictly
    c2, m2 = oracle.flip_refine(Wb, s, np.zeros((K, K)), c, sc, 1000)
    assert (m2 == 0).all() and np.array_equal(c2, c)
    # planted, worked by hand: H = I except H01 = H10 = 0.9, w' = (0.74, 0.70, 0, ...), scale
    # 2^0; round to nearest gives (0.5, 0.5), e = (0.24, 0.20), g = H e = (0.42, 0.416); the
    # best move takes coordinate 0 up to 1.0 (dE = 0.25 - 0.42 = -0.17, against -0.166 for
    # coordinate 1), g becomes (-0.08, -0.034) and no move helps any more
    H = np.eye(32)
    H[0, 1] = H[1, 0] = 0.9
    wv = np.zeros(32, np.float32)
    wv[0], wv[1] = 0.74, 0.70
    codes = np.zeros(16, np.uint8)
    codes[0] = 0x11                                 # codes 1 | 1 << 4: values 0.5, 0.5
    out, n = oracle.flip_refine_row(wv, H, codes, np.array([127], np.uint8), 100)
    assert n == 1 and out[0] == 0x12 and (out[1:] == 0).all(), (n, out[:2])


def pin_flip_refine_local_optimum():
    rng = np.random.default_rng(32)
    N, K, T = 6, 96, 40
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    Wb = (W.view(np.uint32) >> 16).astype(np.uint16)
    s = np.exp(rng.normal(0, 0.5, K)).astype(np.float32)
    x = rng.standard_t(3, size=(T, K)).astype(np.float32)
    x[:, 7] *= 20
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    H = oracle.hessian_full(xb, (np.float32(1.0) / s).astype(np.float32))
    c, sc, _ = oracle.prepare_weight(Wb, s)
    c2, moves = oracle.flip_refine(Wb, s, H, c, sc, 10000)
    assert moves.sum() > 0
    for n in range(N):
        wv = np.concatenate([oracle.transform_block(Wb[n], s, b) for b in range(K // 32)])
        g0, e0 = _local_gains(wv, H, c[n], sc[n])
        g1, e1 = _local_gains(wv, H, c2[n], sc[n])
        assert e1 <= e0 * (1 + 1e-12), n              # never worse than round to nearest
        assert (g1 >= -1e-9 * max(e0, 1e-300)).all(), (n, g1.min())   # no improving move left
        assert int((c2[n] != c[n]).sum()) <= 2 * moves[n]
    # a cap on the rounds is honoured
    c3, m3 = oracle.flip_refine(Wb, s, H, c, sc, 1)
    assert (m3 <= 1).all() and (m3 == np.minimum(moves, 1)).all()


def pin_flip_refine_brute_force():
    """Three coupled coordinates in one block, the rest zero: every code triple is
    enumerated; the refined triple is no worse than round to nearest, is a local
    optimum, and starting from the global optimum no move is made."""
    rng = np.random.default_rng(33)
    for trial in range(6):
        A = rng.standard_normal((3, 3))
        H = np.eye(32)
        H[:3, :3] = A @ A.T + 0.05 * np.eye(3)
        wv = np.zeros(32, np.float32)
        wv[:3] = rng.uniform(-2.5, 2.5, 3).astype(np.float32)
        sc = np.array([127], np.uint8)
        best = None
        for i in range(15):
            for j in range(15):
                for k in range(15):
                    d = wv[:3].astype(np.float64) - FLIP_GRID[[i, j, k]]
                    E = float(d @ H[:3, :3] @ d)
                    if best is None or E < best[0]:
                        best = (E, (i, j, k))
        def codes_of(idx):
            nib = np.zeros(32, np.uint8)
            for p_, gi in enumerate(idx):
                v = FLIP_GRID[gi]
                m = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}[abs(v)]
                nib[p_] = m | (8 if v < 0 and m else 0)
            return (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)
        rtn = tuple(int(np.argmin(np.abs(FLIP_GRID - float(w)))) for w in wv[:3])
        out, n = oracle.flip_refine_row(wv, H, codes_of(rtn), sc, 1000)
        gains, E = _local_gains(wv, H, out, sc)
        _, E_rtn = _local_gains(wv, H, codes_of(rtn), sc)
        assert best[0] <= E + 1e-12 and E <= E_rtn + 1e-12, trial
        assert (gains >= -1e-12).all(), trial
        out2, n2 = oracle.flip_refine_row(wv, H, codes_of(best[1]), sc, 1000)
        assert n2 == 0 and np.array_equal(out2, codes_of(best[1])), trial


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
