"""The no-allocation variant of the W4A4 layer, for callers that cannot allocate device
memory (a runtime that owns the whole memory pool, or a latency-critical loop where an
allocation would stall the device). It must give the same output as the workspace
entry point, call after call, although every call reuses one static scratch array.

Collected last on purpose, and independent of every other test module."""
import ctypes

import numpy as np
import pytest

import oracle
from helpers import assert_gemm_close, bf16_dev, f32_dev, host
from mxfp4_w4a4_post_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MACAQ_ERR_WORKSPACE = 7
NOALLOC_SCRATCH_BYTES = 16 << 20


@pytest.fixture(scope="module")
def mq():
    import mxfp4_w4a4_post_b200 as m
    from mxfp4_w4a4_post_b200 import build
    build.build()
    L = m.lib()
    f = L.macaq_linear_w4a4_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.POINTER(m.MacaqWeight),
                  ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p]
    return m


def noalloc_linear(mq, x, pw, out_dtype):
    import torch
    M = x.shape[0]
    y = torch.empty((M, pw.N), dtype=out_dtype, device=x.device)
    cw = pw.c_struct()
    st = mq.lib().macaq_linear_w4a4_noalloc(
        x.data_ptr(), M, x.stride(0), ctypes.byref(cw), y.data_ptr(), y.stride(0),
        mq.OUT_F32 if out_dtype == torch.float32 else mq.OUT_BF16,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, y


@pytest.mark.parametrize("M,N,K", [(16, 512, 16384), (300, 1000, 1024)])
def test_noalloc_matches_workspace_entry_point(mq, M, N, K):
    """Two calls in a row with different activations (the second call must not see the
    first call's stream-K partial tiles or counts), each against macaq_linear_w4a4."""
    import torch
    base = wl.with_shape(wl.tiny_layer(), M=M, N=N, K=K)
    assert mq.linear_workspace_bytes(M, N, K, torch.float32) <= NOALLOC_SCRATCH_BYTES
    W, s = wl.draw_W(base), wl.draw_s(base)
    pw = mq.prepare_weight(bf16_dev(W), f32_dev(s))
    for seed in (11, 12):
        x = bf16_dev(wl.draw_x(wl.with_shape(base, seed=seed)))
        st, y_na = noalloc_linear(mq, x, pw, torch.float32)
        assert st == 0, mq.STATUS_NAMES.get(st, st)
        y_ws = mq.linear(x, pw, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert_gemm_close(host(y_na), host(y_ws).astype(np.float64), f"noalloc vs linear, seed {seed}")
    assert mq.device_error() == 0


def test_noalloc_against_the_oracle(mq):
    import torch
    L = wl.tiny_layer()
    x, W, s = wl.draw_x(L), wl.draw_W(L), wl.draw_s(L)
    pw = mq.prepare_weight(bf16_dev(W), f32_dev(s))
    st, y = noalloc_linear(mq, bf16_dev(x), pw, torch.float32)
    assert st == 0
    torch.cuda.synchronize()
    rwc, rws, rinv = oracle.prepare_weight(W, s)
    rac, ras = oracle.quant_rows(x, rinv)
    assert_gemm_close(host(y), oracle.gemm_fp64(rac, ras, rwc, rws, L.K), "noalloc tiny layer")


def test_noalloc_rejects_sizes_beyond_the_scratch(mq):
    import torch
    M, N, K = 8192, 256, 4096          # activation codes alone are 16 MiB
    assert mq.linear_workspace_bytes(M, N, K, torch.bfloat16) > NOALLOC_SCRATCH_BYTES
    pw = mq.PreparedWeight(torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda"),
                           torch.zeros(mq.scales_bytes(N, K), dtype=torch.uint8, device="cuda"),
                           torch.ones(K, dtype=torch.float32, device="cuda"), N, K)
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    st, _ = noalloc_linear(mq, x, pw, torch.bfloat16)
    assert st == MACAQ_ERR_WORKSPACE
