"""The C-ABI library loads, exports every entry point include/macaq.h declares, and
its host-side logic (sizes, status names, argument validation) behaves as documented.
No compute call reaches a device here."""
import ctypes
import os
import re

import pytest

import mxfp4_w4a4_post_b200 as mq
from mxfp4_w4a4_post_b200 import build as mq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "macaq.h")


@pytest.fixture(scope="module")
def L():
    mq_build.build()
    return mq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(macaq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["macaq_prepare_weight", "macaq_quant_act", "macaq_linear_w4a4", "macaq_gemm_mxfp4",
                     "macaq_codes_bytes", "macaq_scales_bytes", "macaq_get_device_error",
                     "macaq_status_string"]:
        assert required in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_sizes(L):
    assert L.macaq_codes_bytes(16, 256) == 16 * 128
    assert L.macaq_scales_bytes(16, 256) == 128 * 8          # rows -> 128, 8 blocks
    assert L.macaq_scales_bytes(130, 32 * 13) == 256 * 16    # 13 blocks -> 16
    assert L.macaq_scales_bytes(4096, 4096) == 4096 * 128
    assert L.macaq_codes_bytes(-1, 32) == 0


def test_storage_is_4_25_bits(L):
    K, rows = 4096, 4096
    bits = 8.0 * (L.macaq_codes_bytes(rows, K) + L.macaq_scales_bytes(rows, K)) / (rows * K)
    assert bits == 4.25


def test_status_strings(L):
    for code, name in mq.STATUS_NAMES.items():
        assert L.macaq_status_string(code).decode() == name
    assert L.macaq_version() == 1


def test_validation_rejects_bad_arguments(L):
    a = ctypes.c_void_p(0x1000)       # aligned, never dereferenced: validation fails first
    mis = ctypes.c_void_p(0x1004)
    null = None
    # null pointers
    assert L.macaq_quant_act(null, 4, 64, 64, a, a, a, None) == 1
    assert L.macaq_prepare_weight(a, 4, 64, 64, a, a, a, null, None) == 1
    # K not a multiple of 32
    assert L.macaq_quant_act(a, 4, 48, 48, a, a, a, None) == 3
    # ldx < K, rows < 1
    assert L.macaq_quant_act(a, 4, 64, 32, a, a, a, None) == 1
    assert L.macaq_quant_act(a, 0, 64, 64, a, a, a, None) == 1
    # misaligned pointers / leading dimension
    assert L.macaq_quant_act(mis, 4, 64, 64, a, a, a, None) == 2
    assert L.macaq_quant_act(a, 4, 64, 68, a, a, a, None) == 2
    w = mq.MacaqWeight(0x1000, 0x1000, 0x1000, 128, 256)
    assert L.macaq_gemm_mxfp4(a, a, 4, ctypes.byref(w), a, 64, 0, null, 0, None) == 1   # ldy < N
    assert L.macaq_gemm_mxfp4(a, a, 4, ctypes.byref(w), a, 128, 7, null, 0, None) == 1  # bad dtype
    assert L.macaq_gemm_mxfp4(a, a, 4, ctypes.byref(w), ctypes.c_void_p(0x1002), 128, 0, null, 0, None) == 2
    assert L.macaq_gemm_mxfp4(a, a, 4, ctypes.byref(w), ctypes.c_void_p(0x1001), 128, 1, null, 0, None) == 2
    assert L.macaq_gemm_mxfp4(mis, a, 4, ctypes.byref(w), a, 128, 0, null, 0, None) == 2   # codes
    bad = mq.MacaqWeight(0x1000, 0x1000, 0x1000, 128, 250)
    assert L.macaq_gemm_mxfp4(a, a, 4, ctypes.byref(bad), a, 128, 0, null, 0, None) == 3
    assert L.macaq_linear_w4a4(a, 4, 256, ctypes.byref(w), a, 128, 0, 3, a, 1 << 20, None) == 1  # fused not 0..2
    assert L.macaq_linear_w4a4(a, 4, 256, ctypes.byref(w), a, 128, 0, -1, a, 1 << 20, None) == 1
    # wait self-test: limit outside [1 us, 1 s] or no result array
    res = (ctypes.c_int64 * 10)()
    assert L.macaq_selftest_wait_timeout(0, res, None) == 1
    assert L.macaq_selftest_wait_timeout(1000001, res, None) == 1
    assert L.macaq_selftest_wait_timeout(100, None, None) == 1
    # gathered output: no destinations, too many, a misaligned one
    d_ok = (ctypes.c_uint64 * 2)(0x2000, 0x3000)
    d_mis = (ctypes.c_uint64 * 1)(0x2002)
    d_many = (ctypes.c_uint64 * 65)(*([0x2000] * 65))
    assert L.macaq_linear_w4a4_gather(a, 4, 256, ctypes.byref(w), None, 1, 128, 0, a, 1 << 20, None) == 1
    assert L.macaq_linear_w4a4_gather(a, 4, 256, ctypes.byref(w), d_ok, 0, 128, 0, a, 1 << 20, None) == 1
    assert L.macaq_linear_w4a4_gather(a, 4, 256, ctypes.byref(w), d_many, 65, 128, 0, a, 1 << 20, None) == 1
    assert L.macaq_linear_w4a4_gather(a, 4, 256, ctypes.byref(w), d_mis, 1, 128, 0, a, 1 << 20, None) == 2
    assert L.macaq_linear_w4a4_gather(a, 4, 256, ctypes.byref(w), d_ok, 2, 64, 0, a, 1 << 20, None) == 1  # ldy < N
    assert L.macaq_linear_gather_workspace_bytes(4, 128, 256, 0) == L.macaq_linear_workspace_bytes(4, 128, 256, 0)


def test_multi_linear_validation(L):
    """The shared-input layer checks its arguments before anything is launched."""
    a = ctypes.c_void_p(0x1000)
    ok = mq.MacaqWeight(0x1000, 0x1000, 0x1000, 128, 256)
    ws2 = (mq.MacaqWeight * 2)(ok, mq.MacaqWeight(0x1000, 0x1000, 0x1000, 64, 256))
    ys = (ctypes.c_void_p * 2)(0x2000, 0x3000)
    lds = (ctypes.c_int64 * 2)(128, 64)
    assert L.macaq_multi_linear_workspace_bytes(4, 256, 2) == L.macaq_multi_linear_workspace_bytes(100, 256, 2)
    assert L.macaq_multi_linear_workspace_bytes(0, 256, 2) == 0
    assert L.macaq_multi_linear_w4a4(None, 4, 256, ws2, 2, ys, lds, 0, a, 1 << 24, None) == 1
    assert L.macaq_multi_linear_w4a4(a, 4, 256, ws2, 0, ys, lds, 0, a, 1 << 24, None) == 1
    other_k = (mq.MacaqWeight * 2)(ok, mq.MacaqWeight(0x1000, 0x1000, 0x1000, 64, 512))
    assert L.macaq_multi_linear_w4a4(a, 4, 256, other_k, 2, ys, lds, 0, a, 1 << 24, None) == 1
    bad_inv = (mq.MacaqWeight * 2)(ok, mq.MacaqWeight(0x1000, 0x1000, 0x1004, 64, 256))
    assert L.macaq_multi_linear_w4a4(a, 4, 256, bad_inv, 2, ys, lds, 0, a, 1 << 24, None) == 2
    short_ld = (ctypes.c_int64 * 2)(128, 32)
    assert L.macaq_multi_linear_w4a4(a, 4, 256, ws2, 2, ys, short_ld, 0, a, 1 << 24, None) == 1
    assert L.macaq_multi_linear_w4a4(a, 4, 256, ws2, 2, ys, lds, 0, a, 1024, None) == 7


def test_no_usable_device_is_a_status_not_a_crash(L):
    """Valid arguments on a machine without a usable CUDA device (the nearest this host
    comes to a wrong architecture): every launching entry point returns MACAQ_ERR_CUDA
    after validation, and nothing aborts."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    a = ctypes.c_void_p(0x1000)
    w = mq.MacaqWeight(0x1000, 0x1000, 0x1000, 128, 256)
    d = (ctypes.c_uint64 * 1)(0x2000)
    res = (ctypes.c_int64 * 10)()
    assert L.macaq_quant_act(a, 4, 64, 64, a, a, a, None) == 5
    assert L.macaq_prepare_weight(a, 4, 64, 64, a, a, a, a, None) == 5
    assert L.macaq_gemm_mxfp4(a, a, 4, ctypes.byref(w), a, 128, 0, None, 0, None) == 5
    assert L.macaq_linear_w4a4(a, 4, 256, ctypes.byref(w), a, 128, 0, 0, a, 1 << 24, None) == 5
    assert L.macaq_linear_w4a4_gather(a, 4, 256, ctypes.byref(w), d, 1, 128, 0, a, 1 << 24, None) == 5
    ws2 = (mq.MacaqWeight * 2)(mq.MacaqWeight(0x1000, 0x1000, 0x1000, 128, 256),
                               mq.MacaqWeight(0x1000, 0x1000, 0x1000, 64, 256))
    ys = (ctypes.c_void_p * 2)(0x2000, 0x3000)
    lds = (ctypes.c_int64 * 2)(128, 64)
    assert L.macaq_multi_linear_w4a4(a, 4, 256, ws2, 2, ys, lds, 0, a, 1 << 24, None) == 5
    offs = (ctypes.c_int64 * 3)(0, 3, 4)
    assert L.macaq_grouped_linear_w4a4(a, 256, offs, 2, (mq.MacaqWeight * 2)(w, w), a, 128, 0, a, 1 << 24, None) == 5
    assert L.macaq_selftest_wait_timeout(100, res, None) == 5
    assert L.macaq_get_device_error() == 5
