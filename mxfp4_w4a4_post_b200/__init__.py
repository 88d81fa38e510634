"""MACaQ W4A4 linear layer (MXFP4) on NVIDIA B200: thin Python binding of libmacaq.

Every step of the layer runs in the CUDA kernels behind the C ABI declared in
include/macaq.h; this module only marshals torch tensors (device memory and the
current stream) into those calls. There is no CPU fallback: if the library is missing
or the device is not a B200, calls raise.

    w = prepare_weight(W_bf16, s)          # offline: W' = W diag(s) Hb -> MXFP4
    y = linear(x_bf16, w)                  # online: x diag(s)^-1 Hb -> MXFP4 -> FP4 GEMM
"""
import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmacaq.so")

MACAQ_OK = 0
OUT_F32 = 0
OUT_BF16 = 1

STATUS_NAMES = {
    0: "MACAQ_OK", 1: "MACAQ_ERR_INVALID_ARG", 2: "MACAQ_ERR_MISALIGNED",
    3: "MACAQ_ERR_UNSUPPORTED_SHAPE", 4: "MACAQ_ERR_UNSUPPORTED_DEVICE", 5: "MACAQ_ERR_CUDA",
    6: "MACAQ_ERR_DEVICE_TIMEOUT", 7: "MACAQ_ERR_WORKSPACE", 8: "MACAQ_ERR_UNSUPPORTED",
}


class MacaqError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


class MacaqWeight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("inv_s", ctypes.c_void_p),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64)]


_lib = None


def lib():
    """The loaded libmacaq.so (ctypes), with argument types declared."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmacaq.so not built ({LIB_PATH}); run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, SZ, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
        sig = {
            "macaq_codes_bytes": (SZ, [I64, I64]),
            "macaq_scales_bytes": (SZ, [I64, I64]),
            "macaq_gemm_workspace_bytes": (SZ, [I64, I64, I64, I]),
            "macaq_linear_workspace_bytes": (SZ, [I64, I64, I64, I]),
            "macaq_prepare_weight": (I, [P, I64, I64, I64, P, P, P, P, P]),
            "macaq_quant_act": (I, [P, I64, I64, I64, P, P, P, P]),
            "macaq_gemm_mxfp4": (I, [P, P, I64, ctypes.POINTER(MacaqWeight), P, I64, I, P, SZ, P]),
            "macaq_linear_w4a4": (I, [P, I64, I64, ctypes.POINTER(MacaqWeight), P, I64, I, I, P, SZ, P]),
            "macaq_hessian_bytes": (SZ, [I64]),
            "macaq_hessian_blocks": (I, [P, I64, I64, I64, P, P, P]),
            "macaq_prepare_weight_hessian": (I, [P, I64, I64, I64, P, P, P, P, P, P]),
            "macaq_hessian_full_workspace_bytes": (SZ, [I64, I64]),
            "macaq_hessian_full": (I, [P, I64, I64, I64, P, P, P, SZ, P]),
            "macaq_flip_workspace_bytes": (SZ, [I64, I64]),
            "macaq_flip_refine": (I, [P, I64, I64, I64, P, P, P, P, I, P, P, SZ, P]),
            "macaq_grouped_linear_workspace_bytes": (SZ, [P, I64, I64]),
            "macaq_grouped_linear_w4a4": (I, [P, I64, P, I64, P, P, I64, I, P, SZ, P]),
            "macaq_multi_linear_workspace_bytes": (SZ, [I64, I64, I64]),
            "macaq_multi_linear_w4a4": (I, [P, I64, I64, P, I64, P, P, I, P, SZ, P]),
            "macaq_linear_gather_workspace_bytes": (SZ, [I64, I64, I64, I]),
            "macaq_linear_w4a4_gather": (I, [P, I64, I64, ctypes.POINTER(MacaqWeight), P, I, I64, I, P, SZ, P]),
            "macaq_selftest_wait_timeout": (I, [ctypes.c_uint32, ctypes.POINTER(I64), P]),
            "macaq_get_device_error": (I, []),
            "macaq_status_string": (ctypes.c_char_p, [I]),
            "macaq_version": (I, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status, what):
    if status != MACAQ_OK:
        raise MacaqError(status, what)


def _torch():
    import torch
    return torch


def _stream_ptr(device):
    torch = _torch()
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _out_code(dtype):
    torch = _torch()
    if dtype == torch.float32:
        return OUT_F32
    if dtype == torch.bfloat16:
        return OUT_BF16
    raise ValueError(f"unsupported output dtype {dtype}")


def codes_bytes(rows, K):
    return lib().macaq_codes_bytes(rows, K)


def scales_bytes(rows, K):
    return lib().macaq_scales_bytes(rows, K)


def linear_workspace_bytes(M, N, K, out_dtype=None):
    torch = _torch()
    return lib().macaq_linear_workspace_bytes(M, N, K, _out_code(out_dtype or torch.bfloat16))


def gemm_workspace_bytes(M, N, K, out_dtype=None):
    torch = _torch()
    return lib().macaq_gemm_workspace_bytes(M, N, K, _out_code(out_dtype or torch.bfloat16))


@dataclass
class PreparedWeight:
    """Offline artefact: MXFP4 codes/scales of W' = W diag(s) Hb, and inv_s = 1/s."""
    codes: "object"    # uint8 [N, K/2]
    scales: "object"   # uint8 [scales_bytes(N, K)] (tensor-core atom layout)
    inv_s: "object"    # float32 [K]
    N: int
    K: int

    def c_struct(self):
        return MacaqWeight(self.codes.data_ptr(), self.scales.data_ptr(), self.inv_s.data_ptr(),
                           self.N, self.K)


def _require(t, dtype, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() == 2 and t.stride(1) != 1:
        raise ValueError(f"{name} must have unit stride along its last dimension")


def prepare_weight(W, s, out=None):
    """W: bf16 [N, K] CUDA tensor (row stride W.stride(0)); s: fp32 [K]."""
    torch = _torch()
    _require(W, torch.bfloat16, "W")
    _require(s, torch.float32, "s")
    N, K = W.shape
    dev = W.device
    if out is None:
        out = PreparedWeight(torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                             torch.empty(scales_bytes(N, K), dtype=torch.uint8, device=dev),
                             torch.empty(K, dtype=torch.float32, device=dev), N, K)
    st = lib().macaq_prepare_weight(W.data_ptr(), N, K, W.stride(0), s.data_ptr(), out.codes.data_ptr(),
                                    out.scales.data_ptr(), out.inv_s.data_ptr(), _stream_ptr(dev))
    _check(st, "macaq_prepare_weight")
    return out


def hessian_blocks(x, s, H=None):
    """Calibration activations x: bf16 [T, K]; s: fp32 [K]. Returns the fp64 Gram blocks
    H [K/32, 32, 32] of the transformed rows (the input of prepare_weight_hessian)."""
    torch = _torch()
    _require(x, torch.bfloat16, "x")
    _require(s, torch.float32, "s")
    T, K = x.shape
    if H is None:
        H = torch.empty((K // 32, 32, 32), dtype=torch.float64, device=x.device)
    st = lib().macaq_hessian_blocks(x.data_ptr(), T, K, x.stride(0), s.data_ptr(), H.data_ptr(),
                                    _stream_ptr(x.device))
    _check(st, "macaq_hessian_blocks")
    return H


def prepare_weight_hessian(W, s, H, out=None):
    """prepare_weight with the Hessian exponent search over e0, e0 + 1, e0 - 1 per block."""
    torch = _torch()
    _require(W, torch.bfloat16, "W")
    _require(s, torch.float32, "s")
    N, K = W.shape
    dev = W.device
    if not (isinstance(H, torch.Tensor) and H.is_cuda and H.dtype == torch.float64 and H.is_contiguous()
            and tuple(H.shape) == (K // 32, 32, 32)):
        raise ValueError("H must be a contiguous float64 CUDA tensor [K/32, 32, 32]")
    if out is None:
        out = PreparedWeight(torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                             torch.empty(scales_bytes(N, K), dtype=torch.uint8, device=dev),
                             torch.empty(K, dtype=torch.float32, device=dev), N, K)
    st = lib().macaq_prepare_weight_hessian(W.data_ptr(), N, K, W.stride(0), s.data_ptr(), H.data_ptr(),
                                            out.codes.data_ptr(), out.scales.data_ptr(), out.inv_s.data_ptr(),
                                            _stream_ptr(dev))
    _check(st, "macaq_prepare_weight_hessian")
    return out


def hessian_full(x, s, H=None):
    """Calibration activations x: bf16 [T, K]; s: fp32 [K]. Returns the full fp64 Gram
    matrix H [K, K] of the transformed rows (the input of flip_refine)."""
    torch = _torch()
    _require(x, torch.bfloat16, "x")
    _require(s, torch.float32, "s")
    T, K = x.shape
    if H is None:
        H = torch.empty((K, K), dtype=torch.float64, device=x.device)
    nws = lib().macaq_hessian_full_workspace_bytes(T, K)
    ws = torch.empty(max(nws, 256), dtype=torch.uint8, device=x.device)
    st = lib().macaq_hessian_full(x.data_ptr(), T, K, x.stride(0), s.data_ptr(), H.data_ptr(), ws.data_ptr(),
                                  ws.numel(), _stream_ptr(x.device))
    _check(st, "macaq_hessian_full")
    return H


def flip_refine(W, s, H, w, max_rounds=1 << 20, workspace=None):
    """Flip-Refinement of the prepared weight w's codes, in place. Returns the number of
    moves per row (int32 CUDA tensor [N])."""
    torch = _torch()
    _require(W, torch.bfloat16, "W")
    _require(s, torch.float32, "s")
    N, K = W.shape
    dev = W.device
    moves = torch.empty(N, dtype=torch.int32, device=dev)
    need = lib().macaq_flip_workspace_bytes(N, K)
    ws, ws_bytes = _workspace(need, dev, workspace)
    st = lib().macaq_flip_refine(W.data_ptr(), N, K, W.stride(0), s.data_ptr(), H.data_ptr(), w.codes.data_ptr(),
                                 w.scales.data_ptr(), int(max_rounds), moves.data_ptr(), ws.data_ptr(), ws_bytes,
                                 _stream_ptr(dev))
    _check(st, "macaq_flip_refine")
    return moves


def grouped_linear(x, offsets, weights, out_dtype=None, y=None, workspace=None):
    """MoE experts: rows offsets[g] .. offsets[g+1] - 1 of x go through weights[g]."""
    torch = _torch()
    _require(x, torch.bfloat16, "x")
    G = len(weights)
    if len(offsets) != G + 1:
        raise ValueError("offsets must have len(weights) + 1 entries")
    offs = (ctypes.c_int64 * (G + 1))(*[int(o) for o in offsets])
    ws_structs = (MacaqWeight * G)(*[w.c_struct() for w in weights])
    N, K = weights[0].N, weights[0].K
    M = int(offsets[-1])
    out_dtype = out_dtype or torch.bfloat16
    dev = x.device
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=dev)
    need = lib().macaq_grouped_linear_workspace_bytes(offs, G, K)
    ws, ws_bytes = _workspace(need, dev, workspace)
    st = lib().macaq_grouped_linear_w4a4(x.data_ptr(), x.stride(0), offs, G, ws_structs, y.data_ptr(), y.stride(0),
                                         _out_code(y.dtype), ws.data_ptr(), ws_bytes, _stream_ptr(dev))
    _check(st, "macaq_grouped_linear_w4a4")
    return y


def multi_linear(x, weights, out_dtype=None, ys=None, workspace=None):
    """Several layers that share the input x (q/k/v, gate/up): returns [y_g] with
    y_g = linear(x, weights[g]), from one quantiser launch and one GEMM launch."""
    torch = _torch()
    _require(x, torch.bfloat16, "x")
    M, K = x.shape
    G = len(weights)
    if G == 0 or any(w.K != K for w in weights):
        raise ValueError("weights must be non-empty and share x's K")
    out_dtype = out_dtype or torch.bfloat16
    dev = x.device
    if ys is None:
        ys = [torch.empty((M, w.N), dtype=out_dtype, device=dev) for w in weights]
    for y, w in zip(ys, weights):
        if tuple(y.shape) != (M, w.N) or y.dtype != ys[0].dtype or y.stride(1) != 1:
            raise ValueError("outputs must be [M, N_g] with one dtype and unit column stride")
    ws_structs = (MacaqWeight * G)(*[w.c_struct() for w in weights])
    yp = (ctypes.c_void_p * G)(*[y.data_ptr() for y in ys])
    lds = (ctypes.c_int64 * G)(*[y.stride(0) for y in ys])
    need = lib().macaq_multi_linear_workspace_bytes(M, K, G)
    ws, ws_bytes = _workspace(need, dev, workspace)
    st = lib().macaq_multi_linear_w4a4(x.data_ptr(), M, x.stride(0), ws_structs, G, yp, lds, _out_code(ys[0].dtype),
                                       ws.data_ptr(), ws_bytes, _stream_ptr(dev))
    _check(st, "macaq_multi_linear_w4a4")
    return ys


def quant_act(x, inv_s, codes=None, scales=None):
    """x: bf16 [M, K]; inv_s: fp32 [K]. Returns (codes uint8 [M, K/2], scales uint8)."""
    torch = _torch()
    _require(x, torch.bfloat16, "x")
    _require(inv_s, torch.float32, "inv_s")
    M, K = x.shape
    dev = x.device
    if codes is None:
        codes = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(scales_bytes(M, K), dtype=torch.uint8, device=dev)
    st = lib().macaq_quant_act(x.data_ptr(), M, K, x.stride(0), inv_s.data_ptr(), codes.data_ptr(),
                               scales.data_ptr(), _stream_ptr(dev))
    _check(st, "macaq_quant_act")
    return codes, scales


def _workspace(nbytes, device, workspace):
    torch = _torch()
    if nbytes == 0:
        return None, 0
    if workspace is not None and workspace.numel() >= nbytes:
        return workspace, workspace.numel()
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws, nbytes


def gemm_mxfp4(a_codes, a_scales, M, w, out_dtype=None, y=None, workspace=None):
    """Block-scaled FP4 GEMM on pre-quantised activations: y = A W'^T."""
    torch = _torch()
    out_dtype = out_dtype or torch.bfloat16
    dev = a_codes.device
    if y is None:
        y = torch.empty((M, w.N), dtype=out_dtype, device=dev)
    need = gemm_workspace_bytes(M, w.N, w.K, out_dtype)
    ws, ws_bytes = _workspace(need, dev, workspace)
    cw = w.c_struct()
    st = lib().macaq_gemm_mxfp4(a_codes.data_ptr(), a_scales.data_ptr(), M, ctypes.byref(cw), y.data_ptr(),
                                y.stride(0), _out_code(y.dtype), ws.data_ptr() if ws is not None else None,
                                ws_bytes, _stream_ptr(dev))
    _check(st, "macaq_gemm_mxfp4")
    return y


def linear(x, w, out_dtype=None, y=None, workspace=None, fused=False):
    """The MACaQ W4A4 layer: y = x W^T computed as (x diag(s)^-1 Hb)(Hb diag(s) W^T) in MXFP4.
    fused: False (two launches), True (one launch where that is faster: M <= 2), or
    "always" (one launch for every M <= 32 the kernel takes); in one launch the GEMM
    kernel makes the MXFP4 activations in shared memory itself."""
    torch = _torch()
    _require(x, torch.bfloat16, "x")
    out_dtype = out_dtype or torch.bfloat16
    M, K = x.shape
    if K != w.K:
        raise ValueError(f"x has K={K}, weight has K={w.K}")
    dev = x.device
    if y is None:
        y = torch.empty((M, w.N), dtype=out_dtype, device=dev)
    need = linear_workspace_bytes(M, w.N, K, y.dtype)
    ws, ws_bytes = _workspace(need, dev, workspace)
    cw = w.c_struct()
    st = lib().macaq_linear_w4a4(x.data_ptr(), M, x.stride(0), ctypes.byref(cw), y.data_ptr(), y.stride(0),
                                 _out_code(y.dtype), 2 if fused == "always" else 1 if fused else 0, ws.data_ptr(),
                                 ws_bytes, _stream_ptr(dev))
    _check(st, "macaq_linear_w4a4")
    return y


def linear_gather(x, w, dests, workspace=None):
    """The layer for one rank of a column-parallel cut, written into several outputs:
    dests are CUDA tensors [M, w.N] of one dtype (bf16 or fp32), each a column slice of a
    full-width y (unit column stride, one common row stride), all reachable from x's
    device. Every one receives this rank's columns of y."""
    torch = _torch()
    _require(x, torch.bfloat16, "x")
    M, K = x.shape
    if K != w.K:
        raise ValueError(f"x has K={K}, weight has K={w.K}")
    if not dests:
        raise ValueError("no destinations")
    dt, ld = dests[0].dtype, dests[0].stride(0)
    for d in dests:
        if tuple(d.shape) != (M, w.N) or d.dtype != dt or d.stride(0) != ld or d.stride(1) != 1:
            raise ValueError("destinations must be [M, N] slices with one dtype and row stride")
    addrs = (ctypes.c_uint64 * len(dests))(*[d.data_ptr() for d in dests])
    need = lib().macaq_linear_gather_workspace_bytes(M, w.N, K, _out_code(dt))
    ws, ws_bytes = _workspace(need, x.device, workspace)
    cw = w.c_struct()
    st = lib().macaq_linear_w4a4_gather(x.data_ptr(), M, x.stride(0), ctypes.byref(cw), addrs, len(dests), ld,
                                        _out_code(dt), ws.data_ptr(), ws_bytes, _stream_ptr(x.device))
    _check(st, "macaq_linear_w4a4_gather")
    return dests


def selftest_wait_timeout(limit_us=2000, device=None):
    """Run the bounded-wait self-test kernel on the current stream; returns the ten
    result words of macaq_selftest_wait_timeout as a dict."""
    torch = _torch()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    res = (ctypes.c_int64 * 10)()
    with torch.cuda.device(dev):
        _check(lib().macaq_selftest_wait_timeout(limit_us, res, _stream_ptr(dev)), "macaq_selftest_wait_timeout")
    r = list(res)
    return {"bar_timeout_ok": r[0], "bar_abort_ok": r[1], "bar_done_ok": r[2], "bar_err": r[3],
            "bar_timeout_ns": r[4], "bar_abort_ns": r[5], "set_agreed_ok": r[6], "set_err": r[7],
            "set_timeout_ns": r[8], "set_member_ok": r[9]}


def device_error():
    """Synchronise, read and clear the device error word (MACAQ_OK or a timeout)."""
    return lib().macaq_get_device_error()
