"""Per-call timing of the library on the seeded workloads, for the per-shape figures and
the ncu captures that back them.

    python -m mxfp4_w4a4_post_b200.timing list
    python -m mxfp4_w4a4_post_b200.timing {quant,gemm,linear,hessian,flip} WORKLOAD [--reps R]
                                          [--warmup W] [--fused] [--rows M] [--calib T] [--rounds R]
    python -m mxfp4_w4a4_post_b200.timing moe [--experts G] [--tokens T] [--n N] [--k K]
    python -m mxfp4_w4a4_post_b200.timing tp WORKLOAD [--world G]
    python -m mxfp4_w4a4_post_b200.timing layerset

Inputs are the workload's seeded synthetic tensors (workloads.py), resident on the
device. Before every timed call L2 is flushed by a 256 MiB write and a read of the same
buffer; each call is timed with CUDA events on the current stream and the mean is
printed, one line per measured call:
    quant    macaq_quant_act on x (weights prepared first)
    gemm     macaq_gemm_mxfp4 on the quantised x and the prepared weight
    linear   macaq_linear_w4a4 (fused = 0, or 2 with --fused: one launch whenever possible)
    hessian  macaq_hessian_blocks on T calibration rows (the workload's activation model
             with another seed) and macaq_prepare_weight_hessian on the weight
    moe      macaq_grouped_linear_w4a4 on T tokens routed over G experts (seeded skewed
             counts, tokens sorted by expert), against the same work as G separate
             macaq_linear_w4a4 calls
    tp       one rank's macaq_linear_w4a4 under a column- and a row-parallel cut into G
             pieces (the collective that follows needs several GPUs and is not timed)
    layerset the seven projections of a decoder layer at 256 rows: seven layer calls,
             and by role (q/k/v and gate/up each one macaq_multi_linear_w4a4 call)
    flip     macaq_hessian_full on T calibration rows, then macaq_flip_refine of the
             prepared weight (each timed call starts again from the round-to-nearest
             codes, restored before the flush); also prints the moves per row
"""
import argparse
import sys

import numpy as np

from . import workloads as wl

L2_FLUSH_BYTES = 256 << 20


def all_workloads():
    ws = {L.name: L for L in wl.all_single_layers()}
    ws.update({L.name: L for L in wl.qwen3_32b_layer_decode(256)})
    return ws


def _bf16(torch, a, dev):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)


def _time(torch, fn, flush, reps, warmup):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    total = 0.0
    for i in range(reps):
        flush.fill_(i & 0xFF)
        flush.view(torch.int32).max()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        total += a.elapsed_time(b) * 1e-3
    return total / reps


def moe(a):
    import ctypes
    import torch
    import mxfp4_w4a4_post_b200 as mq
    dev = torch.device("cuda", torch.cuda.current_device())
    G, T, N, K = a.experts, a.tokens, a.n, a.k
    rng = np.random.default_rng(5)
    p = 1.0 / np.arange(1, G + 1) ** 1.2
    counts = np.bincount(rng.choice(G, T, p=p / p.sum()), minlength=G)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    base = wl.with_shape(wl.tiny_layer(), M=T, N=N, K=K)
    x = _bf16(torch, wl.draw_x(base), dev)
    pws = []
    for g in range(G):
        Lg = wl.with_shape(base, M=1, seed=300 + g)
        pws.append(mq.prepare_weight(_bf16(torch, wl.draw_W(Lg), dev), torch.from_numpy(wl.draw_s(Lg)).to(dev)))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
    lib = mq.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    offs = (ctypes.c_int64 * (G + 1))(*offsets.tolist())
    wts = (mq.MacaqWeight * G)(*[w.c_struct() for w in pws])
    gws = torch.empty(lib.macaq_grouped_linear_workspace_bytes(offs, G, K), dtype=torch.uint8, device=dev)
    gargs = (x.data_ptr(), x.stride(0), offs, G, wts, y.data_ptr(), y.stride(0), mq.OUT_BF16, gws.data_ptr(),
             gws.numel(), stream)

    def grouped():
        st = lib.macaq_grouped_linear_w4a4(*gargs)
        if st != 0:
            raise mq.MacaqError(st, "macaq_grouped_linear_w4a4")

    lws = torch.empty(max(mq.linear_workspace_bytes(int(c), N, K, torch.bfloat16) for c in counts if c),
                      dtype=torch.uint8, device=dev)
    cws = [w.c_struct() for w in pws]
    calls = []
    for g in range(G):
        if counts[g]:
            calls.append((x[offsets[g]:].data_ptr(), int(counts[g]), x.stride(0), ctypes.byref(cws[g]),
                          y[offsets[g]:].data_ptr(), y.stride(0), mq.OUT_BF16, 0, lws.data_ptr(), lws.numel(),
                          stream))

    def separate():
        for args in calls:
            st = lib.macaq_linear_w4a4(*args)
            if st != 0:
                raise mq.MacaqError(st, "macaq_linear_w4a4")

    t_g = _time(torch, grouped, flush, a.reps, a.warmup)
    t_s = _time(torch, separate, flush, a.reps, a.warmup)
    flops = 2.0 * T * N * K
    print(f"moe G={G} tokens={T} N={N} K={K} counts={counts.tolist()}")
    print(f"grouped_linear_w4a4 {t_g * 1e6:.1f} us {flops / t_g / 1e12:.1f} TFLOP/s; "
          f"{G} separate linear_w4a4 calls {t_s * 1e6:.1f} us {flops / t_s / 1e12:.1f} TFLOP/s")
    return 1 if mq.device_error() != 0 else 0


def layerset(a):
    """The seven projections of a Qwen3-32B-shaped decoder layer at 256 rows, each with its
    own seeded input, weight and s: as seven macaq_linear_w4a4 calls, and by role, with
    the layers that share an input in one macaq_multi_linear_w4a4 call (q/k/v; gate/up)
    and o and down on their own (four calls)."""
    import ctypes
    import torch
    import mxfp4_w4a4_post_b200 as mq
    dev = torch.device("cuda", torch.cuda.current_device())
    layers = wl.qwen3_32b_layer_decode(256)
    by = {L.name.split("_")[2]: L for L in layers}          # q, k, v, o, gate, up, down
    pws, xs = {}, {}
    for k, L in by.items():
        pws[k] = mq.prepare_weight(_bf16(torch, wl.draw_W(L), dev), torch.from_numpy(wl.draw_s(L)).to(dev))
        xs[k] = _bf16(torch, wl.draw_x(L), dev)
    ys = {k: torch.empty((L.M, L.N), dtype=torch.bfloat16, device=dev) for k, L in by.items()}
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    lib = mq.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    cws = {k: pw.c_struct() for k, pw in pws.items()}
    lws = torch.empty(max(mq.linear_workspace_bytes(L.M, L.N, L.K, torch.bfloat16) for L in layers),
                      dtype=torch.uint8, device=dev)

    def lin_args(k):
        L = by[k]
        return (xs[k].data_ptr(), L.M, xs[k].stride(0), ctypes.byref(cws[k]), ys[k].data_ptr(), ys[k].stride(0),
                mq.OUT_BF16, 0, lws.data_ptr(), lws.numel(), stream)

    def multi_args(keys, x, ws_t):
        G = len(keys)
        wts = (mq.MacaqWeight * G)(*[cws[k] for k in keys])
        yp = (ctypes.c_void_p * G)(*[ys[k].data_ptr() for k in keys])
        lds = (ctypes.c_int64 * G)(*[ys[k].stride(0) for k in keys])
        return (x.data_ptr(), 256, x.stride(0), wts, G, yp, lds, mq.OUT_BF16, ws_t.data_ptr(), ws_t.numel(), stream)

    # the layers that share an input take one input (q/k/v: q's, gate/up: gate's)
    mws1 = torch.empty(lib.macaq_multi_linear_workspace_bytes(256, 5120, 3), dtype=torch.uint8, device=dev)
    mws2 = torch.empty(lib.macaq_multi_linear_workspace_bytes(256, 5120, 2), dtype=torch.uint8, device=dev)
    calls_sep = [(lib.macaq_linear_w4a4, lin_args(k)) for k in ("q", "k", "v", "o", "gate", "up", "down")]
    calls_role = [(lib.macaq_multi_linear_w4a4, multi_args(("q", "k", "v"), xs["q"], mws1)),
                  (lib.macaq_linear_w4a4, lin_args("o")),
                  (lib.macaq_multi_linear_w4a4, multi_args(("gate", "up"), xs["gate"], mws2)),
                  (lib.macaq_linear_w4a4, lin_args("down"))]

    def run(calls):
        def f():
            for fn, args in calls:
                st = fn(*args)
                if st != 0:
                    raise mq.MacaqError(st, fn.__name__)
        return f

    flops = sum(2.0 * L.M * L.N * L.K for L in layers)
    wbytes = sum(L.N * L.K * 0.53125 for L in layers)
    for label, calls in (("seven linear_w4a4 calls", calls_sep), ("by role (4 calls)", calls_role)):
        t = _time(torch, run(calls), flush, a.reps, a.warmup)
        print(f"qwen3_32b decoder-layer set, 256 rows, {label}: {t * 1e6:.1f} us {flops / t / 1e12:.1f} TFLOP/s "
              f"{wbytes / t / 1e9:.0f} GB/s of weights")
    for k in ("q", "k", "v", "o", "gate", "up", "down"):
        t = _time(torch, run([(lib.macaq_linear_w4a4, lin_args(k))]), flush, a.reps, a.warmup)
        print(f"  {by[k].name} linear_w4a4 {t * 1e6:.1f} us")
    for keys, x, ws_t in ((("q", "k", "v"), xs["q"], mws1), (("gate", "up"), xs["gate"], mws2)):
        t = _time(torch, run([(lib.macaq_multi_linear_w4a4, multi_args(keys, x, ws_t))]), flush, a.reps, a.warmup)
        print(f"  multi_linear_w4a4 {'/'.join(keys)} {t * 1e6:.1f} us")
    return 1 if mq.device_error() != 0 else 0


def tp(a, L):
    """One rank's layer call under column- and row-parallel cuts of the workload's weight
    into `--world` pieces (the rank with the largest piece), with the bytes its single
    collective would move; the collective itself needs more than one GPU."""
    import ctypes
    import torch
    import mxfp4_w4a4_post_b200 as mq
    from .tensor_parallel import split_k, split_range
    dev = torch.device("cuda", torch.cuda.current_device())
    M, N, K, g = L.M, L.N, L.K, a.world
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    x = _bf16(torch, wl.draw_x(L), dev)
    W, s = _bf16(torch, wl.draw_W(L), dev), torch.from_numpy(wl.draw_s(L)).to(dev)
    lib = mq.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    print(f"{L.name} M={M} N={N} K={K} world={g}")
    for cut in ("column", "row"):
        if cut == "column":
            n0, n1 = split_range(N, g, 0)
            pw = mq.prepare_weight(W[n0:n1], s)
            xs, out, Nl, Kl = x, torch.bfloat16, n1 - n0, K
            coll = f"all-gather {M * N * 2 / 1e6:.1f} MB bf16"
        else:
            k0, k1 = split_k(K, g, 0)
            pw = mq.prepare_weight(W[:, k0:k1], s[k0:k1].contiguous())
            xs, out, Nl, Kl = x[:, k0:k1], torch.float32, N, k1 - k0
            coll = f"all-reduce {M * N * 4 / 1e6:.1f} MB fp32"
        y = torch.empty((M, Nl), dtype=out, device=dev)
        oc = mq.OUT_BF16 if out == torch.bfloat16 else mq.OUT_F32
        ws = torch.empty(max(256, mq.linear_workspace_bytes(M, Nl, Kl, out)), dtype=torch.uint8, device=dev)
        cw = pw.c_struct()
        args = (xs.data_ptr(), M, xs.stride(0), ctypes.byref(cw), y.data_ptr(), y.stride(0), oc, 0,
                ws.data_ptr(), ws.numel(), stream)

        def run():
            st = lib.macaq_linear_w4a4(*args)
            if st != 0:
                raise mq.MacaqError(st, "macaq_linear_w4a4")

        t = _time(torch, run, flush, a.reps, a.warmup)
        flops = 2.0 * M * Nl * Kl
        print(f"{cut}-parallel rank 0 of {g}: linear_w4a4 {M}x{Nl}x{Kl} {t * 1e6:.1f} us "
              f"{flops / t / 1e12:.1f} TFLOP/s; then {coll}")
    return 1 if mq.device_error() != 0 else 0


def main(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("what", choices=["list", "quant", "gemm", "linear", "hessian", "flip", "moe", "tp", "layerset"])
    p.add_argument("workload", nargs="?")
    p.add_argument("--reps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--fused", action="store_true")
    p.add_argument("--rows", type=int, default=None,
                   help="run the workload's layer on this many rows of x (its first rows), e.g. a capture-sized slice")
    p.add_argument("--calib", type=int, default=2048, help="calibration rows for `hessian` and `flip`")
    p.add_argument("--rounds", type=int, default=256, help="move cap per row for `flip`")
    p.add_argument("--experts", type=int, default=8)
    p.add_argument("--tokens", type=int, default=4096)
    p.add_argument("--n", type=int, default=2048)
    p.add_argument("--k", type=int, default=4096)
    p.add_argument("--world", type=int, default=8, help="tensor-parallel pieces for `tp`")
    a = p.parse_args(argv)
    ws = all_workloads()
    if a.what == "list":
        print("\n".join(ws))
        return 0
    if a.what == "moe":
        return moe(a)
    if a.what == "layerset":
        return layerset(a)
    if a.workload not in ws:
        p.error(f"unknown workload {a.workload!r}; see `list`")
    L = ws[a.workload]
    if a.rows is not None:
        from dataclasses import replace
        L = replace(L, M=a.rows, name=f"{L.name}[rows={a.rows}]")
    if a.what == "tp":
        return tp(a, L)
    import torch
    import mxfp4_w4a4_post_b200 as mq
    dev = torch.device("cuda", torch.cuda.current_device())
    M, N, K = L.M, L.N, L.K
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    W, s = _bf16(torch, wl.draw_W(L), dev), torch.from_numpy(wl.draw_s(L)).to(dev)
    pw = mq.prepare_weight(W, s)
    out = torch.bfloat16 if L.out_dtype == "bf16" else torch.float32
    line = f"{L.name} M={M} N={N} K={K}"
    # the C-ABI calls with their arguments marshalled once, so that host-side Python
    # time stays out of the measured intervals
    import ctypes
    lib = mq.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    cw = pw.c_struct()
    oc = mq.OUT_BF16 if out == torch.bfloat16 else mq.OUT_F32

    def call(fn, *args):
        st = fn(*args)
        if st != 0:
            raise mq.MacaqError(st, fn.__name__)

    if a.what in ("quant", "gemm", "linear"):
        x = _bf16(torch, wl.draw_x(L), dev)
        codes, scales = mq.quant_act(x, pw.inv_s)
        y = torch.empty((M, N), dtype=out, device=dev)
        if a.what == "quant":
            args = (x.data_ptr(), M, K, x.stride(0), pw.inv_s.data_ptr(), codes.data_ptr(), scales.data_ptr(), stream)
            t = _time(torch, lambda: call(lib.macaq_quant_act, *args), flush, a.reps, a.warmup)
            print(f"{line} quant_act {t * 1e6:.2f} us {M * K * 2.53125 / t / 1e9:.1f} GB/s")
        elif a.what == "gemm":
            nws = mq.gemm_workspace_bytes(M, N, K, out)
            ws_t = torch.empty(max(256, nws), dtype=torch.uint8, device=dev)
            args = (codes.data_ptr(), scales.data_ptr(), M, ctypes.byref(cw), y.data_ptr(), y.stride(0), oc,
                    ws_t.data_ptr(), ws_t.numel(), stream)
            t = _time(torch, lambda: call(lib.macaq_gemm_mxfp4, *args), flush, a.reps, a.warmup)
            print(f"{line} gemm_mxfp4 {t * 1e6:.2f} us {2.0 * M * N * K / t / 1e12:.1f} TFLOP/s "
                  f"{(N * K + M * K) * 0.53125 / t / 1e9:.1f} GB/s of operands")
        else:
            ws_t = torch.empty(mq.linear_workspace_bytes(M, N, K, out), dtype=torch.uint8, device=dev)
            args = (x.data_ptr(), M, x.stride(0), ctypes.byref(cw), y.data_ptr(), y.stride(0), oc,
                    2 if a.fused else 0, ws_t.data_ptr(), ws_t.numel(), stream)
            t = _time(torch, lambda: call(lib.macaq_linear_w4a4, *args), flush, a.reps, a.warmup)
            print(f"{line} linear_w4a4 fused={2 if a.fused else 0} {t * 1e6:.2f} us {2.0 * M * N * K / t / 1e12:.1f} TFLOP/s")
    elif a.what == "flip":
        from dataclasses import replace
        xc = _bf16(torch, wl.draw_x(replace(L, M=a.calib, seed=L.seed + 100)), dev)
        hws = torch.empty(lib.macaq_hessian_full_workspace_bytes(a.calib, K), dtype=torch.uint8, device=dev)
        H = torch.empty((K, K), dtype=torch.float64, device=dev)
        hargs = (xc.data_ptr(), a.calib, K, xc.stride(0), s.data_ptr(), H.data_ptr(), hws.data_ptr(), hws.numel(),
                 stream)
        t_h = _time(torch, lambda: call(lib.macaq_hessian_full, *hargs), flush, a.reps, a.warmup)
        codes0 = pw.codes.clone()
        fws = torch.empty(lib.macaq_flip_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
        moves = torch.empty(N, dtype=torch.int32, device=dev)
        fargs = (W.data_ptr(), N, K, W.stride(0), s.data_ptr(), H.data_ptr(), pw.codes.data_ptr(),
                 pw.scales.data_ptr(), a.rounds, moves.data_ptr(), fws.data_ptr(), fws.numel(), stream)

        def refine():
            call(lib.macaq_flip_refine, *fargs)

        total = 0.0
        for i in range(a.warmup + a.reps):
            pw.codes.copy_(codes0)
            flush.fill_(i & 0xFF)
            flush.view(torch.int32).max()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            refine()
            e1.record()
            torch.cuda.synchronize()
            if i >= a.warmup:
                total += e0.elapsed_time(e1) * 1e-3
        t_f = total / a.reps
        mv = moves.float()
        print(f"{line} hessian_full T={a.calib} {t_h * 1e6:.1f} us")
        print(f"{line} flip_refine rounds<={a.rounds} {t_f * 1e6:.1f} us, moves per row mean "
              f"{mv.mean().item():.1f} max {int(mv.max().item())}")
    else:
        from dataclasses import replace
        xc = _bf16(torch, wl.draw_x(replace(L, M=a.calib, seed=L.seed + 100)), dev)
        H = mq.hessian_blocks(xc, s)
        hargs = (xc.data_ptr(), a.calib, K, xc.stride(0), s.data_ptr(), H.data_ptr(), stream)
        t_h = _time(torch, lambda: call(lib.macaq_hessian_blocks, *hargs), flush, a.reps, a.warmup)
        out_w = mq.prepare_weight_hessian(W, s, H)
        pargs = (W.data_ptr(), N, K, W.stride(0), s.data_ptr(), H.data_ptr(), out_w.codes.data_ptr(),
                 out_w.scales.data_ptr(), out_w.inv_s.data_ptr(), stream)
        t_p = _time(torch, lambda: call(lib.macaq_prepare_weight_hessian, *pargs), flush, a.reps, a.warmup)
        print(f"{line} hessian_blocks T={a.calib} {t_h * 1e6:.1f} us "
              f"{2.0 * a.calib * K * 32 / t_h / 1e12:.2f} TFLOP/s fp64")
        print(f"{line} prepare_weight_hessian {t_p * 1e6:.1f} us "
              f"{N * (K // 32) * 3 * 2048 / t_p / 1e12:.2f} TFLOP/s fp64")
    if mq.device_error() != 0:
        print("device error word set", file=sys.stderr)
        return 1
    return 0


if __name__ == "__main__":
    sys.exit(main())
