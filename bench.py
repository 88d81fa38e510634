"""Benchmark of the MACaQ W4A4 linear layer on B200.

One step = the whole path on one batch: offline weight preparation (W' = W diag(s) Hb
-> MXFP4), online activation transform + MXFP4 quantisation, and the block-scaled FP4
GEMM, on the Llama-3-8B gate/up prefill shape (x 4096x4096, W 14336x4096, bf16 out),
seeded synthetic inputs resident in HBM. L2 is flushed before every timed step by a
256 MiB write followed by a 256 MiB read of the same buffer, so the step starts with no
input lines and no dirty lines (whose write-back would be charged to the first kernel) in
L2; each step is timed with CUDA events on the launching stream.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload NAME]
  python bench.py --oracle-table

The `e2e` leg times the same steps from pinned host memory: every step uploads its x,
W and s and reads back its whole y, consecutive steps pipelined over copy-in, compute
and copy-out streams. `--impl reference` times the oracle on the host cores on a
bounded row sample; `--oracle-table` times the oracle per config, single-threaded and
with OpenMP, and uses no GPU.

Under torchrun (N > 1) every rank runs its own replica of the workload (token rows
are independent, no data-path collective): weak scaling, value = all ranks' FLOPs /
max-over-ranks time. Rank 0 prints one JSON line.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "W4A4 linear TFLOPS & quant-kernel GB/s (fraction of B200 roofline)"
UNIT = "TFLOP/s"
QUANT_BYTES_PER_ELEM = 2.0 + 0.5 + 1.0 / 32.0      # bf16 in, E2M1 codes + E8M0 scales out
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 4.0                                   # dense FP4 : BF16 tensor rate on sm_100
GEMM_SOURCES = ("gemm_kernel.cuh", "ptx_sm100.cuh", "macaq_api.cu")
# DRAM bytes (read + write) of one GEMM launch from an ncu capture of this workload, keyed by
# the digest of the GEMM sources it was taken on; any change to them retires the figure
# (traffic is then reported as null until a new capture). Summary: profiles/.
NCU_GEMM_TRAFFIC = {
    "llama3_8b_gate_up_prefill_4096x14336x4096": ("8cfd9d0bbb09657c", 142.389e6),
}


def gemm_source_digest():
    import hashlib
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        with open(os.path.join(ROOT, "mxfp4_w4a4_post_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def gemm_traffic(workload):
    digest, nbytes = NCU_GEMM_TRAFFIC.get(workload, (None, None))
    return nbytes if digest and digest == gemm_source_digest() else None


def workloads_by_name():
    from mxfp4_w4a4_post_b200 import workloads as wl
    ws = {L.name: L for L in wl.all_single_layers()}
    ws.update({L.name: L for L in wl.qwen3_32b_layer_decode(256)})
    return ws


DEFAULT_WORKLOAD = "llama3_8b_gate_up_prefill_4096x14336x4096"


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=500)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--oracle-table", action="store_true",
                   help="time the oracle on the host cores per config (single-threaded and OpenMP) "
                        "and print one JSON line per config and mode; uses no GPU")
    p.add_argument("--sample-rows", type=int, default=None,
                   help="oracle sample size in rows of x (default: 128 for the CPU baseline of the GPU arm; "
                        "for --impl reference, as many rows per step, up to 16, as keep the run within ~150 s)")
    return p.parse_args(argv)


# ------------------------------------------------------------------ helpers ---

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def gemm_flops(L):
    return 2.0 * L.M * L.N * L.K


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(x, device=None):
    """Max over ranks of a float (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(flops_per_rank, seconds_max, world):
    """Whole-job throughput: every rank's work over the slowest rank's time."""
    return flops_per_rank * world / seconds_max / 1e12


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if not self.path or not os.path.exists(self.path):
            return out
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if sm:
            out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                   "samples": len(sm)}
        return out


# ------------------------------------------------------------- our (GPU) arm ---

class DeviceStep:
    """Preallocated device buffers and the three library calls of one step."""

    def __init__(self, L, x, W, s, device):
        import torch
        import mxfp4_w4a4_post_b200 as mq
        self.torch = torch
        self.mq, self.L, self.dev = mq, L, device
        to_bf16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        self.x_host = to_bf16(x).pin_memory()
        self.W_host = to_bf16(W).pin_memory()
        self.s_host = torch.from_numpy(s).pin_memory()
        self.x = self.x_host.to(device)
        self.W = self.W_host.to(device)
        self.s = self.s_host.to(device)
        M, N, K = L.M, L.N, L.K
        self.pw = mq.PreparedWeight(torch.empty((N, K // 2), dtype=torch.uint8, device=device),
                                    torch.empty(mq.scales_bytes(N, K), dtype=torch.uint8, device=device),
                                    torch.empty(K, dtype=torch.float32, device=device), N, K)
        self.a_codes = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
        self.a_scales = torch.empty(mq.scales_bytes(M, K), dtype=torch.uint8, device=device)
        self.out_dtype = torch.bfloat16
        self.y = torch.empty((M, N), dtype=self.out_dtype, device=device)
        self.y_host = torch.empty((M, N), dtype=self.out_dtype).pin_memory()
        nws = mq.gemm_workspace_bytes(M, N, K, self.out_dtype)
        self.ws = torch.empty(max(nws, 256), dtype=torch.uint8, device=device)
        self.flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.launches_per_step = 3                            # prep, quant, gemm: one kernel each
        # The three C-ABI calls with their arguments marshalled once, so that the host
        # enqueues a step in a few microseconds (well inside the L2-flush kernel that
        # precedes it) and the device never waits for the host inside the timed region.
        import ctypes
        lib = mq.lib()
        stream = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
        self._cw = self.pw.c_struct()
        self._calls = [
            (lib.macaq_prepare_weight, (self.W.data_ptr(), N, K, self.W.stride(0), self.s.data_ptr(),
                                        self.pw.codes.data_ptr(), self.pw.scales.data_ptr(),
                                        self.pw.inv_s.data_ptr(), stream)),
            (lib.macaq_quant_act, (self.x.data_ptr(), M, K, self.x.stride(0), self.pw.inv_s.data_ptr(),
                                   self.a_codes.data_ptr(), self.a_scales.data_ptr(), stream)),
            (lib.macaq_gemm_mxfp4, (self.a_codes.data_ptr(), self.a_scales.data_ptr(), M, ctypes.byref(self._cw),
                                    self.y.data_ptr(), self.y.stride(0), mq.OUT_BF16, self.ws.data_ptr(),
                                    self.ws.numel(), stream)),
        ]

    def quant_stream(self, n_buf=8, reps=5):
        """Mean time per macaq_quant_act call over n_buf consecutive calls, each on its own
        copy of x and its own outputs (n_buf x 33.5 MB of inputs for the prefill shape,
        more than twice L2, so every call reads its x from HBM); consecutive launches
        overlap through programmatic dependent launch, as in the step. Best of `reps`
        passes, each after an L2 flush."""
        import ctypes
        torch, mq, L = self.torch, self.mq, self.L
        M, K = L.M, L.K
        lib = mq.lib()
        stream = ctypes.c_void_p(torch.cuda.current_stream(self.dev).cuda_stream)
        bufs = []
        for _ in range(n_buf):
            bufs.append((self.x.clone(), torch.empty((M, K // 2), dtype=torch.uint8, device=self.dev),
                         torch.empty(mq.scales_bytes(M, K), dtype=torch.uint8, device=self.dev)))
        calls = [(x.data_ptr(), M, K, x.stride(0), self.pw.inv_s.data_ptr(), c.data_ptr(), sc.data_ptr(), stream)
                 for x, c, sc in bufs]
        best = None
        for r in range(reps + 1):
            self.flush_l2(r)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for args in calls:
                st = lib.macaq_quant_act(*args)
                if st != 0:
                    raise RuntimeError(f"macaq_quant_act returned {st}")
            e1.record()
            torch.cuda.synchronize(self.dev)
            t = e0.elapsed_time(e1) * 1e-3 / n_buf
            if r > 0:
                best = t if best is None else min(best, t)
        del bufs
        return best

    def flush_l2(self, i):
        """Write, then read back, a buffer twice the L2 size: every line of the step's
        inputs is evicted and the lines left behind are clean."""
        self.flush.fill_(i & 0xFF)
        self.flush.view(self.torch.int32).max()

    def step(self, ev=None):
        """One step. ev: None, (start, end) events around the step, or four events
        around each of the three calls (which serialises the calls' launches)."""
        per_call = ev is not None and len(ev) == 4
        if ev is not None:
            ev[0].record()
        for i, (fn, args) in enumerate(self._calls):
            if per_call and i > 0:
                ev[i].record()
            st = fn(*args)
            if st != 0:
                raise RuntimeError(f"{fn.__name__} returned {st}")
        if ev is not None:
            ev[-1].record()

    def run_e2e_pipelined(self, n):
        """n steps from pinned host buffers with their copies in flight together: step i's
        x, W and s go host -> device on a copy-in stream, its three calls run on a
        compute stream, its y goes device -> host on a copy-out stream; device buffers
        are double-buffered and events order every reuse, so the upload of step i + 1
        and the read-back of step i - 1 overlap step i (PCIe carries both directions at
        once). Every step still copies all of its inputs and all of its result. Returns
        seconds per step (first upload to last read-back, CUDA events)."""
        import ctypes
        torch, mq, dev = self.torch, self.mq, self.x.device
        M, N, K = self.L.M, self.L.N, self.L.K
        s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        lib = mq.lib()
        slots = []
        for k in range(2):
            b = {"x": torch.empty_like(self.x), "W": torch.empty_like(self.W), "s": torch.empty_like(self.s),
                 "y": torch.empty_like(self.y),
                 "pw": mq.PreparedWeight(torch.empty_like(self.pw.codes), torch.empty_like(self.pw.scales),
                                         torch.empty_like(self.pw.inv_s), N, K),
                 "ac": torch.empty_like(self.a_codes), "as": torch.empty_like(self.a_scales),
                 "ws": torch.empty_like(self.ws)}
            b["cw"] = b["pw"].c_struct()
            cs = ctypes.c_void_p(s_comp.cuda_stream)
            b["calls"] = [
                (lib.macaq_prepare_weight, (b["W"].data_ptr(), N, K, b["W"].stride(0), b["s"].data_ptr(),
                                            b["pw"].codes.data_ptr(), b["pw"].scales.data_ptr(),
                                            b["pw"].inv_s.data_ptr(), cs)),
                (lib.macaq_quant_act, (b["x"].data_ptr(), M, K, b["x"].stride(0), b["pw"].inv_s.data_ptr(),
                                       b["ac"].data_ptr(), b["as"].data_ptr(), cs)),
                (lib.macaq_gemm_mxfp4, (b["ac"].data_ptr(), b["as"].data_ptr(), M, ctypes.byref(b["cw"]),
                                        b["y"].data_ptr(), b["y"].stride(0), mq.OUT_BF16, b["ws"].data_ptr(),
                                        b["ws"].numel(), cs)),
            ]
            b["in_done"] = b["comp_done"] = b["out_done"] = None
            slots.append(b)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for i in range(n):
            b = slots[i % 2]
            with torch.cuda.stream(s_in):
                if b["comp_done"] is not None:
                    s_in.wait_event(b["comp_done"])          # the slot's inputs are consumed
                b["x"].copy_(self.x_host, non_blocking=True)
                b["W"].copy_(self.W_host, non_blocking=True)
                b["s"].copy_(self.s_host, non_blocking=True)
                b["in_done"] = torch.cuda.Event()
                b["in_done"].record(s_in)
            s_comp.wait_event(b["in_done"])
            if b["out_done"] is not None:
                s_comp.wait_event(b["out_done"])             # the slot's y has been read back
            for fn, args in b["calls"]:
                st = fn(*args)
                if st != 0:
                    raise RuntimeError(f"{fn.__name__} returned {st}")
            b["comp_done"] = torch.cuda.Event()
            b["comp_done"].record(s_comp)
            s_out.wait_event(b["comp_done"])
            with torch.cuda.stream(s_out):
                self.y_host.copy_(b["y"], non_blocking=True)
                b["out_done"] = torch.cuda.Event()
                b["out_done"].record(s_out)
        e1.record(s_out)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) * 1e-3 / n

    def h2d_bytes(self):
        return self.x.numel() * 2 + self.W.numel() * 2 + self.s.numel() * 4

    def d2h_bytes(self):
        return self.y.numel() * self.y.element_size()


def run_ours(args):
    import torch
    import torch.distributed as dist
    import mxfp4_w4a4_post_b200 as mq
    from mxfp4_w4a4_post_b200 import workloads as wl

    rank, world, local = dist_env()
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)
    mq.lib()
    L = workloads_by_name()[args.workload]
    x, W, s = wl.draw_x(L), wl.draw_W(L), wl.draw_s(L)
    st = DeviceStep(L, x, W, s, device)
    stream = torch.cuda.current_stream(device)

    for _ in range(max(args.warmup, 3)):
        st.flush_l2(1)
        st.step()
    torch.cuda.synchronize(device)
    if mq.device_error() != 0:
        raise RuntimeError("device error word set during warm-up")

    # Timed region 1: whole steps (events only at step boundaries, so consecutive
    # kernels keep their launch overlap). Timed region 2: the same steps with events
    # around each call, for the per-kernel durations of the roofline figures.
    ev_step = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    ev_call = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(args.steps):
            st.flush_l2(i)                        # evict L2 before the step (untimed)
            st.step(ev_step[i])
        for i in range(args.steps):
            st.flush_l2(i)
            st.step(ev_call[i])
        torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    assert mq.device_error() == 0

    t_step = [ev_step[i][0].elapsed_time(ev_step[i][1]) * 1e-3 for i in range(args.steps)]
    t_prep = [ev_call[i][0].elapsed_time(ev_call[i][1]) * 1e-3 for i in range(args.steps)]
    t_quant = [ev_call[i][1].elapsed_time(ev_call[i][2]) * 1e-3 for i in range(args.steps)]
    t_gemm = [ev_call[i][2].elapsed_time(ev_call[i][3]) * 1e-3 for i in range(args.steps)]
    total = reduce_max(sum(t_step), device)
    sec_per_step = total / args.steps
    value = aggregate(gemm_flops(L), sec_per_step, world)

    peaks, peak_src = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    g_avg = reduce_max(statistics.mean(t_gemm), device)
    q_avg = reduce_max(statistics.mean(t_quant), device)
    p_avg = reduce_max(statistics.mean(t_prep), device)
    gemm_tflops = gemm_flops(L) / g_avg / 1e12
    q_bytes = QUANT_BYTES_PER_ELEM * L.M * L.K + 4 * L.K
    p_bytes = QUANT_BYTES_PER_ELEM * L.N * L.K + 8 * L.K
    q_gbs = q_bytes / q_avg / 1e9
    p_gbs = p_bytes / p_avg / 1e9

    q_stream = reduce_max(st.quant_stream(), device)
    q_stream_gbs = q_bytes / q_stream / 1e9

    e2e = None
    if not args.no_e2e:
        n_e2e = max(3, min(args.steps, 30))
        st.run_e2e_pipelined(2)                             # warm-up
        if world > 1:
            dist.barrier()
        t_e2e = reduce_max(st.run_e2e_pipelined(n_e2e), device)
        e2e = {"value": aggregate(gemm_flops(L), t_e2e, world), "unit": UNIT,
               "h2d_bytes_per_step": st.h2d_bytes(), "d2h_bytes_per_step": st.d2h_bytes(),
               "ms_per_step": t_e2e * 1e3, "steps": n_e2e,
               "path": "pinned host x, W, s -> C ABI calls -> pinned host y; uploads, compute and "
                       "read-backs of consecutive steps on three streams (double-buffered)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(L, x, W, s, args.sample_rows or 128)

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": sec_per_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "mxfp4 (e2m1 x e2m1, e8m0 scales, f32 accumulate); transform in f32",
        "data": "synthetic (seeded; Student-t(3) activations with 0.5% x20 outlier channels, N(0,0.02) weights)",
        "config": {"workload": L.name, "M": L.M, "N": L.N, "K": L.K, "out_dtype": "bf16",
                   "step": "prepare_weight + quant_act + gemm_mxfp4",
                   "l2": f"flushed before every timed step ({L2_FLUSH_BYTES >> 20} MiB write, then read)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": gemm_tflops / fp4_peak, "traffic": gemm_traffic(L.name),
                     "kernel": "gemm_mxf4_kernel",
                     "peak_source": f"{peak_src} bf16 burst x {FP4_OVER_BF16:g} (dense FP4:BF16 rate)"},
        "kernels": {
            "gemm_mxfp4": {"us": g_avg * 1e6, "tflops": gemm_tflops, "frac_fp4_peak": gemm_tflops / fp4_peak},
            "quant_act": {"us": q_avg * 1e6, "gbs": q_gbs, "frac_hbm": q_gbs / peaks["hbm_gbs"],
                          "bytes": q_bytes,
                          "us_stream": q_stream * 1e6, "gbs_stream": q_stream_gbs,
                          "frac_hbm_stream": q_stream_gbs / peaks["hbm_gbs"],
                          "stream": "mean per call over 8 consecutive calls on 8 copies of x (268 MB of "
                                    "inputs, > 2x L2), launches overlapped; 'us' is one call between "
                                    "events after an L2 flush, which includes ~5 us of launch gap (an "
                                    "empty kernel measures 5.4 us that way on this box)"},
            "prepare_weight": {"us": p_avg * 1e6, "gbs": p_gbs, "frac_hbm": p_gbs / peaks["hbm_gbs"],
                               "bytes": p_bytes},
            "quant_over_gemm": q_avg / g_avg,
            "hbm_peak_gbs": peaks["hbm_gbs"],
        },
        "e2e": e2e,
        "cpu_baseline": cpu,
        "gpu_launches": st.launches_per_step * args.steps * 2,   # both timed regions
        "clocks": clk.summary(),
    }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)
    return result


# ----------------------------------------------------------- oracle (CPU) ----

def oracle_sample(L, x, W_codes_full, W_scales_full, W, s, rows, prep_rows):
    """One bounded sample of the step on the host cores: weight preparation of
    `prep_rows` rows of W (the sample's share), quantisation of `rows` rows of x and
    their fp64 GEMM against the full prepared weight. Returns seconds."""
    import oracle
    t0 = time.perf_counter()
    oracle.prepare_weight(W[:prep_rows], s)
    inv_s = (np.float32(1.0) / s).astype(np.float32)
    ac, as_ = oracle.quant_rows(x[:rows], inv_s)
    oracle.gemm_fp64(ac, as_, W_codes_full, W_scales_full, L.K)
    return time.perf_counter() - t0


def cpu_baseline(L, x, W, s, rows):
    import oracle
    wc, ws, _ = oracle.prepare_weight(W, s)
    prep_rows = max(1, int(round(L.N * rows / L.M)))
    t = oracle_sample(L, x, wc, ws, W, s, rows, prep_rows)
    flops = 2.0 * rows * L.N * L.K
    return {"value": flops / t / 1e12, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{rows} of {L.M} rows of x (quantise + fp64 GEMM against all {L.N} prepared "
                      f"weight rows) plus the matching {prep_rows}-row share of the weight preparation; "
                      f"single-threaded C, {t:.1f} s"}


def run_reference(args):
    import torch.distributed as dist  # noqa: F401
    from mxfp4_w4a4_post_b200 import workloads as wl
    import oracle

    rank, world, _ = dist_env()
    if rank != 0:
        return None
    L = workloads_by_name()[args.workload]
    x, W, s = wl.draw_x(L, rows=16), wl.draw_W(L), wl.draw_s(L)
    wc, ws, _ = oracle.prepare_weight(W, s)
    rows = args.sample_rows
    if rows is None:
        # size each step's sample so that warm-up + timed steps stay within ~150 s
        t1 = oracle_sample(L, x, wc, ws, W, s, 1, max(1, int(round(L.N / L.M))))
        rows = int(max(1, min(16, 150.0 / (max(1, args.steps + args.warmup) * t1))))
    rows = min(rows, x.shape[0])
    prep_rows = max(1, int(round(L.N * rows / L.M)))
    for _ in range(args.warmup):
        oracle_sample(L, x, wc, ws, W, s, rows, prep_rows)
    times = [oracle_sample(L, x, wc, ws, W, s, rows, prep_rows) for _ in range(args.steps)]
    t = sum(times) / len(times)
    flops = 2.0 * rows * L.N * L.K
    value = flops / t / 1e12
    sample = (f"{rows} of {L.M} rows of x per step (quantise + fp64 GEMM against all {L.N} "
              f"prepared weight rows) plus the matching {prep_rows}-row share of the weight preparation")
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 transform, f64 GEMM", "data": "synthetic (seeded)",
        "config": {"workload": f"{L.name} (sampled: {rows} of {L.M} rows per step)", "M": L.M, "N": L.N,
                   "K": L.K, "out_dtype": "f64", "step": "prepare_weight + quant_act + gemm (bounded row sample)"},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)
    return result


def oracle_configs():
    """(label, workloads, GEMM rows per workload: None = all rows) of the oracle table."""
    from mxfp4_w4a4_post_b200 import workloads as wl
    return [
        ("C1", [wl.tiny_layer()], None),
        ("C2", [wl.llama3_8b_gate_up_prefill()], 256),
        ("C3", [wl.qwen3_32b_up_decode(b) for b in (1, 8, 16, 64)], None),
        ("C4", [wl.qwen3_32b_down_prefill()], 256),
        ("C5", wl.qwen3_32b_layer_decode(256), None),
    ]


def oracle_table(args):
    """The oracle on the host cores, per config, single-threaded and with OpenMP over
    rows: full quantisation of x and preparation of W, and the fp64 GEMM over all rows
    (C1, C3, C5) or over 256 seeded sampled rows of x (C2, C4; the single-threaded run
    of C5 also samples, 64 rows per linear). One JSON line per config and mode; GEMM
    throughput in MAC/s with the full-size time extrapolated from it."""
    import oracle
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    rows_out = []
    for label, layers, gemm_rows in oracle_configs():
        inputs = []
        for L in layers:
            x, W, s = wl_draw(L)
            inputs.append((L, x, W, s))
        for omp in (False, True):
            oracle.set_openmp(omp)
            t_q = t_g = 0.0
            elems = macs = macs_full = 0
            sampled = False
            for L, x, W, s in inputs:
                t0 = time.perf_counter()
                wc, ws, inv = oracle.prepare_weight(W, s)
                ac, as_ = oracle.quant_rows(x, inv)
                t_q += time.perf_counter() - t0
                elems += L.M * L.K + L.N * L.K
                r = gemm_rows
                if r is None and not omp and label == "C5":
                    r = 64
                if r is not None and r < L.M:
                    sampled = True
                    idx = np.sort(np.random.default_rng(0).choice(L.M, r, replace=False)).astype(np.int64)
                else:
                    idx = None
                t0 = time.perf_counter()
                oracle.gemm_fp64(ac, as_, wc, ws, L.K, rows=idx)
                t_g += time.perf_counter() - t0
                n = L.M if idx is None else len(idx)
                macs += n * L.N * L.K
                macs_full += L.M * L.N * L.K
            mac_s = macs / t_g
            line = {
                "oracle_table": label, "mode": "openmp" if omp else "single-thread",
                "threads": cores if omp else 1, "host_cores": cores,
                "workloads": [L.name for L, *_ in inputs],
                "quantise_s": t_q, "quantise_elems": elems, "quantise_melem_per_s": elems / t_q / 1e6,
                "gemm_s": t_g, "gemm_macs": macs, "gemm_mac_per_s": mac_s,
                "gemm_rows": "sampled" if sampled else "all",
                "gemm_full_s_extrapolated" if sampled else "gemm_full_s": macs_full / mac_s,
            }
            print(json.dumps(line), flush=True)
            rows_out.append(line)
    oracle.set_openmp(False)
    return rows_out


def wl_draw(L):
    from mxfp4_w4a4_post_b200 import workloads as wl
    return wl.draw_x(L), wl.draw_W(L), wl.draw_s(L)


def main(argv=None):
    args = parse_args(argv)
    if args.oracle_table:
        oracle_table(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
