"""Benchmark of libbsq on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl bsq|reference]
                    [--workload prefill|tiny] [--no-rows]

A step is one pass of the W4A4 linear layer's hot path over one batch:
quantise the BF16 activations to NVFP4 (scale2 = 1), then the NVFP4 x NVFP4
GEMM into BF16, at M=4096, N=17408, K=5120 (Student-t(4) activations with 1%
outlier channels x20, N(0,0.02) weight quantised once to NVFP4 with its
per-tensor scale2).  `value` is whole-job TFLOP/s (2*M*N*K per step, summed
over ranks).  The same JSON line carries, under "rows", a device-timed
measurement of every other kernel of the path (FP8 GEMV for M = 1, 2, 8, 16
and the lm_head shape, the quantisers, the int8 per-32 GEMM, the row-scaled
FP8 GEMM), each against its roofline.

Multi-GPU: one process per GPU (torchrun), every rank runs the same
per-GPU problem (independent replicas, no data-path collective), timing is
the max over ranks -> "scaling": "weak".

--impl reference times the CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4 GEMM TFLOPS & % FP4 peak; M≤16 FP8 GEMV GB/s & % HBM peak"
WORKLOADS = {
    "prefill": dict(m=4096, n=17408, k=5120),
    "tiny": dict(m=16, n=256, k=512),
}
L2_BYTES = 126 * 1024 * 1024
# dense tensor-core throughput relative to BF16 (NVIDIA B200 datasheet ratios)
RATIO_FP4, RATIO_FP8, RATIO_INT8 = 4.0, 2.0, 2.0
SM_MAX_MHZ = 1965  # B200 clocks.max.sm
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def workload_desc(w):
    return (f"W4A4 linear: NVFP4 activation quantisation + NVFP4xNVFP4 GEMM -> BF16, "
            f"M={w['m']} N={w['n']} K={w['k']}")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------- ranks -----

def rank_info():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def dist_init(backend: str, world: int):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, device) -> float:
    """Max of a float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
    if device.type == "cuda":
        torch.cuda.synchronize(device)


# -------------------------------------------------------------- clocks -----

class ClockSampler:
    """Samples SM clock and clock-event (throttle) reasons through NVML while
    the timed region runs.  Reads only."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.ok = [], 0, False
        self.index, self.period = index, period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
                self.reasons |= int(n.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        reasons = [name for bit, name in self.REASONS.items() if self.reasons & bit and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples),
                "source": "nvml" if self.ok else "unavailable"}


# -------------------------------------------------------------- our arm ----

def _events(torch, n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def time_launches(torch, stream, fn, iters, warm=3):
    """Average device time of fn() over iters back-to-back calls (events on
    the launching stream)."""
    for _ in range(warm):
        fn()
    s, e = _events(torch, 2)
    torch.cuda.synchronize()
    s.record(stream)
    for _ in range(iters):
        fn()
    e.record(stream)
    e.synchronize()
    return s.elapsed_time(e) * 1e-3 / iters


def time_graph(torch, fn, iters, reps=5):
    """Average device time of fn(stream) over iters launches captured into
    one CUDA graph and replayed reps times (events on the replay stream):
    back-to-back kernel time without per-launch host overhead, for kernels
    short enough for that overhead to matter."""
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        for _ in range(3):
            fn(st)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        for _ in range(iters):
            fn(st)
    with torch.cuda.stream(st):
        g.replay()
        s, e = _events(torch, 2)
        st.synchronize()
        s.record(st)
        for _ in range(reps):
            g.replay()
        e.record(st)
    e.synchronize()
    del g
    return s.elapsed_time(e) * 1e-3 / (reps * iters)


def kernel_hash(name):
    with open(os.path.join(ROOT, "int8_gemm_gemv_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def ncu_traffic(profile_json, kernel_file):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the kernel source as it is now."""
    p = os.path.join(ROOT, "profiles", profile_json)
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("kernel_sha256_16") != kernel_hash(kernel_file):
        return None
    return d.get("dram_bytes_per_launch_full_size")


def run_bsq(args, w, peaks, peak_src):
    import torch
    import int8_gemm_gemv_b200 as bsq
    from int8_gemm_gemv_b200 import synth

    rank, world, local = rank_info()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist_init("nccl", world)
    stream = torch.cuda.current_stream(dev)
    m, n, k = w["m"], w["n"], w["k"]

    # ---- inputs: resident in HBM before timing; 3 rotating sets when the
    # working set would otherwise fit in L2
    a_bf, w_bf = synth.w4a4_inputs(m, n, k, seed=0, heavy_tailed=True)
    per_set = m * k * 2 + n * k // 2 + n * k // 16 + m * k // 2 + m * k // 16
    nsets = 1 if args.workload == "tiny" else max(1, -(-2 * L2_BYTES // per_set) + 1)
    a_dev, w_codes = [], []
    amax = torch.empty(1, dtype=torch.float32, device=dev)
    for i in range(nsets):
        a_i = torch.from_numpy(a_bf.view(np.int16)).to(dev) if i == 0 else a_dev[0].clone()
        a_dev.append(a_i)
        wb = torch.from_numpy(w_bf.view(np.int16)).to(dev)
        bsq.bsq_amax_bf16(wb, wb.numel(), amax)
        scale_b2 = float(np.float32(amax.item()) / np.float32(6 * 448))
        wp = torch.empty((n, k // 2), dtype=torch.uint8, device=dev)
        wsf = torch.empty((n, k // 16), dtype=torch.uint8, device=dev)
        bsq.quantize_bf16_to_nvfp4(wb, wp, wsf, scale_b2, n, k)
        w_codes.append((wp, wsf, scale_b2))
        del wb
    ap = [torch.empty((m, k // 2), dtype=torch.uint8, device=dev) for _ in range(nsets)]
    asf = [torch.empty((m, k // 16), dtype=torch.uint8, device=dev) for _ in range(nsets)]
    out = torch.empty((m, n), dtype=torch.int16, device=dev)
    torch.cuda.synchronize()

    def step(i):
        j = i % nsets
        wp, wsf, sb2 = w_codes[j]
        bsq.quantize_bf16_to_nvfp4(a_dev[j], ap[j], asf[j], 1.0, m, k, stream)
        bsq.w4a4_gemm(ap[j], asf[j], wp, wsf, out, 1.0, sb2, m, n, k, stream)

    for i in range(args.warmup):
        step(i)
    t0, t1 = _events(torch, 2)
    barrier(dev)
    launches0 = bsq.debug_launch_count()
    # the timed region: back-to-back steps with no event between the two
    # kernels, so the GEMM's prologue overlaps the quantiser's tail
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        t0.record(stream)
        for i in range(args.steps):
            step(i)
        t1.record(stream)
        t1.synchronize()
    launches = bsq.debug_launch_count() - launches0
    barrier(dev)
    elapsed = t0.elapsed_time(t1) * 1e-3
    t_max = max_over_ranks(elapsed, dev)
    # per-kernel durations: each kernel of the step run alone, back to back
    # over the same rotating input sets, between two events on the stream
    def kernel_time(fn):
        fn(0)
        s0, s1 = _events(torch, 2)
        s0.record(stream)
        for i in range(args.steps):
            fn(i)
        s1.record(stream)
        s1.synchronize()
        return s0.elapsed_time(s1) * 1e-3 / args.steps

    quant_t = kernel_time(lambda i: bsq.quantize_bf16_to_nvfp4(a_dev[i % nsets], ap[i % nsets], asf[i % nsets], 1.0,
                                                               m, k, stream))
    gemm_t = kernel_time(lambda i: bsq.w4a4_gemm(ap[i % nsets], asf[i % nsets], w_codes[i % nsets][0],
                                                 w_codes[i % nsets][1], out, 1.0, w_codes[i % nsets][2], m, n, k,
                                                 stream))
    flops = 2.0 * m * n * k
    value = world * flops * args.steps / t_max / 1e12

    # ---- end to end through the public API: pinned host input in, host
    # output back, every step.  Steps are pipelined the way a serving loop
    # would run them: the input copy, the two kernels and the output copy of
    # a step go on three streams with two buffers, so step i's compute
    # overlaps step i-1's read-back and step i+1's upload (the two copy
    # directions use separate copy engines).  Every step still moves its own
    # input in and its own result out inside the timed region.
    e2e_steps = max(1, min(args.steps, 10))
    a_host = torch.from_numpy(a_bf.view(np.int16)).pin_memory()
    out_host = [torch.empty((m, n), dtype=torch.int16).pin_memory() for _ in range(2)]
    a_stage = [torch.empty_like(a_dev[0]) for _ in range(2)]
    outs = [out] + [torch.empty_like(out)]
    wp, wsf, sb2 = w_codes[0]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {key: [torch.cuda.Event() for _ in range(2)] for key in ("in", "cmp", "out")}
    started = [False, False]

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if started[b]:
                s_in.wait_event(ev["cmp"][b])  # the step before last has read a_stage[b]
            a_stage[b].copy_(a_host, non_blocking=True)
            ev["in"][b].record(s_in)
        stream.wait_event(ev["in"][b])
        if started[b]:
            stream.wait_event(ev["out"][b])  # outs[b] has been read back
        bsq.quantize_bf16_to_nvfp4(a_stage[b], ap[b % nsets], asf[b % nsets], 1.0, m, k, stream)
        bsq.w4a4_gemm(ap[b % nsets], asf[b % nsets], wp, wsf, outs[b], 1.0, sb2, m, n, k, stream)
        ev["cmp"][b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["cmp"][b])
            out_host[b].copy_(outs[b], non_blocking=True)
            ev["out"][b].record(s_out)
        started[b] = True

    e2e_step(0)
    e2e_step(1)
    torch.cuda.synchronize()
    barrier(dev)
    s, e = _events(torch, 2)
    s.record(stream)
    s_in.wait_event(s)
    s_out.wait_event(s)
    for i in range(e2e_steps):
        e2e_step(i)
    for b in range(2):
        stream.wait_event(ev["out"][b])
    e.record(stream)
    e.synchronize()
    e2e_t = max_over_ranks(s.elapsed_time(e) * 1e-3, dev)
    e2e_value = world * flops * e2e_steps / e2e_t / 1e12

    long_region = elapsed > 1.0
    bf16_peak = peaks["bf16_tflops_sustained"] if long_region else peaks["bf16_tflops"]
    fp4_peak = bf16_peak * RATIO_FP4
    achieved = flops / gemm_t / 1e12
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_max / args.steps * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3/16, fp32 accumulate)",
        "data": "synthetic (seeded Student-t(4) activations with 1% outlier channels x20; N(0,0.02) weight)",
        "config": {"workload": workload_desc(w), "m": m, "n": n, "k": k,
                   "l2": (f"{nsets} rotating input sets of {per_set / 1e6:.0f} MB (> 2x L2) plus a "
                          f"{m * n * 2 / 1e6:.0f} MB output" if nsets > 1 else "single set (tiny)"),
                   "parallelism": f"replicas x{world}"},
        "gpu_launches": int(launches),
        "roofline": {"bound": "tensor", "kernel": "w4a4_gemm", "achieved": round(achieved, 1),
                     "peak": round(fp4_peak, 1), "unit": "TFLOP/s", "frac": round(achieved / fp4_peak, 4),
                     "peak_source": (f"{peak_src} bf16 {'sustained' if long_region else 'burst'} "
                                     f"{bf16_peak} x {RATIO_FP4:.0f} (dense FP4/BF16 ratio)"),
                     "traffic": ncu_traffic("w4a4_gemm.json", "gemm_w4a4.cu"),
                     "algorithmic_flops_per_launch": flops},
        "step_breakdown_us": {"quantize_bf16_to_nvfp4": round(quant_t * 1e6, 2), "w4a4_gemm": round(gemm_t * 1e6, 2)},
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "steps": e2e_steps,
                "h2d_bytes_per_step": int(a_host.numel() * 2), "d2h_bytes_per_step": int(out_host[0].numel() * 2),
                "schedule": "input copy, kernels and output copy on three streams, two buffers"},
        "clocks": clk.summary(),
    }
    del a_dev, w_codes, ap, asf, out, a_stage, outs
    torch.cuda.empty_cache()
    if args.rows and args.workload == "prefill":
        line["rows"] = measure_rows(torch, bsq, dev, stream, peaks, peak_src)
    return line, rank


def measure_rows(torch, bsq, dev, stream, peaks, peak_src):
    """Device time of every other kernel of the path at the workload shapes,
    inputs larger than L2 (rotating copies where needed)."""
    hbm = peaks["hbm_gbs"]
    bf16 = peaks["bf16_tflops"]
    rows = {}
    g = torch.Generator(device=dev)
    g.manual_seed(0)

    def bf16_rand(shape, std):
        return (torch.randn(shape, device=dev, generator=g) * std).to(torch.bfloat16)

    def rotate(make, nbytes):
        cnt = max(1, -(-2 * L2_BYTES // max(nbytes, 1)) + 1)
        return [make() for _ in range(cnt)]

    def hbm_row(name, t, nbytes, extra=None):
        r = {"us": round(t * 1e6, 3), "gbs": round(nbytes / t / 1e9, 1), "bytes": int(nbytes),
             "frac_hbm": round(nbytes / t / 1e9 / hbm, 4), "bound": "hbm"}
        if extra:
            r.update(extra)
        rows[name] = r

    # a4: FP8 GEMV, M = 1, 2, 8, 16 at 5120x5120 and M = 2 at 151936x5120
    for (n, k, ms) in ((5120, 5120, (1, 2, 8, 16)), (151936, 5120, (2,))):
        def mk_w():
            wq = torch.empty((n, k), dtype=torch.uint8, device=dev)
            ws = torch.empty((n,), dtype=torch.float32, device=dev)
            src = bf16_rand((n, k), 0.02)
            bsq.quant_rowwise_fp8(src, wq, ws, n, k, stream)
            return wq, ws
        ws_list = rotate(mk_w, n * k)
        # the floor: a read-only kernel launched like the GEMV (one CTA per SM,
        # programmatic stream serialization) over the same rotating copies
        sink = torch.zeros(1, dtype=torch.int32, device=dev)
        itf = [0]

        def floor_fn(st):
            wq, _ = ws_list[itf[0] % len(ws_list)]
            itf[0] += 1
            bsq.debug_stream_read(wq, n * k, sink, 0, st)
        t_floor = time_graph(torch, floor_fn, 4 * len(ws_list))
        hbm_row(f"floor_stream_read_{n}x{k}", t_floor, n * k,
                {"l2": f"{len(ws_list)} rotating weight copies", "kernel": "bsq_debug_stream_read (read only)"})
        for m in ms:
            x = bf16_rand((m, k), 1.0)
            out = torch.empty((m, n), dtype=torch.int16, device=dev)
            it = [0]

            def f(st):
                wq, ws = ws_list[it[0] % len(ws_list)]
                it[0] += 1
                bsq.fp8_gemv_rowscale(x, wq, ws, out, m, n, k, st)
            t = time_graph(torch, f, 4 * len(ws_list))
            hbm_row(f"a4_fp8_gemv_m{m}_n{n}_k{k}", t, n * k + 4 * n + 2 * m * k + 2 * m * n,
                    {"l2": f"{len(ws_list)} rotating weight copies",
                     "frac_of_stream_read_floor": round(t_floor / t, 4)})
        del ws_list
        torch.cuda.empty_cache()

    def rotating(fn_of, inputs, reps_per_input=4):
        """fn(stream) cycling through the input copies."""
        it = [0]

        def f(st):
            fn_of(inputs[it[0] % len(inputs)], st)
            it[0] += 1
        return f, reps_per_input * len(inputs)

    # next row: block-scaled FP8 GEMV (w8a16_gemv_batch4 / _batch2), M = 1, 2, 4
    n, k = 5120, 5120

    def mk_bw():
        wq = torch.empty((n, k), dtype=torch.uint8, device=dev)
        S = torch.empty((n // 128, k // 128), dtype=torch.float32, device=dev)
        bsq.quant_blockfp8(bf16_rand((n, k), 0.02), wq, S, n, k, stream)
        return wq, S
    bw_list = rotate(mk_bw, n * k)
    for m in (1, 2, 4):
        x = bf16_rand((m, k), 1.0)
        out = torch.empty((m, n), dtype=torch.int16, device=dev)
        f, n_it = rotating(lambda ws, st: bsq.fp8_gemv_blockscaled(x, ws[0], ws[1], out, m, n, k, st), bw_list)
        t = time_graph(torch, f, n_it)
        hbm_row(f"next_fp8_gemv_blockscaled_m{m}_n{n}_k{k}", t,
                n * k + 4 * (n // 128) * (k // 128) + 2 * m * k + 2 * m * n,
                {"l2": f"{len(bw_list)} rotating weight copies"})
    del bw_list

    # a1: NVFP4 quantiser, 4096x5120 and 16384x5120 (inputs rotated past L2)
    for m in (4096, 16384):
        k = 5120
        a_list = rotate(lambda: bf16_rand((m, k), 1.0), m * k * 2)
        ap = torch.empty((m, k // 2), dtype=torch.uint8, device=dev)
        asf = torch.empty((m, k // 16), dtype=torch.uint8, device=dev)
        f, n_it = rotating(lambda a, st: bsq.quantize_bf16_to_nvfp4(a, ap, asf, 1.0, m, k, st), a_list)
        t = time_graph(torch, f, n_it)
        hbm_row(f"a1_quantize_bf16_to_nvfp4_{m}x{k}", t, m * k * 2 + m * k // 2 + m * k // 16,
                {"l2": f"{len(a_list)} rotating input copies"})
        del a_list

    # a2: W4A4 GEMM at M = 512 and 16384 (4096 is the headline step)
    n, k = 17408, 5120
    wp = torch.randint(0, 256, (n, k // 2), dtype=torch.uint8, device=dev, generator=g)
    wsf = torch.randint(0x30, 0x40, (n, k // 16), dtype=torch.uint8, device=dev, generator=g)
    for m in (512, 16384):
        ap = torch.randint(0, 256, (m, k // 2), dtype=torch.uint8, device=dev, generator=g)
        asf = torch.randint(0x30, 0x40, (m, k // 16), dtype=torch.uint8, device=dev, generator=g)
        out = torch.empty((m, n), dtype=torch.int16, device=dev)
        t = time_launches(torch, stream, lambda: bsq.w4a4_gemm(ap, asf, wp, wsf, out, 1.0, 1.0, m, n, k, stream), 10)
        tf = 2.0 * m * n * k / t / 1e12
        rows[f"a2_w4a4_gemm_m{m}"] = {"us": round(t * 1e6, 1), "tflops": round(tf, 1),
                                      "frac_fp4": round(tf / (bf16 * RATIO_FP4), 4), "bound": "tensor"}
        del ap, asf, out
    del wp, wsf
    # a2, few activation rows (swapped-operand kernel): the weight stream
    # (N*K/2 + N*K/16 bytes) is the cost; weight copies rotated past L2
    def mk_w4():
        return (torch.randint(0, 256, (n, k // 2), dtype=torch.uint8, device=dev, generator=g),
                torch.randint(0x30, 0x40, (n, k // 16), dtype=torch.uint8, device=dev, generator=g))
    w4_list = rotate(mk_w4, n * k // 2 + n * k // 16)
    for m in (1, 16, 128):
        ap = torch.randint(0, 256, (m, k // 2), dtype=torch.uint8, device=dev, generator=g)
        asf = torch.randint(0x30, 0x40, (m, k // 16), dtype=torch.uint8, device=dev, generator=g)
        out = torch.empty((m, n), dtype=torch.int16, device=dev)
        f, n_it = rotating(lambda w4, st: bsq.w4a4_gemm(ap, asf, w4[0], w4[1], out, 1.0, 1.0, m, n, k, st), w4_list)
        t = time_graph(torch, f, n_it)
        hbm_row(f"a2_w4a4_gemm_small_m{m}", t, n * k // 2 + n * k // 16 + m * k // 2 + m * k // 16 + 2 * m * n,
                {"tflops": round(2.0 * m * n * k / t / 1e12, 1), "l2": f"{len(w4_list)} rotating weight copies"})
        del ap, asf, out
    del w4_list

    # a3: row-wise FP8 quantiser (per-token activations of the FP8 projection)
    m, k = 8192, 5120
    a_list = rotate(lambda: bf16_rand((m, k), 1.0), m * k * 2)
    q = torch.empty((m, k), dtype=torch.uint8, device=dev)
    s = torch.empty((m,), dtype=torch.float32, device=dev)
    f, n_it = rotating(lambda a, st: bsq.quant_rowwise_fp8(a, q, s, m, k, st), a_list)
    t = time_graph(torch, f, n_it)
    hbm_row(f"a3_quant_rowwise_fp8_{m}x{k}", t, m * k * 3 + 4 * m, {"l2": f"{len(a_list)} rotating input copies"})
    a = a_list[0]
    bsq.quant_rowwise_fp8(a, q, s, m, k, stream)
    del a_list

    # a8: block FP8 -> row-wise FP8 requant (one-time weight conversion)
    n, k = 10240, 5120
    wsrc = bf16_rand((n, k), 0.02)

    def mk_block():
        wb = torch.empty((n, k), dtype=torch.uint8, device=dev)
        S = torch.empty((n // 128, k // 128), dtype=torch.float32, device=dev)
        bsq.quant_blockfp8(wsrc, wb, S, n, k, stream)
        return wb, S
    blk_list = rotate(mk_block, n * k)
    wr = torch.empty((n, k), dtype=torch.uint8, device=dev)
    sr = torch.empty((n,), dtype=torch.float32, device=dev)
    f, n_it = rotating(lambda b, st: bsq.requant_blockfp8_to_rowwise(
        bsq.BSQ_FP8_BLOCK_SCALED, b[0], b[1], n, k, wr, sr, st), blk_list)
    t = time_graph(torch, f, n_it)
    hbm_row(f"a8_requant_blockfp8_to_rowwise_{n}x{k}", t, 2 * n * k + 4 * n + 4 * (n // 128) * (k // 128),
            {"l2": f"{len(blk_list)} rotating input copies"})
    wb, S = blk_list[0]
    bsq.requant_blockfp8_to_rowwise(bsq.BSQ_FP8_BLOCK_SCALED, wb, S, n, k, wr, sr, stream)
    del blk_list

    # a9: row-scaled FP8 GEMM 8192 x 10240 x 5120
    m = 8192
    out = torch.empty((m, n), dtype=torch.int16, device=dev)
    t = time_launches(torch, stream, lambda: bsq.fp8_gemm_rowscale(q, s, wr, sr, out, m, n, k, stream), 10)
    tf = 2.0 * m * n * k / t / 1e12
    rows["a9_fp8_gemm_rowscale_8192x10240x5120"] = {"us": round(t * 1e6, 1), "tflops": round(tf, 1),
                                                    "frac_fp8": round(tf / (bf16 * RATIO_FP8), 4), "bound": "tensor"}
    del a, q, s, wsrc, wb, S, wr, sr, out

    # a5 / a6 / a7: the W4A8 int8 path
    n, k, m = 5120, 17408, 2048
    wsrc = bf16_rand((n, k), 0.02)

    def mk_nvfp4():
        wp = torch.empty((n, k // 2), dtype=torch.uint8, device=dev)
        wsf = torch.empty((n, k // 16), dtype=torch.uint8, device=dev)
        bsq.quantize_bf16_to_nvfp4(wsrc, wp, wsf, 1e-5, n, k, stream)
        return wp, wsf
    w_list = rotate(mk_nvfp4, n * k // 2)
    del wsrc
    wi = torch.empty((n, k), dtype=torch.int8, device=dev)
    wis = torch.empty((n, k // 32), dtype=torch.float32, device=dev)
    f, n_it = rotating(lambda wq, st: bsq.requant_w_nvfp4_int8(wq[0], wq[1], 1e-5, wi, wis, n, k, st), w_list, 2)
    t = time_graph(torch, f, n_it, reps=3)
    hbm_row(f"a5_requant_w_nvfp4_int8_{n}x{k}", t, n * k // 2 + n * k // 16 + n * k + n * k // 8,
            {"l2": f"{len(w_list)} rotating input copies"})
    wp, wsf = w_list[0]
    bsq.requant_w_nvfp4_int8(wp, wsf, 1e-5, wi, wis, n, k, stream)
    del w_list
    a_list = rotate(lambda: bf16_rand((m, k), 1.0), m * k * 2)
    ai = torch.empty((m, k), dtype=torch.int8, device=dev)
    ais = torch.empty((m, k // 32), dtype=torch.float32, device=dev)
    f, n_it = rotating(lambda a, st: bsq.quant_act_int8_per32(a, ai, ais, m, k, st), a_list)
    t = time_graph(torch, f, n_it)
    hbm_row(f"a6_quant_act_int8_per32_{m}x{k}", t, m * k * 3 + m * k // 8, {"l2": f"{len(a_list)} rotating input copies"})
    bsq.quant_act_int8_per32(a_list[0], ai, ais, m, k, stream)
    del a_list
    out = torch.empty((m, n), dtype=torch.int16, device=dev)
    t_plain = time_launches(torch, stream, lambda: bsq.int8_blockscaled_gemm(ai, wi, ais, wis, out, m, n, k, stream), 5)
    # the workspace form: the partial last round of tiles split along K
    ws_bytes = bsq.int8_gemm_workspace_bytes()
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    t = time_launches(torch, stream,
                      lambda: bsq.int8_blockscaled_gemm_ws(ai, wi, ais, wis, out, ws, ws_bytes, m, n, k, stream), 5)
    tops = 2.0 * m * n * k / t / 1e12
    # The fold's own roofline: two FP32 lane operations (the scale product and
    # the FMA) per output and 32-block, against every SM's 128 FP32 lanes at
    # the maximum SM clock; the int32 -> FP32 conversions run on the ALU pipe.
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    fold_peak = sms * 128 * SM_MAX_MHZ * 1e6
    fold_rate = 2.0 * m * n * (k // 32) / t
    rows[f"a7_int8_blockscaled_gemm_{m}x{n}x{k}"] = {
        "us": round(t * 1e6, 1), "tops": round(tops, 1), "frac_int8": round(tops / (bf16 * RATIO_INT8), 4),
        "fold_gops": round(fold_rate / 1e9, 1), "fold_peak_gops": round(fold_peak / 1e9, 1),
        "frac_fold": round(fold_rate / fold_peak, 4), "bound": "alu (per-32 FP32 fold on CUDA cores)",
        "call": "int8_blockscaled_gemm_ws (workspace split of the last round)",
        "us_without_workspace": round(t_plain * 1e6, 1)}
    return rows


# ---------------------------------------------------------- reference arm ---

def run_reference(args, w):
    """The CPU oracle, timed on a bounded sample of the workload: each step
    quantises S activation rows and computes their S x N outputs."""
    import oracle
    from int8_gemm_gemv_b200 import synth
    m, n, k = w["m"], w["n"], w["k"]
    threads = oracle.num_threads()
    sample = min(m, max(1, threads)) if args.workload != "tiny" else m
    a_bf, w_bf = synth.w4a4_inputs(m, n, k, seed=0, heavy_tailed=True)
    sb2 = float(np.float32(oracle.amax_bf16(w_bf)) / np.float32(6 * 448))
    wp, wsf = oracle.quant_nvfp4(w_bf, sb2)
    rows = np.arange(sample)

    def step():
        ap, asf = oracle.quant_nvfp4(a_bf[:sample], 1.0)
        oracle.w4a4_gemm(ap, asf, wp, wsf, 1.0, sb2)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    flops = 2.0 * sample * n * k
    value = flops * args.steps / dt / 1e12
    desc = f"{sample} of {m} activation rows per step (quantise + GEMM against all {n} weight rows)"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same seeded inputs as the GPU arm)",
        "config": {"workload": workload_desc(w), "m": m, "n": n, "k": k, "parallelism": "cpu oracle, rank 0"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def cpu_baseline_leg(w):
    """Bounded oracle timing reported beside the GPU line (rank 0, N=1)."""
    import oracle
    from int8_gemm_gemv_b200 import synth
    m, n, k = w["m"], w["n"], w["k"]
    threads = oracle.num_threads()
    sample = min(m, max(8, 16 * threads)) if m > 64 else m  # ~10 s of CPU work
    a_bf, w_bf = synth.w4a4_inputs(m, n, k, seed=0, heavy_tailed=True)
    sb2 = float(np.float32(oracle.amax_bf16(w_bf)) / np.float32(6 * 448))
    wp, wsf = oracle.quant_nvfp4(w_bf, sb2)
    t0 = time.perf_counter()
    ap, asf = oracle.quant_nvfp4(a_bf[:sample], 1.0)
    oracle.w4a4_gemm(ap, asf, wp, wsf, 1.0, sb2)
    dt = time.perf_counter() - t0
    return {"value": round(2.0 * sample * n * k / dt / 1e12, 6), "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{sample} of {m} activation rows (NVFP4 quantise + GEMM vs all {n} weight rows), "
                      f"{dt:.1f} s"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="bsq", choices=["bsq", "reference"])
    ap.add_argument("--workload", default="prefill", choices=sorted(WORKLOADS))
    ap.add_argument("--no-rows", dest="rows", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    rank, world, _ = rank_info()

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, w)), flush=True)
        return 0

    if args.warmup < 3:
        args.warmup = 3
    peaks, src = load_peaks()
    line, rank = run_bsq(args, w, peaks, src)
    if rank == 0 and world == 1 and args.cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_leg(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
