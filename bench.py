#!/usr/bin/env python
"""Benchmark of the fused SVDQuant W4A4 linear (quantizer + block-scaled FP4 GEMM
with the rank-R epilogue) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one full forward of the layer (both kernels) on one batch of the
workload (default: the diffusion-transformer attention projection, M=4096,
K=N=3072, R=32, synthetic seeded inputs).  Prints one JSON line.

Timing: 8 replica sets (own weights, x, y, workspace) rotate so that the
working set (~0.5 GB) is far larger than the 126 MB L2 and every step reads
its inputs from HBM.  The K timed steps are one CUDA-graph replay bracketed by
CUDA events on the launching stream (barrier + synchronize on both sides);
per-kernel averages come from graphs of each stage alone over the same sets.
Multi-GPU (torchrun): independent replicas, one per rank, no collective on the
data path ("replicas only"); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FP4_PER_BF16 = 4.0          # nominal dense FP4 / BF16 tensor throughput ratio on B200 (9 / 2.25 PFLOP/s)
L2_BYTES = 126e6


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def flops_per_step(M, K, N, R):
    return 2.0 * M * N * K + 2.0 * M * K * R + 2.0 * M * N * R


def quant_bytes(M, K, R):
    # x read, codes + scales + L written, proj_down + smooth read (algorithmic).
    return 2.0 * M * K + M * K / 2 + M * K / 16 + 2.0 * M * R + 2.0 * K * R + 2.0 * K


def gemm_bytes(M, K, N, R):
    # codes + scales + L read, weights (codes + scales + proj_up + alpha) read, y written.
    return M * K / 2 + M * K / 16 + 2.0 * M * R + N * K / 2 + N * K / 16 + 2.0 * N * R + 4.0 * N + 2.0 * M * N


def gemm_roofline_bound(M, K, N, R, hbm_gbs, fp4_tflops):
    """The GEMM's roofline bound: "hbm" when its bytes at HBM bandwidth take
    longer than its flops at the FP4 peak (few rows: the weight read), else
    "tensor"."""
    flops = 2.0 * M * N * K + 2.0 * M * N * R
    return "hbm" if gemm_bytes(M, K, N, R) / (hbm_gbs * 1e9) > flops / (fp4_tflops * 1e12) else "tensor"


def source_digest(path):
    """sha256 over a kernel source and every local device header (.cuh) it
    includes, transitively, in first-seen order.  Headers of host-side
    declarations (.h: launch functions and their parameter structs) do not
    change a kernel's device code and are not followed."""
    seen, order = set(), []

    def walk(p):
        if p in seen or not os.path.exists(p):
            return
        seen.add(p)
        order.append(p)
        with open(p, "r", errors="replace") as f:
            for inc in re.findall(r'^\s*#\s*include\s+"([^"]+\.cuh)"', f.read(), re.M):
                walk(os.path.join(os.path.dirname(p), inc))

    walk(os.path.join(ROOT, path))
    h = hashlib.sha256()
    for p in order:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(workload, kernel):
    """DRAM bytes (read + write) per launch from the ncu capture recorded in
    profiles/traffic.json, or None when there is none or the kernel's source
    (its .cu file and the device headers it includes) has changed since."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[workload][kernel]
        if source_digest(rec["source"]) != rec["source_sha256"]:
            return None
        return rec["dram_bytes_per_launch"]
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = None
            try:
                uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            except Exception:
                pass
            h = None
            if uuid:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._nvml, self._h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None

    def _run(self):
        n = self._nvml
        names = {
            "hw_slowdown": getattr(n, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(n, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(n, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(n, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_power_brake_slowdown": getattr(n, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
                r = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for k, bit in names.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(0.0005)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples),
                "source": "nvml, 0.5 ms period, during the timed region"}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value):
    if world == 1:
        return value
    import torch.distributed as dist
    # NCCL reduces device tensors; gloo (the CPU test of this path) host ones.
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measure_fp4_peak(S, stream, local, iters=20000, seconds=1.0):
    """Dense block-scaled FP4 tensor rate of this GPU: one CTA per SM issuing
    back-to-back tcgen05 NVFP4 MMAs (128 x 256 x 64) from shared memory
    (svdq_fp4_mma_loop).  Burst: one launch of ~5 ms; sustained: back-to-back
    launches for about `seconds`, with the SM clock sampled meanwhile."""
    fl_per_iter = 4 * 2.0 * 128 * 256 * 64
    S.svdq_fp4_mma_loop(200, stream)
    torch.cuda.synchronize()

    def run(n):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        ctas = 0
        for _ in range(n):
            ctas = S.svdq_fp4_mma_loop(iters, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        return ctas * iters * n * fl_per_iter / (e0.elapsed_time(e1) * 1e-3) / 1e12, e0.elapsed_time(e1) * 1e-3

    burst = max(run(1)[0] for _ in range(3))
    _, t1 = run(1)
    n = max(1, int(seconds / max(t1, 1e-4)))
    with ClockSampler(local) as clk:
        sustained, _ = run(n)
    if S.svdq_fp4_mma_loop_status() != 0:
        raise SystemExit("FP4 rate loop: bounded wait expired")
    return {"burst_tflops": burst, "sustained_tflops": sustained, "clocks": clk.summary(),
            "how": f"svdq_fp4_mma_loop: one CTA per SM, {iters} x 4 tcgen05 NVFP4 MMAs (128 x 256 x 64) per CTA "
                   f"from shared memory; burst = best of 3 single launches, sustained = {n} launches back to back"}


def cpu_oracle_run(ck, rows):
    from oracle import svdq_oracle as O
    t0 = time.perf_counter()
    y = O.linear_forward(ck, rows=rows)
    dt = time.perf_counter() - t0
    return y, dt


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def run_reference(args, world, rank):
    """The oracle as it stands, timed on the host cores (bounded row sample per step)."""
    from bit_quantized_linear_svdq_b200 import synthetic
    if rank != 0:
        return
    ck = synthetic.load(args.workload)
    rows = np.arange(min(ck.M, args.ref_rows))
    cpu_oracle_run(ck, rows[: min(16, len(rows))])          # warm caches / BLAS threads
    times = []
    for _ in range(max(1, args.warmup if args.warmup < 3 else 1)):
        cpu_oracle_run(ck, rows)
    for _ in range(args.steps):
        _, dt = cpu_oracle_run(ck, rows)
        times.append(dt)
    t = sum(times) / len(times)
    fl = flops_per_step(len(rows), ck.K, ck.N, ck.R)
    value = fl / t / 1e12
    cores = cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(ck, extra={"sample_rows": len(rows)}),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{len(rows)} of {ck.M} token rows of the workload per step "
                                   f"(numpy fp64 GEMM over dequantized NVFP4 + fp32-emulated quantizer)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


METRIC = "W4A4+low-rank linear TFLOPS & % of dense-FP4 roofline at M=4096,K=N=3072,R=32"


def set_bytes(ck):
    """Device bytes one replica set touches per step: the layer's weights,
    x, the workspace (codes, scales, L) and y."""
    M, K, N, R = ck.M, ck.K, ck.N, ck.R
    weights = N * K // 2 + N * K // 16 + 2 * N * R + 2 * K * R + 2 * K + 4 * N
    return weights + 2 * M * K + (M * K // 2 + M * K // 16 + 2 * M * R) + 2 * M * N


def n_sets(ck):
    """Replica sets (each its own layer and inputs) to rotate over, so that
    consecutive steps' data together exceed twice the L2: at least 8."""
    return int(min(64, max(8, -(-2 * L2_BYTES // set_bytes(ck)))))


def config_of(ck, extra=None):
    ns = n_sets(ck)
    total = ns * set_bytes(ck)
    c = {"workload": ck.name, "M": ck.M, "K": ck.K, "N": ck.N, "R": ck.R, "rotate_block": ck.rotate_block,
         "l2": f"inputs and weights rotate over {ns} replica sets ({total / 1e6:.0f} MB) "
               + ("> 126 MB L2" if total > L2_BYTES else "(fits in the 126 MB L2)"),
         "parallelism": "replicas"}
    if extra:
        c.update(extra)
    return c


def run_ours(args, world, rank, local):
    import bit_quantized_linear_svdq_b200 as S
    from bit_quantized_linear_svdq_b200 import synthetic

    S.load_library()
    ck = synthetic.load(args.workload)
    M, K, N, R = ck.M, ck.K, ck.N, ck.R
    if ck.qweight is None:
        # A checkpoint that ships the dense weight: quantize it on the GPU.
        qw, wsc = S.quantize_weight(
            torch.from_numpy(np.ascontiguousarray(ck.dense_weight).view(np.int16)).view(torch.bfloat16).cuda(),
            ck.rotate_block)
        torch.cuda.synchronize()
        ck.qweight, ck.wscales = qw.cpu().numpy(), wsc.cpu().numpy()

    def dev(bits, dtype):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16 if dtype == torch.bfloat16 else np.uint8)) \
            .view(dtype).cuda()

    N_SETS = n_sets(ck)
    sets = []
    for i in range(N_SETS):
        layer = S.SVDQLinear(dev(ck.qweight, torch.uint8), dev(ck.wscales, torch.uint8),
                             dev(ck.proj_down, torch.bfloat16), dev(ck.proj_up, torch.bfloat16),
                             dev(ck.smooth_factor, torch.bfloat16), dev(ck.wcscales, torch.bfloat16),
                             dev(ck.wtscale, torch.bfloat16), rotate_block=ck.rotate_block)
        x = dev(ck.x, torch.bfloat16)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(S.svdq_workspace_bytes(layer.handle, M), dtype=torch.uint8, device="cuda")
        sets.append((layer, x, y, ws))
    stream = torch.cuda.Stream()
    variant = sets[0][0].gemm_kernel(M)

    def step(i, which="both"):
        # "both": the layer as a user calls it (svdq_linear_forward: the
        # quantizer, then the GEMM); "quant" / "gemm": each stage alone,
        # through the split entry points.
        layer, x, y, ws = sets[i % N_SETS]
        if which == "both":
            S.svdq_linear_forward(layer.handle, x.data_ptr(), M, y.data_ptr(), ws.data_ptr(), stream)
        if which == "quant":
            S.svdq_linear_forward_quantize(layer.handle, x.data_ptr(), M, ws.data_ptr(), stream)
        if which == "gemm":
            S.svdq_linear_forward_gemm(layer.handle, M, y.data_ptr(), ws.data_ptr(), stream)

    def graph_of(n, which):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for i in range(N_SETS):                 # eager pass: attributes set, sets initialised
                step(i, which)
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n):
                    step(i, which)
        return g

    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            step(i)
    torch.cuda.synchronize()
    g_full = graph_of(args.steps, "both")
    g_quant = graph_of(args.steps, "quant")
    g_gemm = graph_of(args.steps, "gemm")
    with torch.cuda.stream(stream):
        for g in (g_full, g_quant, g_gemm):    # graph warm-up replays
            g.replay()
    torch.cuda.synchronize()
    for lay, *_ in sets:
        if lay.device_status() != 0:
            raise SystemExit("device error flag set during warm-up")

    def timed(g):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):        # replay() launches on the current stream
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return e0.elapsed_time(e1) / 1e3

    with ClockSampler(local) as clk:
        t_full = timed(g_full)
    t_quant = timed(g_quant)
    t_gemm = timed(g_gemm)
    t_full_max = max_over_ranks(world, t_full)

    # The offline weight quantizer (svdq_quantize_weight) on this layer's
    # weight shape: seeded dense bf16 W ~ N(0, 0.02), one per replica set.
    gen = torch.Generator(device="cuda").manual_seed(7)
    wsets = []
    for i in range(N_SETS):
        w = (torch.randn((N, K), generator=gen, device="cuda") * 0.02).to(torch.bfloat16)
        wsets.append((w, torch.empty((N, K // 2), dtype=torch.uint8, device="cuda"),
                      torch.empty((K // 16, N), dtype=torch.uint8, device="cuda")))

    def wq(i):
        w, qw, wsc = wsets[i % N_SETS]
        S.svdq_quantize_weight(w.data_ptr(), N, K, ck.rotate_block, qw.data_ptr(), wsc.data_ptr(), stream)

    def graph_calls(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for i in range(N_SETS):
                fn(i)
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                for i in range(args.steps):
                    fn(i)
            g.replay()
        torch.cuda.synchronize()
        return g

    g_wq = graph_calls(wq)
    t_wq = timed(g_wq)
    del g_wq, wsets

    # The standalone Hadamard transform, in place on M rows of 4096 bf16.
    HN = 4096
    hsets = [torch.randn((M, HN), generator=gen, device="cuda").to(torch.bfloat16) for _ in range(N_SETS)]

    def ht(i):
        S.svdq_hadamard_transform(hsets[i % N_SETS].data_ptr(), M, HN, 0, stream)

    g_ht = graph_calls(ht)
    t_ht = timed(g_ht)
    del g_ht, hsets

    # The MXFP4 linear with a grouped Hadamard (the FP-Quant forward: fused
    # group-32 rotation + MXFP4 quantizer, then the MXFP4 GEMM) on this
    # layer's shape: seeded W ~ N(0, 0.02) quantized on the GPU, x ~ N(0, 1).
    msets = []
    for i in range(N_SETS):
        w = (torch.randn((N, K), generator=gen, device="cuda") * 0.02).to(torch.bfloat16)
        qw_m, ws_m = S.mxfp4_quantize(w, 32)
        lay_m = S.MXFP4Linear(qw_m, ws_m, alpha=1.0, hadamard_group=32)
        xm = torch.randn((M, K), generator=gen, device="cuda").to(torch.bfloat16)
        ym = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        msets.append((lay_m, xm, ym, lay_m.workspace(M)))
        del w, qw_m, ws_m

    def mxf(i):
        lay_m, xm, ym, wsm = msets[i % N_SETS]
        S.svdq_mxfp4_forward(lay_m.handle, xm.data_ptr(), M, ym.data_ptr(), wsm.data_ptr(), stream)

    g_mx = graph_calls(mxf)
    t_mx = timed(g_mx)
    del g_mx
    for lay_m, *_ in msets:
        if lay_m.device_status() != 0:
            raise SystemExit("device error flag set in the MXFP4 forward")
        lay_m.close()
    del msets

    # End-to-end through the host-buffer C ABI call: H2D of x, forward, D2H of y, sync.
    layer, x, y, ws = sets[0]
    xh = x.cpu().pin_memory()
    yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    for _ in range(2):
        S.svdq_linear_forward_host(layer.handle, xh.data_ptr(), M, yh.data_ptr(), x.data_ptr(), y.data_ptr(),
                                   ws.data_ptr(), stream)
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        S.svdq_linear_forward_host(layer.handle, xh.data_ptr(), M, yh.data_ptr(), x.data_ptr(), y.data_ptr(),
                                   ws.data_ptr(), stream)
    e1.record(stream)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(world, e0.elapsed_time(e1) / 1e3 / e2e_steps)
    for lay, *_ in sets:
        if lay.device_status() != 0:
            raise SystemExit("device error flag set during the timed region")

    fl = flops_per_step(M, K, N, R)
    value = world * fl * args.steps / t_full_max / 1e12
    pk = peaks()
    fp4_nominal = pk["bf16_tflops"] * FP4_PER_BF16
    fp4m = measure_fp4_peak(S, stream, local)
    fp4_peak = fp4m["burst_tflops"]
    us_q = t_quant / args.steps * 1e6
    us_g = t_gemm / args.steps * 1e6
    us_wq = t_wq / args.steps * 1e6
    us_ht = t_ht / args.steps * 1e6
    us_mx = t_mx / args.steps * 1e6
    ht_bytes = 2.0 * 2 * M * HN
    wq_bytes = 2.0 * N * K + N * K / 2 + N * K / 16
    q_gbs = quant_bytes(M, K, R) / (us_q * 1e-6) / 1e9
    g_flops = 2.0 * M * N * K + 2.0 * M * N * R
    g_tf = g_flops / (us_g * 1e-6) / 1e12
    # The GEMM's roofline bound: the slower of its flops at the FP4 peak and
    # its bytes at HBM bandwidth (few rows: the weight read).
    gemm_bound = gemm_roofline_bound(M, K, N, R, pk["hbm_gbs"], fp4_peak)
    kernels = {
        "quantize_act": {"us": us_q, "bound": "hbm", "algorithmic_bytes": quant_bytes(M, K, R),
                         "achieved_gbs": q_gbs, "frac_of_hbm": q_gbs / pk["hbm_gbs"],
                         "traffic": measured_traffic(ck.name, "quantize_act")},
        "quantize_weight": {"us": us_wq, "bound": "hbm", "algorithmic_bytes": wq_bytes,
                            "achieved_gbs": wq_bytes / (us_wq * 1e-6) / 1e9,
                            "frac_of_hbm": wq_bytes / (us_wq * 1e-6) / 1e9 / pk["hbm_gbs"],
                            "traffic": measured_traffic(ck.name, "quantize_weight"),
                            "note": "offline step (dense weight -> NVFP4), on this layer's weight shape"},
        "hadamard_transform": {"us": us_ht, "bound": "hbm", "algorithmic_bytes": ht_bytes,
                               "achieved_gbs": ht_bytes / (us_ht * 1e-6) / 1e9,
                               "frac_of_hbm": ht_bytes / (us_ht * 1e-6) / 1e9 / pk["hbm_gbs"],
                               "traffic": measured_traffic(ck.name, "hadamard_transform"),
                               "note": f"standalone transform, in place on {M} x {HN} bf16"},
        "mxfp4_forward": {"us": us_mx, "bound": "tensor", "algorithmic_flops": 2.0 * M * N * K,
                          "achieved_tflops": 2.0 * M * N * K / (us_mx * 1e-6) / 1e12,
                          "frac_of_fp4": 2.0 * M * N * K / (us_mx * 1e-6) / 1e12 / fp4_peak,
                          "note": "FP-Quant forward on this layer's shape: group-32 Hadamard + MXFP4 quantizer, "
                                  "then the MXFP4 GEMM (two launches), weights quantized on the GPU"},
        "gemm_nvfp4": {"us": us_g, "bound": gemm_bound, "variant": variant, "algorithmic_flops": g_flops,
                       "achieved_tflops": g_tf, "frac_of_fp4": g_tf / fp4_peak,
                       "algorithmic_bytes": gemm_bytes(M, K, N, R),
                       "achieved_gbs": gemm_bytes(M, K, N, R) / (us_g * 1e-6) / 1e9,
                       "frac_of_hbm": gemm_bytes(M, K, N, R) / (us_g * 1e-6) / 1e9 / pk["hbm_gbs"],
                       "traffic": measured_traffic(ck.name, "gemm_nvfp4")},
    }
    if us_g >= us_q and gemm_bound == "hbm":
        g_gbs = gemm_bytes(M, K, N, R) / (us_g * 1e-6) / 1e9
        roof = {"kernel": "gemm_nvfp4 (" + variant + ")", "bound": "hbm", "achieved": g_gbs, "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": g_gbs / pk["hbm_gbs"], "traffic": measured_traffic(ck.name, "gemm_nvfp4"),
                "peak_source": f"{pk['source']} copy bandwidth"}
    elif us_g >= us_q:
        roof = {"kernel": "gemm_nvfp4 (" + variant + ")", "bound": "tensor", "achieved": g_tf, "peak": fp4_peak,
                "unit": "TFLOP/s", "frac": g_tf / fp4_peak, "traffic": measured_traffic(ck.name, "gemm_nvfp4"),
                "peak_source": "measured FP4 burst: " + fp4m["how"],
                "frac_vs_bf16x4": g_tf / fp4_nominal,
                "peak_bf16x4": fp4_nominal,
                "peak_fp4_sustained": fp4m["sustained_tflops"]}
    else:
        roof = {"kernel": "quantize_act", "bound": "hbm", "achieved": q_gbs, "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": q_gbs / pk["hbm_gbs"], "traffic": measured_traffic(ck.name, "quantize_act"),
                "peak_source": f"{pk['source']} copy bandwidth"}
    step_us = t_full_max / args.steps * 1e6
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_us / 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4 (e2m1 x ue4m3/16) -> fp32 accumulate -> bf16", "data": "synthetic",
        "config": config_of(ck),
        "roofline": roof,
        "roofline_step": {"bound": "tensor", "achieved": fl / (step_us * 1e-6) / 1e12, "peak": fp4_peak,
                          "unit": "TFLOP/s", "frac": fl / (step_us * 1e-6) / 1e12 / fp4_peak,
                          "frac_vs_bf16x4": fl / (step_us * 1e-6) / 1e12 / fp4_nominal},
        "fp4_peak": fp4m,
        "kernels": kernels,
        "e2e": {"value": world * fl / t_e2e / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": 2 * M * K,
                "d2h_bytes_per_step": 2 * M * N, "ms_per_step": t_e2e * 1e3,
                "path": "svdq_linear_forward_host (pinned host x/y)"},
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_oracle_run(ck, np.arange(16))
        dts = [cpu_oracle_run(ck, None)[1] for _ in range(max(1, args.cpu_reps))]
        dt = statistics.median(dts)
        line["cpu_baseline"] = {"value": flops_per_step(M, K, N, R) / dt / 1e12, "unit": "TFLOP/s",
                                "cores": cpu_threads(), "kind": "oracle", "seconds": sum(dts),
                                "sample": f"the whole workload ({M} token rows), median of {len(dts)} runs"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    for lay, *_ in sets:
        lay.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=None)
    ap.add_argument("--ref-rows", type=int, default=256,
                    help="token rows of the workload the reference arm (CPU oracle) runs per step")
    ap.add_argument("--cpu-reps", type=int, default=3,
                    help="full-workload oracle runs timed for cpu_baseline (median)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from bit_quantized_linear_svdq_b200 import synthetic
    if args.workload is None:
        args.workload = synthetic.HEADLINE
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup()
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
