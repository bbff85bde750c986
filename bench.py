#!/usr/bin/env python
"""Benchmark of the NVFP4 quantized linear on B200 through the libbsp C ABI.

One step = one pass of the hot path over one batch: the NVFP4 activation quantizer
(bf16 -> E2M1 codes + E4M3 block-16 scales) followed by the block-scaled FP4 GEMM
with the fused alpha * acc + bias -> bf16 epilogue ("BFL (fp8r / nvfp4)", Kernels
table).  Default workload: the attention projection of a rectified-flow image
transformer at 1 MP (4096 tokens, 3072 -> 3072, bias).  Weights are quantized once
before timing (they are stored pre-quantized); the activation global scale is a
calibrated constant computed once.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events on the
launching stream, with the 126 MB L2 flushed (a 256 MiB write) before every step,
outside the events.  The step is one nvfp4_linear call (quantizer, then the GEMM
launched as its programmatic dependent) replayed from a CUDA graph; a second loop
times the two kernels separately, each from its own graph, for the per-kernel figures.
Barrier + synchronize around the timed loop; the per-rank total is reduced with MAX.
With N > 1 (torchrun), every rank runs an independent replica of the same workload
(the linear shards along tokens with no exchange): value = all ranks' FLOPs / max
time, "scaling": "weak".

`--impl reference` times the CPU oracle (oracle/) on a bounded sample of rows of
the same workload, on this host's cores; it is a deliberately slow correctness
reference, not a competing GPU implementation.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "NVFP4 GEMM TFLOPS & % of B200 FP4 peak; act-quantize GB/s & % of HBM"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def parse():
    p = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["bsp", "reference"], default="bsp")
    p.add_argument("--workload", default="nvfp4_attn_1mp")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--m", type=int, default=0,
                   help="token count (rows of A) instead of the workload's own, e.g. the fp8r "
                        "sweep 256 / 1024 / 16384")
    p.add_argument("--dynamic", action="store_true",
                   help="NVFP4: compute the activation global scale from each step's input "
                        "(nvfp4_linear_dynamic) instead of the calibrated constant")
    p.add_argument("--chain", nargs="?", const="fused", default=None,
                   choices=["fused", "unfused"],
                   help="MLP workloads: time the up projection, the re-quantization of its output "
                        "and the down projection as one step; 'fused' (default) re-quantizes in "
                        "the up projection's epilogue (nvfp4_gemm_quant), 'unfused' writes bf16 "
                        "and runs the quantizer on it")
    p.add_argument("--cpu-rows", type=int, default=2048,
                   help="rows of A in the CPU-oracle baseline sample")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def gemm_source_hash() -> str:
    h = hashlib.sha256()
    for name in ("gemm.cu", "bsp_ptx.cuh"):
        with open(os.path.join(ROOT, "block_scaled_precision_act_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """DRAM bytes per GEMM launch from the committed ncu summary, if it was taken on
    the current GEMM source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("source_hash") != gemm_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while the timed loop runs."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if self._h is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and bit != 0x1]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------- replicas (N > 1)
def max_over_ranks(value: float, device) -> float:
    """MAX of a per-rank timing over all ranks of the default process group (the value
    itself when there is no group or it has one rank).  Every rank must call it."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_tflops(flops_per_step: float, ms_per_step: float, world: int) -> float:
    """Whole-job throughput of `world` independent replicas, each doing `flops_per_step`
    per step, timed by the slowest rank's `ms_per_step`."""
    return world * flops_per_step / (ms_per_step * 1e-3) / 1e12


# ---------------------------------------------------------------------- CPU oracle
def cpu_oracle_sample(wl, rows: int, A=None, W=None):
    """Quantize `rows` rows of A and run the fp64 GEMM against the full weight with the
    oracle, as it stands.  Returns (seconds, flops, threads)."""
    import numpy as np
    import oracle
    import torch
    A = wl.A() if A is None else A
    W = wl.W() if W is None else W
    bias = wl.bias_vec()
    m_total = A.shape[0]
    rows = min(rows, m_total)
    idx = torch.from_numpy(np.linspace(0, m_total - 1, rows).astype(np.int64))
    a_rows = A[idx].contiguous()
    b = None if bias is None else bias.float().numpy().astype(np.float64)
    if wl.scheme == "nvfp4":
        gw = oracle.nvfp4_global_scale(W)
        wc, wsf = oracle.nvfp4_quantize(W, gw)          # offline weight prep, untimed
        ga = oracle.nvfp4_global_scale(A)               # calibrated input scale, untimed
        t0 = time.perf_counter()
        ac, asf = oracle.nvfp4_quantize(a_rows, ga)
        oracle.nvfp4_linear(ac, asf, ga, wc, wsf, gw, b)
    else:
        wq, ws = oracle.fp8r_quantize(W)                # offline weight prep, untimed
        t0 = time.perf_counter()
        aq, as_ = oracle.fp8r_quantize(a_rows)
        oracle.fp8r_linear(aq, as_, wq, ws, b)
    dt = time.perf_counter() - t0
    return dt, 2.0 * rows * wl.N * wl.K, oracle.default_threads()


def cpu_quantize_one_thread(wl, rows: int, A=None) -> dict:
    """The oracle's activation quantizer alone on one host thread, over `rows` rows of A
    (the workload's scheme; its algorithmic bytes per element as the GPU kernel's)."""
    import numpy as np
    import oracle
    import torch
    A = wl.A() if A is None else A
    rows = min(rows, A.shape[0])
    idx = torch.from_numpy(np.linspace(0, A.shape[0] - 1, rows).astype(np.int64))
    a_rows = A[idx].contiguous()
    if wl.scheme == "nvfp4":
        g = oracle.nvfp4_global_scale(A)
        t0 = time.perf_counter()
        oracle.nvfp4_quantize(a_rows, g, threads=1)
        per_elt = 2.5625
    else:
        t0 = time.perf_counter()
        oracle.fp8r_quantize(a_rows, threads=1)
        per_elt = 2.0 + 1.0 + 4.0 / a_rows.shape[1]
    dt = time.perf_counter() - t0
    return {"value": rows * a_rows.shape[1] * per_elt / dt / 1e9, "unit": "GB/s", "threads": 1,
            "rows": rows}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synth
    wl = synth.WORKLOADS[args.workload]
    M = args.m if args.m else wl.M
    A, W = (wl.A() if M == wl.M else wl.A_rows(M)), wl.W()
    # size each step's sample so the whole run stays within a few minutes
    dt, _, _ = cpu_oracle_sample(wl, 16, A, W)
    budget_s = 150.0 / max(1, args.steps + args.warmup)
    rows = int(max(8, min(1024, 16 * budget_s / max(dt, 1e-3))))
    for _ in range(args.warmup):
        cpu_oracle_sample(wl, rows, A, W)
    tot, flops, cores = 0.0, 0.0, 1
    for _ in range(args.steps):
        dt, fl, cores = cpu_oracle_sample(wl, rows, A, W)
        tot += dt
        flops += fl
    value = flops / tot / 1e12
    sample = (f"{rows} of {M} rows of A per step (quantize + fp64 GEMM against the "
              f"full {wl.N}x{wl.K} weight); weight quantization untimed")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "M": M, "N": wl.N, "K": wl.K, "bias": wl.bias,
                   "sample_rows": rows},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------- CUDA path
def run_bsp(args):
    import torch
    import torch.distributed as dist
    import synth
    import block_scaled_precision_act_b200 as bsp

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    wl = synth.WORKLOADS[args.workload]
    nvf4 = wl.scheme == "nvfp4"
    if args.chain and not wl.name.startswith("nvfp4_mlp"):
        raise SystemExit("--chain applies to the NVFP4 MLP workloads")
    M = args.m if args.m else wl.M
    N, K = wl.N, wl.K
    A_cpu = wl.A() if M == wl.M else wl.A_rows(M)
    A_host = A_cpu.pin_memory()
    A = A_cpu.to(dev)
    W = wl.W().to(dev)
    bias = wl.bias_vec()
    bias = None if bias is None else bias.to(dev)
    pk, pk_src = peaks()
    hbm = pk["hbm_gbs"]
    mm_peak = (4.0 if nvf4 else 2.0) * pk["bf16_tflops"]   # nominal dense fp4 / fp8 : bf16

    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    flush = torch.empty((L2_FLUSH_BYTES,), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    # per-kernel parts in step order: (name, fn, unit, algorithmic work per launch, peak)
    parts = []
    flops = 2.0 * M * N * K
    if nvf4:
        # untimed preparation: pre-quantized weights and a calibrated activation scale
        gw = bsp.nvfp4_global_scale(W)
        wc, wsf = bsp.nvfp4_quantize_act(W, gw, layout=bsp.SF_MMA)
        ga = bsp.nvfp4_global_scale(A)
        ac = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        asf = torch.empty((bsp.nvfp4_sf_bytes(M, K, bsp.SF_MMA),), dtype=torch.uint8, device=dev)
        ws = torch.empty((bsp.nvfp4_linear_workspace_bytes(M, max(K, N)),), dtype=torch.uint8,
                         device=dev)
        parts.append(("nvfp4_quantize_act", lambda: bsp.nvfp4_quantize_act(
            A, ga, codes=ac, scales=asf, layout=bsp.SF_MMA), "GB/s", M * K * 2.5625, hbm))
        parts.append(("nvfp4_gemm", lambda: bsp.nvfp4_gemm(
            ac, asf, ga, wc, wsf, gw, bias=bias, out=y), "TFLOP/s", flops, mm_peak))
        # the whole path in one call: quantizer, then the GEMM as its programmatic dependent
        step_fns = [lambda: bsp.nvfp4_linear(A, ga, wc, wsf, gw, bias=bias, out=y, workspace=ws)]
        if args.dynamic:
            gdyn = torch.empty((1,), dtype=torch.float32, device=dev)
            parts.insert(0, ("nvfp4_global_scale (dynamic)", lambda: bsp.nvfp4_global_scale(
                A, out=gdyn), "GB/s", M * K * 2.0, hbm))
            step_fns = [lambda: bsp.nvfp4_linear_dynamic(A, wc, wsf, gw, bias=bias, out=y,
                                                         input_scale_out=gdyn, workspace=ws)]
        y_out = y
        if args.chain:
            # MLP down projection on GEMM1's output: a6 re-quantizes it with a scale
            # calibrated (once, untimed) on that output, then GEMM2 [M, K] = Y1 . W2^T
            W2 = wl.W2().to(dev)
            g2w = bsp.nvfp4_global_scale(W2)
            w2c, w2sf = bsp.nvfp4_quantize_act(W2, g2w, layout=bsp.SF_MMA)
            step_fns[0]()
            g2 = bsp.nvfp4_global_scale(y)
            y1c = torch.empty((M, N // 2), dtype=torch.uint8, device=dev)
            y1sf = torch.empty((bsp.nvfp4_sf_bytes(M, N, bsp.SF_MMA),), dtype=torch.uint8,
                               device=dev)
            y2 = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
            gemm2 = ("nvfp4_gemm (down)", lambda: bsp.nvfp4_gemm(
                y1c, y1sf, g2, w2c, w2sf, g2w, out=y2), "TFLOP/s", 2.0 * M * K * N, mm_peak)
            if args.chain == "fused":
                # up projection with the re-quantization in its epilogue: no bf16 Y1
                up_q = ("nvfp4_gemm_quant (up + a6 in the epilogue)", lambda: bsp.nvfp4_gemm_quant(
                    ac, asf, ga, wc, wsf, gw, g2, bias=bias, out_codes=y1c, out_sf=y1sf),
                    "TFLOP/s", flops, mm_peak)
                parts[1] = up_q
                parts.append(gemm2)
                step_fns = [parts[0][1], up_q[1], gemm2[1]]
            else:
                parts.append(("nvfp4_quantize_act (a6, on GEMM1's output)", lambda: bsp.nvfp4_quantize_act(
                    y, g2, codes=y1c, scales=y1sf, layout=bsp.SF_MMA), "GB/s", M * N * 2.5625, hbm))
                parts.append(gemm2)
                step_fns.append(lambda: bsp.nvfp4_linear(y, g2, w2c, w2sf, g2w, out=y2,
                                                         workspace=ws))
            flops += 2.0 * M * K * N
            y_out = y2
    else:
        # untimed preparation: the weight quantized once per row
        wq, wsc = bsp.fp8r_quantize_rows(W)
        aq = torch.empty((M, K), dtype=torch.uint8, device=dev)
        asc = torch.empty((M,), dtype=torch.float32, device=dev)
        lin_ws = torch.empty((bsp.fp8r_linear_workspace_bytes(M, K),), dtype=torch.uint8,
                             device=dev)
        parts.append(("fp8r_quantize_rows", lambda: bsp.fp8r_quantize_rows(
            A, q=aq, row_scale=asc), "GB/s", M * K * 3.0 + 4.0 * M, hbm))
        parts.append(("fp8r_gemm", lambda: bsp.fp8r_gemm(
            aq, asc, wq, wsc, bias=bias, out=y), "TFLOP/s", flops, mm_peak))
        step_fns = [lambda: bsp.fp8r_linear(A, wq, wsc, bias=bias, out=y, workspace=lin_ws)]
        y_out = y
    y_host = torch.empty(tuple(y_out.shape), dtype=torch.bfloat16).pin_memory()

    def step():
        for f in step_fns:
            f()

    for p in parts:
        p[1]()
    step()
    torch.cuda.synchronize(dev)
    if bsp.bsp_last_device_status() != 0:
        raise SystemExit("device status not OK after the first step")
    graphs = [torch.cuda.CUDAGraph() for _ in parts]
    gs = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for g, p in zip(graphs, parts):
            with torch.cuda.graph(g, stream=side):
                p[1]()
        with torch.cuda.graph(gs, stream=side):
            step()
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)

    n_ev = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_ev)]
    for _ in range(args.warmup):
        flush.fill_(1)
        gs.replay()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local)
    with sampler:
        for i in range(args.steps):
            flush.fill_(1)
            ev[i][0].record(stream)
            gs.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        # per-kernel split (roofline of each kernel): the same kernels in step order,
        # each replayed from its own graph, the L2 flushed before each sequence
        kev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(parts) + 1)]
               for _ in range(n_ev)]
        for i in range(args.steps):
            flush.fill_(1)
            kev[i][0].record(stream)
            for j, g in enumerate(graphs):
                g.replay()
                kev[i][j + 1].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    s_ms = [e[0].elapsed_time(e[1]) for e in ev]
    total_ms = sum(s_ms)
    part_ms = [statistics.mean(e[j].elapsed_time(e[j + 1]) for e in kev)
               for j in range(len(parts))]
    total_ms = max_over_ranks(total_ms, dev)
    if bsp.bsp_last_device_status() != 0:
        raise SystemExit("device status not OK after the timed steps")
    if not torch.isfinite(y_out.float()).all():
        raise SystemExit("non-finite output")

    # end to end through the public API: pinned host A in, host Y out, every step
    e2e_steps = max(5, min(args.steps, 50))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    for i in range(e2e_steps + 2):
        if i == 2:
            e0.record(stream)
        A.copy_(A_host, non_blocking=True)
        step()
        y_host.copy_(y_out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dev)

    ms_per_step = total_ms / args.steps
    kernels = {}
    for (name, _, unit, work, peak), ms in zip(parts, part_ms):
        rate = work / (ms * 1e-3) / (1e9 if unit == "GB/s" else 1e12)
        kernels[name] = {"us": 1e3 * ms, unit: rate, "frac_peak": rate / peak, "peak": peak,
                         "work_per_launch": work}
    gname = next(p[0] for p in parts if p[2] == "TFLOP/s")
    gemm_tflops = kernels[gname]["TFLOP/s"]
    if nvf4:
        step_desc = ("nvfp4_linear = nvfp4_quantize_act + nvfp4_gemm (fused alpha, bias, bf16; "
                     "GEMM as programmatic dependent)")
        if args.dynamic:
            step_desc = "nvfp4_linear_dynamic = nvfp4_global_scale of the step's input + " + step_desc
        if args.chain == "fused":
            step_desc = ("nvfp4_quantize_act + nvfp4_gemm_quant (up projection, its output "
                         "re-quantized in the epilogue) + nvfp4_gemm (down projection), each "
                         "GEMM a programmatic dependent of the kernel before it")
        elif args.chain == "unfused":
            step_desc += "; then nvfp4_linear of GEMM1's bf16 output through the down projection"
    else:
        step_desc = ("fp8r_linear = fp8r_quantize_rows + fp8r_gemm (fused row scales, bias, bf16; "
                     "GEMM as programmatic dependent)")
    line = {
        "metric": METRIC,
        "value": replica_tflops(flops, ms_per_step, world),
        "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4" if nvf4 else "fp8_e4m3", "data": "synthetic",
        "config": {"workload": wl.name, "M": M, "N": N, "K": K, "bias": wl.bias,
                   "chain": args.chain, "step": step_desc + ", one CUDA graph",
                   "l2": "flushed before every step (256 MiB write, outside the events)",
                   "parallelism": "replicas" if world > 1 else "single"},
        "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": mm_peak,
                     "unit": "TFLOP/s", "frac": gemm_tflops / mm_peak,
                     "traffic": ncu_traffic(wl.name) if M == wl.M else None,
                     "kernel": gname,
                     "peak_source": f"{pk_src}: {4 if nvf4 else 2} x bf16 burst "
                                    f"{pk['bf16_tflops']} TFLOP/s (nominal dense "
                                    f"{'fp4' if nvf4 else 'fp8'}:bf16 = {4 if nvf4 else 2})"},
        "kernels": kernels,
        "e2e": {"value": replica_tflops(flops, e2e_ms, world), "unit": "TFLOP/s",
                "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": y_out.numel() * 2},
        "gpu_launches": len(parts) * args.steps,
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, fl, cores = cpu_oracle_sample(wl, args.cpu_rows, A_cpu)
        line["cpu_baseline"] = {
            "value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{min(args.cpu_rows, M)} of {M} rows of A: quantize + fp64 GEMM "
                      f"against the full weight ({dt:.1f} s)"
                      + ("; first linear of the chain only" if args.chain else ""),
            "quantize_one_thread": cpu_quantize_one_thread(wl, args.cpu_rows, A_cpu)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graphs, gs
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_bsp(args)


if __name__ == "__main__":
    sys.exit(main())
