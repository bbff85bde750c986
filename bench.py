#!/usr/bin/env python
"""Benchmark of the NVFP4 quantized linear on B200 through the libbsp C ABI.

One step = one pass of the hot path over one batch: the NVFP4 activation quantizer
(bf16 -> E2M1 codes + E4M3 block-16 scales) followed by the block-scaled FP4 GEMM
with the fused alpha * acc + bias -> bf16 epilogue ("BFL (fp8r / nvfp4)", Kernels
table).  Default workload: the attention projection of a rectified-flow image
transformer at 1 MP (4096 tokens, 3072 -> 3072, bias).  Weights are quantized once
before timing (they are stored pre-quantized); the activation global scale is a
calibrated constant computed once.

Timing: W untimed warm-up steps, then EXACTLY K steps captured in one CUDA graph and
replayed between one pair of CUDA events on the launching stream (barrier +
synchronize on both sides).  Step i works on operand set i mod R (activations, weights,
output, workspace); the R sets together hold more than twice the 126 MB L2, so no step
finds its operands in L2.  The per-kernel figures (and the roofline) are taken the same
way, each kernel alone; the isolated figures beside them time one launch per event pair
with the L2 flushed before it, which adds the ~6 us fixed cost of an event pair around a
graph replay.  A default run also measures the suite's other workloads (`configs`: the
4K quantizer and GEMMs, the 1 MP MLP chain fused and unfused, the fp8r token sweep, the
tiny case) under the same clock record.
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
    p.add_argument("--no-configs", action="store_true",
                   help="skip the other workloads of the suite (the `configs` key)")
    p.add_argument("--m", type=int, default=0,
                   help="token count (rows of A) instead of the workload's own, e.g. the fp8r "
                        "sweep 256 / 1024 / 16384")
    p.add_argument("--dynamic", action="store_true",
                   help="NVFP4: compute the activation global scale from each step's input "
                        "(nvfp4_linear_dynamic) instead of the calibrated constant")
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
class Timer:
    """Device timing on the launching stream.

    back_to_back(): n calls captured in ONE CUDA graph and replayed between one pair of
    CUDA events; call i works on operand set i mod len(sets).  The sets together hold
    more than twice the L2, so no call finds its operands in L2 (each was last touched
    len(sets) - 1 calls earlier), and the ~6 us that an event pair around a graph replay
    costs on this machine is paid once per n calls instead of once per call.
    isolated(): one call per graph replay, the L2 flushed (a 256 MiB write) before it,
    outside the events: the per-launch figure with that fixed cost included."""

    def __init__(self, dev, stream):
        import torch
        self.torch = torch
        self.dev, self.stream = dev, stream
        self.side = torch.cuda.Stream(dev)
        self.flush = torch.empty((L2_FLUSH_BYTES,), dtype=torch.uint8, device=dev)
        self.launches = 0          # library kernels launched inside timed regions

    def graph(self, calls):
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        self.side.wait_stream(self.stream)
        with torch.cuda.stream(self.side):
            with torch.cuda.graph(g, stream=self.side):
                for c in calls:
                    c()
        self.stream.wait_stream(self.side)
        torch.cuda.synchronize(self.dev)
        return g

    def upload(self, g):
        """Upload an instantiated graph to the device before it is timed: the first launch
        of a graph otherwise includes the upload, inside the events."""
        import ctypes
        torch = self.torch
        cu = ctypes.CDLL("libcuda.so.1")
        cu.cuGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        r = cu.cuGraphUpload(ctypes.c_void_p(g.raw_cuda_graph_exec()),
                             ctypes.c_void_p(self.stream.cuda_stream))
        if r != 0:
            raise RuntimeError(f"cuGraphUpload failed ({r})")
        torch.cuda.synchronize(self.dev)

    def _replay_timed(self, g):
        torch = self.torch
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        g.replay()
        e1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        return e0.elapsed_time(e1)

    def back_to_back(self, call, sets, n, warmup, kernels_per_call, reps=1):
        """ms per call: median over `reps` replays of a graph of n calls."""
        torch = self.torch
        calls = [(lambda st=sets[i % len(sets)]: call(st)) for i in range(n)]
        g = self.graph(calls)
        gw = self.graph([(lambda st=sets[i % len(sets)]: call(st)) for i in range(warmup)]) \
            if warmup > 0 else None
        if gw is not None:
            gw.replay()
        self.upload(g)
        ts = []
        for _ in range(reps):
            ts.append(self._replay_timed(g) / n)
            self.launches += n * kernels_per_call
        del g, gw
        return statistics.median(ts)

    def isolated(self, call, n, kernels_per_call):
        torch = self.torch
        g = self.graph([call])
        g.replay()
        torch.cuda.synchronize(self.dev)
        ts = []
        for _ in range(n):
            self.flush.fill_(1)
            ts.append(self._replay_timed(g))
            self.launches += kernels_per_call
        del g
        return statistics.mean(ts)


def n_sets(set_bytes: float, l2_bytes: int) -> int:
    """Operand sets for back-to-back timing: together more than twice the L2."""
    return max(2, int(2.0 * l2_bytes // max(set_bytes, 1.0)) + 1)


def rate(work: float, ms: float, unit: str) -> float:
    return work / (ms * 1e-3) / (1e9 if unit == "GB/s" else 1e12)


def entry(ms: float, unit: str, work: float, peak: float, method: str, **extra) -> dict:
    r = rate(work, ms, unit)
    d = {"us": 1e3 * ms, unit: r, "frac_peak": r / peak, "peak": peak,
         "work_per_launch": work, "timing": method}
    d.update(extra)
    return d


B2B = "back_to_back"
ISO = "isolated_l2_flushed"


def nvfp4_prepared(bsp, torch, W, dev):
    gw = bsp.nvfp4_global_scale(W)
    wc, wsf = bsp.nvfp4_quantize_act(W, gw, layout=bsp.SF_MMA)
    return wc, wsf, gw


def measure_configs(args, bsp, torch, T: Timer, dev, l2: int, hbm: float, fp4_peak: float,
                    fp8_peak: float) -> dict:
    """The other workloads of the benchmark suite, measured in the same run (same clock
    record): 4K quantizer and GEMMs, the 1 MP MLP chain fused and unfused, the fp8r token
    sweep, the tiny case.  Every figure is back-to-back (see Timer)."""
    import synth
    n, w = args.steps, args.warmup
    out = {}

    # ---- 4K output: 65536 tokens (quantizer headline of the suite, and its GEMMs)
    wl = synth.WORKLOADS["nvfp4_4k"]
    M, K = wl.M, wl.K
    A = wl.A().to(dev)
    ga = bsp.nvfp4_global_scale(A)
    qsets = [(A if i == 0 else A.clone(), torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
              torch.empty((bsp.nvfp4_sf_bytes(M, K),), dtype=torch.uint8, device=dev))
             for i in range(2)]
    qcall = lambda st: bsp.nvfp4_quantize_act(st[0], ga, codes=st[1], scales=st[2])
    ms = T.back_to_back(qcall, qsets, n, w, 1, reps=3)
    out["nvfp4_4k.quantize_act"] = entry(ms, "GB/s", M * K * 2.5625, hbm, B2B,
                                        shape=[M, K])
    ac, asf = qsets[0][1], qsets[0][2]
    del qsets
    for name, Wt in (("nvfp4_4k.gemm", wl.W()), ("nvfp4_4k_up.gemm",
                                                 synth.WORKLOADS["nvfp4_4k_up"].W())):
        Wd = Wt.to(dev)
        N = Wd.shape[0]
        wc, wsf, gw = nvfp4_prepared(bsp, torch, Wd, dev)
        gsets = [(ac if i == 0 else ac.clone(), asf if i == 0 else asf.clone(), wc, wsf,
                  torch.empty((M, N), dtype=torch.bfloat16, device=dev)) for i in range(2)]
        gcall = lambda st, gw=gw: bsp.nvfp4_gemm(st[0], st[1], ga, st[2], st[3], gw, out=st[4])
        ms = T.back_to_back(gcall, gsets, n, w, 1, reps=3)
        out[name] = entry(ms, "TFLOP/s", 2.0 * M * N * K, fp4_peak, B2B, shape=[M, N, K])
        del gsets, Wd, wc, wsf
    del A, ac, asf
    torch.cuda.empty_cache()

    # ---- MLP pair at 1 MP: up 3072 -> 12288, re-quantization, down 12288 -> 3072
    wl = synth.WORKLOADS["nvfp4_mlp_1mp"]
    M, K, N = wl.M, wl.K, wl.N
    A = wl.A().to(dev)
    ga = bsp.nvfp4_global_scale(A)
    W1, W2 = wl.W().to(dev), wl.W2().to(dev)
    w1c, w1sf, g1 = nvfp4_prepared(bsp, torch, W1, dev)
    w2c, w2sf, g2w = nvfp4_prepared(bsp, torch, W2, dev)
    y1 = bsp.nvfp4_linear(A, ga, w1c, w1sf, g1)
    g2 = bsp.nvfp4_global_scale(y1)          # calibrated once on GEMM1's output, untimed
    set_bytes = M * K * 2 * 2 + M * N * 2 + M * N // 2 + (N * K) * 2 * 0.5625
    R = n_sets(set_bytes, l2)

    def mlp_set(i):
        return dict(A=A if i == 0 else A.clone(),
                    ac=torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
                    asf=torch.empty((bsp.nvfp4_sf_bytes(M, K),), dtype=torch.uint8, device=dev),
                    w1c=w1c if i == 0 else w1c.clone(), w1sf=w1sf if i == 0 else w1sf.clone(),
                    w2c=w2c if i == 0 else w2c.clone(), w2sf=w2sf if i == 0 else w2sf.clone(),
                    y1=torch.empty((M, N), dtype=torch.bfloat16, device=dev),
                    y1c=torch.empty((M, N // 2), dtype=torch.uint8, device=dev),
                    y1sf=torch.empty((bsp.nvfp4_sf_bytes(M, N),), dtype=torch.uint8, device=dev),
                    y2=torch.empty((M, K), dtype=torch.bfloat16, device=dev),
                    ws=torch.empty((bsp.nvfp4_linear_workspace_bytes(M, max(K, N)),),
                                   dtype=torch.uint8, device=dev))
    msets = [mlp_set(i) for i in range(R)]

    def fused(st):
        bsp.nvfp4_quantize_act(st["A"], ga, codes=st["ac"], scales=st["asf"])
        bsp.nvfp4_gemm_quant(st["ac"], st["asf"], ga, st["w1c"], st["w1sf"], g1, g2,
                             out_codes=st["y1c"], out_sf=st["y1sf"])
        bsp.nvfp4_gemm(st["y1c"], st["y1sf"], g2, st["w2c"], st["w2sf"], g2w, out=st["y2"])

    def unfused(st):
        bsp.nvfp4_linear(st["A"], ga, st["w1c"], st["w1sf"], g1, out=st["y1"], workspace=st["ws"])
        bsp.nvfp4_linear(st["y1"], g2, st["w2c"], st["w2sf"], g2w, out=st["y2"],
                         workspace=st["ws"])

    flops = 2.0 * 2.0 * M * N * K
    ms = T.back_to_back(fused, msets, n, w, 3, reps=3)
    out["nvfp4_mlp_1mp.step_fused"] = entry(ms, "TFLOP/s", flops, fp4_peak, B2B, sets=R,
                                           step="quantize + gemm_quant (up, a6 in the epilogue) "
                                                "+ gemm (down)")
    ms = T.back_to_back(unfused, msets, n, w, 4, reps=3)
    out["nvfp4_mlp_1mp.step_unfused"] = entry(ms, "TFLOP/s", flops, fp4_peak, B2B, sets=R,
                                             step="nvfp4_linear (up) + nvfp4_linear (down)")
    for st in msets:
        bsp.nvfp4_quantize_act(st["A"], ga, codes=st["ac"], scales=st["asf"])
        bsp.nvfp4_quantize_act(y1, g2, codes=st["y1c"], scales=st["y1sf"])
    ms = T.back_to_back(lambda st: bsp.nvfp4_gemm_quant(
        st["ac"], st["asf"], ga, st["w1c"], st["w1sf"], g1, g2, out_codes=st["y1c"],
        out_sf=st["y1sf"]), msets, n, w, 1, reps=3)
    out["nvfp4_mlp_1mp.gemm_quant_up"] = entry(ms, "TFLOP/s", 2.0 * M * N * K, fp4_peak, B2B)
    ms = T.back_to_back(lambda st: bsp.nvfp4_gemm(
        st["y1c"], st["y1sf"], g2, st["w2c"], st["w2sf"], g2w, out=st["y2"]), msets, n, w, 1,
        reps=3)
    out["nvfp4_mlp_1mp.gemm_down"] = entry(ms, "TFLOP/s", 2.0 * M * N * K, fp4_peak, B2B)
    del msets, A, W1, W2, y1
    torch.cuda.empty_cache()

    # ---- fp8r: tokens M in {256, 1024, 4096, 16384}, 3072 -> 3072
    wl = synth.WORKLOADS["fp8r_1mp"]
    K, N = wl.K, wl.N
    W = wl.W().to(dev)
    wq, wsc = bsp.fp8r_quantize_rows(W)
    for M in synth.FP8R_M_SWEEP:
        A = wl.A_rows(M).to(dev)
        aq, asc = bsp.fp8r_quantize_rows(A)
        gemm_bytes = M * K + 4 * M + N * K + 4 * N + M * N * 2
        R = n_sets(gemm_bytes, l2)
        fsets = [(aq if i == 0 else aq.clone(), asc if i == 0 else asc.clone(),
                  wq if i == 0 else wq.clone(), wsc if i == 0 else wsc.clone(),
                  torch.empty((M, N), dtype=torch.bfloat16, device=dev)) for i in range(R)]
        ms = T.back_to_back(lambda st: bsp.fp8r_gemm(st[0], st[1], st[2], st[3], out=st[4]),
                            fsets, n, w, 1, reps=3)
        e = entry(ms, "TFLOP/s", 2.0 * M * N * K, fp8_peak, B2B, sets=R)
        # against the HBM roofline too: at few tokens the GEMM is bound by its bytes
        hbm_us = gemm_bytes / (hbm * 1e9) * 1e6
        e["algorithmic_bytes"] = gemm_bytes
        e["hbm_roofline_us"] = hbm_us
        e["frac_hbm_roofline"] = hbm_us / e["us"]
        out[f"fp8r_1mp.gemm_M{M}"] = e
        if M == wl.M:
            qsets = [(A if i == 0 else A.clone(), torch.empty((M, K), dtype=torch.uint8, device=dev),
                      torch.empty((M,), dtype=torch.float32, device=dev))
                     for i in range(n_sets(M * K * 3.0, l2))]
            ms = T.back_to_back(lambda st: bsp.fp8r_quantize_rows(st[0], q=st[1], row_scale=st[2]),
                                qsets, n, w, 1, reps=3)
            out["fp8r_1mp.quantize_rows"] = entry(ms, "GB/s", M * K * 3.0 + 4.0 * M, hbm, B2B)
            lsets = [(qs[0], torch.empty((M, N), dtype=torch.bfloat16, device=dev),
                      torch.empty((bsp.fp8r_linear_workspace_bytes(M, K),), dtype=torch.uint8,
                                  device=dev)) for qs in qsets]
            ms = T.back_to_back(lambda st: bsp.fp8r_linear(st[0], wq, wsc, out=st[1],
                                                           workspace=st[2]),
                                lsets, n, w, 2, reps=3)
            out["fp8r_1mp.step"] = entry(ms, "TFLOP/s", 2.0 * M * N * K, fp8_peak, B2B)
            del qsets, lsets
        del fsets, A, aq, asc
    del W, wq, wsc
    torch.cuda.empty_cache()

    # ---- tiny: 128 x 256 x 256, a latency figure (one quantizer + one GEMM)
    wl = synth.WORKLOADS["nvfp4_tiny"]
    A, W = wl.A().to(dev), wl.W().to(dev)
    ga = bsp.nvfp4_global_scale(A)
    wc, wsf, gw = nvfp4_prepared(bsp, torch, W, dev)
    y = torch.empty((wl.M, wl.N), dtype=torch.bfloat16, device=dev)
    ws = torch.empty((bsp.nvfp4_linear_workspace_bytes(wl.M, wl.K),), dtype=torch.uint8,
                     device=dev)
    ms = T.back_to_back(lambda st: bsp.nvfp4_linear(A, ga, wc, wsf, gw, out=y, workspace=ws),
                        [None], n, w, 2, reps=3)
    out["nvfp4_tiny.step"] = entry(ms, "TFLOP/s", 2.0 * wl.M * wl.N * wl.K, fp4_peak, B2B,
                                   note="launch-latency bound; operands stay in L2")
    return out


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
    fp4_peak, fp8_peak = 4.0 * pk["bf16_tflops"], 2.0 * pk["bf16_tflops"]
    mm_peak = fp4_peak if nvf4 else fp8_peak     # nominal dense fp4 / fp8 : bf16
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    stream = torch.cuda.current_stream(dev)
    T = Timer(dev, stream)

    # One operand set per step: activations in, weights, output, workspace.  Every set
    # holds valid quantized weights (copies of the prepared ones), so each step is one
    # whole, different linear.
    flops = 2.0 * M * N * K
    if nvf4:
        # untimed preparation: pre-quantized weights and a calibrated activation scale
        wc, wsf, gw = nvfp4_prepared(bsp, torch, W, dev)
        ga = bsp.nvfp4_global_scale(A)
        wsb = bsp.nvfp4_linear_workspace_bytes(M, max(K, N))
        set_bytes = M * K * 2 + M * N * 2 + wsb + N * K * 0.5625
    else:
        wq, wsc = bsp.fp8r_quantize_rows(W)
        wsb = bsp.fp8r_linear_workspace_bytes(M, K)
        set_bytes = M * K * 2 + M * N * 2 + wsb + N * K
    R = n_sets(set_bytes, l2)

    def make_set(i):
        st = {"A": A if i == 0 else A.clone(),
              "y": torch.empty((M, N), dtype=torch.bfloat16, device=dev),
              "ws": torch.empty((wsb,), dtype=torch.uint8, device=dev)}
        if nvf4:
            st.update(wc=wc if i == 0 else wc.clone(), wsf=wsf if i == 0 else wsf.clone(),
                      ac=torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
                      asf=torch.empty((bsp.nvfp4_sf_bytes(M, K),), dtype=torch.uint8, device=dev))
        else:
            st.update(wq=wq if i == 0 else wq.clone(), wsc=wsc if i == 0 else wsc.clone(),
                      aq=torch.empty((M, K), dtype=torch.uint8, device=dev),
                      asc=torch.empty((M,), dtype=torch.float32, device=dev))
        return st

    sets = [make_set(i) for i in range(R)]
    gdyn = torch.empty((1,), dtype=torch.float32, device=dev)
    if nvf4 and args.dynamic:
        step_call = lambda st: bsp.nvfp4_linear_dynamic(st["A"], st["wc"], st["wsf"], gw,
                                                        bias=bias, out=st["y"],
                                                        input_scale_out=gdyn, workspace=st["ws"])
        step_kernels = 3
    elif nvf4:
        step_call = lambda st: bsp.nvfp4_linear(st["A"], ga, st["wc"], st["wsf"], gw, bias=bias,
                                                out=st["y"], workspace=st["ws"])
        step_kernels = 2
    else:
        step_call = lambda st: bsp.fp8r_linear(st["A"], st["wq"], st["wsc"], bias=bias,
                                               out=st["y"], workspace=st["ws"])
        step_kernels = 2
    # per-kernel parts of the step: (name, call on a set, unit, work per launch, peak)
    if nvf4:
        parts = [("nvfp4_quantize_act", lambda st: bsp.nvfp4_quantize_act(
                     st["A"], ga, codes=st["ac"], scales=st["asf"]), "GB/s", M * K * 2.5625, hbm),
                 ("nvfp4_gemm", lambda st: bsp.nvfp4_gemm(
                     st["ac"], st["asf"], ga, st["wc"], st["wsf"], gw, bias=bias, out=st["y"]),
                  "TFLOP/s", flops, mm_peak)]
    else:
        parts = [("fp8r_quantize_rows", lambda st: bsp.fp8r_quantize_rows(
                     st["A"], q=st["aq"], row_scale=st["asc"]), "GB/s", M * K * 3.0 + 4.0 * M, hbm),
                 ("fp8r_gemm", lambda st: bsp.fp8r_gemm(
                     st["aq"], st["asc"], st["wq"], st["wsc"], bias=bias, out=st["y"]),
                  "TFLOP/s", flops, mm_peak)]
    for st in sets:                      # every set's quantized activations exist
        parts[0][1](st)
        step_call(st)
    torch.cuda.synchronize(dev)
    if bsp.bsp_last_device_status() != 0:
        raise SystemExit("device status not OK after the first step")

    # ---- the timed steps: W warm-up steps, then EXACTLY K steps back to back
    calls = [(lambda st=sets[i % R]: step_call(st)) for i in range(args.steps)]
    g_timed = T.graph(calls)
    g_warm = T.graph([(lambda st=sets[i % R]: step_call(st)) for i in range(args.warmup)]) \
        if args.warmup > 0 else None
    T.upload(g_timed)
    sampler = ClockSampler(local)
    with sampler:
        if g_warm is not None:
            g_warm.replay()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g_timed.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        total_ms = e0.elapsed_time(e1)
        T.launches += step_kernels * args.steps
        # the same step in isolation (one replay, L2 flushed before it): includes the
        # fixed cost of an event pair around a replay
        iso_step_ms = T.isolated(lambda: step_call(sets[0]), max(3, args.steps // 2),
                                 step_kernels)
        # per-kernel split, back to back over the rotating sets and in isolation
        kernels = {}
        for name, call, unit, work, peak in parts:
            ms_b = T.back_to_back(call, sets, args.steps, args.warmup, 1, reps=3)
            ms_i = T.isolated(lambda call=call: call(sets[0]), max(3, args.steps // 2), 1)
            kernels[name] = entry(ms_b, unit, work, peak, B2B, sets=R)
            kernels[name]["isolated"] = entry(ms_i, unit, work, peak, ISO)
        configs = None
        if rank == 0 and world == 1 and args.workload == "nvfp4_attn_1mp" and not args.m \
                and not args.dynamic and not args.no_configs:
            configs = measure_configs(args, bsp, torch, T, dev, l2, hbm, fp4_peak, fp8_peak)
    total_ms = max_over_ranks(total_ms, dev)
    if bsp.bsp_last_device_status() != 0:
        raise SystemExit("device status not OK after the timed steps")
    y_out = sets[0]["y"]
    if not torch.isfinite(y_out.float()).all():
        raise SystemExit("non-finite output")
    del g_timed, g_warm

    # ---- end to end through the public API: pinned host A in, host Y out, every step
    y_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    st0 = sets[0]
    e2e_steps = max(5, min(args.steps, 50))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    for i in range(e2e_steps + 2):
        if i == 2:
            e0.record(stream)
        st0["A"].copy_(A_host, non_blocking=True)
        step_call(st0)
        y_host.copy_(st0["y"], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dev)

    ms_per_step = total_ms / args.steps
    gname = parts[1][0]
    g = kernels[gname]
    gemm_rate = g["TFLOP/s"]
    if nvf4:
        step_desc = ("nvfp4_linear = nvfp4_quantize_act + nvfp4_gemm (fused alpha, bias, bf16; "
                     "GEMM as programmatic dependent)")
        if args.dynamic:
            step_desc = "nvfp4_linear_dynamic = nvfp4_global_scale of the step's input + " + step_desc
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
                   "step": step_desc + "; the K timed steps are one CUDA graph between one "
                                       "event pair",
                   "l2": (f"inputs larger than L2: step i uses operand set i mod {R} "
                          f"({R} sets of {set_bytes / 2**20:.0f} MiB: activations, weights, "
                          f"output, workspace; > 2 x the {l2 / 2**20:.0f} MiB L2), so no step "
                          f"finds its operands in L2"),
                   "parallelism": "replicas" if world > 1 else "single"},
        "ms_per_step_isolated": iso_step_ms,
        "roofline": {"bound": "tensor", "achieved": gemm_rate, "peak": mm_peak,
                     "unit": "TFLOP/s", "frac": gemm_rate / mm_peak,
                     "traffic": ncu_traffic(wl.name) if M == wl.M else None,
                     "kernel": gname,
                     "timing": (f"{args.steps} launches back to back in one CUDA graph over "
                                f"{R} rotating operand sets (no launch finds its operands in "
                                f"L2), divided by {args.steps}; the isolated single-launch "
                                f"figure (L2 flushed, one event pair) is in kernels"),
                     "peak_source": f"{pk_src}: {4 if nvf4 else 2} x bf16 burst "
                                    f"{pk['bf16_tflops']} TFLOP/s (nominal dense "
                                    f"{'fp4' if nvf4 else 'fp8'}:bf16 = {4 if nvf4 else 2})"},
        "kernels": kernels,
        "e2e": {"value": replica_tflops(flops, e2e_ms, world), "unit": "TFLOP/s",
                "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2},
        "gpu_launches": T.launches,
        "clocks": sampler.summary(),
    }
    if configs is not None:
        line["configs"] = configs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, fl, cores = cpu_oracle_sample(wl, args.cpu_rows, A_cpu)
        line["cpu_baseline"] = {
            "value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{min(args.cpu_rows, M)} of {M} rows of A: quantize + fp64 GEMM "
                      f"against the full weight ({dt:.1f} s)",
            "quantize_one_thread": cpu_quantize_one_thread(wl, args.cpu_rows, A_cpu)}
    if rank == 0:
        print(json.dumps(line), flush=True)
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
