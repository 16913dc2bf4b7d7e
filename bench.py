#!/usr/bin/env python
"""Benchmark of the DyRA approximated linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl dyra|reference]
                    [--layer-only] [--no-cpu-baseline]

One step is one DyRA forward (projection, Gram, solve, residual factor,
output: every stage of Algorithm 1's inference procedure) over the workload's
B x T rows, inputs resident in HBM. The L2 cache is flushed (256 MiB write)
before every step, outside the step's CUDA events. Prints one JSON line.

Under torchrun (N > 1) every rank runs its own replica of the workload on its
own GPU (instances are independent; no collective on the data path); the
step time is the maximum over ranks and `value` counts all ranks' work.

--impl reference times the fp64 CPU oracle on the same workload instead (rank
0 only); that arm is a deliberately slow baseline, not the target.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DyRA linear µs & dense-equiv TFLOP/s vs cuBLAS dense; % of roofline"
UNIT = "TFLOP/s (dense-equivalent)"
HEADLINE = "vit_fc1"
STAGE_KERNELS = {"proj": "ProjPolicy (CTA pairs, or split-K clusters at skinny N)",
                 "gram": "umma_gemm_kernel<GramPolicy>",
                 "solve": "ltilde_kernel (L~ = L G^-1, beside the rank-k factor GEMM)",
                 "rfactor": "RFactorPolicy (Q = T W_res^T; CTA pairs when there are enough tiles)",
                 "out": "umma_gemm_pair_kernel<OutPairPolicy>"}
FLUSH_BYTES = 256 << 20


def peaks():
    p = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
         "source": "fallback"}
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        m = json.load(open(path))
        p.update({k: float(m[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")
                  if k in m})
        p["source"] = "measured"
    return p


def csrc_digest() -> str:
    """Hash of the kernel sources, to tell whether stored ncu counters are current."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "rank_structured_matmul_b200", "csrc")
    for f in sorted(os.listdir(d)):
        h.update(f.encode())
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def stored_traffic(stage: str, workload: str):
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    t = json.load(open(path)).get("%s:%s" % (stage, workload))
    if not t or t.get("csrc_digest") != csrc_digest():
        return None
    return t.get("dram_bytes_per_launch")


# ------------------------------------------------------------ workload ----

def workload_arrays(name: str):
    from synth import generate, spec
    s = spec(name)
    w = generate(s)
    return s, w


def algorithmic(s):
    """FLOPs and compulsory bytes of one forward and of its output stage."""
    es = 2 if s.dtype == "bf16" else 4
    N, di, do, r, k, B = s.N, s.d_in, s.d_out, s.r, s.k, s.B
    flops = {
        "proj": 2.0 * N * di * (r + k),
        "gram": 2.0 * N * k * (di + k),
        "solve": B * (k ** 3 / 3.0 + k ** 3) + 2.0 * N * k * k,
        "rfactor": 2.0 * B * k * di * do,
        "out": 2.0 * N * do * (r + k),
    }
    bytes_ = {
        "proj": es * (N * di + (r + k) * di + N * (r + k)),
        "gram": es * (N * di + N * k + B * k * di) + 4.0 * B * k * k,
        "solve": 4.0 * B * k * k + 2.0 * es * N * k,
        "rfactor": es * (do * di + B * k * di + do * B * k),
        "out": es * (N * do + N * r + N * k + do * r + do * B * k),
    }
    layer_flops = sum(flops.values())
    layer_bytes = es * (N * di + N * do + do * r + di * r + di * k + do * di)
    return flops, bytes_, layer_flops, layer_bytes


def static_matched_rank(s) -> int:
    """Rank r_s of a static-only layer (X V_s) U_s^T whose FLOPs 2 N r_s
    (d_in + d_out) match the DyRA layer's ([DyRA] App. E.4: the static
    baseline of rank r + k + k' with the same FLOPs), rounded down to a
    multiple of 8 (16-byte rows of bf16 factors) and capped at min(d_in, d_out)."""
    _, _, layer_flops, _ = algorithmic(s)
    rs = int(layer_flops // (2.0 * s.N * (s.d_in + s.d_out)))
    rs = min(rs - rs % 8, min(s.d_in, s.d_out) // 8 * 8)
    return max(rs, 8)


# -------------------------------------------------------------- clocks ----

class ClockSampler:
    """SM clock and clock-event reasons sampled every few ms while the timed
    region runs (read-only NVML queries; nvidia-smi as a fallback)."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, cuda_index: int, period_s: float = 0.005):
        self.cuda_index = cuda_index
        self.period = period_s
        self.rows = []
        self.thread = None
        self.stop_flag = False
        self.handle = None
        self.nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = self._handle(pynvml)
        except Exception:
            self.nvml = None
            self.handle = None

    def _handle(self, pynvml):
        import torch
        props = torch.cuda.get_device_properties(self.cuda_index)
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            dom = getattr(props, "pci_domain_id", 0)
            devid = getattr(props, "pci_device_id", 0)
            bus_str = "%08x:%02x:%02x.0" % (dom, bus, devid)
            try:
                return pynvml.nvmlDeviceGetHandleByPciBusId_v2(bus_str)
            except Exception:
                pass
        return pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def _sample(self):
        n, h = self.nvml, self.handle
        sm = n.nvmlDeviceGetClockInfo(h, n.NVML_CLOCK_SM)
        mx = n.nvmlDeviceGetMaxClockInfo(h, n.NVML_CLOCK_SM)
        try:
            bits = n.nvmlDeviceGetCurrentClocksEventReasons(h)
        except Exception:
            bits = n.nvmlDeviceGetCurrentClocksThrottleReasons(h)
        self.rows.append((float(sm), float(mx), int(bits)))

    def _loop(self):
        while not self.stop_flag:
            try:
                self._sample()
            except Exception:
                return
            time.sleep(self.period)

    def start(self):
        if self.handle is None:
            return
        import threading
        self._sample()
        self.thread = threading.Thread(target=self._loop, daemon=True)
        self.thread.start()

    def stop(self):
        if self.handle is None:
            return self._smi_once()
        self.stop_flag = True
        self.thread.join()
        try:
            self._sample()
        except Exception:
            pass
        rows = self.rows
        reasons = sorted(name for name, bit in self.REASONS.items()
                         if any(r[2] & bit for r in rows))
        return {"sm_mhz": float(np.median([r[0] for r in rows])), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(rows), "source": "nvml, every 5 ms"}

    def _smi_once(self):
        fields = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            out = subprocess.run(["nvidia-smi", "-i", str(self.cuda_index),
                                  "--query-gpu=" + fields, "--format=csv,noheader,nounits"],
                                 capture_output=True, text=True, timeout=20).stdout
            f = [x.strip() for x in out.strip().split(",")]
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            return {"sm_mhz": float(f[0]), "sm_max_mhz": float(f[1]),
                    "reasons": [n for n, v in zip(names, f[2:6]) if v.lower() == "active"],
                    "samples": 1, "source": "nvidia-smi after the timed region"}
        except Exception:
            return None


# ------------------------------------------------------------ ranks ----

def max_over_ranks(x: float, world: int, device=None) -> float:
    """The slowest rank's value: every rank takes part, rank order does not matter."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(flops_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job throughput in TFLOP/s: every rank's work over the slowest rank's time."""
    return flops_per_rank * world / seconds / 1e12


# ------------------------------------------------------------ dyra arm ----

def run_dyra(args):
    import torch
    import torch.distributed as dist
    from rank_structured_matmul_b200 import dyra, prep

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    s, w = workload_arrays(args.workload)
    f = prep.prepare_from_svd(w.left, w.sigma, w.right, s.r, s.k, s.lam)
    td = torch.bfloat16 if s.dtype == "bf16" else torch.float32
    layer = dyra.DyraLinear(s.d_in, s.d_out, s.r, s.k, s.dtype)
    layer.load(f.U, f.V, f.P, f.W_res, s.lam)
    X = torch.from_numpy(w.X).to(dev, td)
    Y = torch.empty(s.N, s.d_out, device=dev, dtype=td)
    layer.reserve(s.B, s.T)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def step():
        layer.forward(X, B=s.B, T=s.T, Y=Y)

    def timed(fn, K, W):
        for _ in range(W):
            flush.zero_()
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
        for a, b in ev:
            flush.zero_()
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return float(np.mean([a.elapsed_time(b) for a, b in ev]))

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    # ---- the timed region: K steps, barrier + sync on both sides
    for _ in range(args.warmup):
        flush.zero_()
        step()
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    ms = timed(step, args.steps, 0)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    status = layer.status()
    ms = max_over_ranks(ms, world, dev)

    dense_flops = 2.0 * s.N * s.d_in * s.d_out
    value = job_value(dense_flops, world, ms * 1e-3)
    if args.layer_only:  # the timed steps only (for profiler launch lists)
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                              "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                              "config": {"workload": s.name}, "device_status": status,
                              "layer_only": True}), flush=True)
        layer.close()
        if world > 1:
            dist.destroy_process_group()
        return

    # ---- cuBLAS dense X W^T of the same shape
    Wd = torch.from_numpy(w.weight()).to(dev, td)
    Yd = torch.empty_like(Y)
    dense_ms = timed(lambda: torch.matmul(X, Wd.t(), out=Yd), args.steps, 3)

    # ---- per-stage device time (events between the stage launches); the
    # tensor-core path only (the fp32 path runs plain CUDA-core kernels)
    pk = peaks()
    flops, bytes_, layer_flops, layer_bytes = algorithmic(s)
    umma = s.dtype == "bf16"
    stage_ms = None
    if umma:
        dyra.dyra_debug_set_stage_timing(layer.plan, True)
        acc = {k: [] for k in dyra.STAGES}
        for _ in range(max(5, min(args.steps, 50))):
            flush.zero_()
            step()
            for k2, v in dyra.dyra_debug_stage_times(layer.plan).items():
                acc[k2].append(v)
        dyra.dyra_debug_set_stage_timing(layer.plan, False)
        stage_ms = {k2: float(np.mean(v)) for k2, v in acc.items()}
        dom = max(stage_ms, key=stage_ms.get)
        t_dom = stage_ms[dom] * 1e-3
        tensor_t = flops[dom] / (pk["bf16_tflops"] * 1e12)
        hbm_t = bytes_[dom] / (pk["hbm_gbs"] * 1e9)
        if tensor_t >= hbm_t:
            roof = {"bound": "tensor", "achieved": flops[dom] / t_dom / 1e12,
                    "peak": pk["bf16_tflops"], "unit": "TFLOP/s"}
        else:
            roof = {"bound": "hbm", "achieved": bytes_[dom] / t_dom / 1e9, "peak": pk["hbm_gbs"],
                    "unit": "GB/s"}
        roof["frac"] = roof["achieved"] / roof["peak"]
        roof["traffic"] = stored_traffic(dom, args.workload)
        roof["kernel"] = STAGE_KERNELS[dom]
        roof["peak_source"] = pk["source"] + " burst"
    else:
        # fp32 FFMA: 148 SMs x 128 lanes x 2 FLOP at the maximum SM clock
        fp32_peak = 148 * 128 * 2 * 1.965e9 / 1e12
        roof = {"bound": "alu", "achieved": layer_flops / (ms * 1e-3) / 1e12, "peak": fp32_peak,
                "unit": "TFLOP/s", "traffic": None, "kernel": "whole layer (fp32 CUDA-core path)",
                "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 x 1965 MHz"}
        roof["frac"] = roof["achieved"] / roof["peak"]
    layer_roof_us = max(layer_flops / (pk["bf16_tflops"] * 1e12),
                        layer_bytes / (pk["hbm_gbs"] * 1e9)) * 1e6

    # ---- end to end through the C ABI on host buffers (dyra_forward_batched_host):
    # pinned host X -> device, forward, Y -> pinned host, overlapped by chunks of instances
    Xh = X.cpu().pin_memory()
    Yh = torch.empty(Y.shape, dtype=td).pin_memory()

    def e2e_step():
        layer.forward_host(Xh, B=s.B, T=s.T, Y=Yh)

    e2e_ms = max_over_ranks(timed(e2e_step, args.steps, 2), world, dev)
    e2e_value = job_value(dense_flops, world, e2e_ms * 1e-3)

    # ---- the static-only layer with the same FLOPs (rank r_s, no correction),
    # timed the same way, outside the timed region above
    rs = static_matched_rank(s)
    static = dyra.DyraLinear(s.d_in, s.d_out, rs, 0, s.dtype)
    static.load(torch.as_tensor(np.ascontiguousarray(w.left[:, :rs] * w.sigma[:rs])),
                torch.as_tensor(np.ascontiguousarray(w.right[:, :rs])), None, None, s.lam)
    Ys = torch.empty_like(Y)
    static_ms = max_over_ranks(timed(lambda: static.forward(X, B=s.B, T=s.T, Y=Ys), args.steps, 3),
                               world, dev)
    static_status = static.status()

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": s.dtype, "data": "synthetic (seeded; shapes and statistics "
        "of the workload, random-orthogonal weights with a power-law spectrum)",
        "config": {"workload": s.name, "d_in": s.d_in, "d_out": s.d_out, "r": s.r, "k": s.k,
                   "instances": s.B, "rows_per_instance": s.T, "rows": s.N, "lambda": s.lam,
                   "l2": "flushed before every step (256 MiB write, outside the step events)",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "us_per_layer": ms * 1e3,
        "cublas_dense_us": dense_ms * 1e3,
        "speedup_vs_cublas_dense": dense_ms / ms,
        "dyra_tflops_algorithmic": layer_flops / (ms * 1e-3) / 1e12,
        "layer_roofline": {"us": layer_roof_us, "frac": layer_roof_us / (ms * 1e3),
                           "flops": layer_flops, "bytes": layer_bytes},
        "stage_us": {k2: v * 1e3 for k2, v in stage_ms.items()} if stage_ms else None,
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": X.numel() * X.element_size(),
                "d2h_bytes_per_step": Y.numel() * Y.element_size(), "us": e2e_ms * 1e3},
        "gpu_launches": ((5 if s.k > 0 else 2) if umma else (7 if s.k > 0 else 2)) * args.steps,
        "device_status": status,
        "clocks": clk,
        "static_matched": {"rank": rs, "flops": 2.0 * s.N * rs * (s.d_in + s.d_out),
                           "dyra_flops": layer_flops, "us_per_layer": static_ms * 1e3,
                           "dyra_us_per_layer": ms * 1e3, "device_status": static_status},
    }

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"], line["parity"] = cpu_baseline(s, w, Y)
        line["static_matched"].update(static_errors(s, w, Ys, rs, line["parity"]["rows"]))
    static.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
    layer.close()
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------------- oracle ----

def static_errors(s, w, Ys_gpu, rs, rows):
    """The FLOPs-matched static layer on the oracle's sample rows: its
    approximation error relative to the dense product, and the GPU result
    against the oracle's weight-only product of the same rounded factors."""
    import oracle
    Xr = oracle.round_to(w.X[:rows], s.dtype)
    Us = oracle.round_to(w.left[:, :rs] * w.sigma[:rs], s.dtype)
    Vs = oracle.round_to(w.right[:, :rs], s.dtype)
    Yo = oracle.weight_only(Xr, Us, Vs)
    Yd = oracle.dense(Xr, w.weight())
    Yg = Ys_gpu[:rows].double().cpu().numpy()
    return {"oracle_err_vs_dense": oracle.rel_fro(Yo, Yd),
            "rel_fro_vs_oracle": oracle.rel_fro(Yg, Yo), "rows": rows}


def oracle_inputs(s, w):
    import oracle
    f = oracle.offline_prepare_from_svd(w.left, w.sigma, w.right, s.r, s.k, s.lam)
    return f, [oracle.round_to(a, s.dtype) for a in (w.X, f.U, f.V, f.P, f.W_res)]


def cpu_baseline(s, w, Y_gpu):
    import oracle
    f, (Xr, Ur, Vr, Pr, Wr) = oracle_inputs(s, w)
    cores = len(os.sched_getaffinity(0))
    # time the oracle on whole instances until ~10 s of work (at least one)
    t0 = time.perf_counter()
    Y1 = oracle.inference(Xr[: s.T], Ur, Vr, Pr, Wr, s.lam, 1, s.T)
    t1 = time.perf_counter() - t0
    n_inst = int(max(1, min(s.B, 10.0 // max(t1, 1e-3))))
    t0 = time.perf_counter()
    Yo = oracle.inference(Xr[: n_inst * s.T], Ur, Vr, Pr, Wr, s.lam, n_inst, s.T)
    t = time.perf_counter() - t0
    flops = 2.0 * n_inst * s.T * s.d_in * s.d_out
    base = {"value": flops / t / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": "%d of %d instances (%d rows), fp64 NumPy, %.2f s" % (
                n_inst, s.B, n_inst * s.T, t)}
    Yg = Y_gpu[: n_inst * s.T].double().cpu().numpy()
    W = w.weight()
    rep = oracle.error_report(Xr[: n_inst * s.T], W, oracle.Factors(Ur, Vr, Pr, Wr, f.R0), s.lam,
                              n_inst, s.T, Y=Yo)
    parity = {"rel_fro_vs_oracle": oracle.rel_fro(Yg, Yo), "tol": 1e-2 if s.dtype == "bf16"
              else 1e-5, "rows": n_inst * s.T, "oracle_err_weight_only": rep["err_wo"],
              "oracle_err_dyra": rep["err_dyra"]}
    return base, parity


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    s, w = workload_arrays(args.workload)
    f, (Xr, Ur, Vr, Pr, Wr) = oracle_inputs(s, w)
    cores = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    oracle.inference(Xr[: s.T], Ur, Vr, Pr, Wr, s.lam, 1, s.T)
    t1 = time.perf_counter() - t0
    # each step a bounded sample of whole instances, sized so that the whole
    # run (warm-up included) takes about two minutes of host time
    per_step = 120.0 / (args.steps + args.warmup)
    n_inst = int(max(1, min(s.B, per_step // max(t1, 1e-4))))
    rows = n_inst * s.T
    for _ in range(args.warmup):
        oracle.inference(Xr[:rows], Ur, Vr, Pr, Wr, s.lam, n_inst, s.T)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.inference(Xr[:rows], Ur, Vr, Pr, Wr, s.lam, n_inst, s.T)
        times.append(time.perf_counter() - t0)
    t = float(np.mean(times))
    value = 2.0 * rows * s.d_in * s.d_out / t / 1e12
    sample = "%d of %d instances (%d rows) per step, fp64 NumPy" % (n_inst, s.B, rows)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": s.name, "d_in": s.d_in, "d_out": s.d_out, "r": s.r, "k": s.k,
                       "instances": s.B, "rows_per_instance": s.T, "lambda": s.lam},
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--impl", choices=("dyra", "reference"), default="dyra")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layer-only", action="store_true",
                    help="time the DyRA steps only: no cuBLAS, stage timing, e2e or CPU legs")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed steps
    if args.impl == "reference":
        run_reference(args)
    else:
        run_dyra(args)


if __name__ == "__main__":
    main()
