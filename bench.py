#!/usr/bin/env python
"""Benchmark of the DyRA approximated linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl dyra|reference]
                    [--layer-only] [--no-cpu-baseline] [--no-per-config]

One step is one DyRA forward (projection, Gram, solve, residual factor,
output: every stage of Algorithm 1's inference procedure) over the workload's
B x T rows, inputs resident in HBM. The default workload is the largest
single-GPU configuration, the Llama-shaped up-projection at 8192 tokens
(4096 -> 14336, r = 1024, k = 64). `--workload vit_block` runs the four
ViT-L/16 block linears (qkv, proj, fc1, fc2; 64 x 201 tokens) back to back on
one stream as one step. The L2 cache is flushed (256 MiB write) before every
step, outside the step's CUDA events. Prints one JSON line.

Beside the headline, `per_config` times every workload (each layer of the
synthetic set and the ViT block sequence) against cuBLAS dense X W^T of the
same shape and checks it against the fp64 oracle on sampled rows.

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
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DyRA linear µs & dense-equiv TFLOP/s vs cuBLAS dense; % of roofline"
UNIT = "TFLOP/s (dense-equivalent)"
HEADLINE = "llama_up_8192"
BLOCK = ("vit_block_qkv", "vit_block_proj", "vit_block_fc1", "vit_block_fc2")
STAGE_KERNELS = {"proj": "ProjPolicy (CTA pairs, or split-K clusters at skinny N)",
                 "gram": "umma_gemm_kernel<GramPolicyT<false, false>>",
                 "solve": "ltilde_kernel (L~ = L G^-1, beside the rank-k factor GEMM)",
                 "rfactor": "RFactorPolicy (Q = T W_res^T; CTA pairs when there are enough tiles)",
                 "out": "umma_gemm_pair_kernel<OutPairPolicyT<false, false>>"}
FLUSH_BYTES = 256 << 20
L2_NOTE = "GPU arm: 256 MiB written before every step, outside the step events"
DATA = ("synthetic (seeded; shapes and statistics of the workload, random-orthogonal weights "
        "with a power-law spectrum)")


def workload_names():
    from synth import CONFIGS
    return list(CONFIGS) + ["vit_block"]


def specs_of(workload: str):
    """The layers one step of `workload` runs, in order."""
    from synth import spec
    if workload == "vit_block":
        return [spec(n) for n in BLOCK]
    return [spec(workload)]


def config_of(workload: str, world: int) -> dict:
    """The `config` object of both arms' JSON lines (identical by construction)."""
    ss = specs_of(workload)
    layers = [{"name": s.name, "d_in": s.d_in, "d_out": s.d_out, "r": s.r, "k": s.k,
               "instances": s.B, "rows_per_instance": s.T} for s in ss]
    c = {"workload": workload}
    if len(ss) == 1:
        c.update({k: v for k, v in layers[0].items() if k != "name"})
    else:
        c["layers"] = layers
    c.update({"rows": ss[0].N, "lambda": ss[0].lam, "l2": L2_NOTE,
              "parallelism": "replicas" if world > 1 else "single GPU"})
    return c


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

def algorithmic(s):
    """FLOPs and compulsory bytes of one forward, per stage and for the layer."""
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


def layer_roofline_us(s, pk) -> float:
    """The slower of the layer's FLOPs at the bf16 peak and its compulsory
    bytes at the HBM peak, in µs."""
    _, _, f, b = algorithmic(s)
    return max(f / (pk["bf16_tflops"] * 1e12), b / (pk["hbm_gbs"] * 1e9)) * 1e6


def launches_per_forward(s) -> int:
    """Library kernels one forward launches: five tensor-core stages (two
    without the correction); the fp32 path's CUDA-core chain is seven."""
    if s.dtype == "bf16":
        return 5 if s.k > 0 else 2
    return 7 if s.k > 0 else 2


def static_matched_rank(s) -> int:
    """Rank r_s of a static-only layer (X V_s) U_s^T whose FLOPs 2 N r_s
    (d_in + d_out) match the DyRA layer's ([DyRA] App. E.4: the static
    baseline of rank r + k + k' with the same FLOPs), rounded down to a
    multiple of 8 (16-byte rows of bf16 factors) and capped at min(d_in, d_out)."""
    _, _, layer_flops, _ = algorithmic(s)
    rs = int(layer_flops // (2.0 * s.N * (s.d_in + s.d_out)))
    rs = min(rs - rs % 8, min(s.d_in, s.d_out) // 8 * 8)
    return max(rs, 8)


def parity_rows(s, max_rows: int = 1024):
    """Rows of a workload that the oracle checks: every row of small layers;
    otherwise whole leading instances (multi-instance layers) or evenly
    spaced rows plus the last rows of a single long instance."""
    if s.N <= max_rows:
        return np.arange(s.N)
    if s.B > 1:
        n_inst = max(1, max_rows // s.T)
        return np.arange(n_inst * s.T)
    body = np.linspace(0, s.N - 1, max_rows - 64).astype(np.int64)
    return np.unique(np.concatenate([body, np.arange(s.N - 64, s.N)]))


# -------------------------------------------------------------- clocks ----

class ClockSampler:
    """SM clock and clock-event reasons sampled every 0.2 ms while the timed
    region runs (two read-only NVML queries per sample, the maximum clock read
    once; nvidia-smi as a fallback)."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, cuda_index: int, period_s: float = 0.0002):
        self.cuda_index = cuda_index
        self.period = period_s
        self.rows = []
        self.thread = None
        self.stop_flag = False
        self.handle = None
        self.nvml = None
        self.max_mhz = None
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
        if self.max_mhz is None:
            self.max_mhz = float(n.nvmlDeviceGetMaxClockInfo(h, n.NVML_CLOCK_SM))
        mx = self.max_mhz
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
            if self.period > 0:
                time.sleep(self.period)

    def start(self):
        if self.handle is None:
            return
        import threading
        self.rows, self.stop_flag = [], False
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
                "sm_mhz_min": float(min(r[0] for r in rows)), "reasons": reasons,
                "samples": len(rows),
                "source": "nvml, every %g ms" % (self.period * 1e3) if self.period > 0
                else "nvml, back to back"}

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

class LayerRun:
    """One layer of a workload on the device: its plan with the factors loaded,
    the seeded input X resident in HBM and the output Y."""

    def __init__(self, s, dev, w=None):
        import torch
        from rank_structured_matmul_b200 import dyra, prep
        from synth import generate
        self.s = s
        self.w = w if w is not None else generate(s)
        f = prep.prepare_from_svd(self.w.left, self.w.sigma, self.w.right, s.r, s.k, s.lam)
        self.td = torch.bfloat16 if s.dtype == "bf16" else torch.float32
        self.layer = dyra.DyraLinear(s.d_in, s.d_out, s.r, s.k, s.dtype)
        self.layer.load(f.U, f.V, f.P, f.W_res, s.lam)
        self.X = torch.from_numpy(self.w.X).to(dev, self.td)
        self.Y = torch.empty(s.N, s.d_out, device=dev, dtype=self.td)
        self.layer.reserve(s.B, s.T)
        self.dev = dev
        self.Wd = self.Yd = None
        self.Xh = self.Yh = None

    def step(self):
        self.layer.forward(self.X, B=self.s.B, T=self.s.T, Y=self.Y)

    def dense_step(self):
        import torch
        if self.Wd is None:
            self.Wd = torch.from_numpy(self.w.weight()).to(self.dev, self.td)
            self.Yd = torch.empty_like(self.Y)
        torch.matmul(self.X, self.Wd.t(), out=self.Yd)

    def host_step(self):
        """The forward through the C ABI on pinned host buffers."""
        if self.Xh is None:
            self.Xh = self.X.cpu().pin_memory()
            import torch
            self.Yh = torch.empty(self.Y.shape, dtype=self.td).pin_memory()
        self.layer.forward_host(self.Xh, B=self.s.B, T=self.s.T, Y=self.Yh)

    def free_dense(self):
        self.Wd = self.Yd = None

    def close(self):
        self.layer.close()


class Timer:
    """Mean device time of a step over K launches, each after an L2 flush
    outside its CUDA events (recorded on the current stream)."""

    def __init__(self, dev):
        import torch
        self.flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def __call__(self, fn, K, W):
        import torch
        for _ in range(W):
            self.flush.zero_()
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
        for a, b in ev:
            self.flush.zero_()
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return float(np.mean([a.elapsed_time(b) for a, b in ev]))


def dense_time(timer, fn, steps):
    """cuBLAS dense time of a step: the lower mean of two timed loops (the
    baseline's occasional slow loop would otherwise flatter the comparison)."""
    return min(timer(fn, steps, 3), timer(fn, steps, 0))


def stage_times(runs, timer, n_steps):
    """Mean per-stage device time of each layer (events between the stage
    launches, a separate loop with stage timing switched on), in ms."""
    from rank_structured_matmul_b200 import dyra
    out = []
    for run in runs:
        dyra.dyra_debug_set_stage_timing(run.layer.plan, True)
        acc = {k: [] for k in dyra.STAGES}
        for _ in range(n_steps):
            timer.flush.zero_()
            run.step()
            for k2, v in dyra.dyra_debug_stage_times(run.layer.plan).items():
                acc[k2].append(v)
        dyra.dyra_debug_set_stage_timing(run.layer.plan, False)
        out.append({k2: float(np.mean(v)) for k2, v in acc.items()})
    return out


def dominant_roofline(runs, st, pk, workload):
    """Roofline of the stage with the most device time over the step's
    layers: its algorithmic bytes or FLOPs over its live time."""
    tot = {k: sum(t[k] for t in st) for k in st[0]}
    dom = max(tot, key=tot.get)
    t_dom = tot[dom] * 1e-3
    fl = sum(algorithmic(r.s)[0][dom] for r in runs)
    by = sum(algorithmic(r.s)[1][dom] for r in runs)
    if fl / (pk["bf16_tflops"] * 1e12) >= by / (pk["hbm_gbs"] * 1e9):
        roof = {"bound": "tensor", "achieved": fl / t_dom / 1e12, "peak": pk["bf16_tflops"],
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": by / t_dom / 1e9, "peak": pk["hbm_gbs"],
                "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = stored_traffic(dom, workload)
    roof["kernel"] = STAGE_KERNELS[dom]
    roof["stage"] = dom
    roof["peak_source"] = pk["source"] + " burst"
    return roof


def oracle_check(s, w, Y_gpu, rows=None):
    """The GPU output on sampled rows against the fp64 oracle on the same
    rounded inputs, with the oracle's own errors against the dense product."""
    import oracle
    f, (Xr, Ur, Vr, Pr, Wr) = oracle_inputs(s, w)
    rows = parity_rows(s) if rows is None else rows
    Yo = oracle.inference_rows(Xr, Ur, Vr, Pr, Wr, s.lam, s.B, s.T, rows)
    Yg = Y_gpu[torch_index(rows, Y_gpu.device)].double().cpu().numpy()
    Yd = oracle.dense(Xr[rows], w.weight())
    Ywo = oracle.weight_only(Xr[rows], Ur, Vr)
    return {"rel_fro_vs_oracle": oracle.rel_fro(Yg, Yo),
            "tol": 1e-2 if s.dtype == "bf16" else 1e-5, "rows": int(len(rows)),
            "oracle_err_weight_only": oracle.rel_fro(Ywo, Yd),
            "oracle_err_dyra": oracle.rel_fro(Yo, Yd)}


def torch_index(rows, device):
    import torch
    return torch.as_tensor(np.asarray(rows, dtype=np.int64), device=device)


def per_config(names, dev, pk, steps, warmup, headline_entry=None):
    """Every workload in `names`, timed against cuBLAS dense and checked
    against the oracle. Returns the entries and the clocks sampled while
    they ran."""
    from synth import generate, spec
    timer = Timer(dev)
    entries = {}
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    llama_w = None
    for name in names:
        if headline_entry is not None and name == headline_entry[0]:
            entries[name] = headline_entry[1]
            continue
        ss = specs_of(name)
        runs = []
        for s in ss:
            w = None
            if s.name.startswith("llama_up_"):
                # one 8192-row draw; each sweep point is its N-row prefix
                if llama_w is None:
                    llama_w = generate(spec("llama_up_8192"))
                w = dataclass_prefix(llama_w, s)
            runs.append(LayerRun(s, dev, w))
        seq = lambda: [r.step() for r in runs]
        dense = lambda: [r.dense_step() for r in runs]
        t = timer(seq, steps, warmup)
        td = dense_time(timer, dense, steps)
        flops = sum(2.0 * r.s.N * r.s.d_in * r.s.d_out for r in runs)
        roof_us = sum(layer_roofline_us(r.s, pk) for r in runs)
        e = {"us": t * 1e3, "cublas_dense_us": td * 1e3, "speedup_vs_cublas_dense": td / t,
             "dense_equiv_tflops": flops / (t * 1e-3) / 1e12,
             "layer_roofline_us": roof_us, "layer_roofline_frac": roof_us / (t * 1e3),
             "device_status": max(r.layer.status() for r in runs)}
        checks = [oracle_check(r.s, r.w, r.Y) for r in runs]
        e["rel_fro_vs_oracle"] = max(c["rel_fro_vs_oracle"] for c in checks)
        e["tol"] = checks[0]["tol"]
        e["oracle_err_weight_only"] = [c["oracle_err_weight_only"] for c in checks]
        e["oracle_err_dyra"] = [c["oracle_err_dyra"] for c in checks]
        e["parity_rows"] = [c["rows"] for c in checks]
        if len(runs) > 1:
            e["layers"] = {}
            for r in runs:
                tl = timer(r.step, steps, 3)
                tdl = dense_time(timer, r.dense_step, steps)
                e["layers"][r.s.name] = {"us": tl * 1e3, "cublas_dense_us": tdl * 1e3}
        else:
            e["static_matched"] = static_entry(runs[0], timer, steps)
        for r in runs:
            r.free_dense()
            r.close()
        entries[name] = e
    clk = clocks.stop()
    return entries, clk


def extras(dev, steps, warmup):
    """The NEXT rows, timed and checked like the workloads: the ViT-L fc1 layer
    with a bias and a correction weight ([DyRA] Sec. 2.4), with t = 1.5 and 2
    ALS iterations (Sec. 3.3), with the Newton-Schulz solver (Sec. 2.4), and a
    Monarch static part (App. B) on the ViT-L block proj shape, each beside the
    plain layer's time and checked against the oracle on whole instances."""
    import torch
    import oracle
    from oracle import monarch as mon
    from rank_structured_matmul_b200 import dyra, prep
    from synth import generate, spec
    timer = Timer(dev)
    out = {}
    s = spec("vit_fc1")
    run = LayerRun(s, dev)
    n_inst = 5
    rows = n_inst * s.T
    fo, (Xr, Ur, Vr, Pr, Wr) = oracle_inputs(s, run.w)
    Xs = Xr[:rows]
    base_us = timer(run.step, steps, warmup) * 1e3

    def check(Yo):
        return oracle.rel_fro(run.Y[:rows].double().cpu().numpy(), Yo)

    bias = oracle.round_to(np.random.default_rng(11).standard_normal(s.d_out) * 0.3, "bf16")
    run.layer.set_linear(torch.from_numpy(bias), 0.7)
    us = timer(run.step, steps, warmup) * 1e3
    out["vit_fc1_bias_alpha"] = {
        "us": us, "plain_us": base_us, "overhead": us / base_us - 1.0,
        "rel_fro_vs_oracle": check(oracle.inference(Xs, Ur, Vr, Pr, Wr, s.lam, n_inst, s.T,
                                                    bias=bias, alpha=0.7)),
        "device_status": run.layer.status()}
    run.layer.set_linear(None, 1.0)
    for t in (1.5, 2.0):
        run.layer.set_als_iterations(t)
        us = timer(run.step, steps, warmup) * 1e3
        out["vit_fc1_t%g" % t] = {
            "us": us, "plain_us": base_us, "launches": {1.5: 9, 2.0: 13}[t],
            "rel_fro_vs_oracle": check(oracle.als_inference(Xs, Ur, Vr, Wr, fo.R0, s.lam, n_inst,
                                                            s.T, t)),
            "device_status": run.layer.status()}
    run.layer.set_als_iterations(1)
    dyra.dyra_set_solver(run.layer.plan, dyra.DYRA_SOLVER_NEWTON_SCHULZ, 40)
    us = timer(run.step, steps, warmup) * 1e3
    out["vit_fc1_newton_schulz"] = {
        "us": us, "plain_us": base_us,
        "rel_fro_vs_oracle": check(oracle.inference(Xs, Ur, Vr, Pr, Wr, s.lam, n_inst, s.T)),
        "device_status": run.layer.status()}
    run.close()

    # Monarch static part, b1 = b2 = 32, on the ViT-L block proj shape
    sm = spec("vit_block_proj")
    w = generate(sm)
    b = 32
    f = prep.prepare_monarch(w.weight(), b, b, sm.k, sm.lam)
    td = torch.bfloat16
    layer = dyra.DyraMonarchLinear(sm.d_in, b, b, sm.k, "bf16")
    layer.load(f.Lblocks, f.Rblocks, f.P, f.W_res, sm.lam)
    X = torch.from_numpy(w.X).to(dev, td)
    Y = torch.empty(sm.N, sm.d_out, device=dev, dtype=td)
    mstep = lambda: layer.forward(X, B=sm.B, T=sm.T, Y=Y)
    us = timer(mstep, steps, warmup) * 1e3
    Wd = torch.from_numpy(w.weight()).to(dev, td)
    Yd = torch.empty_like(Y)
    dense_us = dense_time(timer, lambda: torch.matmul(X, Wd.t(), out=Yd), steps) * 1e3
    rd = lambda a: oracle.round_to(np.asarray(a), "bf16")
    Lb, Rb = rd(f.Lblocks.numpy()), rd(f.Rblocks.numpy())
    fr = mon.MonarchFactors(list(Lb), list(Rb), mon.monarch_matrix(list(Lb), list(Rb)).T,
                            rd(f.P.numpy()), rd(f.W_res.numpy()), None)
    Xm = rd(w.X[:rows])
    Yo = mon.monarch_inference(Xm, fr, sm.lam, n_inst, sm.T)
    Ydense = oracle.dense(Xm, w.weight())
    out["vit_block_proj_monarch"] = {
        "us": us, "cublas_dense_us": dense_us, "speedup_vs_cublas_dense": dense_us / us,
        "blocks": [b, b], "k": sm.k,
        "rel_fro_vs_oracle": oracle.rel_fro(Y[:rows].double().cpu().numpy(), Yo),
        "oracle_err_weight_only": oracle.rel_fro(Xm @ fr.What.T, Ydense),
        "oracle_err_dyra": oracle.rel_fro(Yo, Ydense),
        "device_status": layer.status()}
    layer.close()
    return out


def static_entry(run, timer, steps):
    """The FLOPs-matched static layer of one workload ([DyRA] App. E.4; NEXT
    f1): rank, time, and the oracle's error of it and of DyRA against the
    dense product on the parity rows."""
    import torch
    import oracle
    from rank_structured_matmul_b200 import dyra
    s, w = run.s, run.w
    rs = static_matched_rank(s)
    st = dyra.DyraLinear(s.d_in, s.d_out, rs, 0, s.dtype)
    st.load(torch.as_tensor(np.ascontiguousarray(w.left[:, :rs] * w.sigma[:rs])),
            torch.as_tensor(np.ascontiguousarray(w.right[:, :rs])), None, None, s.lam)
    Ys = torch.empty_like(run.Y)
    us = timer(lambda: st.forward(run.X, B=s.B, T=s.T, Y=Ys), steps, 3) * 1e3
    errs = static_errors([(run, rs, st, Ys)])
    out = {"rank": rs, "r_plus_k": s.r + s.k, "us": us, "device_status": st.status(),
           "oracle_err_vs_dense": errs["oracle_err_vs_dense"][0],
           "rel_fro_vs_oracle": errs["rel_fro_vs_oracle"]}
    st.close()
    return out


def dataclass_prefix(w, s):
    """The N-row prefix of a larger draw of the same layer."""
    import dataclasses
    return dataclasses.replace(w, spec=s, X=np.ascontiguousarray(w.X[: s.N]))


def run_dyra(args):
    import torch
    import torch.distributed as dist
    from rank_structured_matmul_b200 import dyra

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    ss = specs_of(args.workload)
    runs = [LayerRun(s, dev) for s in ss]
    timer = Timer(dev)

    def step():
        for r in runs:
            r.step()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    # ---- the timed region: K steps, barrier + sync on both sides
    for _ in range(args.warmup):
        timer.flush.zero_()
        step()
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    ms = timer(step, args.steps, 0)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    status = max(r.layer.status() for r in runs)
    ms = max_over_ranks(ms, world, dev)

    dense_flops = sum(2.0 * r.s.N * r.s.d_in * r.s.d_out for r in runs)
    value = job_value(dense_flops, world, ms * 1e-3)
    if args.layer_only:  # the timed steps only (for profiler launch lists)
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                              "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                              "config": {"workload": args.workload}, "device_status": status,
                              "layer_only": True}), flush=True)
        for r in runs:
            r.close()
        if world > 1:
            dist.destroy_process_group()
        return

    # ---- cuBLAS dense X W^T of the same shapes, timed the same way
    dense_ms = max_over_ranks(dense_time(timer, lambda: [r.dense_step() for r in runs], args.steps),
                              world, dev)
    for r in runs:
        r.free_dense()

    pk = peaks()
    layer_flops = sum(algorithmic(r.s)[2] for r in runs)
    layer_bytes = sum(algorithmic(r.s)[3] for r in runs)
    layer_roof_us = sum(layer_roofline_us(r.s, pk) for r in runs)
    umma = ss[0].dtype == "bf16"
    stage_us = None
    if umma:
        st = stage_times(runs, timer, max(5, min(args.steps, 50)))
        roof = dominant_roofline(runs, st, pk, args.workload)
        stage_us = ({k: v * 1e3 for k, v in st[0].items()} if len(runs) == 1 else
                    {r.s.name: {k: v * 1e3 for k, v in t.items()} for r, t in zip(runs, st)})
    else:
        # fp32 FFMA: 148 SMs x 128 lanes x 2 FLOP at the maximum SM clock
        fp32_peak = 148 * 128 * 2 * 1.965e9 / 1e12
        roof = {"bound": "alu", "achieved": layer_flops / (ms * 1e-3) / 1e12, "peak": fp32_peak,
                "unit": "TFLOP/s", "traffic": None, "kernel": "whole layer (fp32 CUDA-core path)",
                "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 x 1965 MHz"}
        roof["frac"] = roof["achieved"] / roof["peak"]

    # ---- end to end through the C ABI on host buffers (dyra_forward_batched_host):
    # pinned host X -> device, forward, Y -> pinned host, overlapped by chunks of instances
    e2e_ms = max_over_ranks(timer(lambda: [r.host_step() for r in runs], args.steps, 2),
                            world, dev)
    e2e_value = job_value(dense_flops, world, e2e_ms * 1e-3)

    # ---- the static-only layer with the same FLOPs (rank r_s, no correction),
    # timed the same way, outside the timed region above
    statics = []
    for r in runs:
        rs = static_matched_rank(r.s)
        st_layer = dyra.DyraLinear(r.s.d_in, r.s.d_out, rs, 0, r.s.dtype)
        st_layer.load(torch.as_tensor(np.ascontiguousarray(r.w.left[:, :rs] * r.w.sigma[:rs])),
                      torch.as_tensor(np.ascontiguousarray(r.w.right[:, :rs])), None, None,
                      r.s.lam)
        statics.append((r, rs, st_layer, torch.empty_like(r.Y)))
    static_ms = max_over_ranks(
        timer(lambda: [sl.forward(r.X, B=r.s.B, T=r.s.T, Y=Ys) for r, _, sl, Ys in statics],
              args.steps, 3), world, dev)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": ss[0].dtype, "data": DATA,
        "config": config_of(args.workload, world),
        "us_per_layer": ms * 1e3,
        "us_x_sm_mhz": ms * 1e3 * clk["sm_mhz"] if clk else None,
        "cublas_dense_us": dense_ms * 1e3,
        "speedup_vs_cublas_dense": dense_ms / ms,
        "dyra_tflops_algorithmic": layer_flops / (ms * 1e-3) / 1e12,
        "layer_roofline": {"us": layer_roof_us, "frac": layer_roof_us / (ms * 1e3),
                           "flops": layer_flops, "bytes": layer_bytes},
        "stage_us": stage_us,
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": sum(r.X.numel() * r.X.element_size() for r in runs),
                "d2h_bytes_per_step": sum(r.Y.numel() * r.Y.element_size() for r in runs),
                "us": e2e_ms * 1e3, "path": "dyra_forward_batched_host (C ABI, pinned host "
                "buffers, copies inside the timed region)"},
        "gpu_launches": sum(launches_per_forward(r.s) for r in runs) * args.steps,
        "device_status": status,
        "clocks": clk,
        "static_matched": {"rank": [rs for _, rs, _, _ in statics],
                           "flops": sum(2.0 * r.s.N * rs * (r.s.d_in + r.s.d_out)
                                        for r, rs, _, _ in statics),
                           "dyra_flops": layer_flops, "us_per_layer": static_ms * 1e3,
                           "dyra_us_per_layer": ms * 1e3,
                           "device_status": max(sl.status() for _, _, sl, _ in statics)},
    }

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(runs)
        checks = [oracle_check(r.s, r.w, r.Y) for r in runs]
        line["parity"] = {"rel_fro_vs_oracle": max(c["rel_fro_vs_oracle"] for c in checks),
                          "tol": checks[0]["tol"], "rows": [c["rows"] for c in checks],
                          "oracle_err_weight_only": [c["oracle_err_weight_only"] for c in checks],
                          "oracle_err_dyra": [c["oracle_err_dyra"] for c in checks]}
        line["static_matched"].update(static_errors(statics))
    for _, _, sl, _ in statics:
        sl.close()

    if rank == 0 and world == 1 and not args.no_per_config:
        head = (args.workload, {
            "us": ms * 1e3, "cublas_dense_us": dense_ms * 1e3,
            "speedup_vs_cublas_dense": dense_ms / ms,
            "dense_equiv_tflops": dense_flops / (ms * 1e-3) / 1e12,
            "layer_roofline_us": layer_roof_us, "layer_roofline_frac": layer_roof_us / (ms * 1e3),
            "device_status": status,
            "rel_fro_vs_oracle": line.get("parity", {}).get("rel_fro_vs_oracle"),
            "tol": line.get("parity", {}).get("tol"), "note": "the headline's own timed region"})
        if "parity" not in line:
            head = None
        for r in runs:
            r.close()
        runs = []
        entries, clk_pc = per_config(workload_names(), dev, pk, args.per_config_steps, 5, head)
        line["per_config"] = entries
        line["per_config_clocks"] = clk_pc
        line["per_config_steps"] = args.per_config_steps
        line["extras"] = extras(dev, args.per_config_steps, 5)
    for r in runs:
        r.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------------- oracle ----

def static_errors(statics):
    """The FLOPs-matched static layers on the oracle's sample rows: their
    approximation error relative to the dense product, and the GPU result
    against the oracle's weight-only product of the same rounded factors."""
    import oracle
    errs, pars = [], []
    for r, rs, _, Ys in statics:
        s, w = r.s, r.w
        rows = parity_rows(s)
        Xr = oracle.round_to(w.X[rows], s.dtype)
        Us = oracle.round_to(w.left[:, :rs] * w.sigma[:rs], s.dtype)
        Vs = oracle.round_to(w.right[:, :rs], s.dtype)
        Yo = oracle.weight_only(Xr, Us, Vs)
        Yd = oracle.dense(Xr, w.weight())
        Yg = Ys[torch_index(rows, Ys.device)].double().cpu().numpy()
        errs.append(oracle.rel_fro(Yo, Yd))
        pars.append(oracle.rel_fro(Yg, Yo))
    return {"oracle_err_vs_dense": errs, "rel_fro_vs_oracle": max(pars)}


def oracle_inputs(s, w):
    import oracle
    f = oracle.offline_prepare_from_svd(w.left, w.sigma, w.right, s.r, s.k, s.lam)
    return f, [oracle.round_to(a, s.dtype) for a in (w.X, f.U, f.V, f.P, f.W_res)]


def cpu_baseline(runs, budget_s: float = 10.0):
    """The oracle on the host cores over a bounded sample of whole instances
    of each layer of the step (about `budget_s` of work in all)."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    flops, secs, parts = 0.0, 0.0, []
    for r in runs:
        s = r.s
        _, (Xr, Ur, Vr, Pr, Wr) = oracle_inputs(s, r.w)
        t0 = time.perf_counter()
        oracle.inference(Xr[: s.T], Ur, Vr, Pr, Wr, s.lam, 1, s.T)
        t1 = time.perf_counter() - t0
        n_inst = int(max(1, min(s.B, (budget_s / len(runs)) // max(t1, 1e-3))))
        t0 = time.perf_counter()
        oracle.inference(Xr[: n_inst * s.T], Ur, Vr, Pr, Wr, s.lam, n_inst, s.T)
        secs += time.perf_counter() - t0
        flops += 2.0 * n_inst * s.T * s.d_in * s.d_out
        parts.append("%s: %d of %d instances (%d rows)" % (s.name, n_inst, s.B, n_inst * s.T))
    return {"value": flops / secs / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": "; ".join(parts) + "; fp64 NumPy, %.2f s" % secs}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from synth import generate
    ss = specs_of(args.workload)
    prepared = []
    for s in ss:
        _, arrs = oracle_inputs(s, generate(s))
        prepared.append((s, arrs))
    cores = len(os.sched_getaffinity(0))
    # each step a bounded sample of whole instances of every layer, sized so
    # that the whole run (warm-up included) takes about two minutes of host time
    per_step = 120.0 / (args.steps + args.warmup) / len(prepared)
    plan = []
    for s, (Xr, Ur, Vr, Pr, Wr) in prepared:
        t0 = time.perf_counter()
        oracle.inference(Xr[: s.T], Ur, Vr, Pr, Wr, s.lam, 1, s.T)
        t1 = time.perf_counter() - t0
        n_inst = int(max(1, min(s.B, per_step // max(t1, 1e-4))))
        plan.append((s, n_inst, (Xr, Ur, Vr, Pr, Wr)))

    def one_step():
        for s, n, (Xr, Ur, Vr, Pr, Wr) in plan:
            oracle.inference(Xr[: n * s.T], Ur, Vr, Pr, Wr, s.lam, n, s.T)

    for _ in range(args.warmup):
        one_step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        one_step()
        times.append(time.perf_counter() - t0)
    t = float(np.mean(times))
    flops = sum(2.0 * n * s.T * s.d_in * s.d_out for s, n, _ in plan)
    value = flops / t / 1e12
    sample = "; ".join("%s: %d of %d instances (%d rows)" % (s.name, n, s.B, n * s.T)
                       for s, n, _ in plan) + " per step, fp64 NumPy"
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": DATA,
            "config": config_of(args.workload, world),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=HEADLINE, choices=workload_names())
    ap.add_argument("--impl", choices=("dyra", "reference"), default="dyra")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the sweep over every workload after the headline")
    ap.add_argument("--per-config-steps", type=int, default=100)
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
