#!/usr/bin/env python
"""Benchmark of the generalized delta-rule hot path on B200.

One step = one ``gdr_forward_chunked`` call over the GDN-2 bf16 workload
(B=4, H=16, T=4096, d_k=d_v=128, chunk 64; every chunk step a1-a5 runs inside
it), timed with CUDA events on the launching stream.  The decode step
(B=256, H=32, d=128, fp32 state, GDN-2) is timed alongside and reported under
"decode".  Inputs are seeded synthetic data shaped like the pages' workloads
(``matrix_memory_rnn_b200.synth``).

Multi-GPU: every (b, h) sequence is independent, so each rank runs its own full
workload with no collective on the data path (weak scaling); torch.distributed
is used only for the barrier and the max-over-ranks timing.

``--impl reference`` times the fp64 CPU oracle instead, on a bounded sample of
the same workload, and prints the same JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from matrix_memory_rnn_b200 import synth  # noqa: E402

METRIC = "chunked-forward tokens/s and % tensor-core roofline; decode steps/s and HBM GB/s"
UNIT = "tokens/s"
FWD = synth.PRESETS["gdn2_bf16"]
DEC = synth.PRESETS["decode"]
L2_BYTES = 126 * 2 ** 20


def fwd_algorithmic_bytes(w) -> int:
    """q, k, v, erase gate, write gate (bf16), log_w (fp32) in; o (fp32) and S_T out."""
    eb = 2 if w.dtype == "bf16" else 4
    per_token_head = eb * (3 * w.dk + w.dv + w.dv) + 4 * w.dk + 4 * w.dv
    return w.B * w.T * w.H * per_token_head + w.B * w.H * w.dk * w.dv * 4


def fwd_flops(w) -> int:
    """Algorithmic flops of the single-write (GDN-2) chunk form per token-head:
    6 d^2 (state GEMMs Y S0, Q S0, K~^T V~) + 5 C d (L, M, [U Y], M V~) + C^2 / 3 (T^-1)."""
    d, C = w.dk, w.chunk
    return int(w.B * w.T * w.H * (6 * d * d + 5 * C * d + C * C / 3))


def dec_algorithmic_bytes(w) -> int:
    eb = 2
    state = 2 * w.B * w.H * w.dk * w.dv * 4
    tok = w.B * w.H * (eb * (3 * w.dk + 2 * w.dv) + 4 * w.dk + 4 * w.dv)
    return state + tok


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, x in enumerate(r)
                          if x.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------
# CPU side: the oracle as a reported baseline (and the --impl reference arm)
# ----------------------------------------------------------------------------
def oracle_sample_rate(w, budget_s=15.0):
    """Times the fp64 oracle on a bounded sample of workload ``w``: whole heads
    of the full sequence length, as many as fit in about ``budget_s`` seconds.
    Returns (tokens/s scaled to the workload, cores, sample description)."""
    import oracle
    heads = w.B * w.H
    cores = oracle.max_threads()
    one = w.with_(B=1, H=1)
    inp = synth.forward_inputs(one, seed=w.seed)
    t0 = time.perf_counter()
    oracle.forward(w.form, inp["q"], inp["k"], inp["v"], inp["log_w"], inp["e1"], inp["e2"],
                   None, n_threads=1)
    t_one = time.perf_counter() - t0
    n = int(max(1, min(heads, cores * max(1, budget_s // max(t_one, 1e-3)))))
    n = max(cores, n - n % cores) if n >= cores else n
    n = min(n, heads)
    sub = w.with_(B=1, H=n)
    inp = synth.forward_inputs(sub, seed=w.seed)
    t0 = time.perf_counter()
    oracle.forward(w.form, inp["q"], inp["k"], inp["v"], inp["log_w"], inp["e1"], inp["e2"],
                   None, n_threads=cores)
    dt = time.perf_counter() - t0
    token_heads_per_s = n * w.T / dt
    return token_heads_per_s / w.H, cores, f"{n} of {heads} heads x {w.T} tokens, fp64 oracle ({dt:.1f} s)"


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    t_steps = []
    for _ in range(args.warmup):
        oracle_sample_rate(FWD, budget_s=2.0)
    for _ in range(args.steps):
        t_steps.append(oracle_sample_rate(FWD, budget_s=args.ref_budget))
    vals = [v for v, _, _ in t_steps]
    value = statistics.median(vals)
    _, cores, sample = t_steps[-1]
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": FWD.tokens / value * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": FWD.name, "form": FWD.form, "B": FWD.B, "H": FWD.H,
                       "T": FWD.T, "dk": FWD.dk, "dv": FWD.dv, "chunk": FWD.chunk},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# GPU side
# ----------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--algo", default="auto", choices=["auto", "fp32", "tc"])
    ap.add_argument("--decode-steps", type=int, default=50)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-budget", type=float, default=15.0)
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    args.warmup = max(args.warmup, 3)

    import torch
    import torch.distributed as dist
    from matrix_memory_rnn_b200 import gdr

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    peaks = load_peaks()
    stream = torch.cuda.current_stream()

    # ---------------- chunked forward (the headline) ----------------
    w = FWD
    inp = synth.forward_inputs(w, seed=w.seed + 1000 * rank)
    host = {k: None if inp[k] is None else torch.from_numpy(inp[k]) for k in
            ("q", "k", "v", "log_w", "e1", "e2")}
    d = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, w.dtype, dev)
    o = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device=dev)
    S_T = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    ws = gdr.new_workspace(gdr.gdr_forward_workspace_size(w.form, d["q"], d["k"], d["v"],
                                                          d["log_w"], d["e1"], d["e2"],
                                                          w.chunk, args.algo), dev)

    def fwd_step():
        gdr.gdr_forward_chunked(w.form, d["q"], d["k"], d["v"], d["log_w"], d["e1"], d["e2"],
                                None, chunk=w.chunk, algo=args.algo, o=o, S_T=S_T,
                                workspace=ws)

    for _ in range(args.warmup):
        fwd_step()
    torch.cuda.synchronize()
    status = gdr.gdr_read_status(ws)
    if status != "GDR_OK":
        raise RuntimeError(f"device status after warm-up: {status}")

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t_all0, t_all1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_all0.record(stream)
        for i in range(args.steps):
            evs[i][0].record(stream)
            fwd_step()
            evs[i][1].record(stream)
        t_all1.record(stream)
        torch.cuda.synchronize()
        barrier()
    clocks = clk.summary()
    ms_total = max_over_ranks(t_all0.elapsed_time(t_all1))
    ms_kernel = statistics.mean(a.elapsed_time(b) for a, b in evs)
    ms_per_step = ms_total / args.steps
    tokens = w.tokens * world
    value = tokens / (ms_per_step * 1e-3)
    nbytes = fwd_algorithmic_bytes(w)
    nflops = fwd_flops(w)
    achieved = nbytes / (ms_kernel * 1e-3) / 1e9

    # ---------------- e2e through the C-ABI call with host buffers ----------------
    pinned = {k: None if t is None else t.to(d[k].dtype).pin_memory() for k, t in host.items()}
    dev_bufs = {k: None if t is None else torch.empty(t.shape, dtype=t.dtype, device=dev)
                for k, t in pinned.items()}
    o_host = torch.empty(o.shape, dtype=torch.float32, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in pinned.values() if t is not None)
    d2h = o.numel() * 4

    def e2e_step():
        for k, t in pinned.items():
            if t is not None:
                dev_bufs[k].copy_(t, non_blocking=True)
        gdr.gdr_forward_chunked(w.form, dev_bufs["q"], dev_bufs["k"], dev_bufs["v"],
                                dev_bufs["log_w"], dev_bufs["e1"], dev_bufs["e2"], None,
                                chunk=w.chunk, algo=args.algo, o=o, S_T=S_T, workspace=ws)
        o_host.copy_(o, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 10))
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1_.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1_)) / e2e_steps
    e2e_value = tokens / (ms_e2e * 1e-3)

    # ---------------- decode step ----------------
    dw = DEC
    S = torch.from_numpy(synth.decode_state(dw, seed=dw.seed + 1000 * rank)).to(dev)
    pool = [gdr.to_device({k: p[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, "bf16", dev)
            for p in (synth.decode_step_inputs(dw, s, seed=dw.seed + 1000 * rank)
                      for s in range(8))]
    o_dec = torch.empty((dw.B, dw.H, dw.dv), dtype=torch.float32, device=dev)

    def dec_step(i):
        p = pool[i % len(pool)]
        gdr.gdr_decode_step(dw.form, p["q"], p["k"], p["v"], p["log_w"], p["e1"], p["e2"], S,
                            o=o_dec)

    for i in range(args.warmup):
        dec_step(i)
    torch.cuda.synchronize()
    barrier()
    dev0, dev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dev0.record(stream)
    for i in range(args.decode_steps):
        dec_step(i)
    dev1.record(stream)
    torch.cuda.synchronize()
    ms_dec = max_over_ranks(dev0.elapsed_time(dev1)) / args.decode_steps
    dec_bytes = dec_algorithmic_bytes(dw)
    dec_gbs = dec_bytes / (ms_dec * 1e-3) / 1e9

    if world > 1:
        barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        v_cpu, cores, sample = oracle_sample_rate(w, budget_s=15.0)
        cpu = {"value": v_cpu, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "form": w.form, "B": w.B, "H": w.H, "T": w.T,
                   "dk": w.dk, "dv": w.dv, "chunk": w.chunk, "algo": args.algo,
                   "parallelism": f"dp{world} (independent sequences, no collective)",
                   "l2": f"inputs larger than L2 ({nbytes / 2**20:.0f} MiB per step > 126 MiB)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": peaks["source"], "bytes_per_launch": nbytes,
                     "kernel_ms": ms_kernel},
        "tensor": {"flops_per_launch": nflops, "achieved_tflops": nflops / (ms_kernel * 1e-3) / 1e12,
                   "peak_tflops": peaks["bf16_tflops"],
                   "frac": nflops / (ms_kernel * 1e-3) / 1e12 / peaks["bf16_tflops"]},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e},
        "gpu_launches": args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "decode": {"workload": dw.name, "B": dw.B, "H": dw.H, "dk": dw.dk, "dv": dw.dv,
                   "steps": args.decode_steps, "steps_per_s": 1e3 / ms_dec, "ms_per_step": ms_dec,
                   "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": peaks["hbm_gbs"],
                                "unit": "GB/s", "frac": dec_gbs / peaks["hbm_gbs"],
                                "traffic": None, "bytes_per_launch": dec_bytes},
                   "gpu_launches": args.decode_steps},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
