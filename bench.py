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


def fwd_algorithmic_bytes(w, with_write_gate=False) -> int:
    """Algorithmic bytes of one forward call: the recurrence's five token inputs (q, k, v
    and the form's erase arguments at the input dtype, log w fp32) in and o (fp32) out, per
    token and head -- 2048 B on the GDN-2 bf16 d = 128 workload.  The written value is
    v itself (the Muir page feeds the kernel w (.) v); this API also accepts GDN-2's write
    gate as a separate tensor, whose bytes ``with_write_gate`` adds (2304 B per token-head
    there).  The final state (one d_k x d_v block per sequence) is not counted."""
    eb = 2 if w.dtype == "bf16" else 4
    extra = {"gdn2": w.dk + (w.dv if with_write_gate else 0),   # erase gate b (+ write gate)
             "rwkv7": w.dk + 1,          # removal direction a, coefficient c
             "general": 2 * w.dk,        # u, z
             "gla": 0}[w.form]
    per_token_head = eb * (2 * w.dk + w.dv + extra) + 4 * w.dk + 4 * w.dv
    return w.B * w.T * w.H * per_token_head


def bwd_algorithmic_bytes(w) -> int:
    """Reverse mode: the forward's token inputs and dO (fp32) in, every gradient out
    (fp32: q, k, log_w, v and the form's erase arguments)."""
    eb = 2 if w.dtype == "bf16" else 4
    extra = {"gdn2": w.dk + w.dv, "rwkv7": w.dk + 1, "general": 2 * w.dk, "gla": 0}[w.form]
    per_in = eb * (2 * w.dk + w.dv + extra) + 4 * w.dk + 4 * w.dv
    per_out = 4 * (3 * w.dk + w.dv + extra)
    return w.B * w.T * w.H * (per_in + per_out) + w.B * w.H * w.dk * w.dv * 4


def muir_algorithmic_bytes(w) -> int:
    """The Muir mixer: the activations q, k, v and the gate logits z_f, z_b, z_w, z_q, z_g
    in (input dtype), y out (fp32), S_T out."""
    eb = 2 if w.dtype == "bf16" else 4
    per_token_head = eb * (5 * w.dk + 3 * w.dv) + 4 * w.dv
    return w.B * w.T * w.H * per_token_head + w.B * w.H * w.dk * w.dv * 4


def mlstm_algorithmic_bytes(w) -> int:
    """xLSTM's mLSTM cell: q, k, v in (input dtype), the two fp32 gate pre-activations in,
    h out (fp32), the final state out."""
    eb = 2 if w.dtype == "bf16" else 4
    per_token_head = eb * (2 * w.dk + w.dv) + 8 + 4 * w.dv
    return w.B * w.T * w.H * per_token_head + w.B * w.H * (w.dk * w.dv + w.dk + 1) * 4


def fwd_flops(w) -> int:
    """Algorithmic flops of the single-write (GDN-2) chunk form per token-head:
    6 d^2 (state GEMMs Y S0, Q S0, K~^T V~) + 5 C d (L, M, [U Y], M V~) + C^2 / 3 (T^-1)."""
    d, C = w.dk, w.chunk
    return int(w.B * w.T * w.H * (6 * d * d + 5 * C * d + C * C / 3))


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum from one ncu capture of the
# current kernels on a half-size case, scaled by the units processed).  Forward: prep +
# chain, per (b, h, 64-token chunk) of the GDN-2 bf16 d = 128 tensor-core path (B = 2, 2048
# chunks: prep 235.0 MB read + 109.9 MB written, chain 152.1 MB read + 38.7 MB written);
# decode: per (b, h) step of the d = 128 persistent kernel.  Must be re-measured when those
# kernels change.
FWD_TC_TRAFFIC_PER_CHUNK = (235030528 + 109881344 + 152095488 + 38657536) / 2048
DEC_TRAFFIC_PER_HEAD = (137.9e6 + 81.0e6) / (64 * 32)


def dec_algorithmic_bytes(w) -> int:
    eb = 2
    state = 2 * w.B * w.H * w.dk * w.dv * 4
    tok = w.B * w.H * (eb * (3 * w.dk + 2 * w.dv) + 4 * w.dk + 4 * w.dv)
    return state + tok


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own shard of sequences (weak scaling, no collective)."""
    return base + 1000 * rank


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
    """Samples SM clocks and clock-event (throttle) reasons during a timed region.

    Uses NVML from a background thread (about every 2 ms, so even a region of a
    few milliseconds gets samples); falls back to ``nvidia-smi -lms 20``.  Reads
    settings only; changes nothing on the GPU.
    """
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, uuid):
        self.uuid = uuid
        self.samples = []
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self._proc = None
        self._path = None

    def _nvml_loop(self, nv, handle):
        import time as _t
        masks = [(n, getattr(nv, c, 0)) for n, c in self.REASONS]
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
                bits = get_reasons(handle)
                self.samples.append((float(mhz), [n for n, m in masks if bits & m]))
            except Exception:
                pass
            _t.sleep(0.002)

    def __enter__(self):
        try:
            import threading
            import pynvml as nv
            nv.nvmlInit()
            handle = nv.nvmlDeviceGetHandleByUUID(self.uuid)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM))
            self._stop = threading.Event()
            self._thread = threading.Thread(target=self._nvml_loop, args=(nv, handle), daemon=True)
            self._thread.start()
            return self
        except Exception:
            self._thread = None
        try:
            fd, self._path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.uuid}",
                 "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                 "clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self._path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self._proc = None
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
            for line in open(self._path):
                parts = [x.strip() for x in line.split(",")]
                try:
                    self.max_mhz = float(parts[1])
                    self.samples.append((float(parts[0]), [n for (n, _), x in
                                                          zip(self.REASONS, parts[2:6])
                                                          if x.lower() == "active"]))
                except (ValueError, IndexError):
                    continue
            os.unlink(self._path)

    def summary(self):
        if not self.samples:
            return None
        reasons = sorted({r for _, rs in self.samples for r in rs})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


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
    return token_heads_per_s / w.H, cores, (f"{n} of {heads} heads x {w.T} tokens, fp64 oracle: "
                                            f"{dt:.1f} s on {cores} threads = {dt * cores:.0f} CPU-s")


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
class Ctx:
    """Device, stream and the rank plumbing (barrier, max over ranks)."""

    def __init__(self, torch, dist, world, rank, local, device=None):
        self.torch, self.dist = torch, dist
        self.world, self.rank, self.local = world, rank, local
        # the rank plumbing also runs on the host (gloo) for the multi-process tests
        self.dev = device if device is not None else torch.device("cuda", local)
        self.stream = torch.cuda.current_stream() if self.dev.type == "cuda" else None
        self.peaks = load_peaks()
        self.uuid = str(local)
        if self.dev.type == "cuda":
            try:
                self.uuid = "GPU-" + str(torch.cuda.get_device_properties(self.dev).uuid)
            except Exception:
                pass

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max_over_ranks(self, x):
        if self.world == 1:
            return x
        t = self.torch.tensor([x], dtype=self.torch.float64, device=self.dev)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def event(self):
        return self.torch.cuda.Event(enable_timing=True)


def bench_forward(ctx, args, gdr):
    """Device-resident chunked forward: K timed steps, kernel time per launch."""
    torch = ctx.torch
    w = FWD if args.fwd_workload is None else synth.PRESETS[args.fwd_workload]
    if args.fwd_batch is not None:
        w = w.with_(B=args.fwd_batch)
    inp = synth.forward_inputs(w, seed=rank_seed(w.seed, ctx.rank))
    names = ("q", "k", "v", "log_w", "e1", "e2")
    d = gdr.to_device({k: inp[k] for k in names}, w.dtype, ctx.dev)
    o = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device=ctx.dev)
    S_T = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=ctx.dev)
    ws = gdr.new_workspace(gdr.gdr_forward_workspace_size(w.form, d["q"], d["k"], d["v"],
                                                          d["log_w"], d["e1"], d["e2"],
                                                          w.chunk, args.algo), ctx.dev)

    def step(bufs):
        gdr.gdr_forward_chunked(w.form, bufs["q"], bufs["k"], bufs["v"], bufs["log_w"],
                                bufs["e1"], bufs["e2"], None, chunk=w.chunk, algo=args.algo,
                                o=o, S_T=S_T, workspace=ws)

    evs = [(ctx.event(), ctx.event()) for _ in range(args.steps)]
    t0, t1 = ctx.event(), ctx.event()
    # The clock sampler runs from the warm-up through the timed region: a timed
    # region of a few milliseconds is shorter than nvidia-smi's sampling period.
    with ClockSampler(ctx.uuid) as clk:
        for _ in range(max(args.warmup, 1)):
            step(d)
        torch.cuda.synchronize()
        status = gdr.gdr_read_status(ws)
        if status != "GDR_OK":
            raise RuntimeError(f"device status after warm-up: {status}")
        ctx.barrier()
        torch.cuda.synchronize()
        t0.record(ctx.stream)
        for i in range(args.steps):
            evs[i][0].record(ctx.stream)
            step(d)
            evs[i][1].record(ctx.stream)
        t1.record(ctx.stream)
        torch.cuda.synchronize()
        ctx.barrier()
    status = gdr.gdr_read_status(ws)
    if status != "GDR_OK":
        raise RuntimeError(f"device status after the timed steps: {status}")
    ms_total = ctx.max_over_ranks(t0.elapsed_time(t1))
    ms_kernel = statistics.mean(a.elapsed_time(b) for a, b in evs)
    # launches per call: the two-kernel tensor-core path runs a prep and a chain kernel;
    # every other path is one kernel
    kernel = gdr.gdr_forward_kernel_name(w.form, d["q"], d["k"], d["v"], d["log_w"], d["e1"],
                                         d["e2"], chunk=w.chunk, algo=args.algo,
                                         workspace_bytes=ws.numel())
    per_call = 2 if kernel == "tc_split" else 1
    res = {"w": w, "ms_per_step": ms_total / args.steps, "ms_kernel": ms_kernel,
           "clocks": clk.summary(), "launches": args.steps * per_call,
           "launches_per_call": per_call, "kernel": kernel}
    if args.only == "all":
        res["e2e"] = bench_e2e(ctx, args, gdr, w, inp, names, ws)
    return res


def bench_other_workloads(ctx, args, gdr):
    """The other forward workloads, device-resident, through the same call (algo auto):
    milliseconds per call and the HBM roofline fraction of their algorithmic bytes."""
    torch = ctx.torch
    out = []
    for name in ("rwkv7_bf16", "gdn2_long", "rwkv7_f32"):
        w = synth.PRESETS[name]
        inp = synth.forward_inputs(w, seed=rank_seed(w.seed, ctx.rank))
        names = ("q", "k", "v", "log_w", "e1", "e2")
        d = gdr.to_device({k: inp[k] for k in names}, w.dtype, ctx.dev)
        del inp
        ws = gdr.new_workspace(gdr.gdr_forward_workspace_size(w.form, d["q"], d["k"], d["v"],
                                                              d["log_w"], d["e1"], d["e2"],
                                                              w.chunk, args.algo), ctx.dev)
        kernel = gdr.gdr_forward_kernel_name(w.form, d["q"], d["k"], d["v"], d["log_w"], d["e1"],
                                             d["e2"], chunk=w.chunk, algo=args.algo,
                                             workspace_bytes=ws.numel())

        def call():
            return gdr.gdr_forward_chunked(w.form, d["q"], d["k"], d["v"], d["log_w"], d["e1"],
                                           d["e2"], None, chunk=w.chunk, algo=args.algo,
                                           workspace=ws)
        for _ in range(2):
            call()
        torch.cuda.synchronize()
        e0, e1 = ctx.event(), ctx.event()
        n = 5
        e0.record(ctx.stream)
        for _ in range(n):
            call()
        e1.record(ctx.stream)
        torch.cuda.synchronize()
        status = gdr.gdr_read_status(ws)
        if status != "GDR_OK":
            raise RuntimeError(f"device status after {name}: {status}")
        ms = ctx.max_over_ranks(e0.elapsed_time(e1)) / n
        nbytes = fwd_algorithmic_bytes(w)
        gbs = nbytes / (ms * 1e-3) / 1e9
        nbytes_wg = fwd_algorithmic_bytes(w, with_write_gate=True)
        out.append({"workload": name, "form": w.form, "dtype": w.dtype, "B": w.B, "H": w.H,
                    "T": w.T, "dk": w.dk, "dv": w.dv, "chunk": w.chunk, "kernel": kernel,
                    "ms_per_call": ms,
                    "tokens_per_s": w.tokens * ctx.world / (ms * 1e-3),
                    "roofline": {"bound": "hbm", "achieved": gbs, "peak": ctx.peaks["hbm_gbs"],
                                 "unit": "GB/s", "frac": gbs / ctx.peaks["hbm_gbs"],
                                 "bytes_per_call": nbytes,
                                 "frac_with_write_gate": nbytes_wg / (ms * 1e-3) / 1e9
                                 / ctx.peaks["hbm_gbs"]}})
        del d, ws
        torch.cuda.empty_cache()
    return out


def bench_backward(ctx, args, gdr):
    """gdr_backward_chunked on the bf16 forward workloads, device-resident (S0 = 0,
    dS_T = 0, random dO): milliseconds per call and the HBM roofline fraction of the
    algorithmic bytes (inputs and dO in, every gradient out)."""
    torch = ctx.torch
    out = []
    for name in ((args.bwd_workload,) if args.bwd_workload else ("gdn2_bf16", "rwkv7_bf16")):
        w = synth.PRESETS[name]
        if args.bwd_batch:
            w = w.with_(B=args.bwd_batch)
        inp = synth.forward_inputs(w, seed=rank_seed(w.seed, ctx.rank))
        names = ("q", "k", "v", "log_w", "e1", "e2")
        d = gdr.to_device({k: inp[k] for k in names}, w.dtype, ctx.dev)
        del inp
        gen = torch.Generator(device=ctx.dev).manual_seed(rank_seed(w.seed + 100, ctx.rank))
        dO = torch.randn((w.B, w.T, w.H, w.dv), generator=gen, device=ctx.dev)
        ws = gdr.new_workspace(gdr.gdr_backward_workspace_size(w.form, d["q"], d["k"], d["v"],
                                                               d["log_w"], d["e1"], d["e2"]),
                               ctx.dev)
        grads = None

        def call():
            return gdr.gdr_backward_chunked(w.form, d["q"], d["k"], d["v"], d["log_w"], d["e1"],
                                            d["e2"], None, dO, None, workspace=ws, grads=grads)
        grads = call()
        for _ in range(2):
            call()
        torch.cuda.synchronize()
        e0, e1 = ctx.event(), ctx.event()
        n = 5
        e0.record(ctx.stream)
        for _ in range(n):
            call()
        e1.record(ctx.stream)
        torch.cuda.synchronize()
        ms = ctx.max_over_ranks(e0.elapsed_time(e1)) / n
        nbytes = bwd_algorithmic_bytes(w)
        gbs = nbytes / (ms * 1e-3) / 1e9
        out.append({"workload": name, "form": w.form, "dtype": w.dtype, "B": w.B, "H": w.H,
                    "T": w.T, "dk": w.dk, "dv": w.dv, "ms_per_call": ms, "launches_per_call": 3,
                    "tokens_per_s": w.tokens * ctx.world / (ms * 1e-3),
                    "workspace_bytes": int(ws.numel()),
                    "roofline": {"bound": "hbm", "achieved": gbs, "peak": ctx.peaks["hbm_gbs"],
                                 "unit": "GB/s", "frac": gbs / ctx.peaks["hbm_gbs"],
                                 "bytes_per_call": nbytes}})
        del d, ws, grads, dO
        torch.cuda.empty_cache()
    return out


def bench_muir(ctx, args, gdr):
    """gdr_muir_forward (the Muir token mixer around the GDN-2 recurrence) on the headline
    shapes, device-resident, fused (activations inside the tensor-core forward) and with
    the separate prologue kernel: milliseconds per call and the HBM roofline fraction."""
    torch = ctx.torch
    w = synth.PRESETS["gdn2_bf16"]
    inp = synth.muir_inputs(w, seed=rank_seed(w.seed + 10, ctx.rank))
    names = ("q", "k", "v", "zf", "zb", "zw", "zq", "zg")
    d = {k: torch.from_numpy(inp[k]).to(ctx.dev, torch.bfloat16) for k in names}
    par = {k: torch.from_numpy(inp[k]).to(ctx.dev) for k in ("a_log", "gamma_stat", "rms_weight")}
    out = {"workload": "muir on " + w.name, "B": w.B, "H": w.H, "T": w.T, "dk": w.dk, "dv": w.dv}
    nbytes = muir_algorithmic_bytes(w)
    for key, unfused in (("fused", False), ("unfused", True)):
        ws = gdr.new_workspace(gdr.gdr_muir_workspace_size(d["q"], d["k"], d["v"], w.chunk,
                                                           args.algo, unfused), ctx.dev)
        y = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device=ctx.dev)

        def call():
            gdr.gdr_muir_forward(*(d[k] for k in names), par["a_log"], par["gamma_stat"],
                                 par["rms_weight"], 1e-6, None, chunk=w.chunk, algo=args.algo,
                                 unfused=unfused, y=y, want_state=False, workspace=ws)
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        e0, e1 = ctx.event(), ctx.event()
        n = 5
        e0.record(ctx.stream)
        for _ in range(n):
            call()
        e1.record(ctx.stream)
        torch.cuda.synchronize()
        ms = ctx.max_over_ranks(e0.elapsed_time(e1)) / n
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[key] = {"ms_per_call": ms, "tokens_per_s": w.tokens * ctx.world / (ms * 1e-3),
                    "launches_per_call": 3 if not unfused else 4,
                    "roofline": {"bound": "hbm", "achieved": gbs, "peak": ctx.peaks["hbm_gbs"],
                                 "unit": "GB/s", "frac": gbs / ctx.peaks["hbm_gbs"],
                                 "bytes_per_call": nbytes}}
        del ws, y
    del d, par
    torch.cuda.empty_cache()
    return out


def bench_mlstm(ctx, args, gdr):
    """gdr_mlstm_forward (xLSTM's mLSTM cell with the stabilizer) on the bf16 shapes of the
    two forward workloads, device-resident: milliseconds per call and the HBM roofline
    fraction of the algorithmic bytes."""
    torch = ctx.torch
    out = []
    for name in ("gdn2_bf16", "rwkv7_bf16"):
        w = synth.PRESETS[name]
        inp = synth.mlstm_inputs(w, seed=rank_seed(w.seed + 20, ctx.rank))
        d = {k: torch.from_numpy(inp[k]).to(ctx.dev, torch.bfloat16) for k in ("q", "k", "v")}
        g = {k: torch.from_numpy(inp[k]).to(ctx.dev) for k in ("f_pre", "i_pre")}
        h = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device=ctx.dev)

        def call():
            gdr.gdr_mlstm_forward(d["q"], d["k"], d["v"], g["f_pre"], g["i_pre"], h=h,
                                  want_state=False)
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        e0, e1 = ctx.event(), ctx.event()
        n = 5
        e0.record(ctx.stream)
        for _ in range(n):
            call()
        e1.record(ctx.stream)
        torch.cuda.synchronize()
        ms = ctx.max_over_ranks(e0.elapsed_time(e1)) / n
        nbytes = mlstm_algorithmic_bytes(w)
        gbs = nbytes / (ms * 1e-3) / 1e9
        out.append({"workload": "mlstm on " + name, "B": w.B, "H": w.H, "T": w.T, "dk": w.dk,
                    "dv": w.dv, "ms_per_call": ms, "launches_per_call": 1,
                    "tokens_per_s": w.tokens * ctx.world / (ms * 1e-3),
                    "roofline": {"bound": "hbm", "achieved": gbs, "peak": ctx.peaks["hbm_gbs"],
                                 "unit": "GB/s", "frac": gbs / ctx.peaks["hbm_gbs"],
                                 "bytes_per_call": nbytes}})
        del d, g, h
        torch.cuda.empty_cache()
    return out


def bench_gemm_phases(ctx, fwd):
    """The chunked forward's tensor-core phases, measured: the same kernels built with their
    timing hooks (libgdr_timing.so) run the timed forward workload; each MMA group is
    timed from the issue of its first MMA to its completion (the issuing warp waits for every
    group), and its bf16 FLOPs over those cycles, at the SM clock seen during the timed
    forward steps, are compared with the measured dense bf16 peak.  Per kernel (all its
    groups together) and per group."""
    try:
        from matrix_memory_rnn_b200 import phase_timing
        m = phase_timing.measure(batch=fwd["w"].B, calls=2)
        clk = (fwd.get("clocks") or {}).get("sm_mhz") or 1965.0
        fr = phase_timing.gemm_phase_fractions(m, ctx.peaks["bf16_tflops"], clk)
        return {"method": "timing build, same workload: MMA group issue-to-completion cycles, groups "
                          "waited for one at a time; FLOPs of the groups over their cycles at the "
                          "forward's SM clock, against the measured bf16 peak",
                "sm_mhz": clk, "peak_tflops": ctx.peaks["bf16_tflops"],
                "kernels": {k: {"frac": v["frac"], "tflops": v["tflops"],
                                "groups": [{kk: g[kk] for kk in ("group", "cycles", "frac")}
                                           for g in v["groups"]]}
                            for k, v in fr.items()}}
    except Exception as exc:      # the timing build is optional: report why it is missing
        return {"unavailable": f"{type(exc).__name__}: {exc}"}


def bench_e2e(ctx, args, gdr, w, inp, names, ws):
    """The same call with host inputs, as a pipelined loop: every step copies its inputs
    from pinned host memory to the device, runs the forward and copies o back to pinned
    host memory, all inside the timed region.  Two buffer sets on three streams (upload,
    compute, download) let step i + 1's upload and step i - 1's download overlap step i
    (PCIe is full duplex); a buffer is reused only after the step that used it finished."""
    torch = ctx.torch
    host = {k: None if inp[k] is None else torch.from_numpy(inp[k]) for k in names}
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    pinned = {k: None if t is None else
              t.to(torch.float32 if k == "log_w" else tdt).pin_memory() for k, t in host.items()}
    dev = [{k: None if t is None else torch.empty(t.shape, dtype=t.dtype, device=ctx.dev)
            for k, t in pinned.items()} for _ in range(2)]
    o = [torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device=ctx.dev) for _ in range(2)]
    o_host = [torch.empty(o[0].shape, dtype=torch.float32, pin_memory=True) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in pinned.values() if t is not None)
    d2h = o[0].numel() * 4
    s_in, s_out, s_comp = torch.cuda.Stream(), torch.cuda.Stream(), ctx.stream
    in_done, comp_done, out_done = ([ctx.event() for _ in range(2)] for _ in range(3))

    def e2e_step(i):
        b = i % 2
        s_in.wait_event(comp_done[b])        # the step that last read dev[b] has finished
        with torch.cuda.stream(s_in):
            for k, t in pinned.items():
                if t is not None:
                    dev[b][k].copy_(t, non_blocking=True)
            in_done[b].record(s_in)
        s_comp.wait_event(in_done[b])
        s_comp.wait_event(out_done[b])       # o[b] has been read back
        with torch.cuda.stream(s_comp):
            bb = dev[b]
            gdr.gdr_forward_chunked(w.form, bb["q"], bb["k"], bb["v"], bb["log_w"], bb["e1"],
                                    bb["e2"], None, chunk=w.chunk, algo=args.algo, o=o[b],
                                    want_state=False, workspace=ws, stream=s_comp)
            comp_done[b].record(s_comp)
        s_out.wait_event(comp_done[b])
        with torch.cuda.stream(s_out):
            o_host[b].copy_(o[b], non_blocking=True)
            out_done[b].record(s_out)

    n = max(3, min(args.steps, 10))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    ctx.barrier()
    e0, e1 = ctx.event(), ctx.event()
    e0.record(s_in)
    s_comp.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(n):
        e2e_step(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = ctx.max_over_ranks(e0.elapsed_time(e1)) / n
    return {"value": w.tokens * ctx.world / (ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "pipeline": "2 buffer sets; upload, compute and download on separate streams"}


def bench_decode(ctx, args, gdr):
    """Decode step on the resident 1 GiB state, inputs cycled from 8 seeded steps."""
    torch = ctx.torch
    dw = DEC if args.dec_batch is None else DEC.with_(B=args.dec_batch)
    S = torch.from_numpy(synth.decode_state(dw, seed=rank_seed(dw.seed, ctx.rank))).to(ctx.dev)
    names = ("q", "k", "v", "log_w", "e1", "e2")
    pool = [gdr.to_device({k: p[k] for k in names}, "bf16", ctx.dev)
            for p in (synth.decode_step_inputs(dw, s, seed=rank_seed(dw.seed, ctx.rank))
                      for s in range(8))]
    o_dec = torch.empty((dw.B, dw.H, dw.dv), dtype=torch.float32, device=ctx.dev)

    def step(i):
        p = pool[i % len(pool)]
        gdr.gdr_decode_step(dw.form, p["q"], p["k"], p["v"], p["log_w"], p["e1"], p["e2"], S,
                            o=o_dec)

    d0, d1 = ctx.event(), ctx.event()
    with ClockSampler(ctx.uuid) as clk:
        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize()
        ctx.barrier()
        d0.record(ctx.stream)
        for i in range(args.decode_steps):
            step(i)
        d1.record(ctx.stream)
        torch.cuda.synchronize()
    ms = ctx.max_over_ranks(d0.elapsed_time(d1)) / args.decode_steps
    nbytes = dec_algorithmic_bytes(dw)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": dw.name, "form": dw.form, "B": dw.B, "H": dw.H, "dk": dw.dk,
            "dv": dw.dv, "steps": args.decode_steps, "steps_per_s": 1e3 / ms,
            "ms_per_step": ms,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": ctx.peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / ctx.peaks["hbm_gbs"],
                         "traffic": (DEC_TRAFFIC_PER_HEAD * dw.B * dw.H
                                     if dw.dk == dw.dv == 128 and dw.form != "rwkv7" else None),
                         "bytes_per_launch": nbytes, "peak_source": ctx.peaks["source"]},
            "gpu_launches": args.decode_steps, "clocks": clk.summary()}


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
    ap.add_argument("--fwd-workload", default=None, choices=sorted(synth.PRESETS),
                    help="forward workload (default: the GDN-2 headline); for profiler captures")
    ap.add_argument("--fwd-batch", type=int, default=None,
                    help="forward batch B (default: the workload's); smaller values make "
                         "profiler captures cheaper and are not bench results")
    ap.add_argument("--dec-batch", type=int, default=None,
                    help="decode batch B (default: the workload's); for profiler captures")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the timing of the other forward workloads")
    ap.add_argument("--no-mlstm", action="store_true",
                    help="skip the timing of the mLSTM cell (gdr_mlstm_forward)")
    ap.add_argument("--no-muir", action="store_true",
                    help="skip the timing of the Muir mixer (gdr_muir_forward)")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the timing of the reverse mode (gdr_backward_chunked)")
    ap.add_argument("--bwd-workload", default=None, choices=["gdn2_bf16", "rwkv7_bf16"],
                    help="reverse-mode workload (default: both); for profiler captures")
    ap.add_argument("--bwd-batch", type=int, default=None,
                    help="reverse-mode batch B (default: the workload's); for profiler captures")
    ap.add_argument("--no-gemm-phase", action="store_true",
                    help="skip the tensor-core GEMM-phase measurement (timing build, B = 1)")
    ap.add_argument("--only", default="all",
                    choices=["all", "forward", "decode", "backward", "muir", "mlstm"],
                    help="time one part only (profiling runs); the default line needs 'all'")
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
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    ctx = Ctx(torch, dist, world, rank, local)

    fwd = bench_forward(ctx, args, gdr) if args.only in ("all", "forward") else None
    dec = bench_decode(ctx, args, gdr) if args.only in ("all", "decode") else None
    # every rank times its own shard of these too (same collective steps on all ranks)
    others = (bench_other_workloads(ctx, args, gdr)
              if args.only == "all" and not args.no_other_workloads else None)
    bwd = (bench_backward(ctx, args, gdr)
           if (args.only == "all" and not args.no_backward) or args.only == "backward" else None)
    muir = (bench_muir(ctx, args, gdr)
            if (args.only == "all" and not args.no_muir) or args.only == "muir" else None)
    mlstm = (bench_mlstm(ctx, args, gdr)
             if (args.only == "all" and not args.no_mlstm) or args.only == "mlstm" else None)
    gemm = None
    if args.only in ("all", "forward") and not args.no_gemm_phase and fwd is not None:
        gemm = bench_gemm_phases(ctx, fwd)
    ctx.barrier()
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    line = {"metric": METRIC, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic"}
    if fwd is not None:
        w = fwd["w"]
        nbytes, nflops = fwd_algorithmic_bytes(w), fwd_flops(w)
        nbytes_wg = fwd_algorithmic_bytes(w, with_write_gate=True)
        achieved = nbytes / (fwd["ms_kernel"] * 1e-3) / 1e9
        tflops = nflops / (fwd["ms_kernel"] * 1e-3) / 1e12
        line.update({
            "value": w.tokens * world / (fwd["ms_per_step"] * 1e-3),
            "ms_per_step": fwd["ms_per_step"],
            "config": {"workload": w.name, "form": w.form, "B": w.B, "H": w.H, "T": w.T,
                       "dk": w.dk, "dv": w.dv, "chunk": w.chunk, "algo": args.algo,
                       "parallelism": f"dp{world} (independent sequences, no collective)",
                       "l2": f"inputs larger than L2 ({nbytes / 2**20:.0f} MiB per step > 126 MiB)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": ctx.peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / ctx.peaks["hbm_gbs"],
                         "kernel_path": fwd["kernel"],
                         "traffic": (FWD_TC_TRAFFIC_PER_CHUNK * w.B * w.H * -(-w.T // 64)
                                     if fwd["launches_per_call"] == 2 else None),
                         "peak_source": ctx.peaks["source"],
                         "bytes_per_launch": nbytes, "kernel_ms": fwd["ms_kernel"],
                         "bytes_with_write_gate": nbytes_wg,
                         "frac_with_write_gate": nbytes_wg / (fwd["ms_kernel"] * 1e-3) / 1e9
                         / ctx.peaks["hbm_gbs"],
                         "scope": "one forward call (%d kernel launch%s)" % (
                             fwd["launches_per_call"],
                             "es" if fwd["launches_per_call"] > 1 else "")},
            "tensor": {"flops_per_launch": nflops, "achieved_tflops": tflops,
                       "peak_tflops": ctx.peaks["bf16_tflops"],
                       "frac": tflops / ctx.peaks["bf16_tflops"],
                       "gemm_phase": gemm},
            "gpu_launches": fwd["launches"], "clocks": fwd["clocks"]})
        if "e2e" in fwd:
            line["e2e"] = fwd["e2e"]
        if not args.no_cpu_baseline and world == 1:
            v_cpu, cores, sample = oracle_sample_rate(w, budget_s=15.0)
            line["cpu_baseline"] = {"value": v_cpu, "unit": UNIT, "cores": cores,
                                    "kind": "oracle", "sample": sample}
    if dec is not None:
        line["decode"] = dec
    if others is not None:
        line["other_workloads"] = others
    if bwd is not None:
        line["backward"] = bwd
    if muir is not None:
        line["muir"] = muir
    if mlstm is not None:
        line["mlstm"] = mlstm
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
