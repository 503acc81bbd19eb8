"""Per-phase cycle accounting of the two-kernel tensor-core forward (GDN-2, bf16, d = 128, C = 64).

Runs the forward through ``libgdr_timing.so`` (the same kernels with their phase marks filled
in, see ``csrc/gdr_phase_timing.cuh``) and prints, per kernel and phase, the average cycles
per chunk of one recording thread per role: the prep kernel's front and back warp groups and
the chain kernel's thread 0.  Each value is the interval that
ends at the phase's mark, so it includes the time that thread waited for the others there.
A second pass times each tensor-core group from the issue of its first MMA to its completion
(the issuing warp then waits for every group, which changes the schedule, so the two passes
are separate).

Usage: ``python -m matrix_memory_rnn_b200.phase_timing [--batch B] [--calls N]`` (one GPU).
"""
from __future__ import annotations

import argparse
import ctypes

import torch

from . import build, gdr, synth

PREP_PHASES = [
    (1, "front: wait for log w, tiles and write gate"), (5, "front: scan: log decay per thread"),
    (6, "front: scan: block totals, barrier"), (7, "front: scan: exclusive prefix, barrier"),
    (2, "front: scan: pivot and exponentials, barrier"),
    (3, "front: operand tiles and V^"), (4, "front: MMA1 issued, chunk handed over"),
    (0, "front: to the next chunk"),
    (9, "back: wait for the hand-over and MMA1"), (10, "back: L and M"),
    (11, "back: T^-1 and its bf16 copy"), (12, "back: MMA2 issued and waited for"),
    (13, "back: U, Y to the record; next tiles requested"), (8, "back: to the next chunk"),
]
CHAIN_PHASES = [
    (1, "wait for MMA3 ([Q_pi; Y] S0)"), (2, "V~ = U - Y S0"), (3, "MMA4 issued and waited for"),
    (4, "state update and its bf16 copy"), (7, "wait for the next chunk's record"),
    (5, "MMA3 of the next chunk issued"), (6, "O read out"),
    (0, "to the next chunk"),
]
# Tensor-core groups timed in the timing build (issue of the first MMA to completion, the
# issuing warp waiting for each group): (slot, group, label, bf16 FLOPs per group).
C, D, NV = 64, 128, 64
MMA_GROUPS = [   # (slot, group, product, shape, FLOPs)
    (1, 0, "[K^ f; Q f] (K g)^T", "M=128 N=64 K=128", 2 * 128 * C * D),
    (1, 1, "T^-1 [V^ | K^ f]", "M=64 N=128 K=64, x2", 2 * 2 * 64 * D * C),
    (0, 0, "[Q_pi; Y] S0", "M=128 N=64 K=128", 2 * 128 * NV * D),
    (0, 1, "K~^T V~ and [M; *] V~", "M=128 N=64 K=64, x2", 2 * 2 * 128 * NV * C),
]


def load_timing_library():
    lib = ctypes.CDLL(build.build(timing=True))
    lib.gdr_forward_chunked.argtypes = [ctypes.POINTER(gdr.gdr_fwd_args), ctypes.c_void_p]
    lib.gdr_forward_chunked.restype = ctypes.c_int
    u64p = ctypes.POINTER(ctypes.c_ulonglong)
    lib.gdr_phase_timing_read.argtypes = [u64p, u64p, u64p, u64p]
    lib.gdr_phase_timing_read.restype = ctypes.c_int
    lib.gdr_phase_timing_read_log.argtypes = [u64p, ctypes.POINTER(ctypes.c_uint), ctypes.POINTER(ctypes.c_uint)]
    lib.gdr_phase_timing_read_log.restype = ctypes.c_int
    return lib


LOG_CTAS, LOG_ENTRIES = 256, 256   # the timing build's interval log (gdr_phase_timing.cuh)


def union_length(spans):
    """Total length of the union of closed intervals [start, end] (each start <= end)."""
    total = 0
    lo = hi = None
    for a, b in sorted(spans):
        if hi is None or a > hi:
            if hi is not None:
                total += hi - lo
            lo, hi = a, b
        else:
            hi = max(hi, b)
    return total + (hi - lo if hi is not None else 0)


def read_union(lib, flops_of):
    """Reads (and clears) the timing build's MMA interval log and returns, per kernel slot,
    [bf16 FLOPs of the logged groups, the summed per-CTA union of their [start, end]
    intervals in SM cycles, groups logged, groups dropped].  The union counts the cycles in
    which a CTA had at least one group in flight once, however many groups overlapped."""
    iv = (ctypes.c_ulonglong * (2 * LOG_CTAS * LOG_ENTRIES * 2))()
    gr = (ctypes.c_uint * (2 * LOG_CTAS * LOG_ENTRIES))()
    cn = (ctypes.c_uint * (2 * LOG_CTAS))()
    rc = lib.gdr_phase_timing_read_log(iv, gr, cn)
    if rc != 0:
        raise RuntimeError(f"gdr_phase_timing_read_log failed: CUDA error {rc}")
    out = {}
    for slot in (0, 1):
        fl = cyc = 0.0
        logged = dropped = 0
        for cta in range(LOG_CTAS):
            n = cn[slot * LOG_CTAS + cta]
            if not n:
                continue
            k = min(n, LOG_ENTRIES)
            dropped += n - k
            logged += k
            base = (slot * LOG_CTAS + cta) * LOG_ENTRIES
            fl += sum(flops_of[(slot, gr[base + j])] for j in range(k))
            cyc += union_length((iv[2 * (base + j)], iv[2 * (base + j) + 1]) for j in range(k))
        out[slot] = [fl, cyc, logged, dropped]
    return out


# Marks of the two-stream kernel (every form at d = 64): (index, label), thread 0 per CTA.
GENERAL_PHASES = [
    (1, "wait for the chunk's inputs, barrier"), (2, "log-decay scan"),
    (3, "operand tiles, barrier"), (4, "MMA1 issued and waited for"),
    (14, "A, B, M_z, M_k: from TMEM"), (15, "A, B, M_z, M_k: masked, stored"),
    (5, "A, B, M_z, M_k: gate loads, fence, barrier"), (6, "B V, K~^T V issued; T^-1; waited for"),
    (7, "B V as bf16"), (8, "MMA2 [Y_u | W] issued and waited for"),
    (9, "Y_u, W to their tiles"), (10, "MMA3 [Q_pi; Y_u] S0' + M_k V issued and waited for"),
    (11, "V~ formed"), (12, "MMA4 issued and waited for"), (13, "state update and output, barrier"),
    (0, "to the next chunk"),
]


def measure_general(preset="rwkv7_bf16", calls=3):
    """The two-stream tensor-core forward (d = 64) on `preset` through the timing build:
    thread 0's cycles per chunk by phase."""
    lib = load_timing_library()
    lib.gdr_general_timing_read.argtypes = [ctypes.POINTER(ctypes.c_ulonglong)]
    lib.gdr_general_timing_read.restype = ctypes.c_int
    w = synth.PRESETS[preset]
    inp = synth.forward_inputs(w)
    d = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, "bf16")
    o = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device="cuda")
    S_T = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    ws = gdr.new_workspace(gdr.gdr_forward_workspace_size(w.form, d["q"], d["k"], d["v"], d["log_w"],
                                                          d["e1"], d["e2"], 64, "tc"), "cuda")
    a = gdr._fwd_struct(w.form, d["q"], d["k"], d["v"], d["log_w"], d["e1"], d["e2"], None, o, S_T, 64,
                        "tc", ws)
    cycles = (ctypes.c_ulonglong * 16)()

    def run(n):
        for _ in range(n):
            rc = lib.gdr_forward_chunked(ctypes.byref(a), None)
            if rc != 0:
                raise RuntimeError(f"gdr_forward_chunked (timing build) failed: {rc}")
        rc = lib.gdr_general_timing_read(cycles)
        if rc != 0:
            raise RuntimeError(f"gdr_general_timing_read failed: CUDA error {rc}")

    run(1)
    run(calls)
    chunks = w.B * w.H * ((w.T + 63) // 64) * calls
    return w, {i: cycles[i] / chunks for i in range(16)}


def measure_muir(batch=4, calls=3):
    """The Muir mixer, fused (activations inside the prep kernel), on the gdn2_bf16 shapes with
    B = batch, through the timing build: per-phase cycle sums of its prep and chain kernels,
    per chunk (no tensor-core pass)."""
    lib = load_timing_library()
    gdr._declare(lib)
    w = synth.PRESETS["gdn2_bf16"].with_(B=batch)
    inp = synth.muir_inputs(w)
    names = ("q", "k", "v", "zf", "zb", "zw", "zq", "zg")
    d = {k: torch.from_numpy(inp[k]).to("cuda", torch.bfloat16) for k in names}
    par = {k: torch.from_numpy(inp[k]).cuda() for k in ("a_log", "gamma_stat", "rms_weight")}
    cycles = (ctypes.c_ulonglong * 32)()
    threads = (ctypes.c_ulonglong * 2)()
    mma = [(ctypes.c_ulonglong * 16)() for _ in range(2)]
    saved = gdr._lib
    gdr._lib = lib           # the binding's calls go to the timing build meanwhile
    try:
        ws = gdr.new_workspace(gdr.gdr_muir_workspace_size(d["q"], d["k"], d["v"], 64, "tc", False), "cuda")
        y = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device="cuda")

        def run(n):
            for _ in range(n):
                gdr.gdr_muir_forward(*(d[k] for k in names), par["a_log"], par["gamma_stat"],
                                     par["rms_weight"], 1e-6, None, chunk=64, algo="tc",
                                     unfused=False, y=y, want_state=False, workspace=ws)
            rc = lib.gdr_phase_timing_read(cycles, threads, mma[0], mma[1])
            if rc != 0:
                raise RuntimeError(f"gdr_phase_timing_read failed: CUDA error {rc}")

        run(1)
        run(calls)
    finally:
        gdr._lib = saved
    nch = (w.T + 63) // 64
    return {"w": w, "calls": calls, "threads": list(threads), "cycles": list(cycles),
            "prep_chunks": w.B * w.H * nch * calls, "chain_chunks": threads[0] * nch}


def measure(batch=1, calls=3, lib=None, preset="gdn2_bf16"):
    """Runs a GDN-2 bf16 forward workload (default gdn2_bf16: H = 16, T = 4096, with
    B = batch) through the timing build and returns the per-phase cycle sums and the timed
    tensor-core groups, per chunk."""
    lib = lib or load_timing_library()
    w = synth.PRESETS[preset].with_(B=batch)
    inp = synth.forward_inputs(w)
    d = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, "bf16")
    o = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device="cuda")
    S_T = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    ws = gdr.new_workspace(gdr.gdr_forward_workspace_size("gdn2", d["q"], d["k"], d["v"], d["log_w"],
                                                          d["e1"], d["e2"], 64, "tc"), "cuda")
    a = gdr._fwd_struct("gdn2", d["q"], d["k"], d["v"], d["log_w"], d["e1"], d["e2"], None, o, S_T, 64,
                        "tc", ws)
    cycles = (ctypes.c_ulonglong * 32)()
    threads = (ctypes.c_ulonglong * 2)()
    mma_cycles = (ctypes.c_ulonglong * 16)()
    mma_groups = (ctypes.c_ulonglong * 16)()

    def run(n):
        for _ in range(n):
            rc = lib.gdr_forward_chunked(ctypes.byref(a), None)
            if rc != 0:
                raise RuntimeError(f"gdr_forward_chunked (timing build) failed: {rc}")
        rc = lib.gdr_phase_timing_read(cycles, threads, mma_cycles, mma_groups)
        if rc != 0:
            raise RuntimeError(f"gdr_phase_timing_read failed: CUDA error {rc}")

    import os
    os.environ.pop("GDR_TIMING_MMA", None)
    run(1)            # warm-up; reading clears the sums
    run(calls)        # phases, with the kernels' own schedule
    out = {"w": w, "calls": calls, "threads": list(threads), "cycles": list(cycles)}
    os.environ["GDR_TIMING_MMA"] = "1"
    flops_of = {(s_, g): fl for s_, g, _, _, fl in MMA_GROUPS}
    union = {0: [0.0, 0.0, 0, 0], 1: [0.0, 0.0, 0, 0]}
    try:
        read_union(lib, flops_of)     # clear what earlier runs left in the log
        for _ in range(calls):        # tensor-core groups, each waited for by its issuing warp
            run(1)
            for slot, v in read_union(lib, flops_of).items():
                union[slot] = [x + y for x, y in zip(union[slot], v)]
    finally:
        os.environ.pop("GDR_TIMING_MMA", None)
    out["union"] = union
    nch = (w.T + 63) // 64
    # each prep recorder sees every chunk; each chain CTA's recorder the chunks of its sequence
    # (the chain CTAs per call depend on the value-slice width the launch chose)
    out.update({"prep_chunks": w.B * w.H * nch * calls,
                "chain_chunks": out["threads"][0] * nch,
                "mma_cycles": list(mma_cycles), "mma_groups": list(mma_groups)})
    return out


def gemm_phase_fractions(m, peak_tflops, sm_mhz):
    """Per kernel: bf16 FLOPs of its timed tensor-core groups over their summed
    issue-to-completion cycles, as TFLOP/s of the whole GPU at `sm_mhz` (every SM doing the
    same) and as a fraction of `peak_tflops`.  Also per group, and ("union_*") the same FLOPs
    over the cycles in which each CTA had at least one group in flight (overlapping groups
    counted once)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    out = {}
    fl_all = cyc_all = ufl_all = ucyc_all = 0.0
    for slot, name in ((1, "tc_prep_kernel"), (0, "tc_chain_kernel")):
        fl = cyc = 0.0
        groups = []
        for s_, g, what, shape, flops in MMA_GROUPS:
            n = m["mma_groups"][8 * slot + g]
            if s_ != slot or not n:
                continue
            c = m["mma_cycles"][8 * slot + g] / n
            tf = flops / c * sm_mhz * 1e6 * sms / 1e12
            groups.append({"group": f"{what} ({shape})", "count": n, "cycles": c,
                           "tflops": tf, "frac": tf / peak_tflops})
            fl += flops * n
            cyc += m["mma_cycles"][8 * slot + g]
        if cyc:
            tf = fl / cyc * sm_mhz * 1e6 * sms / 1e12
            out[name] = {"tflops": tf, "frac": tf / peak_tflops, "groups": groups}
            u = m.get("union", {}).get(slot)
            if u and u[1]:
                tu = u[0] / u[1] * sm_mhz * 1e6 * sms / 1e12
                out[name].update({"union_tflops": tu, "union_frac": tu / peak_tflops,
                                  "union_groups_logged": u[2], "union_groups_dropped": u[3]})
                ufl_all += u[0]
                ucyc_all += u[1]
            fl_all += fl
            cyc_all += cyc
    if cyc_all:   # the forward call as a whole: every group of both kernels
        tf = fl_all / cyc_all * sm_mhz * 1e6 * sms / 1e12
        out["forward"] = {"tflops": tf, "frac": tf / peak_tflops, "groups": []}
        if ucyc_all:
            tu = ufl_all / ucyc_all * sm_mhz * 1e6 * sms / 1e12
            out["forward"].update({"union_tflops": tu, "union_frac": tu / peak_tflops})
    return out


# Marks of the mLSTM kernel: (index, label) for thread 0 (a P~ / h warp) and for thread 224
# (a K~ warp, the one that also scans the next chunk's gates), in the order of the chunk
# loop; marks 0, 1, 11 and 12 are shared.
MLSTM_PHASES = {
    "thread 0 (P~ and h warps)": [
        (1, "wait for the chunk's tiles, barrier"), (2, "P~ weights (tensor cores on S)"),
        (3, "wait for S"), (4, "S from TMEM, times the weights"),
        (5, "P~ stored, fence, barrier"), (6, "[P~ V | P~ 1] issued; r, g, m"),
        (7, "wait for [P~ V | P~ 1] and [Q C | Q n]"), (8, "h"),
        (9, "wait for [K~^T V | K~^T 1]"), (10, "state update, rows 0..63"),
        (11, "proxy fence"), (12, "barrier (chunk done)"), (0, "to the next chunk"),
    ],
    "thread 224 (K~ warps; warp 7 scans the next chunk's gates)": [
        (1, "wait for the chunk's tiles, barrier"), (2, "diag(f) [V | 1] formed and stored"),
        (3, "barrier (diag(f) [V | 1] done)"), (4, "(warp 2 issues [K~^T V | K~^T 1])"),
        (5, "next chunk's gate scan"), (6, "wait for [Q C | Q n] and [K~^T V | K~^T 1]"),
        (10, "state update, rows 64..127"), (11, "proxy fence"), (12, "barrier (chunk done)"),
        (0, "to the next chunk"),
    ],
}


def measure_mlstm(batch=4, calls=3):
    """The mLSTM cell (bf16, d = 128: the tensor-core kernel) on the GDN-2 bf16 workload's shapes
    through the timing build; returns, for thread 0 and thread 224, the cycles per chunk by
    mark index."""
    lib = ctypes.CDLL(build.build(timing=True))
    lib.gdr_mlstm_forward.argtypes = [ctypes.POINTER(gdr.gdr_mlstm_args), ctypes.c_void_p]
    lib.gdr_mlstm_forward.restype = ctypes.c_int
    lib.gdr_mlstm_timing_read.argtypes = [ctypes.POINTER(ctypes.c_ulonglong)]
    lib.gdr_mlstm_timing_read.restype = ctypes.c_int
    w = synth.PRESETS["gdn2_bf16"].with_(B=batch)
    inp = synth.mlstm_inputs(w)
    d = {k: torch.from_numpy(inp[k]).to("cuda", torch.bfloat16) for k in ("q", "k", "v")}
    g = {k: torch.from_numpy(inp[k]).cuda() for k in ("f_pre", "i_pre")}
    h = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device="cuda")
    a = gdr.gdr_mlstm_args()
    a.dtype, a.B, a.H, a.T, a.dk, a.dv = gdr.DTYPES["bf16"], w.B, w.H, w.T, w.dk, w.dv
    a.q, a.k, a.v = (ctypes.c_void_p(d[x].data_ptr()) for x in ("q", "k", "v"))
    a.f_pre, a.i_pre = ctypes.c_void_p(g["f_pre"].data_ptr()), ctypes.c_void_p(g["i_pre"].data_ptr())
    a.h = ctypes.c_void_p(h.data_ptr())
    cycles = (ctypes.c_ulonglong * 32)()

    def run(n):
        for _ in range(n):
            rc = lib.gdr_mlstm_forward(ctypes.byref(a), None)
            if rc != 0:
                raise RuntimeError(f"gdr_mlstm_forward (timing build) failed: {rc}")
        rc = lib.gdr_mlstm_timing_read(cycles)
        if rc != 0:
            raise RuntimeError(f"gdr_mlstm_timing_read failed: CUDA error {rc}")

    run(1)
    run(calls)
    chunks = w.B * w.H * (w.dv // 64) * ((w.T + 63) // 64) * calls
    return [{i: cycles[16 * r + i] / chunks for i in range(16)} for r in range(2)]


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--batch", type=int, default=None,
                    help="B of the workload (default: 4 for the H=16, T=4096 shapes, the preset's own B "
                         "for --preset gdn2_long)")
    ap.add_argument("--calls", type=int, default=3, help="timed forward calls after one warm-up call")
    ap.add_argument("--peak-tflops", type=float, default=None,
                    help="bf16 dense peak of the whole GPU (default: MEASURED_PEAKS.json's, else 1590)")
    ap.add_argument("--sm-mhz", type=float, default=1965.0,
                    help="SM clock of the run (the cycles are SM cycles)")
    ap.add_argument("--preset", default="gdn2_bf16", choices=["gdn2_bf16", "gdn2_long"],
                    help="forward workload (gdn2_long: B=1, T=65536, the one-launch path)")
    ap.add_argument("--general", action="store_true",
                    help="the two-stream kernel (every form at d = 64) on rwkv7_bf16")
    ap.add_argument("--muir", action="store_true",
                    help="the Muir mixer's fused forward (phases only)")
    ap.add_argument("--mlstm", action="store_true",
                    help="the mLSTM cell's tensor-core kernel instead of the forward")
    args = ap.parse_args(argv)
    batch = args.batch if args.batch is not None else (
        synth.PRESETS[args.preset].B if args.preset == "gdn2_long" and not (args.muir or args.mlstm) else 4)

    if args.mlstm:
        per = measure_mlstm(batch, args.calls)
        print(f"mlstm_tc_kernel, bf16, B={batch}, H=16, T=4096, d=128: cycles per chunk")
        for r, (who, phases) in enumerate(MLSTM_PHASES.items()):
            print(f"\n{who}")
            for i, label in phases:
                print(f"  {label:50s} {per[r][i]:9.0f}")
            print(f"  {'sum':50s} {sum(per[r][i] for i, _ in phases):9.0f}")
        return 0

    if args.general:
        w, per = measure_general(calls=args.calls)
        print(f"tc_general_kernel, {w.form} bf16, B={w.B}, H={w.H}, T={w.T}, d={w.dk}: thread 0's cycles per chunk")
        for i, label in GENERAL_PHASES:
            print(f"  {label:55s} {per[i]:9.0f}")
        print(f"  {'sum':55s} {sum(per[i] for i, _ in GENERAL_PHASES):9.0f}")
        return 0
    m = (measure_muir(batch, args.calls) if args.muir
         else measure(batch, args.calls, preset=args.preset))
    w = m["w"]
    print(f"{'Muir mixer (fused) on ' if args.muir else ''}GDN-2 bf16, B={w.B}, H={w.H}, T={w.T}, d=128, C=64; {args.calls} calls; "
          f"recording threads: prep {m['threads'][1]}, chain {m['threads'][0]}")
    for title, slot, phases, units in (("tc_prep_kernel", 1, PREP_PHASES, m["prep_chunks"]),
                                      ("tc_chain_kernel", 0, CHAIN_PHASES, m["chain_chunks"])):
        print(f"\n{title}: cycles per chunk, by phase")
        total = {}
        for i, label in phases:
            c = m["cycles"][16 * slot + i] / units
            group = label.split(":")[0] if ":" in label else ""
            total[group] = total.get(group, 0.0) + c
            print(f"  {label:50s} {c:9.0f}")
        for g, t in total.items():
            if t:
                print(f"  {'sum' + (' (' + g + ')' if g else ''):50s} {t:9.0f}")
    if args.muir:
        return 0
    peak = args.peak_tflops
    if peak is None:
        import json
        import os
        path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "MEASURED_PEAKS.json")
        peak = json.load(open(path))["bf16_tflops"] if os.path.exists(path) else 1590.0
    fr = gemm_phase_fractions(m, peak, args.sm_mhz)
    print(f"\ntensor-core groups, issue of the first MMA to completion (the issuing warp waits for "
          f"each group); TFLOP/s of the GPU at {args.sm_mhz:.0f} MHz against {peak:.1f} TFLOP/s")
    for name, r in fr.items():
        for g in r["groups"]:
            print(f"  {name:16s} {g['group']:44s} {g['count']:8d} x {g['cycles']:6.0f} cycles "
                  f"= {g['tflops']:7.1f} TFLOP/s ({g['frac']:5.1%})")
        print(f"  {name:16s} {'all GEMM phases':44s} {'':19s} = {r['tflops']:7.1f} TFLOP/s ({r['frac']:5.1%})")
        if "union_tflops" in r:
            extra = (f"  [{r['union_groups_logged']} groups logged, {r['union_groups_dropped']} dropped]"
                     if "union_groups_logged" in r else "")
            print(f"  {name:16s} {'the same over the busy-interval union':44s} {'':19s} = "
                  f"{r['union_tflops']:7.1f} TFLOP/s ({r['union_frac']:5.1%}){extra}")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
