"""Per-phase cycle accounting of the two-kernel tensor-core forward (GDN-2, bf16, d = 128, C = 64).

Runs the forward through ``libgdr_timing.so`` (the same kernels with their phase marks filled
in, see ``csrc/gdr_phase_timing.cuh``) and prints, per kernel and phase, the average cycles
per chunk of one recording thread: the prep kernel's front and back warp groups (one thread
each) and the chain kernel (thread 0).  Each value is the interval that ends at the phase's
mark, so it includes the time that thread waited for the others there.  The timing build runs
somewhat slower than ``libgdr.so``: compare phases with one another, not with bench.py.

Usage: ``python -m matrix_memory_rnn_b200.phase_timing [--batch B] [--calls N]`` (one GPU).
"""
from __future__ import annotations

import argparse
import ctypes

import torch

from . import build, gdr, synth

PREP_PHASES = [
    (1, "front: wait for log w, tiles and write gate"), (2, "front: log-decay scan"),
    (3, "front: operand tiles and V^"), (4, "front: MMA1 issued, chunk handed over"),
    (0, "front: to the next chunk"),
    (9, "back: wait for the hand-over and MMA1"), (10, "back: L and M"),
    (11, "back: T^-1 and its bf16 copy"), (12, "back: MMA2 issued and waited for"),
    (13, "back: U, Y to the record; next tiles requested"), (8, "back: to the next chunk"),
]
CHAIN_PHASES = [
    (1, "wait for MMA3 ([Q_pi; Y] S0)"), (2, "V~ = U - Y S0"), (3, "MMA4 issued and waited for"),
    (4, "state update and its bf16 copy"), (5, "MMA3 of the next chunk issued"), (6, "O read out"),
    (0, "to the next chunk"),
]


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--batch", type=int, default=4, help="B of the GDN-2 bf16 workload (H=16, T=4096)")
    ap.add_argument("--calls", type=int, default=3, help="timed forward calls after one warm-up call")
    args = ap.parse_args(argv)

    lib = ctypes.CDLL(build.build(timing=True))
    lib.gdr_forward_chunked.argtypes = [ctypes.POINTER(gdr.gdr_fwd_args), ctypes.c_void_p]
    lib.gdr_forward_chunked.restype = ctypes.c_int
    u64p = ctypes.POINTER(ctypes.c_ulonglong)
    lib.gdr_phase_timing_read.argtypes = [u64p, u64p]
    lib.gdr_phase_timing_read.restype = ctypes.c_int

    w = synth.PRESETS["gdn2_bf16"].with_(B=args.batch)
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

    def run(n):
        for _ in range(n):
            rc = lib.gdr_forward_chunked(ctypes.byref(a), None)
            if rc != 0:
                raise RuntimeError(f"gdr_forward_chunked (timing build) failed: {rc}")
        rc = lib.gdr_phase_timing_read(cycles, threads)
        if rc != 0:
            raise RuntimeError(f"gdr_phase_timing_read failed: CUDA error {rc}")

    run(1)            # warm-up; reading clears the sums
    run(args.calls)
    nch = (w.T + 63) // 64
    prep_chunks = w.B * w.H * nch * args.calls                # each group's recorder sees every chunk
    chain_chunks = w.B * w.H * (w.dv // 64) * nch * args.calls
    print(f"GDN-2 bf16, B={w.B}, H={w.H}, T={w.T}, d=128, C=64; {args.calls} calls; "
          f"recording threads: prep {threads[1]}, chain {threads[0]}")
    for title, slot, phases, units in (("tc_prep_kernel", 1, PREP_PHASES, prep_chunks),
                                      ("tc_chain_kernel", 0, CHAIN_PHASES, chain_chunks)):
        print(f"\n{title}: cycles per chunk, by phase")
        total = {"front": 0.0, "back": 0.0, "": 0.0}
        for i, label in phases:
            c = cycles[16 * slot + i] / units
            group = label.split(":")[0] if ":" in label else ""
            total[group] += c
            print(f"  {label:50s} {c:9.0f}")
        for g, t in total.items():
            if t:
                print(f"  {'sum' + (' (' + g + ')' if g else ''):50s} {t:9.0f}")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
