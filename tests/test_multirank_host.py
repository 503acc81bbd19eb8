"""Multi-process checks of bench.py's rank plumbing on the host: gloo, world size 2.

The bench shards independent sequences across ranks (no collective on the data
path); the ranks meet only at a barrier around the timed region and in the max
over ranks of the elapsed time.  These run without a GPU.
"""
import datetime
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from matrix_memory_rnn_b200 import synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ctx = bench.Ctx(torch, dist, world, rank, rank, device=torch.device("cpu"))
        ctx.barrier()
        slowest = ctx.max_over_ranks(1.5 + rank)      # rank r "took" 1.5 + r ms
        ctx.barrier()
        q.put((rank, slowest))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barrier_gloo_world2():
    world, port = 2, _free_port()
    mctx = mp.get_context("spawn")
    q = mctx.Queue()
    procs = [mctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(world))
    assert got == [(0, 2.5), (1, 2.5)]          # every rank reports the slowest rank's time


def test_ranks_draw_disjoint_shards():
    w = synth.PRESETS["gdn2_bf16"].with_(B=1, H=2, T=16)
    a = synth.forward_inputs(w, seed=bench.rank_seed(w.seed, 0))
    b = synth.forward_inputs(w, seed=bench.rank_seed(w.seed, 1))
    assert bench.rank_seed(w.seed, 0) == w.seed
    assert not np.array_equal(a["q"], b["q"]) and not np.array_equal(a["log_w"], b["log_w"])


def test_reference_arm_prints_on_rank0_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1",
                                      "--warmup", "0"])
    assert bench.main() == 0
    assert capsys.readouterr().out == ""
