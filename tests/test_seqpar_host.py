"""Sequence parallelism's collective plumbing on the host: gloo, world size 2.

Each rank holds one segment of every sequence; the per-segment steps (segment maps, the
affine composition, the segment's forward) are supplied by the test from the fp64 oracle,
so that what runs here is the product's collective logic in matrix_memory_rnn_b200.seqpar:
the all-gather of the maps, the composition of the earlier ranks' maps into the entry state,
and of the later ranks' maps into the global final state.  The outputs must equal the
oracle's pass over the whole sequence.  No GPU.
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

T_SPLIT = 37


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    rng = np.random.default_rng(3)
    B, T, H, dk, dv = 1, 70, 2, 4, 3
    q, k = rng.standard_normal((B, T, H, dk)), 0.5 * rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    lw = -np.exp(rng.normal(-1.5, 0.5, (B, T, H, dk)))
    e1 = 0.4 * rng.standard_normal((B, T, H, dk))
    e2 = 0.4 * rng.standard_normal((B, T, H, dk))
    S0 = rng.standard_normal((B, H, dk, dv))
    return q, k, v, lw, e1, e2, S0


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from matrix_memory_rnn_b200 import seqpar
        q, k, v, lw, e1, e2, S0 = _problem()
        sl = slice(0, T_SPLIT) if rank == 0 else slice(T_SPLIT, None)
        seg = [a[:, sl] for a in (q, k, v, lw, e1, e2)]
        t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a))

        def maps_fn(form, q_, k_, v_, lw_, e1_, e2_):
            q_, k_, v_, lw_, e1_, e2_ = (x.numpy() for x in (q_, k_, v_, lw_, e1_, e2_))
            B, T, H, dk = q_.shape
            _, Q = oracle.forward(form, q_, k_, v_, lw_, e1_, e2_, None)
            eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk))
            _, M = oracle.forward(form, q_, k_, np.zeros((B, T, H, dk)), lw_, e1_, e2_, eye)
            return t(M), t(Q)

        def compose_fn(M, S_in, Q):
            return Q if S_in is None else torch.matmul(M, S_in) + Q

        def forward_fn(form, q_, k_, v_, lw_, e1_, e2_, S_in):
            o, S = oracle.forward(form, *(x.numpy() for x in (q_, k_, v_, lw_, e1_, e2_)),
                                  None if S_in is None else S_in.numpy())
            return t(o), t(S)

        o, S_T, S_in = seqpar.sequence_parallel_forward(
            "general", *(t(a) for a in seg), t(S0), maps_fn=maps_fn, compose_fn=compose_fn,
            forward_fn=forward_fn)
        out.put((rank, o.numpy(), S_T.numpy()))
    finally:
        dist.destroy_process_group()


def test_sequence_parallel_gloo_world2():
    import oracle
    world, port = 2, _free_port()
    mctx = mp.get_context("spawn")
    out = mctx.Queue()
    procs = [mctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict((r, (o, S)) for r, o, S in (out.get(timeout=240) for _ in range(world)))
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    q, k, v, lw, e1, e2, S0 = _problem()
    o_ref, S_ref = oracle.forward("general", q, k, v, lw, e1, e2, S0)
    o = np.concatenate([got[0][0], got[1][0]], axis=1)
    assert np.max(np.abs(o - o_ref)) < 1e-10 * np.max(np.abs(o_ref))
    for r in range(world):
        assert np.max(np.abs(got[r][1] - S_ref)) < 1e-10 * np.max(np.abs(S_ref))
