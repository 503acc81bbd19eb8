"""Sequence parallelism for long sequences: each rank holds one contiguous segment of the
tokens of every (b, h) sequence.

A segment maps its entry state affinely to its exit state, S_out = M S_in + Q in the
storage orientation ("Muir: Linear Attention with Sensitivity-Allocated Gating and
Matched-Filter Readout", section 4.2 eq. (10), where a chunk's end state is affine in its
start state; a run of chunks composes such maps).  Each rank

  1. computes its segment's map: Q = the forward from S_in = 0, M = the forward from
     S_in = I with v = 0 (the write terms vanish, the transitions remain);
  2. all-gathers the maps (one collective, (d_k^2 + d_k d_v) fp32 per head and rank);
  3. composes the maps of the ranks before it onto the initial state: its entry state;
  4. runs its segment from that entry state: its outputs, and the global final state by
     composing the remaining ranks' maps.

Three forward passes over the local segment instead of one sequential pass over all of
them: worth it when the per-sequence chain latency dominates (few long sequences).  The
steps are the library's own calls (gdr_forward_chunked, gdr_state_compose); they can be
replaced through the keyword arguments, which the host tests use to drive the collective
plumbing on the CPU.
"""
from __future__ import annotations

import torch

from . import gdr

__all__ = ["segment_maps", "compose", "sequence_parallel_forward", "emulate_segments"]


def segment_maps(form, q, k, v, log_w, e1=None, e2=None, *, chunk=64, algo="auto"):
    """(M [B, H, dk, dk], Q [B, H, dk, dv]) of one segment: S_out = M S_in + Q."""
    B, T, H, dk = q.shape
    _, Q = gdr.gdr_forward_chunked(form, q, k, v, log_w, e1, e2, None, chunk=chunk, algo=algo)
    eye = torch.eye(dk, dtype=torch.float32, device=q.device).expand(B, H, dk, dk).contiguous()
    v0 = torch.zeros((B, T, H, dk), dtype=v.dtype, device=v.device)
    # the write gate (GDN-2's e2) only scales v: with v = 0 it is not needed
    e2_m = None if form == "gdn2" else e2
    _, M = gdr.gdr_forward_chunked(form, q, k, v0, log_w, e1, e2_m, eye, chunk=chunk, algo=algo)
    return M, Q


def compose(M, S_in, Q):
    """M S_in + Q per head (gdr_state_compose); S_in None = 0."""
    return gdr.gdr_state_compose(M, S_in, Q)


def _forward(form, q, k, v, log_w, e1, e2, S0, *, chunk, algo):
    return gdr.gdr_forward_chunked(form, q, k, v, log_w, e1, e2, S0, chunk=chunk, algo=algo)


def sequence_parallel_forward(form, q, k, v, log_w, e1=None, e2=None, S0=None, *, chunk=64,
                              algo="auto", group=None, maps_fn=None, compose_fn=None,
                              forward_fn=None):
    """This rank's segment [B, T_r, H, .] of every sequence (ranks in token order).
    Returns (o of the segment, the global final state S_T, this segment's entry state).
    Without an initialized process group it is the plain forward with one segment."""
    import torch.distributed as dist
    maps_fn = maps_fn or (lambda *a: segment_maps(*a, chunk=chunk, algo=algo))
    compose_fn = compose_fn or compose
    forward_fn = forward_fn or (lambda *a: _forward(*a, chunk=chunk, algo=algo))
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    rank = dist.get_rank(group) if world > 1 else 0
    M, Q = maps_fn(form, q, k, v, log_w, e1, e2)
    if world > 1:
        Ms = [torch.empty_like(M) for _ in range(world)]
        Qs = [torch.empty_like(Q) for _ in range(world)]
        dist.all_gather(Ms, M.contiguous(), group=group)
        dist.all_gather(Qs, Q.contiguous(), group=group)
    else:
        Ms, Qs = [M], [Q]
    S_in = S0
    for j in range(rank):
        S_in = compose_fn(Ms[j], S_in, Qs[j])
    o, S_out = forward_fn(form, q, k, v, log_w, e1, e2, S_in)
    S_T = S_out
    for j in range(rank + 1, world):
        S_T = compose_fn(Ms[j], S_T, Qs[j])
    return o, S_T, S_in


def emulate_segments(form, q, k, v, log_w, e1=None, e2=None, S0=None, *, n_seg, chunk=64,
                     algo="auto"):
    """The same algorithm on one device with ``n_seg`` segments run one after another
    (maps of every segment, then entry states, then each segment's pass): for tests of the
    data path where only one GPU is present.  Returns (o [B, T, H, dv], S_T)."""
    T = q.shape[1]
    bounds = [round(i * T / n_seg) for i in range(n_seg + 1)]
    seg = lambda t, i: None if t is None or t.dim() < 3 else t[:, bounds[i]:bounds[i + 1]].contiguous()
    maps = [segment_maps(form, *(seg(t, i) for t in (q, k, v, log_w, e1, e2)), chunk=chunk, algo=algo)
            for i in range(n_seg)]
    outs, S = [], S0
    for i in range(n_seg):
        args = [seg(t, i) for t in (q, k, v, log_w, e1, e2)]
        o, S_out = _forward(form, *args, S, chunk=chunk, algo=algo)
        outs.append(o)
        S = compose(maps[i][0], S, maps[i][1]) if i + 1 < n_seg else S_out
    return torch.cat(outs, dim=1), S
