"""Context-parallel prefill: one long sequence (or a batch of equal-length sequences)
split into consecutive segments, one per rank, prefilled at the same time.

The KDA state after a stretch of tokens is affine in the state before it (the
recurrence of the Ling-3.0-flash article, section "KDA: constant-size memory over a
very long context", multiplies the state by (I - b k k^T) Diag(a) on the left and
adds b k v^T), so a segment's effect on the state is a pair (M, B):
S_end = M S_start + B. Rank r holding segment r

  1. computes its map: M_r = final state from the identity with zero values and
     B_r = final state from zero (two prefills of the segment, d_v = d_k);
  2. all-gathers the maps of every segment (the one exchange: 2 x H x d x d fp32
     per sequence and segment);
  3. folds the maps of the segments before it into its start state,
     S = M_{r-1} (... (M_0 S_0 + B_0) ...) + B_{r-1};
  4. prefills its segment from S: its outputs, and on the last rank the final state.

Every step runs in the library's CUDA kernels (kda_chunk_fwd, kda_state_affine); this
module only orders them and calls torch.distributed for the exchange. The three steps
that touch data are parameters, so the same orchestration runs with other
implementations of them (the tests drive it on CPU ranks with the oracle).
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple


def _torch():
    import torch
    return torch


def _default_prefill(q, k, v, log_alpha, beta, initial_state, N):
    from . import chunk_fwd
    return chunk_fwd(q, k, v, log_alpha, beta, initial_state, None, N=N)


def _default_affine(M, S, B):
    from . import state_affine
    return state_affine(M, S, B)


def segment_map(q, k, v, log_alpha, beta, N: int, prefill: Callable = _default_prefill):
    """(M, B) of one segment of N equal-length sequences (packed [N*T, H, d]):
    M [N, H, d, d] the final state from the identity with zero values, B [N, H, d, d]
    the final state from zero."""
    torch = _torch()
    H, d = q.shape[1], q.shape[2]
    if v.shape[-1] != d:
        raise ValueError("the segment map needs d_v == d_k")
    eye = torch.eye(d, dtype=torch.float32, device=q.device).expand(N, H, d, d).contiguous()
    _, M = prefill(q, k, torch.zeros_like(v), log_alpha, beta, eye, N)
    _, B = prefill(q, k, v, log_alpha, beta, None, N)
    return M, B


def start_state(maps, rank: int, initial_state=None, affine: Callable = _default_affine):
    """Fold the maps of segments 0 .. rank-1 (a list of (M, B)) into the state at the
    start of segment `rank`; None (zero) when rank == 0 and there is no initial state."""
    S = initial_state
    for M, B in maps[:rank]:
        S = affine(M, S, B)
    return S


def context_parallel_prefill(q, k, v, log_alpha, beta, initial_state=None, *, N: int = 1, group=None,
                             prefill: Callable = _default_prefill, affine: Callable = _default_affine
                             ) -> Tuple[object, object]:
    """This rank's segment of N equal-length sequences (packed [N*T_seg, H, d]); segment
    order = rank order in `group`. Returns (out of the segment, state at its end); the
    last rank's state is the sequences' final state. With one rank it is a plain prefill.
    `initial_state` (the state before segment 0) is used by every rank."""
    torch = _torch()
    import torch.distributed as dist
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    rank = dist.get_rank(group) if world > 1 else 0
    if world == 1:
        return prefill(q, k, v, log_alpha, beta, initial_state, N)
    M, B = segment_map(q, k, v, log_alpha, beta, N, prefill)
    both = torch.stack([M, B]).contiguous()
    parts = [torch.empty_like(both) for _ in range(world)]
    dist.all_gather(parts, both, group=group)
    S = start_state([(p[0], p[1]) for p in parts], rank, initial_state, affine)
    return prefill(q, k, v, log_alpha, beta, S, N)


def context_parallel_emulate(q, k, v, log_alpha, beta, initial_state=None, *, N: int, segments: int,
                             prefill: Callable = _default_prefill, affine: Callable = _default_affine):
    """The same steps on one device: each of N equal-length sequences (packed
    [N*T, H, d], T divisible by `segments`) is cut into `segments` consecutive pieces
    that are treated as ranks. Returns (out [N*T, H, d], final state)."""
    torch = _torch()
    NT, H, d = q.shape
    T = NT // N
    if T * N != NT or T % segments:
        raise ValueError("T must split into equal segments")
    ts = T // segments

    def seg(x, i):  # piece i of every sequence, packed
        return x.reshape(N, T, *x.shape[1:])[:, i * ts:(i + 1) * ts].reshape(N * ts, *x.shape[1:]).contiguous()

    pieces = [[seg(x, i) for x in (q, k, v, log_alpha, beta)] for i in range(segments)]
    maps = [segment_map(*p, N=N, prefill=prefill) for p in pieces]
    outs, final = [], None
    for i, p in enumerate(pieces):
        S = start_state(maps, i, initial_state, affine)
        o, final = prefill(*p, S, N)
        outs.append(o.reshape(N, ts, *o.shape[1:]))
    return torch.cat(outs, dim=1).reshape(NT, *outs[0].shape[2:]), final
