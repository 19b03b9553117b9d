"""Context-parallel prefill: one long sequence (or a batch of equal-length sequences)
split into consecutive segments, one per rank, prefilled at the same time.

The KDA state after a stretch of tokens is affine in the state before it (the
recurrence of the Ling-3.0-flash article, section "KDA: constant-size memory over a
very long context", multiplies the state by (I - b k k^T) Diag(a) on the left and
adds b k v^T), so a segment's effect on the state is a pair (M, B):
S_end = M S_start + B. Rank r holding segment r

  1. computes its map: M_r = final state from the identity with zero values and
     B_r = final state from zero;
  2. all-gathers the maps of every segment (the one exchange: 2 x H x d x d fp32
     per sequence and segment);
  3. folds the maps of the segments before it into its start state,
     S = M_{r-1} (... (M_0 S_0 + B_0) ...) + B_{r-1};
  4. prefills its segment from S: its outputs, and on the last rank the final state.

With the library's kernels (KernelEngine) steps 1 and 4 share one pass over the
segment's chunks: kda_segment_maps runs the state-free part of every chunk once and the
recurrence for both maps, and kda_segment_prefill reruns only the recurrence from S on
what the first call left in its workspace, and kda_state_fold folds all the earlier
segments' maps in one launch. Every step runs in the library's CUDA
kernels; this module only orders them and calls torch.distributed for the exchange.
The steps that touch data go through an engine object, so the same orchestration runs
with other implementations of them (the tests drive it on CPU ranks with the oracle,
through PrefillEngine).
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple


def _torch():
    import torch
    return torch


class KernelEngine:
    """The library's kernels: one pass over the segment's chunks for both maps
    (kda_segment_maps), the recurrence alone from the start state (kda_segment_prefill),
    one map applied to a state (kda_state_affine) and the fold of a chain of maps in one
    launch (kda_state_fold)."""

    def maps(self, q, k, v, log_alpha, beta, N: int):
        from . import segment_maps
        return segment_maps(q, k, v, log_alpha, beta, None, N=N)

    def prefill(self, handle, S):
        from . import segment_prefill
        return segment_prefill(handle, S)

    def affine(self, M, S, B):
        from . import state_affine
        return state_affine(M, S, B)

    def fold(self, MB, rank: int, initial_state=None):
        if rank == 0:
            return initial_state
        from . import state_fold
        return state_fold(MB, rank, initial_state)


class PrefillEngine:
    """Any prefill and affine-map functions: the maps from two prefills of the segment
    (the identity with zero values; zero), the segment's own prefill from its start state."""

    def __init__(self, prefill: Callable, affine: Callable):
        self._prefill, self._affine = prefill, affine

    def maps(self, q, k, v, log_alpha, beta, N: int):
        M, B = segment_map(q, k, v, log_alpha, beta, N, self._prefill)
        return M, B, (q, k, v, log_alpha, beta, N)

    def prefill(self, handle, S):
        q, k, v, log_alpha, beta, N = handle
        return self._prefill(q, k, v, log_alpha, beta, S, N)

    def affine(self, M, S, B):
        return self._affine(M, S, B)

    def fold(self, MB, rank: int, initial_state=None):
        return start_state([(MB[j, 0], MB[j, 1]) for j in range(rank)], rank, initial_state, self._affine)


def _engine(engine, prefill, affine):
    if engine is not None:
        return engine
    if prefill is None and affine is None:
        return KernelEngine()
    if prefill is None or affine is None:
        raise ValueError("give both prefill and affine, or an engine")
    return PrefillEngine(prefill, affine)


def segment_map(q, k, v, log_alpha, beta, N: int, prefill: Callable):
    """(M, B) of one segment of N equal-length sequences (packed [N*T, H, d]) from two
    prefills: M [N, H, d, d] the final state from the identity with zero values, B the
    final state from zero."""
    torch = _torch()
    H, d = q.shape[1], q.shape[2]
    if v.shape[-1] != d:
        raise ValueError("the segment map needs d_v == d_k")
    eye = torch.eye(d, dtype=torch.float32, device=q.device).expand(N, H, d, d).contiguous()
    _, M = prefill(q, k, torch.zeros_like(v), log_alpha, beta, eye, N)
    _, B = prefill(q, k, v, log_alpha, beta, None, N)
    return M, B


def start_state(maps, rank: int, initial_state=None, affine: Optional[Callable] = None):
    """Fold the maps of segments 0 .. rank-1 (a list of (M, B)) into the state at the
    start of segment `rank`; None (zero) when rank == 0 and there is no initial state."""
    fold = affine if affine is not None else KernelEngine().affine
    S = initial_state
    for M, B in maps[:rank]:
        S = fold(M, S, B)
    return S


def context_parallel_prefill(q, k, v, log_alpha, beta, initial_state=None, *, N: int = 1, group=None,
                             engine=None, prefill: Optional[Callable] = None,
                             affine: Optional[Callable] = None) -> Tuple[object, object]:
    """This rank's segment of N equal-length sequences (packed [N*T_seg, H, d]); segment
    order = rank order in `group`. Returns (out of the segment, state at its end); the
    last rank's state is the sequences' final state. With one rank it is a plain prefill.
    `initial_state` (the state before segment 0) is used by every rank."""
    torch = _torch()
    import torch.distributed as dist
    eng = _engine(engine, prefill, affine)
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    rank = dist.get_rank(group) if world > 1 else 0
    if world == 1:
        if prefill is not None:
            return prefill(q, k, v, log_alpha, beta, initial_state, N)
        from . import chunk_fwd
        return chunk_fwd(q, k, v, log_alpha, beta, initial_state, None, N=N)
    M, B, handle = eng.maps(q, k, v, log_alpha, beta, N)
    both = torch.stack([M, B]).contiguous()
    gathered = torch.empty((world,) + tuple(both.shape), dtype=both.dtype, device=both.device)
    dist.all_gather(list(gathered.unbind(0)), both, group=group)  # [world, 2, N, H, d, d]
    S = eng.fold(gathered, rank, initial_state)
    return eng.prefill(handle, S)


def context_parallel_emulate(q, k, v, log_alpha, beta, initial_state=None, *, N: int, segments: int,
                             engine=None, prefill: Optional[Callable] = None, affine: Optional[Callable] = None):
    """The same steps on one device: each of N equal-length sequences (packed
    [N*T, H, d], T divisible by `segments`) is cut into `segments` consecutive pieces
    that are treated as ranks. Returns (out [N*T, H, d], final state)."""
    torch = _torch()
    eng = _engine(engine, prefill, affine)
    NT, H, d = q.shape
    T = NT // N
    if T * N != NT or T % segments:
        raise ValueError("T must split into equal segments")
    ts = T // segments

    def seg(x, i):  # piece i of every sequence, packed
        return x.reshape(N, T, *x.shape[1:])[:, i * ts:(i + 1) * ts].reshape(N * ts, *x.shape[1:]).contiguous()

    pieces = [[seg(x, i) for x in (q, k, v, log_alpha, beta)] for i in range(segments)]
    maps = [eng.maps(*p, N) for p in pieces]
    MB = torch.stack([torch.stack([m[0], m[1]]) for m in maps])  # as the all-gather lays them out
    outs, final = [], None
    for i in range(segments):
        S = eng.fold(MB, i, initial_state)
        o, final = eng.prefill(maps[i][2], S)
        outs.append(o.reshape(N, ts, *o.shape[1:]))
    return torch.cat(outs, dim=1).reshape(NT, *outs[0].shape[2:]), final
