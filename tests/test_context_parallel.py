"""Context-parallel prefill (gated_delta_rule_137_b200.context_parallel).

CPU: the orchestration itself (segment maps, the all-gather over a gloo group, the fold,
the final prefill) on 2 and 3 ranks, with the oracle standing in for the prefill and
the affine map, against the oracle's whole-sequence recurrence.
GPU: the single-device emulation with the library's kernels against the oracle."""
import os
import socket

import numpy as np
import pytest

from gated_delta_rule_137_b200 import inputs as I
from oracle import kda_oracle as O


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload(N=2, T=48, H=2, d=8, seed=137201):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((N * T, H, d)) for _ in range(3))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    la = -np.log1p(np.exp(rng.standard_normal((N * T, H, d)))) / 8
    b = 1 / (1 + np.exp(-rng.standard_normal((N * T, H))))
    s0 = rng.standard_normal((N, H, d, d)) * 0.1
    return q, k, v, la, b, s0


def _oracle_prefill(q, k, v, la, b, h0, N):
    import torch
    cu = np.arange(N + 1) * (q.shape[0] // N)
    o, f = O.kda_recurrence(q.numpy(), k.numpy(), v.numpy(), la.numpy(), b.numpy(),
                            None if h0 is None else h0.numpy(), cu)
    return torch.from_numpy(o), torch.from_numpy(f)


def _oracle_affine(M, S, B):
    return B.clone() if S is None else M @ S + B


def _rank_main(rank, world, port, segments_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    from gated_delta_rule_137_b200 import context_parallel as cp
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        N, T = 2, 48
        q, k, v, la, b, s0 = (torch.from_numpy(x) for x in _workload(N, T))
        ts = T // world

        def seg(x):
            return x.reshape(N, T, *x.shape[1:])[:, rank * ts:(rank + 1) * ts].reshape(N * ts, *x.shape[1:]).contiguous()

        out, fin = cp.context_parallel_prefill(seg(q), seg(k), seg(v), seg(la), seg(b), s0, N=N,
                                               prefill=_oracle_prefill, affine=_oracle_affine)
        segments_out.put((rank, out.numpy(), fin.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_ranks_reproduce_the_whole_sequence(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    qout = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, qout)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(qout.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    N, T = 2, 48
    q, k, v, la, b, s0 = _workload(N, T)
    ref_o, ref_f = O.kda_recurrence(q, k, v, la, b, s0, np.arange(N + 1) * T)
    ts = T // world
    got = np.zeros_like(ref_o).reshape(N, T, *ref_o.shape[1:])
    for rank, o, _ in res:
        got[:, rank * ts:(rank + 1) * ts] = o.reshape(N, ts, *o.shape[1:])
    np.testing.assert_allclose(got.reshape(ref_o.shape), ref_o, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(res[-1][2], ref_f, rtol=1e-10, atol=1e-11)


def test_single_rank_is_a_plain_prefill():
    import torch
    from gated_delta_rule_137_b200 import context_parallel as cp
    q, k, v, la, b, s0 = (torch.from_numpy(x) for x in _workload())
    o, f = cp.context_parallel_prefill(q, k, v, la, b, s0, N=2, prefill=_oracle_prefill, affine=_oracle_affine)
    ro, rf = _oracle_prefill(q, k, v, la, b, s0, 2)
    assert torch.equal(o, ro) and torch.equal(f, rf)


def test_emulation_on_one_device_matches_the_recurrence():
    import torch
    from gated_delta_rule_137_b200 import context_parallel as cp
    x = _workload(N=2, T=48)
    o, f = cp.context_parallel_emulate(*(torch.from_numpy(a) for a in x), N=2, segments=4,
                                       prefill=_oracle_prefill, affine=_oracle_affine)
    ref_o, ref_f = O.kda_recurrence(*x, np.arange(3) * 48)
    np.testing.assert_allclose(o.numpy(), ref_o, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(f.numpy(), ref_f, rtol=1e-10, atol=1e-11)


@pytest.mark.gpu
def test_context_parallel_emulation_with_the_kernels():
    """4 segments of a 1024-token sequence (H = 4, d = 128, bf16) through kda_segment_maps,
    kda_state_fold and kda_segment_prefill on one GPU, against the oracle's whole-sequence
    recurrence."""
    import torch
    from gated_delta_rule_137_b200 import build
    build.build()
    import gated_delta_rule_137_b200 as kda
    from gated_delta_rule_137_b200 import context_parallel as cp
    from tests.helpers import assert_prefill_close, to_device, to_host
    w = I.make_prefill([1024], 4, 128, 128, seed=I.SEED_BASE + 51)
    args = [to_device(w.q, "bf16"), to_device(w.k, "bf16"), to_device(w.v, "bf16"), to_device(w.log_alpha, "f32"),
            to_device(w.beta, "f32"), to_device(w.initial_state, "f32")]
    o, f = cp.context_parallel_emulate(*args, N=1, segments=4)
    torch.cuda.synchronize()
    ro, rf = O.kda_recurrence(w.q, w.k, w.v, w.log_alpha, w.beta, w.initial_state, w.cu_seqlens)
    assert_prefill_close(to_host(o), ro, "context-parallel out", stored_bf16=True)
    assert_prefill_close(to_host(f), rf, "context-parallel final state")


@pytest.mark.gpu
def test_state_affine_kernel_against_matmul():
    import torch
    from gated_delta_rule_137_b200 import build
    build.build()
    import gated_delta_rule_137_b200 as kda
    g = torch.Generator(device="cuda").manual_seed(137202)
    M, S, B = (torch.randn(6, 128, 128, generator=g, device="cuda") for _ in range(3))
    ref = (M.double() @ S.double() + B.double())
    for s, b, want in ((S, B, ref), (S, None, M.double() @ S.double()), (None, B, B.double())):
        out = kda.state_affine(M, s, b)
        torch.cuda.synchronize()
        err = (out.double() - want).abs().max().item() / want.abs().max().item()
        assert err < 1e-5, err
    out = B.clone()
    kda.state_affine(M, S, out, out=out)  # in place over B
    torch.cuda.synchronize()
    assert (out.double() - ref).abs().max().item() / ref.abs().max().item() < 1e-5


@pytest.mark.gpu
@pytest.mark.parametrize("maps", [0, 1, 3])
@pytest.mark.parametrize("with_s0", [False, True])
def test_state_fold_kernel_against_matmul(maps, with_s0):
    """kda_state_fold: S <- M_j S + B_j for j < maps, the maps laid out [maps + 1, 2, N, H, d, d]
    (one more than are folded, as a rank below the last sees them), against the chain of
    fp64 products; in place over S0 too."""
    import torch
    from gated_delta_rule_137_b200 import build
    build.build()
    import gated_delta_rule_137_b200 as kda
    g = torch.Generator(device="cuda").manual_seed(137203 + maps)
    MB = torch.randn(maps + 1, 2, 2, 3, 128, 128, generator=g, device="cuda") / 8
    S0 = torch.randn(2, 3, 128, 128, generator=g, device="cuda") if with_s0 else None
    want = S0.double() if with_s0 else torch.zeros(2, 3, 128, 128, dtype=torch.float64, device="cuda")
    for j in range(maps):
        want = MB[j, 0].double() @ want + MB[j, 1].double()
    out = kda.state_fold(MB, maps, S0)
    torch.cuda.synchronize()
    scale = max(want.abs().max().item(), 1.0)
    assert (out.double() - want).abs().max().item() / scale < 1e-5
    if with_s0:
        kda.state_fold(MB, maps, S0, out=S0)
        torch.cuda.synchronize()
        assert (S0.double() - want).abs().max().item() / scale < 1e-5


@pytest.mark.gpu
@pytest.mark.parametrize("lens,H,strong", [([200, 64], 4, False), ([130, 7], 4, True), ([70] * 20, 4, False)])
def test_segment_maps_and_prefill_against_the_oracle(lens, H, strong):
    """kda_segment_maps: M = final state from the identity with zero values, B = final state
    from zero, from one pass over the chunks; kda_segment_prefill from a start state on what
    it left. Ragged sequences, strong decay on the odd chunks (walked), and 80 chains
    (several waves of the doubled slices)."""
    import torch
    from gated_delta_rule_137_b200 import build
    build.build()
    import gated_delta_rule_137_b200 as kda
    from tests.helpers import assert_prefill_close, to_device, to_host
    w = I.make_prefill(lens, H, 128, 128, seed=I.SEED_BASE + 52 + len(lens))
    la = w.log_alpha.copy()
    if strong:
        for n in range(w.N):
            s, e = int(w.cu_seqlens[n]), int(w.cu_seqlens[n + 1])
            la[s:e][((np.arange(e - s) // 64) % 2) == 1] *= 128.0
    cu = to_device(w.cu_seqlens, "i32")
    M, B, handle = kda.segment_maps(to_device(w.q, "bf16"), to_device(w.k, "bf16"), to_device(w.v, "bf16"),
                                    to_device(la, "f32"), to_device(w.beta, "f32"), cu, check_status=True)
    out, fin = kda.segment_prefill(handle, to_device(w.initial_state, "f32"), check_status=True)
    torch.cuda.synchronize()
    eye = np.broadcast_to(np.eye(128), (w.N, H, 128, 128))
    _, rM = O.kda_recurrence(w.q, w.k, np.zeros_like(w.v), la, w.beta, eye, w.cu_seqlens)
    _, rB = O.kda_recurrence(w.q, w.k, w.v, la, w.beta, None, w.cu_seqlens)
    ro, rf = O.kda_recurrence(w.q, w.k, w.v, la, w.beta, w.initial_state, w.cu_seqlens)
    assert_prefill_close(to_host(M), rM, "segment map M")
    assert_prefill_close(to_host(B), rB, "segment map B")
    assert_prefill_close(to_host(out), ro, "segment prefill out", stored_bf16=True)
    assert_prefill_close(to_host(fin), rf, "segment prefill final state")
