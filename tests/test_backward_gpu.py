"""kda_chunk_bwd (gradients of the recurrence) through the C ABI against the oracle's
kda_backward, on packed sequences that span several 8-token checkpoint intervals with
ragged tails, an empty and a one-token sequence, fp32 and bf16 inputs, with and without
the initial state and the final state's gradient; and, at the model shape (one
4096-token sequence of 32 heads), on sampled heads, which the oracle computes alone
because the heads of the recurrence do not interact."""
import numpy as np
import pytest

from gated_delta_rule_137_b200 import inputs as I
from oracle import kda_oracle as O
from tests.helpers import assert_backward_close, to_device, to_host

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "d_log_alpha", "d_beta", "d_initial_state")


@pytest.fixture(scope="module")
def kda():
    import torch
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    from gated_delta_rule_137_b200 import build
    build.build()
    import gated_delta_rule_137_b200 as m
    m.load_library()
    return m


def _gpu(kda, w, d_out, d_final, use_cu=True):
    import torch
    dt = w.qkv_dtype
    grads = kda.chunk_bwd(to_device(w.q, dt), to_device(w.k, dt), to_device(w.v, dt), to_device(w.log_alpha, "f32"),
                          to_device(w.beta, "f32"), to_device(d_out, dt),
                          to_device(w.initial_state, "f32") if w.initial_state is not None else None,
                          to_device(w.cu_seqlens, "i32") if use_cu else None,
                          to_device(d_final, "f32") if d_final is not None else None, N=w.N, check_status=True)
    torch.cuda.synchronize()
    return [to_host(g) for g in grads]


def _check(got, ref):
    for name, g, r in zip(NAMES, got, ref):
        assert g.shape == r.shape, name
        assert_backward_close(g, r, name)


@pytest.mark.parametrize("qkv_dtype", ["f32", "bf16"])
def test_backward_matches_oracle_on_ragged_packed_sequences(kda, qkv_dtype):
    w = I.make_prefill([37, 64, 0, 100, 1, 17], 2, 128, 128, seed=I.SEED_BASE + 60, qkv_dtype=qkv_dtype)
    d_out, d_final = I.make_cotangents(w.total_T, w.N, 2, 128, seed=I.SEED_BASE + 61, qkv_dtype=qkv_dtype)
    got = _gpu(kda, w, d_out, d_final)
    ref = O.kda_backward(w.q, w.k, w.v, w.log_alpha, w.beta, w.initial_state, w.cu_seqlens, d_out, d_final)
    _check(got, ref)
    # the empty sequence passes the final state's gradient straight through
    np.testing.assert_array_equal(got[5][2], d_final[2].astype(np.float64))


def test_backward_equal_lengths_without_states(kda):
    w = I.make_prefill([80, 80, 80], 3, 128, 128, seed=I.SEED_BASE + 62, state_std=0.0)
    d_out, _ = I.make_cotangents(w.total_T, w.N, 3, 128, seed=I.SEED_BASE + 63, final_std=0.0)
    got = _gpu(kda, w, d_out, None, use_cu=False)
    ref = O.kda_backward(w.q, w.k, w.v, w.log_alpha, w.beta, None, w.cu_seqlens, d_out, None)
    _check(got, ref)


def test_backward_many_chains_persistent_grid(kda):
    # more (sequence, head) chains than the 37 four-CTA clusters of the persistent grid
    w = I.make_prefill([20] * 40, 4, 128, 128, seed=I.SEED_BASE + 64)
    d_out, d_final = I.make_cotangents(w.total_T, w.N, 4, 128, seed=I.SEED_BASE + 65)
    got = _gpu(kda, w, d_out, d_final)
    ref = O.kda_backward(w.q, w.k, w.v, w.log_alpha, w.beta, w.initial_state, w.cu_seqlens, d_out, d_final)
    _check(got, ref)


def test_backward_model_shape_sampled_heads(kda):
    w = I.prefill_model_shape()
    d_out, d_final = I.make_cotangents(w.total_T, w.N, w.H, 128, seed=I.SEED_BASE + 66)
    got = _gpu(kda, w, d_out, d_final)
    for h in (0, 17, 31):
        sl = slice(h, h + 1)
        ref = O.kda_backward(w.q[:, sl], w.k[:, sl], w.v[:, sl], w.log_alpha[:, sl], w.beta[:, sl],
                             w.initial_state[:, sl], w.cu_seqlens, d_out[:, sl], d_final[:, sl])
        _check([g[:, sl] for g in got], ref)


def test_backward_of_only_empty_sequences(kda):
    # no tokens at all: the initial state's gradient is the final state's, exactly
    import torch
    H = 2
    z = lambda dt: torch.empty((0, H, 128), dtype=dt, device="cuda")
    cu = torch.zeros(4, dtype=torch.int32, device="cuda")
    d_final = torch.randn(3, H, 128, 128, device="cuda", generator=torch.Generator("cuda").manual_seed(5))
    s0 = torch.zeros(3, H, 128, 128, device="cuda")
    grads = kda.chunk_bwd(z(torch.bfloat16), z(torch.bfloat16), z(torch.bfloat16), z(torch.float32),
                          torch.empty((0, H), device="cuda"), z(torch.bfloat16), s0, cu, d_final, N=3,
                          check_status=True)
    torch.cuda.synchronize()
    assert all(g.numel() == 0 for g in grads[:5])
    assert torch.equal(grads[5], d_final)


def test_backward_flags_bad_seqlens(kda):
    import torch
    w = I.make_prefill([100, 100], 2, 128, 128, seed=I.SEED_BASE + 67)
    d_out, _ = I.make_cotangents(w.total_T, w.N, 2, 128, seed=I.SEED_BASE + 68, final_std=0.0)
    args = [to_device(x, "bf16") for x in (w.q, w.k, w.v)] + [to_device(w.log_alpha, "f32"),
                                                             to_device(w.beta, "f32"), to_device(d_out, "bf16")]
    bad_cu = torch.tensor([0, 150, 120], dtype=torch.int32, device="cuda")  # not monotone, short of total_T
    with pytest.raises(kda.KdaError):
        kda.chunk_bwd(*args, None, bad_cu, None, N=2, check_status=True)
    # a valid call afterwards reports a clean status and matches the oracle
    got = [to_host(g) for g in kda.chunk_bwd(*args, None, to_device(w.cu_seqlens, "i32"), None, N=2,
                                              check_status=True)]
    ref = O.kda_backward(w.q, w.k, w.v, w.log_alpha, w.beta, None, w.cu_seqlens, d_out, None)
    _check(got, ref)
