"""GPU parity: libkda.so (through the C ABI) against the fp64 oracle on the same
seeded inputs. Small cases are compared element by element; the full-size
workloads are compared on sampled (sequence, head) chains that the oracle runs
in full. Tolerances: prefill max|err| <= 2e-2 * RMS per tensor; decode fp32
state max|err| <= 1e-4 * max|ref| (bf16 outputs also get their rounding)."""
import numpy as np
import pytest

from gated_delta_rule_137_b200 import inputs as I
from oracle import kda_oracle as O
from tests.helpers import (assert_decode_out_close, assert_decode_state_close, assert_prefill_close, to_device,
                           to_host)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    import torch
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    from gated_delta_rule_137_b200 import build
    build.build()
    import gated_delta_rule_137_b200 as m
    m.load_library()
    return m


def _upload(w):
    dt = w.qkv_dtype
    return dict(q=to_device(w.q, dt), k=to_device(w.k, dt), v=to_device(w.v, dt),
                log_alpha=to_device(w.log_alpha, "f32"), beta=to_device(w.beta, "f32"),
                initial_state=None if w.initial_state is None else to_device(w.initial_state, "f32"),
                cu_seqlens=to_device(w.cu_seqlens, "i32"))


def _run_prefill(kda, w, varlen=True):
    import torch
    d = _upload(w)
    out, fin = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["initial_state"],
                             d["cu_seqlens"] if varlen else None, N=w.N, check_status=True)
    torch.cuda.synchronize()
    return to_host(out), to_host(fin)


def _oracle_heads(w, heads):
    hs = list(heads)
    s0 = None if w.initial_state is None else w.initial_state[:, hs]
    return O.kda_recurrence(w.q[:, hs], w.k[:, hs], w.v[:, hs], w.log_alpha[:, hs], w.beta[:, hs], s0, w.cu_seqlens)


# --------------------------------------------------------------------------- decode

def test_decode_small_bf16(kda):
    import torch
    w = I.make_decode(3, 2, 128, 128, 5, seed=11)
    st = to_device(w.state, "f32")
    outs = []
    for s in range(w.steps):
        outs.append(to_host(kda.decode_step(to_device(w.q[s], "bf16"), to_device(w.k[s], "bf16"),
                                            to_device(w.v[s], "bf16"), to_device(w.log_alpha[s], "f32"),
                                            to_device(w.beta[s], "f32"), st)))
    torch.cuda.synchronize()
    ref_o, ref_s = O.kda_decode_steps(w.q, w.k, w.v, w.log_alpha, w.beta, w.state)
    assert_decode_out_close(np.stack(outs), ref_o, "decode out")
    assert_decode_state_close(to_host(st), ref_s, "decode state")


def test_decode_small_dims_f32(kda):
    import torch
    rng = np.random.default_rng(12)
    N, H, dk, dv, steps = 2, 3, 16, 8, 4
    q = rng.standard_normal((steps, N, H, dk)).astype(np.float32)
    k = (rng.standard_normal((steps, N, H, dk)) / 4).astype(np.float32)
    v = rng.standard_normal((steps, N, H, dv)).astype(np.float32)
    la = (-rng.random((steps, N, H, dk)) / 4).astype(np.float32)
    b = rng.random((steps, N, H)).astype(np.float32)
    s0 = rng.standard_normal((N, H, dk, dv)).astype(np.float32)
    st = to_device(s0, "f32")
    outs = []
    for s in range(steps):
        outs.append(to_host(kda.decode_step(to_device(q[s], "f32"), to_device(k[s], "f32"), to_device(v[s], "f32"),
                                            to_device(la[s], "f32"), to_device(b[s], "f32"), st)))
    torch.cuda.synchronize()
    ref_o, ref_s = O.kda_decode_steps(q, k, v, la, b, s0)
    assert_decode_state_close(np.stack(outs), ref_o, "decode out (fp32)")
    assert_decode_state_close(to_host(st), ref_s, "decode state (fp32)")


def test_decode_model_shape_64_steps(kda):
    """256 sequences x 32 heads x 128 x 128 fp32 state in place, 64 consecutive steps;
    the oracle follows every 32nd sequence (all heads, all steps)."""
    import torch
    w = I.decode_batch()
    st = to_device(w.state, "f32")
    subset = np.arange(0, w.N, 32)
    outs = []
    for s in range(w.steps):
        o = kda.decode_step(to_device(w.q[s], "bf16"), to_device(w.k[s], "bf16"), to_device(w.v[s], "bf16"),
                            to_device(w.log_alpha[s], "f32"), to_device(w.beta[s], "f32"), st)
        outs.append(to_host(o[torch.as_tensor(subset, device=o.device)]))
    torch.cuda.synchronize()
    ref_o, ref_s = O.kda_decode_steps(w.q, w.k, w.v, w.log_alpha, w.beta, w.state, seq_subset=subset)
    assert_decode_out_close(np.stack(outs), ref_o, "decode out")
    assert_decode_state_close(to_host(st)[subset], ref_s, "decode state")


# --------------------------------------------------------------------------- prefill

def test_prefill_tiny_fp32_d16(kda):
    """B=1, T=64, H=2, d=16 fp32 (zero-padded to the d=128 kernel), chunk-aligned."""
    w = I.tiny_recurrence()
    out, fin = _run_prefill(kda, w, varlen=False)
    ro, rf = O.kda_recurrence(w.q, w.k, w.v, w.log_alpha, w.beta, None, w.cu_seqlens)
    assert_prefill_close(out, ro, "out", stored_bf16=False)
    assert_prefill_close(fin, rf, "final_state")


@pytest.mark.parametrize("lens,H,dk,dv,dtype", [
    ([200], 2, 128, 128, "bf16"),                 # ragged tail, 32-column slices
    ([64, 1, 130, 0, 63, 129], 3, 128, 128, "bf16"),  # varlen, empty and 1-token sequences
    ([150], 1, 128, 128, "f32"),                  # fp32 q/k/v through the staging path
    ([70, 33], 2, 64, 32, "bf16"),                # dk, dv below 128 (zero padding)
    ([96] * 4, 12, 128, 128, "bf16"),             # 48 chains -> 64-column slices
    ([70] * 10, 32, 128, 128, "bf16"),            # 320 chains -> full 128-column CTAs
])
def test_prefill_small_cases(kda, lens, H, dk, dv, dtype):
    w = I.make_prefill(lens, H, dk, dv, seed=sum(lens) + H, qkv_dtype=dtype)
    out, fin = _run_prefill(kda, w)
    ro, rf = O.kda_recurrence(w.q, w.k, w.v, w.log_alpha, w.beta, w.initial_state, w.cu_seqlens)
    assert_prefill_close(out, ro, "out", stored_bf16=(dtype == "bf16"))
    assert_prefill_close(fin, rf, "final_state")


def test_prefill_model_shape_all_heads(kda):
    """B=1, T=4096, H=32, d=128 bf16 with N(0, 0.02^2) initial state (the headline
    workload, through the two-pass kernels the bench times); the oracle runs every head."""
    w = I.prefill_model_shape()
    out, fin = _run_prefill(kda, w, varlen=False)
    ro, rf = _oracle_heads(w, range(w.H))
    assert_prefill_close(out, ro, "out", stored_bf16=True)
    assert_prefill_close(fin, rf, "final_state")


def test_prefill_varlen_sampled(kda):
    """64 packed sequences, lengths U[256, 8192], per-sequence initial states."""
    w = I.varlen_prefill()
    out, fin = _run_prefill(kda, w)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(fin))
    lens = np.diff(w.cu_seqlens)
    longest, shortest = int(np.argmax(lens)), int(np.argmin(lens))
    # the longest sequence on four heads, the shortest on two, and ten more (sequence, head)
    # chains spread over the batch: 16 chains
    picks = [(longest, h) for h in (0, 9, 21, 30)] + [(shortest, h) for h in (5, 31)]
    picks += [(n, (7 * n + 3) % w.H) for n in range(1, w.N, 6)][:10]
    for n, h in picks:
        s, e = int(w.cu_seqlens[n]), int(w.cu_seqlens[n + 1])
        ro, rf = O.kda_recurrence(w.q[s:e, h:h + 1], w.k[s:e, h:h + 1], w.v[s:e, h:h + 1],
                                  w.log_alpha[s:e, h:h + 1], w.beta[s:e, h:h + 1],
                                  w.initial_state[n:n + 1, h:h + 1], np.array([0, e - s]))
        assert_prefill_close(out[s:e, h:h + 1], ro, f"out seq {n} head {h}", stored_bf16=True)
        assert_prefill_close(fin[n:n + 1, h:h + 1], rf, f"final seq {n} head {h}")


def test_prefill_many_short_sequences(kda):
    """1500 packed sequences (more than one 1024-wide block of the chunk-offset scan),
    mostly 0..5 tokens with a few longer ones; oracle on a sample of sequences."""
    rng = np.random.default_rng(I.SEED_BASE + 31)
    lens = [int(x) for x in rng.integers(0, 6, 1500)]
    for i, L in ((3, 70), (1024, 130), (1499, 64)):
        lens[i] = L
    w = I.make_prefill(lens, 1, 128, 128, seed=I.SEED_BASE + 32)
    out, fin = _run_prefill(kda, w)
    picks = sorted(set([3, 1023, 1024, 1025, 1499] + list(range(0, 1500, 97))))
    for n in picks:
        s, e = int(w.cu_seqlens[n]), int(w.cu_seqlens[n + 1])
        ro, rf = O.kda_recurrence(w.q[s:e], w.k[s:e], w.v[s:e], w.log_alpha[s:e], w.beta[s:e],
                                  w.initial_state[n:n + 1], np.array([0, e - s]))
        if e > s:
            assert_prefill_close(out[s:e], ro, f"out seq {n} (len {e - s})", stored_bf16=True)
        assert_prefill_close(fin[n:n + 1], rf, f"final seq {n} (len {e - s})")


def test_prefill_two_pass_limit_and_many_short_sequences(kda):
    """74 (sequence, head) chains run the two-pass kernels, 75 the single-pass kernel (the
    workspace query tells which). 74 packed sequences of 0..130 tokens (empty, single-token
    and chunk-boundary lengths) through the two-pass path against the oracle; then one more
    sequence through the single-pass path, which must agree on the shared sequences."""
    import torch
    rng = np.random.default_rng(I.SEED_BASE + 33)
    lens = [int(x) for x in rng.integers(0, 131, 74)]
    lens[:6] = [0, 1, 63, 64, 65, 128]
    w = I.make_prefill(lens + [40], 1, 128, 128, seed=I.SEED_BASE + 34)
    assert kda.chunk_fwd_workspace_bytes(int(w.cu_seqlens[74]), 74, 1, 128, 128, kda.KDA_DT_BF16) > 256
    assert kda.chunk_fwd_workspace_bytes(int(w.cu_seqlens[75]), 75, 1, 128, 128, kda.KDA_DT_BF16) == 256
    d = _upload(w)
    T74 = int(w.cu_seqlens[74])
    cut = lambda x: x[:T74].contiguous()
    out2, fin2 = kda.chunk_fwd(cut(d["q"]), cut(d["k"]), cut(d["v"]), cut(d["log_alpha"]), cut(d["beta"]),
                               d["initial_state"][:74].contiguous(), d["cu_seqlens"][:75].contiguous(), N=74,
                               check_status=True)
    out1, fin1 = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["initial_state"],
                               d["cu_seqlens"], N=75, check_status=True)
    torch.cuda.synchronize()
    out2, fin2, out1, fin1 = to_host(out2), to_host(fin2), to_host(out1), to_host(fin1)
    ro, rf = O.kda_recurrence(w.q, w.k, w.v, w.log_alpha, w.beta, w.initial_state, w.cu_seqlens)
    assert_prefill_close(out2, ro[:T74], "two-pass out (74 sequences)", stored_bf16=True)
    assert_prefill_close(fin2, rf[:74], "two-pass final states")
    assert_prefill_close(out1, ro, "single-pass out (75 sequences)", stored_bf16=True)
    assert_prefill_close(fin1, rf, "single-pass final states")


def test_prefill_split_and_state_alias(kda):
    """run(T) == run(T1) then run(T - T1) from the carried state, with final_state
    written over initial_state in place; and prefill then one decode step equals
    the prefill of one more token."""
    import torch
    w = I.make_prefill([301], 4, 128, 128, seed=5)
    d = _upload(w)
    T, T1 = 300, 100
    part = lambda x, a, b: x[a:b].contiguous()
    ro, rf = O.kda_recurrence(w.q[:T], w.k[:T], w.v[:T], w.log_alpha[:T], w.beta[:T], w.initial_state,
                              np.array([0, T]))
    out, fin = kda.chunk_fwd(part(d["q"], 0, T), part(d["k"], 0, T), part(d["v"], 0, T),
                             part(d["log_alpha"], 0, T), part(d["beta"], 0, T), d["initial_state"], None, N=1)
    st = d["initial_state"].clone()
    outs = []
    for a, b in ((0, T1), (T1, T)):
        o, _ = kda.chunk_fwd(part(d["q"], a, b), part(d["k"], a, b), part(d["v"], a, b),
                             part(d["log_alpha"], a, b), part(d["beta"], a, b), st, None, N=1, final_state=st)
        outs.append(to_host(o))
    torch.cuda.synchronize()
    assert_prefill_close(to_host(out), ro, "whole out", stored_bf16=True)
    assert_prefill_close(to_host(fin), rf, "whole final")
    assert_prefill_close(np.concatenate(outs), ro, "split out", stored_bf16=True)
    assert_prefill_close(to_host(st), rf, "split final (in place)")
    # one more token through the decode kernel, from the prefill's final state
    ro2, rf2 = O.kda_recurrence(w.q, w.k, w.v, w.log_alpha, w.beta, w.initial_state, w.cu_seqlens)
    sl = slice(T, T + 1)  # one sequence (N=1) of H=4 heads
    od = kda.decode_step(d["q"][sl], d["k"][sl], d["v"][sl], d["log_alpha"][sl], d["beta"][sl], fin)
    torch.cuda.synchronize()
    assert_prefill_close(to_host(od)[0], ro2[T], "decode after prefill", stored_bf16=True)
    assert_prefill_close(to_host(fin), rf2, "state after decode")


def test_prefill_zero_tokens_copies_state(kda):
    import torch
    s0 = torch.randn(2, 3, 128, 128, device="cuda")
    e = torch.empty(0, 3, 128, device="cuda", dtype=torch.bfloat16)
    la = torch.empty(0, 3, 128, device="cuda")
    b = torch.empty(0, 3, device="cuda")
    cu = torch.zeros(3, dtype=torch.int32, device="cuda")
    out, fin = kda.chunk_fwd(e, e, e, la, b, s0, cu, N=2)
    torch.cuda.synchronize()
    assert torch.equal(fin, s0)


def test_device_status_flags(kda):
    """A cu_seqlens that is not monotone is flagged; a decay of 3 nats per token in every
    channel (192 nats per chunk, beyond what e^g e^-g can carry in fp32) is not: those
    chunks are walked token by token and must match the oracle with a clean status."""
    import torch
    w = I.make_prefill([100, 100], 2, 128, 128, seed=9)
    d = _upload(w)
    bad_cu = torch.tensor([0, 150, 120], dtype=torch.int32, device="cuda")  # not monotone
    with pytest.raises(kda.KdaError) as err:
        kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, bad_cu, N=2, check_status=True)
    assert f"0x{kda.DEVFLAG_BAD_SEQLENS:08x}" in str(err.value)
    la = np.full_like(w.log_alpha, -3.0)
    out, fin = kda.chunk_fwd(d["q"], d["k"], d["v"], to_device(la, "f32"), d["beta"], d["initial_state"],
                             d["cu_seqlens"], N=2, check_status=True)
    torch.cuda.synchronize()
    ro, rf = O.kda_recurrence(w.q, w.k, w.v, la, w.beta, w.initial_state, w.cu_seqlens)
    assert_prefill_close(to_host(out), ro, "out at 3 nats per token", stored_bf16=True)
    assert_prefill_close(to_host(fin), rf, "final state at 3 nats per token")
    # a valid call afterwards reports a clean status
    kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, d["cu_seqlens"], N=2, check_status=True)


def test_wait_timeout_is_reported(kda):
    """Every wait inside the kernels is bounded. The diagnostic entry point runs one such
    wait on an mbarrier that nothing arrives at, with a 2 ms budget: it must give up,
    leave KDA_DEVFLAG_WAIT_TIMEOUT in the status word, and leave the context usable."""
    import torch
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    kda.selftest_wait_timeout(ws, 2000)
    with pytest.raises(kda.KdaError) as err:
        kda.workspace_status(ws)
    assert f"0x{kda.DEVFLAG_WAIT_TIMEOUT:08x}" in str(err.value)
    assert kda.workspace_status(ws) == 0  # read and cleared
    w = I.make_prefill([70], 2, 128, 128, seed=10)
    out, fin = _run_prefill(kda, w)  # the context still runs kernels
    ro, rf = O.kda_recurrence(w.q, w.k, w.v, w.log_alpha, w.beta, w.initial_state, w.cu_seqlens)
    assert_prefill_close(out, ro, "out after the timed-out wait", stored_bf16=True)


# ------------------------------------------------------------- strong per-channel decay

def _decay_pattern(w, scale, pattern):
    """log_alpha = -softplus(z) * scale per channel (the generator draws -softplus(z)/16).
    pattern "all": every chunk; "odd": only the odd 64-token chunks of each sequence (the
    even ones keep the generator's mild decay), so fast and walked chunks alternate."""
    la = w.log_alpha * (16.0 * scale)
    if pattern == "odd":
        keep = np.zeros(la.shape[0], dtype=bool)
        for n in range(w.N):
            s, e = int(w.cu_seqlens[n]), int(w.cu_seqlens[n + 1])
            keep[s:e] = ((np.arange(e - s) // 64) % 2) == 0
        la = np.where(keep[:, None, None], w.log_alpha, la)
    return la


@pytest.mark.parametrize("path", ["two-pass", "single-pass"])
@pytest.mark.parametrize("scale,pattern,dtype", [
    (1.0, "all", "bf16"),    # ~0.8 nats per token: chunks near and past the 80-nat line
    (8.0, "all", "bf16"),    # ~6.5 nats per token: every chunk walked
    (8.0, "odd", "bf16"),    # walked and tensor-core chunks alternate along each sequence
    (8.0, "odd", "f32"),
])
def test_prefill_strong_decay(kda, path, scale, pattern, dtype):
    """Per-channel decay far beyond the range of the factorised chunk form, through the
    two-pass kernels (<= 74 chains) and the single-pass kernel (> 74 chains), against the
    oracle's token recurrence; no status flag may be raised."""
    rng = np.random.default_rng(I.SEED_BASE + 41)
    if path == "two-pass":
        lens, H = [200, 64, 7, 131], 4                          # 16 chains, ragged tails
    else:
        lens, H = [int(x) for x in rng.integers(1, 200, 20)], 4  # 80 chains
        lens[:3] = [64, 65, 128]
    w = I.make_prefill(lens, H, 128, 128, seed=I.SEED_BASE + 42 + int(scale), qkv_dtype=dtype)
    la = _decay_pattern(w, scale, pattern)
    need = kda.chunk_fwd_workspace_bytes(w.total_T, w.N, H, 128, 128,
                                         kda.KDA_DT_BF16 if dtype == "bf16" else kda.KDA_DT_F32)
    assert (need > 256) == (path == "two-pass")
    d = _upload(w)
    import torch
    out, fin = kda.chunk_fwd(d["q"], d["k"], d["v"], to_device(la, "f32"), d["beta"], d["initial_state"],
                             d["cu_seqlens"], N=w.N, check_status=True)
    torch.cuda.synchronize()
    ro, rf = O.kda_recurrence(w.q, w.k, w.v, la, w.beta, w.initial_state, w.cu_seqlens)
    assert_prefill_close(to_host(out), ro, f"out ({path}, decay x{scale} {pattern})", stored_bf16=(dtype == "bf16"))
    assert_prefill_close(to_host(fin), rf, f"final state ({path}, decay x{scale} {pattern})")


@pytest.mark.parametrize("lens,H", [([300, 77], 4), ([70] * 40, 2)])  # two-pass; single-pass (80 chains)
def test_mixer_strong_decay(kda, lens, H):
    """The full mixer (conv4 + L2 inside the kernels, sigmoid gate) with strong decay on
    the odd chunks: the walked chunks must see the conv'd, normalised q, k, v."""
    w = I.make_prefill(lens, H, 128, 128, seed=sum(lens) + 43, normalise_qk=False, mixer=True)
    la = _decay_pattern(w, 8.0, "odd")
    import torch
    dt = "bf16"
    out, fin = kda.mixer_fwd(to_device(w.q, dt), to_device(w.k, dt), to_device(w.v, dt), to_device(w.conv_w, "f32"),
                             to_device(la, "f32"), to_device(w.beta, "f32"), to_device(w.gate, dt),
                             to_device(w.initial_state, "f32"), to_device(w.cu_seqlens, "i32"), N=w.N,
                             check_status=True)
    torch.cuda.synchronize()
    ro, rf = O.kda_mixer(w.q, w.k, w.v, w.conv_w, la, w.beta, w.gate, w.cu_seqlens, w.initial_state)
    assert_prefill_close(to_host(out), ro, "strong-decay mixer out", stored_bf16=True)
    assert_prefill_close(to_host(fin), rf, "strong-decay mixer final state")


def test_mixer_gate_from_preactivation_strong(kda):
    """kda_mixer_fwd_gate with per-head scales of 4..8 on softplus(a): about 3-6 nats per
    token, so most chunks are walked with log_alpha made on the device."""
    import torch
    w = I.make_prefill([300, 77], 4, 128, 128, seed=44, normalise_qk=False, mixer=True)
    a_pre, _ = I.make_gate_preactivation(w.q.shape[0], 4, 128, seed=45)
    a_scale = np.array([4.0, 5.0, 6.0, 8.0])
    dt = "bf16"
    out, fin = kda.mixer_fwd_gate(to_device(w.q, dt), to_device(w.k, dt), to_device(w.v, dt),
                                  to_device(w.conv_w, "f32"), to_device(a_pre, "bf16"), to_device(a_scale, "f32"),
                                  to_device(w.beta, "f32"), to_device(w.gate, dt), to_device(w.initial_state, "f32"),
                                  to_device(w.cu_seqlens, "i32"), N=w.N, check_status=True)
    torch.cuda.synchronize()
    la = O.gate_log_alpha(a_pre, a_scale)
    ro, rf = O.kda_mixer(w.q, w.k, w.v, w.conv_w, la, w.beta, w.gate, w.cu_seqlens, w.initial_state)
    assert_prefill_close(to_host(out), ro, "strong gate-from-pre-activation out", stored_bf16=True)
    assert_prefill_close(to_host(fin), rf, "strong gate-from-pre-activation final state")


# --------------------------------------------------------------------------- mixer

def _mixer_oracle_heads(w, heads):
    outs, fins = [], []
    d = w.dk
    for h in heads:
        sl = slice(h * d, (h + 1) * d)
        cw = w.conv_w[:, sl]
        o, f = O.kda_mixer(w.q[:, h:h + 1], w.k[:, h:h + 1], w.v[:, h:h + 1], cw, w.log_alpha[:, h:h + 1],
                           w.beta[:, h:h + 1], w.gate[:, h:h + 1], w.cu_seqlens)
        outs.append(o)
        fins.append(f)
    return np.concatenate(outs, axis=1), np.concatenate(fins, axis=1)


def _run_mixer(kda, w):
    import torch
    dt = "bf16"
    out, fin = kda.mixer_fwd(to_device(w.q, dt), to_device(w.k, dt), to_device(w.v, dt), to_device(w.conv_w, "f32"),
                             to_device(w.log_alpha, "f32"), to_device(w.beta, "f32"), to_device(w.gate, dt), None,
                             to_device(w.cu_seqlens, "i32"), N=w.N, check_status=True)
    torch.cuda.synchronize()
    return to_host(out), to_host(fin)


def test_mixer_small(kda):
    w = I.make_prefill([300, 77], 4, 128, 128, seed=21, state_std=0.0, normalise_qk=False, mixer=True)
    out, fin = _run_mixer(kda, w)
    ro, rf = _mixer_oracle_heads(w, range(4))
    assert_prefill_close(out, ro, "mixer out", stored_bf16=True)
    assert_prefill_close(fin, rf, "mixer final")


def test_mixer_full_size_sampled_heads(kda):
    """B=2, T=32768, H=32, d=128: conv4 + L2 + KDA + sigmoid gate; oracle on 8 heads."""
    w = I.mixer_prefill()
    out, fin = _run_mixer(kda, w)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(fin))
    heads = [0, 3, 8, 13, 17, 22, 28, 31]
    ro, rf = _mixer_oracle_heads(w, heads)
    assert_prefill_close(out[:, heads], ro, "mixer out", stored_bf16=True)
    assert_prefill_close(fin[:, heads], rf, "mixer final")


@pytest.mark.parametrize("lens,H", [([300, 77], 4), ([70] * 40, 2)])  # 8 chains; 80 chains (several waves)
def test_mixer_gate_from_preactivation(kda, lens, H):
    """kda_mixer_fwd_gate: log_alpha = -a_scale[h] softplus(a_pre) made on the device."""
    import torch
    w = I.make_prefill(lens, H, 128, 128, seed=sum(lens) + H + 7, normalise_qk=False, mixer=True)
    a_pre, a_scale = I.make_gate_preactivation(w.q.shape[0], H, 128, seed=sum(lens) + 8)
    dt = "bf16"
    out, fin = kda.mixer_fwd_gate(to_device(w.q, dt), to_device(w.k, dt), to_device(w.v, dt),
                                  to_device(w.conv_w, "f32"), to_device(a_pre, "bf16"), to_device(a_scale, "f32"),
                                  to_device(w.beta, "f32"), to_device(w.gate, dt), to_device(w.initial_state, "f32"),
                                  to_device(w.cu_seqlens, "i32"), N=w.N, check_status=True)
    torch.cuda.synchronize()
    la = O.gate_log_alpha(a_pre, a_scale)
    ro, rf = O.kda_mixer(w.q, w.k, w.v, w.conv_w, la, w.beta, w.gate, w.cu_seqlens, w.initial_state)
    assert_prefill_close(to_host(out), ro, "gate-from-pre-activation mixer out", stored_bf16=True)
    assert_prefill_close(to_host(fin), rf, "gate-from-pre-activation mixer final state")
