"""kda_mixer_decode_step (the serving decode step of the full mixer) through the C ABI
against the oracle's kda_mixer_decode_step: several consecutive steps on sequences
whose states and conv histories sit at permuted slots of larger pools. The out rows and
states are held to the decode tolerance; the rolled conv histories must be bit-exact
(they are copies of bf16 inputs), and the slots no sequence uses must not change."""
import numpy as np
import pytest

from gated_delta_rule_137_b200 import inputs as I
from oracle import kda_oracle as O
from tests.helpers import assert_decode_out_close, assert_decode_state_close, assert_prefill_close, to_device, to_host

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


def _run(kda, w, use_gate=True):
    import torch
    sp = to_device(w.state_pool, "f32")
    cp = to_device(w.conv_pool, "bf16")
    idx = to_device(w.indices, "i32")
    cw = to_device(w.conv_w, "f32")
    status = torch.zeros(64, dtype=torch.int32, device="cuda")
    outs = []
    for s in range(w.steps):
        o = kda.mixer_decode_step(to_device(w.q[s], "bf16"), to_device(w.k[s], "bf16"), to_device(w.v[s], "bf16"),
                                  cw, to_device(w.log_alpha[s], "f32"), to_device(w.beta[s], "f32"),
                                  to_device(w.gate[s], "bf16") if use_gate else None, sp, cp, idx, status=status)
        outs.append(to_host(o))
    torch.cuda.synchronize()
    return np.stack(outs), to_host(sp), cp, int(to_host(status)[0])


def _oracle(w, use_gate=True):
    idx = w.indices
    S, hist = w.state_pool[idx], w.conv_pool[idx]
    outs = []
    for s in range(w.steps):
        o, S, hist = O.kda_mixer_decode_step(w.q[s], w.k[s], w.v[s], w.conv_w, w.log_alpha[s], w.beta[s],
                                             w.gate[s] if use_gate else None, S, hist)
        outs.append(o)
    return np.stack(outs), S, hist


@pytest.mark.parametrize("use_gate", [True, False])
def test_mixer_decode_matches_oracle_on_permuted_pool_slots(kda, use_gate):
    import torch
    w = I.make_mixer_decode(12, 4, 128, 3, 20, seed=I.SEED_BASE + 41)
    out, sp, cp, status = _run(kda, w, use_gate)
    ro, rs, rh = _oracle(w, use_gate)
    assert status == 0
    assert_decode_out_close(out, ro, "mixer decode out")
    assert_decode_state_close(sp[w.indices], rs, "mixer decode state")
    # the history holds copies of bf16 inputs: bit-exact
    got_h = cp.view(torch.int16).cpu().numpy().view(np.uint16)
    ref_h = I.bf16_bits(rh)
    np.testing.assert_array_equal(got_h[w.indices], ref_h)
    unused = np.setdiff1d(np.arange(w.pool), w.indices)
    np.testing.assert_array_equal(sp[unused], w.state_pool[unused].astype(np.float32))
    np.testing.assert_array_equal(got_h[unused], I.bf16_bits(w.conv_pool[unused]))


def test_mixer_decode_flags_an_index_outside_the_pool(kda):
    import torch
    w = I.make_mixer_decode(4, 2, 128, 1, 6, seed=I.SEED_BASE + 42)
    w.indices = np.array([0, 9, 2, -1], dtype=np.int32)  # 9 and -1 are outside [0, 6)
    out, sp, cp, status = _run(kda, w)
    assert status & kda.DEVFLAG_BAD_INDEX
    # the valid sequences still match the oracle, the slots of the others are untouched
    ok = np.array([0, 2])
    w2 = I.make_mixer_decode(4, 2, 128, 1, 6, seed=I.SEED_BASE + 42)
    S, hist = w2.state_pool[[0, 2]], w2.conv_pool[[0, 2]]
    ro, rs, _ = O.kda_mixer_decode_step(w2.q[0][ok], w2.k[0][ok], w2.v[0][ok], w2.conv_w, w2.log_alpha[0][ok],
                                        w2.beta[0][ok], w2.gate[0][ok], S, hist)
    assert_decode_out_close(out[0][ok], ro, "valid rows")
    assert_decode_state_close(sp[[0, 2]], rs, "valid states")
    for slot in (1, 3, 4, 5):
        np.testing.assert_array_equal(sp[slot], w2.state_pool[slot].astype(np.float32))


def _tok(x):
    """[K, N, ...] as drawn by the generator -> [N, K, ...] as the multi-token call takes it."""
    return np.ascontiguousarray(np.swapaxes(x, 0, 1))


@pytest.mark.parametrize("K", [2, 3, 4, 6])  # 2..4: the one-pass block form; 6: token by token
def test_mixer_decode_tokens_without_checkpoints_matches_k_steps(kda, K):
    import torch
    w = I.make_mixer_decode(10, 4, 128, K, 16, seed=I.SEED_BASE + 43 + K)
    sp, cp = to_device(w.state_pool, "f32"), to_device(w.conv_pool, "bf16")
    out = kda.mixer_decode_tokens(to_device(_tok(w.q), "bf16"), to_device(_tok(w.k), "bf16"),
                                  to_device(_tok(w.v), "bf16"), to_device(w.conv_w, "f32"),
                                  to_device(_tok(w.log_alpha), "f32"), to_device(_tok(w.beta), "f32"),
                                  to_device(_tok(w.gate), "bf16"), sp, cp, to_device(w.indices, "i32"))
    torch.cuda.synchronize()
    idx = w.indices
    ro, rs, rh = O.kda_mixer_decode_tokens(_tok(w.q), _tok(w.k), _tok(w.v), w.conv_w, _tok(w.log_alpha),
                                           _tok(w.beta), _tok(w.gate), w.state_pool[idx], w.conv_pool[idx])
    assert_decode_out_close(to_host(out), ro, "K-token out")
    assert_decode_state_close(to_host(sp)[idx], rs[:, -1], "state after K tokens")
    np.testing.assert_array_equal(cp.view(torch.int16).cpu().numpy().view(np.uint16)[idx], I.bf16_bits(rh[:, -1]))


@pytest.mark.parametrize("K", [3, 4, 5])
def test_mixer_decode_tokens_checkpoints_and_commit(kda, K):
    import torch
    w = I.make_mixer_decode(6, 2, 128, K, 9, seed=I.SEED_BASE + 44 + K)
    N, H = 6, 2
    sp, cp = to_device(w.state_pool, "f32"), to_device(w.conv_pool, "bf16")
    idx = to_device(w.indices, "i32")
    sck = torch.full((N, K, H, 128, 128), float("nan"), device="cuda")
    cck = torch.zeros((N, K, H, 3, 3, 128), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(64, dtype=torch.int32, device="cuda")
    out = kda.mixer_decode_tokens(to_device(_tok(w.q), "bf16"), to_device(_tok(w.k), "bf16"),
                                  to_device(_tok(w.v), "bf16"), to_device(w.conv_w, "f32"),
                                  to_device(_tok(w.log_alpha), "f32"), to_device(_tok(w.beta), "f32"),
                                  to_device(_tok(w.gate), "bf16"), sp, cp, idx, state_ckpt=sck, conv_ckpt=cck,
                                  status=status)
    torch.cuda.synchronize()
    # with checkpoints the pools stay as they were
    np.testing.assert_array_equal(to_host(sp), w.state_pool.astype(np.float32))
    ro, rs, rh = O.kda_mixer_decode_tokens(_tok(w.q), _tok(w.k), _tok(w.v), w.conv_w, _tok(w.log_alpha),
                                           _tok(w.beta), _tok(w.gate), w.state_pool[w.indices],
                                           w.conv_pool[w.indices])
    assert_decode_out_close(to_host(out), ro, "K-token out")
    assert_decode_state_close(to_host(sck), rs, "checkpoint states")
    ck_bits = cck.view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(ck_bits, I.bf16_bits(rh))
    # commit: sequence n keeps accepted[n] tokens
    accepted = np.array([0, 1, K, 2, 3, 1], dtype=np.int32)
    kda.mixer_decode_commit(sck, cck, to_device(accepted, "i32"), sp, cp, idx, status=status)
    torch.cuda.synchronize()
    assert int(to_host(status)[0]) == 0
    got_s, got_h = to_host(sp), cp.view(torch.int16).cpu().numpy().view(np.uint16)
    sck_h = to_host(sck)
    for n, a in enumerate(accepted):
        slot = w.indices[n]
        if a == 0:
            np.testing.assert_array_equal(got_s[slot], w.state_pool[slot].astype(np.float32))
            np.testing.assert_array_equal(got_h[slot], I.bf16_bits(w.conv_pool[slot]))
        else:
            np.testing.assert_array_equal(got_s[slot], sck_h[n, a - 1])
            np.testing.assert_array_equal(got_h[slot], ck_bits[n, a - 1])
    unused = np.setdiff1d(np.arange(w.pool), w.indices)
    np.testing.assert_array_equal(got_s[unused], w.state_pool[unused].astype(np.float32))


def test_mixer_decode_one_token_call_is_the_decode_step(kda):
    import torch
    w = I.make_mixer_decode(5, 2, 128, 1, 5, seed=I.SEED_BASE + 45)
    outs = []
    for multi in (False, True):
        sp, cp = to_device(w.state_pool, "f32"), to_device(w.conv_pool, "bf16")
        args = [to_device(x, dt) for x, dt in ((w.q, "bf16"), (w.k, "bf16"), (w.v, "bf16"))]
        if multi:
            o = kda.mixer_decode_tokens(*[a.transpose(0, 1).contiguous() for a in args], to_device(w.conv_w, "f32"),
                                        to_device(_tok(w.log_alpha), "f32"), to_device(_tok(w.beta), "f32"),
                                        to_device(_tok(w.gate), "bf16"), sp, cp)[:, 0]
        else:
            o = kda.mixer_decode_step(*[a[0] for a in args], to_device(w.conv_w, "f32"),
                                      to_device(w.log_alpha[0], "f32"), to_device(w.beta[0], "f32"),
                                      to_device(w.gate[0], "bf16"), sp, cp)
        torch.cuda.synchronize()
        outs.append((to_host(o), to_host(sp)))
    np.testing.assert_array_equal(outs[0][0], outs[1][0])
    np.testing.assert_array_equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("lens,H", [([130, 2, 64, 0], 4),        # 16 chains: the two-pass prefill
                                    ([70] * 19 + [1], 4),       # 80 chains: the single-pass prefill
                                    ([0] + [66] * 18 + [3], 4)])  # single-pass, an empty prompt first
def test_pooled_prefill_hands_over_to_the_decode_step(kda, lens, H):
    """kda_mixer_fwd_pooled over each sequence's first T tokens into permuted slots of
    larger pools, then kda_mixer_decode_step on token T + 1, against oracle.kda_mixer over
    all T + 1 tokens: the prefill's out rows, the pooled states and conv histories after
    the prefill (histories bit-exact: copies of bf16 inputs, zeros before a short prompt),
    the decode's out row and the state after it. Slots no sequence names stay untouched.
    The decode's results sit on a prefill-computed state, so they are held to the prefill's
    bar."""
    import torch
    N, d = len(lens), 128
    w = I.make_prefill([L + 1 for L in lens], H, d, d, seed=I.SEED_BASE + 43 + N, normalise_qk=False, mixer=True)
    cu = w.cu_seqlens
    first = np.concatenate([np.arange(cu[n], cu[n + 1] - 1) for n in range(N)]).astype(np.int64)
    last = cu[1:] - 1
    pcu = np.zeros(N + 1, dtype=np.int32)
    pcu[1:] = np.cumsum(lens)
    pool = N + 5
    rng = np.random.default_rng(I.SEED_BASE + 44)
    slots = rng.permutation(pool)[:N].astype(np.int32)
    sp0 = rng.standard_normal((pool, H, d, d)).astype(np.float32)
    cp0 = I.bf16_round(rng.standard_normal((pool, H, 3, 3, d)).astype(np.float32))
    sp, cp = to_device(sp0, "f32"), to_device(cp0, "bf16")
    idx = to_device(slots, "i32")
    cw = to_device(w.conv_w, "f32")
    sel = lambda x, rows, dt: to_device(x[rows], dt)
    out = kda.mixer_fwd_pooled(sel(w.q, first, "bf16"), sel(w.k, first, "bf16"), sel(w.v, first, "bf16"), cw,
                               sel(w.log_alpha, first, "f32"), sel(w.beta, first, "f32"), sel(w.gate, first, "bf16"),
                               sp, cp, idx, to_device(w.initial_state, "f32"), to_device(pcu, "i32"), N=N,
                               check_status=True)
    torch.cuda.synchronize()
    sp_pre, cp_pre = to_host(sp), cp.view(torch.int16).cpu().numpy().view(np.uint16).copy()
    status = torch.zeros(64, dtype=torch.int32, device="cuda")
    dout = kda.mixer_decode_step(sel(w.q, last, "bf16"), sel(w.k, last, "bf16"), sel(w.v, last, "bf16"), cw,
                                 sel(w.log_alpha, last, "f32"), sel(w.beta, last, "f32"), sel(w.gate, last, "bf16"),
                                 sp, cp, idx, status=status)
    torch.cuda.synchronize()
    assert int(to_host(status)[0]) == 0

    pre = [w.q[first], w.k[first], w.v[first], w.conv_w, w.log_alpha[first], w.beta[first], w.gate[first], pcu]
    ro_pre, rf_pre = O.kda_mixer(*pre, initial_state=w.initial_state)
    ro, rf = O.kda_mixer(w.q, w.k, w.v, w.conv_w, w.log_alpha, w.beta, w.gate, cu, initial_state=w.initial_state)
    assert_prefill_close(to_host(out), ro_pre, "pooled prefill out", stored_bf16=True)
    assert_prefill_close(sp_pre[slots], rf_pre, "pooled prefill state")
    assert_prefill_close(to_host(dout), ro[last], "decode out after the prefill", stored_bf16=True)
    assert_prefill_close(to_host(sp)[slots], rf, "state after prefill + decode")

    def history(rows_of):  # the last three raw rows of each sequence, oldest first, zeros before it
        h = np.zeros((N, H, 3, 3, d))
        for n in range(N):
            rows = rows_of(n)
            for r in range(3):
                t = len(rows) - 3 + r
                if t >= 0:
                    for i, x in enumerate((w.q, w.k, w.v)):
                        h[n, :, i, r] = x[rows[t]]
        return h

    np.testing.assert_array_equal(cp_pre[slots], I.bf16_bits(history(lambda n: np.arange(cu[n], cu[n + 1] - 1))))
    got_h = cp.view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got_h[slots], I.bf16_bits(history(lambda n: np.arange(cu[n], cu[n + 1]))))
    unused = np.setdiff1d(np.arange(pool), slots)
    np.testing.assert_array_equal(to_host(sp)[unused], sp0[unused])
    np.testing.assert_array_equal(got_h[unused], I.bf16_bits(cp0[unused]))


def test_pooled_prefill_flags_a_slot_outside_the_pool(kda):
    """A slot outside [0, pool_size) is reported and that sequence's pools are left alone;
    the other sequences are handed over as usual and every out row is written."""
    import torch
    lens, H, d = [40, 90], 2, 128
    w = I.make_prefill(lens, H, d, d, seed=I.SEED_BASE + 45, normalise_qk=False, mixer=True)
    pool = 3
    sp0 = np.zeros((pool, H, d, d), np.float32)
    cp0 = np.zeros((pool, H, 3, 3, d), np.float32)
    sp, cp = to_device(sp0, "f32"), to_device(cp0, "bf16")
    ws = torch.empty(kda.load_library().kda_mixer_fwd_workspace(w.total_T, 2, H, d, d), dtype=torch.uint8,
                     device="cuda")
    out = kda.mixer_fwd_pooled(to_device(w.q, "bf16"), to_device(w.k, "bf16"), to_device(w.v, "bf16"),
                               to_device(w.conv_w, "f32"), to_device(w.log_alpha, "f32"), to_device(w.beta, "f32"),
                               to_device(w.gate, "bf16"), sp, cp, to_device(np.array([7, 1], np.int32), "i32"),
                               to_device(w.initial_state, "f32"), to_device(w.cu_seqlens, "i32"), N=2, workspace=ws)
    torch.cuda.synchronize()
    with pytest.raises(kda.KdaError) as err:
        kda.workspace_status(ws)
    assert int(str(err.value).split("0x")[-1][:8], 16) == kda.DEVFLAG_BAD_INDEX
    ro, rf = O.kda_mixer(w.q, w.k, w.v, w.conv_w, w.log_alpha, w.beta, w.gate, w.cu_seqlens,
                         initial_state=w.initial_state)
    assert_prefill_close(to_host(out), ro, "out", stored_bf16=True)
    assert_prefill_close(to_host(sp)[1], rf[1], "state of the valid slot")
    np.testing.assert_array_equal(to_host(sp)[[0, 2]], 0.0)
    np.testing.assert_array_equal(to_host(cp)[[0, 2]], 0.0)


def test_pooled_prefill_of_empty_prompts_starts_the_slots(kda):
    """total_T = 0: nothing to prefill; each named slot gets the sequence's initial state (or
    zero) and an all-zero conv history, the other slots are untouched."""
    import torch
    N, H, d, pool = 3, 2, 128, 5
    rng = np.random.default_rng(I.SEED_BASE + 46)
    sp0 = rng.standard_normal((pool, H, d, d)).astype(np.float32)
    cp0 = I.bf16_round(rng.standard_normal((pool, H, 3, 3, d)).astype(np.float32))
    s0 = (0.02 * rng.standard_normal((N, H, d, d))).astype(np.float32)
    slots = np.array([4, 0, 2], dtype=np.int32)
    empty = lambda dt: to_device(np.zeros((0, H, d), np.float32), dt)
    for init in (s0, None):
        sp, cp = to_device(sp0, "f32"), to_device(cp0, "bf16")
        kda.mixer_fwd_pooled(empty("bf16"), empty("bf16"), empty("bf16"), to_device(np.ones((3, H * d, 4), np.float32), "f32"),
                             empty("f32"), to_device(np.zeros((0, H), np.float32), "f32"), None, sp, cp,
                             to_device(slots, "i32"), None if init is None else to_device(init, "f32"),
                             to_device(np.zeros(N + 1, np.int32), "i32"), N=N, check_status=True)
        torch.cuda.synchronize()
        got_s, got_h = to_host(sp), to_host(cp)
        want = np.zeros((N, H, d, d), np.float32) if init is None else init
        np.testing.assert_array_equal(got_s[slots], want)
        np.testing.assert_array_equal(got_h[slots], 0.0)
        np.testing.assert_array_equal(got_s[[1, 3]], sp0[[1, 3]])
        np.testing.assert_array_equal(got_h[[1, 3]], to_host(to_device(cp0, "bf16"))[[1, 3]])
