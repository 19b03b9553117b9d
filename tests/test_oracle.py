"""Pins for the fp64 oracle: facts the pages and the mathematics fix, each chosen
so that a plausible slip in the oracle (a dropped term, a sign, the read before
instead of after the write, decay on the wrong side of the state, a wrong conv
tap order) fails at least one of them. CPU only."""
import json
import os

import numpy as np
import pytest

from oracle import kda_oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


def _rand(seed, T, H, dk, dv, unit_k=True, decay_scale=1.0 / 16):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    la = -np.logaddexp(0, rng.standard_normal((T, H, dk))) * decay_scale
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    return q, k, v, la, beta


def _cu(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)


# --- the state is a fixed d_k x d_v matrix per head, whatever T is ----------------

@pytest.mark.parametrize("T", [1, 64, 65, 300])
def test_state_size_does_not_depend_on_T(T):
    q, k, v, la, b = _rand(1, T, 2, 8, 5)
    out, fin = O.kda_recurrence(q, k, v, la, b, None, _cu([T]))
    assert out.shape == (T, 2, 5)
    assert fin.shape == (1, 2, 8, 5)


# --- alpha = 1, beta = 0: nothing is erased or written --------------------------

def test_no_decay_no_write_keeps_state_and_reads_it():
    T, H, dk, dv = 20, 3, 6, 4
    q, k, v, _, _ = _rand(2, T, H, dk, dv)
    S0 = np.random.default_rng(3).standard_normal((1, H, dk, dv))
    out, fin = O.kda_recurrence(q, k, v, np.zeros((T, H, dk)), np.zeros((T, H)), S0, _cu([T]))
    np.testing.assert_array_equal(fin, S0)
    for t in range(T):
        for h in range(H):
            np.testing.assert_allclose(out[t, h], S0[0, h].T @ q[t, h], rtol=1e-14, atol=1e-14)


# --- the delta rule: alpha = 1, beta = 1, unit key => S_t^T k_t = v_t -----------

def test_delta_rule_reads_back_the_value_just_written():
    T, H, dk, dv = 40, 2, 16, 7
    _, k, v, _, _ = _rand(4, T, H, dk, dv, unit_k=True)
    S0 = np.random.default_rng(5).standard_normal((1, H, dk, dv))
    # query = key makes o_t the read-back S_t^T k_t (after the write)
    out, _ = O.kda_recurrence(k, k, v, np.zeros((T, H, dk)), np.ones((T, H)), S0, _cu([T]))
    np.testing.assert_allclose(out, v, rtol=0, atol=1e-12)


def test_one_hot_keys_overwrite_one_row():
    # alpha = 1, beta = 1 and one-hot keys e_c: the write replaces row c of S by
    # v_t^T and leaves the other rows alone (a plain key -> value table).
    rng = np.random.default_rng(6)
    T, H, dk, dv = 50, 1, 5, 3
    rows = rng.integers(0, dk, T)
    k = np.zeros((T, H, dk))
    k[np.arange(T), 0, rows] = 1.0
    v = rng.standard_normal((T, H, dv))
    S0 = rng.standard_normal((1, H, dk, dv))
    _, fin = O.kda_recurrence(k, k, v, np.zeros((T, H, dk)), np.ones((T, H)), S0, _cu([T]))
    table = {c: S0[0, 0, c].copy() for c in range(dk)}
    for t in range(T):
        table[int(rows[t])] = v[t, 0]
    for c in range(dk):
        np.testing.assert_allclose(fin[0, 0, c], table[c], rtol=0, atol=1e-14)


def test_write_strength_shrinks_the_residual():
    # With alpha = 1 the update is one gradient step of size beta on
    # 1/2 ||S^T k - v||^2, so the residual at k_t is multiplied by (1 - beta |k|^2).
    T, H, dk, dv = 30, 2, 9, 4
    q, k, v, _, b = _rand(7, T, H, dk, dv, unit_k=False)
    S0 = np.random.default_rng(8).standard_normal((1, H, dk, dv))
    _, _, states = O.kda_recurrence(q, k, v, np.zeros((T, H, dk)), b, S0, _cu([T]), return_states=True)
    prev = S0[0]
    for t in range(T):
        for h in range(H):
            before = prev[h].T @ k[t, h] - v[t, h]
            after = states[t, h].T @ k[t, h] - v[t, h]
            np.testing.assert_allclose(after, (1 - b[t, h] * k[t, h] @ k[t, h]) * before, rtol=1e-11, atol=1e-11)
        prev = states[t]


def test_orthonormal_keys_make_an_exact_associative_memory():
    rng = np.random.default_rng(9)
    d, dv = 12, 5
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    k = Qm.T[:, None, :]                      # d orthonormal keys, one head
    v = rng.standard_normal((d, 1, dv))
    _, fin = O.kda_recurrence(k, k, v, np.zeros((d, 1, d)), np.ones((d, 1)), None, _cu([d]))
    np.testing.assert_allclose(fin[0, 0], Qm @ v[:, 0, :], atol=1e-12)
    np.testing.assert_allclose(fin[0, 0].T @ Qm, v[:, 0, :].T, atol=1e-12)


# --- the gated decay acts per key channel, on the rows of S ---------------------

def test_pure_decay_closed_form_per_key_channel():
    T, H, dk, dv = 25, 2, 6, 3                  # dk != dv catches decay on the wrong side
    q, k, v, la, _ = _rand(10, T, H, dk, dv, decay_scale=0.3)
    S0 = np.random.default_rng(11).standard_normal((1, H, dk, dv))
    out, fin = O.kda_recurrence(q, k, v, la, np.zeros((T, H)), S0, _cu([T]))
    cum = np.cumsum(la, axis=0)
    for t in range(T):
        for h in range(H):
            St = np.diag(np.exp(cum[t, h])) @ S0[0, h]
            np.testing.assert_allclose(out[t, h], St.T @ q[t, h], rtol=1e-12, atol=1e-14)
    for h in range(H):
        np.testing.assert_allclose(fin[0, h], np.diag(np.exp(cum[-1, h])) @ S0[0, h], rtol=1e-12)


def test_matrix_product_form_on_tiny_inputs():
    # S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T, built from explicit
    # matrices, against the oracle's residual form.
    T, H, dk, dv = 12, 1, 4, 3
    q, k, v, la, b = _rand(12, T, H, dk, dv, unit_k=False, decay_scale=0.5)
    S0 = np.random.default_rng(13).standard_normal((1, H, dk, dv))
    out, fin = O.kda_recurrence(q, k, v, la, b, S0, _cu([T]))
    S = S0[0, 0]
    for t in range(T):
        kt = k[t, 0][:, None]
        S = (np.eye(dk) - b[t, 0] * kt @ kt.T) @ np.diag(np.exp(la[t, 0])) @ S + b[t, 0] * kt @ v[t, 0][None, :]
        np.testing.assert_allclose(out[t, 0], S.T @ q[t, 0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(fin[0, 0], S, rtol=1e-12, atol=1e-13)


def test_state_norm_bound():
    # ||(I - beta k k^T) Diag(alpha)||_2 <= 1 for unit k, beta in [0,1], alpha <= 1,
    # hence ||S_t||_F <= ||S_{t-1}||_F + beta_t ||v_t||.
    T, H, dk, dv = 60, 3, 10, 6
    q, k, v, la, b = _rand(14, T, H, dk, dv)
    S0 = np.random.default_rng(15).standard_normal((1, H, dk, dv))
    _, _, states = O.kda_recurrence(q, k, v, la, b, S0, _cu([T]), return_states=True)
    prev = S0[0]
    for t in range(T):
        for h in range(H):
            lhs = np.linalg.norm(states[t, h])
            rhs = np.linalg.norm(prev[h]) + b[t, h] * np.linalg.norm(v[t, h])
            assert lhs <= rhs * (1 + 1e-12)
        prev = states[t]


# --- chunked rewrite, splitting and packing ----------------------------------------

@pytest.mark.parametrize("chunk", [1, 4, 16, 64])
def test_chunked_rewrite_equals_recurrence(chunk):
    lens = [100, 1, 64, 37]
    T = sum(lens)
    H, dk, dv = 2, 16, 12
    q, k, v, la, b = _rand(16, T, H, dk, dv, decay_scale=0.4)
    S0 = np.random.default_rng(17).standard_normal((len(lens), H, dk, dv)) * 0.3
    o1, f1 = O.kda_recurrence(q, k, v, la, b, S0, _cu(lens))
    o2, f2 = O.kda_chunked(q, k, v, la, b, S0, _cu(lens), chunk=chunk)
    scale = np.abs(o1).max()
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-11 * scale)
    np.testing.assert_allclose(f2, f1, rtol=0, atol=1e-11 * np.abs(f1).max())


def test_chunked_rewrite_strong_decay():
    # large per-token decay: the pairwise factors are evaluated exactly, so the
    # rewrite still matches where a factorised exp(g) * exp(-g) would overflow
    T, H, dk, dv = 70, 1, 8, 4
    q, k, v, la, b = _rand(18, T, H, dk, dv, decay_scale=8.0)
    o1, f1 = O.kda_recurrence(q, k, v, la, b, None, _cu([T]))
    o2, f2 = O.kda_chunked(q, k, v, la, b, None, _cu([T]), chunk=64)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-11 * np.abs(o1).max())


def test_split_invariance():
    T, T1, H, dk, dv = 90, 33, 2, 8, 8
    q, k, v, la, b = _rand(19, T, H, dk, dv)
    S0 = np.random.default_rng(20).standard_normal((1, H, dk, dv))
    o, f = O.kda_recurrence(q, k, v, la, b, S0, _cu([T]))
    oa, fa = O.kda_recurrence(q[:T1], k[:T1], v[:T1], la[:T1], b[:T1], S0, _cu([T1]))
    ob, fb = O.kda_recurrence(q[T1:], k[T1:], v[T1:], la[T1:], b[T1:], fa, _cu([T - T1]))
    np.testing.assert_allclose(np.concatenate([oa, ob]), o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(fb, f, rtol=1e-13, atol=1e-14)


def test_packed_equals_per_sequence_and_fixed_length():
    lens = [7, 20, 1]
    H, dk, dv = 2, 4, 3
    q, k, v, la, b = _rand(21, sum(lens), H, dk, dv)
    S0 = np.random.default_rng(22).standard_normal((3, H, dk, dv))
    o, f = O.kda_recurrence(q, k, v, la, b, S0, _cu(lens))
    cu = _cu(lens)
    for n in range(3):
        s, e = cu[n], cu[n + 1]
        on, fn = O.kda_recurrence(q[s:e], k[s:e], v[s:e], la[s:e], b[s:e], S0[n:n + 1], _cu([e - s]))
        np.testing.assert_array_equal(on, o[s:e])
        np.testing.assert_array_equal(fn[0], f[n])
    # fixed-length [B, T, ...] is the packed layout with equal lengths
    qb, kb, vb, lab, bb = _rand(23, 2 * 9, H, dk, dv)
    of, ff = O.kda_recurrence(qb.reshape(2, 9, H, dk), kb.reshape(2, 9, H, dk), vb.reshape(2, 9, H, dv),
                              lab.reshape(2, 9, H, dk), bb.reshape(2, 9, H), None, None)
    op, fp = O.kda_recurrence(qb, kb, vb, lab, bb, None, _cu([9, 9]))
    np.testing.assert_array_equal(of.reshape(18, H, dv), op)
    np.testing.assert_array_equal(ff, fp)


def test_empty_sequence_keeps_initial_state():
    H, dk, dv = 2, 4, 3
    q, k, v, la, b = _rand(24, 5, H, dk, dv)
    S0 = np.random.default_rng(25).standard_normal((3, H, dk, dv))
    o, f = O.kda_recurrence(q, k, v, la, b, S0, _cu([2, 0, 3]))
    np.testing.assert_array_equal(f[1], S0[1])
    o2, f2 = O.kda_chunked(q, k, v, la, b, S0, _cu([2, 0, 3]), chunk=4)
    np.testing.assert_array_equal(f2[1], S0[1])


def test_decode_steps_equal_the_token_recurrence():
    steps, N, H, dk, dv = 9, 3, 2, 6, 5
    rng = np.random.default_rng(26)
    q, k, v, la, b = _rand(27, steps * N, H, dk, dv)
    q, k, v, la = (x.reshape(steps, N, H, -1) for x in (q, k, v, la))
    b = b.reshape(steps, N, H)
    S0 = rng.standard_normal((N, H, dk, dv))
    outs, fin = O.kda_decode_steps(q, k, v, la, b, S0)
    # the same tokens as N sequences of length `steps`
    perm = lambda x: x.transpose(1, 0, *range(2, x.ndim)).reshape(N * steps, *x.shape[2:])
    o2, f2 = O.kda_recurrence(perm(q), perm(k), perm(v), perm(la), perm(b), S0, _cu([steps] * N))
    np.testing.assert_allclose(perm(outs), o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(fin, f2, rtol=1e-13, atol=1e-14)
    sub, fsub = O.kda_decode_steps(q, k, v, la, b, S0, seq_subset=np.array([2, 0]))
    np.testing.assert_array_equal(sub, outs[:, [2, 0]])


# --- pre/post stage -------------------------------------------------------------

def test_short_conv_matches_causal_library_convolution():
    rng = np.random.default_rng(28)
    lens = [10, 3, 6]
    C = 5
    x = rng.standard_normal((sum(lens), C))
    w = rng.standard_normal((C, 4))
    y = O.short_conv(x, w, _cu(lens))
    cu = _cu(lens)
    for n in range(len(lens)):
        s, e = cu[n], cu[n + 1]
        for c in range(C):
            # np.convolve flips its kernel: taps reversed puts w[c,3] on the current token
            ref = np.convolve(x[s:e, c], w[c, ::-1])[: e - s]
            np.testing.assert_allclose(y[s:e, c], ref, rtol=1e-13, atol=1e-14)


def test_short_conv_impulse_response_and_sequence_start():
    w = np.array([[1.0, 2.0, 3.0, 4.0]])
    x = np.zeros((8, 1))
    x[2, 0] = 1.0
    y = O.short_conv(x, w, _cu([8]))
    np.testing.assert_array_equal(y[:, 0], [0, 0, 4, 3, 2, 1, 0, 0])
    # a second sequence starting at token 4 does not see the first one's history
    y2 = O.short_conv(x, w, _cu([4, 4]))
    np.testing.assert_array_equal(y2[:, 0], [0, 0, 4, 3, 0, 0, 0, 0])


def test_l2norm_and_gate():
    rng = np.random.default_rng(29)
    x = rng.standard_normal((6, 3, 16)) * 5
    n = O.l2norm(x)
    np.testing.assert_allclose(np.linalg.norm(n, axis=-1), 1.0, rtol=1e-6)
    np.testing.assert_allclose(n / np.linalg.norm(n, axis=-1, keepdims=True), x / np.linalg.norm(x, axis=-1, keepdims=True), rtol=1e-13)
    assert np.all(O.l2norm(np.zeros((2, 4))) == 0)
    o = rng.standard_normal((4, 2, 3))
    np.testing.assert_allclose(O.output_gate(o, np.zeros_like(o)), o / 2, rtol=1e-15)
    np.testing.assert_allclose(O.output_gate(o, np.full_like(o, 60.0)), o, rtol=1e-15)
    assert np.all(np.abs(O.output_gate(o, np.full_like(o, -800.0))) < 1e-300)


def test_mixer_with_identity_conv_and_open_gate_is_the_recurrence():
    lens = [9, 14]
    H, d = 2, 8
    q, k, v, la, b = _rand(30, sum(lens), H, d, d, unit_k=False)
    w = np.zeros((3, H * d, 4))
    w[:, :, 3] = 1.0                          # pass the current token through
    out, fin = O.kda_mixer(q, k, v, w, la, b, np.full((sum(lens), H, d), 60.0), _cu(lens))
    ref, rfin = O.kda_recurrence(O.l2norm(q), O.l2norm(k), v, la, b, None, _cu(lens))
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(fin, rfin, rtol=1e-13, atol=1e-14)


# --- the pages' printed cost-model figures pin the state's shape --------------------

def test_cost_model_figures_pin_state_shape():
    g = json.load(open(os.path.join(HERE, "golden", "cost_model.json")))
    f = g["fields"]
    mla_bytes_per_token = f["mla_layers"] * (f["kv_lora_rank"] + f["qk_rope_head_dim"]) * 2
    assert round(mla_bytes_per_token / 1024, 2) == g["kv_cache_per_token_bf16_kib"]
    # per KDA layer: one d_k x d_v state per head, plus the conv history (kernel - 1
    # tokens) of q, k and v channels, all BF16
    state = f["linear_k_heads"] * f["linear_k_head_dim"] * f["linear_v_head_dim"] * 2
    conv = (f["short_conv_kernel"] - 1) * f["linear_k_heads"] * (2 * f["linear_k_head_dim"] + f["linear_v_head_dim"]) * 2
    total = mla_bytes_per_token * g["context_tokens"] + f["kda_layers"] * (state + conv)
    assert round(total / 2**30, 2) == g["kv_cache_plus_state_at_256k_bf16_gib"]
    # a state of another shape (e.g. d_k x d_k/2, or 16 heads) misses the printed figure
    for wrong in (state // 2, state * 2):
        t2 = mla_bytes_per_token * g["context_tokens"] + f["kda_layers"] * (wrong + conv)
        assert round(t2 / 2**30, 2) != g["kv_cache_plus_state_at_256k_bf16_gib"]


def test_mixer_decode_steps_reproduce_the_mixer_prefill():
    """Decoding a sequence token by token from an empty conv history and a zero state,
    with the serving decode step, gives the prefill mixer's outputs and final state
    (the two take their convolution windows from different code: packed sequences
    with zero history at each start, against a rolling three-row history)."""
    rng = np.random.default_rng(137101)
    N, T, H, d = 3, 9, 2, 8
    q = rng.standard_normal((N, T, H, d))
    k = rng.standard_normal((N, T, H, d))
    v = rng.standard_normal((N, T, H, d))
    la = -np.log1p(np.exp(rng.standard_normal((N, T, H, d)))) / 4
    b = 1 / (1 + np.exp(-rng.standard_normal((N, T, H))))
    g = rng.standard_normal((N, T, H, d))
    w = rng.standard_normal((3, H * d, 4)) * 0.5
    s0 = rng.standard_normal((N, H, d, d)) * 0.1
    packed = lambda x: x.reshape(N * T, *x.shape[2:])
    cu = np.arange(N + 1) * T
    ref_o, ref_s = O.kda_mixer(packed(q), packed(k), packed(v), w, packed(la), packed(b), packed(g), cu, s0)
    S, hist = s0.copy(), np.zeros((N, H, 3, 3, d))
    outs = []
    for t in range(T):
        o, S, hist = O.kda_mixer_decode_step(q[:, t], k[:, t], v[:, t], w, la[:, t], b[:, t], g[:, t], S, hist)
        outs.append(o)
    np.testing.assert_allclose(np.stack(outs, axis=1).reshape(N * T, H, d), ref_o, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S, ref_s, rtol=1e-11, atol=1e-12)
    # the history holds the last three raw rows, oldest first
    np.testing.assert_array_equal(hist[:, :, 0], q[:, T - 3:].transpose(0, 2, 1, 3))
    np.testing.assert_array_equal(hist[:, :, 2], v[:, T - 3:].transpose(0, 2, 1, 3))


def test_mixer_decode_step_with_history_matches_a_longer_prefill():
    """After a prefill of T tokens, one decode step fed the prefill's last three raw rows
    as its history equals the prefill of T + 1 tokens at the last token."""
    rng = np.random.default_rng(137102)
    T, H, d = 6, 2, 8
    mk = lambda *s: rng.standard_normal(s)
    q, k, v, g = mk(T + 1, H, d), mk(T + 1, H, d), mk(T + 1, H, d), mk(T + 1, H, d)
    la = -np.log1p(np.exp(mk(T + 1, H, d))) / 4
    b = 1 / (1 + np.exp(-mk(T + 1, H)))
    w = mk(3, H * d, 4) * 0.5
    o_long, s_long = O.kda_mixer(q, k, v, w, la, b, g, np.array([0, T + 1]))
    _, s_T = O.kda_mixer(q[:T], k[:T], v[:T], w, la[:T], b[:T], g[:T], np.array([0, T]))
    hist = np.stack([x[T - 3:T].transpose(1, 0, 2) for x in (q, k, v)], axis=1)[None]  # [1, H, 3, 3, d]
    o, S, _ = O.kda_mixer_decode_step(q[T:], k[T:], v[T:], w, la[T:], b[T:], g[T:], s_T, hist)
    np.testing.assert_allclose(o[0], o_long[T], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S[0], s_long[0], rtol=1e-11, atol=1e-12)


def test_mixer_decode_tokens_checkpoints_equal_shorter_runs():
    """K tokens at once: the outputs are the single-step outputs, and checkpoint a-1 is
    the state and history after decoding only the first a tokens (what a speculative
    decoder rolls back to); the last checkpoint is the state after all K."""
    rng = np.random.default_rng(137103)
    N, K, H, d = 2, 4, 2, 8
    mk = lambda *s: rng.standard_normal(s)
    q, k, v, g = mk(N, K, H, d), mk(N, K, H, d), mk(N, K, H, d), mk(N, K, H, d)
    la = -np.log1p(np.exp(mk(N, K, H, d))) / 4
    b = 1 / (1 + np.exp(-mk(N, K, H)))
    w = mk(3, H * d, 4) * 0.5
    s0, h0 = mk(N, H, d, d) * 0.1, mk(N, H, 3, 3, d)
    out, states, hists = O.kda_mixer_decode_tokens(q, k, v, w, la, b, g, s0, h0)
    for a in range(1, K + 1):
        S, hist = s0, h0
        for j in range(a):
            o, S, hist = O.kda_mixer_decode_step(q[:, j], k[:, j], v[:, j], w, la[:, j], b[:, j], g[:, j], S, hist)
            np.testing.assert_allclose(out[:, j], o, rtol=0, atol=0)
        np.testing.assert_allclose(states[:, a - 1], S, rtol=0, atol=0)
        np.testing.assert_allclose(hists[:, a - 1], hist, rtol=0, atol=0)


def test_final_state_is_affine_in_the_initial_state():
    """S_end(S0) = M S0 + B with M the run from the identity with zero values and B the
    run from zero: the fact a context-parallel prefill builds on (checked on random S0)."""
    rng = np.random.default_rng(137104)
    T, H, d = 40, 2, 8
    q, k, v = (rng.standard_normal((T, H, d)) for _ in range(3))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    la = -np.log1p(np.exp(rng.standard_normal((T, H, d)))) / 8
    b = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    cu = np.array([0, T])
    eye = np.broadcast_to(np.eye(d), (1, H, d, d)).copy()
    _, M = O.kda_recurrence(q, k, np.zeros_like(v), la, b, eye, cu)
    _, B = O.kda_recurrence(q, k, v, la, b, None, cu)
    S0 = rng.standard_normal((1, H, d, d))
    _, S = O.kda_recurrence(q, k, v, la, b, S0, cu)
    np.testing.assert_allclose(S, M @ S0 + B, rtol=1e-11, atol=1e-12)


def test_softplus_gate_closed_forms():
    # softplus(0) = ln 2; large x -> x; very negative x -> e^x; -softplus <= 0 always
    assert O.softplus(0.0) == pytest.approx(np.log(2.0), rel=1e-15)
    assert O.softplus(50.0) == pytest.approx(50.0, rel=1e-15)
    assert O.softplus(-40.0) == pytest.approx(np.exp(-40.0), rel=1e-12)
    x = np.linspace(-30, 30, 601)
    np.testing.assert_allclose(O.softplus(x), np.log1p(np.exp(x)), rtol=1e-12)
    a = np.random.default_rng(137105).standard_normal((5, 3, 4))
    s = np.array([0.5, 1.0, 2.0])
    la = O.gate_log_alpha(a, s)
    assert np.all(la < 0)
    np.testing.assert_allclose(la[:, 1], -np.log1p(np.exp(a[:, 1])), rtol=1e-12)   # scale 1
    np.testing.assert_allclose(la[:, 2], -2 * np.log1p(np.exp(a[:, 2])), rtol=1e-12)  # linear in the scale


def test_backward_matches_finite_differences():
    """Every gradient of kda_backward against central differences of kda_recurrence
    (tiny packed problem with two sequences, a loss mixing all outputs and the final
    states with fixed random weights)."""
    rng = np.random.default_rng(137106)
    lens, H, d = [4, 3], 2, 3
    TT = sum(lens)
    cu = np.array([0, 4, 7])
    q, k, v = (rng.standard_normal((TT, H, d)) for _ in range(3))
    la = -np.log1p(np.exp(rng.standard_normal((TT, H, d))))
    b = 1 / (1 + np.exp(-rng.standard_normal((TT, H))))
    s0 = rng.standard_normal((2, H, d, d)) * 0.3
    wo, wf = rng.standard_normal((TT, H, d)), rng.standard_normal((2, H, d, d))

    def loss(q_, k_, v_, la_, b_, s0_):
        o, f = O.kda_recurrence(q_, k_, v_, la_, b_, s0_, cu)
        return np.sum(wo * o) + np.sum(wf * f)

    grads = O.kda_backward(q, k, v, la, b, s0, cu, wo, wf)
    args = [q, k, v, la, b, s0]
    eps = 1e-6
    for which, (x, g) in enumerate(zip(args, grads)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            xp, xm = [a.copy() for a in args], [a.copy() for a in args]
            xp[which][i] += eps
            xm[which][i] -= eps
            num[i] = (loss(*xp) - loss(*xm)) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-7, err_msg=f"gradient {which}")


def test_backward_closed_form_without_writes():
    """With beta = 0 and alpha = 1 nothing is written: S_t = S0 for every token, so
    o_t = S0^T q_t and, with G_t = d_final + sum_{s >= t} q_s do_s^T (the gradient of the
    state after token t), the gradients have closed forms: dq_t = S0 do_t, dk = dv = 0,
    dS0 = G_first, dbeta_t = (G_t^T k_t) . (v_t - S0^T k_t), dlog_alpha_t,i =
    sum_j (G_t)_ij (S0)_ij."""
    rng = np.random.default_rng(137107)
    T, H, dk, dv = 6, 2, 4, 3
    q, k = rng.standard_normal((T, H, dk)), rng.standard_normal((T, H, dk))
    v = rng.standard_normal((T, H, dv))
    do = rng.standard_normal((T, H, dv))
    s0 = rng.standard_normal((1, H, dk, dv))
    df = rng.standard_normal((1, H, dk, dv))
    la, b = np.zeros((T, H, dk)), np.zeros((T, H))
    dq, dkk, dvv, dla, db, ds0 = O.kda_backward(q, k, v, la, b, s0, [0, T], do, df)
    S = s0[0]
    for h in range(H):
        G = df[0, h].copy()
        for t in range(T - 1, -1, -1):
            G = G + np.outer(q[t, h], do[t, h])
            np.testing.assert_allclose(dq[t, h], S[h] @ do[t, h], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(db[t, h], (G.T @ k[t, h]) @ (v[t, h] - S[h].T @ k[t, h]), rtol=1e-12,
                                       atol=1e-12)
            np.testing.assert_allclose(dla[t, h], np.sum(G * S[h], axis=1), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(ds0[0, h], G, rtol=1e-12, atol=1e-12)
    assert np.all(dkk == 0) and np.all(dvv == 0)


@pytest.mark.parametrize("factorized", [False, True])
@pytest.mark.parametrize("lens,chunk", [([9, 4, 0, 13], 4), ([70, 5, 64], 64)])
def test_chunked_backward_matches_the_token_backward(lens, chunk, factorized):
    """kda_chunked_backward (the chunk-parallel form: GEMMs, a triangular inverse and a
    reverse running sum per chunk; pairwise or factorized decay) against kda_backward
    (one token at a time): partial and full chunks, an empty sequence, initial states
    and a final-state gradient."""
    rng = np.random.default_rng(137108 + chunk)
    H, dk, dv = 2, 5, 3
    TT = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k = rng.standard_normal((TT, H, dk)), rng.standard_normal((TT, H, dk))
    v = rng.standard_normal((TT, H, dv))
    la = -np.log1p(np.exp(rng.standard_normal((TT, H, dk)))) / 4
    b = 1 / (1 + np.exp(-rng.standard_normal((TT, H))))
    s0 = rng.standard_normal((len(lens), H, dk, dv)) * 0.3
    do = rng.standard_normal((TT, H, dv))
    df = rng.standard_normal((len(lens), H, dk, dv))
    ref = O.kda_backward(q, k, v, la, b, s0, cu, do, df)
    got = O.kda_chunked_backward(q, k, v, la, b, s0, cu, do, df, chunk=chunk, factorized=factorized)
    for name, r, g in zip(("dq", "dk", "dv", "dla", "dbeta", "dS0"), ref, got):
        np.testing.assert_allclose(g, r, rtol=0, atol=1e-10 * np.max(np.abs(r)), err_msg=name)
