"""fp64 CPU oracle for the Kimi Delta Attention (KDA) token mixer.

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's CPU
baseline may import this module; the library never does. It shares no code with
the CUDA path (the seeded input generators are the only common module, and they
hold none of the mixer's arithmetic).

What it computes (all in float64, from the exact input values upcast):

* ``kda_recurrence`` — the token-by-token definition. The pages' KDA section
  ("KDA: constant-size memory over a very long context", Ling-3.0-flash article,
  ai.thesatyajit.com) describes a fixed d_k x d_v state per head that each token
  first decays per key channel (the gated decay alpha_t, "the erase") and then
  writes with the delta rule (the write beta_t k_t v_t^T), read by the query. The
  displayed equation is missing from the extracted page; the reading used is

      S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
      o_t = S_t^T q_t,   alpha_t = exp(log_alpha_t) per key channel,

  i.e. decay acts on the key (row) side and the read happens after the write.
* ``kda_chunked`` — the chunk-parallel rewrite of the same recurrence (WY/UT
  form), written in its plainest matrix form per chunk with the pairwise decay
  factors exp(g_r - g_i) evaluated exactly (no factorisation). It is a
  self-check of the algebra a chunked kernel follows; it must equal
  ``kda_recurrence`` to rounding.
* ``short_conv``, ``l2norm``, ``output_gate`` and ``kda_mixer`` — the fused
  pre/post stage drawn in the article's KDA panel: a short causal depthwise
  convolution (kernel 4, from the model's config field short_conv_kernel_size on
  the llm-architectures-explained page, "Every architecture field") on q, k, v,
  an L2 norm of q and k, and a final sigmoid output gate.
* ``kda_decode_step`` — one token of the recurrence for a batch of sequences,
  updating the state in place (the constant-size state is what makes decode
  cost independent of context length, same article section).
* ``kda_mixer_decode_step`` — one serving decode token of the full mixer: the
  same conv4 / L2 norm / recurrence / gate steps as ``kda_mixer`` applied to one
  new token, with the convolution's last three raw inputs kept per sequence (a
  conv history) instead of the whole sequence.
* ``kda_backward`` — the gradients of ``kda_recurrence`` (of q, k, v, log_alpha,
  beta and the initial state, given the gradients of the outputs and of the final
  state): the chain rule through each token step, taken in reverse order.
* ``gate_log_alpha`` — the decay gate made from its pre-activation, read from
  the article's "softplus" gate as log alpha = -scale_h * softplus(a) per channel
  with one positive scale per head (the pages name the softplus, not its
  parameters).
* ``kda_mixer_decode_tokens`` — K consecutive tokens per sequence through
  ``kda_mixer_decode_step``, keeping the state and history after every token (the
  checkpoints a speculative decoder rolls back to when it accepts fewer tokens).
* ``kda_chunked_backward`` — the same gradients as ``kda_backward`` through the
  chunk-parallel rewrite of ``kda_chunked`` (each chunk's forward reversed step by
  step); a self-check of the algebra a chunked backward kernel would follow, equal
  to ``kda_backward`` to rounding.

Each function is pinned by tests that do not restate it: closed forms, special
cases that reduce to a textbook computation, finite differences, and the agreement
of two independent formulations (token and chunk).

Readings where the pages are silent (the full list is kept with the design
notes): no 1/sqrt(d_k) query scale; log_alpha is given directly (natural log,
<= 0); beta is given in (0, 1); conv tap w[c, 3] multiplies the current token,
zero history at every sequence start, no bias, identity activation; L2 norm is
x / sqrt(sum x^2 + 1e-6); the gate is out * sigmoid(g) with no norm before it.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np
from scipy.special import expit

L2NORM_EPS = 1e-6
CONV_WIDTH = 4


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _packed(q, k, v, log_alpha, beta, cu_seqlens):
    """Accept [B, T, H, d] (fixed length) or [sum_T, H, d] (packed with cu_seqlens)."""
    q, k, v, la, b = _f64(q), _f64(k), _f64(v), _f64(log_alpha), _f64(beta)
    if cu_seqlens is None:
        if q.ndim != 4:
            raise ValueError("fixed-length inputs must be [B, T, H, d]")
        B, T = q.shape[:2]
        cu = np.arange(B + 1, dtype=np.int64) * T
        return (q.reshape(B * T, *q.shape[2:]), k.reshape(B * T, *k.shape[2:]),
                v.reshape(B * T, *v.shape[2:]), la.reshape(B * T, *la.shape[2:]),
                b.reshape(B * T, *b.shape[2:]), cu, (B, T))
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    return q, k, v, la, b, cu, None


def token_step(S: np.ndarray, q_t, k_t, v_t, la_t, beta_t) -> Tuple[np.ndarray, np.ndarray]:
    """One token for every head at once. S [H, dk, dv] -> (S_t, o_t [H, dv]).

    Decay the key rows (Diag(alpha) S), form the delta-rule residual of the
    decayed state at k_t, write beta * k_t (residual)^T, read with q_t.
    """
    S = np.exp(la_t)[:, :, None] * S                       # Diag(alpha_t) S_{t-1}
    pred = np.einsum("hk,hkv->hv", k_t, S)                 # (Diag(alpha) S)^T k_t
    u = beta_t[:, None] * (v_t - pred)                     # beta_t (v_t - prediction)
    S = S + k_t[:, :, None] * u[:, None, :]                # + k_t u^T
    o = np.einsum("hk,hkv->hv", q_t, S)                    # o_t = S_t^T q_t
    return S, o


def kda_recurrence(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None,
                   return_states: bool = False):
    """Token-by-token KDA over packed sequences.

    q, k, log_alpha: [sum_T, H, dk]; v: [sum_T, H, dv]; beta: [sum_T, H];
    initial_state: [N, H, dk, dv] or None (zeros); cu_seqlens: [N+1] or None
    with [B, T, H, d] inputs. Returns (out [like v], final_state [N, H, dk, dv]),
    plus the per-token states [sum_T, H, dk, dv] if ``return_states``.
    """
    q, k, v, la, b, cu, fixed = _packed(q, k, v, log_alpha, beta, cu_seqlens)
    N = len(cu) - 1
    H, dk = k.shape[1], k.shape[2]
    dv = v.shape[2]
    out = np.zeros((q.shape[0], H, dv))
    final = np.zeros((N, H, dk, dv))
    states = np.zeros((q.shape[0], H, dk, dv)) if return_states else None
    for n in range(N):
        S = np.zeros((H, dk, dv)) if initial_state is None else _f64(initial_state[n]).copy()
        for t in range(cu[n], cu[n + 1]):
            S, out[t] = token_step(S, q[t], k[t], v[t], la[t], b[t])
            if return_states:
                states[t] = S
        final[n] = S
    if fixed is not None:
        out = out.reshape(fixed[0], fixed[1], H, dv)
    return (out, final, states) if return_states else (out, final)


def kda_chunked(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, chunk: int = 64):
    """The same result via the chunk-parallel (WY / UT) rewrite.

    Inside a chunk of L tokens that starts from state S0, with g_r the running
    sum of log_alpha up to and including token r (per key channel):
      A[r,i]  = beta_r * sum_c k[r,c] k[i,c] exp(g[r,c] - g[i,c])  for i < r
      T       = (I + A)^-1 Diag(beta)
      W       = T (K * exp(g)),  U~ = T V,  U = U~ - W S0
      P[r,i]  = sum_c q[r,c] k[i,c] exp(g[r,c] - g[i,c])          for i <= r
      O       = (Q * exp(g)) S0 + P U
      S_L     = Diag(exp(g_last)) S0 + (K * exp(g_last - g))^T U
    Chunks never cross a sequence boundary; the last chunk may be partial.
    """
    q, k, v, la, b, cu, fixed = _packed(q, k, v, log_alpha, beta, cu_seqlens)
    N = len(cu) - 1
    H, dk = k.shape[1], k.shape[2]
    dv = v.shape[2]
    out = np.zeros((q.shape[0], H, dv))
    final = np.zeros((N, H, dk, dv))
    for n in range(N):
        S = np.zeros((H, dk, dv)) if initial_state is None else _f64(initial_state[n]).copy()
        for s in range(cu[n], cu[n + 1], chunk):
            e = min(s + chunk, cu[n + 1])
            L = e - s
            Q = q[s:e].transpose(1, 0, 2)                  # [H, L, dk]
            K = k[s:e].transpose(1, 0, 2)
            V = v[s:e].transpose(1, 0, 2)                  # [H, L, dv]
            g = np.cumsum(la[s:e].transpose(1, 0, 2), axis=1)   # [H, L, dk]
            beta_c = b[s:e].T                               # [H, L]
            strict = np.tril(np.ones((L, L), dtype=bool), -1)
            incl = np.tril(np.ones((L, L), dtype=bool), 0)
            # pairwise decay exp(g_r - g_i), only where i <= r (never overflows)
            diff = g[:, :, None, :] - g[:, None, :, :]      # [H, r, i, dk]
            decay = np.where(incl[None, :, :, None], np.exp(np.where(incl[None, :, :, None], diff, 0.0)), 0.0)
            KK = np.einsum("hrc,hic,hric->hri", K, K, decay)
            QK = np.einsum("hrc,hic,hric->hri", Q, K, decay)
            A = beta_c[:, :, None] * np.where(strict, KK, 0.0)
            P = np.where(incl, QK, 0.0)
            eye = np.eye(L)
            Tm = np.linalg.solve(eye[None] + A, np.broadcast_to(eye, (H, L, L))) * beta_c[:, None, :]
            Gam = np.exp(g)
            W = Tm @ (K * Gam)
            Ut = Tm @ V
            U = Ut - W @ S
            O = (Q * Gam) @ S + P @ U
            g_last = g[:, -1, :]                            # [H, dk]
            Kdec = K * np.exp(g_last[:, None, :] - g)
            S = np.exp(g_last)[:, :, None] * S + Kdec.transpose(0, 2, 1) @ U
            out[s:e] = O.transpose(1, 0, 2)
        final[n] = S
    if fixed is not None:
        out = out.reshape(fixed[0], fixed[1], H, dv)
    return out, final


def kda_chunked_backward(q, k, v, log_alpha, beta, initial_state, cu_seqlens, d_out, d_final=None,
                         chunk: int = 64, factorized: bool = False):
    """The gradients of kda_backward, computed through the chunk-parallel rewrite of
    kda_chunked (a blueprint for a tensor-core backward: per chunk only GEMMs, a
    triangular inverse and elementwise work, and one state gradient carried between
    chunks). The forward of one chunk (per head, pairwise decay D[r,i,c] =
    exp(g[r,c] - g[i,c]) for i <= r) is
      KK = sum_c K[r,c] K[i,c] D,  QK = sum_c Q[r,c] K[i,c] D,
      A = Diag(beta) strict(KK),  P = incl(QK),  M = (I + A)^-1,  T = M Diag(beta),
      W = T (K e^g),  U~ = T V,  U = U~ - W S,  O = (Q e^g) S + P U,
      S' = Diag(e^g_last) S + Kdec^T U,  Kdec = K e^(g_last - g).
    Its reverse, given dO and dS' (the next chunk's dS, or d_final):
      dU = P^T dO + Kdec dS';  dS = (Q e^g)^T dO + Diag(e^g_last) dS' - W^T dU;
      dP = incl(dO U^T);  dW = -dU S^T;  dT = dW (K e^g)^T + dU V^T;
      d(K e^g) = T^T dW;  dV = T^T dU;  dM = dT Diag(beta);  dbeta_i += sum_r M[r,i] dT[r,i];
      dA = strict(-M^T dM M^T);  dbeta_r += sum_i dA[r,i] KK[r,i];  dKK = Diag(beta) dA;
    then through the products of K, Q, e^g and D to dK, dQ and dg, and
    dlog_alpha = the reverse running sum of dg within the chunk.

    With ``factorized`` the decay-weighted products are taken as a tensor-core kernel
    would take them, KK = Kt Kh^T and QK = Qt Kh^T with Kt = K e^g, Qt = Q e^g and
    Kh = K e^-g (finite while a chunk's summed decay stays moderate), and their reverse
    is dKt += dKK Kh, dQt += dP Kh, dKh = dKK^T Kt + dP^T Qt.
    """
    q, k, v, la, b = _f64(q), _f64(k), _f64(v), _f64(log_alpha), _f64(beta)
    do = _f64(d_out)
    TT, H, dk = q.shape
    dv = v.shape[2]
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    N = len(cu) - 1
    S0 = np.zeros((N, H, dk, dv)) if initial_state is None else _f64(initial_state)
    dq, dkk, dvv, dla, db = (np.zeros_like(x) for x in (q, k, v, la, b))
    dS0 = np.zeros_like(S0)
    for n in range(N):
        starts = list(range(cu[n], cu[n + 1], chunk))
        # forward: the state at the start of every chunk
        S_at, S = [], S0[n].copy()
        for s in starts:
            e = min(s + chunk, cu[n + 1])
            S_at.append(S)
            _, S = kda_chunked(q[s:e], k[s:e], v[s:e], la[s:e], b[s:e], S[None], [0, e - s], chunk=chunk)
            S = S[0]
        dS = np.zeros((H, dk, dv)) if d_final is None else _f64(d_final)[n].copy()
        for s, S in zip(reversed(starts), reversed(S_at)):
            e = min(s + chunk, cu[n + 1])
            L = e - s
            Q, K = q[s:e].transpose(1, 0, 2), k[s:e].transpose(1, 0, 2)     # [H, L, dk]
            V, dO = v[s:e].transpose(1, 0, 2), do[s:e].transpose(1, 0, 2)   # [H, L, dv]
            be = b[s:e].T                                                   # [H, L]
            g = np.cumsum(la[s:e].transpose(1, 0, 2), axis=1)              # [H, L, dk]
            strict = np.tril(np.ones((L, L), dtype=bool), -1)
            incl = np.tril(np.ones((L, L), dtype=bool), 0)
            diff = g[:, :, None, :] - g[:, None, :, :]
            D = np.where(incl[None, :, :, None], np.exp(np.where(incl[None, :, :, None], diff, 0.0)), 0.0)
            KK = np.einsum("hrc,hic,hric->hri", K, K, D)
            QK = np.einsum("hrc,hic,hric->hri", Q, K, D)
            A = be[:, :, None] * np.where(strict, KK, 0.0)
            P = np.where(incl, QK, 0.0)
            eye = np.eye(L)
            M = np.linalg.solve(eye[None] + A, np.broadcast_to(eye, (H, L, L)))
            T = M * be[:, None, :]
            Gam = np.exp(g)
            Kt, Qt = K * Gam, Q * Gam
            W, Ut = T @ Kt, T @ V
            U = Ut - W @ S
            gl = g[:, -1, :]                                                # [H, dk]
            gam = np.exp(gl)
            Ed = np.exp(gl[:, None, :] - g)                                 # [H, L, dk]
            Kdec = K * Ed
            Tt = lambda x: x.transpose(0, 2, 1)
            # reverse of O = Qt S + P U and S' = Diag(gam) S + Kdec^T U
            dU = Tt(P) @ dO + Kdec @ dS
            dS_prev = Tt(Qt) @ dO + gam[:, :, None] * dS - Tt(W) @ dU
            dP = np.where(incl, dO @ Tt(U), 0.0)
            dQt = dO @ Tt(S)
            dKdec = U @ Tt(dS)
            dgam = np.sum(dS * S, axis=2)                                   # [H, dk]
            # reverse of U = U~ - W S, W = T Kt, U~ = T V
            dW = -dU @ Tt(S)
            dT = dW @ Tt(Kt) + dU @ Tt(V)
            dKt = Tt(T) @ dW
            dV = Tt(T) @ dU
            # reverse of T = M Diag(beta), M = (I + A)^-1, A = Diag(beta) strict(KK)
            dM = dT * be[:, None, :]
            dbe = np.sum(M * dT, axis=1)                                    # over r: [H, i]
            dA = np.where(strict, -Tt(M) @ dM @ Tt(M), 0.0)
            dbe = dbe + np.sum(dA * KK, axis=2)                             # over i: [H, r]
            dKK = be[:, :, None] * dA
            if factorized:
                # reverse of KK = Kt Kh^T, QK = Qt Kh^T, then of Kt, Qt, Kh and Kdec
                Kh = K / Gam
                dKt = dKt + dKK @ Kh
                dQt = dQt + dP @ Kh
                dKh = Tt(dKK) @ Kt + Tt(dP) @ Qt
                dQ = dQt * Gam
                dK = dKt * Gam + dKh / Gam + dKdec * Ed
                dg = dQt * Qt + dKt * Kt - dKh * Kh - dKdec * Kdec
            else:
                # reverse of KK, QK (pairwise decay) and of the e^g, Kdec products
                dQ = dQt * Gam + np.einsum("hri,hic,hric->hrc", dP, K, D)
                dK = (dKt * Gam + dKdec * Ed + np.einsum("hri,hic,hric->hrc", dKK, K, D)
                      + np.einsum("hri,hrc,hric->hic", dKK, K, D) + np.einsum("hri,hrc,hric->hic", dP, Q, D))
                dD = dKK[:, :, :, None] * K[:, :, None, :] * K[:, None, :, :] + \
                    dP[:, :, :, None] * Q[:, :, None, :] * K[:, None, :, :]
                dDD = dD * D
                dg = dQt * Qt + dKt * Kt - dKdec * Kdec + np.sum(dDD, axis=2) - np.sum(dDD, axis=1)
            dg[:, -1, :] += np.sum(dKdec * Kdec, axis=1) + dgam * gam
            dla_c = np.cumsum(dg[:, ::-1, :], axis=1)[:, ::-1, :]          # reverse running sum
            dq[s:e], dkk[s:e], dvv[s:e] = dQ.transpose(1, 0, 2), dK.transpose(1, 0, 2), dV.transpose(1, 0, 2)
            dla[s:e], db[s:e] = dla_c.transpose(1, 0, 2), dbe.T
            dS = dS_prev
        dS0[n] = dS
    return dq, dkk, dvv, dla, db, dS0


def short_conv(x, w, cu_seqlens) -> np.ndarray:
    """Causal depthwise convolution of width 4 on packed [sum_T, C] channels.

    y[t, c] = sum_{j=0..3} w[c, j] * x[t - 3 + j, c], with x taken as zero
    before each sequence's first token; no bias, identity activation.
    """
    x, w = _f64(x), _f64(w)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    y = np.zeros_like(x)
    for n in range(len(cu) - 1):
        s, e = cu[n], cu[n + 1]
        for t in range(s, e):
            for j in range(CONV_WIDTH):
                src = t - (CONV_WIDTH - 1) + j
                if src >= s:
                    y[t] += w[:, j] * x[src]
    return y


def l2norm(x, eps: float = L2NORM_EPS) -> np.ndarray:
    """x / sqrt(sum(x^2) + eps) over the last axis."""
    x = _f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def output_gate(o, g) -> np.ndarray:
    """Final sigmoid output gate: o * sigmoid(g), elementwise."""
    return _f64(o) * expit(_f64(g))


def kda_mixer(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, cu_seqlens,
              initial_state=None):
    """Full mixer stage: conv4 on q, k, v -> L2 norm on q, k -> KDA -> sigmoid gate.

    q_raw, k_raw: [sum_T, H, dk]; v_raw: [sum_T, H, dv]; conv_w: [3, H*d, 4]
    (q, k, v weights); gate: [sum_T, H, dv] or None.
    """
    TT, H, dk = np.shape(q_raw)
    dv = np.shape(v_raw)[2]
    qc = short_conv(np.reshape(q_raw, (TT, H * dk)), conv_w[0], cu_seqlens).reshape(TT, H, dk)
    kc = short_conv(np.reshape(k_raw, (TT, H * dk)), conv_w[1], cu_seqlens).reshape(TT, H, dk)
    vc = short_conv(np.reshape(v_raw, (TT, H * dv)), conv_w[2], cu_seqlens).reshape(TT, H, dv)
    out, final = kda_recurrence(l2norm(qc), l2norm(kc), vc, log_alpha, beta, initial_state, cu_seqlens)
    if gate is not None:
        out = output_gate(out, gate)
    return out, final


def kda_decode_step(q, k, v, log_alpha, beta, state) -> Tuple[np.ndarray, np.ndarray]:
    """One decode token for N sequences: q, k, log_alpha [N, H, dk]; v [N, H, dv];
    beta [N, H]; state [N, H, dk, dv]. Returns (out [N, H, dv], new state)."""
    q, k, v, la, b, S = _f64(q), _f64(k), _f64(v), _f64(log_alpha), _f64(beta), _f64(state)
    out = np.zeros(v.shape)
    new = np.zeros(S.shape)
    for n in range(S.shape[0]):
        new[n], out[n] = token_step(S[n], q[n], k[n], v[n], la[n], b[n])
    return out, new


def kda_decode_steps(q, k, v, log_alpha, beta, state, seq_subset: Optional[np.ndarray] = None):
    """Consecutive decode steps: inputs carry a leading [steps] axis. Optionally only
    a subset of sequences (indices into N) is run. Returns (out [steps, n, H, dv], final)."""
    idx = np.arange(np.shape(state)[0]) if seq_subset is None else np.asarray(seq_subset)
    S = _f64(np.asarray(state)[idx])
    steps = np.shape(q)[0]
    outs = []
    for s in range(steps):
        o, S = kda_decode_step(np.asarray(q[s])[idx], np.asarray(k[s])[idx], np.asarray(v[s])[idx],
                               np.asarray(log_alpha[s])[idx], np.asarray(beta[s])[idx], S)
        outs.append(o)
    return np.stack(outs), S


def kda_mixer_decode_step(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, state, conv_hist):
    """One serving decode token of the full mixer for N sequences (d_k = d_v = d).

    q_raw, k_raw, v_raw [N, H, d]: this token's raw projections; conv_w [3, H*d, 4];
    log_alpha [N, H, d]; beta [N, H]; gate [N, H, d] or None; state [N, H, d, d];
    conv_hist [N, H, 3, 3, d]: for q, k, v (axis 2) the three previous raw rows of
    each sequence, oldest first (zeros before the sequence's first token).

    Steps, as ``kda_mixer`` takes them for one token: y[c] = sum_j w[c, j] x[t-3+j, c]
    over (history, current token); q, k <- l2norm(y); v <- y; the KDA token step
    (``kda_decode_step``); out * sigmoid(gate). The history then drops its oldest row
    and appends the current raw token.
    Returns (out [N, H, d], new state [N, H, d, d], new conv_hist).
    """
    hist = _f64(conv_hist)
    N, H, _, _, d = hist.shape
    w = _f64(conv_w).reshape(3, H, d, CONV_WIDTH)
    ys, new_hist = [], hist.copy()
    for i, x in enumerate((q_raw, k_raw, v_raw)):
        x = _f64(x)
        window = np.concatenate([hist[:, :, i], x[:, :, None, :]], axis=2)  # [N, H, 4, d], oldest first
        ys.append(np.einsum("nhjc,hcj->nhc", window, w[i]))
        new_hist[:, :, i] = window[:, :, 1:]
    out, new_state = kda_decode_step(l2norm(ys[0]), l2norm(ys[1]), ys[2], log_alpha, beta, state)
    if gate is not None:
        out = output_gate(out, gate)
    return out, new_state, new_hist


def kda_mixer_decode_tokens(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, state, conv_hist):
    """K consecutive decode tokens per sequence: q_raw, k_raw, v_raw, log_alpha, gate
    [N, K, H, d]; beta [N, K, H]; state [N, H, d, d]; conv_hist [N, H, 3, 3, d].
    Returns (out [N, K, H, d], states after each token [N, K, H, d, d], histories after
    each token [N, K, H, 3, 3, d]); the last entries are the final state and history."""
    K = np.shape(q_raw)[1]
    S, hist = _f64(state), _f64(conv_hist)
    outs, states, hists = [], [], []
    for j in range(K):
        o, S, hist = kda_mixer_decode_step(np.asarray(q_raw)[:, j], np.asarray(k_raw)[:, j], np.asarray(v_raw)[:, j],
                                           conv_w, np.asarray(log_alpha)[:, j], np.asarray(beta)[:, j],
                                           None if gate is None else np.asarray(gate)[:, j], S, hist)
        outs.append(o)
        states.append(S)
        hists.append(hist)
    return np.stack(outs, axis=1), np.stack(states, axis=1), np.stack(hists, axis=1)


def softplus(x) -> np.ndarray:
    """log(1 + e^x), evaluated without overflow."""
    return np.logaddexp(0.0, _f64(x))


def gate_log_alpha(a_pre, a_scale) -> np.ndarray:
    """log alpha [.., H, d] = -a_scale[h] * softplus(a_pre) (a_scale [H] > 0)."""
    return -_f64(a_scale)[:, None] * softplus(a_pre)


def kda_backward(q, k, v, log_alpha, beta, initial_state, cu_seqlens, d_out, d_final=None):
    """Gradients of kda_recurrence over packed sequences.

    One token step, written with P = Diag(alpha) S_prev, w = P^T k, u = beta (v - w):
        S = P + k u^T,  o = S^T q.
    Walking the tokens backwards with G the gradient of S (the final state's gradient,
    or zero, at the end of each sequence):
        G += q do^T;  dq = S do;  du = G^T k;  dv = beta du;  dbeta = du . (v - w);
        dw = -beta du;  dk = G u + P dw;  dP = G + k dw^T;
        dlog_alpha_i = sum_j dP_ij P_ij;  G <- Diag(alpha) dP  (the gradient of S_prev).
    Returns (dq, dk, dv, dlog_alpha, dbeta, d_initial_state), float64, shapes of the inputs.
    """
    q, k, v, la, b = _f64(q), _f64(k), _f64(v), _f64(log_alpha), _f64(beta)
    do = _f64(d_out)
    TT, H, dk = q.shape
    dv = v.shape[2]
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    N = len(cu) - 1
    S0 = np.zeros((N, H, dk, dv)) if initial_state is None else _f64(initial_state)
    dq, dkk, dvv, dla, db = (np.zeros_like(x) for x in (q, k, v, la, b))
    dS0 = np.zeros_like(S0)
    for n in range(N):
        s, e = cu[n], cu[n + 1]
        # forward, keeping every state
        states = [S0[n]]
        for t in range(s, e):
            S, _ = token_step(states[-1], q[t], k[t], v[t], la[t], b[t])
            states.append(S)
        G = np.zeros((H, dk, dv)) if d_final is None else _f64(d_final)[n].copy()
        for i, t in enumerate(range(e - 1, s - 1, -1)):
            S, Sp = states[len(states) - 1 - i], states[len(states) - 2 - i]
            alpha = np.exp(la[t])                              # [H, dk]
            P = alpha[:, :, None] * Sp                         # [H, dk, dv]
            w = np.einsum("hij,hi->hj", P, k[t])               # [H, dv]
            u = b[t][:, None] * (v[t] - w)
            G = G + np.einsum("hi,hj->hij", q[t], do[t])
            dq[t] = np.einsum("hij,hj->hi", S, do[t])
            du = np.einsum("hij,hi->hj", G, k[t])
            dvv[t] = b[t][:, None] * du
            db[t] = np.sum(du * (v[t] - w), axis=1)
            dw = -b[t][:, None] * du
            dkk[t] = np.einsum("hij,hj->hi", G, u) + np.einsum("hij,hj->hi", P, dw)
            dP = G + np.einsum("hi,hj->hij", k[t], dw)
            dla[t] = np.sum(dP * P, axis=2)
            G = alpha[:, :, None] * dP
        dS0[n] = G
    return dq, dkk, dvv, dla, db, dS0
