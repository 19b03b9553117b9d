"""Seeded synthetic inputs for the KDA token mixer (shared by tests, bench and smoke).

This module draws random numbers and rounds them to the storage dtypes; it holds
none of the mixer's arithmetic. Everything is NumPy on the host, so the values
the CPU oracle sees and the values uploaded to the GPU are the same bits.

Recipe (one NumPy ``default_rng(137000 + config_id)`` per workload; draws are
taken in the order written below):

* q, k ~ N(0, 1) per element, then L2-normalised per (token, head) over d_k
  (except the raw q/k of the full-mixer workload, which the fused pre-stage
  normalises), then rounded to the storage dtype (bf16 RNE, or fp32).
* v ~ N(0, 1), rounded to the storage dtype.
* log_alpha = -softplus(z) / 16, z ~ N(0, 1), one value per key channel, fp32.
  (The gate is "softplus phi" on the pages; /16 keeps a 64-token chunk's decay
  near 3 nats, the regime of a trained model.)
* beta = sigmoid(z), z ~ N(0, 1), one per (token, head), fp32.
* initial states ~ N(0, 0.02^2), fp32.
* full mixer only: depthwise conv weights ~ N(0, 0.5^2) fp32 [3, H*d, 4]
  (q, k, v), output-gate pre-activation g ~ N(0, 1) stored as bf16.
* varlen: 64 lengths ~ U{256..8192} packed through int32 cu_seqlens.

Shapes are token-major packed: q, k, log_alpha [sum_T, H, d_k]; v, g [sum_T, H, d_v];
beta [sum_T, H]; states [N, H, d_k, d_v]. Fixed-length B x T is the same memory
with sum_T = B*T.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

SEED_BASE = 137000


_BLOCK = 1 << 22  # elements per in-place block (keeps temporaries small)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns a float32 copy."""
    out = np.array(x, dtype=np.float32, copy=True)
    _bf16_round_inplace(out)
    return out


def _bf16_round_inplace(x: np.ndarray) -> None:
    flat = x.reshape(-1)
    u = flat.view(np.uint32)
    for s in range(0, flat.size, _BLOCK):
        b = u[s:s + _BLOCK]
        b += np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
        b &= np.uint32(0xFFFF0000)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Bit patterns (uint16) of values that are already bf16-exact float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _normal(rng, shape, scale: float = 1.0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    flat = out.reshape(-1)
    for s in range(0, flat.size, _BLOCK):
        rng.standard_normal(out=flat[s:s + _BLOCK], dtype=np.float32)
    if scale != 1.0:
        flat *= np.float32(scale)
    return out


def _unit_rows_inplace(x: np.ndarray) -> None:
    # input recipe: "q, k ~ N(0,1) then L2-normalised per head" (a distribution
    # choice for the synthetic data, not the library's own normalisation)
    rows = x.reshape(-1, x.shape[-1])
    step = max(1, _BLOCK // x.shape[-1])
    for s in range(0, rows.shape[0], step):
        b = rows[s:s + step]
        n = np.sqrt(np.einsum("ij,ij->i", b, b, dtype=np.float64))
        b /= n[:, None].astype(np.float32)


def _neg_softplus_over_16_inplace(x: np.ndarray) -> None:
    flat = x.reshape(-1)
    for s in range(0, flat.size, _BLOCK):
        b = flat[s:s + _BLOCK]
        np.logaddexp(np.float32(0.0), b, out=b)
        b *= np.float32(-1.0 / 16.0)


def _sigmoid_inplace(x: np.ndarray) -> None:
    flat = x.reshape(-1)
    for s in range(0, flat.size, _BLOCK):
        b = flat[s:s + _BLOCK]
        np.negative(b, out=b)
        np.exp(b, out=b)
        b += np.float32(1.0)
        np.reciprocal(b, out=b)


@dataclasses.dataclass
class Workload:
    name: str
    H: int
    dk: int
    dv: int
    seq_lens: list
    qkv_dtype: str                 # "bf16" or "f32"
    q: np.ndarray                  # float32 arrays holding dtype-exact values
    k: np.ndarray
    v: np.ndarray
    log_alpha: np.ndarray
    beta: np.ndarray
    initial_state: Optional[np.ndarray]
    cu_seqlens: np.ndarray         # int32 [N+1]
    conv_w: Optional[np.ndarray] = None   # [3, H*d, 4] fp32 (full mixer)
    gate: Optional[np.ndarray] = None     # [sum_T, H, dv] bf16-exact (full mixer)
    B: int = 0
    T: int = 0

    @property
    def N(self) -> int:
        return len(self.seq_lens)

    @property
    def total_T(self) -> int:
        return int(self.cu_seqlens[-1])


def make_prefill(seq_lens, H, dk, dv, *, seed=None, rng=None, qkv_dtype="bf16", state_std=0.02,
                 normalise_qk=True, mixer=False, name="prefill", B=0, T=0) -> Workload:
    """Draw one prefill workload. ``seq_lens`` lists the packed sequences."""
    if rng is None:
        rng = np.random.default_rng(seed)
    seq_lens = [int(s) for s in seq_lens]
    cu = np.zeros(len(seq_lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(seq_lens)
    TT = int(cu[-1])
    q = _normal(rng, (TT, H, dk))
    k = _normal(rng, (TT, H, dk))
    v = _normal(rng, (TT, H, dv))
    if normalise_qk:
        _unit_rows_inplace(q)
        _unit_rows_inplace(k)
    if qkv_dtype == "bf16":
        for x in (q, k, v):
            _bf16_round_inplace(x)
    la = _normal(rng, (TT, H, dk))
    _neg_softplus_over_16_inplace(la)
    beta = _normal(rng, (TT, H))
    _sigmoid_inplace(beta)
    s0 = _normal(rng, (len(seq_lens), H, dk, dv), state_std) if state_std else None
    conv_w = gate = None
    if mixer:
        conv_w = _normal(rng, (3, H * dk, 4), 0.5)
        gate = _normal(rng, (TT, H, dv))
        _bf16_round_inplace(gate)
    return Workload(name=name, H=H, dk=dk, dv=dv, seq_lens=seq_lens, qkv_dtype=qkv_dtype,
                    q=q, k=k, v=v, log_alpha=la, beta=beta, initial_state=s0, cu_seqlens=cu,
                    conv_w=conv_w, gate=gate, B=B, T=T)


@dataclasses.dataclass
class DecodeWorkload:
    name: str
    N: int
    H: int
    dk: int
    dv: int
    steps: int
    q: np.ndarray          # [steps, N, H, dk] bf16-exact float32
    k: np.ndarray
    v: np.ndarray          # [steps, N, H, dv]
    log_alpha: np.ndarray  # [steps, N, H, dk] fp32
    beta: np.ndarray       # [steps, N, H] fp32
    state: np.ndarray      # [N, H, dk, dv] fp32


def make_decode(N, H, dk, dv, steps, *, seed, state_std=0.02, name="decode") -> DecodeWorkload:
    rng = np.random.default_rng(seed)
    q = _normal(rng, (steps, N, H, dk))
    k = _normal(rng, (steps, N, H, dk))
    v = _normal(rng, (steps, N, H, dv))
    _unit_rows_inplace(q)
    _unit_rows_inplace(k)
    for x in (q, k, v):
        _bf16_round_inplace(x)
    la = _normal(rng, (steps, N, H, dk))
    _neg_softplus_over_16_inplace(la)
    beta = _normal(rng, (steps, N, H))
    _sigmoid_inplace(beta)
    st = _normal(rng, (N, H, dk, dv), state_std)
    return DecodeWorkload(name=name, N=N, H=H, dk=dk, dv=dv, steps=steps,
                          q=q, k=k, v=v, log_alpha=la, beta=beta, state=st)


def make_gate_preactivation(total_T, H, d, *, seed):
    """The decay gate as its pre-activation: a ~ N(0, 1) rounded to bf16 [total_T, H, d],
    and one scale per head drawn uniformly from [1/32, 1/8] (fp32 [H])."""
    rng = np.random.default_rng(seed)
    a = _normal(rng, (total_T, H, d))
    _bf16_round_inplace(a)
    scale = rng.uniform(1 / 32, 1 / 8, H).astype(np.float64)
    return a, scale


def make_cotangents(total_T, N, H, dv, *, seed, qkv_dtype="bf16", dk=None, final_std=0.1):
    """Gradients fed to the backward: d_out ~ N(0, 1) [total_T, H, dv] (rounded to bf16
    when the inputs are bf16) and d_final ~ N(0, final_std^2) fp32 [N, H, dk, dv]
    (None when final_std is 0)."""
    rng = np.random.default_rng(seed)
    d_out = _normal(rng, (total_T, H, dv))
    if qkv_dtype == "bf16":
        _bf16_round_inplace(d_out)
    d_final = _normal(rng, (N, H, dk or dv, dv), final_std) if final_std else None
    return d_out, d_final


@dataclasses.dataclass
class MixerDecodeWorkload:
    """Serving decode of the full mixer: `steps` tokens for N sequences whose states and
    conv histories live in pools of `pool` slots (slot of sequence n: indices[n])."""
    name: str
    N: int
    H: int
    d: int
    steps: int
    pool: int
    q: np.ndarray          # raw [steps, N, H, d], bf16 values
    k: np.ndarray
    v: np.ndarray
    log_alpha: np.ndarray  # [steps, N, H, d]
    beta: np.ndarray       # [steps, N, H]
    gate: np.ndarray       # [steps, N, H, d], bf16 values
    conv_w: np.ndarray     # [3, H*d, 4]
    state_pool: np.ndarray  # [pool, H, d, d]
    conv_pool: np.ndarray   # [pool, H, 3, 3, d], bf16 values (raw rows, oldest first)
    indices: np.ndarray     # int32 [N], distinct slots


def make_mixer_decode(N, H, d, steps, pool, *, seed, state_std=0.02, name="mixer_decode") -> MixerDecodeWorkload:
    rng = np.random.default_rng(seed)
    q = _normal(rng, (steps, N, H, d))
    k = _normal(rng, (steps, N, H, d))
    v = _normal(rng, (steps, N, H, d))
    gate = _normal(rng, (steps, N, H, d))
    for x in (q, k, v, gate):
        _bf16_round_inplace(x)
    la = _normal(rng, (steps, N, H, d))
    _neg_softplus_over_16_inplace(la)
    beta = _normal(rng, (steps, N, H))
    _sigmoid_inplace(beta)
    conv_w = _normal(rng, (3, H * d, 4), 0.5)
    st = _normal(rng, (pool, H, d, d), state_std)
    hist = _normal(rng, (pool, H, 3, 3, d))
    _bf16_round_inplace(hist)
    idx = rng.permutation(pool)[:N].astype(np.int32)
    return MixerDecodeWorkload(name=name, N=N, H=H, d=d, steps=steps, pool=pool, q=q, k=k, v=v, log_alpha=la,
                               beta=beta, gate=gate, conv_w=conv_w, state_pool=st, conv_pool=hist, indices=idx)


# --- the five named workloads ------------------------------------------------

def tiny_recurrence() -> Workload:
    """B=1, T=64, H=2, d_k=d_v=16, fp32 q/k/v, zero initial state."""
    return make_prefill([64], 2, 16, 16, seed=SEED_BASE + 0, qkv_dtype="f32", state_std=0.0,
                        name="tiny_B1_T64_H2_d16_f32", B=1, T=64)


def prefill_model_shape(T: int = 4096) -> Workload:
    """B=1, T=4096, H=32, d_k=d_v=128, bf16 q/k/v, initial state ~ N(0, 0.02^2)."""
    return make_prefill([T], 32, 128, 128, seed=SEED_BASE + 1, name=f"prefill_B1_T{T}_H32_d128_bf16",
                        B=1, T=T)


def mixer_prefill(B: int = 2, T: int = 32768) -> Workload:
    """B=2, T=32768, H=32, d=128: raw bf16 q/k/v through conv4 + L2 norm, sigmoid output gate."""
    return make_prefill([T] * B, 32, 128, 128, seed=SEED_BASE + 2, state_std=0.0, normalise_qk=False,
                        mixer=True, name=f"mixer_B{B}_T{T}_H32_d128_bf16", B=B, T=T)


def decode_batch(N: int = 256, steps: int = 64) -> DecodeWorkload:
    """256 sequences x 32 heads, one token each, 64 consecutive steps, fp32 state in place."""
    return make_decode(N, 32, 128, 128, steps, seed=SEED_BASE + 3, name=f"decode_N{N}_H32_d128_steps{steps}")


def varlen_prefill(n_seqs: int = 64, lo: int = 256, hi: int = 8192) -> Workload:
    """64 packed sequences, lengths ~ U{256..8192} (drawn first), per-sequence initial states."""
    rng = np.random.default_rng(SEED_BASE + 4)
    lens = [int(x) for x in rng.integers(lo, hi + 1, n_seqs)]
    return make_prefill(lens, 32, 128, 128, rng=rng, name=f"varlen_{n_seqs}seqs_H32_d128_bf16")
