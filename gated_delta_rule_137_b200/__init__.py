"""Python binding of libkda.so — a B200 (sm_100a) implementation of the Kimi Delta
Attention (KDA) token mixer.

The binding only marshals arguments: torch tensors supply device memory and the
current CUDA stream, and every step of the computation runs in the library's CUDA
kernels. There is no CPU fallback: if libkda.so is missing or fails to load, the
calls raise.

    out, final = chunk_fwd(q, k, v, log_alpha, beta, initial_state, cu_seqlens)
    out        = decode_step(q, k, v, log_alpha, beta, state)      # state in place
    out, final = mixer_fwd(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, ...)
    out        = mixer_decode_step(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate,
                                   state_pool, conv_pool, state_indices)  # pools in place
    dq, dk, dv, dla, dbeta, dh0 = chunk_bwd(q, k, v, log_alpha, beta, d_out, ...)

Shapes (token-major, packed): q, k, log_alpha [total_T, H, dk]; v [total_T, H, dv];
beta [total_T, H]; states [N, H, dk, dv]; cu_seqlens int32 [N+1] (device).
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkda.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "kda.h")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_WORKSPACE, KDA_ERR_CUDA, KDA_ERR_RANGE = range(6)
KDA_DT_F32, KDA_DT_BF16 = 0, 1
DEVFLAG_BAD_SEQLENS = 0x1
DEVFLAG_DECAY_RANGE = 0x2  # reserved: no entry point sets it
DEVFLAG_BAD_INDEX = 0x4
DEVFLAG_WAIT_TIMEOUT = 0x80000000

_lib = None


class KdaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_STATUS_NAMES = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED", 3: "KDA_ERR_WORKSPACE",
                 4: "KDA_ERR_CUDA", 5: "KDA_ERR_RANGE"}

_vp, _i32, _i64, _sz, _u32p = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.POINTER(ctypes.c_uint32)

_SIGNATURES = {
    "kda_status_string": (ctypes.c_char_p, [_i32]),
    "kda_last_error": (ctypes.c_char_p, []),
    "kda_version": (ctypes.c_char_p, []),
    "kda_chunk_fwd_workspace": (_sz, [_i64, _i32, _i32, _i32, _i32, _i32]),
    "kda_chunk_fwd": (_i32, [_vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _i32,
                             _vp, _vp, _vp, _sz, _vp]),
    "kda_decode_step": (_i32, [_vp, _vp, _vp, _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp]),
    "kda_mixer_fwd_workspace": (_sz, [_i64, _i32, _i32, _i32, _i32]),
    "kda_mixer_fwd": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _i32,
                             _vp, _vp, _vp, _sz, _vp]),
    "kda_mixer_fwd_pooled": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _i32,
                                    _vp, _vp, _vp, _vp, _i32, _vp, _sz, _vp]),
    "kda_workspace_status": (_i32, [_vp, _vp, _u32p]),
    "kda_mixer_fwd_noalloc_status": (_i32, [_vp, _u32p]),
    "kda_selftest_wait_timeout": (_i32, [_vp, _sz, ctypes.c_uint32, _vp]),
    "kda_state_fold": (_i32, [_vp, _i32, _vp, _vp, _i64, _i32, _vp]),
    "kda_segment_maps_workspace": (_sz, [_i64, _i32, _i32, _i32, _i32]),
    "kda_segment_maps": (_i32, [_vp, _vp, _vp, _i32, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _i32, _vp, _vp,
                                _vp, _sz, _vp]),
    "kda_segment_prefill": (_i32, [_vp, _sz, _i32, _vp, _vp, _i64, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "kda_mixer_fwd_noalloc": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _i32,
                                     _vp, _vp, _vp]),
    "kda_mixer_decode_step": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32,
                                     _i32, _vp, _vp, _vp]),
    "kda_mixer_decode_tokens": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32,
                                       _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "kda_mixer_decode_commit": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
    "kda_state_affine": (_i32, [_vp, _vp, _vp, _vp, _i64, _i32, _vp]),
    "kda_mixer_fwd_gate_workspace": (_sz, [_i64, _i32, _i32, _i32, _i32]),
    "kda_mixer_fwd_gate": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _i32,
                                  _vp, _vp, _vp, _sz, _vp]),
    "kda_chunk_bwd_workspace": (_sz, [_i64, _i32, _i32, _i32, _i32]),
    "kda_chunk_bwd": (_i32, [_vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _i32,
                             _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
}


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libkda.so and declare its C signatures. Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"{path} is missing: build it with `python -m gated_delta_rule_137_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def header_functions(path: str = HEADER_PATH) -> list:
    """Names of the functions include/kda.h declares."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", text)))


def _check(status: int) -> None:
    if status != KDA_OK:
        raise KdaError(status, load_library().kda_last_error().decode())


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return KDA_DT_BF16
    if t.dtype == torch.float32:
        return KDA_DT_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return _torch().cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def chunk_fwd_workspace_bytes(total_T: int, N: int, H: int, dk: int, dv: int, dtype_code: int) -> int:
    return int(load_library().kda_chunk_fwd_workspace(total_T, N, H, dk, dv, dtype_code))


def chunk_fwd(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, *, N: Optional[int] = None,
              out=None, final_state=None, output_final_state: bool = True, workspace=None, stream=None,
              check_status: bool = False) -> Tuple[object, object]:
    """Chunked KDA prefill (kda_chunk_fwd). q, k, log_alpha [T, H, dk] or [B, T, H, dk]."""
    torch = _torch()
    lib = load_library()
    if q.dim() == 4:  # fixed-length [B, T, H, d]
        B, T = q.shape[:2]
        q, k, v, log_alpha = (x.reshape(B * T, *x.shape[2:]) for x in (q, k, v, log_alpha))
        beta = beta.reshape(B * T, -1)
        N = B
        shape_back = (B, T)
    else:
        shape_back = None
    total_T, H, dk = q.shape
    dv = v.shape[-1]
    if N is None:
        if cu_seqlens is None:
            raise ValueError("N is needed when cu_seqlens is not given")
        N = cu_seqlens.numel() - 1
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((total_T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    need = int(lib.kda_chunk_fwd_workspace(total_T, N, H, dk, dv, dt))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(lib.kda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(log_alpha), _ptr(beta), _ptr(initial_state),
                             _ptr(cu_seqlens), total_T, N, H, dk, dv, _ptr(out), _ptr(final_state),
                             _ptr(workspace), workspace.numel(), _stream(stream)))
    if check_status:
        workspace_status(workspace, stream)
    if shape_back is not None:
        out = out.reshape(*shape_back, H, dv)
    return out, final_state


def decode_step(q, k, v, log_alpha, beta, state, *, out=None, stream=None):
    """One decode token per (sequence, head); `state` [N, H, dk, dv] fp32 is updated in place."""
    torch = _torch()
    lib = load_library()
    N, H, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    _check(lib.kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(log_alpha), _ptr(beta),
                               _ptr(state), N, H, dk, dv, _ptr(out), _stream(stream)))
    return out


def mixer_fwd(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate=None, initial_state=None, cu_seqlens=None, *,
              N: Optional[int] = None, out=None, final_state=None, output_final_state: bool = True,
              workspace=None, stream=None, check_status: bool = False):
    """Full mixer prefill (kda_mixer_fwd): conv4 -> L2 norm -> KDA -> sigmoid gate."""
    torch = _torch()
    lib = load_library()
    total_T, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    if N is None:
        if cu_seqlens is None:
            raise ValueError("N is needed when cu_seqlens is not given")
        N = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((total_T, H, dv), dtype=torch.bfloat16, device=q_raw.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q_raw.device)
    need = int(lib.kda_mixer_fwd_workspace(total_T, N, H, dk, dv))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q_raw.device)
    _check(lib.kda_mixer_fwd(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_w), _ptr(log_alpha), _ptr(beta),
                             _ptr(gate), _ptr(initial_state), _ptr(cu_seqlens), total_T, N, H, dk, dv, _ptr(out),
                             _ptr(final_state), _ptr(workspace), workspace.numel(), _stream(stream)))
    if check_status:
        workspace_status(workspace, stream)
    return out, final_state


def mixer_fwd_pooled(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, state_pool, conv_pool,
                     state_indices=None, initial_state=None, cu_seqlens=None, *, N: Optional[int] = None, out=None,
                     workspace=None, stream=None, check_status: bool = False):
    """Full mixer prefill handing its sequences to the serving decode (kda_mixer_fwd_pooled):
    final states into state_pool[slot] fp32 [P, H, 128, 128], the last three raw q, k, v rows
    into conv_pool[slot] bf16 [P, H, 3, 3, 128]. Returns out."""
    torch = _torch()
    lib = load_library()
    total_T, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    if N is None:
        if cu_seqlens is None:
            raise ValueError("N is needed when cu_seqlens is not given")
        N = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((total_T, H, dv), dtype=torch.bfloat16, device=q_raw.device)
    need = int(lib.kda_mixer_fwd_workspace(total_T, N, H, dk, dv))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q_raw.device)
    _check(lib.kda_mixer_fwd_pooled(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_w), _ptr(log_alpha), _ptr(beta),
                                    _ptr(gate), _ptr(initial_state), _ptr(cu_seqlens), total_T, N, H, dk, dv,
                                    _ptr(out), _ptr(state_pool), _ptr(conv_pool), _ptr(state_indices),
                                    state_pool.shape[0], _ptr(workspace), workspace.numel(), _stream(stream)))
    if check_status:
        workspace_status(workspace, stream)
    return out


def mixer_decode_step(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, state_pool, conv_pool,
                      state_indices=None, *, out=None, status=None, stream=None):
    """Serving decode step of the full mixer (kda_mixer_decode_step): one token per
    sequence, q_raw/k_raw/v_raw/gate bf16 [N, H, 128]; state_pool fp32 [P, H, 128, 128]
    and conv_pool bf16 [P, H, 3, 3, 128] updated in place; state_indices int32 [N] or
    None (slot n). `status`: a device uint32 tensor (>= 4 bytes) for device flags."""
    torch = _torch()
    lib = load_library()
    N, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    if out is None:
        out = torch.empty((N, H, dv), dtype=torch.bfloat16, device=q_raw.device)
    _check(lib.kda_mixer_decode_step(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_w), _ptr(log_alpha),
                                     _ptr(beta), _ptr(gate), _ptr(state_pool), _ptr(conv_pool), _ptr(state_indices),
                                     state_pool.shape[0], N, H, dk, dv, _ptr(out), _ptr(status), _stream(stream)))
    return out


def mixer_decode_tokens(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate, state_pool, conv_pool,
                        state_indices=None, *, out=None, state_ckpt=None, conv_ckpt=None, status=None, stream=None):
    """K tokens per sequence (kda_mixer_decode_tokens): q_raw/k_raw/v_raw/gate bf16
    [N, K, H, 128]; with state_ckpt fp32 [N, K, H, 128, 128] and conv_ckpt bf16
    [N, K, H, 3, 3, 128] the pools stay unchanged (see mixer_decode_commit)."""
    torch = _torch()
    lib = load_library()
    N, K, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    if out is None:
        out = torch.empty((N, K, H, dv), dtype=torch.bfloat16, device=q_raw.device)
    _check(lib.kda_mixer_decode_tokens(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_w), _ptr(log_alpha),
                                       _ptr(beta), _ptr(gate), _ptr(state_pool), _ptr(conv_pool),
                                       _ptr(state_indices), state_pool.shape[0], N, K, H, dk, dv, _ptr(out),
                                       _ptr(state_ckpt), _ptr(conv_ckpt), _ptr(status), _stream(stream)))
    return out


def mixer_decode_commit(state_ckpt, conv_ckpt, accepted, state_pool, conv_pool, state_indices=None, *,
                        status=None, stream=None):
    """Install checkpoint accepted[n] - 1 into each sequence's slot (kda_mixer_decode_commit)."""
    lib = load_library()
    N, K, H, d = state_ckpt.shape[:4]
    _check(lib.kda_mixer_decode_commit(_ptr(state_ckpt), _ptr(conv_ckpt), _ptr(accepted), _ptr(state_pool),
                                       _ptr(conv_pool), _ptr(state_indices), state_pool.shape[0], N, K, H, d,
                                       _ptr(status), _stream(stream)))


def state_affine(M, S=None, B=None, *, out=None, stream=None):
    """out = M S + B over [..., 128, 128] fp32 matrices (kda_state_affine); S or B None = 0."""
    torch = _torch()
    lib = load_library()
    d = M.shape[-1]
    count = M.numel() // (d * d)
    if out is None:
        out = torch.empty_like(M)
    _check(lib.kda_state_affine(_ptr(M), _ptr(S), _ptr(B), _ptr(out), count, d, _stream(stream)))
    return out


def mixer_fwd_gate(q_raw, k_raw, v_raw, conv_w, a_pre, a_scale, beta, gate=None, initial_state=None,
                   cu_seqlens=None, *, N: Optional[int] = None, out=None, final_state=None,
                   output_final_state: bool = True, workspace=None, stream=None, check_status: bool = False):
    """Full mixer prefill with log_alpha = -a_scale[h] * softplus(a_pre) made on the
    device (kda_mixer_fwd_gate); a_pre bf16 [T, H, 128], a_scale fp32 [H]."""
    torch = _torch()
    lib = load_library()
    total_T, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    if N is None:
        if cu_seqlens is None:
            raise ValueError("N is needed when cu_seqlens is not given")
        N = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((total_T, H, dv), dtype=torch.bfloat16, device=q_raw.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q_raw.device)
    need = int(lib.kda_mixer_fwd_gate_workspace(total_T, N, H, dk, dv))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q_raw.device)
    _check(lib.kda_mixer_fwd_gate(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_w), _ptr(a_pre), _ptr(a_scale),
                                  _ptr(beta), _ptr(gate), _ptr(initial_state), _ptr(cu_seqlens), total_T, N, H, dk, dv,
                                  _ptr(out), _ptr(final_state), _ptr(workspace), workspace.numel(), _stream(stream)))
    if check_status:
        workspace_status(workspace, stream)
    return out, final_state


def chunk_bwd_workspace_bytes(total_T: int, N: int, H: int, dk: int = 128, dv: int = 128) -> int:
    return int(load_library().kda_chunk_bwd_workspace(total_T, N, H, dk, dv))


def chunk_bwd(q, k, v, log_alpha, beta, d_out, initial_state=None, cu_seqlens=None, d_final_state=None, *,
              N: Optional[int] = None, output_d_initial_state: bool = True, workspace=None, stream=None,
              check_status: bool = False):
    """Backward of the recurrence (kda_chunk_bwd). Packed [total_T, H, 128] inputs as for
    chunk_fwd; d_out like v. Returns fp32 (dq, dk, dv, d_log_alpha, d_beta,
    d_initial_state or None)."""
    torch = _torch()
    lib = load_library()
    total_T, H, dk = q.shape
    dv = v.shape[-1]
    if N is None:
        if cu_seqlens is None:
            raise ValueError("N is needed when cu_seqlens is not given")
        N = cu_seqlens.numel() - 1
    dt = _dtype_code(q)
    f32 = dict(dtype=torch.float32, device=q.device)
    dq, dk_, dv_, dla = (torch.empty((total_T, H, n), **f32) for n in (dk, dk, dv, dk))
    dbeta = torch.empty((total_T, H), **f32)
    dh0 = torch.empty((N, H, dk, dv), **f32) if output_d_initial_state else None
    need = int(lib.kda_chunk_bwd_workspace(total_T, N, H, dk, dv))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(lib.kda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(log_alpha), _ptr(beta), _ptr(initial_state),
                             _ptr(cu_seqlens), total_T, N, H, dk, dv, _ptr(d_out), _ptr(d_final_state), _ptr(dq),
                             _ptr(dk_), _ptr(dv_), _ptr(dla), _ptr(dbeta), _ptr(dh0), _ptr(workspace),
                             workspace.numel(), _stream(stream)))
    if check_status:
        workspace_status(workspace, stream)
    return dq, dk_, dv_, dla, dbeta, dh0


def workspace_status(workspace, stream=None) -> int:
    """Reads and clears the device status word; raises KdaError(KDA_ERR_RANGE) if set."""
    lib = load_library()
    flags = ctypes.c_uint32(0)
    st = lib.kda_workspace_status(_ptr(workspace), _stream(stream), ctypes.byref(flags))
    if st not in (KDA_OK, KDA_ERR_RANGE):
        _check(st)
    if st == KDA_ERR_RANGE:
        raise KdaError(st, f"device status flags 0x{flags.value:08x}")
    return flags.value


def mixer_fwd_noalloc(q_raw, k_raw, v_raw, conv_w, log_alpha, beta, gate=None, initial_state=None,
                      cu_seqlens=None, *, N: Optional[int] = None, out=None, final_state=None,
                      output_final_state: bool = True, stream=None, check_status: bool = False):
    """Full mixer prefill without a workspace (kda_mixer_fwd_noalloc): the scratch is a
    fixed array inside the library (total_T * H <= 16384 token-heads)."""
    torch = _torch()
    lib = load_library()
    total_T, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    if N is None:
        if cu_seqlens is None:
            raise ValueError("N is needed when cu_seqlens is not given")
        N = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((total_T, H, dv), dtype=torch.bfloat16, device=q_raw.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q_raw.device)
    _check(lib.kda_mixer_fwd_noalloc(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_w), _ptr(log_alpha),
                                     _ptr(beta), _ptr(gate), _ptr(initial_state), _ptr(cu_seqlens), total_T, N, H,
                                     dk, dv, _ptr(out), _ptr(final_state), _stream(stream)))
    if check_status:
        noalloc_status(stream)
    return out, final_state


def noalloc_status(stream=None) -> int:
    """Reads and clears the status word of kda_mixer_fwd_noalloc on the current device;
    raises KdaError(KDA_ERR_RANGE) if a flag was set."""
    lib = load_library()
    flags = ctypes.c_uint32(0)
    st = lib.kda_mixer_fwd_noalloc_status(_stream(stream), ctypes.byref(flags))
    if st not in (KDA_OK, KDA_ERR_RANGE):
        _check(st)
    if st == KDA_ERR_RANGE:
        raise KdaError(st, f"device status flags 0x{flags.value:08x}")
    return flags.value


def selftest_wait_timeout(workspace, budget_us: int, stream=None) -> None:
    """Runs the bounded-wait diagnostic (kda_selftest_wait_timeout): one thread waits on
    an mbarrier that nothing arrives at and gives up after budget_us, setting
    DEVFLAG_WAIT_TIMEOUT in the workspace's status word (read it with workspace_status)."""
    lib = load_library()
    _check(lib.kda_selftest_wait_timeout(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                         budget_us, _stream(stream)))


class SegmentMaps:
    """What kda_segment_maps leaves for kda_segment_prefill: the workspace holding the
    segment's per-chunk operands, and the sizes and dtype they were made with."""

    def __init__(self, workspace, cu_seqlens, total_T: int, N: int, H: int, dtype_code: int, device):
        self.workspace, self.cu_seqlens = workspace, cu_seqlens
        self.total_T, self.N, self.H, self.dtype_code, self.device = total_T, N, H, dtype_code, device


def segment_maps(q, k, v, log_alpha, beta, cu_seqlens=None, *, N: Optional[int] = None, workspace=None,
                 stream=None, check_status: bool = False):
    """(M, B, handle) of a segment (kda_segment_maps): S_end = M S_start + B for each of its
    sequences; `handle` feeds segment_prefill."""
    torch = _torch()
    lib = load_library()
    total_T, H, dk = q.shape
    dv = v.shape[-1]
    if N is None:
        if cu_seqlens is None:
            raise ValueError("N is needed when cu_seqlens is not given")
        N = cu_seqlens.numel() - 1
    dt = _dtype_code(q)
    f32 = dict(dtype=torch.float32, device=q.device)
    M, B = torch.empty((N, H, dk, dv), **f32), torch.empty((N, H, dk, dv), **f32)
    need = int(lib.kda_segment_maps_workspace(total_T, N, H, dk, dv))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(lib.kda_segment_maps(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(log_alpha), _ptr(beta), _ptr(cu_seqlens),
                                total_T, N, H, dk, dv, _ptr(M), _ptr(B), _ptr(workspace), workspace.numel(),
                                _stream(stream)))
    if check_status:
        workspace_status(workspace, stream)
    return M, B, SegmentMaps(workspace, cu_seqlens, total_T, N, H, dt, q.device)


def segment_prefill(handle: SegmentMaps, initial_state=None, *, out=None, final_state=None,
                    output_final_state: bool = True, stream=None, check_status: bool = False):
    """The segment of `handle` prefilled from `initial_state` (kda_segment_prefill)."""
    torch = _torch()
    lib = load_library()
    h = handle
    if out is None:
        dtype = torch.float32 if h.dtype_code == KDA_DT_F32 else torch.bfloat16
        out = torch.empty((h.total_T, h.H, 128), dtype=dtype, device=h.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((h.N, h.H, 128, 128), dtype=torch.float32, device=h.device)
    _check(lib.kda_segment_prefill(_ptr(h.workspace), h.workspace.numel(), h.dtype_code, _ptr(initial_state),
                                   _ptr(h.cu_seqlens), h.total_T, h.N, h.H, 128, 128, _ptr(out), _ptr(final_state),
                                   _stream(stream)))
    if check_status:
        workspace_status(h.workspace, stream)
    return out, final_state


def state_fold(MB, maps: int, S0=None, *, out=None, stream=None):
    """S <- M_j S + B_j for j < maps (kda_state_fold); MB [>= maps, 2, ..., 128, 128] fp32
    (M then B of each map), S0 like one M or None (zero)."""
    torch = _torch()
    lib = load_library()
    d = MB.shape[-1]
    count = MB[0, 0].numel() // (d * d)
    if out is None:
        out = torch.empty(MB.shape[2:], dtype=torch.float32, device=MB.device)
    _check(lib.kda_state_fold(_ptr(MB), maps, _ptr(S0), _ptr(out), count, d, _stream(stream)))
    return out
