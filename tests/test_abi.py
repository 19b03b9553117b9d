"""The C-ABI library: it loads, exports every function include/kda.h declares, and
rejects bad arguments on the host before touching the GPU (CPU tests), plus
device-side error paths (GPU tests)."""
import ctypes
import subprocess

import numpy as np
import pytest

import gated_delta_rule_137_b200 as kda

FAKE = 0x10000  # 16-byte aligned non-null address; never dereferenced by host checks


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_137_b200 import build
    build.build()
    return kda.load_library()


def test_exports_match_header(lib):
    declared = kda.header_functions()
    assert set(declared) >= {"kda_chunk_fwd", "kda_decode_step", "kda_mixer_fwd", "kda_chunk_fwd_workspace",
                             "kda_mixer_fwd_workspace", "kda_workspace_status", "kda_status_string",
                             "kda_last_error", "kda_version"}
    out = subprocess.run(["nm", "-D", "--defined-only", kda.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [f for f in declared if f not in exported]
    assert not missing, f"declared but not exported: {missing}"
    # nothing else of ours leaks out of the library
    ours = {s for s in exported if s.startswith("kda")}
    assert ours == set(declared)
    for f in declared:
        assert getattr(lib, f) is not None


def test_status_strings(lib):
    for code, name in [(0, b"KDA_OK"), (1, b"KDA_ERR_INVALID_ARG"), (2, b"KDA_ERR_UNSUPPORTED"),
                       (3, b"KDA_ERR_WORKSPACE"), (4, b"KDA_ERR_CUDA"), (5, b"KDA_ERR_RANGE")]:
        assert lib.kda_status_string(code) == name
    assert lib.kda_version().decode().count(".") == 2


def test_workspace_query(lib):
    item = 147968  # two-pass scratch per (64-token chunk, head)
    ws = lib.kda_chunk_fwd_workspace(4096, 1, 32, 128, 128, kda.KDA_DT_BF16)
    # status word + chunk offsets + items for at most 4096/64 + 1 chunks per head
    assert ws == 256 + 256 + (64 + 1) * 32 * item
    assert ws % 256 == 0
    full = lib.kda_chunk_fwd_workspace(64, 1, 2, 128, 128, kda.KDA_DT_F32)
    small = lib.kda_chunk_fwd_workspace(64, 1, 2, 16, 16, kda.KDA_DT_F32)
    assert small > full  # zero-padded staging copies for d < 128
    assert full == 256 + 256 + 2 * 2 * item  # bound min(T/64 + N, T) = 2 chunks, 2 heads
    assert lib.kda_chunk_fwd_workspace(0, 1, 2, 128, 128, kda.KDA_DT_F32) == 256  # no tokens: status word only
    assert lib.kda_chunk_fwd_workspace(64, 1, 2, 0, 16, kda.KDA_DT_F32) == 0
    assert lib.kda_chunk_fwd_workspace(64, 1, 2, 129, 16, kda.KDA_DT_BF16) == 0
    assert lib.kda_chunk_fwd_workspace(64, 1, 2, 16, 16, 7) == 0
    # beyond 32 GiB of scratch, or beyond 74 (sequence, head) chains, the single-pass kernel
    # runs and the query drops the scratch
    huge_T = (1 << 31) - 1024
    assert lib.kda_chunk_fwd_workspace(huge_T, 1, 32, 128, 128, kda.KDA_DT_BF16) == 256
    assert lib.kda_chunk_fwd_workspace(4096, 3, 25, 128, 128, kda.KDA_DT_BF16) == 256  # 75 chains
    assert lib.kda_chunk_fwd_workspace(4096, 2, 37, 128, 128, kda.KDA_DT_BF16) > 256   # 74 chains
    assert lib.kda_mixer_fwd_workspace(1000, 2, 32, 128, 128) == 256 + 256 + (1000 // 64 + 2) * 32 * item
    assert lib.kda_mixer_fwd_workspace(1000, 2, 32, 64, 64) == 0


def _chunk(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dt=kda.KDA_DT_BF16, la=FAKE, beta=FAKE, h0=None, cu=None, total_T=128, N=1,
             H=2, dk=128, dv=128, out=FAKE * 2, ht=None, ws=FAKE * 3, ws_bytes=1 << 20, stream=None)
    a.update(kw)
    return lib.kda_chunk_fwd(a["q"], a["k"], a["v"], a["dt"], a["la"], a["beta"], a["h0"], a["cu"], a["total_T"],
                             a["N"], a["H"], a["dk"], a["dv"], a["out"], a["ht"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("bad,status", [
    (dict(dk=0), kda.KDA_ERR_INVALID_ARG),
    (dict(dv=129), kda.KDA_ERR_INVALID_ARG),
    (dict(H=0), kda.KDA_ERR_INVALID_ARG),
    (dict(N=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(total_T=-5), kda.KDA_ERR_INVALID_ARG),
    (dict(dt=3), kda.KDA_ERR_INVALID_ARG),
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(out=None), kda.KDA_ERR_INVALID_ARG),
    (dict(beta=FAKE + 4), kda.KDA_ERR_INVALID_ARG),           # misaligned
    (dict(N=3, total_T=128), kda.KDA_ERR_INVALID_ARG),        # equal lengths need T % N == 0
    (dict(N=0, total_T=64), kda.KDA_ERR_INVALID_ARG),
    (dict(cu=FAKE + 2), kda.KDA_ERR_INVALID_ARG),             # cu_seqlens not 4-byte aligned
    (dict(ws=None), kda.KDA_ERR_WORKSPACE),
    (dict(ws_bytes=16), kda.KDA_ERR_WORKSPACE),
    (dict(h0=FAKE * 8, ht=FAKE * 8 + 1024), kda.KDA_ERR_INVALID_ARG),  # partial state overlap
    (dict(out=FAKE), kda.KDA_ERR_INVALID_ARG),                # out aliases q
])
def test_chunk_fwd_rejects_bad_arguments(lib, bad, status):
    assert _chunk(lib, **bad) == status
    assert lib.kda_last_error()  # a message explains it


def test_chunk_fwd_empty_batch_is_a_no_op(lib):
    assert _chunk(lib, N=0, total_T=0) == kda.KDA_OK
    assert lib.kda_last_error() == b""


def test_decode_rejects_bad_arguments(lib):
    args = [FAKE, FAKE, FAKE, kda.KDA_DT_BF16, FAKE, FAKE, FAKE * 4, 4, 2, 128, 128, FAKE * 16, None]
    bad = list(args); bad[9] = 0
    assert lib.kda_decode_step(*bad) == kda.KDA_ERR_INVALID_ARG
    bad = list(args); bad[10] = 30  # dv not a multiple of 4
    assert lib.kda_decode_step(*bad) == kda.KDA_ERR_UNSUPPORTED
    bad = list(args); bad[6] = FAKE * 4 + 8  # state misaligned
    assert lib.kda_decode_step(*bad) == kda.KDA_ERR_INVALID_ARG
    bad = list(args); bad[11] = FAKE * 4  # out overlaps state
    assert lib.kda_decode_step(*bad) == kda.KDA_ERR_INVALID_ARG
    bad = list(args); bad[0] = None
    assert lib.kda_decode_step(*bad) == kda.KDA_ERR_INVALID_ARG
    ok = list(args); ok[7] = 0  # N = 0: nothing to do
    assert lib.kda_decode_step(*ok) == kda.KDA_OK


def test_mixer_rejects_bad_arguments(lib):
    base = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 128, 1, 2, 128, 128, FAKE * 2, None, FAKE * 3,
            1 << 24, None]
    bad = list(base); bad[12] = 64; bad[13] = 64
    assert lib.kda_mixer_fwd(*bad) == kda.KDA_ERR_UNSUPPORTED
    bad = list(base); bad[3] = None
    assert lib.kda_mixer_fwd(*bad) == kda.KDA_ERR_INVALID_ARG
    bad = list(base); bad[17] = 100
    assert lib.kda_mixer_fwd(*bad) == kda.KDA_ERR_WORKSPACE
    assert lib.kda_workspace_status(None, None, None) == kda.KDA_ERR_INVALID_ARG


def test_binding_fails_loudly_without_the_library(tmp_path):
    import importlib
    mod = importlib.import_module("gated_delta_rule_137_b200")
    saved = mod._lib
    try:
        mod._lib = None
        with pytest.raises(OSError):
            mod.load_library(str(tmp_path / "nope.so"))
    finally:
        mod._lib = saved


def test_mixer_decode_rejects_bad_arguments(lib):
    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, w=FAKE, la=FAKE, b=FAKE, g=None, sp=FAKE * 4, cp=FAKE * 64, idx=None,
                 pool=8, N=4, H=2, dk=128, dv=128, out=FAKE * 128, status=None)
        a.update(kw)
        return lib.kda_mixer_decode_step(a["q"], a["k"], a["v"], a["w"], a["la"], a["b"], a["g"], a["sp"], a["cp"],
                                         a["idx"], a["pool"], a["N"], a["H"], a["dk"], a["dv"], a["out"], a["status"],
                                         None)
    assert call(dk=64, dv=64) == kda.KDA_ERR_UNSUPPORTED
    assert call(pool=0) == kda.KDA_ERR_INVALID_ARG
    assert call(N=9) == kda.KDA_ERR_INVALID_ARG             # no indices: slot n needs n < pool_size
    assert call(q=None) == kda.KDA_ERR_INVALID_ARG
    assert call(sp=FAKE * 4 + 8) == kda.KDA_ERR_INVALID_ARG  # misaligned state pool
    assert call(idx=FAKE + 2) == kda.KDA_ERR_INVALID_ARG     # misaligned indices
    assert call(out=FAKE * 4) == kda.KDA_ERR_INVALID_ARG     # out overlaps the state pool
    assert call(N=0) == kda.KDA_OK                           # nothing to do
    assert b"pool_size" in lib.kda_last_error() or lib.kda_last_error() == b""


def test_mixer_decode_tokens_and_commit_reject_bad_arguments(lib):
    base = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE * 4, FAKE * 64, None, 8, 4, 3, 2, 128, 128, FAKE * 128,
            None, None, None, None]
    bad = list(base); bad[12] = -1                 # K < 0
    assert lib.kda_mixer_decode_tokens(*bad) == kda.KDA_ERR_INVALID_ARG
    bad = list(base); bad[17] = FAKE * 256         # state checkpoint without the history checkpoint
    assert lib.kda_mixer_decode_tokens(*bad) == kda.KDA_ERR_INVALID_ARG
    bad = list(base); bad[12] = 0                  # K = 0: nothing to do
    assert lib.kda_mixer_decode_tokens(*bad) == kda.KDA_OK
    cbase = [FAKE, FAKE * 2, FAKE * 3, FAKE * 4, FAKE * 5, None, 8, 4, 3, 2, 128, None, None]
    bad = list(cbase); bad[2] = None                # accepted missing
    assert lib.kda_mixer_decode_commit(*bad) == kda.KDA_ERR_INVALID_ARG
    bad = list(cbase); bad[8] = 0                   # K = 0
    assert lib.kda_mixer_decode_commit(*bad) == kda.KDA_ERR_INVALID_ARG
    bad = list(cbase); bad[10] = 64                 # d != 128
    assert lib.kda_mixer_decode_commit(*bad) == kda.KDA_ERR_UNSUPPORTED


def test_state_affine_rejects_bad_arguments(lib):
    assert lib.kda_state_affine(FAKE, FAKE * 2, FAKE * 3, FAKE * 4, 2, 64, None) == kda.KDA_ERR_UNSUPPORTED
    assert lib.kda_state_affine(None, FAKE * 2, FAKE * 3, FAKE * 4, 2, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_state_affine(FAKE, FAKE * 2, FAKE * 3, FAKE * 4, -1, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_state_affine(FAKE, FAKE * 2, FAKE * 3, FAKE + 8, 2, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_state_affine(FAKE, FAKE * 2, None, FAKE * 2, 2, 128, None) == kda.KDA_ERR_INVALID_ARG  # out is S
    assert lib.kda_state_affine(FAKE, None, None, FAKE * 4, 0, 128, None) == kda.KDA_OK  # nothing to do


def test_chunk_bwd_workspace_formula(lib):
    # status word + plan + one fp32 state per 8 tokens (8 per 64-token chunk bound) and head
    def expect(T, N, H):
        plan = -(-(N + 1) * 4 // 256) * 256
        chunks = min(T // 64 + N, T)
        ckpt = -(-(chunks * 8 * H * 128 * 128 * 4) // 256) * 256
        return 256 + plan + ckpt
    assert lib.kda_chunk_bwd_workspace(0, 3, 2, 128, 128) == 256 + 256   # status + plan only
    for T, N, H in [(4096, 1, 32), (300, 5, 2), (1, 1, 1), (262144, 64, 32)]:
        assert lib.kda_chunk_bwd_workspace(T, N, H, 128, 128) == expect(T, N, H)
    assert lib.kda_chunk_bwd_workspace(4096, 1, 32, 64, 128) == 0   # only dk == dv == 128
    assert lib.kda_chunk_bwd_workspace(-1, 1, 32, 128, 128) == 0


def test_chunk_bwd_rejects_bad_arguments(lib):
    ws = lib.kda_chunk_bwd_workspace(128, 2, 2, 128, 128)
    # disjoint 16-byte aligned fake ranges, 1 MiB apart (each tensor here is < 1 MiB)
    f = [0x10000000 + i * (1 << 20) for i in range(16)]

    def call(q=f[0], la=f[1], beta=f[2], d_out=f[3], dq=f[4], dbeta=f[5], cu=None, T=128, N=2, dk=128,
             ws_bytes=ws, dtype=kda.KDA_DT_BF16):
        return lib.kda_chunk_bwd(q, f[6], f[7], dtype, la, beta, None, cu, T, N, 2, dk, 128, d_out, None, dq, f[8],
                                 f[9], f[10], dbeta, None, f[11], ws_bytes, None)
    assert call(dk=64) == kda.KDA_ERR_UNSUPPORTED
    assert call(dtype=7) == kda.KDA_ERR_INVALID_ARG
    assert call(d_out=None) == kda.KDA_ERR_INVALID_ARG
    assert call(dbeta=None) == kda.KDA_ERR_INVALID_ARG
    assert call(q=f[0] + 8) == kda.KDA_ERR_INVALID_ARG         # misaligned
    assert call(beta=f[2] + 2) == kda.KDA_ERR_INVALID_ARG      # beta needs 4-byte alignment
    assert call(T=129) == kda.KDA_ERR_INVALID_ARG              # not a multiple of N without cu_seqlens
    assert call(ws_bytes=ws - 256) == kda.KDA_ERR_WORKSPACE
    assert call(T=0, N=0) == kda.KDA_OK                        # empty batch: nothing to do


def test_chunk_bwd_rejects_overlapping_outputs(lib):
    T, N, H = 64, 1, 2
    tok = T * H * 128
    ws = lib.kda_chunk_bwd_workspace(T, N, H, 128, 128)
    # disjoint 16-byte aligned fake ranges, 1 MiB apart (each tensor here is < 1 MiB)
    base = [0x10000000 + i * (1 << 20) for i in range(16)]
    q, k, v, la, beta, dout, dq, dk, dv, dla, dbeta, wsp = base[:12]

    def call(**kw):
        a = dict(q=q, k=k, v=v, la=la, beta=beta, dout=dout, dq=dq, dk=dk, dv=dv, dla=dla, dbeta=dbeta)
        a.update(kw)
        return lib.kda_chunk_bwd(a["q"], a["k"], a["v"], kda.KDA_DT_BF16, a["la"], a["beta"], None, None, T, N, H,
                                 128, 128, a["dout"], None, a["dq"], a["dk"], a["dv"], a["dla"], a["dbeta"], None,
                                 wsp, ws, None)
    assert call(dq=q) == kda.KDA_ERR_INVALID_ARG                  # an output on an input
    assert call(dla=la + 16 * (tok // 8)) == kda.KDA_ERR_INVALID_ARG  # partly inside log_alpha
    assert call(dk=dq) == kda.KDA_ERR_INVALID_ARG                 # two outputs on each other
    assert call(dbeta=dv + 256) == kda.KDA_ERR_INVALID_ARG


def test_mixer_pooled_rejects_bad_arguments(lib):
    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, w=FAKE, la=FAKE, b=FAKE, g=None, h0=None, cu=None, T=128, N=2, H=2, dk=128,
                 dv=128, out=FAKE * 2, sp=FAKE * 256, cp=FAKE * 1024, idx=None, pool=8, ws=FAKE * 3, wsb=1 << 24)
        a.update(kw)
        return lib.kda_mixer_fwd_pooled(a["q"], a["k"], a["v"], a["w"], a["la"], a["b"], a["g"], a["h0"], a["cu"],
                                        a["T"], a["N"], a["H"], a["dk"], a["dv"], a["out"], a["sp"], a["cp"],
                                        a["idx"], a["pool"], a["ws"], a["wsb"], None)
    assert call(dk=64, dv=64) == kda.KDA_ERR_UNSUPPORTED
    assert call(pool=0) == kda.KDA_ERR_INVALID_ARG
    assert call(pool=1) == kda.KDA_ERR_INVALID_ARG              # no indices: slot n needs n < pool_size
    assert call(sp=None) == kda.KDA_ERR_INVALID_ARG
    assert call(cp=FAKE * 1024 + 8) == kda.KDA_ERR_INVALID_ARG  # misaligned history pool
    assert call(idx=FAKE + 2) == kda.KDA_ERR_INVALID_ARG        # misaligned indices
    assert call(out=FAKE * 256) == kda.KDA_ERR_INVALID_ARG      # out overlaps the state pool
    assert call(h0=FAKE * 256) == kda.KDA_ERR_INVALID_ARG       # the start states inside the pool
    assert call(wsb=100) == kda.KDA_ERR_WORKSPACE
    assert call(N=0, T=0) == kda.KDA_OK                         # nothing to do


def test_state_fold_rejects_bad_arguments(lib):
    assert lib.kda_state_fold(FAKE, 2, None, FAKE * 64, 2, 64, None) == kda.KDA_ERR_UNSUPPORTED
    assert lib.kda_state_fold(FAKE, -1, None, FAKE * 64, 2, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_state_fold(None, 2, None, FAKE * 64, 2, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_state_fold(FAKE, 2, None, FAKE * 64 + 4, 2, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_state_fold(FAKE, 2, None, FAKE * 2, 2, 128, None) == kda.KDA_ERR_INVALID_ARG  # out in the maps
    assert lib.kda_state_fold(FAKE, 2, FAKE * 64 + 16, FAKE * 64, 2, 128, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_state_fold(None, 0, None, None, 0, 128, None) == kda.KDA_OK  # nothing to do
