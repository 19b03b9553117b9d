"""kda_mixer_fwd_noalloc: the full mixer for callers that may not allocate device
memory (no workspace argument; scratch is a fixed array inside the library).

Checked through the C ABI against kda_mixer_fwd (the workspace entry point) and
against the oracle on the same inputs, on two calls in a row (the second call reuses
the scratch the first one left behind), within the parity tolerance of the other
prefill tests; its status word is read with kda_mixer_fwd_noalloc_status. This file
is collected last so that a stop-at-first-failure run has already run the rest of
the suite.
"""
import ctypes

import numpy as np
import pytest

from gated_delta_rule_137_b200 import inputs as I
from oracle import kda_oracle as O
from tests.helpers import assert_prefill_close, to_device, to_host

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


def _ptr(t):
    return None if t is None else t.data_ptr()


def test_mixer_noalloc_matches_workspace_entry_point(kda):
    import torch
    lib = kda.load_library()
    w = I.make_prefill([300, 77, 5], 4, 128, 128, seed=4242, normalise_qk=False, mixer=True)
    dt = "bf16"
    q, k, v = to_device(w.q, dt), to_device(w.k, dt), to_device(w.v, dt)
    cw, la, b = to_device(w.conv_w, "f32"), to_device(w.log_alpha, "f32"), to_device(w.beta, "f32")
    g, h0, cu = to_device(w.gate, dt), to_device(w.initial_state, "f32"), to_device(w.cu_seqlens, "i32")
    ref_out, ref_fin = kda.mixer_fwd(q, k, v, cw, la, b, g, h0, cu, N=w.N)
    torch.cuda.synchronize()
    ref_out, ref_fin = to_host(ref_out), to_host(ref_fin)
    ora_out, ora_fin = O.kda_mixer(w.q, w.k, w.v, w.conv_w, w.log_alpha, w.beta, w.gate, w.cu_seqlens,
                                   w.initial_state)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full((w.total_T, 4, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        fin = torch.full((w.N, 4, 128, 128), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.kda_mixer_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(cw), _ptr(la), _ptr(b), _ptr(g), _ptr(h0),
                                       _ptr(cu), w.total_T, w.N, 4, 128, 128, _ptr(out), _ptr(fin), stream)
        assert st == kda.KDA_OK, lib.kda_last_error().decode()
        torch.cuda.synchronize()
        assert_prefill_close(to_host(out), ref_out, f"noalloc out (call {call + 1})", stored_bf16=True)
        assert_prefill_close(to_host(fin), ref_fin, f"noalloc final state (call {call + 1})")
        assert_prefill_close(to_host(out), ora_out, f"noalloc out vs oracle (call {call + 1})", stored_bf16=True)
        assert_prefill_close(to_host(fin), ora_fin, f"noalloc final state vs oracle (call {call + 1})")
        assert kda.noalloc_status() == 0


def test_mixer_noalloc_rejects_problems_beyond_its_scratch(kda):
    lib = kda.load_library()
    fake = 0x10000
    # 1024 tokens x 32 heads exceeds the 16384 token-head capacity: refused before any launch
    st = lib.kda_mixer_fwd_noalloc(fake, fake, fake, fake, fake, fake, None, None, None, 1024, 1, 32, 128, 128,
                                   fake * 2, None, None)
    assert st == kda.KDA_ERR_UNSUPPORTED
    assert b"static scratch capacity" in lib.kda_last_error()


def test_mixer_noalloc_warm_up_call_launches_nothing(kda):
    """total_T = N = 0 with no tensors: the set-up a caller makes before capturing or
    filling the device; it succeeds and writes nothing."""
    import torch
    lib = kda.load_library()
    st = lib.kda_mixer_fwd_noalloc(None, None, None, None, None, None, None, None, None, 0, 0, 32, 128, 128,
                                   None, None, torch.cuda.current_stream().cuda_stream)
    assert st == kda.KDA_OK, lib.kda_last_error().decode()


def test_mixer_noalloc_strong_decay_and_status(kda):
    """Strong decay (about 6.5 nats per token on the odd chunks, walked token by token)
    through the no-alloc path against the oracle with a clean status word; then a
    cu_seqlens that is not monotone, which the status reader must report."""
    import torch
    w = I.make_prefill([150, 70], 4, 128, 128, seed=4343, normalise_qk=False, mixer=True)
    la = w.log_alpha.copy()
    for n in range(w.N):
        s0, e0 = int(w.cu_seqlens[n]), int(w.cu_seqlens[n + 1])
        odd = ((np.arange(e0 - s0) // 64) % 2) == 1
        la[s0:e0][odd] *= 128.0
    dt = "bf16"
    args = (to_device(w.q, dt), to_device(w.k, dt), to_device(w.v, dt), to_device(w.conv_w, "f32"),
            to_device(la, "f32"), to_device(w.beta, "f32"), to_device(w.gate, dt), to_device(w.initial_state, "f32"))
    out, fin = kda.mixer_fwd_noalloc(*args, to_device(w.cu_seqlens, "i32"), N=w.N, check_status=True)
    torch.cuda.synchronize()
    ro, rf = O.kda_mixer(w.q, w.k, w.v, w.conv_w, la, w.beta, w.gate, w.cu_seqlens, w.initial_state)
    assert_prefill_close(to_host(out), ro, "noalloc strong-decay out", stored_bf16=True)
    assert_prefill_close(to_host(fin), rf, "noalloc strong-decay final state")
    bad_cu = torch.tensor([0, 200, 150], dtype=torch.int32, device="cuda")  # not monotone
    kda.mixer_fwd_noalloc(*args, bad_cu, N=w.N)
    with pytest.raises(kda.KdaError) as err:
        kda.noalloc_status()
    assert f"0x{kda.DEVFLAG_BAD_SEQLENS:08x}" in str(err.value)
    assert kda.noalloc_status() == 0  # read and cleared
