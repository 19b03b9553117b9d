"""Shared test utilities: upload seeded workloads to the GPU and compare with the oracle."""
from __future__ import annotations

import numpy as np

# Tolerances, written once and used by every parity test.
PREFILL_TOL = 2e-2      # max |gpu - oracle| <= PREFILL_TOL * RMS(oracle), per tensor
DECODE_TOL = 1e-4       # max |gpu - oracle| <= DECODE_TOL * max|oracle| (fp32 state)
BF16_HALF_ULP = 2.0 ** -8  # relative rounding of one bf16 store (8 significant bits)


def to_device(x, dtype: str, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype == "bf16":
        return t.to(device=device, dtype=torch.bfloat16)
    if dtype == "f32":
        return t.to(device=device, dtype=torch.float32)
    if dtype == "i32":
        return t.to(device=device, dtype=torch.int32)
    raise ValueError(dtype)


def to_host(t) -> np.ndarray:
    import torch
    return t.detach().to(dtype=torch.float64, device="cpu").numpy()


def rms(x) -> float:
    return float(np.sqrt(np.mean(np.square(x))))


def assert_prefill_close(got, ref, what: str, stored_bf16: bool = False):
    """max |gpu - oracle| <= PREFILL_TOL * RMS(oracle); a tensor the library stores in
    bf16 additionally carries that store's rounding, at most half a bf16 ulp
    (<= 2^-8 |x|) per element. Even the exact result, stored in bf16, exceeds the bare
    2e-2 * RMS bar on heavy-tailed outputs (0.0218 * RMS on the 10 x 70-token, 32-head
    case), so the bar applies to the computed value and the store is added to it."""
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    scale = rms(ref)
    bound = PREFILL_TOL * scale + (BF16_HALF_ULP * np.abs(ref) if stored_bf16 else 0.0)
    over = np.abs(got - ref) - bound
    err = float(np.max(np.abs(got - ref)))
    assert np.all(over <= 0), (f"{what}: max|err|={err:.3e} ({err / scale:.4f} RMS), worst excess over the "
                               f"bound {float(np.max(over)):.3e}")
    return err / scale


def assert_decode_state_close(got, ref, what: str):
    err = float(np.max(np.abs(got - ref)))
    scale = float(np.max(np.abs(ref)))
    assert err <= DECODE_TOL * scale, f"{what}: max|err|={err:.3e} > {DECODE_TOL}*max|ref|={DECODE_TOL * scale:.3e}"
    return err / scale


def assert_decode_out_close(got, ref, what: str):
    # fp32 arithmetic within DECODE_TOL, plus the rounding of the bf16 store
    bound = DECODE_TOL * np.max(np.abs(ref)) + BF16_HALF_ULP * np.abs(ref) * 1.0001
    over = np.abs(got - ref) - bound
    assert np.all(over <= 0), f"{what}: worst excess {float(np.max(over)):.3e}"


# The backward runs token by token in fp32. Per step each gradient element is a sum of at
# most 2 x 128 fp32 products (unit roundoff 2^-24 ~ 6e-8, so <= 1.5e-5 relative per step
# in the worst case), and the gradient of the state is carried through maps of norm <= 1
# (alpha <= 1, beta in (0, 1), |k| = 1), so rounding adds up at most linearly along a
# sequence: T x 1.5e-5 bounds it (1.5e-3 at 100 tokens) and random signs make it grow like
# sqrt(T). 1e-3 of the largest magnitude holds every case tested here with room, while a
# dropped term, a wrong sign or a transposed operand moves gradients by O(1) of it.
BWD_TOL = 1e-3


def assert_backward_close(got, ref, what: str):
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = float(np.max(np.abs(got - ref)))
    scale = float(np.max(np.abs(ref)))
    assert err <= BWD_TOL * scale, f"{what}: max|err|={err:.3e} > {BWD_TOL}*max|ref|={BWD_TOL * scale:.3e}"
    return err / scale
