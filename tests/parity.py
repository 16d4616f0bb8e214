"""Shared helpers of the GPU parity tests: tolerances and host/device conversion.

Tolerances (stated for the path as a whole): every floating-point output tensor
has max |err| <= 2e-2 x RMS(oracle tensor); every final DeltaNet state has
relative Frobenius error <= 1e-2; integer / index / bit-copy outputs are exact.

Per-kernel tests of steps whose output is stored in bf16 add an elementwise
term BF16_ELEM x |oracle| to the bound: storing a value in bf16 alone moves it
by up to 2^-9 of its magnitude, and a heavy-tailed intermediate (a SwiGLU
product, an attention output over few keys) can hold values far above its RMS.
2^-8 allows that storage rounding plus the bf16 rounding of one operand.
"""
import numpy as np
import torch

TOL_RMS = 2e-2
TOL_STATE = 1e-2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


BF16_ELEM = 2.0 ** -8


def assert_rms_close(got, want, tol=TOL_RMS, what="", elem=0.0, scale=None):
    """max over elements of |got - want| - elem * scale <= tol * RMS(want);
    scale defaults to |want| (the magnitude the stored value is rounded at)."""
    got = f64(got) if isinstance(got, torch.Tensor) else np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    rms = float(np.sqrt(np.mean(want * want)))
    if not got.size:
        return 0.0
    sc = np.abs(want) if scale is None else np.asarray(scale, dtype=np.float64)
    excess = np.abs(got - want) - elem * sc
    i = int(np.argmax(excess))
    err = float(np.abs(got - want).flat[i])
    assert excess.flat[i] <= tol * rms, (
        f"{what}: err {err:.3e} at {np.unravel_index(i, got.shape)} (want {want.flat[i]:.4g}) "
        f"> {tol} x rms {rms:.3e} + {elem:.3g} x |want|")
    return float(np.max(np.abs(got - want))) / rms if rms > 0 else 0.0


def assert_state_close(got, want, tol=TOL_STATE, what="state"):
    got = f64(got) if isinstance(got, torch.Tensor) else np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    # relative Frobenius error per state matrix (last two axes)
    num = np.sqrt(np.sum((got - want) ** 2, axis=(-2, -1)))
    den = np.sqrt(np.sum(want ** 2, axis=(-2, -1)))
    rel = num / np.maximum(den, 1e-30)
    worst = float(rel.max())
    assert worst <= tol, f"{what}: worst relative Frobenius error {worst:.3e} > {tol}"
    return worst


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 (what the device stores)."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()
