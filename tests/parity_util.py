"""Helpers for GPU-vs-oracle parity tests: tolerances and comparisons."""

import numpy as np
import torch

# y: max-abs error bounds; S, z: max|diff| / max|ref| bounds.
Y_TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}
STATE_TOL = {torch.float32: 1e-5, torch.bfloat16: 1e-2}


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64))))


def assert_y(got, ref, dtype, what="y"):
    err = max_abs(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err <= Y_TOL[dtype], f"{what}: max-abs error {err:.3e} > {Y_TOL[dtype]:.0e}"
    return err


def assert_state(got, ref, dtype, what="S"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite state"
    rel = max_abs(got, ref) / max(1e-30, float(np.max(np.abs(ref))))
    assert rel <= STATE_TOL[dtype], f"{what}: relative error {rel:.3e} > {STATE_TOL[dtype]:.0e}"
    return rel
