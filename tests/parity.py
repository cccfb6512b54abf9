"""Helpers for GPU-vs-oracle parity tests.

The floating-point bar, elementwise:
  |gpu - ref| <= max(1e-5 * max(|ref|, 1e-3 * rms(ref)), 2^-22 * max|ref|)
- max relative error 1e-5, with a floor for values that cross zero;
- plus 4 units in the last place of the array's largest magnitude: a value
  that comes out of a cancellation (a weight stepped to near zero, a sum of
  terms of both signs) keeps the absolute rounding of its operands, which
  are as large as the array's values; two correct implementations that
  round an operand differently (an fp64 sum taken in another order, rounded
  to fp32) differ by that much.  The term decides only for values below
  about 2% of the array's largest.
Integer results (key packing, key -> offset maps) must be equal.
"""
from __future__ import annotations

import numpy as np
import torch

REL = 1e-5
FLOOR = 1e-3
ULPS_OF_MAX = 2.0 ** -22  # 4 ulp of fp32 at the array's largest magnitude


def close_report(gpu: np.ndarray, ref: np.ndarray) -> dict:
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    if ref.size == 0:
        return dict(ok=True, max_abs=0.0, max_rel=0.0, exact=1.0, n=0)
    finite = np.isfinite(ref)
    rms = float(np.sqrt(np.mean(ref[finite] ** 2))) if finite.any() else 0.0
    top = float(np.max(np.abs(ref[finite]))) if finite.any() else 0.0
    bound = np.maximum(REL * np.maximum(np.abs(ref), FLOOR * rms), ULPS_OF_MAX * top)
    diff = np.abs(gpu - ref)
    ok = bool(np.all((diff <= bound) | (np.isnan(gpu) & np.isnan(ref))))
    rel = diff / np.maximum(np.abs(ref), 1e-30)
    return dict(ok=ok, max_abs=float(np.nanmax(diff)), max_rel=float(np.nanmax(rel)),
                exact=float(np.mean(gpu == ref)), n=int(ref.size))


def assert_close(gpu, ref, what=""):
    r = close_report(gpu, ref)
    assert r["ok"], f"{what}: {r}"
    return r


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()
