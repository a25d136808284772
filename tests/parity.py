"""Comparison rules for the CUDA path against the fp64 oracle.

Tolerances (written here, used by every GPU parity test):
  * fp32 storage: relative L2 error <= 1e-5 against the fp64 result.
  * fp16 / bf16 storage: the oracle's y is first rounded to the storage dtype
    (round-to-nearest-even, the rounding the kernel's own store applies), then
    relative L2 <= 2e-3 and, element by element,
        |y - ref| <= max(1e-2 * RMS(ref), 1 ulp of the storage dtype at |ref|).
    The ulp term is needed because one output ulp at the largest values
    (|y| ~ 20 RMS) already exceeds 1e-2 RMS for bf16: a kernel whose fp32
    result lands half an ulp off a rounding boundary of the oracle's value
    rounds to the neighbouring representable number.
"""
from __future__ import annotations

import numpy as np
import torch

TOL_F32_REL = 1e-5
TOL_16_REL = 2e-3
TOL_16_MAXABS_RMS = 1e-2


def round_to(ref64: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    return torch.from_numpy(ref64).to(dtype).double().numpy()


def ulp(x: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    mant = {torch.float16: 10, torch.bfloat16: 7, torch.float32: 23}[dtype]
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    e = np.maximum(e, {torch.float16: -14, torch.bfloat16: -126, torch.float32: -126}[dtype])
    return np.exp2(e - mant)


def compare(y: torch.Tensor, ref64: np.ndarray, dtype: torch.dtype) -> dict:
    """Return the error figures and whether they pass the rules above."""
    got = y.detach().double().cpu().numpy()
    assert got.shape == ref64.shape, (got.shape, ref64.shape)
    assert np.all(np.isfinite(got)), "non-finite output"
    if dtype == torch.float32:
        rel = float(np.linalg.norm(got - ref64) / max(np.linalg.norm(ref64), 1e-300))
        return {"rel_l2": rel, "ok": rel <= TOL_F32_REL}
    ref = round_to(ref64, dtype)
    diff = np.abs(got - ref)
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    rms = float(np.sqrt(np.mean(ref ** 2)))
    bound = np.maximum(TOL_16_MAXABS_RMS * rms, ulp(ref, dtype))
    worst = float(np.max(diff / bound)) if diff.size else 0.0
    raw_rel = float(np.linalg.norm(got - ref64) / max(np.linalg.norm(ref64), 1e-300))
    return {"rel_l2": rel, "raw_rel_l2": raw_rel, "max_abs": float(diff.max(initial=0.0)),
            "rms": rms, "worst_over_bound": worst, "ok": rel <= TOL_16_REL and worst <= 1.0}


def assert_close(y, ref64, dtype, what=""):
    r = compare(y, ref64, dtype)
    assert r["ok"], f"{what}: {r}"
    return r
