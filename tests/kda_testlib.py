"""Helpers shared by the GPU parity tests (inputs, oracle calls, metrics)."""
from __future__ import annotations

import numpy as np
import torch

# Relative-L2 bars: fp32-input workloads and bf16-input workloads.
TOL_FP32 = 1e-5
TOL_BF16 = 2e-3


def tol_for(dtype) -> float:
    return TOL_FP32 if dtype == torch.float32 else TOL_BF16


def f64(t):
    """Exact upcast of the bits a kernel consumed (or produced) to float64."""
    if t is None:
        return None
    return t.detach().to("cpu").to(torch.float64).numpy()


def rel_l2(x, ref) -> float:
    x, ref = np.asarray(x, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def bf16_floor(ref) -> float:
    """Relative-L2 of rounding the float64 reference itself to bfloat16: the
    error floor any bf16 output carries before kernel error is added."""
    r = torch.from_numpy(np.asarray(ref, dtype=np.float64))
    return rel_l2(r.to(torch.bfloat16).to(torch.float64).numpy(), ref)


def to_cuda(inputs: dict) -> dict:
    return {n: (None if t is None else t.cuda()) for n, t in inputs.items()}


def report(name, got, ref, tol, dtype):
    err = rel_l2(got, ref)
    floor = bf16_floor(ref) if dtype == torch.bfloat16 else 0.0
    print(f"{name}: rel_l2={err:.3e} (bf16 floor {floor:.3e}, bar {tol:.0e})")
    assert np.isfinite(np.asarray(got)).all(), f"{name}: non-finite output"
    assert err <= tol, f"{name}: rel_l2 {err:.3e} > {tol:.0e}"
    return err
