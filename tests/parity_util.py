"""Comparison helpers shared by the GPU parity tests (no attention arithmetic here)."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances of the GPU path against the fp64 oracle (bf16 inputs, fp32 accumulate):
O_MAX_ABS = 1e-2
O_REL_FRO = 5e-3
GRAD_REL_FRO = 1e-2


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rel_fro(got: np.ndarray, ref: np.ndarray) -> float:
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def max_abs(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.max(np.abs(got - ref))) if got.size else 0.0


def report(name: str, got: np.ndarray, ref: np.ndarray) -> str:
    idx = np.unravel_index(np.argmax(np.abs(got - ref)), got.shape) if got.size else ()
    return (f"{name}: max_abs={max_abs(got, ref):.3e} rel_fro={rel_fro(got, ref):.3e} "
            f"worst@{tuple(int(i) for i in idx)} got={got[idx] if got.size else 0:.5f} "
            f"ref={ref[idx] if got.size else 0:.5f}")


def check_o(got, ref, what=""):
    msg = report("O" + what, got, ref)
    assert max_abs(got, ref) <= O_MAX_ABS and rel_fro(got, ref) <= O_REL_FRO, msg
    return msg


def check_grad(name, got, ref, what=""):
    msg = report(name + what, got, ref)
    assert rel_fro(got, ref) <= GRAD_REL_FRO, msg
    return msg
