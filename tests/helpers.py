"""Shared test utilities: device transfer of synthetic inputs and the parity
criteria of the layer.

Tolerance (GEMM outputs against the fp64 oracle, which is not rounded):
  relative Frobenius error  ||Y - Yref||_F / ||Yref||_F  <= 5e-3, and
  every element             |Y - Yref| <= 2e-2 * (|Yref| + rms(Yref)).
Dequantized weights and the exact-integer regime are compared bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch

FROB_TOL = 5e-3
ELEM_TOL = 2e-2


def bf16_tensor(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bits_of_bf16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().double().numpy()


def parity(y: np.ndarray, ref: np.ndarray) -> tuple[float, float]:
    """(relative Frobenius error, worst element ratio to its bound)."""
    diff = y - ref
    rms = float(np.sqrt(np.mean(ref * ref)))
    frob = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    bound = ELEM_TOL * (np.abs(ref) + rms)
    worst = float(np.max(np.abs(diff) / np.maximum(bound, 1e-300)))
    return frob, worst


def assert_parity(y: np.ndarray, ref: np.ndarray, what: str = "") -> None:
    frob, worst = parity(y, ref)
    assert frob <= FROB_TOL, f"{what}: relative Frobenius error {frob:.3e} > {FROB_TOL}"
    assert worst <= 1.0, f"{what}: an element exceeds 2e-2*(|ref|+rms) by x{worst:.2f}"


def assert_sampled_parity(y_samples: np.ndarray, ref_samples: np.ndarray, rms_ref: float,
                          what: str = "") -> None:
    """Element bound on sampled outputs, with rms taken from the samples."""
    diff = y_samples - ref_samples
    bound = ELEM_TOL * (np.abs(ref_samples) + rms_ref)
    worst = float(np.max(np.abs(diff) / bound))
    frob = float(np.linalg.norm(diff) / max(np.linalg.norm(ref_samples), 1e-300))
    assert frob <= FROB_TOL, f"{what}: sampled relative error {frob:.3e}"
    assert worst <= 1.0, f"{what}: a sampled element exceeds its bound by x{worst:.2f}"
