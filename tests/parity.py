"""Helpers shared by the GPU parity tests: tolerances and tensor plumbing.

Tolerance for the GEMM output Y (bf16) against the oracle's fp64 result R
(the block-scaled GEMM computed exactly from the quantized operands):
  pointwise   |Y - R| <= 4e-3 |R| + 1e-2 rms(R)      (against unrounded R)
  aggregate   ||Y - bf16(R)||_F <= 1e-3 ||bf16(R)||_F
The pointwise bound leaves room for the final bf16 rounding (at most 2^-9
relative, 1.95e-3) plus fp32 accumulation error; the aggregate bound is
taken against the bf16-rounded R, because bf16 rounding alone moves the
Frobenius norm by about 1.7e-3 relative to R.
Quantized codes and scales must match the oracle bit for bit.
"""
import numpy as np
import torch

import oracle
import workloads as wl

PW_REL = 4e-3
PW_RMS = 1e-2
FRO_REL = 1e-3


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return wl.to_torch_bf16(bits).cuda()


def u8(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.uint8).cpu().numpy()


def f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def check_gemm(y: np.ndarray, R: np.ndarray, label: str = "") -> dict:
    """Assert the tolerance above; returns the measured error figures."""
    y = np.asarray(y, dtype=np.float64)
    R = np.asarray(R, dtype=np.float64)
    assert y.shape == R.shape, (y.shape, R.shape)
    assert np.all(np.isfinite(y)), label
    rms = float(np.sqrt(np.mean(R * R))) if R.size else 0.0
    d = np.abs(y - R)
    lim = PW_REL * np.abs(R) + PW_RMS * rms
    worst = float(np.max(d / np.maximum(lim, 1e-300))) if R.size else 0.0
    Rb = oracle.bf16_rne(R)
    nrm = float(np.linalg.norm(Rb))
    fro = float(np.linalg.norm(y - Rb) / nrm) if nrm > 0 else float(np.linalg.norm(y))
    assert np.all(d <= lim), f"{label}: pointwise bound exceeded (worst ratio {worst:.3f})"
    assert fro <= FRO_REL, f"{label}: relative Frobenius {fro:.3e} > {FRO_REL}"
    return {"worst_ratio": worst, "fro_vs_bf16R": fro}
