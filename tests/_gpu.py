"""Helpers for the GPU parity tests: move seeded problems to the device, run the library
through its C ABI binding, and compare with the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import bit_weight_only_w2_b200 as lb

# Per-element bound: |gpu - ref| <= RTOL * |ref| + ATOL_RMS * rms(ref), ref = fp64 oracle.
RTOL = 1e-2
ATOL_RMS = 1e-2


def dev_problem(prob, device="cuda"):
    """Device tensors for a synth.Problem; W packed on the GPU by the library."""
    codes = torch.from_numpy(prob.codes).to(device)
    packed = lb.pack(codes, prob.spec.bits)
    x = None
    if prob.x_bf16 is not None:
        x = torch.from_numpy(prob.x_bf16.view(np.int16)).to(device).view(torch.bfloat16)
    s = torch.from_numpy(prob.scales).to(device)
    z = torch.from_numpy(prob.zeros).to(device) if prob.zeros is not None else None
    return x, packed, s, z


def oracle_packed(prob):
    p, bad = oracle.pack(prob.codes, prob.spec.bits)
    assert bad == 0
    return p


def y_to_f64(y: torch.Tensor) -> np.ndarray:
    return y.float().cpu().numpy().astype(np.float64)


def check_close(got: np.ndarray, ref: np.ndarray, rms: float | None = None, what: str = ""):
    if rms is None:
        rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    err = np.abs(got - ref)
    bound = RTOL * np.abs(ref) + ATOL_RMS * rms
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        worst = float(np.max(err / np.maximum(bound, 1e-300)))
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance "
                             f"(worst err/bound {worst:.3f}); first at {idx.tolist()}")
    return float(np.max(err / np.maximum(bound, 1e-300))) if err.size else 0.0
