"""Shared helpers of the GPU parity tests: moving seeded inputs to the device and
the comparison rules.

Tolerances (stated once, used by every parity test):
* index outputs (clusters, neighbour tables, KNN tables): bit-exact;
* bf16 forward outputs: max |gpu - oracle| <= 1e-2 where |oracle| < 4; where
  |oracle| >= 4 a bf16 result cannot be closer than half a bf16 ulp (1/64 in
  [4, 8)), so those few outputs are held to half an ulp + 1e-3 and counted;
* log-sum-exp: max abs error <= 1e-3;
* gradients: max |gpu - oracle| <= 2e-2 * max |oracle| per tensor.
"""
from __future__ import annotations

import os

import numpy as np
import torch

FWD_ATOL = 1e-2
LSE_ATOL = 1e-3
GRAD_RTOL = 2e-2

# forward outputs held to half an ulp instead of FWD_ATOL, per (test, output): reported at
# the end of the session by tests/conftest.py
LARGE_OUTPUTS: dict[str, tuple[int, int]] = {}


def dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def bf16(a: np.ndarray) -> torch.Tensor:
    """float32 array holding bf16 values -> bf16 CUDA tensor (exact)."""
    return dev(a.astype(np.float32), torch.bfloat16)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_fwd(gpu: np.ndarray, ref: np.ndarray, what: str) -> dict:
    err = np.abs(gpu - ref)
    big = np.abs(ref) >= 4.0
    small_err = float(err[~big].max()) if (~big).any() else 0.0
    assert small_err <= FWD_ATOL, f"{what}: max abs err {small_err:.3e} > {FWD_ATOL}"
    if big.any():
        half_ulp = 2.0 ** (np.floor(np.log2(np.abs(ref[big]))) - 8)
        assert np.all(err[big] <= half_ulp + 1e-3), f"{what}: large outputs off by more than half an ulp"
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    n0, m0 = LARGE_OUTPUTS.get(f"{test} {what}", (0, 0))
    LARGE_OUTPUTS[f"{test} {what}"] = (n0 + int(big.sum()), m0 + int(big.size))
    return {"max_abs": small_err, "n_large": int(big.sum())}


def check_grad(gpu: np.ndarray, ref: np.ndarray, what: str) -> float:
    scale = float(np.abs(ref).max())
    err = float(np.abs(gpu - ref).max())
    tol = GRAD_RTOL * max(scale, 1e-30)
    assert err <= tol, f"{what}: max abs err {err:.3e} > {GRAD_RTOL} * {scale:.3e}"
    return err / max(scale, 1e-30)
