"""Helpers shared by the GPU parity tests: run the oracle and the CUDA library
on the same seeded inputs and compare.

The metric is max|gpu - ref| / max|ref| per output tensor; the limits are
1e-4 for float32 runs and 2e-2 for bf16-input / float32-accumulate runs.
"""
from __future__ import annotations

import numpy as np
import torch

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def rel_err(got, ref) -> float:
    got = np.asarray(got.detach().float().cpu().numpy() if isinstance(got, torch.Tensor) else got,
                     np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    denom = np.max(np.abs(ref))
    if denom == 0.0:
        return float(np.max(np.abs(got)))
    return float(np.max(np.abs(got - ref)) / denom)


def assert_close(name, got, ref, tol):
    e = rel_err(got, ref)
    assert e <= tol, f"{name}: max|err|/max|ref| = {e:.3e} > {tol:.1e}"
    return e


def oracle_inputs(inp: dict) -> dict:
    """float32 numpy views of the (possibly bf16-rounded) host inputs."""
    return {k: (v.float().numpy() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def to_device(inp: dict, device="cuda") -> dict:
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
