"""Shared parity helpers for the GPU tests: tolerances, error metrics, and the
packing of decode steps into the oracle's packed-sequence layout.

Tolerances (gated delta rule, bf16 inputs): output max|o - o_ref| / rms(o_ref)
<= 1e-2 and final-state relative Frobenius error <= 1e-3 per sequence; fp32
inputs: <= 1e-4 for both. The oracle is always fed the exact values the
kernel consumed (bf16 values upcast exactly).
"""
import numpy as np
import torch

O_TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-4}
S_TOL = {torch.bfloat16: 1e-3, torch.float32: 1e-4}


def f64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def o_err(o, o_ref):
    o, o_ref = f64(o), f64(o_ref)
    rms = np.sqrt(np.mean(o_ref ** 2))
    return float(np.max(np.abs(o - o_ref)) / rms)


def state_err(S, S_ref):
    """Max over sequences of ||S - S_ref||_F / ||S_ref||_F; S is [N, ...]."""
    S, S_ref = f64(S), f64(S_ref)
    N = S.shape[0]
    d = (S - S_ref).reshape(N, -1)
    r = S_ref.reshape(N, -1)
    return float(np.max(np.linalg.norm(d, axis=1) / np.linalg.norm(r, axis=1)))


def bf16_out_bound(o_ref):
    """Extra allowance when the output itself is stored in bf16: half a bf16
    ulp of |o_ref| (2^-8 relative covers it), as a fraction of rms(o_ref)."""
    o_ref = f64(o_ref)
    return float(np.max(np.abs(o_ref)) * 2.0 ** -8 / np.sqrt(np.mean(o_ref ** 2)))


def close_elementwise(got, ref, rtol, atol):
    got, ref = f64(got), f64(ref)
    bad = np.abs(got - ref) > rtol * np.abs(ref) + atol
    return int(bad.sum()), float(np.max(np.abs(got - ref)))
