"""Shared helpers for the parity tests: seeded inputs -> device tensors, metrics."""
from __future__ import annotations

import numpy as np

from exact_io_aware_100_b200 import inputs

# Tolerances fixed for this path: bf16 I/O with fp32 accumulation.
MAX_ABS = 2e-2      # O, dQ, dK, dV
REL_L2 = 5e-3       # O, dQ, dK, dV
LSE_ABS = 1e-3      # fp32 logsumexp


def to_device(x: np.ndarray, dtype: str):
    import torch
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def to_f64(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def errors(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = got - ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff) / denom) if denom > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_close(name, got, ref, max_abs=MAX_ABS, rel_l2=REL_L2, scale_max_abs=False):
    """max-abs and relative-L2 bounds.  With scale_max_abs the max-abs bound is
    multiplied by max(1, max|ref|): for stress inputs whose outputs are far from
    unit scale, where a bf16 output ulp alone exceeds the unit-scale bound."""
    if scale_max_abs:
        max_abs = max_abs * max(1.0, float(np.abs(np.asarray(ref)).max()))
    ma, rl = errors(got, ref)
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    assert ma <= max_abs and rl <= rel_l2, f"{name}: max_abs={ma:.3e} rel_l2={rl:.3e}"
    return ma, rl


def assert_close_bwd(name, got, ref, operand_bound, max_abs=MAX_ABS, rel_l2=REL_L2):
    """Gradient check with the error terms the arithmetic itself fixes, per element:
        |got - ref| <= max_abs + 2^-8 |ref| + operand_bound,
    and the relative-L2 bound unchanged.

    2^-8 |ref|: the bf16 output's own rounding (a correctly rounded bf16 value is
    within 2^-8 |x| of x; at |x| >= 8 that alone exceeds a 2e-2 absolute bound).
    operand_bound: the oracle's ``bwd_operand_rounding_bound`` for the same inputs,
    the most that rounding the products' operands P and dS to bf16 can move the
    entry.  Used where gradients reach several units (keys scaled x2, grouped
    heads), where the absolute bound alone is below what bf16 operands allow."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    ma, rl = errors(got, ref)
    excess = np.abs(got - ref) - (max_abs + 2.0 ** -8 * np.abs(ref) + np.asarray(operand_bound, np.float64))
    worst = float(excess.max()) if excess.size else -1.0
    assert worst <= 0 and rl <= rel_l2, f"{name}: max_abs={ma:.3e} rel_l2={rl:.3e} excess={worst:.3e}"
    return ma, rl


def assert_lse(got, ref, tol=LSE_ABS):
    ma = float(np.abs(np.asarray(got, np.float64) - ref).max())
    assert np.isfinite(got).all() and ma <= tol, f"lse: max_abs={ma:.3e}"
    return ma


def make_case(B, H, N, d, seed, k_scale=1.0, dtype="bf16", names=("q", "k", "v")):
    """Seeded inputs of one shape: (host arrays as generated, float64 values)."""
    shape = (B, H, N, d)
    host = {n: inputs.make_tensor(seed, n, shape, k_scale if n == "k" else 1.0, dtype) for n in names}
    f64 = {n: inputs.to_f64(host[n], dtype) for n in names}
    return host, f64
