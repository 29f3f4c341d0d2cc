"""Comparison helpers for the GPU-vs-oracle parity tests."""

import numpy as np

from exact_attention_137_b200.workloads import to_f64

# bf16 inputs, fp32 accumulation: max |dO| <= 2e-2, mean |dO| <= 2e-3, |dLSE| <= 1e-3.
BF16_TOL = dict(max_o=2e-2, mean_o=2e-3, lse=1e-3)
# fp32 inputs and arithmetic: max error <= 1e-4.
F32_TOL = dict(max_o=1e-4, mean_o=1e-4, lse=1e-4)


def compare(o, lse, o_ref, lse_ref, tol, what=""):
    """Element-wise comparison; -inf LSE entries (rows with no visible key) must match exactly."""
    o = to_f64(o)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    d = np.abs(o - o_ref)
    stats = dict(max_o=float(d.max(initial=0.0)), mean_o=float(d.mean()) if d.size else 0.0)
    if lse is not None:
        lse = to_f64(lse)
        lse_ref = np.asarray(lse_ref, dtype=np.float64)
        neg = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(lse), neg), f"{what}: -inf LSE rows differ"
        dl = np.abs(lse[~neg] - lse_ref[~neg])
        stats["lse"] = float(dl.max(initial=0.0))
    assert stats["max_o"] <= tol["max_o"], f"{what}: max |dO| {stats}"
    assert stats["mean_o"] <= tol["mean_o"], f"{what}: mean |dO| {stats}"
    if lse is not None:
        assert stats["lse"] <= tol["lse"], f"{what}: max |dLSE| {stats}"
    return stats


# Gradients (bf16 in and out, fp32 accumulation, P and dS rounded to bf16 as MMA operands,
# O rounded to bf16 by the forward): errors are judged relative to the reference's size.
GRAD_TOL = dict(max_rel=2e-2, mean_rel=1e-2)


def compare_grad(got, ref, tol=GRAD_TOL, what=""):
    """max|d| / max|ref| and mean|d| / mean|ref| within tolerance."""
    got = to_f64(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite gradient"
    d = np.abs(got - ref)
    scale_max = max(float(np.abs(ref).max(initial=0.0)), 1e-30)
    scale_mean = max(float(np.abs(ref).mean()) if ref.size else 0.0, 1e-30)
    stats = dict(max_rel=float(d.max(initial=0.0)) / scale_max, mean_rel=(float(d.mean()) if d.size else 0.0) / scale_mean)
    assert stats["max_rel"] <= tol["max_rel"], f"{what}: {stats}"
    assert stats["mean_rel"] <= tol["mean_rel"], f"{what}: {stats}"
    return stats
