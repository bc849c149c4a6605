"""Comparison helpers for the parity tests (tolerances from the targets:
max|dO| <= 1e-2, mean|dO| <= 1e-3, |dLSE| <= 1e-3, rel-L2 of dQ/dK/dV <= 2e-2)."""

import numpy as np

O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3
GRAD_REL_L2 = 2e-2


def o_errors(o_gpu, o_ref):
    d = np.abs(np.asarray(o_gpu, np.float64) - np.asarray(o_ref, np.float64))
    return float(d.max()) if d.size else 0.0, float(d.mean()) if d.size else 0.0


def assert_o_close(o_gpu, o_ref, what="O"):
    mx, mean = o_errors(o_gpu, o_ref)
    assert mx <= O_MAX_ABS, f"{what}: max|diff| {mx:.3e} > {O_MAX_ABS}"
    assert mean <= O_MEAN_ABS, f"{what}: mean|diff| {mean:.3e} > {O_MEAN_ABS}"
    return mx, mean


def assert_lse_close(lse_gpu, lse_ref, what="LSE"):
    a = np.asarray(lse_gpu, np.float64)
    b = np.asarray(lse_ref, np.float64)
    inf_a, inf_b = np.isneginf(a), np.isneginf(b)
    assert np.array_equal(inf_a, inf_b), f"{what}: -inf pattern differs ({inf_a.sum()} vs {inf_b.sum()})"
    fin = ~inf_b
    mx = float(np.abs(a[fin] - b[fin]).max()) if fin.any() else 0.0
    assert mx <= LSE_MAX_ABS, f"{what}: max|diff| {mx:.3e} > {LSE_MAX_ABS}"
    return mx


def rel_l2(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / n) if n > 0 else float(np.linalg.norm(x))


def assert_grad_close(x, ref, what):
    r = rel_l2(x, ref)
    assert r <= GRAD_REL_L2, f"{what}: rel-L2 {r:.3e} > {GRAD_REL_L2}"
    return r
