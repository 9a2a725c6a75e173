"""Comparison rules shared by the parity tests.

fp32 outputs:  |y - y_ref| <= 1e-5 * (1 + |y_ref|)               (elementwise)
bf16 outputs:  |y - y_ref| <= ulp_bf16(y_ref) + 1e-5 * (1 + |y_ref|)
               (one bf16 unit in the last place of the exact value; the second term only
               matters where |y_ref| is so small that one bf16 ulp is below the fp32
               accumulation error). The strict one-ulp count is reported as well.
States are compared through what the (a, b, p) representation leaves unique:
               rho = a / b and lambda = p + ln b, each within 1e-5 * (1 + |ref|).
Reductions (dw, du) over n terms: |d - d_ref| <= 1e-5 * (1 + sum |terms|).
Gradients dk, dv (each a sum over the later tokens a token reaches, plus the current
               token's term): |d - d_ref| <= 1e-5 * (1 + sum |terms|) elementwise, with
               sum |terms| the oracle's dk_abs, dv_abs. Where the terms do not cancel this
               is the fp32 rule; where they do, a float evaluation rounds at the size of
               the terms, not of their difference. dr (a product) keeps the fp32 rule.
"""
import numpy as np

FP32_TOL = 1e-5


def fp32_bad(y, ref, tol=FP32_TOL):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(y - ref)
    bound = tol * (1.0 + np.abs(ref))
    bad = ~(err <= bound)
    return bad, err, bound


def assert_fp32_close(y, ref, what="y", tol=FP32_TOL):
    bad, err, bound = fp32_bad(y, ref, tol)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err / np.maximum(bound, 1e-300), 0)),
                             err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements outside 1e-5*(1+|ref|); worst at "
            f"{tuple(int(x) for x in i)}: got {np.asarray(y)[i]!r}, ref {np.asarray(ref)[i]!r}")
    return float((err / np.maximum(bound, 1e-300)).max()) if err.size else 0.0


def assert_grad_close(got, ref, ref_abs, what, tol=FP32_TOL):
    """dk / dv against the oracle, bounded by the size of their terms; returns the worst
    error as a fraction of the bound."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    bound = tol * (1.0 + np.asarray(ref_abs, dtype=np.float64))
    bad = ~(err <= bound)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err / bound, 0)), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements outside 1e-5*(1+sum|terms|); "
            f"worst at {tuple(int(x) for x in i)}: got {got[i]!r}, ref {ref[i]!r}, "
            f"sum|terms| {float(np.asarray(ref_abs)[i])!r}")
    return float((err / bound).max()) if err.size else 0.0


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (8 significant bits), for normal |x|."""
    ax = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    e = np.floor(np.log2(ax))
    return 2.0 ** (e - 7)


def assert_bf16_close(y_bf16_as_f32, ref, what="y"):
    y = np.asarray(y_bf16_as_f32, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(y - ref)
    ulp = bf16_ulp(ref)
    bound = ulp + FP32_TOL * (1.0 + np.abs(ref))
    bad = ~(err <= bound)
    strict = int((~(err <= ulp)).sum())
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err / bound, 0)), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} bf16 outputs beyond 1 ulp + 1e-5(1+|ref|);"
            f" worst at {tuple(int(x) for x in i)}: got {y[i]!r}, ref {ref[i]!r}")
    return {"strict_1ulp_violations": strict, "n": int(y.size),
            "max_err_in_ulps": float((err / ulp).max()) if y.size else 0.0}


def assert_state_close(a, b, p, A_ref, B_ref, what="state", tol=FP32_TOL):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    p = np.asarray(p, dtype=np.float64)
    rho, rho_ref = a / b, np.asarray(A_ref) / np.asarray(B_ref)
    lam, lam_ref = p + np.log(b), np.log(np.asarray(B_ref))
    assert_fp32_close(rho, rho_ref, what + ".a/b", tol)
    assert_fp32_close(lam, lam_ref, what + ".p+ln(b)", tol)
