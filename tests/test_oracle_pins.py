"""Pins for the fp64 oracle: each test ties it to something other than itself.

The pages print no worked numeric example, so the oracle is pinned by: two independent
forms of the same definition (parallel sum vs recurrence), a textbook library route
(SciPy softmax), closed forms for special cases, exact rational arithmetic, invariants
(a convex combination stays within the range of its points) and finite differences.
A plausible slip in the oracle (a dropped current-token term, a decay that starts one
step early or late, a sign of w, u on the wrong term, a transposed index, a wrong
gradient accumulator order) fails at least one of these.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
import wkv_inputs


def _rand(B, T, C, seed, k_std=1.0, logw=(-3.0, 1.0)):
    g = np.random.Generator(np.random.PCG64(seed))
    w = np.exp(g.uniform(*logw, size=C))
    u = g.uniform(-1, 1, size=C)
    k = g.normal(0, k_std, size=(B, T, C))
    v = g.standard_normal((B, T, C))
    r = g.standard_normal((B, T, C))
    return w, u, k, v, r


def test_parallel_form_equals_recurrence():
    # "关键设计 2" gives both forms of the same operator.
    w, u, k, v, r = _rand(3, 40, 7, 1)
    y1 = oracle.wkv_direct(w, u, k, v, r)
    y2 = oracle.wkv_recurrent(w, u, k, v, r)
    np.testing.assert_allclose(y1, y2, rtol=1e-12, atol=1e-13)


def test_parallel_form_equals_recurrence_with_initial_state():
    w, u, k, v, r = _rand(2, 25, 5, 2)
    g = np.random.Generator(np.random.PCG64(3))
    A0 = g.standard_normal((2, 5)) * 3.0
    B0 = g.uniform(0.5, 4.0, size=(2, 5))
    y1 = oracle.wkv_direct(w, u, k, v, r, A0, B0)
    y2 = oracle.wkv_recurrent(w, u, k, v, r, A0, B0)
    np.testing.assert_allclose(y1, y2, rtol=1e-12, atol=1e-13)


def test_matches_scipy_softmax_route():
    # The operator as causal attention with logits k_i - (t-1-i)w and u + k_t.
    w, u, k, v, _ = _rand(1, 12, 4, 4, k_std=2.0)
    ys = oracle.wkv_softmax_form(w, u, k[0], v[0])
    yd = oracle.wkv_direct(w, u, k, v)[0]
    np.testing.assert_allclose(yd, ys, rtol=1e-12, atol=1e-13)


def test_single_token_gives_v():
    w, u, k, v, _ = _rand(4, 1, 9, 5, k_std=5.0)
    for f in (oracle.wkv_direct, oracle.wkv_recurrent):
        np.testing.assert_allclose(f(w, u, k, v), v, rtol=1e-15, atol=0)


def test_constant_value_is_reproduced():
    w, u, k, _, _ = _rand(2, 30, 6, 6, k_std=3.0)
    v = np.broadcast_to(np.linspace(-2, 2, 6), (2, 30, 6)).copy()
    for f in (oracle.wkv_direct, oracle.wkv_recurrent):
        np.testing.assert_allclose(f(w, u, k, v), v, rtol=1e-14, atol=1e-15)


def test_output_within_prefix_range():
    w, u, k, v, _ = _rand(2, 50, 8, 7, k_std=3.0)
    y = oracle.wkv_recurrent(w, u, k, v)
    lo = np.minimum.accumulate(v, axis=1)
    hi = np.maximum.accumulate(v, axis=1)
    eps = 1e-12
    assert np.all(y >= lo - eps) and np.all(y <= hi + eps)


def test_gate_multiplies_by_sigmoid():
    w, u, k, v, r = _rand(1, 10, 3, 8)
    np.testing.assert_allclose(oracle.wkv_direct(w, u, k, v, r),
                               oracle.wkv_direct(w, u, k, v) / (1 + np.exp(-r)), rtol=1e-14)


def test_fast_decay_leaves_last_two_tokens():
    # w -> large: every token older than i = t-1 is forgotten (the most recent past token
    # is not decayed: exponent -(t-1-i)w is zero for i = t-1).
    _, u, k, v, _ = _rand(2, 20, 5, 9)
    w = np.full(5, 80.0)
    y = oracle.wkv_recurrent(w, u, k, v)
    ek_prev, ecur = np.exp(k[:, :-1]), np.exp(u + k[:, 1:])
    want = (ek_prev * v[:, :-1] + ecur * v[:, 1:]) / (ek_prev + ecur)
    np.testing.assert_allclose(y[:, 1:], want, rtol=1e-13)
    np.testing.assert_allclose(y[:, 0], v[:, 0], rtol=1e-15)


def test_huge_bonus_gives_current_value():
    w, _, k, v, _ = _rand(1, 15, 4, 10)
    u = np.full(4, 60.0)
    np.testing.assert_allclose(oracle.wkv_direct(w, u, k, v), v, rtol=1e-12, atol=1e-12)


def test_no_decay_is_prefix_weighted_mean():
    # w -> 0: a softmax-weighted mean over the whole prefix, by cumulative sums.
    _, u, k, v, _ = _rand(2, 30, 3, 11)
    w = np.full(3, 1e-14)
    y = oracle.wkv_direct(w, u, k, v)
    ek = np.exp(k)
    past_num = np.cumsum(ek * v, axis=1) - ek * v
    past_den = np.cumsum(ek, axis=1) - ek
    cur = np.exp(u + k)
    want = (past_num + cur * v) / (past_den + cur)
    np.testing.assert_allclose(y, want, rtol=1e-11)


@pytest.mark.parametrize("j", [0, 3, 9])
def test_geometric_closed_form(j):
    # k constant and v a unit impulse at token j: the weights are a geometric sequence.
    T, C = 14, 3
    w = np.array([0.05, 0.7, 2.5])
    u = np.array([-0.4, 0.3, 1.1])
    k = np.full((1, T, C), 1.7)
    v = np.zeros((1, T, C))
    v[0, j, :] = 1.0
    y = oracle.wkv_recurrent(w, u, k, v)[0]
    for t in range(T):                      # 0-based t; token t has t past tokens
        past = (1 - np.exp(-t * w)) / (1 - np.exp(-w))   # sum_{m=0}^{t-1} e^{-m w}
        den = past + np.exp(u)
        if t < j:
            want = np.zeros(C)
        elif t == j:
            want = np.exp(u) / den
        else:
            want = np.exp(-(t - 1 - j) * w) / den
        np.testing.assert_allclose(y[t], want, rtol=1e-12, atol=1e-15)


def test_exact_rational_example():
    # e^{-w} = 1/2, e^{u} = 3, e^{k_i} = i + 1: every weight is rational.
    T = 7
    vs = [3, -1, 4, 1, -5, 9, 2]
    half = Fraction(1, 2)
    want = []
    for t in range(T):
        num = sum(half ** (t - 1 - i) * (i + 1) * vs[i] for i in range(t))
        den = sum(half ** (t - 1 - i) * (i + 1) for i in range(t))
        num += 3 * (t + 1) * vs[t]
        den += 3 * (t + 1)
        want.append(num / den)
    w = np.array([math.log(2.0)])
    u = np.array([math.log(3.0)])
    k = np.log(np.arange(1, T + 1, dtype=np.float64)).reshape(1, T, 1)
    v = np.array(vs, dtype=np.float64).reshape(1, T, 1)
    for f in (oracle.wkv_direct, oracle.wkv_recurrent):
        y = f(w, u, k, v)[0, :, 0]
        np.testing.assert_allclose(y, [float(q) for q in want], rtol=1e-14)


def test_split_invariance_of_state():
    # Encoding a sequence in two segments and handing the state over gives the same
    # output and final state as one pass.
    w, u, k, v, r = _rand(2, 33, 4, 12)
    y, A, Bd = oracle.wkv_recurrent(w, u, k, v, r, want_state=True)
    y1, A1, B1 = oracle.wkv_recurrent(w, u, k[:, :20], v[:, :20], r[:, :20], want_state=True)
    y2 = oracle.wkv_direct(w, u, k[:, 20:], v[:, 20:], r[:, 20:], A1, B1)
    _, A2, B2 = oracle.wkv_recurrent(w, u, k[:, 20:], v[:, 20:], r[:, 20:], A1, B1,
                                     want_state=True)
    np.testing.assert_allclose(np.concatenate([y1, y2], axis=1), y, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(A2, A, rtol=1e-12)
    np.testing.assert_allclose(B2, Bd, rtol=1e-12)


def test_decode_steps_reproduce_forward():
    w, u, k, v, r = _rand(3, 12, 5, 13)
    y = oracle.wkv_direct(w, u, k, v, r)
    A = np.zeros((3, 1, 5))
    Bd = np.zeros((3, 1, 5))
    for t in range(12):
        yt, A, Bd = oracle.wkv_decode(w[None], u[None], k[:, t:t + 1], v[:, t:t + 1],
                                      r[:, t:t + 1], A, Bd)
        np.testing.assert_allclose(yt[:, 0], y[:, t], rtol=1e-12, atol=1e-13)


def test_decode_matches_single_step_restatement():
    d = wkv_inputs.decode_batch(seed=3, N=4, L=3, C=8)
    A, Bd = oracle.state_from_scaled(d.a, d.b, d.p)
    k, v, r = d.step(0)
    y, A1, B1 = oracle.wkv_decode(d.w, d.u, k, v, None, A, Bd)
    for n in range(4):
        for l in range(3):
            yy, (na, nb) = oracle.wkv_single_step(d.w[l], d.u[l], k[n, l], v[n, l],
                                                  (A[n, l], Bd[n, l]))
            np.testing.assert_allclose(y[n, l], yy, rtol=1e-13)
            np.testing.assert_allclose(A1[n, l], na, rtol=1e-13)
            np.testing.assert_allclose(B1[n, l], nb, rtol=1e-13)


def _loss(w, u, k, v, r, dy):
    return float(np.sum(oracle.wkv_direct(w, u, k, v, r) * dy))


@pytest.mark.parametrize("gate", [True, False])
def test_backward_matches_central_differences(gate):
    B, T, C = 2, 8, 3
    w, u, k, v, r = _rand(B, T, C, 14)
    if not gate:
        r = None
    dy = np.random.Generator(np.random.PCG64(15)).standard_normal((B, T, C))
    g = oracle.wkv_backward(w, u, k, v, r, dy)
    h = 1e-6

    def fd(name, arr, idx):
        plus = {"w": w, "u": u, "k": k, "v": v, "r": r}
        a1 = arr.copy(); a1[idx] += h
        a2 = arr.copy(); a2[idx] -= h
        plus[name] = a1
        lp = _loss(plus["w"], plus["u"], plus["k"], plus["v"], plus["r"], dy)
        plus[name] = a2
        lm = _loss(plus["w"], plus["u"], plus["k"], plus["v"], plus["r"], dy)
        return (lp - lm) / (2 * h)

    for name, arr, grad in (("k", k, g["dk"]), ("v", v, g["dv"])):
        for idx in np.ndindex(arr.shape):
            assert fd(name, arr, idx) == pytest.approx(grad[idx], rel=1e-6, abs=1e-8), \
                (name, idx)
    for name, arr, grad in (("w", w, g["dw"]), ("u", u, g["du"])):
        for c in range(C):
            assert fd(name, arr, (c,)) == pytest.approx(grad[c], rel=1e-6, abs=1e-8), \
                (name, c)
    if gate:
        for idx in np.ndindex(r.shape):
            assert fd("r", r, idx) == pytest.approx(g["dr"][idx], rel=1e-6, abs=1e-8)
    else:
        assert g["dr"] is None
    assert np.all(g["dw_abs"] >= np.abs(g["dw"])) and np.all(g["du_abs"] >= np.abs(g["du"]))


def test_spike_inputs_stay_finite_and_in_range():
    # The bf16 workload's k has entries of +60: e^{62} is far inside fp64's range.
    x = wkv_inputs.long_bf16(seed=0, B=1, T=256, C=64)
    y = oracle.wkv_recurrent(x.w, x.u, x.k, x.v)
    assert np.all(np.isfinite(y))
    lo = np.minimum.accumulate(x.v.astype(np.float64), axis=1)
    hi = np.maximum.accumulate(x.v.astype(np.float64), axis=1)
    assert np.all(y >= lo - 1e-12) and np.all(y <= hi + 1e-12)
    yd = oracle.wkv_direct(x.w, x.u, x.k[:, :64], x.v[:, :64])
    np.testing.assert_allclose(yd, y[:, :64], rtol=1e-12, atol=1e-13)


def test_golden_fixture_regression():
    # Values written by tests/golden/make_golden.py from the oracle; keeps the oracle
    # from drifting between commits.
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_forward_seed0.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    x = wkv_inputs.tiny_forward(seed=0)
    y = oracle.wkv_direct(x.w, x.u, x.k, x.v, x.r)
    for b, t, c, val in rows:
        assert y[int(b), int(t), int(c)] == pytest.approx(float(val), rel=1e-13, abs=1e-15)


def _loss_state(w, u, k, v, r, dy, A0, B0, gA, gB):
    y, AT, BT = oracle.wkv_recurrent(w, u, k, v, r, A0, B0, want_state=True)
    return float(np.sum(y * dy) + np.sum(gA * AT) + np.sum(gB * BT))


def test_backward_state_matches_central_differences():
    # The stateful backward (gradients through an entering and a leaving state) against
    # central differences of sum(dy y) + gA A_T + gB B_T computed with the recurrence.
    B, T, C = 2, 7, 3
    w, u, k, v, r = _rand(B, T, C, 31)
    g = np.random.Generator(np.random.PCG64(32))
    dy = g.standard_normal((B, T, C))
    A0 = g.standard_normal((B, C))
    B0 = g.uniform(0.5, 2.0, (B, C))
    gA = g.standard_normal((B, C))
    gB = g.standard_normal((B, C))
    res = oracle.wkv_backward_state(w, u, k, v, r, dy, A0, B0, gA, gB)
    h = 1e-6
    args = {"w": w, "u": u, "k": k, "v": v, "r": r, "A0": A0, "B0": B0}

    def fd(name, idx):
        a = dict(args)
        p = a[name].copy(); p[idx] += h; a[name] = p
        lp = _loss_state(a["w"], a["u"], a["k"], a["v"], a["r"], dy, a["A0"], a["B0"], gA, gB)
        m = args[name].copy(); m[idx] -= h; a[name] = m
        lm = _loss_state(a["w"], a["u"], a["k"], a["v"], a["r"], dy, a["A0"], a["B0"], gA, gB)
        return (lp - lm) / (2 * h)

    for name, key in (("k", "dk"), ("v", "dv"), ("r", "dr"), ("w", "dw"), ("u", "du"),
                      ("A0", "dA0"), ("B0", "dB0")):
        for idx in np.ndindex(args[name].shape):
            assert fd(name, idx) == pytest.approx(res[key][idx], rel=1e-6, abs=1e-8), (name, idx)
    assert np.all(res["dw_abs"] >= np.abs(res["dw"])) and np.all(res["du_abs"] >= np.abs(res["du"]))
    assert np.all(res["dA0_abs"] >= np.abs(res["dA0"])) and np.all(res["dB0_abs"] >= np.abs(res["dB0"]))


def test_backward_state_without_state_is_the_analytic_backward():
    # Two independent derivations: the adjoint of the recurrence with empty state and
    # zero final-state gradient, and the closed-form sums beta, gamma, betad, gammad.
    w, u, k, v, r = _rand(3, 33, 4, 33)
    dy = np.random.Generator(np.random.PCG64(34)).standard_normal((3, 33, 4))
    a = oracle.wkv_backward(w, u, k, v, r, dy)
    b = oracle.wkv_backward_state(w, u, k, v, r, dy)
    for n in ("dk", "dv", "dr", "dw", "du"):
        np.testing.assert_allclose(b[n], a[n], rtol=1e-12, atol=1e-13, err_msg=n)
    np.testing.assert_allclose(b["dw_abs"], a["dw_abs"], rtol=1e-12, err_msg="dw_abs")
    np.testing.assert_allclose(b["du_abs"], a["du_abs"], rtol=1e-12, err_msg="du_abs")


def test_backward_state_chains_over_a_split_sequence():
    # Training a sequence in two consecutive pieces: the second piece starts from the
    # first's final state; its initial-state gradient is the first piece's final-state
    # gradient. Together they must give the whole sequence's gradients.
    B, T, C, T1 = 2, 30, 3, 11
    w, u, k, v, r = _rand(B, T, C, 35)
    g = np.random.Generator(np.random.PCG64(36))
    dy = g.standard_normal((B, T, C))
    A0 = g.standard_normal((B, C))
    B0 = g.uniform(0.5, 2.0, (B, C))
    gA = g.standard_normal((B, C))
    gB = g.standard_normal((B, C))
    whole = oracle.wkv_backward_state(w, u, k, v, r, dy, A0, B0, gA, gB)
    _, Am, Bm = oracle.wkv_recurrent(w, u, k[:, :T1], v[:, :T1], r[:, :T1], A0, B0,
                                     want_state=True)
    second = oracle.wkv_backward_state(w, u, k[:, T1:], v[:, T1:], r[:, T1:], dy[:, T1:],
                                       Am, Bm, gA, gB)
    first = oracle.wkv_backward_state(w, u, k[:, :T1], v[:, :T1], r[:, :T1], dy[:, :T1],
                                      A0, B0, second["dA0"], second["dB0"])
    for n in ("dk", "dv", "dr"):
        np.testing.assert_allclose(np.concatenate([first[n], second[n]], axis=1), whole[n],
                                   rtol=1e-11, atol=1e-12, err_msg=n)
    for n in ("dw", "du"):
        np.testing.assert_allclose(first[n] + second[n], whole[n], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(first["dA0"], whole["dA0"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(first["dB0"], whole["dB0"], rtol=1e-11, atol=1e-12)


def _grad_terms_brute(w, u, k, v, r, dy, A0=None, B0=None, gA=None, gB=None):
    """dk_abs, dv_abs by listing the terms of dk_i and dv_i one by one from the parallel
    form (plain loops, tiny inputs): token i reaches output t >= i with the weight
    e^{k_i - (t-1-i)w} / D_t (t > i) or e^{u+k_i} / D_t (t = i), and the final state with
    e^{k_i - (T-1-i)w}; D_t, wkv_t are the definition's sums written out."""
    B, T, C = k.shape
    dka = np.zeros((B, T, C))
    dva = np.zeros((B, T, C))
    for b in range(B):
        for c in range(C):
            D = np.empty(T)
            wkv = np.empty(T)
            for t in range(T):
                num = den = 0.0
                if A0 is not None:
                    num += math.exp(-t * w[c]) * A0[b, c]
                    den += math.exp(-t * w[c]) * B0[b, c]
                for i in range(t):
                    e = math.exp(-(t - 1 - i) * w[c] + k[b, i, c])
                    num += e * v[b, i, c]
                    den += e
                e = math.exp(u[c] + k[b, t, c])
                D[t] = den + e
                wkv[t] = (num + e * v[b, t, c]) / D[t]
            g = dy[b, :, c] * (1.0 / (1.0 + np.exp(-r[b, :, c])) if r is not None else 1.0)
            for i in range(T):
                vi = abs(v[b, i, c])
                e = math.exp(u[c] + k[b, i, c]) * abs(g[i]) / D[i]
                sv, sk = e, e * (vi + abs(wkv[i]))
                for t in range(i + 1, T):
                    e = math.exp(k[b, i, c] - (t - 1 - i) * w[c]) * abs(g[t]) / D[t]
                    sv += e
                    sk += e * (vi + abs(wkv[t]))
                if gA is not None:
                    e = math.exp(k[b, i, c] - (T - 1 - i) * w[c])
                    sv += e * abs(gA[b, c])
                    sk += e * (vi * abs(gA[b, c]) + abs(gB[b, c]))
                dva[b, i, c] = sv
                dka[b, i, c] = sk
    return dka, dva


def test_gradient_term_scales_match_brute_force():
    # dk_abs, dv_abs (the scale of the terms behind each dk, dv element) against the terms
    # listed one by one, for the plain backward and through a state.
    B, T, C = 2, 9, 3
    w, u, k, v, r = _rand(B, T, C, 40, k_std=2.0)
    g = np.random.Generator(np.random.PCG64(41))
    dy = g.standard_normal((B, T, C))
    a = oracle.wkv_backward(w, u, k, v, r, dy)
    dka, dva = _grad_terms_brute(w, u, k, v, r, dy)
    np.testing.assert_allclose(a["dk_abs"], dka, rtol=1e-12)
    np.testing.assert_allclose(a["dv_abs"], dva, rtol=1e-12)
    A0 = g.standard_normal((B, C))
    B0 = g.uniform(0.5, 2.0, (B, C))
    gA = g.standard_normal((B, C))
    gB = g.standard_normal((B, C))
    s = oracle.wkv_backward_state(w, u, k, v, r, dy, A0, B0, gA, gB)
    dka, dva = _grad_terms_brute(w, u, k, v, r, dy, A0, B0, gA, gB)
    np.testing.assert_allclose(s["dk_abs"], dka, rtol=1e-12)
    np.testing.assert_allclose(s["dv_abs"], dva, rtol=1e-12)
    for res in (a, s):
        assert np.all(res["dv_abs"] >= np.abs(res["dv"]) * (1 - 1e-12))
        assert np.all(res["dk_abs"] >= np.abs(res["dk"]) * (1 - 1e-12))


def test_gradient_term_scales_without_cancellation():
    # dy >= 0 and v >= 0 (hence wkv >= 0): every term of dv is non-negative, so
    # dv_abs = dv; dk's terms are e^{..} h (v_i - wkv_t), so dk_abs = sum e^{..} h (v_i +
    # wkv_t) = 2 v_i dv_i - dk_i.
    B, T, C = 2, 50, 4
    w, u, k, v, r = _rand(B, T, C, 42, k_std=2.0)
    v = np.abs(v)
    dy = np.abs(np.random.Generator(np.random.PCG64(43)).standard_normal((B, T, C)))
    for res in (oracle.wkv_backward(w, u, k, v, r, dy),
                oracle.wkv_backward_state(w, u, k, v, r, dy)):
        np.testing.assert_allclose(res["dv_abs"], res["dv"], rtol=1e-12)
        np.testing.assert_allclose(res["dk_abs"], 2 * v * res["dv"] - res["dk"], rtol=1e-10,
                                   atol=1e-13)


# ---- RWKV-7 generalised-delta-rule recurrence (research report, section 1.3.3) ----

def _unit_rows(g, shape):
    x = g.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def test_wkv7_delta_rule_stores_the_latest_pair():
    # w = 1, a = -k^, b = k^ (unit k^) makes the transition I - k^T k^, so after each token
    # the state maps the token's key exactly to its value: S_t k^_t^T = v_t. Reading the
    # state with r_t = k^_t therefore returns v_t, whatever came before.
    g = np.random.Generator(np.random.PCG64(40))
    B, T, H, N = 2, 9, 3, 6
    kh = _unit_rows(g, (B, T, H, N))
    v = g.standard_normal((B, T, H, N))
    S0 = g.standard_normal((B, H, N, N))
    y = oracle.wkv7_recurrent(kh, np.ones((B, T, H, N)), kh, v, -kh, kh, S0)
    np.testing.assert_allclose(y, v, rtol=1e-12, atol=1e-12)


def test_wkv7_reflection_preserves_the_state_norm():
    # w = 1, a = -2 k^, b = k^: the transition I - 2 k^T k^ is a reflection (orthogonal), so
    # with v = 0 every row of S keeps its length; with k = 0 nothing is written.
    g = np.random.Generator(np.random.PCG64(41))
    B, T, H, N = 1, 12, 2, 5
    kh = _unit_rows(g, (B, T, H, N))
    S0 = g.standard_normal((B, H, N, N))
    zero = np.zeros((B, T, H, N))
    _, ST = oracle.wkv7_recurrent(zero, np.ones((B, T, H, N)), zero, zero, -2 * kh, kh, S0,
                                  want_state=True)
    np.testing.assert_allclose(np.linalg.norm(ST, axis=-1), np.linalg.norm(S0, axis=-1),
                               rtol=1e-12)


def test_wkv7_without_delta_term_is_decayed_linear_attention():
    # a = b = 0: S_t = sum_{s<=t} v_s^T (k_s * D_{s,t}) with D_{s,t} = prod_{s<u<=t} w_u (per key
    # channel), so y_t = sum_{s<=t} v_s <k_s * D_{s,t}, r_t>: attention with per-channel
    # decayed scores, summed here pair by pair.
    g = np.random.Generator(np.random.PCG64(42))
    B, T, H, N = 2, 7, 2, 4
    r, k, v = (g.standard_normal((B, T, H, N)) for _ in range(3))
    w = g.uniform(0.3, 1.0, (B, T, H, N))
    zero = np.zeros((B, T, H, N))
    y = oracle.wkv7_recurrent(r, w, k, v, zero, zero)
    ref = np.zeros_like(y)
    for bb in range(B):
        for h in range(H):
            for t in range(T):
                for s in range(t + 1):
                    D = np.prod(w[bb, s + 1:t + 1, h], axis=0) if t > s else np.ones(N)
                    ref[bb, t, h] += v[bb, s, h] * np.dot(k[bb, s, h] * D, r[bb, t, h])
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_wkv7_scalar_head_closed_form():
    # N = 1: s_t = s_{t-1} (w_t + a_t b_t) + v_t k_t, a scalar linear recurrence with the
    # closed form s_T = s_0 prod_t m_t + sum_i v_i k_i prod_{j>i} m_j, m = w + a b.
    g = np.random.Generator(np.random.PCG64(43))
    T = 15
    r, k, v, a, b = (g.standard_normal((1, T, 1, 1)) for _ in range(5))
    w = g.uniform(0.2, 1.0, (1, T, 1, 1))
    s0 = np.array([[[[0.7]]]])
    y, sT = oracle.wkv7_recurrent(r, w, k, v, a, b, s0, want_state=True)
    m = (w + a * b)[0, :, 0, 0]
    vk = (v * k)[0, :, 0, 0]
    for t in range(T):
        st = s0[0, 0, 0, 0] * np.prod(m[:t + 1]) + sum(vk[i] * np.prod(m[i + 1:t + 1])
                                                       for i in range(t + 1))
        assert y[0, t, 0, 0] == pytest.approx(st * r[0, t, 0, 0], rel=1e-12, abs=1e-14)
    assert sT[0, 0, 0, 0] == pytest.approx(s0[0, 0, 0, 0] * np.prod(m)
                                           + sum(vk[i] * np.prod(m[i + 1:]) for i in range(T)),
                                           rel=1e-12)


def test_wkv7_split_with_state_handover():
    g = np.random.Generator(np.random.PCG64(44))
    B, T, H, N, T1 = 2, 20, 2, 5, 8
    r, k, v = (g.standard_normal((B, T, H, N)) for _ in range(3))
    w = g.uniform(0.5, 1.0, (B, T, H, N))
    kh = _unit_rows(g, (B, T, H, N))
    a, b = -kh, kh * g.uniform(0, 1, (B, T, H, 1))
    S0 = g.standard_normal((B, H, N, N))
    y, ST = oracle.wkv7_recurrent(r, w, k, v, a, b, S0, want_state=True)
    y1, S1 = oracle.wkv7_recurrent(r[:, :T1], w[:, :T1], k[:, :T1], v[:, :T1], a[:, :T1],
                                   b[:, :T1], S0, want_state=True)
    y2, S2 = oracle.wkv7_recurrent(r[:, T1:], w[:, T1:], k[:, T1:], v[:, T1:], a[:, T1:],
                                   b[:, T1:], S1, want_state=True)
    np.testing.assert_allclose(np.concatenate([y1, y2], axis=1), y, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(S2, ST, rtol=1e-13, atol=1e-13)


def _wkv7_chunked(r, w, k, v, a, b, S0, L):
    """One head's recurrence in the chunked (triangular-solve) form, fp64: within a chunk,
    with gamma_t = w_1 ... w_t per key channel, the decay-normalised state is S_0 plus rank-one
    terms x_s (b_s / gamma_s)^T + v_s (k_s / gamma_s)^T, where x_t = S_{t-1} a_t solves a
    unit-triangular system over the chunk's tokens. A different algorithm from the token
    loop (no state update per token), so it pins the oracle's indexing and transposes."""
    T, N = k.shape
    S = S0.copy()
    y = np.empty((T, N))
    for c0 in range(0, T, L):
        n = min(L, T - c0)
        sl = slice(c0, c0 + n)
        gam = np.cumprod(w[sl], axis=0)                  # gamma_t, t = 1 .. n
        gprev = np.vstack([np.ones((1, N)), gam[:-1]])   # gamma_{t-1}
        at, bt, kt, rt = gprev * a[sl], b[sl] / gam, k[sl] / gam, gam * r[sl]
        V = v[sl]
        X = np.zeros((n, N))
        for t in range(n):                               # forward substitution
            X[t] = S @ at[t] + sum(X[s] * (bt[s] @ at[t]) + V[s] * (kt[s] @ at[t])
                                   for s in range(t))
        for t in range(n):
            y[c0 + t] = S @ rt[t] + sum(X[s] * (bt[s] @ rt[t]) + V[s] * (kt[s] @ rt[t])
                                        for s in range(t + 1))
        g = gam[-1]
        S = S * g[None, :] + sum(np.outer(X[s], g * bt[s]) + np.outer(V[s], g * kt[s])
                                 for s in range(n))
    return y, S


@pytest.mark.parametrize("L", [1, 4, 8])
def test_wkv7_matches_the_chunked_form(L):
    # Generic inputs (a, b not tied to k), decays in (0.5, 1], a ragged last chunk.
    g = np.random.Generator(np.random.PCG64(45))
    B, T, H, N = 1, 19, 2, 6
    r, k, v, a, b = (g.standard_normal((B, T, H, N)) * 0.5 for _ in range(5))
    w = g.uniform(0.5, 1.0, (B, T, H, N))
    S0 = g.standard_normal((B, H, N, N))
    y, ST = oracle.wkv7_recurrent(r, w, k, v, a, b, S0, want_state=True)
    for h in range(H):
        yc, Sc = _wkv7_chunked(r[0, :, h], w[0, :, h], k[0, :, h], v[0, :, h], a[0, :, h],
                               b[0, :, h], S0[0, h], L)
        np.testing.assert_allclose(y[0, :, h], yc, rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(ST[0, h], Sc, rtol=1e-10, atol=1e-10)
