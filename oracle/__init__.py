"""fp64 CPU oracle for RWKV's WKV operator: TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package. The product (the CUDA library and its Python binding) never does,
and this package imports nothing from it.

Two parts:

* ``wkv_oracle.c`` (built into ``libwkv_oracle.so`` by :func:`build`), plain C in
  double precision: the O(T^2) parallel form, the unstabilised recurrence, the decode
  step, the analytic backward, the backward through an entering and leaving state (the
  recurrence's adjoint), and RWKV-7's generalised-delta-rule recurrence (research report
  "RWKV模型深度研究报告", section 1.3.3);
* a few NumPy routines for tiny inputs that restate the operator through other
  routes: a causal softmax over logits (the operator as attention with
  query-independent weights), and one inference step written from the single-token
  description.

Sources (page title, section): "RWKV（Receptance Weighted Key Value）概念", section 3.2
(the wkv_t equation, the receptance gate) and section 3.1 (linear-attention view);
"RWKV - 把 RNN 重新带回 Transformer 时代的线性大模型", "一句话总结" (recurrence),
"关键设计 2" (parallel form and RNN cell), "关键设计 4" (single-token inference).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wkv_oracle.c")
_LIB = os.path.join(_HERE, "libwkv_oracle.so")


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (no fast-math: IEEE double throughout)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-Wall",
                               "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int64
        lib.oracle_wkv_direct.argtypes = [I, I, I] + [P] * 8
        lib.oracle_wkv_recurrent.argtypes = [I, I, I] + [P] * 10
        lib.oracle_wkv_decode.argtypes = [I, I, I] + [P] * 8
        lib.oracle_wkv_backward.argtypes = [I, I, I] + [P] * 15
        lib.oracle_wkv_backward_state.argtypes = [I, I, I] + [P] * 23
        lib.oracle_wkv7_recurrent.argtypes = [I, I, I, I] + [P] * 9
        for f in (lib.oracle_wkv_direct, lib.oracle_wkv_recurrent, lib.oracle_wkv_decode,
                  lib.oracle_wkv_backward, lib.oracle_wkv_backward_state,
                  lib.oracle_wkv7_recurrent):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    return None if x is None else x.ctypes.data


def _check(rc):
    if rc != 0:
        raise RuntimeError("oracle call failed (bad argument or out of memory)")


def wkv_direct(w, u, k, v, r=None, A0=None, B0=None):
    """O(T^2) parallel form; k, v, r (B,T,C). Returns y (B,T,C) float64."""
    w, u, k, v, r, A0, B0 = map(_f64, (w, u, k, v, r, A0, B0))
    B, T, C = k.shape
    y = np.empty((B, T, C))
    _check(_load().oracle_wkv_direct(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
                                     _ptr(y), _ptr(A0), _ptr(B0)))
    return y


def wkv_recurrent(w, u, k, v, r=None, A0=None, B0=None, want_state=False):
    """Unstabilised fp64 recurrence. Returns y, or (y, A_T, B_T) with want_state."""
    w, u, k, v, r, A0, B0 = map(_f64, (w, u, k, v, r, A0, B0))
    B, T, C = k.shape
    y = np.empty((B, T, C))
    A1 = np.empty((B, C)) if want_state else None
    B1 = np.empty((B, C)) if want_state else None
    _check(_load().oracle_wkv_recurrent(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
                                        _ptr(y), _ptr(A0), _ptr(B0), _ptr(A1), _ptr(B1)))
    return (y, A1, B1) if want_state else y


def wkv_decode(w, u, k, v, r, A, Bd):
    """One token for [N,L,C] states; w, u [L,C]. Returns (y, A', B') as new arrays."""
    w, u, k, v, r = map(_f64, (w, u, k, v, r))
    A = np.array(A, dtype=np.float64, copy=True, order="C")
    Bd = np.array(Bd, dtype=np.float64, copy=True, order="C")
    N, L, C = k.shape
    y = np.empty((N, L, C))
    _check(_load().oracle_wkv_decode(N, L, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
                                     _ptr(y), _ptr(A), _ptr(Bd)))
    return y, A, Bd


def wkv_backward(w, u, k, v, r, dy):
    """Analytic fp64 gradients. Returns dict dk, dv, dw, du, dr (dr None if r is None),
    and dw_abs, du_abs, dk_abs, dv_abs: the sums of |term| behind dw, du, dk and dv."""
    w, u, k, v, r, dy = map(_f64, (w, u, k, v, r, dy))
    B, T, C = k.shape
    dk = np.empty((B, T, C))
    dv = np.empty((B, T, C))
    dr = np.empty((B, T, C)) if r is not None else None
    dw = np.empty(C)
    du = np.empty(C)
    dwa = np.empty(C)
    dua = np.empty(C)
    dka = np.empty((B, T, C))
    dva = np.empty((B, T, C))
    _check(_load().oracle_wkv_backward(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
                                       _ptr(dy), _ptr(dk), _ptr(dv), _ptr(dw), _ptr(du),
                                       _ptr(dr), _ptr(dwa), _ptr(dua), _ptr(dka), _ptr(dva)))
    return {"dk": dk, "dv": dv, "dw": dw, "du": du, "dr": dr, "dw_abs": dwa, "du_abs": dua,
            "dk_abs": dka, "dv_abs": dva}


def wkv_backward_state(w, u, k, v, r, dy, A0=None, B0=None, gA=None, gB=None):
    """Gradients of sum(dy * y) + sum(gA * A_T) + sum(gB * B_T) for the forward from the
    true initial state (A0, B0) [B, C] (None: empty), by the step-by-step adjoint of the
    recurrence. Returns dict dk, dv, dw, du, dr (None if r is None), dA0, dB0 [B, C], and
    dw_abs, du_abs, dA0_abs, dB0_abs, dk_abs, dv_abs: the same sums run on absolute
    values."""
    w, u, k, v, r, dy, A0, B0, gA, gB = map(_f64, (w, u, k, v, r, dy, A0, B0, gA, gB))
    B, T, C = k.shape
    dk = np.empty((B, T, C))
    dv = np.empty((B, T, C))
    dr = np.empty((B, T, C)) if r is not None else None
    dw, du, dwa, dua = (np.empty(C) for _ in range(4))
    dA0, dB0, dA0a, dB0a = (np.empty((B, C)) for _ in range(4))
    dka = np.empty((B, T, C))
    dva = np.empty((B, T, C))
    _check(_load().oracle_wkv_backward_state(
        B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(dy), _ptr(A0), _ptr(B0),
        _ptr(gA), _ptr(gB), _ptr(dk), _ptr(dv), _ptr(dw), _ptr(du), _ptr(dr), _ptr(dA0),
        _ptr(dB0), _ptr(dwa), _ptr(dua), _ptr(dA0a), _ptr(dB0a), _ptr(dka), _ptr(dva)))
    return {"dk": dk, "dv": dv, "dw": dw, "du": du, "dr": dr, "dA0": dA0, "dB0": dB0,
            "dw_abs": dwa, "du_abs": dua, "dA0_abs": dA0a, "dB0_abs": dB0a,
            "dk_abs": dka, "dv_abs": dva}


def wkv7_recurrent(r, w, k, v, a, b, S0=None, want_state=False):
    """RWKV-7 generalised-delta-rule recurrence per head; r, w, k, v, a, b (B, T, H, N),
    S0 (B, H, N, N) or None. Returns y (B, T, H, N), or (y, S_T) with want_state."""
    r, w, k, v, a, b, S0 = map(_f64, (r, w, k, v, a, b, S0))
    B, T, H, N = k.shape
    y = np.empty((B, T, H, N))
    S1 = np.empty((B, H, N, N)) if want_state else None
    _check(_load().oracle_wkv7_recurrent(B, T, H, N, _ptr(r), _ptr(w), _ptr(k), _ptr(v),
                                         _ptr(a), _ptr(b), _ptr(y), _ptr(S0), _ptr(S1)))
    return (y, S1) if want_state else y


def state_from_scaled(a, b, p):
    """(a, b, p) with numerator a e^p and denominator b e^p -> true (A, B) in fp64."""
    a, b, p = (np.asarray(x, dtype=np.float64) for x in (a, b, p))
    s = np.exp(p)
    return a * s, b * s


# ---------------------------------------------------------------------------------------
# Tiny-input restatements through other routes (NumPy / SciPy, fp64).
# ---------------------------------------------------------------------------------------

def wkv_softmax_form(w, u, k, v):
    """wkv as causal attention with query-independent logits.

    Section 3.1/3.2 of the concept page reads the operator as attention whose weights
    decay with distance; written that way, wkv_t is a softmax over the logits
    {k_i - (t-1-i) w : i < t} together with u + k_t for the current token, applied to v.
    SciPy's softmax does the normalisation. k, v (T, C); w, u (C,). Returns (T, C).
    """
    from scipy.special import softmax

    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    T, C = k.shape
    out = np.empty((T, C))
    for c in range(C):
        for t in range(T):
            logits = np.empty(t + 1)
            for i in range(t):
                logits[i] = k[i, c] - (t - 1 - i) * float(w[c])
            logits[t] = float(u[c]) + k[t, c]
            out[t, c] = softmax(logits) @ v[: t + 1, c]
    return out


def wkv_single_step(w, u, k, v, state):
    """One inference step per the single-token description: the output uses the stored
    numerator/denominator plus the current token weighted by e^{u+k}; afterwards both
    decay by e^{-w} and take in e^{k} (times v for the numerator).
    state = (num, den) arrays (C,). Returns (wkv, (num', den'))."""
    num, den = (np.asarray(x, dtype=np.float64) for x in state)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    bonus = np.exp(np.asarray(u, dtype=np.float64) + k)
    out = (num + bonus * v) / (den + bonus)
    keep = np.exp(-np.asarray(w, dtype=np.float64))
    return out, (keep * num + np.exp(k) * v, keep * den + np.exp(k))
