"""GPU parity of wkv7_forward (through the C ABI): RWKV-7's generalised-delta-rule
recurrence per head against the fp64 oracle (pinned on the CPU by the delta-rule, reflection,
decayed-attention and closed-form tests)."""
import numpy as np
import pytest

import oracle
import wkv_inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def W():
    import rwkv_linear_attention_wkv_b200 as W
    return W


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def close(got, ref, what, tol=1e-5):
    # fp32 against fp64 over sums of N = 64 products per step, scale-relative
    got = np.asarray(got, dtype=np.float64)
    scale = 1.0 + np.abs(ref)
    err = np.abs(got - ref) / scale
    assert np.all(err <= tol), (what, float(err.max()))


def run(W, x, with_state=True):
    y, ST = W.wkv7_forward(dev(x.r), dev(x.w), dev(x.k), dev(x.v), dev(x.a), dev(x.b),
                           state=dev(x.S0) if with_state else None)
    assert W.wkv_stream_status() == 0
    ref, Sref = oracle.wkv7_recurrent(x.r, x.w, x.k, x.v, x.a, x.b,
                                      x.S0 if with_state else None, want_state=True)
    return y.cpu().numpy(), ST.cpu().numpy(), ref, Sref


@pytest.mark.parametrize("shape", [(1, 1, 1), (2, 37, 3), (1, 256, 2), (3, 100, 4),
                                   (1, 1000, 1)])
@pytest.mark.parametrize("with_state", [True, False])
def test_wkv7_shapes(W, shape, with_state):
    B, T, H = shape
    x = wkv_inputs.rwkv7_inputs(B, T, H, seed=T + H)
    y, ST, ref, Sref = run(W, x, with_state)
    close(y, ref, "y")
    close(ST, Sref, "state")


@pytest.mark.parametrize("shape", [(2, 37, 3), (1, 300, 4)])
def test_wkv7_without_delta_term(W, shape):
    # a = b = 0: S_t = S_{t-1} diag(w_t) + v_t^T k_t, per-channel decayed linear attention
    # with a matrix-valued state per head (the form of the report's section 1.3.2, with a
    # data-dependent decay).
    B, T, H = shape
    x = wkv_inputs.rwkv7_inputs(B, T, H, seed=60 + T)
    x.a[...] = 0.0
    x.b[...] = 0.0
    y, ST, ref, Sref = run(W, x)
    close(y, ref, "y")
    close(ST, Sref, "state")


def test_wkv7_delta_rule_on_gpu(W):
    # w = 1, a = -k^, b = k^: the state stores the latest (key, value) pair exactly, so
    # reading with r = k^ returns v (to fp32 rounding).
    g = np.random.Generator(np.random.PCG64(50))
    B, T, H, N = 2, 40, 3, 64
    kh = g.standard_normal((B, T, H, N))
    kh /= np.linalg.norm(kh, axis=-1, keepdims=True)
    v = g.standard_normal((B, T, H, N))
    one = np.ones((B, T, H, N))
    y, _ = W.wkv7_forward(dev(kh), dev(one), dev(kh), dev(v), dev(-kh), dev(kh))
    assert W.wkv_stream_status() == 0
    close(y.cpu().numpy(), v, "y = v")
    ref = oracle.wkv7_recurrent(*(np.float32(t).astype(np.float64) for t in
                                  (kh, one, kh, v, -kh, kh)))
    close(y.cpu().numpy(), ref, "y")


def test_wkv7_split_and_in_place_state(W):
    x = wkv_inputs.rwkv7_inputs(2, 300, 2, seed=51)
    t = {n: dev(getattr(x, n)) for n in ("r", "w", "k", "v", "a", "b")}
    st = dev(x.S0)
    y_all, s_all = W.wkv7_forward(*(t[n] for n in "rwkvab"), state=st.clone())
    ys = []
    for lo, hi in ((0, 77), (77, 300)):
        ys.append(W.wkv7_forward(*(t[n][:, lo:hi].contiguous() for n in "rwkvab"), state=st,
                                 state_out=st)[0])
    assert W.wkv_stream_status() == 0
    ref, Sref = oracle.wkv7_recurrent(x.r, x.w, x.k, x.v, x.a, x.b, x.S0, want_state=True)
    y_split = torch.cat(ys, 1).cpu().numpy()
    close(y_split, ref, "y, in two pieces")
    close(st.cpu().numpy(), Sref, "state, in two pieces")
    close(y_all.cpu().numpy(), ref, "y, one pass")
    close(y_split, y_all.cpu().numpy().astype(np.float64), "pieces against one pass")


def test_wkv7_argument_checks(W):
    import ctypes
    P = lambda n: ctypes.c_void_p(n)  # noqa: E731
    f = W.lib.wkv7_forward
    ok = P(4096)
    assert f(1, 4, 2, 32, *([ok] * 7), None, None, None) == 5     # N != 64
    assert f(1, 4, 2, 64, P(4100), *([ok] * 6), None, None, None) == 2  # not 16-B aligned
    assert f(1, 4, 2, 64, None, *([ok] * 6), None, None, None) == 1
    assert f(0, 4, 2, 64, *([None] * 9), None) == 0


def test_wkv7_larger_shape_sampled(W):
    # The benchmark's head count at a shorter sequence: every head, against the oracle.
    x = wkv_inputs.rwkv7_inputs(1, 512, 64, seed=52)
    y, ST, ref, Sref = run(W, x)
    close(y, ref, "y")
    close(ST, Sref, "state")


def test_wkv7_benchmark_shape_sampled(W):
    # The benchmark's launch: 8 x 4096 tokens x 64 heads; 16 seeded heads in full against
    # the oracle (heads are independent).
    x = wkv_inputs.rwkv7_inputs(8, 4096, 64, seed=0)
    y, S = W.wkv7_forward(*(dev(getattr(x, n)) for n in "rwkvab"), state=dev(x.S0))
    assert W.wkv_stream_status() == 0
    g = np.random.Generator(np.random.PCG64(5))
    for f in g.choice(8 * 64, 16, replace=False):
        b, h = int(f) // 64, int(f) % 64
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
        ref, Sref = oracle.wkv7_recurrent(*(getattr(x, n)[sl] for n in "rwkvab"),
                                          x.S0[b:b + 1, h:h + 1], want_state=True)
        close(y[sl].cpu().numpy(), ref, f"y of head ({b}, {h})")
        close(S[b:b + 1, h:h + 1].cpu().numpy(), Sref, f"state of head ({b}, {h})")
