"""GPU parity of wkv_mstate_forward (through the C ABI): the matrix-valued-state WKV with a
per-key-channel decay (the RWKV-5/6 form, the delta-rule update with a = b = 0), computed
chunkwise on the tensor cores, against the fp64 oracle's recurrence (pinned on the CPU,
among others, by decayed linear attention summed pair by pair)."""
import ctypes

import numpy as np
import pytest

import oracle
import wkv_inputs
from wkv_check import FP32_TOL

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

WKV_ERR_RANGE = 7


@pytest.fixture(scope="module")
def W():
    import rwkv_linear_attention_wkv_b200 as W
    return W


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def close(got, ref, what, tol=FP32_TOL):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref) / (1.0 + np.abs(ref))
    assert np.all(err <= tol), (what, float(err.max()))
    return float(err.max()) if err.size else 0.0


def inputs(B, T, H, seed):
    x = wkv_inputs.rwkv7_inputs(B, T, H, seed=seed)
    x.a[...] = 0.0
    x.b[...] = 0.0
    return x


def run(W, x, with_state=True):
    y, S = W.wkv_mstate_forward(dev(x.r), dev(x.w), dev(x.k), dev(x.v),
                                state=dev(x.S0) if with_state else None)
    assert W.wkv_stream_status() == 0
    ref, Sref = oracle.wkv7_recurrent(x.r, x.w, x.k, x.v, x.a, x.b,
                                      x.S0 if with_state else None, want_state=True)
    return y.cpu().numpy(), S.cpu().numpy(), ref, Sref


@pytest.mark.parametrize("shape", [(1, 1, 1), (2, 37, 3), (1, 64, 2), (1, 65, 1),
                                   (1, 256, 2), (3, 100, 4), (1, 1000, 1)])
@pytest.mark.parametrize("with_state", [True, False])
def test_mstate_shapes(W, shape, with_state):
    # one chunk, one partial chunk, exact chunk multiples and ragged tails, several heads
    # and batch rows, with and without an initial state
    B, T, H = shape
    x = inputs(B, T, H, seed=7 * T + H)
    y, S, ref, Sref = run(W, x, with_state)
    close(y, ref, "y")
    close(S, Sref, "state")


def test_mstate_long_sequence(W):
    # 2048 tokens: 32 chunks chained through the state ring
    x = inputs(1, 2048, 2, seed=3)
    y, S, ref, Sref = run(W, x)
    close(y, ref, "y")
    close(S, Sref, "state")


def test_mstate_bench_heads_sampled(W):
    # The benchmark's 64 heads over 512 tokens, every head against the oracle.
    x = inputs(1, 512, 64, seed=52)
    y, S, ref, Sref = run(W, x)
    close(y, ref, "y")
    close(S, Sref, "state")


def test_mstate_split_and_in_place_state(W):
    # Two pieces chained through the state (updated in place) give the one-pass result;
    # both against the oracle.
    x = inputs(2, 300, 2, seed=51)
    t = {n: dev(getattr(x, n)) for n in "rwkv"}
    st = dev(x.S0)
    y_all, s_all = W.wkv_mstate_forward(*(t[n] for n in "rwkv"), state=st.clone())
    ys = []
    for lo, hi in ((0, 77), (77, 300)):
        ys.append(W.wkv_mstate_forward(*(t[n][:, lo:hi].contiguous() for n in "rwkv"),
                                       state=st, state_out=st)[0])
    assert W.wkv_stream_status() == 0
    ref, Sref = oracle.wkv7_recurrent(x.r, x.w, x.k, x.v, x.a, x.b, x.S0, want_state=True)
    close(torch.cat(ys, 1).cpu().numpy(), ref, "y, in two pieces")
    close(st.cpu().numpy(), Sref, "state, in two pieces")
    close(y_all.cpu().numpy(), ref, "y, one pass")
    close(s_all.cpu().numpy(), Sref, "state, one pass")


def test_mstate_matches_recurrence_kernel(W):
    # Same inputs through wkv7_forward (token-by-token recurrence, a = b = 0): both within
    # the tolerance of the oracle, and of each other.
    x = inputs(2, 200, 3, seed=9)
    args = [dev(getattr(x, n)) for n in "rwkv"]
    y1, s1 = W.wkv_mstate_forward(*args, state=dev(x.S0))
    y2, s2 = W.wkv7_forward(*args, dev(x.a), dev(x.b), state=dev(x.S0))
    assert W.wkv_stream_status() == 0
    close(y1.cpu().numpy(), y2.cpu().numpy().astype(np.float64), "y")
    close(s1.cpu().numpy(), s2.cpu().numpy().astype(np.float64), "state")


def test_mstate_deterministic(W):
    x = inputs(2, 400, 4, seed=11)
    args = [dev(getattr(x, n)) for n in "rwkv"]
    a = W.wkv_mstate_forward(*args, state=dev(x.S0))
    b = W.wkv_mstate_forward(*args, state=dev(x.S0))
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_mstate_decay_out_of_range_is_reported(W):
    # w = 0.01 on every token: the decay over half a chunk (1e-62) is beyond the range of
    # the factorisation; the call reports WKV_ERR_RANGE and the next call is clean.
    x = inputs(1, 128, 1, seed=12)
    x.w[...] = 0.01
    W.wkv_mstate_forward(*(dev(getattr(x, n)) for n in "rwkv"))
    assert W.wkv_stream_status() == WKV_ERR_RANGE
    assert W.wkv_status_string(WKV_ERR_RANGE) == "WKV_ERR_RANGE"
    x = inputs(1, 128, 1, seed=13)
    y, S, ref, Sref = run(W, x)
    close(y, ref, "y after the reported call")


def test_mstate_no_tokens_and_arguments(W):
    f = W.lib.wkv_mstate_forward
    P = ctypes.c_void_p
    ok = P(4096)
    assert f(1, 4, 2, 32, *([ok] * 5), None, None, None) == 5      # N != 64
    assert f(1, 4, 2, 64, P(4100), *([ok] * 4), None, None, None) == 2  # misaligned
    assert f(1, 4, 2, 64, None, *([ok] * 4), None, None, None) == 1
    assert f(0, 4, 2, 64, *([None] * 7), None) == 0
    s0 = torch.randn(2, 3, 64, 64, device="cuda")
    s1 = torch.empty_like(s0)
    z = torch.empty((2, 0, 3, 64), device="cuda")
    W.wkv_mstate_forward(z, z, z, z, state=s0, state_out=s1)
    assert W.wkv_stream_status() == 0
    assert torch.equal(s0, s1)


def _sampled_heads(x, y, S, picks):
    """y (B, T, H, N) and S (B, H, N, N) of the listed (b, h) heads against the oracle run
    on those heads alone (heads are independent)."""
    for b, h in picks:
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
        ref, Sref = oracle.wkv7_recurrent(*(getattr(x, n)[sl] for n in "rwkvab"),
                                          x.S0[b:b + 1, h:h + 1], want_state=True)
        close(y[sl].cpu().numpy(), ref, f"y of head ({b}, {h})")
        close(S[b:b + 1, h:h + 1].cpu().numpy(), Sref, f"state of head ({b}, {h})")


def test_mstate_benchmark_shape_sampled(W):
    # The benchmark's launch: 8 x 4096 tokens x 64 heads (32768 chunks on the persistent
    # CTAs); 16 seeded heads in full against the oracle.
    x = inputs(8, 4096, 64, seed=0)
    y, S = W.wkv_mstate_forward(*(dev(getattr(x, n)) for n in "rwkv"), state=dev(x.S0))
    assert W.wkv_stream_status() == 0
    g = np.random.Generator(np.random.PCG64(5))
    picks = [(int(f) // 64, int(f) % 64) for f in g.choice(8 * 64, 16, replace=False)]
    _sampled_heads(x, y, S, picks)
