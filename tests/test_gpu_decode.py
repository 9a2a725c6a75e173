"""GPU parity of wkv_decode_step (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest

import oracle
import wkv_inputs
from wkv_check import assert_fp32_close, assert_state_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def W():
    import rwkv_linear_attention_wkv_b200 as W
    return W


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _run(W, d, steps, sample_n, gate=True):
    a, b, p = dev(d.a), dev(d.b), dev(d.p)
    w, u = dev(d.w), dev(d.u)
    A, Bd = oracle.state_from_scaled(d.a[sample_n], d.b[sample_n], d.p[sample_n])
    for s in range(steps):
        k, v, r = d.step(s)
        y = W.wkv_decode_step(w, u, dev(k), dev(v), dev(r) if gate else None, a, b, p)
        yr, A, Bd = oracle.wkv_decode(d.w, d.u, k[sample_n], v[sample_n],
                                      r[sample_n] if gate else None, A, Bd)
        assert_fp32_close(y.cpu().numpy()[sample_n], yr, f"y step {s}")
    assert W.wkv_stream_status() == 0
    assert_state_close(a.cpu().numpy()[sample_n], b.cpu().numpy()[sample_n],
                       p.cpu().numpy()[sample_n], A, Bd, f"state after {steps} steps")


@pytest.mark.parametrize("N,L,C", [(3, 2, 64), (2, 3, 37), (1, 1, 1), (5, 4, 130)])
def test_decode_small(W, N, L, C):
    d = wkv_inputs.decode_batch(seed=N + L + C, N=N, L=L, C=C)
    _run(W, d, 20, np.arange(N))
    d = wkv_inputs.decode_batch(seed=N * L * C, N=N, L=L, C=C)
    _run(W, d, 5, np.arange(N), gate=False)


def test_decode_full_size_64_chained_steps(W):
    # 256 sequences x 32 layers x 4096 channels, 64 chained steps; the oracle follows 8
    # seeded sequences (all layers and channels) through every step.
    d = wkv_inputs.decode_batch(seed=0)
    pick = np.sort(np.random.Generator(np.random.PCG64(99)).choice(d.N, 8, replace=False))
    _run(W, d, 64, pick)


def test_decode_steps_reproduce_forward(W):
    # T decode steps from the empty state give the forward pass's output.
    x = wkv_inputs.make_inputs(2, 50, 64, seed=21, k_std=2.0)
    y_fwd = W.wkv_forward(dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(x.r)).cpu().numpy()
    a = torch.zeros((2, 1, 64), device="cuda")
    b = torch.zeros((2, 1, 64), device="cuda")
    p = torch.full((2, 1, 64), -1e38, device="cuda")
    ys = []
    for t in range(50):
        ys.append(W.wkv_decode_step(dev(x.w[None]), dev(x.u[None]),
                                    dev(x.k[:, t:t + 1]), dev(x.v[:, t:t + 1]),
                                    dev(x.r[:, t:t + 1]), a, b, p).cpu().numpy()[:, 0])
    ref = oracle.wkv_recurrent(x.w, x.u, x.k, x.v, x.r)
    assert_fp32_close(np.stack(ys, 1), ref, "decode")
    assert_fp32_close(y_fwd, ref, "forward")


def _steps_vs_single(W, d, S, sample_n, gate=True):
    """wkv_decode_steps over S tokens against S wkv_decode_step calls (bit for bit, every
    element) and against the oracle chained S times on the sequences sample_n."""
    w, u = dev(d.w), dev(d.u)
    N, L, C = d.N, d.L, d.C
    k = torch.empty((S, N, L, C), device="cuda")
    v = torch.empty_like(k)
    r = torch.empty_like(k) if gate else None
    for s in range(S):
        ks, vs, rs = d.step(s)
        k[s].copy_(torch.from_numpy(ks))
        v[s].copy_(torch.from_numpy(vs))
        if gate:
            r[s].copy_(torch.from_numpy(rs))
    a, b, p = dev(d.a), dev(d.b), dev(d.p)
    y = W.wkv_decode_steps(w, u, k, v, r, a, b, p)
    assert W.wkv_stream_status() == 0
    a1, b1, p1 = dev(d.a), dev(d.b), dev(d.p)
    A, Bd = oracle.state_from_scaled(d.a[sample_n], d.b[sample_n], d.p[sample_n])
    for s in range(S):
        ys = W.wkv_decode_step(w, u, k[s], v[s], r[s] if gate else None, a1, b1, p1)
        assert torch.equal(ys, y[s]), f"step {s}: differs from the single-token step"
        kh, vh = k[s].cpu().numpy()[sample_n], v[s].cpu().numpy()[sample_n]
        rh = r[s].cpu().numpy()[sample_n] if gate else None
        yr, A, Bd = oracle.wkv_decode(d.w, d.u, kh, vh, rh, A, Bd)
        assert_fp32_close(y[s].cpu().numpy()[sample_n], yr, f"y step {s}")
    assert W.wkv_stream_status() == 0
    for t, t1 in ((a, a1), (b, b1), (p, p1)):
        assert torch.equal(t, t1), "final state differs from the single-token steps"
    assert_state_close(a.cpu().numpy()[sample_n], b.cpu().numpy()[sample_n],
                       p.cpu().numpy()[sample_n], A, Bd, f"state after {S} tokens")


@pytest.mark.parametrize("N,L,C,S", [(3, 2, 64, 20), (2, 3, 37, 7), (1, 1, 1, 5),
                                     (5, 4, 130, 9), (4, 2, 8, 1)])
@pytest.mark.parametrize("gate", [True, False])
def test_decode_steps_small(W, N, L, C, S, gate):
    d = wkv_inputs.decode_batch(seed=7 * N + L + C + S, N=N, L=L, C=C)
    _steps_vs_single(W, d, S, np.arange(N), gate)


def test_decode_steps_full_size_64_tokens(W):
    # 256 sequences x 32 layers x 4096 channels, 64 tokens in one call: every element
    # against 64 single-token calls, and the oracle following 8 seeded sequences (all
    # layers and channels) through every token.
    d = wkv_inputs.decode_batch(seed=0)
    pick = np.sort(np.random.Generator(np.random.PCG64(99)).choice(d.N, 8, replace=False))
    _steps_vs_single(W, d, 64, pick)


def test_decode_steps_arguments(W):
    import ctypes
    P = ctypes.c_void_p
    ok = P(4096)
    f = W.lib.wkv_decode_steps
    assert f(2, 1, 4, -1, *([ok] * 9), None) == 1            # negative S
    assert f(2, 1, 4, 0, *([ok] * 9), None) == 0             # no tokens: nothing to do
    assert f(2, 1, 4, 3, ok, ok, None, *([ok] * 6), None) == 1   # k missing
    assert f(2, 1, 4, 3, ok, ok, P(4098), *([ok] * 6), None) == 2  # k misaligned
    assert f(2, 1, 4, 1 << 31, *([ok] * 9), None) == 5       # S beyond int32
