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
