"""GPU parity of wkv_backward_state (through the C ABI): the backward through an entering
and a leaving state, against the fp64 oracle's adjoint of the recurrence (itself pinned
to central differences on the CPU)."""
import numpy as np
import pytest

import oracle
import wkv_inputs
from wkv_check import assert_fp32_close, assert_grad_close

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("bwd_path")]


@pytest.fixture(scope="module")
def W():
    import rwkv_linear_attention_wkv_b200 as W
    return W


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def make_state(B, C, seed):
    """An initial state in the (a, b, p) representation and final-state gradients."""
    g = np.random.Generator(np.random.PCG64(seed))
    a0 = g.standard_normal((B, C)).astype(np.float32)
    b0 = g.uniform(0.5, 2.0, (B, C)).astype(np.float32)
    p0 = g.normal(0.0, 2.0, (B, C)).astype(np.float32)
    ga1 = g.standard_normal((B, C)).astype(np.float32)
    gb1 = g.standard_normal((B, C)).astype(np.float32)
    return a0, b0, p0, ga1, gb1


def assert_sum_close(got, ref, scale, what):
    err = np.abs(np.asarray(got, dtype=np.float64) - ref)
    bound = 1e-5 * (1.0 + scale)
    assert np.all(err <= bound), (what, float((err / bound).max()))


def run(W, x, a0, b0, p0, ga1, gb1, with_state=True, with_grad=True, plain=False):
    """GPU stateful backward and the oracle's, compared. Returns the GPU results."""
    st = (dev(a0), dev(b0), dev(p0)) if with_state else None
    # p1 of the final state the forward returns (the representation ga1, gb1 refer to)
    y, (a1, b1, p1) = W.wkv_forward_state(dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(x.r),
                                          state=st)
    gs = (dev(ga1), dev(gb1), p1) if with_grad else None
    g = W.wkv_backward_state(dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(x.r), dev(x.dy),
                             state=st, grad_state=gs,
                             _entry=("wkv_testing_backward_state_plain" if plain
                                     else "wkv_backward_state"))
    assert W.wkv_stream_status() == 0
    p1h = p1.cpu().numpy().astype(np.float64)
    A0 = B0 = gA = gB = None
    if with_state:
        A0, B0 = oracle.state_from_scaled(a0, b0, p0)
    if with_grad:
        gA = ga1.astype(np.float64) * np.exp(-p1h)
        gB = gb1.astype(np.float64) * np.exp(-p1h)
    ref = oracle.wkv_backward_state(x.w, x.u, x.k, x.v, x.r, x.dy, A0, B0, gA, gB)
    for n in ("dk", "dv"):
        assert_grad_close(g[n].cpu().numpy(), ref[n], ref[n + "_abs"], n)
    assert_fp32_close(g["dr"].cpu().numpy(), ref["dr"], "dr")
    for n in ("dw", "du"):
        assert_sum_close(g[n].cpu().numpy(), ref[n], ref[n + "_abs"], n)
    # da0 = e^{p0} dL/dA0, db0 = e^{p0} dL/dB0, dp0 = a0 da0 + b0 db0
    e0 = np.exp(p0.astype(np.float64)) if with_state else np.zeros_like(ref["dA0"])
    da0 = e0 * ref["dA0"]
    db0 = e0 * ref["dB0"]
    assert_sum_close(g["da0"].cpu().numpy(), da0, e0 * ref["dA0_abs"], "da0")
    assert_sum_close(g["db0"].cpu().numpy(), db0, e0 * ref["dB0_abs"], "db0")
    if with_state:
        dp0 = a0 * da0 + b0 * db0
        scale = np.abs(a0) * e0 * ref["dA0_abs"] + b0 * e0 * ref["dB0_abs"]
        assert_sum_close(g["dp0"].cpu().numpy(), dp0, scale, "dp0")
    return g


@pytest.mark.parametrize("shape", [(2, 40, 64), (1, 33, 37), (3, 100, 8), (2, 95, 96),
                                   (1, 257, 5), (3, 1001, 100), (1, 16, 32), (1, 17, 32),
                                   (1, 1, 4)])
@pytest.mark.parametrize("plain", [False, True])
def test_backward_state_shapes(W, shape, plain):
    B, T, C = shape
    x = wkv_inputs.make_inputs(B, T, C, seed=T * 3 + C, k_std=2.0, with_dy=True)
    run(W, x, *make_state(B, C, T + C), plain=plain)


@pytest.mark.parametrize("with_state,with_grad", [(True, False), (False, True)])
def test_backward_state_one_side_only(W, with_state, with_grad):
    x = wkv_inputs.make_inputs(2, 150, 64, seed=4, k_std=2.0, with_dy=True)
    run(W, x, *make_state(2, 64, 5), with_state=with_state, with_grad=with_grad)


@pytest.mark.parametrize("shape", [(2, 97, 4096), (3, 40, 2752)])
@pytest.mark.parametrize("spike_frac", [0.0, 1e-3])
def test_backward_state_many_channels(W, shape, spike_frac):
    # Thousands of channels with a state on both sides, with and without k spikes (+60 on
    # 0.1% of the entries). With spikes, dv and dk hold sums whose terms nearly cancel; the
    # bound scales with the terms (the oracle's dk_abs, dv_abs).
    B, T, C = shape
    x = wkv_inputs.make_inputs(B, T, C, seed=T + C, k_std=2.0, spike_frac=spike_frac,
                               with_dy=True)
    run(W, x, *make_state(B, C, T))


def test_backward_state_spikes(W):
    x = wkv_inputs.make_inputs(2, 300, 64, seed=8, logw_range=(-6, 2), u_bound=2.0, k_std=3.0,
                               spike_frac=0.01, with_dy=True)
    run(W, x, *make_state(2, 64, 9))


def test_backward_state_without_state_equals_backward(W):
    x = wkv_inputs.make_inputs(2, 300, 96, seed=10, k_std=2.0, with_dy=True)
    a = W.wkv_backward(dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(x.r), dev(x.dy))
    b = W.wkv_backward_state(dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(x.r), dev(x.dy))
    for n in ("dk", "dv", "dr", "dw", "du"):
        assert torch.equal(a[n], b[n]), n
    assert torch.count_nonzero(b["da0"]) == 0 and torch.count_nonzero(b["db0"]) == 0


def test_backward_state_chains_over_pieces(W):
    # Three consecutive pieces, chained through the state and its gradients, give the
    # whole sequence's gradients (to within the fp32 tolerances against the oracle).
    B, T, C = 2, 700, 64
    x = wkv_inputs.make_inputs(B, T, C, seed=11, k_std=2.0, with_dy=True)
    a0, b0, p0, ga1, gb1 = make_state(B, C, 12)
    cuts = [0, 230, 481, T]
    w, u = dev(x.w), dev(x.u)
    pieces = []
    st = (dev(a0), dev(b0), dev(p0))
    for i in range(3):
        sl = slice(cuts[i], cuts[i + 1])
        k, v, r = dev(x.k[:, sl]), dev(x.v[:, sl]), dev(x.r[:, sl])
        _, st_out = W.wkv_forward_state(w, u, k, v, r, state=st)
        pieces.append((sl, st, st_out))
        st = st_out
    grad = (dev(ga1), dev(gb1), st[2])
    res = [None] * 3
    for i in (2, 1, 0):
        sl, st_in, _ = pieces[i]
        g = W.wkv_backward_state(w, u, dev(x.k[:, sl]), dev(x.v[:, sl]), dev(x.r[:, sl]),
                                 dev(x.dy[:, sl]), state=st_in, grad_state=grad)
        res[i] = g
        grad = (g["da0"], g["db0"], st_in[2])
    assert W.wkv_stream_status() == 0
    A0, B0 = oracle.state_from_scaled(a0, b0, p0)
    p1 = st[2].cpu().numpy().astype(np.float64)
    ref = oracle.wkv_backward_state(x.w, x.u, x.k, x.v, x.r, x.dy, A0, B0,
                                    ga1 * np.exp(-p1), gb1 * np.exp(-p1))
    for n in ("dk", "dv", "dr"):
        got = np.concatenate([g[n].cpu().numpy() for g in res], axis=1)
        if n == "dr":
            assert_fp32_close(got, ref[n], n)
        else:
            assert_grad_close(got, ref[n], ref[n + "_abs"], n)
    for n in ("dw", "du"):
        got = sum(g[n].cpu().numpy().astype(np.float64) for g in res)
        assert_sum_close(got, ref[n], ref[n + "_abs"], n)
    e0 = np.exp(p0.astype(np.float64))
    assert_sum_close(res[0]["da0"].cpu().numpy(), e0 * ref["dA0"], e0 * ref["dA0_abs"], "da0")
    assert_sum_close(res[0]["db0"].cpu().numpy(), e0 * ref["dB0"], e0 * ref["dB0_abs"], "db0")


def test_backward_state_no_tokens_passes_the_state_through(W):
    B, C = 2, 8
    a0, b0, p0, ga1, gb1 = make_state(B, C, 13)
    p1 = p0 + np.float32(0.5)
    z = torch.zeros((B, 0, C), device="cuda")
    g = W.wkv_backward_state(dev(np.ones(C)), dev(np.zeros(C)), z, z, z, z,
                             state=(dev(a0), dev(b0), dev(p0)),
                             grad_state=(dev(ga1), dev(gb1), dev(p1)))
    assert W.wkv_stream_status() == 0
    f = np.exp(p0.astype(np.float64) - p1)
    np.testing.assert_allclose(g["da0"].cpu().numpy(), ga1 * f, rtol=1e-6)
    np.testing.assert_allclose(g["db0"].cpu().numpy(), gb1 * f, rtol=1e-6)
    np.testing.assert_allclose(g["dp0"].cpu().numpy(), a0 * ga1 * f + b0 * gb1 * f,
                               rtol=1e-5, atol=1e-6)
    assert torch.count_nonzero(g["dw"]) == 0 and torch.count_nonzero(g["du"]) == 0


def test_backward_state_training_shape(W):
    # The 169M-model training shape with a state on both sides, and determinism.
    x = wkv_inputs.training_shape(seed=1)
    B, C = x.k.shape[0], x.k.shape[2]
    g1 = run(W, x, *make_state(B, C, 14))
    a0, b0, p0, ga1, gb1 = make_state(B, C, 14)
    st = (dev(a0), dev(b0), dev(p0))
    _, (a1, b1, p1) = W.wkv_forward_state(dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(x.r),
                                          state=st)
    g2 = W.wkv_backward_state(dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(x.r), dev(x.dy),
                              state=st, grad_state=(dev(ga1), dev(gb1), p1))
    for n in ("dk", "dv", "dr", "dw", "du", "da0", "db0", "dp0"):
        assert torch.equal(g1[n], g2[n]), n
