"""GPU parity of wkv_backward (through the C ABI) against the fp64 analytic oracle, which
is itself pinned to central finite differences on the CPU."""
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
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def check(W, x, gate=True, want_dr=True, plain=False):
    r = dev(x.r) if gate else None
    g = W.wkv_backward(dev(x.w), dev(x.u), dev(x.k), dev(x.v), r, dev(x.dy), want_dr=want_dr,
                       _entry="wkv_testing_backward_plain" if plain else "wkv_backward")
    assert W.wkv_stream_status() == 0
    ref = oracle.wkv_backward(x.w, x.u, x.k, x.v, x.r if gate else None, x.dy)
    assert_grad_close(g["dk"].cpu().numpy(), ref["dk"], ref["dk_abs"], "dk")
    assert_grad_close(g["dv"].cpu().numpy(), ref["dv"], ref["dv_abs"], "dv")
    if gate and want_dr:
        assert_fp32_close(g["dr"].cpu().numpy(), ref["dr"], "dr")
    else:
        assert g["dr"] is None
    for n in ("dw", "du"):
        got = g[n].cpu().numpy().astype(np.float64)
        err = np.abs(got - ref[n])
        bound = 1e-5 * (1.0 + ref[n + "_abs"])
        assert np.all(err <= bound), (n, float((err / bound).max()))
    return g


@pytest.mark.parametrize("shape", [(1, 1, 4), (2, 40, 64), (1, 33, 37), (3, 100, 8),
                                   (2, 95, 96), (1, 257, 5)])
@pytest.mark.parametrize("gate", [True, False])
def test_backward_shapes(W, shape, gate):
    B, T, C = shape
    x = wkv_inputs.make_inputs(B, T, C, seed=T * 7 + C, k_std=2.0, with_dy=True)
    check(W, x, gate)
    check(W, x, gate, plain=True)


def test_backward_without_dr(W):
    x = wkv_inputs.make_inputs(2, 70, 32, seed=3, with_dy=True)
    check(W, x, gate=True, want_dr=False)


def test_backward_extreme_parameters(W):
    x = wkv_inputs.make_inputs(2, 70, 64, seed=5, k_std=2.0, with_dy=True)
    x.w[:16] = 30.0
    x.u[16:32] = 40.0
    x.w[32:48] = 1e-4
    check(W, x)


def test_backward_spikes(W):
    x = wkv_inputs.make_inputs(2, 300, 64, seed=8, logw_range=(-6, 2), u_bound=2.0, k_std=3.0,
                               spike_frac=0.01, with_dy=True)
    check(W, x)


def test_backward_training_shape_full(W):
    # The 169M-model training shape B=16, T=1024, C=768: every element of dk, dv, dr and
    # dw, du against the oracle.
    x = wkv_inputs.training_shape(seed=0)
    g1 = check(W, x)
    # Deterministic: the carries of the time-parallel reverse are chained in a fixed order
    # and dw, du are reduced in a fixed order, so a second call gives identical bits.
    for _ in range(2):
        g2 = W.wkv_backward(dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(x.r), dev(x.dy))
        for n in ("dk", "dv", "dw", "du", "dr"):
            assert torch.equal(g1[n], g2[n]), n
    # The serial form (plain loads and stores) against the oracle at the same shape.
    check(W, x, plain=True)


@pytest.mark.parametrize("shape", [(3, 1001, 100), (1, 4100, 32), (2, 64, 36), (1, 16, 32),
                                   (1, 17, 32)])
def test_backward_time_parallel_segments(W, shape):
    # Many 64-token segments (one carry hop each), a ragged last chunk and segment, a
    # partial 32-channel group, and the one-chunk / one-segment edges.
    B, T, C = shape
    x = wkv_inputs.make_inputs(B, T, C, seed=B * 31 + T, k_std=2.0, with_dy=True)
    check(W, x)


@pytest.mark.parametrize("shape", [(3, 150, 2752), (1, 67, 8192), (2, 33, 4100)])
@pytest.mark.parametrize("gate", [True, False])
def test_backward_many_channels(W, shape, gate):
    # Thousands of channels with k spikes and decays from e^-6 to e^2: many independent
    # 32-channel groups per segment, ragged T (a partial last chunk) and a partial group
    # (C = 4100).
    B, T, C = shape
    x = wkv_inputs.make_inputs(B, T, C, seed=C + T, logw_range=(-6, 2), u_bound=2.0,
                               k_std=3.0, spike_frac=1e-3, with_dy=True)
    check(W, x, gate)


def test_backward_workspace_checks(W):
    import ctypes
    x = wkv_inputs.make_inputs(1, 10, 8, seed=1, with_dy=True)
    k = dev(x.k)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        W.wkv_backward(dev(x.w), dev(x.u), k, dev(x.v), dev(x.r), dev(x.dy), workspace=small)
    ws = torch.empty(W.wkv_backward_workspace_bytes(1, 10, 8), dtype=torch.uint8, device="cuda")
    t = [torch.empty_like(k) for _ in range(3)]
    dwdu = [torch.empty(8, device="cuda") for _ in range(2)]
    P = lambda a: ctypes.c_void_p(a.data_ptr())  # noqa: E731
    rc = W.lib.wkv_backward(1, 10, 8, P(dev(x.w)), P(dev(x.u)), P(k), P(dev(x.v)), P(dev(x.r)),
                            P(dev(x.dy)), P(t[0]), P(t[1]), P(dwdu[0]), P(dwdu[1]), P(t[2]),
                            P(ws), 8, None)
    assert rc == 1  # WKV_ERR_INVALID_ARG: workspace too small
    # No tokens: parameter gradients are zero.
    z = torch.zeros((1, 0, 8), device="cuda")
    g = W.wkv_backward(dev(x.w), dev(x.u), z, z, z, z)
    assert torch.count_nonzero(g["dw"]) == 0 and torch.count_nonzero(g["du"]) == 0


def test_backward_wait_gives_up_and_reports(W):
    # The last segment of the time-parallel reverse pass withholds its map: the earlier
    # segments' bounded waits give up after 1 ms, flag the error word and end.
    import ctypes
    s = torch.cuda.current_stream()
    rc = W.lib.wkv_testing_backward_timeout(1_000_000, ctypes.c_void_p(s.cuda_stream))
    assert rc == 0
    assert W.wkv_stream_status() == 4          # WKV_ERR_TIMEOUT
    assert W.wkv_stream_status() == 0          # cleared
    x = wkv_inputs.make_inputs(1, 200, 32, seed=21, with_dy=True)  # context still usable
    check(W, x)
