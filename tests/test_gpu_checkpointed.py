"""GPU parity of the checkpointed training pair (through the C ABI):
wkv_forward_checkpointed writes y and the backward's chunk checkpoints;
wkv_backward_checkpointed takes them instead of forming them. Both are compared with the
fp64 oracle (forward recurrence; adjoint of the recurrence, pinned on the CPU to central
differences), and the checkpoints with the ones the backward's own pass forms."""
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


def run(W, x, with_state=False, with_grad=False, gate=True, seed=0):
    """Checkpointed forward and backward against the oracle. Returns (y, grads, ws)."""
    B, T, C = x.k.shape
    a0, b0, p0, ga1, gb1 = make_state(B, C, seed)
    st = (dev(a0), dev(b0), dev(p0)) if with_state else None
    w, u, k, v = dev(x.w), dev(x.u), dev(x.k), dev(x.v)
    r = dev(x.r) if gate else None
    y, ws = W.wkv_forward_checkpointed(w, u, k, v, r, state=st)
    assert W.wkv_stream_status() == 0
    A0 = B0 = None
    if with_state:
        A0, B0 = oracle.state_from_scaled(a0, b0, p0)
    yref = oracle.wkv_recurrent(x.w, x.u, x.k, x.v, x.r if gate else None, A0, B0)
    assert_fp32_close(y.cpu().numpy(), yref, "y")
    gs = None
    gA = gB = None
    if with_grad:
        # the final state's p1, as wkv_forward_state reports it
        _, (_, _, p1) = W.wkv_forward_state(w, u, k, v, r, state=st)
        gs = (dev(ga1), dev(gb1), p1)
        p1h = p1.cpu().numpy().astype(np.float64)
        gA = ga1.astype(np.float64) * np.exp(-p1h)
        gB = gb1.astype(np.float64) * np.exp(-p1h)
    g = W.wkv_backward_checkpointed(w, u, k, v, r, dev(x.dy), ws, state=st, grad_state=gs)
    assert W.wkv_stream_status() == 0
    ref = oracle.wkv_backward_state(x.w, x.u, x.k, x.v, x.r if gate else None, x.dy,
                                    A0, B0, gA, gB)
    for n in ("dk", "dv"):
        assert_grad_close(g[n].cpu().numpy(), ref[n], ref[n + "_abs"], n)
    if gate:
        assert_fp32_close(g["dr"].cpu().numpy(), ref["dr"], "dr")
    for n in ("dw", "du"):
        assert_sum_close(g[n].cpu().numpy(), ref[n], ref[n + "_abs"], n)
    if with_state:
        e0 = np.exp(p0.astype(np.float64))
        assert_sum_close(g["da0"].cpu().numpy(), e0 * ref["dA0"], e0 * ref["dA0_abs"], "da0")
        assert_sum_close(g["db0"].cpu().numpy(), e0 * ref["dB0"], e0 * ref["dB0_abs"], "db0")
    return y, g, ws


@pytest.mark.parametrize("shape", [(2, 40, 64), (1, 33, 36), (3, 100, 8), (2, 95, 96),
                                   (1, 257, 4), (3, 1001, 100), (1, 16, 32), (1, 17, 32),
                                   (1, 1, 4), (2, 64, 32), (1, 48, 40)])
@pytest.mark.parametrize("gate", [True, False])
def test_checkpointed_pair_shapes(W, shape, gate):
    B, T, C = shape
    x = wkv_inputs.make_inputs(B, T, C, seed=T * 5 + C, k_std=2.0, with_dy=True)
    run(W, x, gate=gate)


@pytest.mark.parametrize("with_state,with_grad", [(True, False), (False, True), (True, True)])
def test_checkpointed_pair_with_state(W, with_state, with_grad):
    x = wkv_inputs.make_inputs(2, 150, 64, seed=31, k_std=2.0, with_dy=True)
    run(W, x, with_state=with_state, with_grad=with_grad, seed=32)


def test_checkpointed_pair_spikes_and_fast_decay(W):
    # k spikes (a single token dominating its chunk's scale) and decays from e^-6 to e^2
    # (windows of 16, 4 and 1 tokens), where a checkpoint that the recomputation does not
    # reproduce exactly would show.
    x = wkv_inputs.make_inputs(2, 300, 64, seed=33, logw_range=(-6, 2), u_bound=2.0, k_std=3.0,
                               spike_frac=0.01, with_dy=True)
    run(W, x, with_state=True, with_grad=True, seed=34)


def test_checkpointed_pair_generic_output(W):
    # |u - w| beyond the single-exponential bound in some warps.
    x = wkv_inputs.make_inputs(2, 70, 64, seed=35, k_std=2.0, with_dy=True)
    x.w[:32] = 90.0
    x.u[32:] = 95.0
    run(W, x)


def ckpt_region(W, ws, B, T, C):
    """The checkpoints [B, ceil(T/16), C, 4] in a backward workspace: after the 256-aligned
    block of chain flags (16 bytes + 8 per time segment of 64 tokens and 32-channel group)."""
    a256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
    nch = (T + 15) // 16
    nitems = B * ((C + 31) // 32) * ((nch + 3) // 4)
    off = a256(16 + 8 * nitems)
    n = B * nch * C * 16
    return ws[off:off + n].view(torch.float32).view(B, nch, C, 4)


def test_checkpoints_match_the_backward_pass(W):
    # The forward's checkpoints and the ones the backward's own pass forms describe the same
    # states: same a / b and log-scale Q + pl + log2(b), to fp32 rounding.
    B, T, C = 2, 500, 96
    x = wkv_inputs.make_inputs(B, T, C, seed=36, k_std=2.0, with_dy=True)
    w, u, k, v, r, dy = dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(x.r), dev(x.dy)
    _, ws1 = W.wkv_forward_checkpointed(w, u, k, v, r)
    ws2 = torch.zeros_like(ws1)
    W.wkv_backward(w, u, k, v, r, dy, workspace=ws2)
    assert W.wkv_stream_status() == 0
    c1 = ckpt_region(W, ws1, B, T, C).cpu().numpy().astype(np.float64)
    c2 = ckpt_region(W, ws2, B, T, C).cpu().numpy().astype(np.float64)
    # chunk 0: the empty state on both sides
    assert np.array_equal(c1[:, 0], c2[:, 0])
    c1, c2 = c1[:, 1:], c2[:, 1:]
    assert_fp32_close(c1[..., 0] / c1[..., 1], c2[..., 0] / c2[..., 1], "a/b")
    assert_fp32_close(c1[..., 2] + c1[..., 3] + np.log2(c1[..., 1]),
                      c2[..., 2] + c2[..., 3] + np.log2(c2[..., 1]), "log2 scale")


def test_checkpointed_pair_training_shape_and_determinism(W):
    x = wkv_inputs.training_shape(seed=2)
    y1, g1, _ = run(W, x)
    w, u, k, v, r = dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(x.r)
    y2, ws = W.wkv_forward_checkpointed(w, u, k, v, r)
    g2 = W.wkv_backward_checkpointed(w, u, k, v, r, dev(x.dy), ws)
    g3 = W.wkv_backward_checkpointed(w, u, k, v, r, dev(x.dy), ws)  # the workspace is reused
    assert W.wkv_stream_status() == 0
    assert torch.equal(y1, y2)
    # the streaming kernel of wkv_forward (B * C = 12288 channels), checkpoints aside
    assert torch.equal(y2, W.wkv_forward(w, u, k, v, r))
    for n in ("dk", "dv", "dr", "dw", "du"):
        assert torch.equal(g1[n], g2[n]), n
        assert torch.equal(g2[n], g3[n]), n


def test_checkpointed_pair_refuses_other_shapes(W):
    # C not a multiple of 4 has no time-parallel path: both calls refuse.
    C = 6
    z = torch.zeros((1, 20, C), device="cuda")
    one, zero = torch.ones(C, device="cuda"), torch.zeros(C, device="cuda")
    with pytest.raises(W.WkvError) as e:
        W.wkv_forward_checkpointed(one, zero, z, z, z)
    assert e.value.status == 5  # WKV_ERR_UNSUPPORTED
    ws = torch.zeros(W.wkv_backward_workspace_bytes(1, 20, C), dtype=torch.uint8, device="cuda")
    with pytest.raises(W.WkvError) as e:
        W.wkv_backward_checkpointed(one, zero, z, z, z, z, ws)
    assert e.value.status == 5
    assert W.wkv_stream_status() == 0
