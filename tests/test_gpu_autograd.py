"""The autograd wrapper (rwkv_linear_attention_wkv_b200.autograd): its forward and the
gradients PyTorch's backward collects through it are bit for bit those of the C-ABI calls
it marshals (wkv_forward_checkpointed, wkv_backward_checkpointed), and they match the fp64
oracle (y within 1e-5 (1 + |y|); dk, dv within the term-scale rule, dw, du within it)."""
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


def dev(a, grad=False):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda().requires_grad_(grad)


@pytest.mark.parametrize("gate", [True, False])
def test_autograd_matches_the_c_abi_and_the_oracle(W, gate):
    from rwkv_linear_attention_wkv_b200.autograd import wkv
    x = wkv_inputs.make_inputs(2, 200, 96, seed=31, with_dy=True, k_std=2.0)
    w, u, k, v = (dev(getattr(x, n), True) for n in ("w", "u", "k", "v"))
    r = dev(x.r, True) if gate else None
    dy = dev(x.dy)
    y = wkv(w, u, k, v, r)
    (y * dy).sum().backward()
    assert W.wkv_stream_status() == 0
    # the same calls directly
    y2, ws = W.wkv_forward_checkpointed(*(t.detach() for t in (w, u, k, v)),
                                        None if r is None else r.detach())
    g = W.wkv_backward_checkpointed(*(t.detach() for t in (w, u, k, v)),
                                    None if r is None else r.detach(), dy, ws, want_dr=gate)
    assert torch.equal(y.detach(), y2)
    for name, t in (("dw", w), ("du", u), ("dk", k), ("dv", v)) + ((("dr", r),) if gate else ()):
        assert torch.equal(t.grad, g[name]), name
    # and against the oracle
    ref = oracle.wkv_backward(x.w, x.u, x.k, x.v, x.r if gate else None, x.dy)
    y_ref = oracle.wkv_recurrent(x.w, x.u, x.k, x.v, x.r if gate else None)
    assert_fp32_close(y.detach().cpu().numpy(), y_ref, "y")
    for name, t in (("dk", k), ("dv", v)):
        assert_grad_close(t.grad.cpu().numpy(), ref[name], ref[name + "_abs"], name)
    for name, t in (("dw", w), ("du", u)):
        assert_grad_close(t.grad.cpu().numpy(), ref[name], ref[name + "_abs"], name)
    if gate:
        assert_fp32_close(r.grad.cpu().numpy(), ref["dr"], "dr")


def test_autograd_only_some_inputs_need_grad(W):
    from rwkv_linear_attention_wkv_b200.autograd import wkv
    x = wkv_inputs.make_inputs(1, 64, 32, seed=32, with_dy=True)
    w, u = dev(x.w), dev(x.u)
    k = dev(x.k, True)
    v, r = dev(x.v), dev(x.r)
    y = wkv(w, u, k, v, r)
    (y * dev(x.dy)).sum().backward()
    assert k.grad is not None and w.grad is None and v.grad is None
