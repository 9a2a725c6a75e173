"""CUDA graphs over the C ABI.

Every entry point is stream-ordered: its launches, clears and any scratch it needs
(stream-ordered allocation) go onto the caller's stream with no host synchronisation, so a
caller can capture a whole step once and replay it. These tests capture a training step
(forward + backward, both pairs), the 7B-shaped bf16 forward's call pattern, the chunked
long-sequence forward (which allocates and frees its scratch inside the call) and a
multi-token decode. They write new inputs into the captured tensors and replay: each
replay must give exactly (bit for bit) what the same calls give run eagerly on those
inputs.
"""
import numpy as np
import pytest

import wkv_inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def W():
    import rwkv_linear_attention_wkv_b200 as W
    return W


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def capture(fn):
    """fn run once eagerly (first-call set-up outside the capture), then captured."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def refill(tensors, seed):
    """New values in place (same storage, so the captured graph reads them)."""
    x = wkv_inputs.make_inputs(*tensors["k"].shape, seed=seed, with_dy="dy" in tensors,
                               k_std=2.0, spike_frac=1e-3)
    for n, t in tensors.items():
        t.copy_(dev(getattr(x, n)).to(t.dtype))


def _train_tensors(B, T, C, seed):
    x = wkv_inputs.make_inputs(B, T, C, seed=seed, with_dy=True)
    return {n: dev(getattr(x, n)) for n in ("w", "u", "k", "v", "r", "dy")}


def _grads_like(k, B, C):
    out = {n: torch.empty_like(k) for n in ("dk", "dv", "dr")}
    out["dw"] = torch.empty(C, device="cuda")
    out["du"] = torch.empty(C, device="cuda")
    return out


@pytest.mark.usefixtures("bwd_path")
@pytest.mark.parametrize("pair", ["checkpointed", "plain"])
def test_training_step_replay_is_bitwise_eager(W, pair):
    B, T, C = 4, 300, 256
    t = _train_tensors(B, T, C, seed=61)
    ws = torch.empty(W.wkv_backward_workspace_bytes(B, T, C), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(t["k"])
    out = _grads_like(t["k"], B, C)
    args = [t[n] for n in ("w", "u", "k", "v", "r")]

    def step():
        if pair == "checkpointed":
            W.wkv_forward_checkpointed(*args, y=y, workspace=ws)
            W.wkv_backward_checkpointed(*args, t["dy"], ws, out=out)
        else:
            W.wkv_forward(*args, y=y)
            W.wkv_backward(*args, t["dy"], workspace=ws, out=out)

    g = capture(step)
    for seed in (62, 63):
        refill({n: t[n] for n in ("k", "v", "r", "dy")}, seed)
        g.replay()
        torch.cuda.synchronize()
        assert W.wkv_stream_status() == 0
        got = {"y": y.clone(), **{n: o.clone() for n, o in out.items()}}
        step()  # eagerly, same inputs
        torch.cuda.synchronize()
        assert W.wkv_stream_status() == 0
        assert torch.equal(got["y"], y), "y"
        for n, o in out.items():
            assert torch.equal(got[n], o), n


def test_bf16_forward_replay_is_bitwise_eager(W):
    def bf16_inputs(seed):
        # k, v, r hold bf16-representable values (exact in the conversion)
        x = wkv_inputs.make_inputs(2, 1000, 512, seed=seed, dtype="bf16", k_std=3.0,
                                   spike_frac=1e-3)
        return x, [dev(getattr(x, n)).to(torch.bfloat16) for n in ("k", "v", "r")]

    x, (k, v, r) = bf16_inputs(71)
    w, u = dev(x.w), dev(x.u)
    y = torch.empty_like(k)
    g = capture(lambda: W.wkv_forward_bf16(w, u, k, v, r, y=y))
    for seed in (72, 73):
        for dst, src in zip((k, v, r), bf16_inputs(seed)[1]):
            dst.copy_(src)
        g.replay()
        torch.cuda.synchronize()
        got = y.clone()
        W.wkv_forward_bf16(w, u, k, v, r, y=y)
        torch.cuda.synchronize()
        assert W.wkv_stream_status() == 0
        assert torch.equal(got.view(torch.int16), y.view(torch.int16))


def test_chunked_forward_with_state_replay_is_bitwise_eager(W):
    # Few channels and a long sequence: the chunked path, whose scratch is allocated and
    # freed on the stream inside the call (allocation nodes in the graph).
    B, T, C = 1, 4000, 128
    x = wkv_inputs.make_inputs(B, T, C, seed=81)
    t = {n: dev(getattr(x, n)) for n in ("w", "u", "k", "v", "r")}
    y = torch.empty_like(t["k"])
    st_in = tuple(torch.full((B, C), v, device="cuda") for v in (0.3, 1.5, 0.2))
    st_out = tuple(torch.empty((B, C), device="cuda") for _ in range(3))

    def fwd():
        W.wkv_forward_state(*(t[n] for n in ("w", "u", "k", "v", "r")), state=st_in, y=y,
                            state_out=st_out)

    g = capture(fwd)
    for seed in (82, 83):
        refill({n: t[n] for n in ("k", "v", "r")}, seed)
        g.replay()
        torch.cuda.synchronize()
        got = (y.clone(),) + tuple(s.clone() for s in st_out)
        fwd()
        torch.cuda.synchronize()
        assert W.wkv_stream_status() == 0
        for a, b_ in zip(got, (y,) + st_out):
            assert torch.equal(a, b_)


def test_decode_steps_replay_advances_the_state_like_eager_calls(W):
    d = wkv_inputs.decode_batch(seed=91, N=8, L=4, C=512)
    S = 6
    kvr = [np.stack(z) for z in zip(*(d.step(s) for s in range(S)))]
    w, u = dev(d.w), dev(d.u)
    k, v, r = (dev(z) for z in kvr)
    state_g = [dev(z) for z in (d.a, d.b, d.p)]
    state_e = [s.clone() for s in state_g]
    y = torch.empty_like(k)
    # the capture's own eager warm-up call advances state_g once: keep state_e in step
    g = capture(lambda: W.wkv_decode_steps(w, u, k, v, r, *state_g, y=y))
    W.wkv_decode_steps(w, u, k, v, r, *state_e, y=torch.empty_like(k))
    y_e = torch.empty_like(k)
    for _ in range(2):  # each replay decodes the next S tokens from the state it left
        g.replay()
        W.wkv_decode_steps(w, u, k, v, r, *state_e, y=y_e)
        torch.cuda.synchronize()
        assert W.wkv_stream_status() == 0
        assert torch.equal(y, y_e)
        for a, b_ in zip(state_g, state_e):
            assert torch.equal(a, b_)
