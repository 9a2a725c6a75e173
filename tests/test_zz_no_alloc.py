"""wkv_forward_state_static: the stateful forward that allocates no device memory.

Some callers cannot allocate device memory at the point where they run the operator: a
serving loop that must not risk the implicit device synchronisation an allocation can
bring, an application whose memory manager owns all device memory, or a deployment that
forbids dynamic allocation once started. For them the library keeps the chunked path's
scratch in a fixed array of its own device memory (8 MiB + 64 KiB) instead of allocating
it per call. These tests call that entry point through the C ABI:

* on two calls in a row (the second reuses the scratch the first left behind), its
  results are bit for bit those of wkv_forward_state (the same fixed-order kernel), both
  match the fp64 oracle within the fp32 tolerance, and the device's free memory does not
  move across a call;
* the largest documented problem (one sequence of 32768 tokens x 2048 channels) runs, and
  one more 256-token segment is refused with WKV_ERR_SCRATCH_LIMIT.

The file is collected last, so a run that stops at the first failure has run every other
test before it.
"""
import ctypes

import numpy as np
import pytest

import oracle
import wkv_inputs
from wkv_check import assert_fp32_close, assert_state_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

WKV_ERR_SCRATCH_LIMIT = 6


@pytest.fixture(scope="module")
def W():
    import rwkv_linear_attention_wkv_b200 as W
    f = W.lib.wkv_forward_state_static
    f.argtypes = [ctypes.c_int64] * 3 + [ctypes.c_void_p] * 13
    f.restype = ctypes.c_int
    # The first call on a device looks up the array's address (and may load the library's
    # device code): make it here, so that every test's free-memory check sees a later call.
    x = wkv_inputs.make_inputs(1, 600, 32, seed=7)
    w, u, k, v, r = (dev(a) for a in (x.w, x.u, x.k, x.v, x.r))
    y = torch.empty_like(k)
    out = [torch.empty((x.B, x.C), device="cuda") for _ in range(3)]
    assert static_call(W, x.B, x.T, x.C, w, u, k, v, r, y, None, out) == 0
    assert W.wkv_stream_status() == 0
    return W


def P(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def static_call(W, B, T, C, w, u, k, v, r, y, state, out):
    a0, b0, p0 = state if state is not None else (None, None, None)
    return W.lib.wkv_forward_state_static(
        B, T, C, P(w), P(u), P(k), P(v), P(r), P(y), P(a0), P(b0), P(p0), P(out[0]),
        P(out[1]), P(out[2]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def run_both(W, x, state=None):
    """The static entry point, then wkv_forward_state on the same inputs. Returns the
    static call's y and state, the allocating call's, and the device's free bytes just
    before and just after the static call."""
    w, u, k, v, r = dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(x.r)
    y = torch.empty_like(k)
    st = [torch.empty((x.B, x.C), device="cuda") for _ in range(3)]
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    rc = static_call(W, x.B, x.T, x.C, w, u, k, v, r, y, state, st)
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    assert rc == 0, W.wkv_status_string(rc)
    assert W.wkv_stream_status() == 0
    y_ref, st_ref = W.wkv_forward_state(w, u, k, v, r, state=state)
    assert W.wkv_stream_status() == 0
    return y, st, y_ref, st_ref, (free_before, free_after)


def check_against_oracle(x, y, st, A0=None, B0=None):
    ref, A1, B1 = oracle.wkv_recurrent(x.w, x.u, x.k, x.v, x.r, A0, B0, want_state=True)
    assert_fp32_close(y.cpu().numpy(), ref, "y")
    assert_state_close(*(s.cpu().numpy() for s in st), A1, B1, "final state")


def test_static_scratch_matches_allocating_entry_point_twice(W):
    # Few channels and a long sequence: the chunked (scratch-using) path.
    x1 = wkv_inputs.make_inputs(2, 3000, 256, seed=101, k_std=2.0)
    y, st, y_ref, st_ref, _ = run_both(W, x1)
    assert torch.equal(y, y_ref), "y, first call"
    for s, s_ref in zip(st, st_ref):
        assert torch.equal(s, s_ref), "state, first call"
    check_against_oracle(x1, y, st)
    # Second call in a row, other inputs and an initial state: the shared scratch still
    # holds the first call's flags and carries. The address lookup is done by now, so the
    # call must leave the device's free memory exactly as it was.
    x2 = wkv_inputs.make_inputs(2, 2500, 256, seed=202, k_std=2.0)
    state = tuple(t.clone() for t in st_ref)
    y2, st2, y2_ref, st2_ref, (free0, free1) = run_both(W, x2, state=state)
    assert torch.equal(y2, y2_ref), "y, second call"
    for s, s_ref in zip(st2, st2_ref):
        assert torch.equal(s, s_ref), "state, second call"
    A0, B0 = oracle.state_from_scaled(*(t.cpu().numpy() for t in state))
    check_against_oracle(x2, y2, st2, A0, B0)
    assert free1 == free0, f"device free memory moved by {free0 - free1} bytes"


def test_static_scratch_at_its_documented_limit(W):
    # One sequence of 32768 tokens x 2048 channels: 8192 items of scratch, the largest
    # documented problem. Bitwise equal to the allocating entry point; a sample of
    # channels against the oracle (channels are independent).
    x = wkv_inputs.make_inputs(1, 32768, 2048, seed=303)
    y, st, y_ref, st_ref, (free0, free1) = run_both(W, x)
    assert torch.equal(y, y_ref)
    for s, s_ref in zip(st, st_ref):
        assert torch.equal(s, s_ref)
    assert free1 == free0, f"device free memory moved by {free0 - free1} bytes"
    cols = slice(1000, 1032)
    xs = wkv_inputs.WkvInputs(**{**x.__dict__, "C": 32, "w": x.w[cols], "u": x.u[cols],
                                 "k": x.k[:, :, cols], "v": x.v[:, :, cols],
                                 "r": x.r[:, :, cols]})
    check_against_oracle(xs, y[:, :, cols], [s[:, cols] for s in st])


@pytest.mark.parametrize("shape", [(1, 33024, 2048), (1, 65536, 4096)])
def test_static_scratch_rejects_problems_beyond_its_size(W, shape):
    # 33024 tokens x 2048 channels is one 256-token segment more than the limit (8256
    # items); 65536 x 4096 needs about 33 MiB.
    B, T, C = shape
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the size check comes first
    rc = W.lib.wkv_forward_state_static(B, T, C, *([fake] * 6), None, None, None,
                                        None, None, None, None)
    assert rc == WKV_ERR_SCRATCH_LIMIT
    assert W.wkv_status_string(rc) == "WKV_ERR_SCRATCH_LIMIT"
