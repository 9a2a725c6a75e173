"""wkv_forward_state_static: the stateful forward that allocates no device memory.

Some callers cannot allocate device memory at the point where they run the operator: a
serving loop that must not risk the implicit device synchronisation an allocation can
bring, an application whose memory manager owns all device memory, or a deployment that
forbids dynamic allocation once started. For them the library keeps the chunked path's scratch
of the chunked path in a fixed 8 MiB array of its own device memory instead of allocating
it per call. This test calls that entry point through the C ABI and checks it against
wkv_forward_state on two calls in a row (the second reuses the scratch the first left
behind), with the tolerance the other fp32 tests use. It lives in a file of its own that
pytest collects last.
"""
import ctypes

import numpy as np
import pytest

import wkv_inputs
from wkv_check import assert_fp32_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

WKV_ERR_SCRATCH_LIMIT = 6


@pytest.fixture(scope="module")
def W():
    import rwkv_linear_attention_wkv_b200 as W
    f = W.lib.wkv_forward_state_static
    f.argtypes = [ctypes.c_int64] * 3 + [ctypes.c_void_p] * 13
    f.restype = ctypes.c_int
    return W


def P(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def call_static(W, x, state=None):
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    w, u, k, v, r = dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(x.r)
    y = torch.empty_like(k)
    st = [torch.empty((x.B, x.C), device="cuda") for _ in range(3)]
    a0, b0, p0 = state if state is not None else (None, None, None)
    rc = W.lib.wkv_forward_state_static(
        x.B, x.T, x.C, P(w), P(u), P(k), P(v), P(r), P(y), P(a0), P(b0), P(p0),
        P(st[0]), P(st[1]), P(st[2]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, W.wkv_status_string(rc)
    assert W.wkv_stream_status() == 0
    y_ref, st_ref = W.wkv_forward_state(w, u, k, v, r, state=state)
    assert W.wkv_stream_status() == 0
    return y, st, y_ref, st_ref


def test_static_scratch_matches_allocating_entry_point_twice(W):
    # Few channels and a long sequence: the chunked (scratch-using) path.
    x1 = wkv_inputs.make_inputs(2, 3000, 256, seed=101, k_std=2.0)
    y, st, y_ref, st_ref = call_static(W, x1)
    assert_fp32_close(y.cpu().numpy(), y_ref.cpu().numpy(), "y, first call")
    for s, s_ref in zip(st, st_ref):
        assert_fp32_close(s.cpu().numpy(), s_ref.cpu().numpy(), "state, first call")
    # Second call in a row, other inputs and an initial state: the shared scratch still
    # holds the first call's flags and carries.
    x2 = wkv_inputs.make_inputs(2, 2500, 256, seed=202, k_std=2.0)
    y2, st2, y2_ref, st2_ref = call_static(W, x2, state=tuple(t.clone() for t in st_ref))
    assert_fp32_close(y2.cpu().numpy(), y2_ref.cpu().numpy(), "y, second call")
    for s, s_ref in zip(st2, st2_ref):
        assert_fp32_close(s.cpu().numpy(), s_ref.cpu().numpy(), "state, second call")


def test_static_scratch_rejects_problems_beyond_its_size(W):
    # One sequence of 65536 tokens x 4096 channels needs about 33 MiB of scratch.
    B, T, C = 1, 65536, 4096
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the size check comes first
    rc = W.lib.wkv_forward_state_static(B, T, C, *([fake] * 6), None, None, None,
                                        None, None, None, None)
    assert rc == WKV_ERR_SCRATCH_LIMIT
    assert W.wkv_status_string(rc) == "WKV_ERR_SCRATCH_LIMIT"
