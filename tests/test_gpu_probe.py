"""The pipe-throughput probe (wkv_testing_pipe_rate) that gives the bench's SFU and FP32
roofline denominators: its rates must lie near the unit-count figures (148 SMs x 16 MUFU
operations, or x 128 FMA lanes x 2 flops, per clock at up to 1965 MHz), since a probe
whose work was optimised away, or that counted it wrongly, would be far off; bad arguments
are refused before anything runs."""
import ctypes

import pytest

pytestmark = pytest.mark.gpu

NOMINAL_EX2 = 148 * 16 * 1965e6
NOMINAL_FLOPS = 148 * 128 * 2 * 1965e6


@pytest.fixture(scope="module")
def W():
    import rwkv_linear_attention_wkv_b200 as W
    return W


def rate(W, pipe, iters):
    out = ctypes.c_double(0.0)
    rc = W.lib.wkv_testing_pipe_rate(pipe, iters, ctypes.byref(out), None)
    return rc, out.value


def test_ex2_rate_is_near_the_mufu_unit_count(W):
    rc, r = rate(W, 0, 20000)
    assert rc == 0
    assert 0.4 * NOMINAL_EX2 < r < 1.2 * NOMINAL_EX2, r


def test_ffma2_rate_is_near_the_fma_unit_count(W):
    rc, r = rate(W, 1, 100000)
    assert rc == 0
    assert 0.4 * NOMINAL_FLOPS < r < 1.2 * NOMINAL_FLOPS, r


def test_probe_arguments(W):
    f = W.lib.wkv_testing_pipe_rate
    out = ctypes.c_double(0.0)
    assert f(2, 10, ctypes.byref(out), None) == 1        # unknown pipe
    assert f(0, 0, ctypes.byref(out), None) == 1         # no iterations
    assert f(0, 1 << 31, ctypes.byref(out), None) == 1   # too many
    assert f(0, 10, None, None) == 1                     # nowhere to write
