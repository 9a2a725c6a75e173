"""Host-side checks of the C-ABI library that need no GPU: it loads, exports every symbol
the headers declare, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def W():
    import rwkv_linear_attention_wkv_b200 as W
    return W


def declared_symbols():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"WKV_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return names


def test_library_exports_every_declared_symbol(W):
    names = declared_symbols()
    assert "wkv_forward" in names and "wkv_backward" in names and len(names) >= 10
    for n in names:
        assert hasattr(W.lib, n), n


def test_status_strings(W):
    assert [W.wkv_status_string(i) for i in range(6)] == [
        "WKV_OK", "WKV_ERR_INVALID_ARG", "WKV_ERR_ALIGNMENT", "WKV_ERR_CUDA",
        "WKV_ERR_TIMEOUT", "WKV_ERR_UNSUPPORTED"]
    assert W.wkv_status_string(99) == "WKV_ERR_UNKNOWN"
    assert W.lib.wkv_version() >= 10000


def P(x):
    return ctypes.c_void_p(x)


def test_forward_argument_checks(W):
    f = W.lib.wkv_forward
    ok = P(4096)
    assert f(-1, 1, 1, ok, ok, ok, ok, ok, ok, None) == 1
    assert f(1, -1, 1, ok, ok, ok, ok, ok, ok, None) == 1
    assert f(1, 1, 1, None, ok, ok, ok, ok, ok, None) == 1      # w missing
    assert f(1, 1, 1, ok, ok, None, ok, ok, ok, None) == 1      # k missing
    assert f(1, 1, 1, ok, ok, ok, ok, None, None, None) == 1    # y missing
    assert f(1, 1, 4, ok, ok, P(4098), ok, None, ok, None) == 2  # k not 4-byte aligned
    assert f(0, 5, 5, None, None, None, None, None, None, None) == 0   # empty
    assert f(5, 5, 0, None, None, None, None, None, None, None) == 0
    assert f(1, 1 << 31, 4, ok, ok, ok, ok, ok, ok, None) == 5       # T too large
    g = W.lib.wkv_forward_bf16
    assert g(1, 1, 8, ok, ok, P(4097), ok, None, ok, None) == 2      # bf16 needs 2-byte
    st = W.lib.wkv_forward_state
    # state pointers must come as a full triple
    assert st(1, 1, 4, ok, ok, ok, ok, None, ok, ok, None, None, None, None, None, None) == 1
    assert st(1, 1, 4, ok, ok, ok, ok, None, ok, None, None, None, ok, ok, None, None) == 1


def test_decode_and_backward_argument_checks(W):
    ok = P(4096)
    d = W.lib.wkv_decode_step
    assert d(-1, 1, 1, *([ok] * 9), None) == 1
    assert d(1, 1, 1, ok, ok, ok, ok, None, ok, ok, ok, None, None) == 1   # p missing
    assert d(0, 4, 4, *([None] * 9), None) == 0
    assert d(1, 1, 1, ok, ok, P(4099), ok, None, ok, ok, ok, ok, None) == 2
    bw = W.lib.wkv_backward
    need = W.wkv_backward_workspace_bytes(2, 64, 32)
    args = [ok] * 5 + [ok] * 6
    assert bw(2, 64, 32, *args, ok, need - 1, None) == 1                    # too small
    assert bw(2, 64, 32, *args, P(4096 + 128), need, None) == 1             # not 256-aligned
    assert bw(2, 64, 32, ok, ok, ok, ok, None, ok, ok, ok, ok, ok, ok, ok, need, None) == 1
    assert bw(-2, 64, 32, *args, ok, need, None) == 1


def test_backward_workspace_size(W):
    # Chain flags (16 bytes of tickets, then two words per segment item), the forward state
    # (a, b, Q, pl) entering every 16-token chunk and after the last token, per-segment
    # partials of dw and du, and per segment item of 4 chunks and lane: its forward
    # aggregate (1 float4), reverse map (2 float4) and reverse carry (1 float4).
    def a256(x):
        return (x + 255) // 256 * 256
    for B, T, C in ((16, 1024, 768), (1, 33, 5), (3, 1, 4096)):
        nch = (T + 15) // 16
        nseg = (nch + 3) // 4
        nitems = B * ((C + 31) // 32) * nseg
        want = (a256(16 + 8 * nitems) + a256(B * nch * C * 16) + a256(B * C * 16)
                + 2 * a256(B * nseg * C * 4) + a256(nitems * 32 * 16) + a256(nitems * 32 * 32)
                + a256(nitems * 32 * 16))
        assert W.wkv_backward_workspace_bytes(B, T, C) == want


def test_backward_state_argument_checks(W):
    ok = P(4096)
    bs = W.lib.wkv_backward_state
    need = W.wkv_backward_workspace_bytes(2, 64, 32)
    base = [ok] * 6                      # w, u, k, v, r, dy
    outs = [ok] * 5                      # dk, dv, dw, du, dr
    full = [ok] * 3

    def call(B, st, gs, ds, ws=ok, nb=need):
        return bs(B, 64, 32, *base, *st, *gs, *outs, *ds, ws, nb, None)

    none3 = [None] * 3
    # each of the three triples must be all NULL or all non-NULL
    assert call(2, [ok, None, ok], none3, none3) == 1
    assert call(2, none3, [ok, ok, None], none3) == 1
    assert call(2, none3, none3, [None, ok, ok]) == 1
    assert call(2, full, full, full, nb=need - 1) == 1          # workspace too small
    assert call(2, full, full, [ok, ok, P(4098)]) == 2          # dp0 not 4-byte aligned
    assert call(-2, full, full, full) == 1
    assert call(0, full, full, full) == 0                       # no batch rows: nothing


def test_checkpointed_pair_argument_checks(W):
    # Refusals that happen before anything is enqueued (no GPU needed).
    ok = P(4096)
    need = W.wkv_backward_workspace_bytes(2, 64, 32)
    fc = W.lib.wkv_forward_checkpointed
    none3 = [None] * 3
    assert fc(2, 64, 32, ok, ok, ok, ok, ok, ok, *none3, ok, need - 1, None) == 1  # short
    assert fc(2, 64, 32, ok, ok, ok, ok, ok, ok, *none3, None, need, None) == 1    # no ws
    assert fc(2, 64, 32, ok, ok, ok, ok, ok, ok, *none3, P(4352 + 16), need, None) == 1
    assert fc(2, 64, 32, ok, ok, ok, ok, ok, ok, ok, None, ok, ok, need, None) == 1  # a0 triple
    assert fc(2, 64, 32, ok, ok, ok, ok, ok, P(4098), *none3, ok, need, None) == 2   # y align
    assert fc(-1, 64, 32, ok, ok, ok, ok, ok, ok, *none3, ok, need, None) == 1
    assert fc(2, 0, 32, ok, ok, ok, ok, ok, ok, *none3, None, 0, None) == 0         # no tokens
    bc = W.lib.wkv_backward_checkpointed
    base = [ok] * 6
    outs = [ok] * 5
    assert bc(2, 64, 32, *base, *none3, *none3, *outs, *none3, ok, need - 1, None) == 1
    assert bc(2, 64, 32, *base, [ok, None, ok][0], None, ok, *none3, *outs, *none3, ok, need,
              None) == 1
    assert bc(0, 64, 32, *base, *none3, *none3, *outs, *none3, ok, need, None) == 0


def declared_signatures():
    """{name: [parameter types]} of every WKV_API function in include/*.h."""
    sigs = {}
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        text = re.sub(r"/\*.*?\*/", " ", open(os.path.join(ROOT, "include", h)).read(), flags=re.S)
        for m in re.finditer(r"WKV_API\s+[\w\s\*]+?\b(\w+)\s*\(([^)]*)\)\s*;", text):
            params = [p.strip() for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
            sigs[m.group(1)] = [re.sub(r"\s+\w+$", "", p) for p in params]
    return sigs


def test_binding_matches_the_declarations(W):
    # Every function the binding types matches its declaration parameter for parameter:
    # 64-bit sizes, ints, size_t and pointers (including the stream) where the header has them.
    from rwkv_linear_attention_wkv_b200 import _SIGS
    sigs = declared_signatures()
    # (size_t and uint64_t are the same 64-bit unsigned type on this ABI, as are their
    # ctypes names)
    kinds = {ctypes.c_int64: "i64", ctypes.c_int: "int", ctypes.c_size_t: "u64",
             ctypes.c_uint64: "u64", ctypes.c_void_p: "ptr"}

    def kind(t):
        t = t.replace("const ", "").strip()
        if t.endswith("*") or t == "cudaStream_t":
            return "ptr"
        return {"int64_t": "i64", "int": "int", "size_t": "u64", "uint64_t": "u64"}[t]

    def ctype_kind(a):  # typed pointers (e.g. POINTER(c_double)) are pointers too
        return "ptr" if isinstance(a, type) and issubclass(a, ctypes._Pointer) else kinds[a]

    for name, (args, _) in _SIGS.items():
        assert name in sigs, name
        assert [ctype_kind(a) for a in args] == [kind(t) for t in sigs[name]], name


def test_backward_path_hook_values(W):
    # The test hook that chooses the backward's reverse pass is host-only state: 0..3 are
    # accepted, anything else is refused, and the automatic choice is restored.
    f = W.lib.wkv_testing_set_backward_path
    try:
        for path in (0, 1, 2, 3):
            assert f(path) == 0
        for path in (-1, 4, 100):
            assert f(path) == 1  # WKV_ERR_INVALID_ARG
    finally:
        assert f(0) == 0


def test_pipe_probe_argument_checks(W):
    # Refused before anything touches a device.
    out = ctypes.c_double(0.0)
    f = W.lib.wkv_testing_pipe_rate
    assert f(7, 10, ctypes.byref(out), None) == 1
    assert f(0, 0, ctypes.byref(out), None) == 1
    assert f(1, -5, ctypes.byref(out), None) == 1
    assert f(0, 10, None, None) == 1


def test_binding_refuses_host_tensors_and_wrong_dtypes(W):
    # The product path has no CPU implementation: the binding refuses host tensors (and
    # objects that are not tensors) before anything is launched, rather than computing
    # anywhere else.
    import torch
    C = 8
    w, u = torch.ones(C), torch.zeros(C)
    k = v = r = torch.zeros(1, 4, C)
    with pytest.raises(ValueError, match="CUDA tensor"):
        W.wkv_forward(w, u, k, v, r)
    with pytest.raises(ValueError, match="CUDA tensor"):
        W.wkv_forward_bf16(w, u, k.bfloat16(), v.bfloat16(), r.bfloat16())
    with pytest.raises(ValueError, match="CUDA tensor"):
        W.wkv_backward(w, u, k, v, r, k)
    with pytest.raises(TypeError, match="torch.Tensor"):
        W.wkv_forward(w, u, k.numpy(), v, r)
