"""Python binding of libwkv.so, the B200 (sm_100a) WKV library.

Argument marshalling only: every function checks the torch tensors it is given (device,
dtype, contiguity, shape), allocates outputs the caller did not pass, and calls the C
entry point of the same name (include/wkv.h) on the current CUDA stream. All arithmetic
runs in the library's CUDA kernels; there is no fallback. Importing this package fails
loudly when libwkv.so has not been built.
"""
from __future__ import annotations

import ctypes
import os

__all__ = ["wkv_forward", "wkv_forward_bf16", "wkv_forward_state", "wkv_decode_step",
           "wkv_decode_steps",
           "wkv_backward", "wkv_backward_state", "wkv_backward_workspace_bytes",
           "wkv_forward_checkpointed", "wkv_backward_checkpointed",
           "wkv7_forward", "wkv_mstate_forward", "wkv_stream_status", "wkv_status_string", "WkvError", "lib",
           "LIB_PATH"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libwkv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python rwkv_linear_attention_wkv_b200/build.py`"
        " (the WKV operator has no non-CUDA implementation)")

lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int64
_SIGS = {
    "wkv_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "wkv_version": ([], ctypes.c_int),
    "wkv_forward": ([_I, _I, _I] + [_P] * 6 + [_P], ctypes.c_int),
    "wkv_forward_bf16": ([_I, _I, _I] + [_P] * 6 + [_P], ctypes.c_int),
    "wkv_forward_state": ([_I, _I, _I] + [_P] * 12 + [_P], ctypes.c_int),
    "wkv_decode_step": ([_I, _I, _I] + [_P] * 9 + [_P], ctypes.c_int),
    "wkv_decode_steps": ([_I, _I, _I, _I] + [_P] * 9 + [_P], ctypes.c_int),
    "wkv_stream_status": ([_P], ctypes.c_int),
    "wkv_backward_workspace_bytes": ([_I, _I, _I], ctypes.c_size_t),
    "wkv_backward": ([_I, _I, _I] + [_P] * 12 + [ctypes.c_size_t, _P], ctypes.c_int),
    "wkv_testing_backward_plain": ([_I, _I, _I] + [_P] * 12 + [ctypes.c_size_t, _P],
                                   ctypes.c_int),
    "wkv_backward_state": ([_I, _I, _I] + [_P] * 21 + [ctypes.c_size_t, _P], ctypes.c_int),
    "wkv7_forward": ([_I, _I, _I, _I] + [_P] * 9 + [_P], ctypes.c_int),
    "wkv_mstate_forward": ([_I, _I, _I, _I] + [_P] * 7 + [_P], ctypes.c_int),
    "wkv_forward_checkpointed": ([_I, _I, _I] + [_P] * 10 + [ctypes.c_size_t, _P], ctypes.c_int),
    "wkv_backward_checkpointed": ([_I, _I, _I] + [_P] * 21 + [ctypes.c_size_t, _P],
                                  ctypes.c_int),
    "wkv_testing_backward_state_plain": ([_I, _I, _I] + [_P] * 21 + [ctypes.c_size_t, _P],
                                         ctypes.c_int),
    "wkv_testing_lookback_timeout": ([ctypes.c_uint64, _P], ctypes.c_int),
    "wkv_testing_backward_timeout": ([ctypes.c_uint64, _P], ctypes.c_int),
    "wkv_testing_forward_plain": ([_I, _I, _I] + [_P] * 6 + [ctypes.c_int, _P], ctypes.c_int),
    "wkv_testing_set_backward_path": ([ctypes.c_int], ctypes.c_int),
    "wkv_testing_pipe_rate": ([ctypes.c_int, _I, ctypes.POINTER(ctypes.c_double), _P],
                              ctypes.c_int),
}
for _name, (_args, _res) in _SIGS.items():
    try:
        _f = getattr(lib, _name)
    except AttributeError as _e:
        raise ImportError(f"{LIB_PATH} lacks {_name}: it is older than the sources; rebuild it "
                          "with `python rwkv_linear_attention_wkv_b200/build.py`") from _e
    _f.argtypes = _args
    _f.restype = _res


class WkvError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {wkv_status_string(status)} ({status})")
        self.status = status


def wkv_status_string(status: int) -> str:
    return lib.wkv_status_string(int(status)).decode()


def _torch():
    import torch
    return torch


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, name, dtype, shape=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _dims(t, name, n):
    """Whether t has n dimensions; t must be a tensor (checked before its shape is read)."""
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    return t.dim() == n


def _call(fn, *args):
    rc = getattr(lib, fn)(*args)
    if rc != 0:
        raise WkvError(fn, rc)


def _fwd_common(w, u, k, v, r, y, dtype):
    torch = _torch()
    if not _dims(k, "k", 3):
        raise ValueError("k must be (B, T, C)")
    B, T, C = k.shape
    _need(k, "k", dtype)
    _need(v, "v", dtype, (B, T, C))
    if r is not None:
        _need(r, "r", dtype, (B, T, C))
    _need(w, "w", torch.float32, (C,))
    _need(u, "u", torch.float32, (C,))
    if y is None:
        y = torch.empty((B, T, C), dtype=dtype, device=k.device)
    _need(y, "y", dtype, (B, T, C))
    return B, T, C, y


def wkv_forward(w, u, k, v, r=None, y=None, stream=None):
    """fp32 forward: y = sigmoid(r) * wkv (no gate when r is None). Returns y."""
    torch = _torch()
    B, T, C, y = _fwd_common(w, u, k, v, r, y, torch.float32)
    _call("wkv_forward", B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(y),
          _stream(stream))
    return y


def wkv_forward_bf16(w, u, k, v, r=None, y=None, stream=None):
    """bf16 in/out forward (fp32 arithmetic). Returns y (bf16)."""
    torch = _torch()
    B, T, C, y = _fwd_common(w, u, k, v, r, y, torch.bfloat16)
    _call("wkv_forward_bf16", B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(y),
          _stream(stream))
    return y


def wkv_forward_state(w, u, k, v, r=None, state=None, y=None, state_out=None,
                      want_state=True, stream=None):
    """fp32 forward with state. state = (a, b, p) fp32 [B, C] or None (empty).

    Returns (y, (a1, b1, p1)), or (y, None) with want_state=False. state_out may be given
    (and may be the same tensors as state) to write the final state in place.
    """
    torch = _torch()
    B, T, C, y = _fwd_common(w, u, k, v, r, y, torch.float32)
    a0 = b0 = p0 = None
    if state is not None:
        a0, b0, p0 = state
        for n, t in (("a0", a0), ("b0", b0), ("p0", p0)):
            _need(t, n, torch.float32, (B, C))
    a1 = b1 = p1 = None
    if want_state:
        if state_out is None:
            state_out = tuple(torch.empty((B, C), dtype=torch.float32, device=k.device)
                              for _ in range(3))
        a1, b1, p1 = state_out
        for n, t in (("a1", a1), ("b1", b1), ("p1", p1)):
            _need(t, n, torch.float32, (B, C))
    _call("wkv_forward_state", B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(y),
          _ptr(a0), _ptr(b0), _ptr(p0), _ptr(a1), _ptr(b1), _ptr(p1), _stream(stream))
    return y, ((a1, b1, p1) if want_state else None)


def wkv_decode_step(w, u, k, v, r, a, b, p, y=None, stream=None):
    """One token for [N, L, C] states; w, u [L, C]; (a, b, p) updated in place. Returns y."""
    torch = _torch()
    if not _dims(k, "k", 3):
        raise ValueError("k must be (N, L, C)")
    N, L, C = k.shape
    f32 = torch.float32
    _need(k, "k", f32)
    for n, t in (("v", v), ("a", a), ("b", b), ("p", p)):
        _need(t, n, f32, (N, L, C))
    if r is not None:
        _need(r, "r", f32, (N, L, C))
    _need(w, "w", f32, (L, C))
    _need(u, "u", f32, (L, C))
    if y is None:
        y = torch.empty((N, L, C), dtype=f32, device=k.device)
    _need(y, "y", f32, (N, L, C))
    _call("wkv_decode_step", N, L, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(y),
          _ptr(a), _ptr(b), _ptr(p), _stream(stream))
    return y


def wkv_decode_steps(w, u, k, v, r, a, b, p, y=None, stream=None):
    """S chained tokens for [N, L, C] states in one call: k, v, r (S, N, L, C); w, u
    [L, C]; (a, b, p) updated in place. Returns y (S, N, L, C)."""
    torch = _torch()
    if not _dims(k, "k", 4):
        raise ValueError("k must be (S, N, L, C)")
    S, N, L, C = k.shape
    f32 = torch.float32
    _need(k, "k", f32)
    _need(v, "v", f32, (S, N, L, C))
    if r is not None:
        _need(r, "r", f32, (S, N, L, C))
    for n, t in (("a", a), ("b", b), ("p", p)):
        _need(t, n, f32, (N, L, C))
    _need(w, "w", f32, (L, C))
    _need(u, "u", f32, (L, C))
    if y is None:
        y = torch.empty((S, N, L, C), dtype=f32, device=k.device)
    _need(y, "y", f32, (S, N, L, C))
    _call("wkv_decode_steps", N, L, C, S, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
          _ptr(y), _ptr(a), _ptr(b), _ptr(p), _stream(stream))
    return y


def wkv_backward_workspace_bytes(B: int, T: int, C: int) -> int:
    return int(lib.wkv_backward_workspace_bytes(B, T, C))


def wkv_backward(w, u, k, v, r, dy, want_dr=True, workspace=None, out=None, stream=None,
                 _entry="wkv_backward"):
    """fp32 gradients of sum(dy * y) for y = wkv_forward(w, u, k, v, r).

    Returns a dict with dk, dv (B, T, C), dw, du (C,) and dr (B, T, C; None when r is None
    or want_dr is False). `workspace` (uint8 CUDA tensor of at least
    wkv_backward_workspace_bytes(B, T, C) bytes) is allocated when not given; `out` may
    hold preallocated dk, dv, dw, du, dr tensors.
    """
    torch = _torch()
    f32 = torch.float32
    if not _dims(k, "k", 3):
        raise ValueError("k must be (B, T, C)")
    B, T, C = k.shape
    _need(k, "k", f32)
    for n, t in (("v", v), ("dy", dy)):
        _need(t, n, f32, (B, T, C))
    if r is not None:
        _need(r, "r", f32, (B, T, C))
    _need(w, "w", f32, (C,))
    _need(u, "u", f32, (C,))
    out = dict(out or {})
    dev = k.device
    for n, shape in (("dk", (B, T, C)), ("dv", (B, T, C)), ("dw", (C,)), ("du", (C,))):
        if out.get(n) is None:
            out[n] = torch.empty(shape, dtype=f32, device=dev)
        _need(out[n], n, f32, shape)
    if r is not None and want_dr:
        if out.get("dr") is None:
            out["dr"] = torch.empty((B, T, C), dtype=f32, device=dev)
        _need(out["dr"], "dr", f32, (B, T, C))
    else:
        out["dr"] = None
    nbytes = wkv_backward_workspace_bytes(B, T, C)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    if not workspace.is_cuda or workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError(f"workspace must be a CUDA tensor of at least {nbytes} bytes")
    _call(_entry, B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(dy),
          _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dw"]), _ptr(out["du"]), _ptr(out["dr"]),
          _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    return out


def wkv_backward_state(w, u, k, v, r, dy, state=None, grad_state=None, want_dr=True,
                       workspace=None, out=None, stream=None, _entry="wkv_backward_state"):
    """fp32 gradients for y, (a1, b1, p1) = wkv_forward_state(w, u, k, v, r, state).

    `state` = (a0, b0, p0) or None (empty); `grad_state` = (ga1, gb1, p1): the gradients
    of a later loss with respect to the final state's a1, b1, and that state's p1; or None.
    Returns the dict of wkv_backward plus da0, db0, dp0 (B, C). Chaining: pass a piece's
    (da0, db0, p0) as the previous piece's grad_state.
    """
    torch = _torch()
    f32 = torch.float32
    if not _dims(k, "k", 3):
        raise ValueError("k must be (B, T, C)")
    B, T, C = k.shape
    _need(k, "k", f32)
    for n, t in (("v", v), ("dy", dy)):
        _need(t, n, f32, (B, T, C))
    if r is not None:
        _need(r, "r", f32, (B, T, C))
    _need(w, "w", f32, (C,))
    _need(u, "u", f32, (C,))
    st = tuple(state) if state is not None else (None, None, None)
    gs = tuple(grad_state) if grad_state is not None else (None, None, None)
    for n, t in zip(("a0", "b0", "p0", "ga1", "gb1", "p1"), st + gs):
        if t is not None:
            _need(t, n, f32, (B, C))
    out = dict(out or {})
    dev = k.device
    for n, shape in (("dk", (B, T, C)), ("dv", (B, T, C)), ("dw", (C,)), ("du", (C,)),
                     ("da0", (B, C)), ("db0", (B, C)), ("dp0", (B, C))):
        if out.get(n) is None:
            out[n] = torch.empty(shape, dtype=f32, device=dev)
        _need(out[n], n, f32, shape)
    if r is not None and want_dr:
        if out.get("dr") is None:
            out["dr"] = torch.empty((B, T, C), dtype=f32, device=dev)
        _need(out["dr"], "dr", f32, (B, T, C))
    else:
        out["dr"] = None
    nbytes = wkv_backward_workspace_bytes(B, T, C)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    if not workspace.is_cuda or workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError(f"workspace must be a CUDA tensor of at least {nbytes} bytes")
    _call(_entry, B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(dy),
          *(_ptr(t) for t in st + gs),
          _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dw"]), _ptr(out["du"]), _ptr(out["dr"]),
          _ptr(out["da0"]), _ptr(out["db0"]), _ptr(out["dp0"]),
          _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    return out


def wkv_forward_checkpointed(w, u, k, v, r=None, state=None, y=None, workspace=None,
                             stream=None):
    """fp32 forward of a training step that also writes the backward's checkpoints.

    y as wkv_forward_state(w, u, k, v, r, state) (no final state); the checkpoints go into
    `workspace` (uint8 CUDA tensor of at least wkv_backward_workspace_bytes(B, T, C) bytes,
    allocated when not given). Returns (y, workspace); hand the workspace, unchanged, to
    wkv_backward_checkpointed with the same w, u, k, v and state.
    """
    torch = _torch()
    f32 = torch.float32
    if not _dims(k, "k", 3):
        raise ValueError("k must be (B, T, C)")
    B, T, C = k.shape
    _need(k, "k", f32)
    _need(v, "v", f32, (B, T, C))
    if r is not None:
        _need(r, "r", f32, (B, T, C))
    _need(w, "w", f32, (C,))
    _need(u, "u", f32, (C,))
    st = tuple(state) if state is not None else (None, None, None)
    for n, t in zip(("a0", "b0", "p0"), st):
        if t is not None:
            _need(t, n, f32, (B, C))
    if y is None:
        y = torch.empty((B, T, C), dtype=f32, device=k.device)
    _need(y, "y", f32, (B, T, C))
    nbytes = wkv_backward_workspace_bytes(B, T, C)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=k.device)
    if not workspace.is_cuda or workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError(f"workspace must be a CUDA tensor of at least {nbytes} bytes")
    _call("wkv_forward_checkpointed", B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
          _ptr(y), *(_ptr(t) for t in st), _ptr(workspace),
          workspace.numel() * workspace.element_size(), _stream(stream))
    return y, workspace


def wkv_backward_checkpointed(w, u, k, v, r, dy, workspace, state=None, grad_state=None,
                              want_dr=True, out=None, stream=None):
    """wkv_backward_state, using the checkpoints wkv_forward_checkpointed left in
    `workspace` (same w, u, k, v and state) instead of forming them again."""
    if workspace is None:
        raise ValueError("workspace: the one wkv_forward_checkpointed filled")
    return wkv_backward_state(w, u, k, v, r, dy, state=state, grad_state=grad_state,
                              want_dr=want_dr, workspace=workspace, out=out, stream=stream,
                              _entry="wkv_backward_checkpointed")


def wkv7_forward(r, w, k, v, a, b, state=None, y=None, state_out=None, want_state=True,
                 stream=None):
    """RWKV-7 recurrence per head: r, w, k, v, a, b fp32 (B, T, H, N), N = 64; state
    (B, H, N, N) or None (zero). Returns (y, S_T), or (y, None) with want_state=False.
    state_out may be given (and may be `state` itself)."""
    torch = _torch()
    f32 = torch.float32
    if not _dims(k, "k", 4):
        raise ValueError("k must be (B, T, H, N)")
    B, T, H, N = k.shape
    for n, t in (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("b", b)):
        _need(t, n, f32, (B, T, H, N))
    if y is None:
        y = torch.empty((B, T, H, N), dtype=f32, device=k.device)
    _need(y, "y", f32, (B, T, H, N))
    if state is not None:
        _need(state, "state", f32, (B, H, N, N))
    s1 = None
    if want_state:
        s1 = state_out if state_out is not None else torch.empty((B, H, N, N), dtype=f32,
                                                                 device=k.device)
        _need(s1, "state_out", f32, (B, H, N, N))
    _call("wkv7_forward", B, T, H, N, _ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
          _ptr(y), _ptr(state), _ptr(s1), _stream(stream))
    return y, s1


def wkv_mstate_forward(r, w, k, v, state=None, y=None, state_out=None, want_state=True,
                       stream=None):
    """Matrix-valued-state WKV (per-key-channel decay, no delta term), chunked on the tensor
    cores: r, w, k, v fp32 (B, T, H, N), N = 64; state (B, H, N, N) or None (zero). Returns
    (y, S_T), or (y, None) with want_state=False. state_out may be `state` itself."""
    torch = _torch()
    f32 = torch.float32
    if not _dims(k, "k", 4):
        raise ValueError("k must be (B, T, H, N)")
    B, T, H, N = k.shape
    for n, t in (("r", r), ("w", w), ("k", k), ("v", v)):
        _need(t, n, f32, (B, T, H, N))
    if y is None:
        y = torch.empty((B, T, H, N), dtype=f32, device=k.device)
    _need(y, "y", f32, (B, T, H, N))
    if state is not None:
        _need(state, "state", f32, (B, H, N, N))
    s1 = None
    if want_state:
        s1 = state_out if state_out is not None else torch.empty((B, H, N, N), dtype=f32,
                                                                 device=k.device)
        _need(s1, "state_out", f32, (B, H, N, N))
    _call("wkv_mstate_forward", B, T, H, N, _ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(y),
          _ptr(state), _ptr(s1), _stream(stream))
    return y, s1


def wkv_stream_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device-side status code."""
    return int(lib.wkv_stream_status(_stream(stream)))
