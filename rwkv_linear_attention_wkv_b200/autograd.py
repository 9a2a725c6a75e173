"""The WKV operator as a PyTorch autograd function (argument marshalling only).

The news page "RWKV CUDA linear attention GPU" describes the CUDA operator being used
from PyTorch through an autograd function whose forward and backward are fused kernels.
This module is that wrapper over the library's C ABI: the forward is
`wkv_forward_checkpointed` (y, and the state entering every 16-token chunk kept in a
workspace saved for the backward), the backward is `wkv_backward_checkpointed` (dk, dv,
dr, dw, du from those checkpoints). Nothing here computes: every number comes from the
library's kernels, on the current CUDA stream, in fp32.

    y = wkv(w, u, k, v, r)        # w, u: (C,) fp32, w > 0; k, v, r: (B, T, C) fp32 CUDA
    (y * dy).sum().backward()     # gradients for w, u, k, v and r

w is the positive decay itself (the per-token factor is e^{-w}), so w's gradient is with
respect to w, not log w. r may be None (no gate).
"""
import torch

from . import wkv_backward_checkpointed, wkv_forward_checkpointed


class WKVFunction(torch.autograd.Function):
    """y = sigmoid(r) * wkv(w, u, k, v) with its gradients from the library's kernels."""

    @staticmethod
    def forward(ctx, w, u, k, v, r):
        w, u, k, v = (t.contiguous() for t in (w, u, k, v))
        r = None if r is None else r.contiguous()
        y, workspace = wkv_forward_checkpointed(w, u, k, v, r)
        ctx.save_for_backward(w, u, k, v, r, workspace)
        ctx.has_r = r is not None
        return y

    @staticmethod
    def backward(ctx, dy):
        w, u, k, v, r, workspace = ctx.saved_tensors
        g = wkv_backward_checkpointed(w, u, k, v, r if ctx.has_r else None, dy.contiguous(),
                                      workspace, want_dr=ctx.has_r)
        return g["dw"], g["du"], g["dk"], g["dv"], g["dr"]


def wkv(w, u, k, v, r=None):
    """Differentiable WKV: see WKVFunction."""
    return WKVFunction.apply(w, u, k, v, r)
