"""B200-native sum-of-Kronecker-products linear layer.

    y = x W + bias,   W = sum_{i<r} kron(S (.) A_i, B_i)

(page "kronecker-layer-benchmark", section "1. Build W, then multiply") computed
with the vec trick by the hand-written sm_100a kernels of libkronlinear.so; W is
never materialised.  ``native`` is the ctypes binding of the C ABI
(include/kron_linear.h); ``KronLinearFunction`` / ``KronLinear`` wrap it for
autograd.  PyTorch is used for device memory and streams only.

The same library holds the Kronecker-sparse factor of the page "Fast Inference
with Kronecker-Sparse Matrices" (support kron(I_a, kron(1_{b x c}, I_d)),
include/ks_linear.h): ``native.ks_forward`` / ``native.ks_backward``, wrapped by
``KSLinearFunction`` / ``KSLinear``.
"""
from __future__ import annotations

import math

import torch

from . import accounting, native
from .native import KronError, backward, forward, workspace_size

__all__ = ["native", "accounting", "forward", "backward", "workspace_size", "KronError",
           "KronLinearFunction", "KronLinear", "kron_linear", "KSLinearFunction", "KSLinear",
           "ks_linear"]


class KronLinearFunction(torch.autograd.Function):
    """Autograd wrapper: forward and backward both run in the CUDA library.

    Nothing but the inputs is saved; the backward recomputes X_n B_i on chip.
    Factor gradients come back in float32 and are cast to the parameters' dtype.
    ``l1`` > 0 makes S's gradient include that of the penalty l1 * sum|S| (added in the
    library's dS epilogue); the penalty's value is not part of the output.
    """

    @staticmethod
    def forward(ctx, x, S, A, B, bias, dtype, flags, l1=0.0):
        ctx.save_for_backward(x, S, A, B)
        ctx.dtype, ctx.flags, ctx.has_bias, ctx.l1 = dtype, flags, bias is not None, l1
        return forward(x, S, A, B, bias, dtype=dtype, flags=flags)

    @staticmethod
    def backward(ctx, dY):
        x, S, A, B = ctx.saved_tensors
        g = backward(x, S, A, B, dY.contiguous(), dtype=ctx.dtype, flags=ctx.flags,
                     need_dx=ctx.needs_input_grad[0], need_dbias=ctx.has_bias, l1=ctx.l1)
        cast = lambda t, like: None if t is None else t.to(like.dtype)
        dbias = cast(g["dbias"], S) if ctx.has_bias else None
        return (g["dX"], cast(g["dS"], S), cast(g["dA"], A), cast(g["dB"], B), dbias,
                None, None, None)


def kron_linear(x, S, A, B, bias=None, dtype="tf32", flags=0, l1=0.0):
    return KronLinearFunction.apply(x, S, A, B, bias, dtype, flags, l1)


class KronLinear(torch.nn.Module):
    """Drop-in linear layer with W = sum_i kron(S (.) A_i, B_i), W of shape
    (p*m1) x (q*m2); initialised as on the page "kronecker-layer-benchmark"
    (S = ones, A_i ~ randn/sqrt(p), B_i ~ randn/sqrt(m1), bias = zeros).

    ``l1`` > 0 trains S under the page's penalty l1 * sum|S| with its gradient fused into
    the backward's dS epilogue; the loss the caller computes then leaves the penalty out."""

    def __init__(self, in_features, out_features, block_in, block_out=None, rank=1,
                 bias=True, dtype="tf32", flags=0, device=None, l1=0.0):
        super().__init__()
        block_out = block_in if block_out is None else block_out
        if in_features % block_in or out_features % block_out:
            raise ValueError("features must be multiples of the block size")
        p, q = in_features // block_in, out_features // block_out
        t = native.io_dtype(dtype)
        kw = dict(device=device, dtype=t)
        self.S = torch.nn.Parameter(torch.ones(p, q, **kw))
        self.A = torch.nn.Parameter(torch.randn(rank, p, q, **kw) / math.sqrt(p))
        self.B = torch.nn.Parameter(torch.randn(rank, block_in, block_out, **kw) / math.sqrt(block_in))
        self.bias = torch.nn.Parameter(torch.zeros(out_features, **kw)) if bias else None
        self.path, self.flags, self.l1 = dtype, flags, float(l1)

    def forward(self, x):
        shp = x.shape
        y = kron_linear(x.reshape(-1, shp[-1]).contiguous(), self.S, self.A, self.B, self.bias,
                        self.path, self.flags, self.l1)
        return y.reshape(*shp[:-1], y.shape[-1])


class KSLinearFunction(torch.autograd.Function):
    """Autograd wrapper of the Kronecker-sparse factor; both passes run in the CUDA library."""

    @staticmethod
    def forward(ctx, x, w, bias):
        ctx.save_for_backward(x, w)
        ctx.has_bias = bias is not None
        return native.ks_forward(x, w, bias)

    @staticmethod
    def backward(ctx, dY):
        x, w = ctx.saved_tensors
        g = native.ks_backward(x, w, dY.contiguous(), need_dx=ctx.needs_input_grad[0],
                               need_dbias=ctx.has_bias)
        return g["dX"], g["dw"], g["dbias"]


def ks_linear(x, w, bias=None):
    return KSLinearFunction.apply(x, w, bias)


class KSLinear(torch.nn.Module):
    """Linear layer y = x K + bias whose weight K is Kronecker-sparse with pattern
    (a, b, c, d): supp K = kron(I_a, kron(1_{b x c}, I_d)), in = a*b*d, out = a*c*d.
    The a*d dense b x c blocks are initialised with std 1/sqrt(b) (each output sums b
    inputs); FP32 only.  Butterfly and Monarch layers are sequences of these."""

    def __init__(self, a, b, c, d, bias=True, device=None):
        super().__init__()
        kw = dict(device=device, dtype=torch.float32)
        self.pattern = (a, b, c, d)
        self.w = torch.nn.Parameter(torch.randn(a, d, b, c, **kw) / math.sqrt(b))
        self.bias = torch.nn.Parameter(torch.zeros(a * c * d, **kw)) if bias else None

    def forward(self, x):
        shp = x.shape
        y = ks_linear(x.reshape(-1, shp[-1]).contiguous(), self.w, self.bias)
        return y.reshape(*shp[:-1], y.shape[-1])
