"""Token-chunked linear layer with an activation, whose backward recomputes instead of storing.

Helios kernels article, section "内核三 TiledLinear": the layer y = act(x W^T + b) runs along the
token dimension in chunks (each chunk's output written into the full output), and the backward
keeps no intermediate activation: it recomputes each chunk's pre-activation z from x, then
forms that chunk's gradients. Memory for the layer's intermediates falls with the chunk count;
the price is the recomputed forward. The default chunk count is ceil(tokens / hidden).

Where each step runs (all on this library's kernels):
  * forward and recompute: ``gn_norm_linear_fwd`` with ``GN_NORM_NONE`` (the tcgen05 kernels; the
    bias and activation in their epilogue);
  * dz = dy * act'(z): ``gn_linear_act_grad``, the recompute with the activation gradient applied
    where the accumulators are read back (z never reaches memory);
  * dx = dz W: ``gn_norm_linear_fwd`` on dz with W^T (``gn_transpose``, once per backward) as the
    weight operand;
  * dW += dz^T x: ``gn_linear_acc_f32`` on the transposed chunk operands (the tokens, over which
    the product contracts, made contiguous by ``gn_transpose``), accumulating in fp32 in place;
  * db += sum dz: ``gn_colsum_bf16`` (fixed order).
This module only orchestrates chunks (host logic); every elementwise and fused step is a kernel
of the library.
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import transformer_norm_rope_b200 as gn


def default_chunks(tokens: int, hidden: int) -> int:
    """The chunk count the article's layer picks when none is given: ceil(tokens / hidden)."""
    return max(1, math.ceil(tokens / max(1, hidden)))


def _bounds(rows: int, chunks: int):
    step = math.ceil(rows / chunks) if rows else 0
    # 8-row multiples keep every chunk's rows 16-byte aligned for the kernels
    step = (step + 7) // 8 * 8 if step else 0
    r0 = 0
    while r0 < rows:
        r1 = min(rows, r0 + step)
        yield r0, r1
        r0 = r1


def prepare(W, bias=None):
    """The layer weight in the form the forward kernels read (bf16 W as is, bias as fp32)."""
    Wf, _, d = gn.norm_linear_prepare(W, None, None, bias, norm="none")
    return Wf, d


def forward(x, Wf, d, act: str = "silu", chunks: Optional[int] = None):
    """y [M, N] = act(x W^T + b), computed chunk by chunk along the M tokens of x [M, K]."""
    torch = gn._torch()
    M, K = x.shape
    N = Wf.shape[0]
    chunks = chunks or default_chunks(M, K)
    y = torch.empty((M, N), dtype=x.dtype, device=x.device)
    for r0, r1 in _bounds(M, chunks):
        gn.norm_linear_fwd(x[r0:r1], Wf, None, d, norm="none", epilogue=act, save_stats=False, out=y[r0:r1])
    return y


def backward(x, Wf, d, dy, act: str = "silu", chunks: Optional[int] = None) -> Tuple:
    """Gradients of sum(dy * y) -> (dx [M, K] bf16, dW [N, K] fp32, db [N] fp32), recomputing each
    chunk's pre-activation instead of reading a stored one."""
    torch = gn._torch()
    M, K = x.shape
    N = Wf.shape[0]
    chunks = chunks or default_chunks(M, K)
    dx = torch.empty_like(x)
    dW = torch.zeros((N, K), dtype=torch.float32, device=x.device)
    db = torch.zeros(N, dtype=torch.float32, device=x.device)
    Wt = gn.transpose(Wf)  # [K, N]: the weight operand of dx = dz W
    ws = torch.empty(max(gn.gn_colsum_bf16_workspace(N), 16), dtype=torch.uint8, device=x.device)
    for r0, r1 in _bounds(M, chunks):
        xc = x[r0:r1]
        dz = gn.linear_act_grad(xc, Wf, d, dy[r0:r1], epilogue=act)
        gn.norm_linear_fwd(dz, Wt, None, None, norm="none", epilogue="none", save_stats=False, out=dx[r0:r1])
        # dW += dz^T x contracts over the chunk's tokens: both operands with the tokens contiguous
        # (zero-padded to a multiple of 8 tokens)
        gn.linear_acc_f32(gn.transpose(dz), gn.transpose(xc), dW)
        gn.colsum_bf16(dz, db, accumulate=True, ws=ws)
    return dx, dW, db


def _function_class():
    torch = gn._torch()

    class _TiledLinear(torch.autograd.Function):
        @staticmethod
        def forward(ctx, x, W, bias, act, chunks):
            Wf, d = prepare(W, bias)
            ctx.save_for_backward(x, Wf, d)
            ctx.act, ctx.chunks = act, chunks
            ctx.w_dtype = W.dtype
            ctx.b_dtype = None if bias is None else bias.dtype
            return forward(x, Wf, d, act, chunks)

        @staticmethod
        def backward(ctx, dy):
            x, Wf, d = ctx.saved_tensors
            dx, dW, db = backward(x, Wf, d, dy.contiguous(), ctx.act, ctx.chunks)
            return dx, dW.to(ctx.w_dtype), (None if ctx.b_dtype is None else db.to(ctx.b_dtype)), None, None

    return _TiledLinear


_FUNCTION = None


class TiledLinearFunction:
    """torch.autograd.Function form: saves only x (and the weight), recomputes in backward."""

    @staticmethod
    def apply(x, W, bias, act: str = "silu", chunks: Optional[int] = None):
        global _FUNCTION
        if _FUNCTION is None:
            _FUNCTION = _function_class()
        return _FUNCTION.apply(x, W, bias, act, chunks)
