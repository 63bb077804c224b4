"""Token-chunked linear layer with an activation, whose backward recomputes instead of storing.

Helios kernels article, section "内核三 TiledLinear": the layer y = act(x W^T + b) runs along the
token dimension in chunks (each chunk's output written into the full output), and the backward
keeps no intermediate activation: it recomputes each chunk's pre-activation z from x, then
forms that chunk's gradients. Memory for the layer's intermediates falls with the chunk count;
the price is the recomputed forward. The default chunk count is ceil(tokens / hidden).
With the activation fused into the tensor-core epilogue the forward has no intermediate, so it
runs unchunked by default; the backward's intermediate is each chunk's dz.

Where each step runs (all on this library's kernels):
  * forward and recompute: ``gn_norm_linear_fwd`` with ``GN_NORM_NONE`` (the tcgen05 kernels; the
    bias and activation in their epilogue);
  * dz = dy * act'(z): ``gn_linear_act_grad``, the recompute with the activation gradient applied
    where the accumulators are read back (z never reaches memory);
  * dx = dz W: ``gn_linear_bf16`` with W read as an MN-major operand (no transposed copy);
  * dW += dz^T x: ``gn_linear_acc_f32`` contracting over the chunk's tokens, both operands read
    MN-major straight from dz and x, accumulating in fp32 in place;
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


# rows of one tensor-core output tile (a pair of SMs covers 256 rows)
_TILE_ROWS = 256


def _bounds(rows: int, chunks: int):
    """Contiguous row ranges of about rows / chunks rows each. Every range starts on a multiple of
    8 rows (16-byte aligned rows for the kernels) and, where that keeps the number of ranges, on a
    multiple of the 256-row output tile, so that no chunk's products pay for a partly empty tile
    row in the middle of the tensor."""
    step = math.ceil(rows / chunks) if rows else 0
    step8 = (step + 7) // 8 * 8 if step else 0
    step_t = (step + _TILE_ROWS - 1) // _TILE_ROWS * _TILE_ROWS if step else 0
    if step and math.ceil(rows / step_t) == math.ceil(rows / step8):
        step8 = step_t
    r0 = 0
    while r0 < rows:
        r1 = min(rows, r0 + step8)
        yield r0, r1
        r0 = r1


def prepare(W, bias=None):
    """The layer weight in the form the forward kernels read (bf16 W as is, bias as fp32)."""
    Wf, _, d = gn.norm_linear_prepare(W, None, None, bias, norm="none")
    return Wf, d


def forward(x, Wf, d, act: str = "silu", chunks: Optional[int] = None):
    """y [M, N] = act(x W^T + b) for x [M, K]. The activation is applied where the tensor-core
    kernel reads its accumulators back, so the forward keeps no intermediate at all: by default
    (chunks None) it runs as one launch over every token; with a chunk count it runs chunk by
    chunk (the same values, bit for bit: the rows are independent)."""
    torch = gn._torch()
    M, K = x.shape
    N = Wf.shape[0]
    y = torch.empty((M, N), dtype=x.dtype, device=x.device)
    for r0, r1 in _bounds(M, chunks or 1):
        gn.norm_linear_fwd(x[r0:r1], Wf, None, d, norm="none", epilogue=act, save_stats=False, out=y[r0:r1])
    return y


def _stream_pair(device):
    """The caller's current stream and a second stream (from torch's pool) for the dx products."""
    torch = gn._torch()
    return torch.cuda.current_stream(device), torch.cuda.Stream(device=device)


def _event():
    return gn._torch().cuda.Event()


def backward(x, Wf, d, dy, act: str = "silu", chunks: Optional[int] = None) -> Tuple:
    """Gradients of sum(dy * y) -> (dx [M, K] bf16, dW [N, K] fp32, db [N] fp32), recomputing each
    chunk's pre-activation instead of reading a stored one (default chunk count ceil(M / K)).

    Per chunk, on the caller's stream: dz = dy * act'(x W^T + b), then dW += dz^T x and db += sum
    dz (both accumulate, so they stay in chunk order on one stream); on a second stream, dx = dz W
    for the chunk's rows (independent of the accumulations, so its tiles fill the SMs the others
    leave idle in their last wave). dz is double-buffered: the recompute of chunk i+2 waits for
    the dx product of chunk i, the one other reader of its buffer."""
    torch = gn._torch()
    M, K = x.shape
    N = Wf.shape[0]
    chunks = chunks or default_chunks(M, K)
    bounds = list(_bounds(M, chunks))
    dx = torch.empty_like(x)
    dW = torch.zeros((N, K), dtype=torch.float32, device=x.device)
    db = torch.zeros(N, dtype=torch.float32, device=x.device)
    ws = torch.empty(max(gn.gn_colsum_bf16_workspace(N), 16), dtype=torch.uint8, device=x.device)
    rows = max(r1 - r0 for r0, r1 in bounds) if bounds else 0
    dz_buf = [torch.empty((rows, N), dtype=x.dtype, device=x.device) for _ in range(min(2, len(bounds)))]
    main, side = _stream_pair(x.device)
    dz_ready = [_event() for _ in bounds]
    dx_done = [_event() for _ in bounds]
    for i, (r0, r1) in enumerate(bounds):
        dz = dz_buf[i % 2][: r1 - r0]
        if i >= 2:
            main.wait_event(dx_done[i - 2])  # the dx product of chunk i-2 has read this buffer
        xc = x[r0:r1]
        gn.linear_act_grad(xc, Wf, d, dy[r0:r1], epilogue=act, out=dz, stream=main)
        dz_ready[i].record(main)
        side.wait_event(dz_ready[i])
        # dx = dz W: W [N, K] is the [contraction, output] operand, read MN-major
        gn.linear_bf16(dz, Wf, out=dx[r0:r1], b_mn=True, stream=side)
        dx_done[i].record(side)
        # dW += dz^T x contracts over the chunk's tokens, the rows of both dz and x: both MN-major
        gn.linear_acc_f32(dz, xc, dW, a_mn=True, b_mn=True, stream=main)
        gn.colsum_bf16(dz, db, accumulate=True, ws=ws, stream=main)
    if bounds:
        main.wait_event(dx_done[-1])  # every dx product (and every use of the buffers) is done
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
