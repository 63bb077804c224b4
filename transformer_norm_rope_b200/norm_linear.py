"""A row normalization followed by a linear layer and an activation, as one training op.

Janus-Pro inference page, section 4.1 (LayerNorm, the first linear projection and SiLU in one
kernel) and HY-Motion optimization page, section 3.1 (LayerNorm merged with the matrix
multiplication after it): y = act(norm(x) W^T + bias), norm = LayerNorm (weight g, bias beta)
or RMSNorm (weight g, Gemma 1 + g optionally).

Forward: ``gn_norm_linear_prepare`` folds g (and beta) into the weight once, then
``gn_norm_linear_fwd`` streams the raw x through the tensor cores with the row statistics
applied in the epilogue; the statistics (mean, rstd) are saved for the backward.

Backward, by the chain rule, every step on this library's kernels:
  * xn = norm(x): ``gn_layernorm_fwd`` / ``gn_rmsnorm_fwd`` (the normalized rows, bf16);
  * dz = dy * act'(xn W^T + bias): ``gn_linear_act_grad`` (z recomputed, never stored), or, when
    the forward kept z (``forward_keeping_z``: the product with no activation, then
    ``gn_act_fwd``), ``gn_act_grad`` on the stored z: one elementwise pass instead of a product;
  * dxn = dz W: ``gn_linear_bf16`` with W read MN-major;
  * dW = dz^T xn: ``gn_linear_acc_f32`` with both operands read MN-major (fp32);
  * dbias = sum dz: ``gn_colsum_bf16``;
  * dx, dg (, dbeta) = the normalization's backward with dxn as the gradient of its output and
    the saved statistics: ``gn_layernorm_bwd`` / ``gn_rmsnorm_bwd``.
This module only orders the calls and allocates their outputs.
"""
from __future__ import annotations

from typing import Tuple

import transformer_norm_rope_b200 as gn


def forward(x, g, beta, W, bias, eps: float, norm: str = "ln", gemma: bool = False, act: str = "none"):
    """y [M, N] = act(norm(x) W^T + bias) -> (y, mean [M] or None, rstd [M]) for x [M, K], W [N, K]."""
    Wf, c, d = gn.norm_linear_prepare(W, g, beta if norm == "ln" else None, bias, norm=norm, gemma=gemma)
    return gn.norm_linear_fwd(x, Wf, c, d, eps=eps, norm=norm, epilogue=act)


def forward_keeping_z(x, g, beta, W, bias, eps: float, norm: str = "ln", gemma: bool = False, act: str = "none"):
    """The same layer keeping its pre-activation for the backward -> (y, mean or None, rstd, z [M, N]
    bf16): the product with no activation writes z, then y = act(z) elementwise (y is z itself when
    act is "none"). One more pass over [M, N] than ``forward``, one product fewer in ``backward``."""
    Wf, c, d = gn.norm_linear_prepare(W, g, beta if norm == "ln" else None, bias, norm=norm, gemma=gemma)
    z, mean, rstd = gn.norm_linear_fwd(x, Wf, c, d, eps=eps, norm=norm, epilogue="none")
    y = z if act == "none" else gn.act_fwd(z, epilogue=act)
    return y, mean, rstd, z


def backward(x, g, beta, W, bias, mean, rstd, dy, eps: float, norm: str = "ln", gemma: bool = False,
             act: str = "none", z=None) -> Tuple:
    """Gradients of sum(dy * y) -> (dx [M, K] bf16, dg [K] fp32, dbeta [K] fp32 or None, dW [N, K] fp32,
    dbias [N] fp32 or None), from the saved statistics of the forward (mean is unused by RMSNorm)
    and, if given, the pre-activation z that ``forward_keeping_z`` kept (else z is recomputed)."""
    torch = gn._torch()
    M, K = x.shape
    N = W.shape[0]
    if norm == "ln":
        xn, _, _ = gn.layernorm_fwd(x, g, beta, eps, save_stats=False)
    elif norm == "rms":
        if g is None:
            raise ValueError("the RMSNorm backward needs the norm weight g")
        xn, _ = gn.rmsnorm_fwd(x, g, eps, gemma=gemma, save_stats=False)
    else:
        raise ValueError(f"norm {norm!r}: 'ln' or 'rms'")
    Wp, _, d = gn.norm_linear_prepare(W, None, None, bias, norm="none")  # W as is, bias as fp32
    dz = gn.linear_act_grad(xn, Wp, d, dy, epilogue=act) if z is None else gn.act_grad(z, dy, epilogue=act)
    dxn = gn.linear_bf16(dz, Wp, b_mn=True)
    dW = torch.zeros((N, K), dtype=torch.float32, device=x.device)
    gn.linear_acc_f32(dz, xn, dW, a_mn=True, b_mn=True)
    dbias = gn.colsum_bf16(dz, torch.empty(N, dtype=torch.float32, device=x.device)) if bias is not None else None
    if norm == "ln":
        dx, dg, dbeta = gn.layernorm_bwd(x, g, beta, mean, rstd, dxn)
        return dx, dg, dbeta, dW, dbias
    dx, dg = gn.rmsnorm_bwd(x, g, rstd, dxn, gemma=gemma)
    return dx, dg, None, dW, dbias


def _function_class():
    torch = gn._torch()

    class _NormLinear(torch.autograd.Function):
        @staticmethod
        def forward(ctx, x, g, beta, W, bias, eps, norm, gemma, act, keep_z):
            if keep_z:
                y, mean, rstd, z = forward_keeping_z(x, g, beta, W, bias, eps, norm, gemma, act)
            else:
                (y, mean, rstd), z = forward(x, g, beta, W, bias, eps, norm, gemma, act), None
            ctx.save_for_backward(x, g, beta, W, bias, mean, rstd, z)
            ctx.cfg = (eps, norm, gemma, act)
            return y

        @staticmethod
        def backward(ctx, dy):
            x, g, beta, W, bias, mean, rstd, z = ctx.saved_tensors
            eps, norm, gemma, act = ctx.cfg
            dx, dg, dbeta, dW, dbias = backward(x, g, beta, W, bias, mean, rstd, dy.contiguous(), eps, norm, gemma,
                                                act, z=z)

            def cast(t, like):
                return None if t is None or like is None else t.to(like.dtype)

            return (dx, cast(dg, g), cast(dbeta, beta), dW.to(W.dtype), cast(dbias, bias), None, None, None, None,
                    None)

    return _NormLinear


_FUNCTION = None


class NormLinearFunction:
    """torch.autograd.Function form: saves x, the parameters and the row statistics, and with
    keep_z also the pre-activation (one product fewer in the backward, [M, N] bf16 more memory)."""

    @staticmethod
    def apply(x, g, beta, W, bias, eps: float = 1e-5, norm: str = "ln", gemma: bool = False, act: str = "none",
              keep_z: bool = False):
        global _FUNCTION
        if _FUNCTION is None:
            _FUNCTION = _function_class()
        return _FUNCTION.apply(x, g, beta, W, bias, eps, norm, gemma, act, keep_z)


__all__ = ["forward", "forward_keeping_z", "backward", "NormLinearFunction"]
