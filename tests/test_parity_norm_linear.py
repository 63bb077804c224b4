"""Normalization + linear layer on the tensor cores (gn_norm_linear_prepare / gn_norm_linear_fwd)
against the fp64 oracle: y = act(norm(x) W^T + bias) for LayerNorm and RMSNorm, the three
epilogues, the Gemma offset, ragged M, N and K, and the benchmark size on sampled rows.

Tolerance: the bf16 output tolerance (1.6e-2 relative + 1e-2 absolute). The kernel multiplies by
Wf = bf16(g W), one bf16 rounding per weight, where the unfused layer rounds the normalized
activations instead; with W ~ N(0, 1/K) and unit-scale outputs either rounding perturbs an output
by about 1e-3 (random over K terms), an order of magnitude inside the bound. The row statistics
(fp32: each piece of the row centred on its own mean, the pieces combined with Chan's pairwise
update) are checked at 1e-5 relative."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests._util import assert_close, to_dev, to_np
from transformer_norm_rope_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _inputs(M, N, K, seed, norm, gemma=False):
    d = wl.layernorm(M=M, N=K, dtype="bf16", seed=seed)  # rows with their own mean and scale
    g = np.random.default_rng(seed + 100)
    bf = lambda a: wl.bf16_bits(np.asarray(a, dtype=np.float32))  # noqa: E731
    W = bf(g.standard_normal((N, K)) / math.sqrt(K))
    gw = bf(0.1 * g.standard_normal(K) + (0.0 if gemma else 1.0))  # Gemma stores w with w' = 1 + w
    beta = bf(0.1 * g.standard_normal(K)) if norm == "ln" else None
    bias = bf(0.1 * g.standard_normal(N))
    return d["x"], gw, beta, W, bias


def _run(gpu, x, gw, beta, W, bias, eps, norm, gemma, epi):
    Wf, c, dd = gpu.norm_linear_prepare(to_dev(W), to_dev(gw), None if beta is None else to_dev(beta), to_dev(bias),
                                        norm=norm, gemma=gemma)
    y, mu, rs = gpu.norm_linear_fwd(to_dev(x), Wf, c, dd, eps=eps, norm=norm, epilogue=epi)
    torch.cuda.synchronize()
    return y, mu, rs


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 520, 1024), (257, 264, 1000), (64, 40, 136)])
@pytest.mark.parametrize("norm,epi,gemma", [("ln", "silu", False), ("ln", "none", False), ("rms", "gelu_tanh", False),
                                            ("rms", "none", True)])
def test_norm_linear_matches_oracle(gpu, M, N, K, norm, epi, gemma):
    x, gw, beta, W, bias = _inputs(M, N, K, seed=M + N + K, norm=norm, gemma=gemma)
    eps = 1e-5
    y, mu, rs = _run(gpu, x, gw, beta, W, bias, eps, norm, gemma, epi)
    ref, rmu, rrs = oracle.norm_linear(x, gw, beta, W, bias, eps, norm, gemma=gemma, act=epi)
    assert_close(to_np(y), ref, "bf16", f"y {norm} {epi} {M}x{N}x{K}")
    assert_close(to_np(rs), rrs, (1e-5, 0.0), "rstd")
    if norm == "ln":
        assert_close(to_np(mu), rmu, (1e-5, 1e-6), "mean")
    assert gpu.device_error(clear=True) == 0


def test_norm_linear_repeat_calls_are_identical(gpu):
    x, gw, beta, W, bias = _inputs(256, 512, 512, seed=5, norm="ln")
    a = _run(gpu, x, gw, beta, W, bias, 1e-5, "ln", False, "silu")[0]
    b = _run(gpu, x, gw, beta, W, bias, 1e-5, "ln", False, "silu")[0]
    assert torch.equal(a, b)


def test_norm_linear_empty_and_unsupported(gpu):
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((256, 64), dtype=torch.bfloat16, device="cuda")
    Wf, c, d = gpu.norm_linear_prepare(W, norm="ln")
    y, _, _ = gpu.norm_linear_fwd(x, Wf, c, d)
    assert y.shape == (0, 256)
    W60 = torch.zeros((256, 60), dtype=torch.bfloat16, device="cuda")
    Wf60, c60, d60 = gpu.norm_linear_prepare(W60, norm="ln")
    with pytest.raises(gpu.GnError):  # K % 8: the rows of x and W are not 16-byte tiles
        gpu.norm_linear_fwd(torch.zeros((4, 60), dtype=torch.bfloat16, device="cuda"), Wf60, c60, d60)


@pytest.mark.slow
def test_norm_linear_full_size_sampled_rows(gpu):
    # the benchmark shape: x [32768, 5120] (LayerNorm rows), W [5120, 5120], SiLU; the oracle
    # checks 48 rows spread over the tiles (first, last, ragged positions inside tiles)
    M, N, K = 32768, 5120, 5120
    x, gw, beta, W, bias = _inputs(M, N, K, seed=0, norm="ln")
    y, mu, rs = _run(gpu, x, gw, beta, W, bias, 1e-5, "ln", False, "silu")
    rows = np.unique(np.concatenate([np.arange(0, M, M // 40), [1, 127, 128, 129, M - 129, M - 2, M - 1]]))
    ref, rmu, rrs = oracle.norm_linear(x[rows], gw, beta, W, bias, 1e-5, "ln", act="silu")
    assert_close(to_np(y)[rows], ref, "bf16", "full-size y")
    assert_close(to_np(rs)[rows], rrs, (1e-5, 0.0), "full-size rstd")
    assert gpu.device_error(clear=True) == 0


@pytest.mark.parametrize("M,N,K", [(300, 264, 520), (257, 520, 1000), (64, 40, 136)])
@pytest.mark.parametrize("norm,act,gemma", [("ln", "silu", False), ("ln", "gelu_tanh", False), ("rms", "silu", True),
                                            ("rms", "none", False)])
def test_norm_linear_backward_matches_oracle(gpu, M, N, K, norm, act, gemma):
    """The training backward of the fused layer (normalized rows recomputed, activation gradient in
    the product's epilogue, dW and the gradient of the normalized rows on the tensor cores, then the
    normalization's backward with the forward's saved statistics) against the oracle's chain rule
    in fp64. dx within the bf16 gradient tolerance; dW, dbias and the norm's dg, dbeta (sums over
    the rows) relative to their scale."""
    from transformer_norm_rope_b200 import norm_linear as nl

    x, gw, beta, W, bias = _inputs(M, N, K, seed=M + N + K, norm=norm, gemma=gemma)
    dy = wl.bf16_bits(np.random.default_rng(M * N).standard_normal((M, N)).astype(np.float32))
    eps = 1e-5
    dev = [None if a is None else to_dev(a) for a in (x, gw, beta, W, bias, dy)]
    xt, gt, bt, Wt, biast, dyt = dev
    y, mu, rs = nl.forward(xt, gt, bt, Wt, biast, eps, norm, gemma, act)
    dx, dg, dbeta, dW, db = nl.backward(xt, gt, bt, Wt, biast, mu, rs, dyt, eps, norm, gemma, act)
    torch.cuda.synchronize()
    rdx, rdg, rdbeta, rdW, rdb = oracle.norm_linear_bwd(x, gw, beta, W, bias, dy, eps, norm, gemma=gemma, act=act)
    tag = f"{norm} {act} gemma={gemma} {M}x{N}x{K}"
    assert_close(to_np(dx), rdx, "grad_bf16", tag + " dx")
    for name, got, ref in (("dg", dg, rdg), ("dbeta", dbeta, rdbeta), ("dW", dW, rdW), ("dbias", db, rdb)):
        if ref is None:
            assert got is None, name
            continue
        sc = float(np.abs(ref).max())
        assert_close(to_np(got), ref, (2e-2, 2e-2 * sc), tag + " " + name)
    assert gpu.device_error(clear=True) == 0


def test_norm_linear_autograd_function_matches_backward(gpu):
    from transformer_norm_rope_b200 import norm_linear as nl

    x, gw, beta, W, bias = _inputs(256, 264, 512, seed=7, norm="ln")
    dy = to_dev(wl.bf16_bits(np.random.default_rng(8).standard_normal((256, 264)).astype(np.float32)))
    leaves = [to_dev(a).requires_grad_() for a in (x, gw, beta, W, bias)]
    y = nl.NormLinearFunction.apply(*leaves, 1e-5, "ln", False, "silu")
    y.backward(dy)
    xt, gt, bt, Wt, biast = (to_dev(a) for a in (x, gw, beta, W, bias))
    _, mu, rs = nl.forward(xt, gt, bt, Wt, biast, 1e-5, "ln", False, "silu")
    ref = nl.backward(xt, gt, bt, Wt, biast, mu, rs, dy, 1e-5, "ln", False, "silu")
    torch.cuda.synchronize()
    assert torch.equal(leaves[0].grad, ref[0])
    for leaf, r in zip(leaves[1:], (ref[1], ref[2], ref[3], ref[4])):
        assert leaf.grad.dtype == leaf.dtype and torch.equal(leaf.grad, r.to(leaf.dtype))


def _spread_rows(M):
    """Rows over the whole range: first, last, tile edges (128 / 256 / 512 row tiles) and a spread."""
    return np.unique(np.concatenate([np.arange(0, M, M // 40), [1, 127, 128, 129, 255, 256, 511, 512, M - 129, M - 2,
                                                                 M - 1]]))


@pytest.mark.slow
def test_norm_linear_backward_full_size_sampled_rows(gpu):
    """The training backward at the benchmark's shape (x [32768, 5120], W [5120, 5120], LayerNorm,
    SiLU): dx is row-local given the weights, so the oracle's chain rule on sampled rows gives their
    exact dx; dW, dbias, dg and dbeta sum over all rows and are checked at the small shapes."""
    from transformer_norm_rope_b200 import norm_linear as nl

    d = wl.norm_linear(seed=0)
    M, N = d["x"].shape[0], d["W"].shape[0]
    dy = wl.normal(0, 91, M * N, "bf16").reshape(M, N)
    xt, gt, bt, Wt, biast = (to_dev(d[k]) for k in ("x", "g", "beta", "W", "bias"))
    dyt = to_dev(dy)
    _, mu, rs = nl.forward(xt, gt, bt, Wt, biast, d["eps"], "ln", False, "silu")
    dx = nl.backward(xt, gt, bt, Wt, biast, mu, rs, dyt, d["eps"], "ln", False, "silu")[0]
    torch.cuda.synchronize()
    rows = _spread_rows(M)
    rdx = oracle.norm_linear_bwd(d["x"][rows], d["g"], d["beta"], d["W"], d["bias"], dy[rows], d["eps"], "ln",
                                 act="silu")[0]
    assert_close(to_np(dx)[rows], rdx, "grad_bf16", "full-size norm + linear dx")
    assert gpu.device_error(clear=True) == 0


@pytest.mark.parametrize("M,N,K", [(300, 264, 520), (64, 40, 136)])
@pytest.mark.parametrize("norm,act", [("ln", "silu"), ("rms", "gelu_tanh"), ("ln", "none")])
def test_norm_linear_keeping_z_matches_oracle(gpu, M, N, K, norm, act):
    """The training form that keeps the pre-activation: the product with no activation writes z,
    gn_act_fwd forms y from it, and the backward takes dz = dy act'(z) from the stored z
    (gn_act_grad) instead of recomputing the product. Against the oracle's forward and chain rule,
    at the tolerances of the recomputing form; the autograd form with keep_z gives the same
    gradients as the explicit backward."""
    from transformer_norm_rope_b200 import norm_linear as nl

    x, gw, beta, W, bias = _inputs(M, N, K, seed=M + K, norm=norm)
    dy = wl.bf16_bits(np.random.default_rng(M + N).standard_normal((M, N)).astype(np.float32))
    eps = 1e-5
    xt, gt, bt, Wt, biast, dyt = (None if a is None else to_dev(a) for a in (x, gw, beta, W, bias, dy))
    y, mu, rs, zt = nl.forward_keeping_z(xt, gt, bt, Wt, biast, eps, norm, False, act)
    grads = nl.backward(xt, gt, bt, Wt, biast, mu, rs, dyt, eps, norm, False, act, z=zt)
    torch.cuda.synchronize()
    ry, _, _ = oracle.norm_linear(x, gw, beta, W, bias, eps, norm, act=act)
    rz, _, _ = oracle.norm_linear(x, gw, beta, W, bias, eps, norm, act="none")
    tag = f"keep z {norm} {act} {M}x{N}x{K}"
    assert_close(to_np(y), ry, "bf16", tag + " y")
    assert_close(to_np(zt), rz, "bf16", tag + " z")
    ref = oracle.norm_linear_bwd(x, gw, beta, W, bias, dy, eps, norm, act=act)
    assert_close(to_np(grads[0]), ref[0], "grad_bf16", tag + " dx")
    for name, got, r in zip(("dg", "dbeta", "dW", "dbias"), grads[1:], ref[1:]):
        if r is None:
            assert got is None, name
            continue
        sc = float(np.abs(r).max())
        assert_close(to_np(got), r, (2e-2, 2e-2 * sc), tag + " " + name)
    leaves = [None if a is None else to_dev(a).requires_grad_() for a in (x, gw, beta, W, bias)]
    out = nl.NormLinearFunction.apply(*leaves, eps, norm, False, act, True)
    out.backward(dyt)
    torch.cuda.synchronize()
    assert torch.equal(out.detach(), y)
    assert torch.equal(leaves[0].grad, grads[0])
    for leaf, r in zip(leaves[1:], grads[1:]):
        if leaf is not None:
            assert torch.equal(leaf.grad, r.to(leaf.dtype))
    assert gpu.device_error(clear=True) == 0
