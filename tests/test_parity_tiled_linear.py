"""The token-chunked linear layer (TiledLinear, Helios kernels article, section "内核三
TiledLinear"): forward y = act(x W^T + b) chunk by chunk on the tensor-core kernels, backward
recomputing each chunk's pre-activation. Checked against the fp64 oracle (forward: the plain
linear + activation; backward: its gradients), and chunked against unchunked: the forward rows
are independent, so y must be bit-identical for every chunk count.

Tolerances: y as any bf16 output (1.6e-2 rel + 1e-2 abs); dx, dW, db as bf16 gradients (2e-2 rel
+ 2e-2 abs, dW and db relative to their scale: they sum over all rows)."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests._util import assert_close, to_dev, to_np
from transformer_norm_rope_b200 import tiled_linear as tl
from transformer_norm_rope_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _inputs(M, N, K, seed):
    g = np.random.default_rng(seed)
    bf = lambda a: wl.bf16_bits(np.asarray(a, dtype=np.float32))  # noqa: E731
    x = bf(g.standard_normal((M, K)))
    W = bf(g.standard_normal((N, K)) / math.sqrt(K))
    b = bf(0.1 * g.standard_normal(N))
    dy = bf(g.standard_normal((M, N)))
    return x, W, b, dy


@pytest.mark.parametrize("M,N,K,chunks", [(1000, 768, 512, None), (300, 264, 1024, 3), (64, 256, 128, 1)])
@pytest.mark.parametrize("act", ["silu", "gelu_tanh"])
def test_tiled_linear_matches_oracle(gpu, M, N, K, chunks, act):
    x, W, b, dy = _inputs(M, N, K, seed=M + N)
    Wf, d = tl.prepare(to_dev(W), to_dev(b))
    y = tl.forward(to_dev(x), Wf, d, act, chunks)
    dx, dW, db = tl.backward(to_dev(x), Wf, d, to_dev(dy), act, chunks)
    torch.cuda.synchronize()
    ry, _, _ = oracle.norm_linear(x, None, None, W, b, 0.0, "none", act=act)
    assert_close(to_np(y), ry, "bf16", f"y {act}")
    rdx, rdW, rdb = oracle.linear_act_bwd(x, W, b, dy, act)
    assert_close(to_np(dx), rdx, "grad_bf16", "dx")
    for name, got, ref in (("dW", dW, rdW), ("db", db, rdb)):
        sc = float(np.abs(ref).max())
        assert_close(to_np(got), ref, (2e-2, 2e-2 * sc), name)
    assert gpu.device_error(clear=True) == 0


def test_chunking_changes_no_forward_value(gpu):
    x, W, b, dy = _inputs(2048, 512, 512, seed=9)
    Wf, d = tl.prepare(to_dev(W), to_dev(b))
    ys = [tl.forward(to_dev(x), Wf, d, "silu", c) for c in (1, 4, 7)]
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])


def test_autograd_function_matches_backward(gpu):
    x, W, b, dy = _inputs(512, 256, 256, seed=4)
    xt, Wt, bt = to_dev(x).requires_grad_(), to_dev(W).requires_grad_(), to_dev(b).requires_grad_()
    y = tl.TiledLinearFunction.apply(xt, Wt, bt, "silu", 2)
    y.backward(to_dev(dy))
    Wf, d = tl.prepare(to_dev(W), to_dev(b))
    dx, dW, db = tl.backward(to_dev(x), Wf, d, to_dev(dy), "silu", 2)
    torch.cuda.synchronize()
    assert torch.equal(xt.grad, dx)
    assert torch.equal(Wt.grad, dW.to(torch.bfloat16)) and torch.equal(bt.grad, db.to(torch.bfloat16))


def test_act_grad_matches_oracle_derivative(gpu):
    g = np.random.default_rng(1)
    for dt, tol in (("f32", (1e-5, 1e-6)), ("bf16", (1.6e-2, 1e-2))):
        n = 4099  # a ragged tail
        z = g.standard_normal(n).astype(np.float32) * 3
        dy = g.standard_normal(n).astype(np.float32)
        if dt == "bf16":
            z, dy = wl.bf16_bits(z), wl.bf16_bits(dy)
        for act in ("none", "silu", "gelu_tanh"):
            dz = gpu.act_grad(to_dev(z), to_dev(dy), epilogue=act)
            torch.cuda.synchronize()
            zf = z.astype(np.float64) if dt == "f32" else wl.bf16_to_f32(z).astype(np.float64)
            gf = dy.astype(np.float64) if dt == "f32" else wl.bf16_to_f32(dy).astype(np.float64)
            ref = gf * np.array([oracle.act_grad(act, v) for v in zf])
            assert_close(to_np(dz), ref, tol, f"act_grad {dt} {act}")


@pytest.mark.parametrize("rows,cols", [(300, 264), (64, 5120), (1000, 72), (8, 8)])
def test_transpose_and_column_sums(gpu, rows, cols):
    """The backward's memory-bound steps: the transpose is exact (bit for bit, zero-padded up to
    a multiple of 8 rows) and the column sums match the fp64 sums of the same bf16 values."""
    g = np.random.default_rng(rows)
    a = wl.bf16_bits(g.standard_normal((rows, cols)).astype(np.float32))
    t = to_dev(a)
    tt = gpu.transpose(t)
    r8 = (rows + 7) // 8 * 8
    assert tuple(tt.shape) == (cols, r8)
    assert torch.equal(tt[:, :rows], t.t()) and bool((tt[:, rows:] == 0).all())
    out = torch.full((cols,), 1.5, dtype=torch.float32, device="cuda")
    gpu.colsum_bf16(t, out, accumulate=True)
    ref = wl.bf16_to_f32(a).astype(np.float64).sum(0) + 1.5
    assert_close(to_np(out), ref, (1e-5, 1e-5 * float(np.abs(ref).max())), "colsum")
    a2 = gpu.colsum_bf16(t, torch.empty(cols, dtype=torch.float32, device="cuda"))
    b2 = gpu.colsum_bf16(t, torch.empty(cols, dtype=torch.float32, device="cuda"))
    assert torch.equal(a2, b2)  # fixed order


@pytest.mark.parametrize("M,N,K", [(300, 264, 1024), (5120, 512, 1000), (100, 600, 200)])
def test_fp32_accumulating_product(gpu, M, N, K):
    """C += A B^T on the tensor cores with an fp32 accumulator updated in place, against the fp64
    product of the same bf16 operands (K padded with zeros to a multiple of 8 by the transpose
    path where the caller needs it; here K is a multiple of 8)."""
    g = np.random.default_rng(M + N + K)
    A = wl.bf16_bits(g.standard_normal((M, K)).astype(np.float32))
    B = wl.bf16_bits(g.standard_normal((N, K)).astype(np.float32))
    C0 = g.standard_normal((M, N)).astype(np.float32)
    C = to_dev(C0)
    gpu.linear_acc_f32(to_dev(A), to_dev(B), C)
    torch.cuda.synchronize()
    ref = C0.astype(np.float64) + wl.bf16_to_f32(A).astype(np.float64) @ wl.bf16_to_f32(B).astype(np.float64).T
    assert_close(to_np(C), ref, (1e-5, 1e-4 * math.sqrt(K)), "C += A B^T")
    assert gpu.device_error(clear=True) == 0
