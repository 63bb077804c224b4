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
def test_column_sums(gpu, rows, cols):
    """The backward's memory-bound step: the column sums match the fp64 sums of the same bf16
    values, and repeat bit for bit (fixed order)."""
    g = np.random.default_rng(rows)
    a = wl.bf16_bits(g.standard_normal((rows, cols)).astype(np.float32))
    t = to_dev(a)
    out = torch.full((cols,), 1.5, dtype=torch.float32, device="cuda")
    gpu.colsum_bf16(t, out, accumulate=True)
    ref = wl.bf16_to_f32(a).astype(np.float64).sum(0) + 1.5
    assert_close(to_np(out), ref, (1e-5, 1e-5 * float(np.abs(ref).max())), "colsum")
    a2 = gpu.colsum_bf16(t, torch.empty(cols, dtype=torch.float32, device="cuda"))
    b2 = gpu.colsum_bf16(t, torch.empty(cols, dtype=torch.float32, device="cuda"))
    assert torch.equal(a2, b2)  # fixed order


# shapes: a single-CTA tile with few rows (M <= 128), two-accumulator tiles (N <= 256), pair
# tiles (M > 128 and N > 256) with M, N, K not multiples of the tiles (N a multiple of 8: the
# output rows stay 16-byte aligned); a stored row is a multiple of 8 elements (K for a K-major
# operand, M or N for an MN-major one), so K is ragged only where both operands are MN-major
PRODUCT_SHAPES = [(100, 600, 200), (104, 600, 200), (300, 264, 1000), (296, 264, 1000), (5120, 512, 1000),
                  (1000, 776, 328), (136, 1032, 1001)]
LAYOUTS = [(False, False), (True, False), (False, True), (True, True)]


def _skip_unaligned(M, N, K, a_mn, b_mn):
    """Stored rows must be whole 16-byte vectors: K for a K-major operand, M / N for MN-major."""
    if (K % 8 and not (a_mn and b_mn)) or (a_mn and M % 8) or (b_mn and N % 8):
        pytest.skip("a stored row that is not a multiple of 8 elements")


def _product_operands(M, N, K, a_mn, b_mn, seed):
    """Logical A [M, K], B [N, K] (bf16 bits) and their stored forms in the requested layouts."""
    g = np.random.default_rng(seed)
    A = wl.bf16_bits(g.standard_normal((M, K)).astype(np.float32))
    B = wl.bf16_bits(g.standard_normal((N, K)).astype(np.float32))
    As = np.ascontiguousarray(A.T) if a_mn else A
    Bs = np.ascontiguousarray(B.T) if b_mn else B
    return A, B, to_dev(As), to_dev(Bs)


@pytest.mark.parametrize("M,N,K", PRODUCT_SHAPES)
@pytest.mark.parametrize("a_mn,b_mn", LAYOUTS)
def test_fp32_accumulating_product(gpu, M, N, K, a_mn, b_mn):
    """C += A B^T on the tensor cores with an fp32 accumulator updated in place, every operand
    layout, against the oracle's fp64 linear layer (no norm, no activation) of the same bf16
    operands plus the starting C."""
    _skip_unaligned(M, N, K, a_mn, b_mn)
    A, B, As, Bs = _product_operands(M, N, K, a_mn, b_mn, seed=M + N + K)
    C0 = np.random.default_rng(K).standard_normal((M, N)).astype(np.float32)
    C = to_dev(C0)
    gpu.linear_acc_f32(As, Bs, C, a_mn=a_mn, b_mn=b_mn)
    torch.cuda.synchronize()
    prod, _, _ = oracle.norm_linear(A, None, None, B, None, 0.0, "none")
    ref = C0.astype(np.float64) + prod
    assert_close(to_np(C), ref, (1e-5, 1e-4 * math.sqrt(K)), f"C += A B^T (a_mn={a_mn}, b_mn={b_mn})")
    assert gpu.device_error(clear=True) == 0


@pytest.mark.parametrize("M,N,K", PRODUCT_SHAPES)
@pytest.mark.parametrize("a_mn,b_mn", LAYOUTS)
def test_bf16_product(gpu, M, N, K, a_mn, b_mn):
    """y = A B^T + d in bf16, every operand layout, against the oracle's fp64 linear layer of the
    same operands (tolerance: the bf16 rounding of y)."""
    _skip_unaligned(M, N, K, a_mn, b_mn)
    A, B, As, Bs = _product_operands(M, N, K, a_mn, b_mn, seed=3 * M + N + K)
    bias = wl.bf16_bits((0.1 * np.random.default_rng(N).standard_normal(N)).astype(np.float32))
    d = torch.from_numpy(wl.bf16_to_f32(bias)).cuda()
    y = gpu.linear_bf16(As, Bs, d, a_mn=a_mn, b_mn=b_mn)
    torch.cuda.synchronize()
    ref, _, _ = oracle.norm_linear(A, None, None, B, bias, 0.0, "none")
    assert_close(to_np(y), ref, "bf16", f"y = A B^T + d (a_mn={a_mn}, b_mn={b_mn})")
    assert gpu.device_error(clear=True) == 0


@pytest.mark.slow
def test_tiled_linear_full_size_sampled_rows(gpu):
    """The benchmark's TiledLinear (x [32768, 5120], W [5120, 5120], SiLU, 7 backward chunks): y and
    dx are row-local given the weights, so the oracle on sampled rows - both ends of every chunk,
    tile edges and a spread - gives their exact values; dW and db sum over all rows and are checked
    at the small shapes."""
    M, N, K = 32768, 5120, 5120
    x = wl.normal(0, 92, M * K, "bf16").reshape(M, K)
    W = wl.normal(0, 93, N * K, "bf16", scale=1.0 / math.sqrt(K)).reshape(N, K)
    b = wl.normal(0, 94, N, "bf16", scale=0.1)
    dy = wl.normal(0, 95, M * N, "bf16").reshape(M, N)
    Wf, d = tl.prepare(to_dev(W), to_dev(b))
    y = tl.forward(to_dev(x), Wf, d, "silu")
    dx = tl.backward(to_dev(x), Wf, d, to_dev(dy), "silu")[0]
    torch.cuda.synchronize()
    bounds = list(tl._bounds(M, tl.default_chunks(M, K)))
    rows = np.unique(np.concatenate([np.arange(0, M, M // 32), [r for b0, b1 in bounds for r in (b0, b0 + 1, b1 - 1)],
                                     [127, 128, 255, 256, M - 1]]))
    ry, _, _ = oracle.norm_linear(x[rows], None, None, W, b, 0.0, "none", act="silu")
    rdx = oracle.linear_act_bwd(x[rows], W, b, dy[rows], "silu")[0]
    assert_close(to_np(y)[rows], ry, "bf16", "full-size tiled y")
    assert_close(to_np(dx)[rows], rdx, "grad_bf16", "full-size tiled dx")
    assert gpu.device_error(clear=True) == 0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("act", ["silu", "gelu_tanh", "none"])
def test_elementwise_activation_and_gradient(gpu, dtype, act):
    """gn_act_fwd (y = act(z)) and gn_act_grad (dz = dy act'(z)) element by element against the
    oracle's activation and derivative, on a ragged length (a tail shorter than one 16-byte vector)
    and in place (y over z, dz over dy)."""
    n = 4099
    g = np.random.default_rng(n)
    zf = (3.0 * g.standard_normal(n)).astype(np.float32)
    dyf = g.standard_normal(n).astype(np.float32)
    conv = (lambda a: wl.bf16_bits(a)) if dtype == "bf16" else (lambda a: a)  # noqa: E731
    zh, dyh = conv(zf), conv(dyf)
    zt, dyt = to_dev(zh), to_dev(dyh)
    widen = (lambda a: (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)) if dtype == "bf16" else \
        (lambda a: a.astype(np.float64))  # noqa: E731
    zr, dyr = widen(zh), widen(dyh)
    ry = np.array([oracle.act(act, v) for v in zr])
    rdz = np.array([dv * oracle.act_grad(act, v) for v, dv in zip(zr, dyr)])
    tol = "bf16" if dtype == "bf16" else "f32"
    y = gpu.act_fwd(zt, epilogue=act)
    dz = gpu.act_grad(zt, dyt, epilogue=act)
    torch.cuda.synchronize()
    assert_close(to_np(y), ry, tol, f"act {act} {dtype}")
    assert_close(to_np(dz), rdz, "grad_bf16" if dtype == "bf16" else "f32", f"act' {act} {dtype}")
    gpu.act_fwd(zt, epilogue=act, out=zt)  # in place
    gpu.act_grad(to_dev(zh), dyt, epilogue=act, out=dyt)
    torch.cuda.synchronize()
    assert torch.equal(zt, y) and torch.equal(dyt, dz)
    assert gpu.device_error(clear=True) == 0
