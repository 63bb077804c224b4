"""GPU parity of the RMSNorm and LayerNorm kernels against the fp64 oracle.

Small cases span several CTAs and row tiles, ragged tails (hidden not a multiple of the
16-byte vector), both launch shapes (lane group per row for short rows, CTA per row with the
TMA pipeline for long rows), strided rows, in-place outputs and empty inputs. The full-size
cases run the exact launch configuration the benchmark times and compare every output element,
every saved statistic and the complete weight gradients with the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from transformer_norm_rope_b200 import workloads as wl
from tests import _fullsize as fs
from tests._util import assert_close, grad_tol, io_tol, to_dev, to_np, wgrad_tol


def to_rows(a):
    """Generator matrix -> device tensor whose rows start on 16-byte boundaries (row stride
    padded when the width is ragged, as the C ABI requires)."""
    import transformer_norm_rope_b200 as gn

    t = to_dev(a)
    out = gn.empty_rows(t.shape, t.dtype, t.device)
    out.copy_(t)
    return out

pytestmark = pytest.mark.gpu

EPIS = ["none", "gelu_tanh", "silu"]
# (rows, hidden): PR1 shape; group path (short rows, incl. lanes < 32 and ragged tails);
# CTA path (long rows, ragged tails, more rows than the persistent grid)
SHAPES = [(256, 1024), (33, 72), (129, 1000), (5, 9), (65, 2051), (300, 5120), (3, 8192), (1200, 1536)]


def rms_case(rows, hidden, dtype, gemma, seed=0):
    d = wl.rmsnorm(M=rows, N=hidden, dtype=dtype, gemma=gemma, seed=seed, outliers=rows >= 100)
    return d


@pytest.mark.parametrize("rows,hidden", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_rmsnorm_fwd_bwd(gpu, rows, hidden, dtype):
    if dtype == "f32" and hidden > 4096:
        hidden = 4096  # fp32 backward rows stop at 4096
    for gemma, epi in ((False, "none"), (True, "gelu_tanh"), (False, "silu")):
        d = rms_case(rows, hidden, dtype, gemma)
        x, w, dy = to_rows(d["x"]), to_dev(d["w"]), to_rows(d["dy"])
        y, r = gpu.rmsnorm_fwd(x, w, d["eps"], gemma=gemma, epilogue=epi)
        dx, dw = gpu.rmsnorm_bwd(x, w, r, dy, gemma=gemma, epilogue=epi)
        torch.cuda.synchronize()
        ry, rr = oracle.rmsnorm_fwd(d["x"], d["w"], d["eps"], gemma=gemma, act=epi)
        rdx, rdw = oracle.rmsnorm_bwd(d["x"], d["w"], d["dy"], d["eps"], gemma=gemma, act=epi)
        tag = f"rms {dtype} {rows}x{hidden} gemma={gemma} {epi}"
        assert_close(to_np(y), ry, io_tol(dtype), tag + " y")
        assert_close(to_np(r), rr, "stat", tag + " inv_rms")
        assert_close(to_np(dx), rdx, grad_tol(dtype), tag + " dx")
        assert_close(to_np(dw), rdw, wgrad_tol(dtype, rdw), tag + " dw")


@pytest.mark.parametrize("rows,hidden", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_layernorm_fwd_bwd(gpu, rows, hidden, dtype):
    if dtype == "f32" and hidden > 4096:
        hidden = 4096
    for epi, affine in (("gelu_tanh", True), ("none", True), ("silu", False)):
        d = wl.layernorm(M=rows, N=hidden, dtype=dtype)
        w = d["w"] if affine else None
        b = d["b"] if affine else None
        x, dy = to_rows(d["x"]), to_rows(d["dy"])
        wt = to_dev(w) if affine else None
        bt = to_dev(b) if affine else None
        y, mu, rs = gpu.layernorm_fwd(x, wt, bt, d["eps"], epilogue=epi)
        dx, dw, db = gpu.layernorm_bwd(x, wt, bt, mu, rs, dy, epilogue=epi)
        torch.cuda.synchronize()
        ry, rmu, rrs = oracle.layernorm_fwd(d["x"], w, b, d["eps"], act=epi)
        rdx, rdw, rdb = oracle.layernorm_bwd(d["x"], w, b, d["dy"], d["eps"], act=epi)
        tag = f"ln {dtype} {rows}x{hidden} {epi} affine={affine}"
        assert_close(to_np(y), ry, io_tol(dtype), tag + " y")
        # the mean is compared with an absolute floor: rows are centred anywhere in (-2, 2)
        assert_close(to_np(mu), rmu, (1e-5, 1e-6), tag + " mean")
        assert_close(to_np(rs), rrs, "stat", tag + " rstd")
        assert_close(to_np(dx), rdx, grad_tol(dtype), tag + " dx")
        assert_close(to_np(dw), rdw, wgrad_tol(dtype, rdw), tag + " dw")
        assert_close(to_np(db), rdb, wgrad_tol(dtype, rdb), tag + " db")


@pytest.mark.parametrize("path,warps,stages", [(0, 0, 0), (1, 0, 0), (1, 0, 4), (2, 4, 3), (2, 0, 4), (2, 5, 2),
                                               (3, 0, 0), (3, 6, 3), (3, 0, 2), (2, 20, 1), (3, 13, 1)])
def test_norm_forward_kernels_of_long_rows(gpu, path, warps, stages):
    """The forward kernels of long rows - the CTA-per-row pipeline (fwd_path 1), one warp per row
    with the LayerNorm statistics in two passes (fwd_path 2) or one shifted pass (fwd_path 3), and
    the default (RMSNorm: the CTA kernel, LayerNorm: the shifted warp kernel) - at several warp and
    stage counts, against the oracle, ragged tails included. A row whose stages do not fit the
    warp kernel falls back to the CTA kernel."""
    try:
        gpu.tune("fwd_path", path)
        gpu.tune("fwd_warps", warps)
        gpu.tune("stages", stages)
        for rows, hidden, dtype in ((300, 5120, "bf16"), (65, 2051, "bf16"), (77, 1000, "f32"), (129, 8192, "bf16"),
                                    (41, 1027, "f32"), (50, 3500, "bf16"), (30, 6000, "bf16")):
            d = wl.rmsnorm(M=rows, N=hidden, dtype=dtype, gemma=True, outliers=False)
            y, r = gpu.rmsnorm_fwd(to_rows(d["x"]), to_dev(d["w"]), d["eps"], gemma=True, epilogue="gelu_tanh")
            ry, rr = oracle.rmsnorm_fwd(d["x"], d["w"], d["eps"], gemma=True, act="gelu_tanh")
            tag = f"path {path} warps {warps} stages {stages} {dtype} {rows}x{hidden}"
            assert_close(to_np(y), ry, io_tol(dtype), tag + " rms y")
            assert_close(to_np(r), rr, "stat", tag + " rms inv_rms")
            dl = wl.layernorm(M=rows, N=hidden, dtype=dtype)
            for epi in ("gelu_tanh", "silu"):
                y, mu, rs = gpu.layernorm_fwd(to_rows(dl["x"]), to_dev(dl["w"]), to_dev(dl["b"]), dl["eps"], epilogue=epi)
                ry, rmu, rrs = oracle.layernorm_fwd(dl["x"], dl["w"], dl["b"], dl["eps"], act=epi)
                assert_close(to_np(y), ry, io_tol(dtype), tag + f" ln {epi} y")
                assert_close(to_np(mu), rmu, (1e-5, 1e-6), tag + " ln mean")
                assert_close(to_np(rs), rrs, "stat", tag + " ln rstd")
    finally:
        for key in ("fwd_path", "fwd_warps", "stages"):
            gpu.tune(key, 0)
    assert gpu.device_error(clear=True) == 0


@pytest.mark.parametrize("hidden", [72, 5120])
def test_strided_rows_and_in_place(gpu, hidden):
    rows, ld = 40, hidden + 64
    d = wl.rmsnorm(M=rows, N=hidden, dtype="bf16", outliers=False)
    base = torch.zeros(rows, ld, dtype=torch.bfloat16, device="cuda")
    base[:, :hidden] = to_dev(d["x"])
    xs = base[:, :hidden]
    w = to_dev(d["w"])
    y, r = gpu.rmsnorm_fwd(xs, w, d["eps"])
    ry, rr = oracle.rmsnorm_fwd(d["x"], d["w"], d["eps"])
    assert_close(to_np(y), ry, "bf16", "strided rms y")
    gpu.rmsnorm_fwd(xs, w, d["eps"], out=xs)  # in place on a strided view
    assert_close(to_np(xs), ry, "bf16", "in-place rms y")
    assert torch.all(base[:, hidden:] == 0), "padding between rows was written"
    dl = wl.layernorm(M=rows, N=hidden, dtype="bf16")
    x = to_dev(dl["x"])
    gpu.layernorm_fwd(x, to_dev(dl["w"]), to_dev(dl["b"]), dl["eps"], epilogue="gelu_tanh", out=x)
    ry, _, _ = oracle.layernorm_fwd(dl["x"], dl["w"], dl["b"], dl["eps"], act="gelu_tanh")
    assert_close(to_np(x), ry, "bf16", "in-place ln y")


def test_empty_rows(gpu):
    x = torch.empty(0, 512, dtype=torch.bfloat16, device="cuda")
    w = torch.ones(512, dtype=torch.bfloat16, device="cuda")
    y, r = gpu.rmsnorm_fwd(x, w)
    assert y.shape == (0, 512)
    dx, dw = gpu.rmsnorm_bwd(x, w, r, x)
    dxl, dwl, dbl = gpu.layernorm_bwd(x, w, None, r, r, x)
    torch.cuda.synchronize()
    assert torch.all(dw == 0) and torch.all(dwl == 0) and torch.all(dbl == 0)


def test_unsupported_hidden_is_reported(gpu):
    x = torch.zeros(2, 40000, dtype=torch.bfloat16, device="cuda")
    w = torch.ones(40000, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gpu.GnError) as e:
        gpu.rmsnorm_bwd(x, w, torch.ones(2, device="cuda"), x)
    assert e.value.status == gpu.GN_ERR_UNSUPPORTED


@pytest.mark.parametrize("dtype,fwd_max,bwd_max", [("bf16", 20480, 10240), ("f32", 10240, 5120)])
def test_widest_rows(gpu, dtype, fwd_max, bwd_max):
    """The widest rows each path takes (the CTA-per-row kernels: 320 consumer threads, at most 8
    vectors a thread forward and 4 backward) match the oracle; one 16-byte vector more is
    refused with GN_ERR_UNSUPPORTED before anything is launched."""
    vec = 8 if dtype == "bf16" else 4
    for hidden, bwd in ((fwd_max, False), (bwd_max, True)):
        d = wl.rmsnorm(M=3, N=hidden, dtype=dtype, gemma=True, outliers=False)
        x, w = to_rows(d["x"]), to_dev(d["w"])
        y, r = gpu.rmsnorm_fwd(x, w, d["eps"], gemma=True, epilogue="silu")
        ry, rr = oracle.rmsnorm_fwd(d["x"], d["w"], d["eps"], gemma=True, act="silu")
        assert_close(to_np(y), ry, io_tol(dtype), f"rms {dtype} {hidden} y")
        dl = wl.layernorm(M=3, N=hidden, dtype=dtype)
        xl, wt, bt = to_rows(dl["x"]), to_dev(dl["w"]), to_dev(dl["b"])
        yl, mu, rs = gpu.layernorm_fwd(xl, wt, bt, dl["eps"], epilogue="gelu_tanh")
        ryl, _, _ = oracle.layernorm_fwd(dl["x"], dl["w"], dl["b"], dl["eps"], act="gelu_tanh")
        assert_close(to_np(yl), ryl, io_tol(dtype), f"ln {dtype} {hidden} y")
        if bwd:
            dx, dw = gpu.rmsnorm_bwd(x, w, r, to_rows(d["dy"]), gemma=True, epilogue="silu")
            rdx, rdw = oracle.rmsnorm_bwd(d["x"], d["w"], d["dy"], d["eps"], gemma=True, act="silu")
            assert_close(to_np(dx), rdx, grad_tol(dtype), f"rms {dtype} {hidden} dx")
            assert_close(to_np(dw), rdw, wgrad_tol(dtype, rdw), f"rms {dtype} {hidden} dw")
            dxl, dwl, dbl = gpu.layernorm_bwd(xl, wt, bt, mu, rs, to_rows(dl["dy"]), epilogue="gelu_tanh")
            rdxl, rdwl, rdbl = oracle.layernorm_bwd(dl["x"], dl["w"], dl["b"], dl["dy"], dl["eps"], act="gelu_tanh")
            assert_close(to_np(dxl), rdxl, grad_tol(dtype), f"ln {dtype} {hidden} dx")
            assert_close(to_np(dwl), rdwl, wgrad_tol(dtype, rdwl), f"ln {dtype} {hidden} dw")
            assert_close(to_np(dbl), rdbl, wgrad_tol(dtype, rdbl), f"ln {dtype} {hidden} db")
    torch.cuda.synchronize()
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    for hidden, bwd in ((fwd_max + vec, False), (bwd_max + vec, True)):
        x = torch.zeros(2, hidden, dtype=tdt, device="cuda")
        w = torch.ones(hidden, dtype=tdt, device="cuda")
        st = torch.ones(2, device="cuda")
        calls = [lambda: gpu.rmsnorm_bwd(x, w, st, x), lambda: gpu.layernorm_bwd(x, w, w, st, st, x)] if bwd else \
            [lambda: gpu.rmsnorm_fwd(x, w), lambda: gpu.layernorm_fwd(x, w, w)]
        for call in calls:
            with pytest.raises(gpu.GnError) as e:
                call()
            assert e.value.status == gpu.GN_ERR_UNSUPPORTED, hidden
    assert gpu.device_error(clear=True) == 0


def _degenerate_rows(hidden, rng):
    """Rows the statistics can trip on: all zero, constant, a large mean with a small spread (the
    shifted one-pass variance must not cancel), one outlier, a tiny scale, alternating signs."""
    j = np.arange(hidden)
    rows = [np.zeros(hidden), np.full(hidden, 3.5), 1000.0 + 8.0 * (j % 2), np.where(j == hidden // 3, 500.0, 0.25),
            1e-3 * rng.standard_normal(hidden), np.where(j % 2 == 0, 1.0, -1.0)]
    return np.stack(rows).astype(np.float32)


@pytest.mark.parametrize("hidden,dtype", [(5120, "bf16"), (64, "bf16"), (1000, "f32"), (2051, "bf16")])
def test_degenerate_rows(gpu, hidden, dtype):
    """Zero, constant, far-off-centre, outlier, tiny and alternating rows through every norm
    kernel (CTA, warp and lane-group paths by row width) against the oracle: y and the saved
    statistics of the forwards, dx and the weight gradients of the backwards."""
    rng = np.random.default_rng(hidden)
    xf = _degenerate_rows(hidden, rng)
    conv = (lambda a: wl.bf16_bits(a)) if dtype == "bf16" else (lambda a: a.astype(np.float32))  # noqa: E731
    x = conv(xf)
    w = conv((1.0 + 0.1 * rng.standard_normal(hidden)).astype(np.float32))
    b = conv((0.1 * rng.standard_normal(hidden)).astype(np.float32))
    dy = conv(rng.standard_normal(xf.shape).astype(np.float32))
    xt, wt, bt, dyt = to_rows(x), to_dev(w), to_dev(b), to_rows(dy)
    for gemma, eps in ((False, 1e-6), (True, 1e-5)):
        y, r = gpu.rmsnorm_fwd(xt, wt, eps, gemma=gemma, epilogue="silu")
        dx, dw = gpu.rmsnorm_bwd(xt, wt, r, dyt, gemma=gemma, epilogue="silu")
        torch.cuda.synchronize()
        ry, rr = oracle.rmsnorm_fwd(x, w, eps, gemma=gemma, act="silu")
        rdx, rdw = oracle.rmsnorm_bwd(x, w, dy, eps, gemma=gemma, act="silu")
        tag = f"rms {dtype} {hidden} gemma={gemma}"
        assert_close(to_np(y), ry, io_tol(dtype), tag + " y")
        assert_close(to_np(r), rr, "stat", tag + " inv_rms")
        assert_close(to_np(dx), rdx, grad_tol(dtype), tag + " dx")
        assert_close(to_np(dw), rdw, wgrad_tol(dtype, rdw), tag + " dw")
    eps = 1e-5
    y, mu, rs = gpu.layernorm_fwd(xt, wt, bt, eps, epilogue="gelu_tanh")
    dx, dw, db = gpu.layernorm_bwd(xt, wt, bt, mu, rs, dyt, epilogue="gelu_tanh")
    torch.cuda.synchronize()
    ry, rmu, rrs = oracle.layernorm_fwd(x, w, b, eps, act="gelu_tanh")
    rdx, rdw, rdb = oracle.layernorm_bwd(x, w, b, dy, eps, act="gelu_tanh")
    tag = f"ln {dtype} {hidden}"
    assert_close(to_np(y), ry, io_tol(dtype), tag + " y")
    assert_close(to_np(mu), rmu, (1e-5, 1e-6), tag + " mean")
    assert_close(to_np(rs), rrs, "stat", tag + " rstd")
    assert_close(to_np(dx), rdx, grad_tol(dtype), tag + " dx")
    assert_close(to_np(dw), rdw, wgrad_tol(dtype, rdw), tag + " dw")
    assert_close(to_np(db), rdb, wgrad_tol(dtype, rdb), tag + " db")
    assert gpu.device_error(clear=True) == 0


def test_deterministic_weight_gradients(gpu):
    d = wl.rmsnorm(M=3000, N=5120, dtype="bf16")
    x, w, dy = to_dev(d["x"]), to_dev(d["w"]), to_dev(d["dy"])
    _, r = gpu.rmsnorm_fwd(x, w, d["eps"])
    a = gpu.rmsnorm_bwd(x, w, r, dy)
    b = gpu.rmsnorm_bwd(x, w, r, dy)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.slow
@pytest.mark.parametrize("gemma", [False, True])
def test_rmsnorm_full_size(gpu, gemma):
    """The benchmark's launch (x[15360, 5120] bf16, 1% outlier rows): y, inv_rms and dx on every
    row against the oracle (chunks of rows on host worker processes), dw complete."""
    cfg = wl.RMSNORM_MAIN
    d = wl.rmsnorm(M=cfg["M"], N=cfg["N"], dtype="bf16", gemma=gemma)
    x, w, dy = to_dev(d["x"]), to_dev(d["w"]), to_dev(d["dy"])
    y, r = gpu.rmsnorm_fwd(x, w, d["eps"], gemma=gemma)
    dx, dw = gpu.rmsnorm_bwd(x, w, r, dy, gemma=gemma)
    torch.cuda.synchronize()
    M, N = x.shape

    def jobs():
        for r0, r1 in fs.row_chunks(M, N):
            yield fs.job_rms, (d["x"][r0:r1], d["w"], d["dy"][r0:r1], d["eps"], gemma, fs.bits(y[r0:r1]),
                               fs.bits(r[r0:r1]), fs.bits(dx[r0:r1]), f"rows {r0}:{r1}")

    v = fs.run(jobs(), f"full rms gemma={gemma}")
    n = v.assert_ok()
    assert n == {"y": M * N, "inv_rms": M, "dx": M * N}
    assert_close(to_np(dw), v.parts["dw"], "grad_bf16", "full rms dw")


@pytest.mark.slow
def test_layernorm_full_size(gpu):
    """The benchmark's launch (x[32768, 5120] bf16, tanh-GeLU): y, mean, rstd and dx on every row
    against the oracle, dw and db complete."""
    cfg = wl.LAYERNORM_MAIN
    d = wl.layernorm(M=cfg["M"], N=cfg["N"], dtype="bf16")
    x, w, b, dy = (to_dev(d[k]) for k in ("x", "w", "b", "dy"))
    y, mu, rs = gpu.layernorm_fwd(x, w, b, d["eps"], epilogue="gelu_tanh")
    dx, dw, db = gpu.layernorm_bwd(x, w, b, mu, rs, dy, epilogue="gelu_tanh")
    torch.cuda.synchronize()
    M, N = x.shape

    def jobs():
        for r0, r1 in fs.row_chunks(M, N):
            yield fs.job_ln, (d["x"][r0:r1], d["w"], d["b"], d["dy"][r0:r1], d["eps"], "gelu_tanh",
                              fs.bits(y[r0:r1]), fs.bits(mu[r0:r1]), fs.bits(rs[r0:r1]), fs.bits(dx[r0:r1]),
                              f"rows {r0}:{r1}")

    v = fs.run(jobs(), "full ln")
    n = v.assert_ok()
    assert n == {"y": M * N, "mean": M, "rstd": M, "dx": M * N}
    assert_close(to_np(dw), v.parts["dw"], "grad_bf16", "full ln dw")
    assert_close(to_np(db), v.parts["db"], "grad_bf16", "full ln db")


def _shifted(t):
    """The same values in storage that starts 2 bytes past a 16-byte boundary."""
    buf = torch.empty(t.numel() + 8, dtype=t.dtype, device=t.device)
    off = (2 - buf.data_ptr() % 16) % 16 // t.element_size() if t.element_size() == 2 else 1
    out = buf[off:off + t.numel()]
    out.copy_(t)
    return out


@pytest.mark.parametrize("hidden", [2051, 5120])
def test_unaligned_weights_give_the_aligned_result(gpu, hidden):
    # weights need no alignment: whole 16-byte vectors of an aligned weight are staged with one
    # load each, an unaligned one element by element; the staged values, hence every output,
    # must be the same bits
    d = wl.layernorm(M=300, N=hidden, dtype="bf16")
    x, dy = to_rows(d["x"]), to_rows(d["dy"])
    w, b = to_dev(d["w"]), to_dev(d["b"])
    ws, bs = _shifted(w), _shifted(b)
    assert ws.data_ptr() % 16 != 0 and torch.equal(ws, w)
    for epi in ("gelu_tanh", "none"):
        a = gpu.layernorm_fwd(x, w, b, d["eps"], epilogue=epi)
        u = gpu.layernorm_fwd(x, ws, bs, d["eps"], epilogue=epi)
        ga = gpu.layernorm_bwd(x, w, b, a[1], a[2], dy, epilogue=epi)
        gu = gpu.layernorm_bwd(x, ws, bs, a[1], a[2], dy, epilogue=epi)
        torch.cuda.synchronize()
        for p, q in zip(a + ga, u + gu):
            assert torch.equal(p, q), f"layernorm {epi} {hidden}"
    r = wl.rmsnorm(M=300, N=hidden, dtype="bf16", gemma=True)
    xr, dyr, wr = to_rows(r["x"]), to_rows(r["dy"]), to_dev(r["w"])
    wrs = _shifted(wr)
    a = gpu.rmsnorm_fwd(xr, wr, r["eps"], gemma=True, epilogue="silu")
    u = gpu.rmsnorm_fwd(xr, wrs, r["eps"], gemma=True, epilogue="silu")
    ga = gpu.rmsnorm_bwd(xr, wr, a[1], dyr, gemma=True, epilogue="silu")
    gu = gpu.rmsnorm_bwd(xr, wrs, a[1], dyr, gemma=True, epilogue="silu")
    torch.cuda.synchronize()
    for p, q in zip(a + ga, u + gu):
        assert torch.equal(p, q), f"rmsnorm {hidden}"
    assert gpu.device_error(clear=True) == 0


def test_fp32_gelu_far_below_zero(gpu):
    """fp32 rows whose pre-activations reach far below zero (z down to about -12), where the
    tanh-GeLU and its derivative are 1e-7 .. 1e-3 and 1 + tanh(u) must not be formed from a
    tanh(u) that rounds to -1: LayerNorm with a bias near -6 and RMSNorm with a weight near -4,
    forward and backward through the CTA and warp kernels, against the oracle at the fp32
    tolerances."""
    rng = np.random.default_rng(11)
    for rows, hidden in ((64, 1000), (40, 2051)):
        x = rng.standard_normal((rows, hidden)).astype(np.float32)
        dy = rng.standard_normal((rows, hidden)).astype(np.float32)
        w = (1.0 + 0.1 * rng.standard_normal(hidden)).astype(np.float32)
        b = (-6.0 + 0.5 * rng.standard_normal(hidden)).astype(np.float32)
        xt, dyt, wt, bt = to_rows(x), to_rows(dy), to_dev(w), to_dev(b)
        y, mu, rs = gpu.layernorm_fwd(xt, wt, bt, 1e-5, epilogue="gelu_tanh")
        dx, dw, db = gpu.layernorm_bwd(xt, wt, bt, mu, rs, dyt, epilogue="gelu_tanh")
        torch.cuda.synchronize()
        ry, _, _ = oracle.layernorm_fwd(x, w, b, 1e-5, act="gelu_tanh")
        rdx, rdw, rdb = oracle.layernorm_bwd(x, w, b, dy, 1e-5, act="gelu_tanh")
        tag = f"ln f32 {rows}x{hidden} far below zero"
        assert_close(to_np(y), ry, "f32", tag + " y")
        assert_close(to_np(dx), rdx, "f32", tag + " dx")
        assert_close(to_np(dw), rdw, wgrad_tol("f32", rdw), tag + " dw")
        assert_close(to_np(db), rdb, wgrad_tol("f32", rdb), tag + " db")
        wr = (-4.0 + 0.1 * rng.standard_normal(hidden)).astype(np.float32)
        y, r = gpu.rmsnorm_fwd(xt, to_dev(wr), 1e-6, epilogue="gelu_tanh")
        dx, dw = gpu.rmsnorm_bwd(xt, to_dev(wr), r, dyt, epilogue="gelu_tanh")
        torch.cuda.synchronize()
        ry, _ = oracle.rmsnorm_fwd(x, wr, 1e-6, act="gelu_tanh")
        rdx, rdw = oracle.rmsnorm_bwd(x, wr, dy, 1e-6, act="gelu_tanh")
        tag = f"rms f32 {rows}x{hidden} far below zero"
        assert_close(to_np(y), ry, "f32", tag + " y")
        assert_close(to_np(dx), rdx, "f32", tag + " dx")
        assert_close(to_np(dw), rdw, wgrad_tol("f32", rdw), tag + " dw")
    assert gpu.device_error(clear=True) == 0
