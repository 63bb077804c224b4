"""GPU parity of the in-place interleaved RoPE and the fused qk-norm + RoPE against the oracle.

Small cases cover several units per CTA and several CTAs, one or two tensors (k may be
absent), head dims from 8 to 264 (including widths whose lanes per head are not a power of
two, for the plain rotation), slabs split across heads (the backward stages four tensors),
and empty inputs. The full-size cases run the benchmark's launch configuration and compare
every output element, every saved statistic and the complete weight gradients with the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from transformer_norm_rope_b200 import workloads as wl
from tests import _fullsize as fs
from tests._util import assert_close, grad_tol, io_tol, to_dev, to_np, wgrad_tol

pytestmark = pytest.mark.gpu

ROPE_SHAPES = [(1, 256, 8, 128, "f32"), (2, 37, 5, 64, "bf16"), (1, 300, 40, 128, "bf16"),
               (3, 11, 2, 8, "bf16"), (1, 17, 3, 96, "bf16"), (2, 9, 2, 264, "bf16"), (1, 40, 6, 72, "f32")]


@pytest.mark.parametrize("B,S,H,D,dtype", ROPE_SHAPES)
@pytest.mark.parametrize("with_k", [True, False])
def test_rope_fwd_bwd_in_place(gpu, B, S, H, D, dtype, with_k):
    d = wl.rope(B=B, S=S, H=H, D=D, dtype=dtype)
    q, k = to_dev(d["q"]), to_dev(d["k"]) if with_k else None
    cos, sin = to_dev(d["cos"]), to_dev(d["sin"])
    gpu.rope_apply_(q, k, cos, sin, +1)
    torch.cuda.synchronize()
    tol = io_tol(dtype)
    assert_close(to_np(q), oracle.rope(d["q"], d["cos"], d["sin"], +1), tol, "rope fwd q")
    if with_k:
        assert_close(to_np(k), oracle.rope(d["k"], d["cos"], d["sin"], +1), tol, "rope fwd k")
    # the backward is the same call with sin negated, applied in place to the gradient
    qf = q.clone()
    gpu.rope_apply_(q, k, cos, sin, -1)
    torch.cuda.synchronize()
    qf_np = qf.cpu().view(torch.int16).numpy().view(np.uint16) if dtype == "bf16" else qf.cpu().numpy()
    assert_close(to_np(q), oracle.rope(qf_np, d["cos"], d["sin"], -1), tol, "rope bwd q")
    assert_undone(q, to_dev(d["q"]), dtype, "rope bwd(fwd)")


def assert_undone(back, orig, dtype, what):
    """bwd(fwd(x)) returns x up to the output roundings. Each rounding of a rotated pair errs
    by at most u|pair| per element (unit roundoff u = 2^-8 for bf16, 2^-24 for fp32); rotating back keeps
    the pair error's norm (at most sqrt(2) u |pair|) and the final store adds u |pair|, so
    |bwd(fwd(x)) - x| <= (sqrt(2) + 1) u |pair| elementwise, plus fp32 arithmetic slack."""
    u = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -24
    o = orig.float()
    pair = o.reshape(*o.shape[:-1], -1, 2).norm(dim=-1).repeat_interleave(2, dim=-1)
    bound = (2 ** 0.5 + 1) * u * pair + 1e-6 * (1 + pair)
    diff = (back.float() - o).abs()
    assert bool((diff <= bound).all()), f"{what}: max excess {(diff - bound).max().item():.3g}"


def test_rope_position_zero_is_identity(gpu):
    d = wl.rope(B=2, S=4, H=3, D=128, dtype="bf16")
    q = to_dev(d["q"])
    gpu.rope_apply_(q, None, to_dev(d["cos"]), to_dev(d["sin"]), +1)
    torch.cuda.synchronize()
    assert torch.equal(q[:, 0], to_dev(d["q"])[:, 0])  # cos = 1, sin = 0: bit-exact


def test_rope_empty(gpu):
    q = torch.empty(1, 0, 4, 128, dtype=torch.bfloat16, device="cuda")
    t = torch.empty(0, 64, device="cuda")
    gpu.rope_apply_(q, None, t, t, +1)


QK_SHAPES = [(2, 37, 5, 128, "bf16"), (1, 64, 40, 128, "bf16"), (1, 50, 8, 128, "f32"), (2, 21, 3, 64, "bf16"),
             (1, 30, 4, 8, "bf16"), (1, 19, 7, 32, "f32"), (1, 24, 4, 256, "bf16")]


@pytest.mark.parametrize("B,S,H,D,dtype", QK_SHAPES)
@pytest.mark.parametrize("gemma", [False, True])
def test_qknorm_rope_fwd_bwd(gpu, B, S, H, D, dtype, gemma):
    d = wl.qknorm_rope(B=B, S=S, H=H, D=D, dtype=dtype)
    if gemma:  # Gemma weights sit around 0: w' = 1 + w
        d["wq"] = wl.normal(0, wl.S_WQ, D, dtype, scale=0.1)
        d["wk"] = wl.normal(0, wl.S_WK, D, dtype, scale=0.1)
    q, k, wq, wk = (to_dev(d[n]) for n in ("q", "k", "wq", "wk"))
    cos, sin = to_dev(d["cos"]), to_dev(d["sin"])
    qo, ko, rq, rk = gpu.qknorm_rope_fwd(q, k, wq, wk, cos, sin, d["eps"], gemma=gemma)
    dq, dk, dwq, dwk = gpu.qknorm_rope_bwd(q, k, wq, wk, cos, sin, rq, rk, to_dev(d["dq_out"]),
                                           to_dev(d["dk_out"]), gemma=gemma)
    torch.cuda.synchronize()
    for name, x, w, dy, out, r, dx, dw in (("q", d["q"], d["wq"], d["dq_out"], qo, rq, dq, dwq),
                                           ("k", d["k"], d["wk"], d["dk_out"], ko, rk, dk, dwk)):
        ro, rr = oracle.qknorm_rope_fwd(x, w, d["cos"], d["sin"], d["eps"], gemma=gemma)
        rdx, rdw = oracle.qknorm_rope_bwd(x, w, d["cos"], d["sin"], dy, d["eps"], gemma=gemma)
        tag = f"qk {name} {dtype} {B}x{S}x{H}x{D} gemma={gemma}"
        assert_close(to_np(out), ro, io_tol(dtype), tag + " out")
        assert_close(to_np(r), rr, "stat", tag + " inv_rms")
        assert_close(to_np(dx), rdx, grad_tol(dtype), tag + " dx")
        assert_close(to_np(dw), rdw, wgrad_tol(dtype, rdw), tag + " dw")


def test_qknorm_rope_without_k(gpu):
    d = wl.qknorm_rope(B=1, S=33, H=6, D=128, dtype="bf16")
    q, wq = to_dev(d["q"]), to_dev(d["wq"])
    cos, sin = to_dev(d["cos"]), to_dev(d["sin"])
    qo, ko, rq, rk = gpu.qknorm_rope_fwd(q, None, wq, None, cos, sin, d["eps"])
    dq, dk, dwq, dwk = gpu.qknorm_rope_bwd(q, None, wq, None, cos, sin, rq, None, to_dev(d["dq_out"]), None)
    torch.cuda.synchronize()
    assert ko is None and dk is None and dwk is None
    ro, _ = oracle.qknorm_rope_fwd(d["q"], d["wq"], d["cos"], d["sin"], d["eps"])
    rdx, rdw = oracle.qknorm_rope_bwd(d["q"], d["wq"], d["cos"], d["sin"], d["dq_out"], d["eps"])
    assert_close(to_np(qo), ro, "bf16", "q only out")
    assert_close(to_np(dq), rdx, "grad_bf16", "q only dx")
    assert_close(to_np(dwq), rdw, "grad_bf16", "q only dw")


@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "f32"), (64, "bf16")])
def test_qknorm_rope_degenerate_heads(gpu, D, dtype):
    """Heads the per-head statistic can trip on - all zero (inv_rms = 1/sqrt(eps), output 0),
    constant, a single large element, a tiny scale - next to ordinary heads, at position 0 (the
    identity rotation) and beyond, forward and backward against the oracle."""
    d = wl.qknorm_rope(B=1, S=4, H=6, D=D, dtype=dtype)
    rng = np.random.default_rng(D)
    j = np.arange(D)
    special = [np.zeros(D), np.full(D, -2.0), np.where(j == 5, 300.0, 0.0), 1e-3 * rng.standard_normal(D)]
    conv = (lambda a: wl.bf16_bits(a.astype(np.float32))) if dtype == "bf16" else (lambda a: a.astype(np.float32))  # noqa
    for name in ("q", "k"):
        for s_, row in enumerate(special):
            d[name][0, s_, s_ % 6] = conv(row)
    q, k, wq, wk = (to_dev(d[n]) for n in ("q", "k", "wq", "wk"))
    cos, sin = to_dev(d["cos"]), to_dev(d["sin"])
    qo, ko, rq, rk = gpu.qknorm_rope_fwd(q, k, wq, wk, cos, sin, d["eps"])
    dq, dk, dwq, dwk = gpu.qknorm_rope_bwd(q, k, wq, wk, cos, sin, rq, rk, to_dev(d["dq_out"]), to_dev(d["dk_out"]))
    torch.cuda.synchronize()
    for name, x, w, dy, out, r, dx, dw in (("q", d["q"], d["wq"], d["dq_out"], qo, rq, dq, dwq),
                                           ("k", d["k"], d["wk"], d["dk_out"], ko, rk, dk, dwk)):
        ro, rr = oracle.qknorm_rope_fwd(x, w, d["cos"], d["sin"], d["eps"])
        rdx, rdw = oracle.qknorm_rope_bwd(x, w, d["cos"], d["sin"], dy, d["eps"])
        tag = f"qk degenerate {name} {dtype} D={D}"
        assert_close(to_np(out), ro, io_tol(dtype), tag + " out")
        assert_close(to_np(r), rr, "stat", tag + " inv_rms")
        assert_close(to_np(dx), rdx, grad_tol(dtype), tag + " dx")
        assert_close(to_np(dw), rdw, wgrad_tol(dtype, rdw), tag + " dw")
    assert gpu.device_error(clear=True) == 0


def test_qknorm_unsupported_head_dim(gpu):
    q = torch.zeros(1, 2, 2, 96, dtype=torch.bfloat16, device="cuda")
    w = torch.ones(96, dtype=torch.bfloat16, device="cuda")
    t = torch.zeros(2, 48, device="cuda")
    with pytest.raises(gpu.GnError) as e:
        gpu.qknorm_rope_fwd(q, None, w, None, t, t)
    assert e.value.status == gpu.GN_ERR_UNSUPPORTED


@pytest.mark.slow
def test_rope_full_size(gpu):
    """The benchmark's launch (q, k [1, 32760, 40, 128] bf16): the forward on every element
    against the oracle, the backward on every element against the oracle applied to the
    forward's bf16 output (the backward's actual input), and the round-trip bound on every
    element."""
    c = wl.ROPE_MAIN
    d = wl.rope(**c)
    q, k = to_dev(d["q"]), to_dev(d["k"])
    cos, sin = to_dev(d["cos"]), to_dev(d["sin"])
    gpu.rope_apply_(q, k, cos, sin, +1)
    qf, kf = q.clone(), k.clone()
    gpu.rope_apply_(q, k, cos, sin, -1)
    torch.cuda.synchronize()
    B, S, H, D = q.shape

    def jobs():
        for name, fwd, bwd in (("q", qf, q), ("k", kf, k)):
            for s0, s1 in fs.token_chunks(S, B * H * D):
                yield fs.job_rope, (d[name][:, s0:s1], d["cos"][s0:s1], d["sin"][s0:s1], fs.bits(fwd[:, s0:s1]),
                                    fs.bits(bwd[:, s0:s1]), f"{name} tokens {s0}:{s1}")

    n = fs.run(jobs(), "full rope").assert_ok()
    assert n == {"fwd": 2 * B * S * H * D, "bwd": 2 * B * S * H * D}
    for name, t in (("q", q), ("k", k)):
        assert_undone(t, to_dev(d[name]), "bf16", f"full rope bwd(fwd) {name}")


@pytest.mark.slow
def test_qknorm_rope_full_size(gpu):
    """The benchmark's launch (q, k [2, 76800, 40, 128] bf16): out, inv_rms and dx of both
    tensors on every element against the oracle (chunks of tokens on host worker processes),
    dw_q and dw_k complete."""
    c = wl.QKNORM_MAIN
    d = wl.qknorm_rope(**c)
    q, k, wq, wk = (to_dev(d[n]) for n in ("q", "k", "wq", "wk"))
    cos, sin = to_dev(d["cos"]), to_dev(d["sin"])
    qo, ko, rq, rk = gpu.qknorm_rope_fwd(q, k, wq, wk, cos, sin, d["eps"])
    dq, dk, dwq, dwk = gpu.qknorm_rope_bwd(q, k, wq, wk, cos, sin, rq, rk, to_dev(d["dq_out"]), to_dev(d["dk_out"]))
    torch.cuda.synchronize()
    B, S, H, D = q.shape
    for name, x, w, dy, out, r, dx, dw in (("q", "q", "wq", "dq_out", qo, rq, dq, dwq),
                                           ("k", "k", "wk", "dk_out", ko, rk, dk, dwk)):
        def jobs():
            for s0, s1 in fs.token_chunks(S, B * H * D):
                yield fs.job_qk, (d[x][:, s0:s1], d[w], d["cos"][s0:s1], d["sin"][s0:s1], d[dy][:, s0:s1], d["eps"],
                                  False, fs.bits(out[:, s0:s1]), fs.bits(r[:, s0:s1]), fs.bits(dx[:, s0:s1]),
                                  f"{name} tokens {s0}:{s1}")

        v = fs.run(jobs(), f"full qk {name}")
        n = v.assert_ok()
        assert n == {"out": B * S * H * D, "inv_rms": B * S * H, "dx": B * S * H * D}
        assert_close(to_np(dw), v.parts["dw"], "grad_bf16", f"full qk {name} dw")
