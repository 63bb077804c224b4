"""Pins of the fp64 oracle to things other than itself (CPU only).

Each group checks the oracle against what the source pages and the mathematics fix:
hand-worked cases (tests/golden/hand_cases.json), closed forms and invariants, special
cases that reduce to a library routine (torch fp64 CPU functions and autograd, numpy complex
arithmetic, math.erf), and central finite differences of the oracle's own forward for every
backward. The cases are chosen so that a dropped term, a wrong sign, a swapped index or a
transposed operand in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from transformer_norm_rope_b200 import workloads as wl

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")))
ACTS = ["none", "gelu_tanh", "silu"]
rng = np.random.default_rng(1234)


def t64(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64))


def torch_act(act, z):
    if act == "gelu_tanh":
        return F.gelu(z, approximate="tanh")
    if act == "silu":
        return F.silu(z)
    return z


# ---------------------------------------------------------------- hand-worked cases


def test_hand_rmsnorm():
    for key, gemma in (("rmsnorm_3_4", False), ("rmsnorm_gemma_zero_weight", True)):
        c = GOLD[key]
        y, r = oracle.rmsnorm_fwd(np.array([c["x"]]), np.array(c["w"]), c["eps"], gemma=gemma)
        np.testing.assert_allclose(y[0], c["y"], rtol=0, atol=1e-15)
        np.testing.assert_allclose(r[0], c["inv_rms"], rtol=0, atol=1e-15)


def test_hand_layernorm():
    c = GOLD["layernorm_1_3"]
    y, mu, rs = oracle.layernorm_fwd(np.array([c["x"]]), None, None, c["eps"])
    np.testing.assert_allclose(y[0], c["y"], atol=1e-15)
    assert mu[0] == c["mean"] and rs[0] == c["rstd"]
    c = GOLD["layernorm_1_2_3_4_affine"]
    y, mu, rs = oracle.layernorm_fwd(np.array([c["x"]]), np.array(c["w"]), np.array(c["b"]), c["eps"])
    np.testing.assert_allclose(y[0], c["y"], atol=1e-14)
    np.testing.assert_allclose([mu[0], rs[0]], [c["mean"], c["rstd"]], atol=1e-15)


def test_hand_rope():
    for key in ("rope_quarter_turn", "rope_3_4_5"):
        c = GOLD[key]
        x = np.array(c["x"]).reshape(1, 1, 1, 2)
        cs, sn = np.array([c["cos"]]), np.array([c["sin"]])
        np.testing.assert_allclose(oracle.rope(x, cs, sn, +1).ravel(), c["fwd"], atol=1e-15)
        back = oracle.rope(np.array(c["fwd"]).reshape(1, 1, 1, 2), cs, sn, -1).ravel()
        np.testing.assert_allclose(back, c["x"], atol=1e-15)
        if "bwd" in c:
            np.testing.assert_allclose(oracle.rope(x, cs, sn, -1).ravel(), c["bwd"], atol=1e-15)


def test_hand_activations():
    c = GOLD["silu_ln3"]
    assert abs(oracle.act("silu", c["z"]) - c["silu"]) < 1e-15
    assert abs(oracle.act_grad("silu", c["z"]) - c["silu_grad"]) < 1e-15
    c = GOLD["gelu_tanh_zero"]
    assert oracle.act("gelu_tanh", c["z"]) == c["gelu"]
    assert oracle.act_grad("gelu_tanh", c["z"]) == c["gelu_grad"]
    assert oracle.act("silu", 0.0) == 0.0 and oracle.act_grad("silu", 0.0) == 0.5


# ---------------------------------------------------------------- activations


def test_gelu_tanh_close_to_exact_gelu():
    # The tanh form approximates z * Phi(z) (Phi via math.erf) to a few 1e-4 everywhere;
    # dropping the cubic term or using a wrong constant moves it by > 1e-2 near |z| ~ 2.
    zs = np.linspace(-8, 8, 4001)
    err = max(abs(oracle.act("gelu_tanh", z) - z * 0.5 * (1 + math.erf(z / math.sqrt(2)))) for z in zs)
    assert err < 5e-4


def test_gelu_tanh_limits_and_printed_constant():
    assert abs(oracle.act("gelu_tanh", 12.0) - 12.0) < 1e-12
    assert abs(oracle.act("gelu_tanh", -12.0)) < 1e-12
    # the page prints the constant as 0.79788456; the oracle's sqrt(2/pi) agrees to 1e-9
    for z in (-3.0, -0.5, 0.7, 2.5):
        page = 0.5 * z * (1 + math.tanh(0.79788456 * (z + 0.044715 * z ** 3)))
        assert abs(oracle.act("gelu_tanh", z) - page) < 1e-8


@pytest.mark.parametrize("act", ACTS)
def test_activation_matches_torch(act):
    z = np.linspace(-9, 9, 301)
    ref = torch_act(act, t64(z)).numpy()
    got = np.array([oracle.act(act, v) for v in z])
    np.testing.assert_allclose(got, ref, rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("act", ACTS)
def test_activation_grad_matches_fd_and_autograd(act):
    z = np.linspace(-7, 7, 141)
    h = 1e-6
    fd = np.array([(oracle.act(act, v + h) - oracle.act(act, v - h)) / (2 * h) for v in z])
    got = np.array([oracle.act_grad(act, v) for v in z])
    np.testing.assert_allclose(got, fd, rtol=1e-7, atol=1e-8)
    zt = t64(z).requires_grad_()
    torch_act(act, zt).sum().backward()
    np.testing.assert_allclose(got, zt.grad.numpy(), rtol=1e-13, atol=1e-14)


def test_silu_odd_part_identity():
    # silu(z) - silu(-z) = z because sigmoid(z) + sigmoid(-z) = 1
    for z in (-4.0, -1.3, 0.2, 3.3, 9.0):
        assert abs(oracle.act("silu", z) - oracle.act("silu", -z) - z) < 1e-14


# ---------------------------------------------------------------- RMSNorm


def test_rmsnorm_unit_rms_rows():
    x = rng.standard_normal((9, 33)) * rng.uniform(0.1, 30, (9, 1))
    y, r = oracle.rmsnorm_fwd(x, np.ones(33), 0.0)
    np.testing.assert_allclose(np.sqrt((y ** 2).mean(1)), 1.0, rtol=1e-14)
    eps = 0.25
    y, _ = oracle.rmsnorm_fwd(x, np.ones(33), eps)
    ms = (x ** 2).mean(1)
    np.testing.assert_allclose(np.sqrt((y ** 2).mean(1)), np.sqrt(ms / (ms + eps)), rtol=1e-13)


@pytest.mark.parametrize("act", ACTS)
def test_rmsnorm_scale_invariance(act):
    x = rng.standard_normal((4, 20))
    w = 1 + 0.1 * rng.standard_normal(20)
    y1, r1 = oracle.rmsnorm_fwd(x, w, 0.0, act=act)
    y2, r2 = oracle.rmsnorm_fwd(50.0 * x, w, 0.0, act=act)
    np.testing.assert_allclose(y1, y2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(r1, 50.0 * r2, rtol=1e-14)


@pytest.mark.parametrize("act", ACTS)
@pytest.mark.parametrize("gemma", [False, True])
def test_rmsnorm_matches_torch_fp64(act, gemma):
    x = rng.standard_normal((7, 48)) * 3
    w = 0.1 * rng.standard_normal(48) + (0.0 if gemma else 1.0)
    dy = rng.standard_normal((7, 48))
    eps = 1e-6
    xt = t64(x).requires_grad_()
    wt = t64(w).requires_grad_()
    yt = torch_act(act, F.rms_norm(xt, (48,), (1.0 + wt) if gemma else wt, eps))
    (yt * t64(dy)).sum().backward()
    y, r = oracle.rmsnorm_fwd(x, w, eps, gemma=gemma, act=act)
    dx, dw = oracle.rmsnorm_bwd(x, w, dy, eps, gemma=gemma, act=act)
    np.testing.assert_allclose(y, yt.detach().numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(r, 1.0 / np.sqrt((x ** 2).mean(1) + eps), rtol=1e-14)
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dw, wt.grad.numpy(), rtol=1e-11, atol=1e-12)


def test_rmsnorm_gemma_is_plain_with_weight_plus_one():
    x = rng.standard_normal((5, 24))
    w = 0.1 * rng.standard_normal(24)
    dy = rng.standard_normal((5, 24))
    for act in ACTS:
        a = oracle.rmsnorm_fwd(x, w, 1e-6, gemma=True, act=act)
        b = oracle.rmsnorm_fwd(x, w + 1.0, 1e-6, gemma=False, act=act)
        np.testing.assert_allclose(a[0], b[0], rtol=1e-15, atol=1e-15)
        ga = oracle.rmsnorm_bwd(x, w, dy, 1e-6, gemma=True, act=act)
        gb = oracle.rmsnorm_bwd(x, w + 1.0, dy, 1e-6, gemma=False, act=act)
        np.testing.assert_allclose(ga[0], gb[0], rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(ga[1], gb[1], rtol=1e-13, atol=1e-15)


def _fd_grad(f, a, h=1e-6):
    g = np.zeros_like(a)
    flat, gf = a.reshape(-1), g.reshape(-1)
    for i in range(flat.size):
        o = flat[i]
        flat[i] = o + h
        up = f()
        flat[i] = o - h
        dn = f()
        flat[i] = o
        gf[i] = (up - dn) / (2 * h)
    return g


@pytest.mark.parametrize("act", ACTS)
@pytest.mark.parametrize("gemma", [False, True])
def test_rmsnorm_bwd_finite_differences(act, gemma):
    M, N, eps = 3, 7, 1e-3
    x = rng.standard_normal((M, N))
    w = rng.standard_normal(N) * 0.3 + (0.0 if gemma else 1.0)
    dy = rng.standard_normal((M, N))
    loss = lambda: float((oracle.rmsnorm_fwd(x, w, eps, gemma=gemma, act=act)[0] * dy).sum())
    dx, dw = oracle.rmsnorm_bwd(x, w, dy, eps, gemma=gemma, act=act)
    np.testing.assert_allclose(dx, _fd_grad(loss, x), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dw, _fd_grad(loss, w), rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("act", ACTS)
def test_rmsnorm_bwd_orthogonal_to_x_at_zero_eps(act):
    # y depends on x only through x / rms(x), so dx . x = 0 per row when eps = 0
    x = rng.standard_normal((6, 40))
    dx, _ = oracle.rmsnorm_bwd(x, 1 + 0.1 * rng.standard_normal(40), rng.standard_normal((6, 40)),
                               0.0, act=act)
    assert np.abs((dx * x).sum(1)).max() < 1e-12


def test_rmsnorm_bf16_and_f32_inputs_widen_exactly():
    x = rng.standard_normal((3, 16)).astype(np.float32)
    bits = wl.bf16_bits(x)
    widened = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    w = np.ones(16, np.float32)
    a = oracle.rmsnorm_fwd(bits, wl.bf16_bits(w), 1e-6)
    b = oracle.rmsnorm_fwd(widened, w.astype(np.float64), 1e-6)
    np.testing.assert_array_equal(a[0], b[0])
    c = oracle.rmsnorm_fwd(x, w, 1e-6)
    d = oracle.rmsnorm_fwd(x.astype(np.float64), w.astype(np.float64), 1e-6)
    np.testing.assert_array_equal(c[0], d[0])


def test_rmsnorm_rows_are_independent():
    x = rng.standard_normal((8, 12))
    w = 1 + 0.1 * rng.standard_normal(12)
    y, r = oracle.rmsnorm_fwd(x, w, 1e-6)
    for m in (0, 5, 7):
        ym, rm = oracle.rmsnorm_fwd(x[m:m + 1], w, 1e-6)
        np.testing.assert_array_equal(ym[0], y[m])
        assert rm[0] == r[m]


# ---------------------------------------------------------------- LayerNorm


def test_layernorm_zero_mean_unit_variance():
    x = rng.standard_normal((10, 37)) * rng.uniform(0.5, 3, (10, 1)) + rng.uniform(-2, 2, (10, 1))
    y, mu, rs = oracle.layernorm_fwd(x, None, None, 0.0)
    assert np.abs(y.mean(1)).max() < 1e-14
    np.testing.assert_allclose(y.var(1), 1.0, rtol=1e-13)
    np.testing.assert_allclose(mu, x.mean(1), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(rs, 1 / np.sqrt(x.var(1)), rtol=1e-13)


def test_layernorm_shift_invariance():
    x = rng.standard_normal((4, 21))
    w, b = 1 + 0.1 * rng.standard_normal(21), 0.1 * rng.standard_normal(21)
    for act in ACTS:
        y1 = oracle.layernorm_fwd(x, w, b, 1e-5, act=act)[0]
        y2 = oracle.layernorm_fwd(x + 1.75, w, b, 1e-5, act=act)[0]
        np.testing.assert_allclose(y1, y2, rtol=1e-12, atol=1e-13)


def test_layernorm_none_weight_bias_are_one_zero():
    x = rng.standard_normal((3, 10))
    a = oracle.layernorm_fwd(x, None, None, 1e-5, act="silu")[0]
    b = oracle.layernorm_fwd(x, np.ones(10), np.zeros(10), 1e-5, act="silu")[0]
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("act", ACTS)
def test_layernorm_matches_torch_fp64(act):
    M, N, eps = 6, 40, 1e-5
    x = rng.standard_normal((M, N)) * 2 + 1.5
    w, b = 1 + 0.1 * rng.standard_normal(N), 0.1 * rng.standard_normal(N)
    dy = rng.standard_normal((M, N))
    xt, wt, bt = (t64(a).requires_grad_() for a in (x, w, b))
    yt = torch_act(act, F.layer_norm(xt, (N,), wt, bt, eps))
    (yt * t64(dy)).sum().backward()
    y, mu, rs = oracle.layernorm_fwd(x, w, b, eps, act=act)
    dx, dw, db = oracle.layernorm_bwd(x, w, b, dy, eps, act=act)
    np.testing.assert_allclose(y, yt.detach().numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dw, wt.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(db, bt.grad.numpy(), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("act", ACTS)
def test_layernorm_bwd_finite_differences(act):
    M, N, eps = 3, 6, 1e-3
    x = rng.standard_normal((M, N)) + 0.5
    w, b = 1 + 0.3 * rng.standard_normal(N), 0.3 * rng.standard_normal(N)
    dy = rng.standard_normal((M, N))
    loss = lambda: float((oracle.layernorm_fwd(x, w, b, eps, act=act)[0] * dy).sum())
    dx, dw, db = oracle.layernorm_bwd(x, w, b, dy, eps, act=act)
    np.testing.assert_allclose(dx, _fd_grad(loss, x), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dw, _fd_grad(loss, w), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(db, _fd_grad(loss, b), rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("act", ACTS)
def test_layernorm_bwd_sums_to_zero(act):
    # y is invariant to adding a constant to a row, so each row of dx sums to 0 (any eps)
    x = rng.standard_normal((5, 30))
    dx, _, _ = oracle.layernorm_bwd(x, 1 + 0.1 * rng.standard_normal(30), 0.1 * rng.standard_normal(30),
                                    rng.standard_normal((5, 30)), 1e-5, act=act)
    assert np.abs(dx.sum(1)).max() < 1e-12


# ---------------------------------------------------------------- rotary embedding


def _angles(S, D, p0=0, theta=10000.0):
    i = np.arange(D // 2)
    return (np.arange(p0, p0 + S)[:, None]) * theta ** (-2.0 * i / D)[None, :]


@pytest.mark.parametrize("sign", [+1, -1])
def test_rope_is_complex_multiplication(sign):
    B, S, H, D = 2, 5, 3, 8
    x = rng.standard_normal((B, S, H, D))
    ang = _angles(S, D, p0=3)
    out = oracle.rope(x, np.cos(ang), np.sin(ang), sign)
    z = x[..., 0::2] + 1j * x[..., 1::2]
    ref = z * np.exp(1j * sign * ang)[None, :, None, :]
    np.testing.assert_allclose(out[..., 0::2], ref.real, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(out[..., 1::2], ref.imag, rtol=1e-14, atol=1e-15)


def test_rope_identity_at_position_zero_and_norm_preserving():
    B, S, H, D = 1, 6, 4, 16
    cos, sin = wl.rope_tables(S, D)
    assert np.all(cos[0] == 1) and np.all(sin[0] == 0)
    x = rng.standard_normal((B, S, H, D))
    out = oracle.rope(x, cos, sin, +1)
    np.testing.assert_array_equal(out[:, 0], x[:, 0])
    n_in = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    n_out = out[..., 0::2] ** 2 + out[..., 1::2] ** 2
    # tables are fp32-rounded, so cos^2 + sin^2 = 1 only to ~1e-7
    np.testing.assert_allclose(n_out, n_in, rtol=3e-7)
    a = _angles(S, D)
    out64 = oracle.rope(x, np.cos(a), np.sin(a), +1)
    np.testing.assert_allclose(out64[..., 0::2] ** 2 + out64[..., 1::2] ** 2, n_in, rtol=1e-14)


def test_rope_inverse_and_angle_additivity():
    B, S, H, D = 2, 7, 2, 12
    x = rng.standard_normal((B, S, H, D))
    a1, a2 = _angles(S, D, p0=11), _angles(S, D, p0=5, theta=500.0)
    back = oracle.rope(oracle.rope(x, np.cos(a1), np.sin(a1), +1), np.cos(a1), np.sin(a1), -1)
    np.testing.assert_allclose(back, x, rtol=0, atol=1e-14)
    two = oracle.rope(oracle.rope(x, np.cos(a1), np.sin(a1), +1), np.cos(a2), np.sin(a2), +1)
    one = oracle.rope(x, np.cos(a1 + a2), np.sin(a1 + a2), +1)
    np.testing.assert_allclose(two, one, rtol=1e-13, atol=1e-14)


def test_rope_backward_is_adjoint():
    # <R x, g> = <x, R^T g>, with R^T the sin-negated rotation
    B, S, H, D = 1, 9, 3, 10
    x, g = rng.standard_normal((2, B, S, H, D))
    a = _angles(S, D)
    lhs = (oracle.rope(x, np.cos(a), np.sin(a), +1) * g).sum()
    rhs = (x * oracle.rope(g, np.cos(a), np.sin(a), -1)).sum()
    assert abs(lhs - rhs) < 1e-12


def test_rope_table_rows_follow_token_not_batch_or_head():
    B, S, H, D = 3, 4, 5, 8
    x = np.broadcast_to(rng.standard_normal(D), (B, S, H, D)).copy()
    a = _angles(S, D)
    out = oracle.rope(x, np.cos(a), np.sin(a), +1)
    for s in range(S):
        np.testing.assert_array_equal(out[:, s], np.broadcast_to(out[0, s, 0], (B, H, D)))
    assert not np.allclose(out[0, 1, 0], out[0, 2, 0])


# ---------------------------------------------------------------- qk-norm + rotary embedding


def _torch_qk(xt, wt, cos, sin, eps, gemma):
    n = F.rms_norm(xt, (xt.shape[-1],), (1.0 + wt) if gemma else wt, eps)
    z = torch.view_as_complex(n.reshape(*n.shape[:-1], -1, 2).contiguous())
    rot = torch.polar(torch.ones_like(t64(cos)), torch.atan2(t64(sin), t64(cos)))
    out = torch.view_as_real(z * rot[None, :, None, :]).reshape(n.shape)
    return out


@pytest.mark.parametrize("gemma", [False, True])
def test_qknorm_rope_matches_torch_fp64(gemma):
    B, S, H, D, eps = 2, 5, 3, 16, 1e-6
    x = rng.standard_normal((B, S, H, D)) * 2
    w = 0.1 * rng.standard_normal(D) + (0.0 if gemma else 1.0)
    dy = rng.standard_normal((B, S, H, D))
    a = _angles(S, D, p0=2)
    cos, sin = np.cos(a), np.sin(a)
    xt, wt = t64(x).requires_grad_(), t64(w).requires_grad_()
    ot = _torch_qk(xt, wt, cos, sin, eps, gemma)
    (ot * t64(dy)).sum().backward()
    out, r = oracle.qknorm_rope_fwd(x, w, cos, sin, eps, gemma=gemma)
    dx, dw = oracle.qknorm_rope_bwd(x, w, cos, sin, dy, eps, gemma=gemma)
    np.testing.assert_allclose(out, ot.detach().numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(r, 1 / np.sqrt((x ** 2).mean(-1) + eps), rtol=1e-14)
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dw, wt.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_qknorm_rope_bwd_finite_differences():
    B, S, H, D, eps = 1, 3, 2, 8, 1e-3
    x = rng.standard_normal((B, S, H, D))
    w = 1 + 0.3 * rng.standard_normal(D)
    dy = rng.standard_normal((B, S, H, D))
    a = _angles(S, D, p0=1)
    cos, sin = np.cos(a), np.sin(a)
    loss = lambda: float((oracle.qknorm_rope_fwd(x, w, cos, sin, eps)[0] * dy).sum())
    dx, dw = oracle.qknorm_rope_bwd(x, w, cos, sin, dy, eps)
    np.testing.assert_allclose(dx, _fd_grad(loss, x), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dw, _fd_grad(loss, w), rtol=1e-6, atol=1e-8)


def test_qknorm_rope_is_composition_of_norm_and_rope():
    B, S, H, D = 1, 4, 3, 8
    x = rng.standard_normal((B, S, H, D))
    w = 1 + 0.1 * rng.standard_normal(D)
    cos, sin = wl.rope_tables(S, D)
    out, r = oracle.qknorm_rope_fwd(x, w, cos, sin, 1e-6)
    n, r2 = oracle.rmsnorm_fwd(x.reshape(-1, D), w, 1e-6)
    np.testing.assert_array_equal(out, oracle.rope(n.reshape(x.shape), cos, sin, +1))
    np.testing.assert_array_equal(r.ravel(), r2)


# ---- normalization followed by the linear layer (Janus-Pro page, section 4.1; HY-Motion page,
# section 3.1) -------------------------------------------------------------------------------


def test_hand_norm_linear():
    # LayerNorm of [1, 3]: mean 2, variance 1 (eps 0), xn = [-1, 1]; W = [[1, 2]], bias 0.5
    y, mu, rs = oracle.norm_linear(np.array([[1.0, 3.0]]), np.ones(2), np.zeros(2), np.array([[1.0, 2.0]]),
                                   np.array([0.5]), 0.0, "ln")
    assert y[0, 0] == 1.5 and mu[0] == 2.0 and rs[0] == 1.0
    # RMSNorm of [3, 4]: mean square 12.5; W = [[1, 1]] -> 7 / sqrt(12.5); with SiLU on top
    y, mu, rs = oracle.norm_linear(np.array([[3.0, 4.0]]), np.ones(2), None, np.array([[1.0, 1.0]]), None, 0.0, "rms")
    assert y[0, 0] == pytest.approx(7 / math.sqrt(12.5), rel=1e-15) and mu[0] == 0.0
    z = 7 / math.sqrt(12.5) + 0.25
    y, _, _ = oracle.norm_linear(np.array([[3.0, 4.0]]), np.ones(2), None, np.array([[1.0, 1.0]]), np.array([0.25]),
                                 0.0, "rms", act="silu")
    assert y[0, 0] == pytest.approx(z / (1 + math.exp(-z)), rel=1e-14)


@pytest.mark.parametrize("norm,act,gemma", [("ln", "none", False), ("ln", "silu", False), ("ln", "gelu_tanh", False),
                                            ("rms", "silu", False), ("rms", "none", True)])
def test_norm_linear_is_the_norm_then_a_matmul(norm, act, gemma):
    # the normalization (pinned above) followed by numpy's fp64 matrix product, bias and the
    # activation; W is deliberately not square, so a transposed operand cannot pass
    M, N, K, eps = 7, 5, 24, 1e-5
    x = rng.standard_normal((M, K)) * 2 + 0.7
    g = 1 + 0.2 * rng.standard_normal(K)
    beta = 0.3 * rng.standard_normal(K)
    W = rng.standard_normal((N, K)) / math.sqrt(K)
    bias = rng.standard_normal(N)
    y, mu, rs = oracle.norm_linear(x, g, beta, W, bias, eps, norm, gemma=gemma, act=act)
    if norm == "ln":
        xn, m2, r2 = oracle.layernorm_fwd(x, g, beta, eps)
        np.testing.assert_array_equal(mu, m2)
    else:
        xn, r2 = oracle.rmsnorm_fwd(x, g, eps, gemma=gemma)
        assert not mu.any()
    np.testing.assert_array_equal(rs, r2)
    z = xn @ W.T + bias
    ref = np.vectorize(lambda v: oracle.act(act, v))(z)
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-13)


def test_norm_linear_with_identity_weight_is_the_norm():
    M, K = 4, 16
    x = rng.standard_normal((M, K))
    g, beta = 1 + 0.1 * rng.standard_normal(K), 0.1 * rng.standard_normal(K)
    y, _, _ = oracle.norm_linear(x, g, beta, np.eye(K), None, 1e-6, "ln")
    np.testing.assert_allclose(y, oracle.layernorm_fwd(x, g, beta, 1e-6)[0], rtol=1e-15, atol=1e-15)
    # output feature n reads row n of W: a one-hot row picks one normalized column
    W = np.zeros((3, K))
    W[0, 5], W[1, 0], W[2, K - 1] = 1.0, 1.0, 1.0
    y, _, _ = oracle.norm_linear(x, g, beta, W, None, 1e-6, "ln")
    xn = oracle.layernorm_fwd(x, g, beta, 1e-6)[0]
    np.testing.assert_array_equal(y, xn[:, [5, 0, K - 1]])


# ---- the linear layer with an activation, forward and backward (Helios kernels article,
# section "内核三 TiledLinear": chunking along the tokens changes none of these values) ----------


@pytest.mark.parametrize("act", ["none", "silu", "gelu_tanh"])
def test_linear_act_matches_torch_fp64(act):
    M, N, K = 6, 5, 7
    x, W, b = rng.standard_normal((M, K)), rng.standard_normal((N, K)), rng.standard_normal(N)
    dy = rng.standard_normal((M, N))
    xt, Wt, bt = t64(x).requires_grad_(), t64(W).requires_grad_(), t64(b).requires_grad_()
    z = F.linear(xt, Wt, bt)
    y = {"none": lambda v: v, "silu": F.silu, "gelu_tanh": lambda v: F.gelu(v, approximate="tanh")}[act](z)
    (y * t64(dy)).sum().backward()
    yo, _, _ = oracle.norm_linear(x, None, None, W, b, 0.0, "none", act=act)
    np.testing.assert_allclose(yo, y.detach().numpy(), rtol=1e-12, atol=1e-12)
    dx, dW, db = oracle.linear_act_bwd(x, W, b, dy, act)
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dW, Wt.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(db, bt.grad.numpy(), rtol=1e-11, atol=1e-12)


def test_linear_act_bwd_finite_differences():
    M, N, K = 3, 4, 5
    x, W, b = rng.standard_normal((M, K)), rng.standard_normal((N, K)), rng.standard_normal(N)
    dy = rng.standard_normal((M, N))
    loss = lambda: float((oracle.norm_linear(x, None, None, W, b, 0.0, "none", act="silu")[0] * dy).sum())
    dx, dW, db = oracle.linear_act_bwd(x, W, b, dy, "silu")
    np.testing.assert_allclose(dx, _fd_grad(loss, x), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dW, _fd_grad(loss, W), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(db, _fd_grad(loss, b), rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("norm,act,gemma", [("ln", "silu", False), ("ln", "gelu_tanh", False), ("rms", "silu", True),
                                            ("rms", "none", False)])
def test_norm_linear_bwd_finite_differences(norm, act, gemma):
    """The backward of the normalization followed by the linear layer, against central differences
    of the oracle's own forward (fp64): every gradient, every element. A dropped term of the
    norm's backward, a transposed product or a wrong chain-rule order fails here."""
    M, N, K = 3, 4, 6
    x = rng.standard_normal((M, K)) * 2.0 + 0.5
    g = 1.0 + 0.3 * rng.standard_normal(K)
    beta = 0.2 * rng.standard_normal(K) if norm == "ln" else None
    W, b = rng.standard_normal((N, K)), rng.standard_normal(N)
    dy = rng.standard_normal((M, N))
    eps = 1e-3
    loss = lambda: float((oracle.norm_linear(x, g, beta, W, b, eps, norm, gemma=gemma, act=act)[0] * dy).sum())
    dx, dg, dbeta, dW, db = oracle.norm_linear_bwd(x, g, beta, W, b, dy, eps, norm, gemma=gemma, act=act)
    for got, var in ((dx, x), (dg, g), (dW, W), (db, b)) + (((dbeta, beta),) if norm == "ln" else ()):
        np.testing.assert_allclose(got, _fd_grad(loss, var), rtol=1e-6, atol=1e-8)
    if norm != "ln":
        assert dbeta is None
