"""The torch helpers validate every tensor before its pointer reaches the C ABI, which sees raw
pointers only (CPU): a tensor of the wrong size, dtype, layout or device raises in Python, and the
argument patterns that the GPU tests and the benchmark use pass. The library calls and the CUDA
stream are replaced by recording stubs, and CPU tensors stand in for device tensors."""
import pytest
import torch

import transformer_norm_rope_b200 as gn

bf = torch.bfloat16
f32 = torch.float32


@pytest.fixture
def stub(monkeypatch):
    calls = []
    monkeypatch.setattr(gn, "_on_gpu", lambda t: True)
    monkeypatch.setattr(gn, "_stream", lambda stream=None: 0)
    for name in gn.SIGNATURES:
        if name.endswith("_workspace"):
            monkeypatch.setattr(gn, name, lambda *a: 1024)
        else:
            monkeypatch.setattr(gn, name, lambda *a, _n=name: calls.append(_n) or gn.GN_OK)
    return calls


def z(*shape, dtype=bf):
    return torch.zeros(shape, dtype=dtype)


def test_cpu_tensors_are_refused_before_any_call():
    with pytest.raises(ValueError, match="CUDA"):
        gn.rmsnorm_fwd(z(4, 64), z(64))
    with pytest.raises(ValueError, match="CUDA"):
        gn.rope_apply_(z(1, 2, 3, 8), None, z(2, 4, dtype=f32), z(2, 4, dtype=f32))
    with pytest.raises(ValueError, match="CUDA"):
        gn.act_grad(z(8), z(8))


def test_norm_helpers(stub):
    x, w, dy = z(6, 64), z(64), z(6, 64)
    y, r = gn.rmsnorm_fwd(x, w)
    gn.rmsnorm_bwd(x, w, r, dy)
    base = z(6, 128)
    gn.rmsnorm_fwd(base[:, :64], w, out=base[:, :64])  # strided rows, in place
    y, mu, rs = gn.layernorm_fwd(x, w, None)
    gn.layernorm_bwd(x, None, w, mu, rs, dy)
    e = z(0, 64)
    gn.layernorm_bwd(e, w, None, z(0, dtype=f32), z(0, dtype=f32), e)
    assert stub == ["gn_rmsnorm_fwd", "gn_rmsnorm_bwd", "gn_rmsnorm_fwd", "gn_layernorm_fwd",
                    "gn_layernorm_bwd", "gn_layernorm_bwd"]
    bad = [
        lambda: gn.rmsnorm_fwd(x, z(63)),  # weight shorter than the row
        lambda: gn.rmsnorm_fwd(x, z(64, dtype=f32)),  # weight dtype
        lambda: gn.rmsnorm_fwd(x, w, out=z(6, 32)),
        lambda: gn.rmsnorm_fwd(z(6, 64, dtype=f32), w),
        lambda: gn.rmsnorm_fwd(z(64, 6).t(), w),  # last dimension strided
        lambda: gn.rmsnorm_bwd(x, w, z(5, dtype=f32), dy),  # one inv_rms per row
        lambda: gn.rmsnorm_bwd(x, w, z(6, dtype=bf), dy),
        lambda: gn.rmsnorm_bwd(x, w, z(6, dtype=f32), z(6, 32)),
        lambda: gn.rmsnorm_bwd(x, w, None, dy),
        lambda: gn.layernorm_fwd(x, z(32), None),
        lambda: gn.layernorm_fwd(x, None, z(64, dtype=f32)),
        lambda: gn.layernorm_bwd(x, w, None, z(6, dtype=f32), z(7, dtype=f32), dy),
        lambda: gn.layernorm_bwd(x, w, None, z(6, dtype=f32), z(12, dtype=f32)[::2], dy),
    ]
    for f in bad:
        with pytest.raises((ValueError, TypeError)):
            f()
    assert len(stub) == 6  # none of the refused calls reached the library


def test_rotary_helpers(stub):
    B, S, H, D = 2, 5, 3, 16
    q, k, t = z(B, S, H, D), z(B, S, H, D), z(S, D // 2, dtype=f32)
    gn.rope_apply_(q, k, t, t)
    gn.rope_apply_(q, None, t, t, -1)
    qo, ko, rq, rk = gn.qknorm_rope_fwd(q, k, z(D), z(D), t, t)
    gn.qknorm_rope_bwd(q, k, z(D), z(D), t, t, rq, rk, qo, ko)
    gn.qknorm_rope_fwd(q, None, z(D), None, t, t)
    gn.qknorm_rope_bwd(q, None, z(D), None, t, t, rq, None, qo, None)
    assert len(stub) == 6
    bad = [
        lambda: gn.rope_apply_(q, z(B, S, H, 8), t, t),
        lambda: gn.rope_apply_(q, z(B, S, H, D, dtype=f32), t, t),
        lambda: gn.rope_apply_(q, None, z(S, D, dtype=f32), t),  # [S, D] table
        lambda: gn.rope_apply_(q, None, t, z(S - 1, D // 2, dtype=f32)),
        lambda: gn.rope_apply_(q, None, t.to(torch.float64), t),
        lambda: gn.rope_apply_(z(B, S, D, H).transpose(2, 3), None, t, t),
        lambda: gn.rope_apply_(z(S, H, D), None, t, t),
        lambda: gn.qknorm_rope_fwd(q, k, z(D), None, t, t),  # k without its weight
        lambda: gn.qknorm_rope_fwd(q, None, z(D // 2), None, t, t),
        lambda: gn.qknorm_rope_bwd(q, k, z(D), z(D), t, t, rq, z(B * S * H - 1, dtype=f32), qo, ko),
        lambda: gn.qknorm_rope_bwd(q, k, z(D), z(D), t, t, rq, rk, qo, None),
        lambda: gn.qknorm_rope_bwd(q, None, z(D), None, t, t, rq, None, z(B, S, H, 8), None),
    ]
    for f in bad:
        with pytest.raises((ValueError, TypeError)):
            f()
    assert len(stub) == 6


def test_linear_helpers(stub):
    M, N, K = 12, 32, 64
    W = z(N, K)
    Wf, c, d = gn.norm_linear_prepare(W, z(K), z(K), z(N), norm="ln")
    gn.norm_linear_fwd(z(M, K), Wf, c, d, norm="ln")
    Wn, _, dn = gn.norm_linear_prepare(W, None, None, z(N), norm="none")
    y = z(M, N)
    gn.norm_linear_fwd(z(M, K)[4:8], Wn, None, dn, norm="none", out=y[4:8])
    gn.act_grad(y, z(M, N), out=y)
    gn.act_fwd(y, out=y)
    assert stub == ["gn_norm_linear_prepare", "gn_norm_linear_fwd", "gn_norm_linear_prepare",
                    "gn_norm_linear_fwd", "gn_act_grad", "gn_act_fwd"]
    bad = [
        lambda: gn.norm_linear_prepare(W, z(N), None, None),  # g is over K
        lambda: gn.norm_linear_prepare(W, None, None, z(K)),  # bias is over N
        lambda: gn.norm_linear_prepare(z(N, K, 2), None, None, None),
        lambda: gn.norm_linear_fwd(z(M, K + 8), Wf, c, d, norm="ln"),
        lambda: gn.norm_linear_fwd(z(M, K), Wf, None, d, norm="ln"),  # LayerNorm needs c
        lambda: gn.norm_linear_fwd(z(M, K), Wf, c, z(N), norm="ln"),  # d is fp32
        lambda: gn.norm_linear_fwd(z(M, K), Wf, c, d, norm="ln", out=z(M, N + 1)),
        lambda: gn.norm_linear_fwd(z(M, K, dtype=f32), Wf, c, d, norm="ln"),
        lambda: gn.act_grad(z(M, N), z(M, N + 1)),
        lambda: gn.act_grad(z(M, N, dtype=f32), z(M, N)),
        lambda: gn.act_grad(z(N, M).t(), z(M, N)),
        lambda: gn.act_grad(z(M, N), z(M, N), out=z(M, N, dtype=f32)),
        lambda: gn.act_fwd(z(N, M).t()),
        lambda: gn.act_fwd(z(M, N), out=z(M, N + 1)),
        lambda: gn.act_fwd(z(M, N), out=z(M, N, dtype=f32)),
    ]
    for f in bad:
        with pytest.raises((ValueError, TypeError)):
            f()
    assert len(stub) == 6


def test_tiled_linear_autograd_plumbing(stub, monkeypatch):
    # with the kernels stubbed, the values are meaningless; the test checks that the autograd
    # form saves what it needs, returns one gradient per input, of the input's dtype and shape,
    # and runs every step of every chunk on the library's entry points
    from transformer_norm_rope_b200 import tiled_linear as tl

    class _Sync:  # stands in for a CUDA stream and a CUDA event (no GPU here)
        def wait_event(self, e):
            pass

        def record(self, s=None):
            pass

    monkeypatch.setattr(tl, "_stream_pair", lambda device: (_Sync(), _Sync()))
    monkeypatch.setattr(tl, "_event", _Sync)
    M, N, K = 24, 16, 32
    x = z(M, K).requires_grad_()
    W = z(N, K).requires_grad_()
    b = z(N).requires_grad_()
    y = tl.TiledLinearFunction.apply(x, W, b, "silu", 3)
    assert y.shape == (M, N) and y.dtype == bf
    y.backward(z(M, N))
    assert x.grad.shape == x.shape and W.grad.shape == W.shape and b.grad.shape == b.shape
    assert x.grad.dtype == W.grad.dtype == b.grad.dtype == bf
    x2 = z(M, K).requires_grad_()
    tl.TiledLinearFunction.apply(x2, W, None, "gelu_tanh", None).backward(z(M, N))
    assert x2.grad.shape == x2.shape
    chunks = 3 + 1  # 3 chunks, then ceil(24 / 32) = 1
    assert stub.count("gn_norm_linear_fwd") == 3 + 1  # the forward: chunked on request, else one launch
    for step in ("gn_linear_act_grad", "gn_linear_bf16", "gn_linear_acc_f32", "gn_colsum_bf16"):
        assert stub.count(step) == chunks, step  # the backward, per chunk


@pytest.mark.parametrize("rows,chunks", [(32768, 7), (1000, 2), (300, 2), (64, 1), (5000, 5), (1, 1), (0, 3),
                                         (4100, 16), (257, 2), (9999, 3)])
def test_tiled_linear_chunk_bounds(rows, chunks):
    """Chunks tile the rows in order, start on 8-row boundaries, keep the count that 8-row rounding
    gives, and start on 256-row tile boundaries whenever that keeps the count."""
    from transformer_norm_rope_b200 import tiled_linear as tl

    b = list(tl._bounds(rows, chunks))
    assert all(b[i][1] == b[i + 1][0] for i in range(len(b) - 1))
    assert (b[0][0], b[-1][1]) == (0, rows) if rows else b == []
    assert all(r1 > r0 for r0, r1 in b) and all(r0 % 8 == 0 for r0, _ in b)
    if rows:
        step8 = -(-(-(-rows // chunks)) // 8) * 8
        assert len(b) == -(-rows // step8)
        step256 = -(-(-(-rows // chunks)) // 256) * 256
        if -(-rows // step256) == len(b):
            assert all(r0 % 256 == 0 for r0, _ in b)
