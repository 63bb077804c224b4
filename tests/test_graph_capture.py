"""The library's calls inside a CUDA graph.

Every entry point allocates nothing, never synchronizes and launches on the stream it is given,
so a sequence of calls can be captured once (torch.cuda.graph) and replayed: each replay must
give the outputs that the same calls give when launched directly, bit for bit (every kernel here
is deterministic), and it must agree with the oracle. The sequence covers every kernel family:
the norm forwards and backwards with their column reductions (launched with programmatic
dependent launch, which a graph keeps as a programmatic edge), RoPE in place, qk-norm + RoPE,
the fused norm + linear on pairs of SMs and the TiledLinear gradient products.
"""
import pytest
import torch

import oracle
import transformer_norm_rope_b200 as gn
from transformer_norm_rope_b200 import workloads as wl
from tests._util import assert_close, grad_tol, io_tol, to_dev, to_np

pytestmark = pytest.mark.gpu


def _inputs():
    r = wl.rmsnorm(M=300, N=5120, dtype="bf16", gemma=True, outliers=False)
    ln = wl.layernorm(M=300, N=5120, dtype="bf16")
    o = wl.rope(B=1, S=96, H=40, D=128, dtype="bf16")
    q = wl.qknorm_rope(B=2, S=48, H=40, D=128, dtype="bf16")
    nl = wl.norm_linear(M=520, N=1024, K=1024)
    host = {"r": r, "ln": ln, "o": o, "q": q, "nl": nl}
    t = {
        "rx": to_dev(r["x"]), "rw": to_dev(r["w"]), "rdy": to_dev(r["dy"]),
        "lx": to_dev(ln["x"]), "lw": to_dev(ln["w"]), "lb": to_dev(ln["b"]), "ldy": to_dev(ln["dy"]),
        "oq": to_dev(o["q"]), "ok": to_dev(o["k"]), "ocos": to_dev(o["cos"]), "osin": to_dev(o["sin"]),
        "qq": to_dev(q["q"]), "qk": to_dev(q["k"]), "qwq": to_dev(q["wq"]), "qwk": to_dev(q["wk"]),
        "qcos": to_dev(q["cos"]), "qsin": to_dev(q["sin"]), "qdq": to_dev(q["dq_out"]), "qdk": to_dev(q["dk_out"]),
        "nx": to_dev(nl["x"]), "ng": to_dev(nl["g"]), "nbeta": to_dev(nl["beta"]), "nW": to_dev(nl["W"]),
        "nbias": to_dev(nl["bias"]),
    }
    t["ndy"] = torch.randn(520, 1024, generator=torch.Generator().manual_seed(1)).to("cuda", torch.bfloat16)
    return host, t


def _sequence(t, prep):
    """Forward and backward calls of every kernel family on the tensors in t -> their outputs."""
    out = {}
    y, r = gn.rmsnorm_fwd(t["rx"], t["rw"], 1e-6, gemma=True, epilogue="silu")
    dx, dw = gn.rmsnorm_bwd(t["rx"], t["rw"], r, t["rdy"], gemma=True, epilogue="silu")
    out.update(ry=y, rr=r, rdx=dx, rdw=dw)
    y, mu, rs = gn.layernorm_fwd(t["lx"], t["lw"], t["lb"], 1e-5, epilogue="gelu_tanh")
    dx, dw, db = gn.layernorm_bwd(t["lx"], t["lw"], t["lb"], mu, rs, t["ldy"], epilogue="gelu_tanh")
    out.update(ly=y, lmu=mu, lrs=rs, ldx=dx, ldw=dw, ldb=db)
    q, k = t["oq"].clone(), t["ok"].clone()  # RoPE is in place: rotate fresh copies every replay
    gn.rope_apply_(q, k, t["ocos"], t["osin"], sign=+1)
    out.update(oq=q, ok=k)
    qo, ko, rq, rk = gn.qknorm_rope_fwd(t["qq"], t["qk"], t["qwq"], t["qwk"], t["qcos"], t["qsin"], 1e-6)
    dq, dk, dwq, dwk = gn.qknorm_rope_bwd(t["qq"], t["qk"], t["qwq"], t["qwk"], t["qcos"], t["qsin"], rq, rk,
                                          t["qdq"], t["qdk"])
    out.update(qqo=qo, qko=ko, qrq=rq, qrk=rk, qdq=dq, qdk=dk, qdwq=dwq, qdwk=dwk)
    Wf, c, d, Wp, dp = prep
    y, mu, rs = gn.norm_linear_fwd(t["nx"], Wf, c, d, eps=1e-5, norm="ln", epilogue="silu")
    out.update(ny=y, nmu=mu, nrs=rs)
    # the TiledLinear gradient products on the linear layer with input x (no norm)
    dz = gn.linear_act_grad(t["nx"], Wp, dp, t["ndy"], epilogue="silu")
    dxl = gn.linear_bf16(dz, Wp, b_mn=True)
    dW = torch.zeros(Wp.shape, dtype=torch.float32, device="cuda")
    gn.linear_acc_f32(dz, t["nx"], dW, a_mn=True, b_mn=True)
    dbl = gn.colsum_bf16(dz, torch.empty(Wp.shape[0], dtype=torch.float32, device="cuda"))
    out.update(ndz=dz, ndx=dxl, ndW=dW, ndb=dbl)
    return out


def test_captured_sequence_replays_bit_for_bit():
    host, t = _inputs()
    Wf, c, d = gn.norm_linear_prepare(t["nW"], t["ng"], t["nbeta"], t["nbias"], norm="ln")
    Wp, _, dp = gn.norm_linear_prepare(t["nW"], None, None, t["nbias"], norm="none")
    prep = (Wf, c, d, Wp, dp)
    eager = _sequence(t, prep)  # also the warm-up: every kernel's module is loaded before capture
    torch.cuda.synchronize()
    n0 = gn.gn_launch_count()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        static = _sequence(t, prep)
    captured = gn.gn_launch_count() - n0
    assert captured > 0
    for _ in range(3):
        g.replay()
        torch.cuda.synchronize()
        assert gn.gn_launch_count() - n0 == captured  # a replay launches from the graph, not the host
        for k, v in eager.items():
            assert torch.equal(static[k], v), k
    # and the replayed outputs are right, not only repeatable
    r, ln, o, q = host["r"], host["ln"], host["o"], host["q"]
    ry, _ = oracle.rmsnorm_fwd(r["x"], r["w"], 1e-6, gemma=True, act="silu")
    rdx, _ = oracle.rmsnorm_bwd(r["x"], r["w"], r["dy"], 1e-6, gemma=True, act="silu")
    assert_close(to_np(static["ry"]), ry, io_tol("bf16"), "rms y")
    assert_close(to_np(static["rdx"]), rdx, grad_tol("bf16"), "rms dx")
    ly, _, _ = oracle.layernorm_fwd(ln["x"], ln["w"], ln["b"], 1e-5, act="gelu_tanh")
    ldx, _, _ = oracle.layernorm_bwd(ln["x"], ln["w"], ln["b"], ln["dy"], 1e-5, act="gelu_tanh")
    assert_close(to_np(static["ly"]), ly, io_tol("bf16"), "ln y")
    assert_close(to_np(static["ldx"]), ldx, grad_tol("bf16"), "ln dx")
    oq = oracle.rope(o["q"], o["cos"], o["sin"], sign=+1)
    assert_close(to_np(static["oq"]), oq, io_tol("bf16"), "rope q")
    qo, _ = oracle.qknorm_rope_fwd(q["q"], q["wq"], q["cos"], q["sin"], 1e-6)
    assert_close(to_np(static["qqo"]), qo, io_tol("bf16"), "qk q")
    assert gn.device_error(clear=True) == 0
