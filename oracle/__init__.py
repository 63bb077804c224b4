"""fp64 CPU oracle for the row-normalization and rotary-embedding path (numpy front end).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline / reference arm may import this package. The CUDA library and its Python binding
never do, and the oracle imports nothing from them.

The arithmetic lives in ``gn_oracle.c`` (plain C, double precision, one loop over rows per
operation); this module only marshals numpy arrays. Input arrays may be ``float64``,
``float32`` or ``uint16`` (raw bfloat16 bit patterns). Outputs are ``float64``.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

F64, F32, BF16 = 0, 1, 2
ACT_NONE, ACT_GELU_TANH, ACT_SILU = 0, 1, 2
NORM_RMS, NORM_LN, NORM_NONE = 0, 1, 2
_ACTS = {"none": ACT_NONE, "gelu_tanh": ACT_GELU_TANH, "silu": ACT_SILU}

_lib = None


def _load():
    global _lib
    if _lib is None:
        # GN_ORACLE_LIB lets the mutation test load a deliberately broken copy of the oracle
        lib = C.CDLL(os.environ.get("GN_ORACLE_LIB") or _build.build())
        vp, i64, dbl, ci = C.c_void_p, C.c_int64, C.c_double, C.c_int
        lib.oracle_act.argtypes = [ci, dbl]
        lib.oracle_act.restype = dbl
        lib.oracle_act_grad.argtypes = [ci, dbl]
        lib.oracle_act_grad.restype = dbl
        lib.oracle_rmsnorm_fwd.argtypes = [vp, ci, vp, ci, i64, i64, dbl, ci, ci, vp, vp]
        lib.oracle_rmsnorm_bwd.argtypes = [vp, ci, vp, ci, vp, ci, i64, i64, dbl, ci, ci, vp, vp]
        lib.oracle_layernorm_fwd.argtypes = [vp, ci, vp, vp, ci, i64, i64, dbl, ci, vp, vp, vp]
        lib.oracle_layernorm_bwd.argtypes = [vp, ci, vp, vp, ci, vp, ci, i64, i64, dbl, ci, vp, vp, vp]
        lib.oracle_rope.argtypes = [vp, ci, vp, vp, ci, i64, i64, i64, i64, ci, vp]
        lib.oracle_qknorm_rope_fwd.argtypes = [vp, ci, vp, ci, vp, vp, ci, i64, i64, i64, i64, dbl, ci, vp, vp]
        lib.oracle_qknorm_rope_bwd.argtypes = [vp, ci, vp, ci, vp, vp, ci, vp, ci, i64, i64, i64, i64, dbl, ci, vp, vp]
        lib.oracle_norm_linear.argtypes = [vp, ci, vp, vp, ci, vp, ci, vp, ci, i64, i64, i64, dbl, ci, ci, ci,
                                           vp, vp, vp]
        lib.oracle_linear_act_bwd.argtypes = [vp, ci, vp, ci, vp, ci, vp, ci, i64, i64, i64, ci, vp, vp, vp]
        for f in ("oracle_rmsnorm_fwd", "oracle_rmsnorm_bwd", "oracle_layernorm_fwd",
                  "oracle_layernorm_bwd", "oracle_rope", "oracle_qknorm_rope_fwd",
                  "oracle_qknorm_rope_bwd", "oracle_norm_linear", "oracle_linear_act_bwd"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def _in(a):
    """(contiguous array, element-type code) for an input array."""
    if a is None:
        return None, F64
    a = np.ascontiguousarray(a)
    if a.dtype == np.float64:
        return a, F64
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.uint16:
        return a, BF16
    raise TypeError(f"oracle input dtype {a.dtype} (want float64, float32 or uint16 bf16 bits)")


def _p(a):
    return None if a is None else a.ctypes.data


def _act(act):
    return _ACTS[act] if isinstance(act, str) else int(act)


def act(kind, z: float) -> float:
    return _load().oracle_act(_act(kind), float(z))


def act_grad(kind, z: float) -> float:
    return _load().oracle_act_grad(_act(kind), float(z))


def rmsnorm_fwd(x, w, eps, gemma=False, act="none"):
    """y[M,N], inv_rms[M] for x[M,N], w[N]."""
    x, xd = _in(x)
    w, wd = _in(w)
    M, N = x.shape
    y = np.empty((M, N))
    r = np.empty(M)
    _load().oracle_rmsnorm_fwd(_p(x), xd, _p(w), wd, M, N, eps, int(gemma), _act(act), _p(y), _p(r))
    return y, r


def rmsnorm_bwd(x, w, dy, eps, gemma=False, act="none", want_dx=True):
    """dx[M,N] (None unless want_dx), dw[N]."""
    x, xd = _in(x)
    w, wd = _in(w)
    dy, gd = _in(dy)
    M, N = x.shape
    dx = np.empty((M, N)) if want_dx else None
    dw = np.empty(N)
    _load().oracle_rmsnorm_bwd(_p(x), xd, _p(w), wd, _p(dy), gd, M, N, eps, int(gemma), _act(act),
                               _p(dx), _p(dw))
    return dx, dw


def layernorm_fwd(x, w, b, eps, act="none"):
    """y[M,N], mean[M], rstd[M]; w or b may be None (1 and 0)."""
    x, xd = _in(x)
    w, wd = _in(w)
    b, bd = _in(b)
    if w is not None and b is not None and wd != bd:
        raise TypeError("w and b must share a dtype")
    M, N = x.shape
    y = np.empty((M, N))
    mu = np.empty(M)
    rs = np.empty(M)
    _load().oracle_layernorm_fwd(_p(x), xd, _p(w), _p(b), wd if w is not None else bd, M, N, eps,
                                 _act(act), _p(y), _p(mu), _p(rs))
    return y, mu, rs


def layernorm_bwd(x, w, b, dy, eps, act="none", want_dx=True):
    """dx[M,N] (None unless want_dx), dw[N], db[N]."""
    x, xd = _in(x)
    w, wd = _in(w)
    b, bd = _in(b)
    dy, gd = _in(dy)
    M, N = x.shape
    dx = np.empty((M, N)) if want_dx else None
    dw = np.empty(N)
    db = np.empty(N)
    _load().oracle_layernorm_bwd(_p(x), xd, _p(w), _p(b), wd if w is not None else bd, _p(dy), gd,
                                 M, N, eps, _act(act), _p(dx), _p(dw), _p(db))
    return dx, dw, db


def _tables(cos, sin):
    cos, cd = _in(cos)
    sin, sd = _in(sin)
    if cd != sd:
        raise TypeError("cos and sin must share a dtype")
    return cos, sin, cd


def rope(x, cos, sin, sign=+1):
    """Rotary embedding of x[B,S,H,D] with tables [S, D/2]; returns a new float64 array."""
    x, xd = _in(x)
    cos, sin, td = _tables(cos, sin)
    B, S, H, D = x.shape
    assert cos.shape == (S, D // 2) and sin.shape == (S, D // 2)
    out = np.empty(x.shape)
    _load().oracle_rope(_p(x), xd, _p(cos), _p(sin), td, B, S, H, D, int(sign), _p(out))
    return out


def qknorm_rope_fwd(x, w, cos, sin, eps, gemma=False, want_out=True):
    """out[B,S,H,D] (None unless want_out), inv_rms[B,S,H]: per-head RMSNorm then the forward
    rotary embedding."""
    x, xd = _in(x)
    w, wd = _in(w)
    cos, sin, td = _tables(cos, sin)
    B, S, H, D = x.shape
    out = np.empty(x.shape) if want_out else None
    r = np.empty((B, S, H))
    _load().oracle_qknorm_rope_fwd(_p(x), xd, _p(w), wd, _p(cos), _p(sin), td, B, S, H, D, eps,
                                   int(gemma), _p(out), _p(r))
    return out, r


def qknorm_rope_bwd(x, w, cos, sin, dy, eps, gemma=False, want_dx=True):
    """dx[B,S,H,D] (None unless want_dx), dw[D]."""
    x, xd = _in(x)
    w, wd = _in(w)
    cos, sin, td = _tables(cos, sin)
    dy, gd = _in(dy)
    B, S, H, D = x.shape
    dx = np.empty(x.shape) if want_dx else None
    dw = np.empty(D)
    _load().oracle_qknorm_rope_bwd(_p(x), xd, _p(w), wd, _p(cos), _p(sin), td, _p(dy), gd, B, S, H,
                                   D, eps, int(gemma), _p(dx), _p(dw))
    return dx, dw


def norm_linear(x, g, beta, W, bias, eps, norm="ln", gemma=False, act="none"):
    """y[M,N] = act(norm(x) W^T + bias), mean[M], rstd[M] for x[M,K], W[N,K]: the normalized
    row (LayerNorm with weight g and bias beta, or RMSNorm with weight g), then the linear layer.
    beta (RMSNorm: ignored) and bias may be None."""
    x, xd = _in(x)
    g, gd = _in(g)
    beta, bd = _in(beta)
    W, wd = _in(W)
    bias, bsd = _in(bias)
    if norm == "ln" and beta is not None and gd != bd:
        raise TypeError("g and beta must share a dtype")
    M, K = x.shape
    N = W.shape[0]
    assert W.shape == (N, K)
    y = np.empty((M, N))
    mu = np.empty(M)
    rs = np.empty(M)
    code = {"ln": NORM_LN, "rms": NORM_RMS, "none": NORM_NONE}[norm]
    _load().oracle_norm_linear(_p(x), xd, _p(g), _p(beta if norm == "ln" else None), gd, _p(W), wd, _p(bias), bsd,
                               M, N, K, eps, code, int(gemma), _act(act), _p(y), _p(mu), _p(rs))
    return y, mu, rs


def norm_linear_bwd(x, g, beta, W, bias, dy, eps, norm="ln", gemma=False, act="none"):
    """Gradients of sum(dy * act(norm(x) W^T + bias)) for the layer that normalizes the rows of x
    and feeds them to the linear layer (Janus-Pro inference page, section 4.1; HY-Motion page,
    section 3.1): -> dx [M,K], dg [K], dbeta [K] (LayerNorm; None for RMSNorm), dW [N,K],
    dbias [N]. By the chain rule: the normalized rows xn = norm(x) in fp64, the linear layer's
    gradients at xn (dxn, dW, dbias), then the normalization's backward with dxn as the gradient of
    its output. RMSNorm needs its weight g."""
    if norm == "ln":
        xn, _, _ = layernorm_fwd(x, g, beta, eps)
        dxn, dW, db = linear_act_bwd(xn, W, bias, dy, act)
        dx, dg, dbeta = layernorm_bwd(x, g, beta, dxn, eps)
        return dx, dg, dbeta, dW, db
    if norm != "rms":
        raise ValueError(f"norm {norm!r}")
    if g is None:
        raise ValueError("RMSNorm needs its weight g")
    xn, _ = rmsnorm_fwd(x, g, eps, gemma=gemma)
    dxn, dW, db = linear_act_bwd(xn, W, bias, dy, act)
    dx, dg = rmsnorm_bwd(x, g, dxn, eps, gemma=gemma)
    return dx, dg, None, dW, db


def linear_act_bwd(x, W, bias, dy, act="none"):
    """Gradients of sum(dy * act(x W^T + bias)): dx[M,K], dW[N,K], dbias[N]."""
    x, xd = _in(x)
    W, wd = _in(W)
    bias, bd = _in(bias)
    dy, gd = _in(dy)
    M, K = x.shape
    N = W.shape[0]
    dx, dW, db = np.empty((M, K)), np.empty((N, K)), np.empty(N)
    _load().oracle_linear_act_bwd(_p(x), xd, _p(W), wd, _p(bias), bd, _p(dy), gd, M, N, K, _act(act), _p(dx),
                                  _p(dW), _p(db))
    return dx, dW, db
