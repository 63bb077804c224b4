"""Python binding of libgn: fused row normalization and interleaved RoPE on B200 (sm_100a).

Two layers, both argument marshalling only (every step of the computation runs in the CUDA
kernels of ``libgn.so``):

* ``gn_*`` functions with the names and argument lists of the C ABI in ``include/gn.h``
  (pointers as Python ints, ``stream`` as an int handle). They return the ``gn_status`` code.
* torch-tensor helpers (``rmsnorm_fwd``, ``rope_apply_``, ...) that allocate outputs with
  torch, pass ``data_ptr()`` values and the current CUDA stream, and raise ``GnError`` on a
  non-zero status.

There is no fallback: if ``libgn.so`` is missing or cannot be loaded, every call raises.
Build it with ``python -m transformer_norm_rope_b200._build``.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgn.so")

GN_OK, GN_ERR_NULL, GN_ERR_SHAPE, GN_ERR_ALIGN, GN_ERR_DTYPE, GN_ERR_WORKSPACE, \
    GN_ERR_UNSUPPORTED, GN_ERR_CUDA = range(8)
GN_F32, GN_BF16 = 0, 1
GN_EPI_NONE, GN_EPI_GELU_TANH, GN_EPI_SILU = 0, 1, 2
GN_NORM_RMS, GN_NORM_LN, GN_NORM_NONE = 0, 1, 2
GN_DEVERR_WAIT_TIMEOUT = 1
EPILOGUES = {"none": GN_EPI_NONE, "gelu_tanh": GN_EPI_GELU_TANH, "silu": GN_EPI_SILU}

_vp, _i64, _f32, _int, _sz = C.c_void_p, C.c_int64, C.c_float, C.c_int, C.c_size_t
_st = C.c_int

# name -> (restype, argtypes), in the order of include/gn.h
SIGNATURES = {
    "gn_status_string": (C.c_char_p, [_st]),
    "gn_rmsnorm_fwd": (_st, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _f32, _int, _int, _int, _vp]),
    "gn_rmsnorm_bwd_workspace": (_sz, [_i64, _i64, _int]),
    "gn_rmsnorm_bwd": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _i64, _i64, _i64, _i64, _i64,
                             _int, _int, _int, _vp]),
    "gn_layernorm_fwd": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _f32, _int, _int,
                               _vp]),
    "gn_layernorm_bwd_workspace": (_sz, [_i64, _i64, _int]),
    "gn_layernorm_bwd": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _i64, _i64, _i64,
                               _i64, _i64, _int, _int, _vp]),
    "gn_rope_apply_inplace": (_st, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _int, _int, _vp]),
    "gn_qknorm_rope_fwd": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                 _i64, _f32, _int, _int, _vp]),
    "gn_qknorm_rope_bwd_workspace": (_sz, [_i64, _i64, _i64, _i64, _int]),
    "gn_qknorm_rope_bwd": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                 _vp, _sz, _i64, _i64, _i64, _i64, _int, _int, _vp]),
    "gn_qknorm_rope_bwd_noalloc": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                         _i64, _i64, _i64, _i64, _int, _int, _vp]),
    "gn_norm_linear_prepare": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _int, _int, _int, _vp]),
    "gn_norm_linear_fwd": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _f32, _int,
                                 _int, _int, _vp]),
    "gn_linear_act_grad": (_st, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _int, _int, _vp]),
    "gn_linear_bf16": (_st, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _int, _int, _int, _vp]),
    "gn_linear_acc_f32": (_st, [_vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _int, _int, _int, _vp]),
    "gn_colsum_bf16_workspace": (_sz, [_i64]),
    "gn_colsum_bf16": (_st, [_vp, _vp, _vp, _sz, _i64, _i64, _i64, _int, _int, _vp]),
    "gn_act_grad": (_st, [_vp, _vp, _vp, _i64, _int, _int, _vp]),
    "gn_act_fwd": (_st, [_vp, _vp, _i64, _int, _int, _vp]),
    "gn_launch_count": (C.c_uint64, []),
    "gn_device_error": (_st, [C.POINTER(C.c_uint), _int]),
    "gn_selftest_wait_timeout": (_st, [C.c_uint32, _vp]),
    "gn_tune": (_st, [C.c_char_p, _int]),
}

_lib = None


class GnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def load():
    """Load libgn.so (once). Raises if it is missing: there is no fallback path."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m transformer_norm_rope_b200._build`")
        lib = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def _c(name):
    def call(*args):
        return getattr(load(), name)(*args)

    call.__name__ = name
    call.__doc__ = f"Direct call of the C entry point {name} (see include/gn.h)."
    return call


for _name in SIGNATURES:
    globals()[_name] = _c(_name)
del _name


def status_string(status: int) -> str:
    try:
        return load().gn_status_string(status).decode()
    except Exception:  # noqa: BLE001 - message helper must not mask the original error
        return f"gn_status {status}"


def check(status: int, where: str = "libgn") -> None:
    if status != GN_OK:
        raise GnError(status, where)


# ---------------------------------------------------------------- torch helpers

def _torch():
    import torch

    return torch


def _dt(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return GN_BF16
    if t.dtype == torch.float32:
        return GN_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bfloat16 or float32)")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    torch = _torch()
    return (stream or torch.cuda.current_stream()).cuda_stream


def _epi(epi) -> int:
    return EPILOGUES[epi] if isinstance(epi, str) else int(epi)


def _on_gpu(t) -> bool:
    return t.is_cuda


def _need(t, name, *, like=None, shape=None, numel=None, dtype=None, contiguous=True, optional=False):
    """Validate a tensor argument before its pointer reaches the library, which sees raw
    pointers only: a wrong size, dtype or layout there would read or write out of bounds.
    Checks (in this order) presence, shape or element count, dtype, contiguity, and that it
    lives on the device of `like` (always a CUDA device)."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not _on_gpu(t):
        raise ValueError(f"{name} must be a CUDA tensor (the library runs on the GPU only)")
    if like is not None and t.device != like.device:
        raise ValueError(f"{name} is on {t.device}, the other operands on {like.device}")


def _rows(x, name="x", like=None, dtype=None):
    """(rows, hidden, ld) of a CUDA tensor whose last dim is contiguous and whose leading dims
    collapse to one row stride."""
    _need(x, name, like=like, dtype=dtype, contiguous=False)
    if x.dim() < 1 or x.stride(-1) != 1:
        raise ValueError(f"last dimension of {name} must be contiguous")
    hidden = x.shape[-1]
    x2 = x.reshape(-1, hidden) if x.dim() != 2 else x
    if x2.data_ptr() != x.data_ptr():
        raise ValueError("rows of x must form one strided matrix")
    ld = x2.stride(0) if x2.shape[0] > 1 else hidden
    return x2.shape[0], hidden, ld


def empty_rows(shape, dtype, device):
    """Uninitialised tensor of `shape` whose rows start on 16-byte boundaries: the row stride
    is the last dimension rounded up to 16 bytes (a strided view when that adds padding)."""
    torch = _torch()
    shape = tuple(shape)
    hidden = shape[-1]
    es = torch.empty((), dtype=dtype).element_size()
    ld = (hidden * es + 15) // 16 * 16 // es
    rows = 1
    for n in shape[:-1]:
        rows *= n
    strides, acc = [1], ld
    for n in reversed(shape[:-1]):
        strides.insert(0, acc)
        acc *= n
    base = torch.empty(rows * ld, dtype=dtype, device=device)
    return base.as_strided(shape, strides)


def rmsnorm_fwd(x, w, eps=1e-6, gemma=False, epilogue="none", out=None, save_stats=True, stream=None):
    """y = epi(x * rsqrt(mean(x^2) + eps) * w') -> (y, inv_rms[rows] fp32 or None)."""
    torch = _torch()
    rows, hidden, ld = _rows(x)
    _need(w, "w", like=x, shape=(hidden,), dtype=x.dtype)
    y = empty_rows(x.shape, x.dtype, x.device) if out is None else out
    _need(y, "out", like=x, shape=x.shape, contiguous=False)
    _, _, ldy = _rows(y, "out", like=x, dtype=x.dtype)
    r = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device) if save_stats else None
    check(gn_rmsnorm_fwd(_ptr(x), _ptr(w), _ptr(y), _ptr(r), rows, hidden, ld, ldy, eps, int(gemma),
                         _epi(epilogue), _dt(x), _stream(stream)), "gn_rmsnorm_fwd")
    return y, r


def rmsnorm_bwd(x, w, inv_rms, dy, gemma=False, epilogue="none", want_dw=True, stream=None):
    """-> (dx, dw fp32 or None)."""
    torch = _torch()
    rows, hidden, ld = _rows(x)
    _need(w, "w", like=x, shape=(hidden,), dtype=x.dtype)
    _need(inv_rms, "inv_rms", like=x, numel=rows, dtype=torch.float32)
    _need(dy, "dy", like=x, shape=x.shape, contiguous=False)
    _, _, lddy = _rows(dy, "dy", like=x, dtype=x.dtype)
    dx = empty_rows(x.shape, x.dtype, x.device)
    _, _, lddx = _rows(dx)
    dw = torch.empty(hidden, dtype=torch.float32, device=x.device) if want_dw else None
    nws = gn_rmsnorm_bwd_workspace(rows, hidden, _dt(x)) if want_dw else 0
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=x.device) if want_dw else None
    check(gn_rmsnorm_bwd(_ptr(x), _ptr(w), _ptr(inv_rms), _ptr(dy), _ptr(dx), _ptr(dw), _ptr(ws), nws,
                         rows, hidden, ld, lddy, lddx, int(gemma), _epi(epilogue), _dt(x),
                         _stream(stream)), "gn_rmsnorm_bwd")
    return dx, dw


def layernorm_fwd(x, w=None, b=None, eps=1e-5, epilogue="none", out=None, save_stats=True, stream=None):
    """y = epi((x - mean) * rstd * w + b) -> (y, mean, rstd)."""
    torch = _torch()
    rows, hidden, ld = _rows(x)
    _need(w, "w", like=x, shape=(hidden,), dtype=x.dtype, optional=True)
    _need(b, "b", like=x, shape=(hidden,), dtype=x.dtype, optional=True)
    y = empty_rows(x.shape, x.dtype, x.device) if out is None else out
    _need(y, "out", like=x, shape=x.shape, contiguous=False)
    _, _, ldy = _rows(y, "out", like=x, dtype=x.dtype)
    mk = (lambda: torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device))
    mu, rs = (mk(), mk()) if save_stats else (None, None)
    check(gn_layernorm_fwd(_ptr(x), _ptr(w), _ptr(b), _ptr(y), _ptr(mu), _ptr(rs), rows, hidden, ld, ldy,
                           eps, _epi(epilogue), _dt(x), _stream(stream)), "gn_layernorm_fwd")
    return y, mu, rs


def layernorm_bwd(x, w, b, mean, rstd, dy, epilogue="none", want_wgrad=True, stream=None):
    """-> (dx, dw, db) (dw, db fp32 or None)."""
    torch = _torch()
    rows, hidden, ld = _rows(x)
    _need(w, "w", like=x, shape=(hidden,), dtype=x.dtype, optional=True)
    _need(b, "b", like=x, shape=(hidden,), dtype=x.dtype, optional=True)
    _need(mean, "mean", like=x, numel=rows, dtype=torch.float32)
    _need(rstd, "rstd", like=x, numel=rows, dtype=torch.float32)
    _need(dy, "dy", like=x, shape=x.shape, contiguous=False)
    _, _, lddy = _rows(dy, "dy", like=x, dtype=x.dtype)
    dx = empty_rows(x.shape, x.dtype, x.device)
    _, _, lddx = _rows(dx)
    mk = (lambda: torch.empty(hidden, dtype=torch.float32, device=x.device))
    dw, db = (mk(), mk()) if want_wgrad else (None, None)
    nws = gn_layernorm_bwd_workspace(rows, hidden, _dt(x)) if want_wgrad else 0
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=x.device) if want_wgrad else None
    check(gn_layernorm_bwd(_ptr(x), _ptr(w), _ptr(b), _ptr(mean), _ptr(rstd), _ptr(dy), _ptr(dx), _ptr(dw),
                           _ptr(db), _ptr(ws), nws, rows, hidden, ld, lddy, lddx, _epi(epilogue), _dt(x),
                           _stream(stream)), "gn_layernorm_bwd")
    return dx, dw, db


def _bshd(q):
    _need(q, "q")
    if q.dim() != 4:
        raise ValueError("rotary tensors must be contiguous [B, S, H, D]")
    return q.shape


def _tables(q, cos, sin):
    torch = _torch()
    _, S, _, D = q.shape
    _need(cos, "cos", like=q, shape=(S, D // 2), dtype=torch.float32)
    _need(sin, "sin", like=q, shape=(S, D // 2), dtype=torch.float32)


def rope_apply_(q, k, cos, sin, sign=+1, stream=None):
    """In-place interleaved RoPE of q (and k, may be None); sign=-1 is the backward."""
    B, S, H, D = _bshd(q)
    _need(k, "k", like=q, shape=q.shape, dtype=q.dtype, optional=True)
    _tables(q, cos, sin)
    check(gn_rope_apply_inplace(_ptr(q), _ptr(k), _ptr(cos), _ptr(sin), B, S, H, D, int(sign), _dt(q),
                                _stream(stream)), "gn_rope_apply_inplace")
    return q, k


def qknorm_rope_fwd(q, k, wq, wk, cos, sin, eps=1e-6, gemma=False, stream=None):
    """-> (q_out, k_out, inv_rms_q, inv_rms_k); k may be None."""
    torch = _torch()
    B, S, H, D = _bshd(q)
    _need(k, "k", like=q, shape=q.shape, dtype=q.dtype, optional=True)
    _need(wq, "wq", like=q, shape=(D,), dtype=q.dtype)
    _need(wk, "wk", like=q, shape=(D,), dtype=q.dtype, optional=k is None)
    _tables(q, cos, sin)
    qo = torch.empty_like(q)
    ko = torch.empty_like(k) if k is not None else None
    rq = torch.empty((B, S, H), dtype=torch.float32, device=q.device)
    rk = torch.empty((B, S, H), dtype=torch.float32, device=q.device) if k is not None else None
    check(gn_qknorm_rope_fwd(_ptr(q), _ptr(k), _ptr(wq), _ptr(wk), _ptr(cos), _ptr(sin), _ptr(qo), _ptr(ko),
                             _ptr(rq), _ptr(rk), B, S, H, D, eps, int(gemma), _dt(q), _stream(stream)),
          "gn_qknorm_rope_fwd")
    return qo, ko, rq, rk


def qknorm_rope_bwd(q, k, wq, wk, cos, sin, inv_rms_q, inv_rms_k, dq_out, dk_out, gemma=False,
                    want_dw=True, stream=None):
    """-> (dq, dk, dwq, dwk)."""
    torch = _torch()
    B, S, H, D = _bshd(q)
    _need(k, "k", like=q, shape=q.shape, dtype=q.dtype, optional=True)
    _need(wq, "wq", like=q, shape=(D,), dtype=q.dtype)
    _need(wk, "wk", like=q, shape=(D,), dtype=q.dtype, optional=k is None)
    _tables(q, cos, sin)
    _need(inv_rms_q, "inv_rms_q", like=q, numel=B * S * H, dtype=torch.float32)
    _need(dq_out, "dq_out", like=q, shape=q.shape, dtype=q.dtype)
    if k is not None:
        _need(inv_rms_k, "inv_rms_k", like=q, numel=B * S * H, dtype=torch.float32)
        _need(dk_out, "dk_out", like=q, shape=q.shape, dtype=q.dtype)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k) if k is not None else None
    dwq = torch.empty(D, dtype=torch.float32, device=q.device) if want_dw else None
    dwk = torch.empty(D, dtype=torch.float32, device=q.device) if (want_dw and k is not None) else None
    nws = gn_qknorm_rope_bwd_workspace(B, S, H, D, _dt(q)) if want_dw else 0
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=q.device) if want_dw else None
    check(gn_qknorm_rope_bwd(_ptr(q), _ptr(k), _ptr(wq), _ptr(wk), _ptr(cos), _ptr(sin), _ptr(inv_rms_q),
                             _ptr(inv_rms_k), _ptr(dq_out), _ptr(dk_out), _ptr(dq), _ptr(dk), _ptr(dwq),
                             _ptr(dwk), _ptr(ws), nws, B, S, H, D, int(gemma), _dt(q), _stream(stream)),
          "gn_qknorm_rope_bwd")
    return dq, dk, dwq, dwk


def _norm(norm) -> int:
    return {"rms": GN_NORM_RMS, "ln": GN_NORM_LN, "none": GN_NORM_NONE}[norm] if isinstance(norm, str) else int(norm)


def norm_linear_prepare(W, g=None, beta=None, bias=None, norm="ln", gemma=False, stream=None):
    """Fold the norm weight into the layer weight W [N, K] (bf16): -> (Wf [N, K] bf16, c [N] fp32
    or None, d [N] fp32)."""
    torch = _torch()
    _need(W, "W")
    if W.dim() != 2:
        raise ValueError("W must be [N, K]")
    N, K = W.shape
    _need(g, "g", like=W, shape=(K,), dtype=W.dtype, optional=True)
    _need(beta, "beta", like=W, shape=(K,), dtype=W.dtype, optional=True)
    _need(bias, "bias", like=W, shape=(N,), dtype=W.dtype, optional=True)
    Wf = torch.empty_like(W)
    c = torch.empty(N, dtype=torch.float32, device=W.device) if _norm(norm) == GN_NORM_LN else None
    d = torch.empty(N, dtype=torch.float32, device=W.device)
    check(gn_norm_linear_prepare(_ptr(W), _ptr(g), _ptr(beta), _ptr(bias), _ptr(Wf), _ptr(c), _ptr(d), N, K,
                                 _norm(norm), int(gemma), _dt(W), _stream(stream)), "gn_norm_linear_prepare")
    return Wf, c, d


def norm_linear_fwd(x, Wf, c, d, eps=1e-5, norm="ln", epilogue="none", save_stats=True, out=None, stream=None):
    """y [M, N] = act(norm(x) W^T + bias) from x [M, K] and the prepared (Wf, c, d):
    -> (y, mean, rstd) (statistics fp32 [M], or None). `out` may give y (rows of a larger
    tensor included: its row stride is passed on)."""
    torch = _torch()
    if x.dim() != 2:
        raise ValueError("x must be [M, K]")
    M, K = x.shape
    _rows(x)
    _need(Wf, "Wf", like=x, dtype=x.dtype)
    if Wf.dim() != 2 or Wf.shape[1] != K:
        raise ValueError(f"Wf has shape {tuple(Wf.shape)}, expected [N, {K}]")
    N = Wf.shape[0]
    _need(c, "c", like=x, shape=(N,), dtype=torch.float32, optional=_norm(norm) != GN_NORM_LN)
    _need(d, "d", like=x, shape=(N,), dtype=torch.float32, optional=True)
    y = torch.empty((M, N), dtype=x.dtype, device=x.device) if out is None else out
    _need(y, "out", like=x, shape=(M, N), contiguous=False)
    _rows(y, "out", like=x, dtype=x.dtype)
    plain = _norm(norm) == GN_NORM_NONE
    mu = None if plain else torch.empty(M, dtype=torch.float32, device=x.device)  # the kernels need both
    rs = None if plain else torch.empty(M, dtype=torch.float32, device=x.device)
    check(gn_norm_linear_fwd(_ptr(x), _ptr(Wf), _ptr(c), _ptr(d), _ptr(y), _ptr(mu), _ptr(rs), M, N, K,
                             x.stride(0), y.stride(0), eps, _norm(norm), _epi(epilogue), _dt(x),
                             _stream(stream)), "gn_norm_linear_fwd")
    return (y, mu, rs) if save_stats else (y, None, None)


def act_grad(z, dy, epilogue="silu", out=None, stream=None):
    """dz = dy * act'(z), elementwise (contiguous tensors of one dtype)."""
    _need(dy, "dy")
    _need(z, "z", like=dy, shape=dy.shape, dtype=dy.dtype)
    dz = torch_empty_like(dy) if out is None else out
    _need(dz, "out", like=dy, shape=dy.shape, dtype=dy.dtype)
    check(gn_act_grad(_ptr(z), _ptr(dy), _ptr(dz), dy.numel(), _epi(epilogue), _dt(dy), _stream(stream)),
          "gn_act_grad")
    return dz


def act_fwd(z, epilogue="silu", out=None, stream=None):
    """y = act(z), elementwise (contiguous; out may be z itself)."""
    _need(z, "z")
    y = torch_empty_like(z) if out is None else out
    _need(y, "out", like=z, shape=z.shape, dtype=z.dtype)
    check(gn_act_fwd(_ptr(z), _ptr(y), z.numel(), _epi(epilogue), _dt(z), _stream(stream)), "gn_act_fwd")
    return y


def linear_act_grad(x, Wf, d, dy, epilogue="silu", out=None, stream=None):
    """dz = dy * act'(x Wf^T + d) [M, N] (bf16) on the tensor-core kernels (z never stored)."""
    _rows(x)
    M, K = x.shape
    _need(Wf, "Wf", like=x, dtype=x.dtype)
    if Wf.dim() != 2 or Wf.shape[1] != K:
        raise ValueError(f"Wf has shape {tuple(Wf.shape)}, expected [N, {K}]")
    N = Wf.shape[0]
    _need(d, "d", like=x, shape=(N,), dtype=_torch().float32, optional=True)
    _need(dy, "dy", like=x, shape=(M, N), dtype=x.dtype, contiguous=False)
    _rows(dy, "dy", like=x, dtype=x.dtype)
    dz = _torch().empty((M, N), dtype=x.dtype, device=x.device) if out is None else out
    _need(dz, "out", like=x, shape=(M, N), dtype=x.dtype, contiguous=False)
    _rows(dz, "out", like=x, dtype=x.dtype)
    check(gn_linear_act_grad(_ptr(x), _ptr(Wf), _ptr(d), _ptr(dy), _ptr(dz), M, N, K, x.stride(0), dy.stride(0),
                             dz.stride(0), _epi(epilogue), _dt(x), _stream(stream)), "gn_linear_act_grad")
    return dz


GN_K_MAJOR, GN_MN_MAJOR = 0, 1


def _operands(A, B, a_mn, b_mn):
    """(M, N, K) of the product A B^T from the stored operands: A is [M, K], or [K, M] when a_mn
    (MN-major); B is [N, K], or [K, N] when b_mn."""
    _rows(A, "A")
    _rows(B, "B", like=A, dtype=A.dtype)
    if A.dim() != 2 or B.dim() != 2:
        raise ValueError("A and B must be 2-D")
    M, K = (A.shape[1], A.shape[0]) if a_mn else A.shape
    N, KB = (B.shape[1], B.shape[0]) if b_mn else B.shape
    if KB != K:
        raise ValueError(f"contraction sizes differ: A gives {K}, B gives {KB}")
    return M, N, K


def linear_bf16(A, B, d=None, out=None, a_mn=False, b_mn=False, stream=None):
    """y [M, N] = A B^T (+ d) in bf16 on the tensor-core kernels; a_mn / b_mn: the operand is
    stored transposed ([K, M] / [K, N])."""
    torch = _torch()
    M, N, K = _operands(A, B, a_mn, b_mn)
    _need(d, "d", like=A, shape=(N,), dtype=torch.float32, optional=True)
    y = torch.empty((M, N), dtype=A.dtype, device=A.device) if out is None else out
    _need(y, "out", like=A, shape=(M, N), dtype=A.dtype, contiguous=False)
    _rows(y, "out", like=A, dtype=A.dtype)
    check(gn_linear_bf16(_ptr(A), _ptr(B), _ptr(d), _ptr(y), M, N, K, A.stride(0), B.stride(0), y.stride(0),
                         GN_MN_MAJOR if a_mn else GN_K_MAJOR, GN_MN_MAJOR if b_mn else GN_K_MAJOR, _dt(A),
                         _stream(stream)), "gn_linear_bf16")
    return y


def linear_acc_f32(A, B, C, a_mn=False, b_mn=False, stream=None):
    """C [M, N] (fp32, in place) += A B^T (bf16) on the tensor-core kernels; a_mn / b_mn: the
    operand is stored transposed ([K, M] / [K, N])."""
    torch = _torch()
    M, N, K = _operands(A, B, a_mn, b_mn)
    _need(C, "C", like=A, shape=(M, N), dtype=torch.float32, contiguous=False)
    _rows(C, "C", like=A, dtype=torch.float32)
    check(gn_linear_acc_f32(_ptr(A), _ptr(B), _ptr(C), M, N, K, A.stride(0), B.stride(0), C.stride(0),
                            GN_MN_MAJOR if a_mn else GN_K_MAJOR, GN_MN_MAJOR if b_mn else GN_K_MAJOR, _dt(A),
                            _stream(stream)), "gn_linear_acc_f32")
    return C


def colsum_bf16(src, out, accumulate=False, ws=None, stream=None):
    """out [cols] (fp32) = (or +=) column sums of src [rows, cols] (bf16), fixed order."""
    torch = _torch()
    rows, cols, ld = _rows(src, "src")
    _need(out, "out", like=src, shape=(cols,), dtype=torch.float32)
    nws = gn_colsum_bf16_workspace(cols)
    if ws is None:
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=src.device)
    _need(ws, "ws", like=src, numel=ws.numel(), dtype=torch.uint8)
    check(gn_colsum_bf16(_ptr(src), _ptr(out), _ptr(ws), ws.numel(), rows, cols, ld, int(accumulate), _dt(src),
                         _stream(stream)), "gn_colsum_bf16")
    return out


def torch_empty_like(t):
    return _torch().empty_like(t)


def device_error(clear: bool = False) -> int:
    w = C.c_uint(0)
    check(gn_device_error(C.byref(w), int(clear)), "gn_device_error")
    return w.value


def tune(key: str, value: int) -> None:
    check(gn_tune(key.encode(), int(value)), "gn_tune")
