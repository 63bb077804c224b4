"""The C-ABI library loads, exports every symbol include/gn.h declares, and rejects bad
arguments on the host before touching the GPU (CPU only: no kernel is launched)."""
import os
import re
import subprocess

import pytest

import transformer_norm_rope_b200 as gn
from transformer_norm_rope_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gn.h")


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return gn.load()


def declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gn_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared() == sorted(gn.SIGNATURES), "binding signature table differs from include/gn.h"


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", gn.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (gn_[a-z0-9_]+)$", out, flags=re.M))
    missing = [s for s in declared() if s not in exported]
    assert not missing, missing


def test_library_is_built_for_sm100a(lib):
    # the build compiles every source for sm_100a only (no PTX for other targets, no JIT)
    assert _build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert not _build.stale(), "libgn.so is older than its sources"


def test_status_strings(lib):
    for s in range(8):
        assert gn.status_string(s).startswith("GN_")


P = 1 << 20  # a 16-byte aligned fake pointer value: validation fails before it is dereferenced


def test_rmsnorm_argument_checks(lib):
    f = gn.gn_rmsnorm_fwd
    assert f(None, P, P, None, 4, 64, 64, 64, 1e-6, 0, 0, gn.GN_BF16, None) == gn.GN_ERR_NULL
    assert f(P, None, P, None, 4, 64, 64, 64, 1e-6, 0, 0, gn.GN_BF16, None) == gn.GN_ERR_NULL
    assert f(P, P, P, None, 4, 0, 64, 64, 1e-6, 0, 0, gn.GN_BF16, None) == gn.GN_ERR_SHAPE
    assert f(P, P, P, None, -1, 64, 64, 64, 1e-6, 0, 0, gn.GN_BF16, None) == gn.GN_ERR_SHAPE
    assert f(P, P, P, None, 4, 64, 32, 64, 1e-6, 0, 0, gn.GN_BF16, None) == gn.GN_ERR_SHAPE
    assert f(P + 2, P, P, None, 4, 64, 64, 64, 1e-6, 0, 0, gn.GN_BF16, None) == gn.GN_ERR_ALIGN
    assert f(P, P, P, None, 4, 64, 68, 64, 1e-6, 0, 0, gn.GN_BF16, None) == gn.GN_ERR_ALIGN
    assert f(P, P, P, None, 4, 64, 64, 64, 1e-6, 0, 0, 5, None) == gn.GN_ERR_DTYPE
    assert f(P, P, P, None, 4, 64, 64, 64, 1e-6, 0, 9, gn.GN_BF16, None) == gn.GN_ERR_DTYPE
    # empty input: valid, nothing launched
    assert f(P, P, P, None, 0, 64, 64, 64, 1e-6, 0, 0, gn.GN_BF16, None) == gn.GN_OK
    b = gn.gn_rmsnorm_bwd
    assert b(P, P, None, P, P, P, P, 1 << 20, 4, 64, 64, 64, 64, 0, 0, gn.GN_BF16, None) == gn.GN_ERR_NULL
    assert b(P, P, P, P, P + 8, P, P, 1 << 20, 4, 64, 64, 64, 64, 0, 0, gn.GN_BF16, None) == gn.GN_ERR_ALIGN


def test_layernorm_argument_checks(lib):
    f = gn.gn_layernorm_fwd
    assert f(None, None, None, P, None, None, 4, 64, 64, 64, 1e-5, 0, gn.GN_BF16, None) == gn.GN_ERR_NULL
    assert f(P, None, None, P, None, None, 4, 64, 64, 66, 1e-5, 0, gn.GN_BF16, None) == gn.GN_ERR_ALIGN
    assert f(P, None, None, P, None, None, 0, 64, 64, 64, 1e-5, 0, gn.GN_BF16, None) == gn.GN_OK
    b = gn.gn_layernorm_bwd
    assert b(P, None, None, None, P, P, P, None, None, None, 0, 4, 64, 64, 64, 64, 0, gn.GN_BF16,
             None) == gn.GN_ERR_NULL


def test_rope_argument_checks(lib):
    f = gn.gn_rope_apply_inplace
    assert f(None, None, P, P, 1, 4, 2, 128, 1, gn.GN_BF16, None) == gn.GN_ERR_NULL
    assert f(P, None, None, P, 1, 4, 2, 128, 1, gn.GN_BF16, None) == gn.GN_ERR_NULL
    assert f(P, None, P, P, 1, 4, 2, 127, 1, gn.GN_BF16, None) == gn.GN_ERR_SHAPE
    assert f(P, None, P, P, 1, 4, 2, 12, 1, gn.GN_BF16, None) == gn.GN_ERR_SHAPE
    assert f(P, None, P, P, 1, 4, 2, 128, 0, gn.GN_BF16, None) == gn.GN_ERR_SHAPE
    assert f(P + 4, None, P, P, 1, 4, 2, 128, 1, gn.GN_BF16, None) == gn.GN_ERR_ALIGN
    assert f(P, None, P, P, 0, 4, 2, 128, 1, gn.GN_BF16, None) == gn.GN_OK


def test_qknorm_argument_checks(lib):
    f = gn.gn_qknorm_rope_fwd
    assert f(P, None, None, None, P, P, P, None, None, None, 1, 4, 2, 128, 1e-6, 0, gn.GN_BF16,
             None) == gn.GN_ERR_NULL
    # D = 96 bf16 is 12 vectors per head: not a power of two
    assert f(P, None, P, None, P, P, P, None, None, None, 1, 4, 2, 96, 1e-6, 0, gn.GN_BF16,
             None) == gn.GN_ERR_UNSUPPORTED
    b = gn.gn_qknorm_rope_bwd
    assert b(P, None, P, None, P, P, None, None, P, None, P, None, None, None, None, 0, 1, 4, 2, 128, 0,
             gn.GN_BF16, None) == gn.GN_ERR_NULL


def test_tune_rejects_unknown_keys(lib):
    assert gn.gn_tune(b"nope", 1) == gn.GN_ERR_SHAPE
    assert gn.gn_tune(b"stages", -1) == gn.GN_ERR_SHAPE
    assert gn.gn_tune(b"vpt", 3) == gn.GN_ERR_SHAPE
    assert gn.gn_tune(b"stages", 0) == gn.GN_OK


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    import importlib

    monkeypatch.setattr(gn, "_lib", None)
    monkeypatch.setattr(gn, "LIB_PATH", str(tmp_path / "libgn.so"))
    with pytest.raises(RuntimeError, match="missing"):
        gn.load()
    importlib.reload(gn)


def test_norm_linear_argument_checks(lib):
    f = gn.gn_norm_linear_fwd
    LN, RMS = gn.GN_NORM_LN, gn.GN_NORM_RMS
    ok = (P, P, P, P, P, P, P, 256, 512, 1024, 1024, 512, 1e-5)
    assert f(*ok, LN, 0, gn.GN_F32, None) == gn.GN_ERR_UNSUPPORTED
    assert f(*ok, LN, 0, 7, None) == gn.GN_ERR_DTYPE
    assert f(*ok, LN, 9, gn.GN_BF16, None) == gn.GN_ERR_DTYPE
    assert f(*ok, 5, 0, gn.GN_BF16, None) == gn.GN_ERR_SHAPE
    assert f(P, P, P, P, P, P, P, 256, 512, 1020, 1024, 512, 1e-5, LN, 0, gn.GN_BF16, None) == gn.GN_ERR_SHAPE
    assert f(P, P, P, P, P, P, P, 256, 512, 1024, 1000, 512, 1e-5, LN, 0, gn.GN_BF16, None) == gn.GN_ERR_SHAPE
    assert f(None, P, P, P, P, P, P, 256, 512, 1024, 1024, 512, 1e-5, LN, 0, gn.GN_BF16, None) == gn.GN_ERR_NULL
    assert f(P, P, None, P, P, P, P, 256, 512, 1024, 1024, 512, 1e-5, LN, 0, gn.GN_BF16, None) == gn.GN_ERR_NULL
    assert f(P, P, P, P, P, None, P, 256, 512, 1024, 1024, 512, 1e-5, LN, 0, gn.GN_BF16, None) == gn.GN_ERR_NULL
    assert f(P, P, P, P, P, P, None, 256, 512, 1024, 1024, 512, 1e-5, LN, 0, gn.GN_BF16, None) == gn.GN_ERR_NULL
    assert f(P + 8, P, P, P, P, P, P, 256, 512, 1024, 1024, 512, 1e-5, LN, 0, gn.GN_BF16,
             None) == gn.GN_ERR_ALIGN
    # RMSNorm needs no c; empty inputs launch nothing
    assert f(P, P, None, None, P, None, P, 0, 512, 1024, 1024, 512, 1e-5, RMS, 0, gn.GN_BF16, None) == gn.GN_OK
    p = gn.gn_norm_linear_prepare
    assert p(None, None, None, None, P, P, P, 8, 64, LN, 0, gn.GN_BF16, None) == gn.GN_ERR_NULL
    assert p(P, None, None, None, P, None, P, 8, 64, LN, 0, gn.GN_BF16, None) == gn.GN_ERR_NULL
    assert p(P, None, None, None, P, P, P, 8, 0, LN, 0, gn.GN_BF16, None) == gn.GN_ERR_SHAPE
    assert p(P, None, None, None, P, P, P, 0, 64, LN, 0, gn.GN_BF16, None) == gn.GN_OK


def test_activation_argument_checks(lib):
    for f, args in ((gn.gn_act_fwd, lambda z, y, n: (z, y, n)), (gn.gn_act_grad, lambda z, y, n: (z, P, y, n))):
        assert f(*args(P, P, 64), gn.GN_EPI_SILU, 7, None) == gn.GN_ERR_DTYPE
        assert f(*args(P, P, 64), 9, gn.GN_BF16, None) == gn.GN_ERR_DTYPE
        assert f(*args(P, P, -1), gn.GN_EPI_SILU, gn.GN_BF16, None) == gn.GN_ERR_SHAPE
        assert f(*args(P, P, 0), gn.GN_EPI_SILU, gn.GN_BF16, None) == gn.GN_OK  # nothing launched
        assert f(*args(None, P, 64), gn.GN_EPI_SILU, gn.GN_BF16, None) == gn.GN_ERR_NULL
        assert f(*args(P, None, 64), gn.GN_EPI_SILU, gn.GN_BF16, None) == gn.GN_ERR_NULL
        assert f(*args(P + 8, P, 64), gn.GN_EPI_SILU, gn.GN_BF16, None) == gn.GN_ERR_ALIGN
        assert f(*args(P, P + 4, 64), gn.GN_EPI_SILU, gn.GN_BF16, None) == gn.GN_ERR_ALIGN
