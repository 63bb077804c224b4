"""The complete full-size comparison machinery (tests/_fullsize.py), checked on the CPU: chunked
oracle runs on spawned worker processes must accept outputs that match the oracle, find a
single wrong element anywhere, and return the weight-gradient parts whose sum is the oracle's
whole-tensor gradient."""
import numpy as np

import oracle
from tests import _fullsize as fs
from transformer_norm_rope_b200 import workloads as wl


def _bf16(a):
    return wl.bf16_bits(np.asarray(a, dtype=np.float32))


def _rms_jobs(d, y, r, dx, M, N):
    for r0, r1 in fs.row_chunks(M, N, elems=4 * N):
        yield fs.job_rms, (d["x"][r0:r1], d["w"], d["dy"][r0:r1], d["eps"], False, y[r0:r1], r[r0:r1], dx[r0:r1],
                           f"rows {r0}:{r1}")


def test_chunked_comparison_accepts_exact_and_finds_one_wrong_element():
    M, N = 37, 72
    d = wl.rmsnorm(M=M, N=N, dtype="bf16", seed=4, outliers=False)
    ry, rr = oracle.rmsnorm_fwd(d["x"], d["w"], d["eps"])
    rdx, rdw = oracle.rmsnorm_bwd(d["x"], d["w"], d["dy"], d["eps"])
    y, r, dx = _bf16(ry), rr.astype(np.float32), _bf16(rdx)
    v = fs.run(_rms_jobs(d, y, r, dx, M, N), "exact")
    assert v.assert_ok() == {"y": M * N, "inv_rms": M, "dx": M * N}
    np.testing.assert_allclose(v.parts["dw"], rdw, rtol=1e-12, atol=1e-12)
    bad = dx.copy()
    bad[29, 50] ^= np.uint16(0x0100)  # one element, in the last chunk, off by a few percent
    v = fs.run(_rms_jobs(d, y, r, bad, M, N), "planted")
    try:
        v.assert_ok()
    except AssertionError as e:
        msg = str(e)
    else:
        raise AssertionError("the planted error was not found")
    assert "dx: 1 of" in msg and "rows 28:32" in msg and "(1, 50)" in msg, msg
