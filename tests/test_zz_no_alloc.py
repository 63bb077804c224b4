"""gn_qknorm_rope_bwd_noalloc: the backward for callers that cannot allocate device memory
(code inside another framework's callback or plugin, or a process whose memory another
allocator owns). It keeps its per-block partial sums in a fixed array inside the library
instead of a caller workspace. This file is collected last on purpose.

The tests call both C entry points directly (ctypes, raw device pointers) on the same inputs.
Both run the same kernel on the same grid and sum the partials in the same fixed order, so the
no-allocation variant must give the workspace variant's results bit for bit: on two calls in a
row (the second call reuses the array the first one filled), with and without k, and it must
refuse, before launching anything, a call whose partials would not fit the array.
"""
import pytest
import torch

from transformer_norm_rope_b200 import workloads as wl
from tests._util import to_dev

pytestmark = pytest.mark.gpu

FIXED_BYTES = 1 << 20  # size of the library's fixed partial-sum array


def _inputs(gpu, B, S, H, D, seed):
    d = wl.qknorm_rope(B=B, S=S, H=H, D=D, dtype="bf16", seed=seed)
    t = {n: to_dev(d[n]) for n in ("q", "k", "wq", "wk", "cos", "sin", "dq_out", "dk_out")}
    _, _, t["rq"], t["rk"] = gpu.qknorm_rope_fwd(t["q"], t["k"], t["wq"], t["wk"], t["cos"], t["sin"], d["eps"])
    return t


def _ptr(t):
    return None if t is None else t.data_ptr()


def _outputs(q, with_k, D):
    nan = float("nan")
    dq = torch.full_like(q, nan)
    dk = torch.full_like(q, nan) if with_k else None
    dwq = torch.full((D,), nan, dtype=torch.float32, device=q.device)
    dwk = torch.full((D,), nan, dtype=torch.float32, device=q.device) if with_k else None
    return dq, dk, dwq, dwk


def _call_ws(gpu, t, with_k, stream):
    q = t["q"]
    B, S, H, D = q.shape
    k = t["k"] if with_k else None
    dq, dk, dwq, dwk = _outputs(q, with_k, D)
    nws = gpu.gn_qknorm_rope_bwd_workspace(B, S, H, D, gpu.GN_BF16)
    ws = torch.empty(nws, dtype=torch.uint8, device=q.device)
    gpu.check(gpu.gn_qknorm_rope_bwd(q.data_ptr(), _ptr(k), t["wq"].data_ptr(), _ptr(t["wk"] if with_k else None),
                                     t["cos"].data_ptr(), t["sin"].data_ptr(), t["rq"].data_ptr(),
                                     _ptr(t["rk"] if with_k else None), t["dq_out"].data_ptr(),
                                     _ptr(t["dk_out"] if with_k else None), dq.data_ptr(), _ptr(dk), dwq.data_ptr(),
                                     _ptr(dwk), ws.data_ptr(), nws, B, S, H, D, 0, gpu.GN_BF16, stream),
              "gn_qknorm_rope_bwd")
    return dq, dk, dwq, dwk


def _call_noalloc(gpu, t, with_k, stream, outs=None):
    q = t["q"]
    B, S, H, D = q.shape
    k = t["k"] if with_k else None
    dq, dk, dwq, dwk = outs if outs is not None else _outputs(q, with_k, D)
    st = gpu.gn_qknorm_rope_bwd_noalloc(q.data_ptr(), _ptr(k), t["wq"].data_ptr(),
                                        _ptr(t["wk"] if with_k else None), t["cos"].data_ptr(), t["sin"].data_ptr(),
                                        t["rq"].data_ptr(), _ptr(t["rk"] if with_k else None),
                                        t["dq_out"].data_ptr(), _ptr(t["dk_out"] if with_k else None), dq.data_ptr(),
                                        _ptr(dk), dwq.data_ptr(), _ptr(dwk), B, S, H, D, 0, gpu.GN_BF16, stream)
    return st, (dq, dk, dwq, dwk)


@pytest.mark.parametrize("with_k", [True, False])
def test_noalloc_backward_matches_workspace_backward(gpu, with_k):
    t = _inputs(gpu, B=2, S=96, H=40, D=128, seed=3)
    stream = torch.cuda.current_stream().cuda_stream
    ref = _call_ws(gpu, t, with_k, stream)
    torch.cuda.synchronize()
    for call in range(2):
        st, got = _call_noalloc(gpu, t, with_k, stream)
        gpu.check(st, "gn_qknorm_rope_bwd_noalloc")
        torch.cuda.synchronize()
        for name, a, b in zip(("dq", "dk", "dwq", "dwk"), got, ref):
            if b is None:
                assert a is None
                continue
            assert torch.equal(a, b), f"no-alloc call {call + 1} (k {'given' if with_k else 'absent'}): {name} differs"
    assert gpu.device_error() == 0


def test_noalloc_refuses_partials_beyond_the_fixed_array(gpu):
    """A call whose per-block partials (2 * D * 4 bytes for each block of the persistent grid)
    exceed the fixed array returns GN_ERR_WORKSPACE and leaves every output untouched. Head dim
    256 with one head per unit and four consumer warps per block gives a grid of more than 512
    blocks; the workspace query reports grid * 2 * D * 4 bytes for the larger grid of the plain
    and Gemma variants, so the variant with that grid must be refused (the other may run)."""
    B, S, H, D = 1, 4096, 4, 256
    t = _inputs(gpu, B=B, S=S, H=H, D=D, seed=5)
    stream = torch.cuda.current_stream().cuda_stream
    found = None
    try:
        for unit_bytes, group_rows, stages in ((0, 0, 0), (2048, 4, 0), (2048, 4, 2), (1024, 4, 2), (512, 4, 2)):
            gpu.tune("unit_bytes", unit_bytes)
            gpu.tune("group_rows", group_rows)
            gpu.tune("stages", stages)
            need = gpu.gn_qknorm_rope_bwd_workspace(B, S, H, D, gpu.GN_BF16)
            if need > FIXED_BYTES:
                found = (unit_bytes, group_rows, stages, need)
                break
        assert found is not None, "no launch shape on this device needs more than the fixed array"
        refused = 0
        for gemma in (0, 1):
            q = t["q"]
            dq, dk, dwq, dwk = _outputs(q, True, D)
            st = gpu.gn_qknorm_rope_bwd_noalloc(q.data_ptr(), t["k"].data_ptr(), t["wq"].data_ptr(),
                                                t["wk"].data_ptr(), t["cos"].data_ptr(), t["sin"].data_ptr(),
                                                t["rq"].data_ptr(), t["rk"].data_ptr(), t["dq_out"].data_ptr(),
                                                t["dk_out"].data_ptr(), dq.data_ptr(), dk.data_ptr(), dwq.data_ptr(),
                                                dwk.data_ptr(), B, S, H, D, gemma, gpu.GN_BF16, stream)
            torch.cuda.synchronize()
            if st == gpu.GN_ERR_WORKSPACE:
                refused += 1
                for o in (dq, dk, dwq, dwk):  # nothing was launched: the NaN fill is intact
                    assert torch.isnan(o).all()
            else:
                assert st == gpu.GN_OK, f"{found} gemma={gemma}: status {st}"
        assert refused >= 1, f"{found}: no variant refused"
    finally:
        for key in ("unit_bytes", "group_rows", "stages"):
            gpu.tune(key, 0)
    assert gpu.device_error() == 0
