"""gn_qknorm_rope_bwd_noalloc: the backward for callers that cannot allocate device memory
(code inside another framework's callback or plugin, or a process whose memory another
allocator owns). It keeps its per-block partial sums in a fixed array inside the library
instead of a caller workspace. This file is collected last on purpose.

The test calls both C entry points directly (ctypes, raw device pointers) on the same inputs
and requires the no-allocation variant to match the workspace variant within the gradient
tolerance, on two calls in a row (the second call reuses the array the first one filled).
"""
import numpy as np
import pytest
import torch

from transformer_norm_rope_b200 import workloads as wl
from tests._util import assert_close, to_dev, to_np

pytestmark = pytest.mark.gpu


def test_noalloc_backward_matches_workspace_backward(gpu):
    d = wl.qknorm_rope(B=2, S=96, H=40, D=128, dtype="bf16", seed=3)
    q, k, wq, wk = (to_dev(d[n]) for n in ("q", "k", "wq", "wk"))
    cos, sin = to_dev(d["cos"]), to_dev(d["sin"])
    dqo, dko = to_dev(d["dq_out"]), to_dev(d["dk_out"])
    _, _, rq, rk = gpu.qknorm_rope_fwd(q, k, wq, wk, cos, sin, d["eps"])
    B, S, H, D = q.shape
    stream = torch.cuda.current_stream().cuda_stream

    # reference: the entry point with a caller-owned workspace
    dq0, dk0 = torch.empty_like(q), torch.empty_like(k)
    dwq0 = torch.empty(D, dtype=torch.float32, device="cuda")
    dwk0 = torch.empty(D, dtype=torch.float32, device="cuda")
    nws = gpu.gn_qknorm_rope_bwd_workspace(B, S, H, D, gpu.GN_BF16)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    gpu.check(gpu.gn_qknorm_rope_bwd(q.data_ptr(), k.data_ptr(), wq.data_ptr(), wk.data_ptr(), cos.data_ptr(),
                                     sin.data_ptr(), rq.data_ptr(), rk.data_ptr(), dqo.data_ptr(), dko.data_ptr(),
                                     dq0.data_ptr(), dk0.data_ptr(), dwq0.data_ptr(), dwk0.data_ptr(),
                                     ws.data_ptr(), nws, B, S, H, D, 0, gpu.GN_BF16, stream))
    torch.cuda.synchronize()

    for call in range(2):
        dq, dk = torch.full_like(q, float("nan")), torch.full_like(k, float("nan"))
        dwq = torch.full((D,), float("nan"), dtype=torch.float32, device="cuda")
        dwk = torch.full((D,), float("nan"), dtype=torch.float32, device="cuda")
        gpu.check(gpu.gn_qknorm_rope_bwd_noalloc(q.data_ptr(), k.data_ptr(), wq.data_ptr(), wk.data_ptr(),
                                                 cos.data_ptr(), sin.data_ptr(), rq.data_ptr(), rk.data_ptr(),
                                                 dqo.data_ptr(), dko.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                                 dwq.data_ptr(), dwk.data_ptr(), B, S, H, D, 0, gpu.GN_BF16,
                                                 stream), "gn_qknorm_rope_bwd_noalloc")
        torch.cuda.synchronize()
        tag = f"no-alloc call {call + 1}"
        assert_close(to_np(dq), to_np(dq0), "grad_bf16", tag + " dq")
        assert_close(to_np(dk), to_np(dk0), "grad_bf16", tag + " dk")
        assert_close(to_np(dwq), to_np(dwq0), "grad_bf16", tag + " dwq")
        assert_close(to_np(dwk), to_np(dwk0), "grad_bf16", tag + " dwk")
    assert gpu.device_error() == 0
