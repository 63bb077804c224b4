"""Failure detection without a GPU fault: every wait of the kernels is bounded. A kernel that
waits on an mbarrier phase nothing completes must give up after its limit, record the
timeout in the device error word and return, and the context must keep working."""
import pytest
import torch

from transformer_norm_rope_b200 import workloads as wl
from tests._util import assert_close, to_dev, to_np

import oracle

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_reports(gpu):
    gpu.device_error(clear=True)
    stream = torch.cuda.current_stream().cuda_stream
    gpu.check(gpu.gn_selftest_wait_timeout(20000, stream), "gn_selftest_wait_timeout")  # 20 ms
    word = gpu.device_error(clear=True)
    assert word & gpu.GN_DEVERR_WAIT_TIMEOUT
    assert gpu.device_error() == 0
    # the context is still usable: a normal call afterwards is correct and reports nothing
    d = wl.rmsnorm(M=64, N=5120, dtype="bf16", outliers=False)
    y, r = gpu.rmsnorm_fwd(to_dev(d["x"]), to_dev(d["w"]), d["eps"])
    torch.cuda.synchronize()
    ry, _ = oracle.rmsnorm_fwd(d["x"], d["w"], d["eps"])
    assert_close(to_np(y), ry, "bf16", "rmsnorm after the timeout self-test")
    assert gpu.device_error() == 0


def test_selftest_rejects_bad_limits(gpu):
    assert gpu.gn_selftest_wait_timeout(0, None) == gpu.GN_ERR_SHAPE
    assert gpu.gn_selftest_wait_timeout(2000000, None) == gpu.GN_ERR_SHAPE
