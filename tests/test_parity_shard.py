"""Token sharding with the CUDA kernels, on one GPU: the qk-norm + RoPE backward and the RMSNorm
backward run on each rank's shard (its tokens or rows, its RoPE table rows, its saved
statistics) exactly as a rank of a data-parallel job would, one shard after another. The dx
shards must concatenate to the unsharded kernel's dx bit for bit (rows are independent and the
per-row arithmetic does not depend on the launch), and the sum of the shards' weight gradients -
what the all-reduce of the gradient bucket computes - must match the unsharded dw and the oracle
within the gradient tolerance."""
import numpy as np
import pytest
import torch

import oracle
from tests._util import assert_close, to_dev, to_np
from transformer_norm_rope_b200 import workloads as wl
from transformer_norm_rope_b200.shard import GradBucket, shard_bounds, token_shard

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_qknorm_rope_backward_matches_unsharded(gpu, world):
    d = wl.qknorm_rope(B=2, S=101, H=40, D=128, dtype="bf16", seed=11)
    q, k, wq, wk = (to_dev(d[n]) for n in ("q", "k", "wq", "wk"))
    cos, sin = to_dev(d["cos"]), to_dev(d["sin"])
    dqo, dko = to_dev(d["dq_out"]), to_dev(d["dk_out"])
    _, _, rq, rk = gpu.qknorm_rope_fwd(q, k, wq, wk, cos, sin, d["eps"])
    dq, dk, dwq, dwk = gpu.qknorm_rope_bwd(q, k, wq, wk, cos, sin, rq, rk, dqo, dko)

    bucket = GradBucket({"dwq": 128, "dwk": 128}, "cuda")
    parts_q, parts_k = [], []
    for r in range(world):
        sh = lambda t, dim=1: token_shard(t, world, r, dim)  # noqa: E731
        a = gpu.qknorm_rope_bwd(sh(q), sh(k), wq, wk, sh(cos, 0), sh(sin, 0), sh(rq), sh(rk), sh(dqo), sh(dko))
        parts_q.append(a[0])
        parts_k.append(a[1])
        bucket["dwq"].add_(a[2])  # what the all-reduce over the ranks sums
        bucket["dwk"].add_(a[3])
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts_q, dim=1), dq) and torch.equal(torch.cat(parts_k, dim=1), dk)
    ref = oracle.qknorm_rope_bwd(d["q"], d["wq"], d["cos"], d["sin"], d["dq_out"], d["eps"], want_dx=False)[1]
    assert_close(to_np(bucket["dwq"]), ref, "grad_bf16", "sharded dwq vs oracle")
    # the shards' partial sums add in another order than the whole launch's: fp32 reassociation
    for name, got, whole in (("dwq", bucket["dwq"], dwq), ("dwk", bucket["dwk"], dwk)):
        w = to_np(whole)
        assert_close(to_np(got), w, (1e-4, 1e-4 * float(np.abs(w).max())), "sharded vs whole " + name)
    assert gpu.device_error(clear=True) == 0


def test_sharded_rmsnorm_backward_matches_unsharded(gpu):
    d = wl.rmsnorm(M=1000, N=5120, dtype="bf16", seed=12)
    x, w, dy = to_dev(d["x"]), to_dev(d["w"]), to_dev(d["dy"])
    _, r = gpu.rmsnorm_fwd(x, w, d["eps"])
    dx, dw = gpu.rmsnorm_bwd(x, w, r, dy)
    world = 4
    g = GradBucket({"dw": 5120}, "cuda")
    parts = []
    for rank in range(world):
        r0, r1 = shard_bounds(x.shape[0], world, rank)
        a = gpu.rmsnorm_bwd(x[r0:r1], w, r[r0:r1], dy[r0:r1])
        parts.append(a[0])
        g["dw"].add_(a[1])
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts), dx)
    w = to_np(dw)
    assert_close(to_np(g["dw"]), w, (1e-4, 1e-4 * float(np.abs(w).max())), "sharded vs whole dw")
    assert gpu.device_error(clear=True) == 0
