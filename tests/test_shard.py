"""Token sharding over ranks (CPU): shard bounds, table slicing, the gradient bucket and its
all-reduce over a world of 2 gloo ranks, and - with the fp64 oracle standing in for each rank's
kernels - that running the backward on token shards and summing the weight gradients over the
ranks gives the unsharded result."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from transformer_norm_rope_b200 import workloads as wl
from transformer_norm_rope_b200.shard import GradBucket, shard_bounds, token_shard


@pytest.mark.parametrize("n", [0, 1, 2, 7, 64, 1000, 76800])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_bounds_tile_the_range(n, world):
    b = [shard_bounds(n, world, r) for r in range(world)]
    assert b[0][0] == 0 and b[-1][1] == n
    for (s0, s1), (t0, _) in zip(b, b[1:]):
        assert s1 == t0
    sizes = [s1 - s0 for s0, s1 in b]
    assert max(sizes) - min(sizes) <= 1 and all(s >= 0 for s in sizes)


def test_shard_bounds_reject_bad_requests():
    for n, w, r in [(5, 0, 0), (5, 2, 2), (5, 2, -1), (-1, 2, 0)]:
        with pytest.raises(ValueError):
            shard_bounds(n, w, r)


def test_token_shards_concatenate_to_the_tensor():
    x = torch.arange(2 * 11 * 3 * 8, dtype=torch.float32).reshape(2, 11, 3, 8)
    parts = [token_shard(x, 4, r) for r in range(4)]
    assert all(p.is_contiguous() for p in parts)
    assert torch.equal(torch.cat(parts, dim=1), x)
    tab = torch.arange(11 * 4, dtype=torch.float32).reshape(11, 4)
    assert torch.equal(torch.cat([token_shard(tab, 4, r, dim=0) for r in range(4)]), tab)
    # a rank's slice of the RoPE tables is the table of its own positions
    cos, sin = wl.rope_tables(11, 8)
    for r in range(3):
        s0, s1 = shard_bounds(11, 3, r)
        c, s = wl.rope_tables(s1 - s0, 8, p0=s0)
        np.testing.assert_array_equal(token_shard(torch.from_numpy(cos), 3, r, 0).numpy(), c)
        np.testing.assert_array_equal(token_shard(torch.from_numpy(sin), 3, r, 0).numpy(), s)


def test_bucket_views_are_aligned_disjoint_and_zeroed():
    g = GradBucket({"a": 5, "b": 128, "c": 3}, "cpu")
    assert [g[k].numel() for k in g.names()] == [5, 128, 3]
    for k in g.names():
        assert g[k].data_ptr() % 16 == 0 and torch.count_nonzero(g[k]) == 0
    g["a"].fill_(1.0)
    g["b"].fill_(2.0)
    g["c"].fill_(3.0)
    assert float(g.flat.sum()) == 5 * 1 + 128 * 2 + 3 * 3
    g.allreduce()  # no process group: a no-op
    assert float(g.flat.sum()) == 5 + 256 + 9
    with pytest.raises(ValueError):
        GradBucket({"a": 0}, "cpu")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


# the sharded-backward case: qk-norm + RoPE on tokens, RMSNorm on rows (small, fp64 oracle)
QK = dict(B=2, S=13, H=3, D=16, eps=1e-6)
RMS = dict(M=37, N=48, eps=1e-6)


def _qk_inputs():
    B, S, H, D = QK["B"], QK["S"], QK["H"], QK["D"]
    g = np.random.default_rng(7)
    x = g.standard_normal((B, S, H, D))
    dy = g.standard_normal((B, S, H, D))
    w = 1 + 0.1 * g.standard_normal(D)
    cos, sin = wl.rope_tables(S, D, 10000.0)
    return x, dy, w, cos, sin


def _rms_inputs():
    g = np.random.default_rng(8)
    x = g.standard_normal((RMS["M"], RMS["N"]))
    dy = g.standard_normal((RMS["M"], RMS["N"]))
    w = 1 + 0.1 * g.standard_normal(RMS["N"])
    return x, dy, w


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        # 1. the bucket sums over the ranks, every view at once
        g = GradBucket({"dw": 5, "db": 6}, "cpu")
        g["dw"].fill_(rank + 1.0)
        g["db"].copy_(torch.arange(6, dtype=torch.float32) * (rank + 1))
        g.allreduce()
        bucket = (g["dw"].tolist(), g["db"].tolist())

        # 2. qk-norm + RoPE backward on this rank's tokens (and table rows), dw summed
        x, dy, w, cos, sin = _qk_inputs()
        s0, s1 = shard_bounds(QK["S"], ws, rank)
        dx, dw = oracle.qknorm_rope_bwd(x[:, s0:s1], w, cos[s0:s1], sin[s0:s1], dy[:, s0:s1], QK["eps"])
        t = torch.from_numpy(dw.copy())
        dist.all_reduce(t)
        qk = (s0, s1, dx, t.numpy())

        # 3. RMSNorm backward on this rank's rows
        x, dy, w = _rms_inputs()
        r0, r1 = shard_bounds(RMS["M"], ws, rank)
        dxr, dwr = oracle.rmsnorm_bwd(x[r0:r1], w, dy[r0:r1], RMS["eps"])
        t = torch.from_numpy(dwr.copy())
        dist.all_reduce(t)
        rms = (r0, r1, dxr, t.numpy())
        q.put((rank, bucket, qk, rms))
    finally:
        dist.destroy_process_group()


def test_sharded_backward_over_two_gloo_ranks_matches_the_unsharded_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(2)), key=lambda r: r[0])
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for _, (dw, db), _, _ in res:
        assert dw == [3.0] * 5 and db == [3.0 * i for i in range(6)]

    x, dy, w, cos, sin = _qk_inputs()
    dx_ref, dw_ref = oracle.qknorm_rope_bwd(x, w, cos, sin, dy, QK["eps"])
    dx = np.concatenate([r[2][2] for r in res], axis=1)
    assert [r[2][:2] for r in res] == [(0, 7), (7, 13)]
    np.testing.assert_array_equal(dx, dx_ref)  # rows are independent: bit-identical
    for r in res:
        np.testing.assert_allclose(r[2][3], dw_ref, rtol=1e-12, atol=1e-12)

    x, dy, w = _rms_inputs()
    dxr_ref, dwr_ref = oracle.rmsnorm_bwd(x, w, dy, RMS["eps"])
    np.testing.assert_array_equal(np.concatenate([r[3][2] for r in res]), dxr_ref)
    for r in res:
        np.testing.assert_allclose(r[3][3], dwr_ref, rtol=1e-12, atol=1e-12)
