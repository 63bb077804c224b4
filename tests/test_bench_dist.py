"""Host logic of the benchmark (CPU): byte accounting, the multi-rank timing reduction over a
world of 2 gloo ranks, the token partition of the multi-GPU run (2 gloo ranks each generate
their shard of one global problem, run the oracle's backward on it and sum the weight
gradients with the bucket all-reduce), the all-cores oracle run, and the oracle (reference)
arm's JSON line on a tiny sample."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_match_the_workload_table():
    b = bench.algorithmic_bytes(bench.sizes(1.0))
    mb = {k: round(v / 1e6, 1) for k, v in b.items()}
    assert mb["rmsnorm_fwd"] == 314.6 and mb["rmsnorm_bwd"] == 472.0
    assert mb["layernorm_fwd"] == 671.4 and mb["layernorm_bwd"] == 1007.0
    assert mb["rope_fwd"] == 1358.6 and mb["rope_bwd"] == 1358.6
    assert mb["qknorm_rope_fwd"] == 6379.9 and mb["qknorm_rope_bwd"] == 9525.7


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        dev = torch.device("cpu")
        bench.barrier(ws, dev)
        # rank r processed 1e9*(r+1) bytes in (r+1) seconds: the job moved 3e9 bytes and the
        # slowest rank took 2 s, so the whole-job figure is 1.5 GB/s (not the mean of ratios)
        v, el = bench.throughput_gbs(1e9 * (rank + 1), float(rank + 1), ws, dev)
        mx = bench.reduce_over_ranks(rank * 10.0, ws, dev, "max")
        q.put((rank, v, el, mx))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, v, el, mx in res:
        assert v == pytest.approx(1.5) and el == 2.0 and mx == 10.0


def _shard_worker(rank, ws, port, q):
    import oracle
    from transformer_norm_rope_b200.shard import GradBucket

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        z = bench.sizes(0.002)
        host = bench.gen_inputs(z, 0, ("rms", "qk"), ws, rank)
        r, k = host["rms"], host["qk"]
        grads = GradBucket({"rdw": z["rms"]["N"], "qdwq": z["qk"]["D"]}, torch.device("cpu"))
        rdx, rdw = oracle.rmsnorm_bwd(r["x"], r["w"], r["dy"], r["eps"])
        qdx, qdw = oracle.qknorm_rope_bwd(k["q"], k["wq"], k["cos"], k["sin"], k["dq_out"], k["eps"])
        grads["rdw"].copy_(torch.from_numpy(rdw))
        grads["qdwq"].copy_(torch.from_numpy(qdw))
        grads.allreduce()
        q.put((rank, r["x"], k["q"], k["cos"], rdx, qdx, grads["rdw"].numpy().copy(), grads["qdwq"].numpy().copy()))
    finally:
        dist.destroy_process_group()


def test_token_partition_tiles_one_global_problem_over_two_gloo_ranks():
    import oracle

    z = bench.sizes(0.002)
    g = bench.global_sizes(z, 2)
    for fam in ("rms", "ln", "rope", "qk"):  # the shards tile the global rows / tokens in rank order
        key = "M" if fam in ("rms", "ln") else "S"
        b0, b1 = bench.shard_ranges(z, 2, 0)[fam], bench.shard_ranges(z, 2, 1)[fam]
        assert b0[0] == 0 and b0[1] == b1[0] and b1[1] == g[fam][key] and b0[1] - b0[0] == z[fam][key]
    rows, grows = bench.rows_of(z), bench.rows_of(g)
    assert all(2 * rows[k] == grows[k] for k in rows)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(2)), key=lambda t: t[0])
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    whole = bench.gen_inputs(g, 0, ("rms", "qk"))
    r, k = whole["rms"], whole["qk"]
    np.testing.assert_array_equal(np.concatenate([res[0][1], res[1][1]]), r["x"])
    np.testing.assert_array_equal(np.concatenate([res[0][2], res[1][2]], axis=1), k["q"])
    np.testing.assert_array_equal(np.concatenate([res[0][3], res[1][3]]), k["cos"])  # table rows by position
    rdx, rdw = oracle.rmsnorm_bwd(r["x"], r["w"], r["dy"], r["eps"])
    qdx, qdw = oracle.qknorm_rope_bwd(k["q"], k["wq"], k["cos"], k["sin"], k["dq_out"], k["eps"])
    np.testing.assert_array_equal(np.concatenate([res[0][4], res[1][4]]), rdx)  # rows are independent
    np.testing.assert_array_equal(np.concatenate([res[0][5], res[1][5]], axis=1), qdx)
    for rank in range(2):  # every rank holds the all-reduced (fp32) sum of the shards' gradients
        np.testing.assert_allclose(res[rank][6], rdw, rtol=1e-5, atol=1e-5 * np.abs(rdw).max())
        np.testing.assert_allclose(res[rank][7], qdw, rtol=1e-5, atol=1e-5 * np.abs(qdw).max())


def test_all_cores_oracle_run_covers_the_sample():
    z = bench.sizes(0.001)
    kernels = ["rmsnorm_fwd", "layernorm_bwd", "rope_fwd", "qknorm_rope_bwd"]
    t, done = bench.oracle_all_cores(z, 0, kernels, 1.0, 3)
    nb = bench.algorithmic_bytes(z)
    assert t > 0 and done == pytest.approx(sum(nb[k] for k in kernels))


def test_oracle_pool_runs_repeat():
    """A pool's processes keep their inputs between runs: every run covers the same sample."""
    z = bench.sizes(0.001)
    kernels = ["rmsnorm_bwd", "rope_bwd"]
    pool = bench.OraclePool(z, 0, kernels, 0.5, 2)
    try:
        runs = [pool.run() for _ in range(3)]
    finally:
        pool.close()
    assert all(t > 0 for t, _ in runs)
    assert len({b for _, b in runs}) == 1
    assert all(not p.is_alive() for p in pool.procs)


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--scale", "0.002", "--steps", "2",
                        "--warmup", "1"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["unit"] == "GB/s" and out["value"] > 0
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["cores"] == bench.host_cores()
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["metric"] == bench.METRIC


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--scale", "0.001", "--steps", "1",
                        "--warmup", "0"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
