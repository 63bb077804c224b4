"""Complete comparison of full-size GPU results with the fp64 oracle, spread over host processes.

The full-size workloads hold up to 786 M elements per tensor. Every output element is compared
with the oracle: the rows (or tokens) are cut into chunks, each chunk's inputs and GPU outputs
go to a worker process that runs the oracle on the chunk and checks the outputs against it with
the suite's element-wise tolerances, and returns only the verdict (plus its share of the weight
gradients, summed here in chunk order). The pool is started with ``spawn``: a process forked
after the first CUDA call could hang.
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np

from tests._util import TOL

CHUNK_ELEMS = 1 << 23  # elements of one tensor per chunk (16 MiB of bf16)


def workers() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def bits(t):
    """torch tensor -> numpy: bf16 as uint16 bit patterns, fp32 as float32 (both exact)."""
    import torch

    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _wide(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _check(name, got, ref, tol, where):
    """{name: (n_bad, n, worst)}; worst = (chunk, index within the chunk, got, ref) or None."""
    rtol, atol = TOL[tol] if isinstance(tol, str) else tol
    ref = np.asarray(ref, dtype=np.float64)
    g = _wide(got).reshape(-1)
    r = ref.reshape(-1)
    nonfinite = ~np.isfinite(g)
    excess = np.abs(g - r) - (atol + rtol * np.abs(r))
    bad = (excess > 0) | nonfinite
    nbad = int(bad.sum())
    worst = None
    if nbad:
        i = int(np.argmax(np.where(nonfinite, np.inf, excess)))
        worst = (where, tuple(int(j) for j in np.unravel_index(i, ref.shape)), float(g[i]), float(r[i]))
    return {name: (nbad, g.size, worst)}


# ------------------------------------------------------------------ chunk jobs (run in workers)

def job_rms(x, w, dy, eps, gemma, y, r, dx, where):
    import oracle

    ry, rr = oracle.rmsnorm_fwd(x, w, eps, gemma=gemma)
    rdx, rdw = oracle.rmsnorm_bwd(x, w, dy, eps, gemma=gemma)
    out = {}
    out.update(_check("y", y, ry, "bf16", where))
    out.update(_check("inv_rms", r, rr, "stat", where))
    out.update(_check("dx", dx, rdx, "grad_bf16", where))
    return out, {"dw": rdw}


def job_ln(x, w, b, dy, eps, act, y, mu, rs, dx, where):
    import oracle

    ry, rmu, rrs = oracle.layernorm_fwd(x, w, b, eps, act=act)
    rdx, rdw, rdb = oracle.layernorm_bwd(x, w, b, dy, eps, act=act)
    out = {}
    out.update(_check("y", y, ry, "bf16", where))
    out.update(_check("mean", mu, rmu, (1e-5, 1e-6), where))
    out.update(_check("rstd", rs, rrs, "stat", where))
    out.update(_check("dx", dx, rdx, "grad_bf16", where))
    return out, {"dw": rdw, "db": rdb}


def job_rope(x, cos, sin, fwd, bwd, where):
    """x [B, Sc, H, D] input chunk; fwd: the GPU's forward result on it; bwd: the GPU's
    backward (sin negated) applied to fwd. The backward is checked against the oracle applied
    to the GPU's own forward output, the input the backward kernel actually read."""
    import oracle

    out = {}
    out.update(_check("fwd", fwd, oracle.rope(x, cos, sin, +1), "bf16", where))
    out.update(_check("bwd", bwd, oracle.rope(fwd, cos, sin, -1), "bf16", where))
    return out, {}


def job_qk(x, w, cos, sin, dy, eps, gemma, o, r, dx, where):
    import oracle

    ro, rr = oracle.qknorm_rope_fwd(x, w, cos, sin, eps, gemma=gemma)
    rdx, rdw = oracle.qknorm_rope_bwd(x, w, cos, sin, dy, eps, gemma=gemma)
    out = {}
    out.update(_check("out", o, ro, "bf16", where))
    out.update(_check("inv_rms", r, rr, "stat", where))
    out.update(_check("dx", dx, rdx, "grad_bf16", where))
    return out, {"dw": rdw}


def _call(job):
    fn, args = job
    return fn(*args)


# ------------------------------------------------------------------ driver (main process)

class Verdict:
    """Accumulates the chunk verdicts of one comparison and the summed weight-gradient parts."""

    def __init__(self, what):
        self.what = what
        self.bad = {}
        self.parts = {}

    def add(self, res):
        checks, parts = res
        for k, (nbad, n, worst) in checks.items():
            b, tot, w = self.bad.get(k, (0, 0, None))
            self.bad[k] = (b + nbad, tot + n, w if w is not None else worst)
        for k, v in parts.items():
            self.parts[k] = self.parts[k] + v if k in self.parts else np.array(v, dtype=np.float64)

    def assert_ok(self):
        msgs = [f"{self.what} {k}: {b} of {n} elements out of tolerance; worst of the first failing chunk "
                f"(chunk, index, got, ref) {w}"
                for k, (b, n, w) in sorted(self.bad.items()) if b]
        assert not msgs, "\n".join(msgs)
        return {k: n for k, (_, n, _) in self.bad.items()}


def run(jobs, what, window=None):
    """Runs the (fn, args) jobs (an iterator, consumed lazily) on a spawn pool with a bounded
    number in flight; results are folded in job order."""
    v = Verdict(what)
    ctx = mp.get_context("spawn")
    nw = workers()
    window = window or 2 * nw
    with ctx.Pool(nw) as pool:
        pending = []
        for job in jobs:
            pending.append(pool.apply_async(_call, (job,)))
            if len(pending) >= window:
                v.add(pending.pop(0).get())
        for p in pending:
            v.add(p.get())
    return v


def row_chunks(M, N, elems=CHUNK_ELEMS):
    step = max(1, elems // max(1, N))
    for r0 in range(0, M, step):
        yield r0, min(M, r0 + step)


def token_chunks(S, per_token, elems=CHUNK_ELEMS):
    step = max(1, elems // max(1, per_token))
    for s0 in range(0, S, step):
        yield s0, min(S, s0 + step)
