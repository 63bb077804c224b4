"""Seeded synthetic inputs for the norm + rotary-embedding path.

This module produces input bytes only; it holds none of the operations' arithmetic. The
same arrays feed the CUDA library (after a host-to-device copy) and the fp64 CPU oracle, so
both sides always see identical inputs.

Random streams. Every tensor draws from its own counter-based Philox stream keyed by
``(seed, stream id, chunk index)`` with chunks of ``CHUNK`` elements, so the first k elements
of a stream do not depend on how many are drawn in total (a smaller row count gives a prefix
of the full tensor) nor on how many threads generate it.

bfloat16 arrays are ``uint16`` bit patterns, rounded once from float32 with
round-to-nearest-even.

Shapes and distributions follow the video-DiT style workloads the source pages describe
(hidden 5120, 40 heads of 128, sequences of tens of thousands of tokens):

* ``rmsnorm``: x[M,N] ~ N(0,1) with 1% of rows (chosen without replacement) scaled by 50,
  weight 1 + 0.1 N(0,1) (plain) or 0.1 N(0,1) (Gemma offset), dy ~ N(0,1).
* ``layernorm``: row r ~ N(mu_r, sigma_r^2), mu_r ~ U(-2,2), sigma_r ~ U(0.5,3),
  weight 1 + 0.1 N(0,1), bias 0.1 N(0,1), dy ~ N(0,1).
* ``rope``: q, k [B,S,H,D] ~ N(0,1); fp32 tables cos/sin[S, D/2] for positions p = 0..S-1,
  angle p * theta^(-2i/D) evaluated in float64, then rounded to float32.
* ``qknorm_rope``: q, k [B,S,H,D] ~ N(0,1), weights 1 + 0.1 N(0,1) of length D, tables as
  above, dq_out, dk_out ~ N(0,1).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import math

import numpy as np

CHUNK = 1 << 22

# stream ids: one per tensor role, fixed forever so inputs never change meaning
S_X, S_W, S_B, S_DY, S_ROWS, S_MU, S_SIGMA, S_Q, S_K, S_WQ, S_WK, S_DQ, S_DK, S_LW, S_LB = range(1, 16)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest, ties to even. No NaN input."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).copy()
    u += np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float32 (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _gen(seed: int, stream: int, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[int(seed), (int(stream) << 32) | int(chunk)]))


def _draw(seed: int, stream: int, start: int, n: int, fill) -> None:
    """Elements [start, start + n) of a stream, chunk by chunk: fill(lo, hi, a) receives the
    float32 draws a of the global element range [lo, hi). A chunk is always drawn from its own
    start, so a range gives exactly the elements the whole-tensor draw has there."""
    if n <= 0:
        return
    c0, c1 = start // CHUNK, (start + n - 1) // CHUNK

    def work(c):
        lo, hi = max(start, c * CHUNK), min(start + n, (c + 1) * CHUNK)
        a = _gen(seed, stream, c).standard_normal(hi - c * CHUNK, dtype=np.float32)
        fill(lo, hi, a[lo - c * CHUNK:])

    if c1 == c0:
        work(c0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, range(c0, c1 + 1)))


def normal(seed: int, stream: int, n: int, dtype: str = "bf16", scale: float = 1.0,
           offset: float = 0.0, row_len: int = 0, row_scale=None, start: int = 0) -> np.ndarray:
    """Elements [start, start + n) of offset + scale * N(0,1) from one stream, as bf16 bits or
    float32.

    ``row_scale`` (indexed by the global row, element index // row_len, float32) multiplies each
    row after the scale and offset, before the single rounding to the output type."""
    out = np.empty(n, dtype=np.uint16 if dtype == "bf16" else np.float32)

    def fill(lo, hi, a):
        if scale != 1.0:
            a *= np.float32(scale)
        if offset != 0.0:
            a += np.float32(offset)
        if row_scale is not None:
            a *= row_scale[np.arange(lo, hi, dtype=np.int64) // row_len]
        out[lo - start:hi - start] = bf16_bits(a) if dtype == "bf16" else a

    _draw(seed, stream, start, n, fill)
    return out


def uniform(seed: int, stream: int, n: int, lo: float, hi: float) -> np.ndarray:
    return _gen(seed, stream, 0).uniform(lo, hi, n).astype(np.float32)


def outlier_rows(seed: int, M: int, frac: float = 0.01, factor: float = 50.0) -> np.ndarray:
    """float32 per-row multipliers: floor(frac*M) rows chosen without replacement get factor."""
    k = int(np.floor(frac * M))
    s = np.ones(M, dtype=np.float32)
    if k:
        s[_gen(seed, S_ROWS, 0).choice(M, size=k, replace=False)] = np.float32(factor)
    return s


def rope_tables(S: int, D: int, theta: float = 10000.0, p0: int = 0):
    """fp32 cos/sin [S, D/2] for positions p0..p0+S-1: angle p * theta^(-2i/D) in float64."""
    i = np.arange(D // 2, dtype=np.float64)
    freq = theta ** (-2.0 * i / D)
    ang = np.arange(p0, p0 + S, dtype=np.float64)[:, None] * freq[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


# ---- the workloads ----------------------------------------------------------------------------


def _range(total: int, part) -> tuple:
    lo, hi = (0, total) if part is None else (int(part[0]), int(part[1]))
    if not 0 <= lo <= hi <= total:
        raise ValueError(f"range {part} outside [0, {total}]")
    return lo, hi


def rmsnorm(M: int = 15360, N: int = 5120, dtype: str = "bf16", gemma: bool = False,
            outliers: bool = True, seed: int = 0, rows=None) -> dict:
    """``rows=(r0, r1)`` gives rows r0..r1-1 of the M-row workload (the outlier rows are still
    chosen among all M rows)."""
    r0, r1 = _range(M, rows)
    rs = outlier_rows(seed, M) if outliers else None
    return {
        "x": normal(seed, S_X, (r1 - r0) * N, dtype, row_len=N, row_scale=rs, start=r0 * N).reshape(r1 - r0, N),
        "w": normal(seed, S_W, N, dtype, scale=0.1, offset=0.0 if gemma else 1.0),
        "dy": normal(seed, S_DY, (r1 - r0) * N, dtype, start=r0 * N).reshape(r1 - r0, N),
        "eps": 1e-6, "gemma": gemma, "dtype": dtype,
    }


def layernorm(M: int = 32768, N: int = 5120, dtype: str = "bf16", seed: int = 0, rows=None) -> dict:
    """``rows=(r0, r1)`` gives rows r0..r1-1 of the M-row workload."""
    r0, r1 = _range(M, rows)
    mu = uniform(seed, S_MU, M, -2.0, 2.0)
    sg = uniform(seed, S_SIGMA, M, 0.5, 3.0)
    x = np.empty((r1 - r0) * N, dtype=np.uint16 if dtype == "bf16" else np.float32)

    def fill(lo, hi, a):
        rr = np.arange(lo, hi, dtype=np.int64) // N
        a = mu[rr] + sg[rr] * a
        x[lo - r0 * N:hi - r0 * N] = bf16_bits(a) if dtype == "bf16" else a

    _draw(seed, S_X, r0 * N, (r1 - r0) * N, fill)
    return {
        "x": x.reshape(r1 - r0, N),
        "w": normal(seed, S_W, N, dtype, scale=0.1, offset=1.0),
        "b": normal(seed, S_B, N, dtype, scale=0.1),
        "dy": normal(seed, S_DY, (r1 - r0) * N, dtype, start=r0 * N).reshape(r1 - r0, N),
        "eps": 1e-5, "dtype": dtype,
    }


def _tokens(seed: int, stream: int, B: int, S: int, H: int, D: int, s0: int, s1: int, dtype: str) -> np.ndarray:
    """Tokens s0..s1-1 of every batch entry of a [B, S, H, D] stream tensor."""
    per = H * D
    return np.stack([normal(seed, stream, (s1 - s0) * per, dtype, start=(b * S + s0) * per)
                     for b in range(B)]).reshape(B, s1 - s0, H, D)


def rope(B: int = 1, S: int = 32760, H: int = 40, D: int = 128, dtype: str = "bf16",
         theta: float = 10000.0, seed: int = 0, tokens=None) -> dict:
    """``tokens=(s0, s1)`` gives tokens s0..s1-1 of the S-token workload, with the table rows of
    their positions s0..s1-1."""
    s0, s1 = _range(S, tokens)
    cos, sin = rope_tables(s1 - s0, D, theta, p0=s0)
    return {
        "q": _tokens(seed, S_Q, B, S, H, D, s0, s1, dtype),
        "k": _tokens(seed, S_K, B, S, H, D, s0, s1, dtype),
        "cos": cos, "sin": sin, "dtype": dtype,
    }


def qknorm_rope(B: int = 2, S: int = 76800, H: int = 40, D: int = 128, dtype: str = "bf16",
                theta: float = 10000.0, seed: int = 0, grads: bool = True, tokens=None) -> dict:
    """``tokens=(s0, s1)`` gives tokens s0..s1-1 of the S-token workload, with the table rows of
    their positions s0..s1-1."""
    s0, s1 = _range(S, tokens)
    cos, sin = rope_tables(s1 - s0, D, theta, p0=s0)
    d = {
        "q": _tokens(seed, S_Q, B, S, H, D, s0, s1, dtype),
        "k": _tokens(seed, S_K, B, S, H, D, s0, s1, dtype),
        "wq": normal(seed, S_WQ, D, dtype, scale=0.1, offset=1.0),
        "wk": normal(seed, S_WK, D, dtype, scale=0.1, offset=1.0),
        "cos": cos, "sin": sin, "eps": 1e-6, "dtype": dtype,
    }
    if grads:
        d["dq_out"] = _tokens(seed, S_DQ, B, S, H, D, s0, s1, dtype)
        d["dk_out"] = _tokens(seed, S_DK, B, S, H, D, s0, s1, dtype)
    return d


# The five workloads: the fp32 parity case and the four bf16 long-sequence cases.
PR1_RMSNORM = dict(M=256, N=1024, dtype="f32", outliers=False)
PR1_ROPE = dict(B=1, S=256, H=8, D=128, dtype="f32")
RMSNORM_MAIN = dict(M=15360, N=5120, dtype="bf16")
LAYERNORM_MAIN = dict(M=32768, N=5120, dtype="bf16")
ROPE_MAIN = dict(B=1, S=32760, H=40, D=128, dtype="bf16")
QKNORM_MAIN = dict(B=2, S=76800, H=40, D=128, dtype="bf16")


def norm_linear(M: int = 32768, N: int = 5120, K: int = 5120, seed: int = 0) -> dict:
    """LayerNorm rows x[M, K] (the layernorm recipe: row mean ~ U(-2, 2), row scale ~ U(0.5, 3)),
    norm weight g = 1 + 0.1 N(0, 1) and bias beta = 0.1 N(0, 1) over K, then the linear layer
    W[N, K] ~ N(0, 1/K) (unit-scale outputs) with bias 0.1 N(0, 1) over N; all bf16."""
    d = layernorm(M=M, N=K, dtype="bf16", seed=seed)
    return {
        "x": d["x"], "g": d["w"], "beta": d["b"],
        "W": normal(seed, S_LW, N * K, "bf16", scale=1.0 / math.sqrt(K)).reshape(N, K),
        "bias": normal(seed, S_LB, N, "bf16", scale=0.1),
        "eps": 1e-5,
    }
