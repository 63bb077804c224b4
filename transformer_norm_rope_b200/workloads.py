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


def normal(seed: int, stream: int, n: int, dtype: str = "bf16", scale: float = 1.0,
           offset: float = 0.0, row_len: int = 0, row_scale=None) -> np.ndarray:
    """n draws of offset + scale * N(0,1) from one stream, as bf16 bits or float32.

    ``row_scale`` (length n // row_len, float32) multiplies row r after the scale and offset,
    before the single rounding to the output type."""
    out = np.empty(n, dtype=np.uint16 if dtype == "bf16" else np.float32)

    def work(c):
        s, e = c * CHUNK, min(n, (c + 1) * CHUNK)
        a = _gen(seed, stream, c).standard_normal(e - s, dtype=np.float32)
        if scale != 1.0:
            a *= np.float32(scale)
        if offset != 0.0:
            a += np.float32(offset)
        if row_scale is not None:
            rows = np.arange(s, e, dtype=np.int64) // row_len
            a *= row_scale[rows]
        out[s:e] = bf16_bits(a) if dtype == "bf16" else a

    nchunks = (n + CHUNK - 1) // CHUNK
    if nchunks <= 1:
        for c in range(nchunks):
            work(c)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, range(nchunks)))
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


def rmsnorm(M: int = 15360, N: int = 5120, dtype: str = "bf16", gemma: bool = False,
            outliers: bool = True, seed: int = 0) -> dict:
    rs = outlier_rows(seed, M) if outliers else None
    return {
        "x": normal(seed, S_X, M * N, dtype, row_len=N, row_scale=rs).reshape(M, N),
        "w": normal(seed, S_W, N, dtype, scale=0.1, offset=0.0 if gemma else 1.0),
        "dy": normal(seed, S_DY, M * N, dtype).reshape(M, N),
        "eps": 1e-6, "gemma": gemma, "dtype": dtype,
    }


def layernorm(M: int = 32768, N: int = 5120, dtype: str = "bf16", seed: int = 0) -> dict:
    mu = uniform(seed, S_MU, M, -2.0, 2.0)
    sg = uniform(seed, S_SIGMA, M, 0.5, 3.0)
    x = np.empty(M * N, dtype=np.uint16 if dtype == "bf16" else np.float32)

    def work(c):
        s, e = c * CHUNK, min(M * N, (c + 1) * CHUNK)
        a = _gen(seed, S_X, c).standard_normal(e - s, dtype=np.float32)
        rows = np.arange(s, e, dtype=np.int64) // N
        a = mu[rows] + sg[rows] * a
        x[s:e] = bf16_bits(a) if dtype == "bf16" else a

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(work, range((M * N + CHUNK - 1) // CHUNK)))
    return {
        "x": x.reshape(M, N),
        "w": normal(seed, S_W, N, dtype, scale=0.1, offset=1.0),
        "b": normal(seed, S_B, N, dtype, scale=0.1),
        "dy": normal(seed, S_DY, M * N, dtype).reshape(M, N),
        "eps": 1e-5, "dtype": dtype,
    }


def rope(B: int = 1, S: int = 32760, H: int = 40, D: int = 128, dtype: str = "bf16",
         theta: float = 10000.0, seed: int = 0) -> dict:
    n = B * S * H * D
    cos, sin = rope_tables(S, D, theta)
    return {
        "q": normal(seed, S_Q, n, dtype).reshape(B, S, H, D),
        "k": normal(seed, S_K, n, dtype).reshape(B, S, H, D),
        "cos": cos, "sin": sin, "dtype": dtype,
    }


def qknorm_rope(B: int = 2, S: int = 76800, H: int = 40, D: int = 128, dtype: str = "bf16",
                theta: float = 10000.0, seed: int = 0, grads: bool = True) -> dict:
    n = B * S * H * D
    cos, sin = rope_tables(S, D, theta)
    d = {
        "q": normal(seed, S_Q, n, dtype).reshape(B, S, H, D),
        "k": normal(seed, S_K, n, dtype).reshape(B, S, H, D),
        "wq": normal(seed, S_WQ, D, dtype, scale=0.1, offset=1.0),
        "wk": normal(seed, S_WK, D, dtype, scale=0.1, offset=1.0),
        "cos": cos, "sin": sin, "eps": 1e-6, "dtype": dtype,
    }
    if grads:
        d["dq_out"] = normal(seed, S_DQ, n, dtype).reshape(B, S, H, D)
        d["dk_out"] = normal(seed, S_DK, n, dtype).reshape(B, S, H, D)
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
