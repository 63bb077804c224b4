"""Seeded input generator: determinism, prefix property, distributions, bf16 rounding (CPU)."""
import numpy as np
import torch

from transformer_norm_rope_b200 import workloads as wl


def test_bf16_rounding_matches_torch():
    a = np.random.default_rng(0).standard_normal(100_000).astype(np.float32) * 100
    a[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.0, 65504.0]  # ties go to even
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(wl.bf16_bits(a), ref)
    np.testing.assert_array_equal(wl.bf16_to_f32(ref), torch.from_numpy(a).to(torch.bfloat16).float().numpy())


def test_streams_are_deterministic_and_prefix_stable():
    a = wl.normal(0, wl.S_X, 3 * wl.CHUNK + 17)
    b = wl.normal(0, wl.S_X, wl.CHUNK + 5)
    np.testing.assert_array_equal(a[: b.size], b)
    c = wl.normal(1, wl.S_X, 100)
    assert not np.array_equal(a[:100], c)
    d = wl.normal(0, wl.S_DY, 100)
    assert not np.array_equal(a[:100], d)


def test_rmsnorm_recipe():
    d = wl.rmsnorm(M=1000, N=256)
    x = wl.bf16_to_f32(d["x"])
    rms = np.sqrt((x.astype(np.float64) ** 2).mean(1))
    big = rms > 10
    assert big.sum() == 10  # floor(1% of 1000) rows scaled by 50
    np.testing.assert_allclose(rms[big].mean(), 50, rtol=0.05)
    np.testing.assert_allclose(rms[~big].mean(), 1, rtol=0.05)
    w = wl.bf16_to_f32(d["w"])
    assert abs(w.mean() - 1) < 0.03 and abs(w.std() - 0.1) < 0.02
    g = wl.rmsnorm(M=10, N=256, gemma=True)
    assert abs(wl.bf16_to_f32(g["w"]).mean()) < 0.03


def test_layernorm_recipe():
    d = wl.layernorm(M=400, N=512)
    x = wl.bf16_to_f32(d["x"]).astype(np.float64)
    mu, sd = x.mean(1), x.std(1)
    assert mu.min() > -2.3 and mu.max() < 2.3 and mu.max() - mu.min() > 3
    assert sd.min() > 0.4 and sd.max() < 3.3
    assert abs(wl.bf16_to_f32(d["b"]).std() - 0.1) < 0.02


def test_rope_tables():
    cos, sin = wl.rope_tables(300, 128)
    assert cos.shape == (300, 64) and cos.dtype == np.float32
    assert np.all(cos[0] == 1) and np.all(sin[0] == 0)
    # row p, pair i: angle p * 10000^(-2i/128); pair 0 has frequency 1
    np.testing.assert_allclose(cos[:, 0], np.cos(np.arange(300)), atol=1e-7)
    np.testing.assert_allclose(sin[7, 32], np.sin(7 * 10000 ** -0.5), atol=1e-7)


def test_qknorm_recipe_shapes():
    d = wl.qknorm_rope(B=2, S=16, H=4, D=128)
    assert d["q"].shape == (2, 16, 4, 128) and d["q"].dtype == np.uint16
    assert d["dq_out"].shape == d["q"].shape and d["wq"].shape == (128,)
    assert not np.array_equal(d["q"], d["k"])


def test_norm_linear_recipe():
    d = wl.norm_linear(M=64, N=96, K=512, seed=3)
    assert d["x"].shape == (64, 512) and d["W"].shape == (96, 512) and d["bias"].shape == (96,)
    assert all(d[k].dtype == np.uint16 for k in ("x", "g", "beta", "W", "bias"))  # bf16 bit patterns
    W = wl.bf16_to_f32(d["W"]).astype(np.float64)
    assert abs(W.std() * np.sqrt(512) - 1) < 0.05  # W ~ N(0, 1/K): unit-scale outputs
    g = wl.bf16_to_f32(d["g"])
    assert abs(g.mean() - 1) < 0.03 and abs(g.std() - 0.1) < 0.02
    # the rows are the LayerNorm recipe's rows with the same seed, the layer weights their own streams
    np.testing.assert_array_equal(d["x"], wl.layernorm(M=64, N=512, dtype="bf16", seed=3)["x"])
    e = wl.norm_linear(M=8, N=96, K=512, seed=3)
    np.testing.assert_array_equal(e["W"], d["W"])  # weights do not depend on the row count
    assert not np.array_equal(wl.norm_linear(M=8, N=96, K=512, seed=4)["W"], d["W"])


def test_row_and_token_ranges_are_slices_of_the_whole():
    # ranges cross chunk boundaries (CHUNK = 4 Mi elements) and keep the global outlier rows,
    # row statistics and table positions
    M, N = 1000, 5120
    full = wl.rmsnorm(M=M, N=N, seed=2)
    part = wl.rmsnorm(M=M, N=N, seed=2, rows=(811, 997))
    np.testing.assert_array_equal(part["x"], full["x"][811:997])
    np.testing.assert_array_equal(part["dy"], full["dy"][811:997])
    np.testing.assert_array_equal(part["w"], full["w"])
    full = wl.layernorm(M=900, N=5120, seed=1)
    part = wl.layernorm(M=900, N=5120, seed=1, rows=(3, 850))
    np.testing.assert_array_equal(part["x"], full["x"][3:850])
    np.testing.assert_array_equal(part["dy"], full["dy"][3:850])
    full = wl.rope(B=2, S=900, H=40, D=128, seed=5)
    part = wl.rope(B=2, S=900, H=40, D=128, seed=5, tokens=(450, 900))
    for k in ("q", "k"):
        np.testing.assert_array_equal(part[k], full[k][:, 450:900])
    for k in ("cos", "sin"):
        np.testing.assert_array_equal(part[k], full[k][450:900])
    full = wl.qknorm_rope(B=2, S=900, H=40, D=128, seed=6)
    part = wl.qknorm_rope(B=2, S=900, H=40, D=128, seed=6, tokens=(1, 420))
    for k in ("q", "k", "dq_out", "dk_out"):
        np.testing.assert_array_equal(part[k], full[k][:, 1:420])
    for k in ("cos", "sin", "wq", "wk"):
        np.testing.assert_array_equal(part[k], full[k][1:420] if k in ("cos", "sin") else full[k])
