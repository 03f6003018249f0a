"""The synthetic inputs follow their stated recipe (shapes, dtypes, seeds, distributions, the
outlier channels, the correlated case's off-diagonal ratio), on the CPU."""

import math

import numpy as np
import pytest
import torch

import workloads as wl


def test_config_shapes_and_dtypes():
    names = [c.name for c in wl.CONFIGS]
    assert names == ["tiny", "q_proj", "gate_up", "down_proj", "hessian_at_scale"]
    q = wl.CONFIGS[1]
    assert (q.N, q.K, q.T, q.chunk, q.group, q.damp) == (5120, 5120, 8192, 512, 128, 0.01)
    assert q.n_chunks == 16 and q.w_dtype == "bf16" and q.x_dtype == "bf16"
    assert (wl.CONFIGS[2].N, wl.CONFIGS[2].K, wl.CONFIGS[2].T) == (17408, 5120, 65536)
    assert (wl.CONFIGS[3].N, wl.CONFIGS[3].K) == (5120, 17408)
    assert wl.CONFIGS[4].K == 6144 and wl.CONFIGS[4].n_chunks == 512


def test_draws_are_seeded_and_streams_independent():
    cfg = wl.small_config(wl.CONFIGS[1], N=32, K=256, T=1024)
    assert torch.equal(wl.make_weights(cfg), wl.make_weights(cfg))
    assert torch.equal(wl.make_activations(cfg), wl.make_activations(cfg))
    a = wl.make_activation_chunk(cfg, 0)
    b = wl.make_activation_chunk(cfg, 1)
    assert not torch.equal(a, b)
    other = wl.small_config(wl.CONFIGS[1], N=32, K=256, T=1024, seed=99)
    assert not torch.equal(wl.make_weights(cfg), wl.make_weights(other))
    # chunks concatenate to the whole X
    X = wl.make_activations(cfg)
    assert torch.equal(X[:512], a) and torch.equal(X[512:], b)


def test_outlier_channels_are_one_percent_times_twenty():
    cfg = wl.CONFIGS[1]
    s = wl.channel_scales(cfg).double()
    z = torch.exp(torch.randn(cfg.K, generator=wl._gen("cpu", cfg.seed, wl._STREAM_SCALES), dtype=torch.float64))
    ratio = (s / z.float().double()).numpy()
    n_out = int(math.floor(0.01 * cfg.K))
    assert n_out == 51
    assert np.sum(np.isclose(ratio, 20.0, rtol=1e-6)) == n_out
    assert np.sum(np.isclose(ratio, 1.0, rtol=1e-6)) == cfg.K - n_out


def test_weight_distributions():
    tiny = wl.CONFIGS[0]
    W = wl.make_weights(tiny).double()
    assert W.dtype == torch.float64 and W.abs().max() <= 1.0
    assert abs(float(W.mean())) < 0.05 and abs(float(W.var()) - 1.0 / 3.0) < 0.03
    q = wl.small_config(wl.CONFIGS[1], N=256, K=512, T=8)
    Wq = wl.make_weights(q)
    assert Wq.dtype == torch.bfloat16
    assert float(Wq.float().std()) == pytest.approx(0.02, rel=0.02)
    d = wl.small_config(wl.CONFIGS[3], N=256, K=512, T=8)
    assert float(wl.make_weights(d).float().std()) == pytest.approx(0.015, rel=0.02)


def test_activations_bf16_are_round_to_nearest_even_of_fp32():
    cfg = wl.small_config(wl.CONFIGS[1], N=1, K=64, T=64)
    x = wl.make_activations(cfg)
    assert x.dtype == torch.bfloat16
    s = wl.channel_scales(cfg, 64)
    g = wl._gen("cpu", cfg.seed, wl._STREAM_X, 0)
    ref = (torch.randn((64, 64), generator=g, dtype=torch.float32) * s[None, :]).to(torch.bfloat16)
    assert torch.equal(x, ref)


def test_down_proj_activations_are_non_negative():
    cfg = wl.small_config(wl.CONFIGS[3], N=1, K=128, T=256)
    assert float(wl.make_activations(cfg).float().min()) >= 0.0


def test_correlated_case_off_diagonal_ratio():
    cfg = wl.correlated_config(8, 256, T=4096)
    X = wl.make_activations(cfg).double().numpy()
    H = X.T @ X
    off = H[~np.eye(256, dtype=bool)]
    ratio = np.sqrt(np.mean(off ** 2)) / np.mean(np.diag(H))
    assert ratio == pytest.approx(0.79, abs=0.06)
