"""Seeded synthetic inputs for the quantisation path: weights W, calibration activations X.

This module only draws random numbers with the shapes and distributions of the layer
configurations below; it holds none of the method's arithmetic (no Hessian, no
factorisation, no quantiser).  Both the CUDA path and the oracle consume the same bytes
made here.

Recipe (all draws from torch's seeded generators, fp32, then cast with round-to-nearest-
even when the dtype is bf16):

* tiny layer: W fp32 [64, 128] ~ U(-1, 1); X fp32 [512, 128], X[t, k] = N(0,1) * s_k with
  s_k = exp(0.5 * N(0,1)); group 32.
* q_proj-like: W bf16 [5120, 5120] ~ N(0, 0.02^2); X bf16 [8192, 5120] as 16 chunks of
  512, X[t, k] = N(0,1) * s_k, s_k = exp(N(0,1)) and floor(1% * K) outlier channels with
  s_k * 20; group 128.
* gate/up-like: W bf16 [17408, 5120] ~ N(0, 0.02^2); X bf16 [65536, 5120] as above.
* down_proj-like: W bf16 [5120, 17408] ~ N(0, 0.015^2); X bf16 [65536, 17408],
  X[t, k] = |N(0,1)| * s_k with s_k = exp(N(0,1)).
* Hessian-at-scale: 512 chunks of X bf16 [8192, 6144] with the q_proj distribution.
* correlated (a parity case, not a benchmark layer): X[t, k] = sum_r w_r z[t, r] a[r, k]
  + sigma * n[t, k] with w = (1, 0.3, 0.2, 0.1), a, z, n ~ N(0,1) and sigma^2 = 0.132, so
  that the off-diagonal RMS of X^T X is about 0.79 of its mean diagonal.

Seeds: each config has a seed (its index); every stream (W, channel scales, outlier pick,
X chunk c, ...) gets its own generator seeded from (seed, stream id, chunk).
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    index: int
    N: int            # output features (rows of W); 0 for the Hessian-only pipeline
    K: int            # input features (columns of W, channels of X)
    T: int            # calibration tokens
    chunk: int        # tokens per generated chunk
    group: int        # quantisation group size along K
    damp: float       # damping, relative to mean(diag H)
    w_dtype: str      # "f32" | "bf16"
    x_dtype: str      # "f32" | "bf16"
    w_dist: str       # "uniform1" | "normal"
    w_std: float
    x_dist: str       # "lognormal0.5" | "lognormal1_outliers" | "halfnormal_lognormal1" | "correlated"
    use_imatrix: bool  # qerr weighted by diag(H)/T
    seed: int

    @property
    def n_chunks(self) -> int:
        return (self.T + self.chunk - 1) // self.chunk


CONFIGS = [
    LayerConfig("tiny", 0, 64, 128, 512, 512, 32, 0.01, "f32", "f32", "uniform1", 1.0,
                "lognormal0.5", False, 0),
    LayerConfig("q_proj", 1, 5120, 5120, 8192, 512, 128, 0.01, "bf16", "bf16", "normal", 0.02,
                "lognormal1_outliers", False, 1),
    LayerConfig("gate_up", 2, 17408, 5120, 65536, 8192, 128, 0.01, "bf16", "bf16", "normal", 0.02,
                "lognormal1_outliers", True, 2),
    LayerConfig("down_proj", 3, 5120, 17408, 65536, 8192, 128, 0.01, "bf16", "bf16", "normal", 0.015,
                "halfnormal_lognormal1", False, 3),
    LayerConfig("hessian_at_scale", 4, 0, 6144, 4194304, 8192, 128, 0.01, "bf16", "bf16", "normal", 0.0,
                "lognormal1_outliers", False, 4),
]

_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}

_STREAM_W = 1
_STREAM_SCALES = 2
_STREAM_OUTLIERS = 3
_STREAM_X = 1000
_STREAM_LATENT = 7


def _seed(seed: int, stream: int, chunk: int = 0) -> int:
    return (seed * 1_000_003 + stream * 65_537 + chunk) & 0x7FFF_FFFF_FFFF


def _gen(device, seed: int, stream: int, chunk: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(seed, stream, chunk))
    return g


def torch_dtype(name: str) -> torch.dtype:
    return _TORCH_DTYPE[name]


def channel_scales(cfg: LayerConfig, K: int | None = None) -> torch.Tensor:
    """Per-channel activation scales s_k (fp32, CPU)."""
    K = cfg.K if K is None else K
    g = _gen("cpu", cfg.seed, _STREAM_SCALES)
    z = torch.randn(K, generator=g, dtype=torch.float64)
    if cfg.x_dist == "lognormal0.5":
        s = torch.exp(0.5 * z)
    elif cfg.x_dist in ("lognormal1_outliers", "halfnormal_lognormal1"):
        s = torch.exp(z)
    elif cfg.x_dist == "correlated":
        s = torch.ones(K, dtype=torch.float64)
    else:
        raise ValueError(cfg.x_dist)
    if cfg.x_dist == "lognormal1_outliers":
        n_out = int(math.floor(0.01 * K))
        go = _gen("cpu", cfg.seed, _STREAM_OUTLIERS)
        pick = torch.randperm(K, generator=go)[:n_out]
        s[pick] *= 20.0
    return s.to(torch.float32)


def make_weights(cfg: LayerConfig, device="cpu", N: int | None = None, K: int | None = None) -> torch.Tensor:
    """W [N, K] in cfg.w_dtype."""
    N = cfg.N if N is None else N
    K = cfg.K if K is None else K
    g = _gen(device, cfg.seed, _STREAM_W)
    if cfg.w_dist == "uniform1":
        w = torch.rand((N, K), generator=g, device=device, dtype=torch.float32) * 2.0 - 1.0
    elif cfg.w_dist == "normal":
        w = torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * cfg.w_std
    else:
        raise ValueError(cfg.w_dist)
    return w.to(_TORCH_DTYPE[cfg.w_dtype])


def make_activation_chunk(cfg: LayerConfig, c: int, device="cpu", scales: torch.Tensor | None = None,
                          rows: int | None = None, K: int | None = None) -> torch.Tensor:
    """Chunk c of X: [rows (default cfg.chunk, the last chunk may be short), K] in cfg.x_dtype."""
    K = cfg.K if K is None else K
    if rows is None:
        rows = min(cfg.chunk, cfg.T - c * cfg.chunk)
    if scales is None:
        scales = channel_scales(cfg, K)
    g = _gen(device, cfg.seed, _STREAM_X, c)
    if cfg.x_dist == "correlated":
        w = torch.tensor([1.0, 0.3, 0.2, 0.1], device=device)
        ga = _gen(device, cfg.seed, _STREAM_LATENT)
        a = torch.randn((4, K), generator=ga, device=device, dtype=torch.float32)
        z = torch.randn((rows, 4), generator=g, device=device, dtype=torch.float32)
        n = torch.randn((rows, K), generator=g, device=device, dtype=torch.float32)
        x = (z * w) @ a + math.sqrt(0.132) * n
    else:
        x = torch.randn((rows, K), generator=g, device=device, dtype=torch.float32)
        if cfg.x_dist == "halfnormal_lognormal1":
            x = x.abs()
        x = x * scales.to(device)[None, :]
    return x.to(_TORCH_DTYPE[cfg.x_dtype])


def make_activations(cfg: LayerConfig, device="cpu", T: int | None = None, K: int | None = None) -> torch.Tensor:
    """All of X [T, K] (chunks concatenated); only for configs that fit in memory."""
    K = cfg.K if K is None else K
    T = cfg.T if T is None else T
    scales = channel_scales(cfg, K)
    parts = []
    c = 0
    done = 0
    while done < T:
        rows = min(cfg.chunk, T - done)
        parts.append(make_activation_chunk(cfg, c, device, scales, rows=rows, K=K))
        done += rows
        c += 1
    return torch.cat(parts, 0)


def correlated_config(N: int, K: int, T: int, group: int = 128, seed: int = 11) -> LayerConfig:
    """A layer whose activations share a low-rank latent factor (strong GPTQ compensation)."""
    return LayerConfig("correlated", -1, N, K, T, T, group, 0.01, "f32", "f32", "uniform1", 1.0,
                       "correlated", False, seed)


def small_config(base: LayerConfig, N: int, K: int, T: int, group: int | None = None,
                 seed: int | None = None) -> LayerConfig:
    """The distribution of `base` at other sizes (ragged and edge-case parity runs)."""
    return dataclasses.replace(base, N=N, K=K, T=T, chunk=max(1, min(base.chunk, T)),
                               group=base.group if group is None else group,
                               seed=base.seed if seed is None else seed)
