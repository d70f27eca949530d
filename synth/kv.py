"""Synthetic rank-structured KV caches shaped like the JoLT paper's model caches.

The JoLT abstract ("A JoLT for the KV Cache", arXiv 2607.12550v2, Abstract) evaluates
on real Mistral-7B-v0.3 (GQA) and LLaMA-2-13B (MHA) caches, which are not available
here. These generators stand in for them with the same shapes: every layer's K (and V)
tensor X in R^{H x T x D} is

    X[h] = U diag(S_h) V^T + sigma * N(0, 1)

with U (T x K) and V (D x K) Gaussian with unit-norm columns, S_h[k] = exp(-k / rho)
* (0.5 + u[h, k]), u ~ U(0, 1) drawn per head and component, and, for the tensors that
carry them, 4 fixed feature channels scaled by 8 after the noise is added. rho is 12 for
the single-layer case and U[8, 16] per layer otherwise (shared by that layer's K and V).

Values are rounded to bf16 (round to nearest even) for the bf16 workloads, so the oracle
and the CUDA path see the same tensor. Random draws come from numpy PCG64 streams keyed
by (config seed, layer, kind, sequence); the torch variant uses the same recipe with
torch's device generator for the multi-GB workloads and is never compared draw-for-draw
with the numpy one (the oracle always takes the tensor the GPU actually used).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np

KIND_K, KIND_V = 0, 1


@dataclass(frozen=True)
class KVConfig:
    name: str
    layers: int
    heads: int
    tokens: int
    head_dim: int
    dtype: str                 # "bf16" or "f32"
    has_v: bool
    rank: int                  # K of the generator
    rho: float | None          # fixed decay, or None for U[8,16] per layer
    sigma: float
    outliers_on: tuple         # kinds whose tensor gets the 4 outlier channels
    groups: int
    split_kv: bool
    ratios: tuple              # compression ratios N: budget = bf16 bytes / N
    encoders: tuple            # "exact" and/or "sketch"
    bits: tuple = tuple(range(9))
    batch: int = 1
    seed: int = 0
    extra: dict = field(default_factory=dict)


def _mk():
    base = dict(head_dim=128, sigma=0.02, outliers_on=(KIND_K,))
    cfgs = [
        KVConfig(name="c0_single_layer_k_t256_f32", layers=1, heads=8, tokens=256, dtype="f32",
                 has_v=False, rank=64, rho=12.0, groups=1, split_kv=False, ratios=(2.0,),
                 encoders=("exact",), seed=1000, **base),
        KVConfig(name="c1_mistral7b_gqa_l32_h8_t1024", layers=32, heads=8, tokens=1024, dtype="bf16",
                 has_v=True, rank=64, rho=None, groups=4, split_kv=True, ratios=(2.0, 3.0),
                 encoders=("sketch", "exact"), seed=1001, **base),
        KVConfig(name="c2_llama2_13b_mha_l40_h40_t4096", layers=40, heads=40, tokens=4096, dtype="bf16",
                 has_v=True, rank=96, rho=None, groups=5, split_kv=True, ratios=(2.0,),
                 encoders=("sketch",), seed=1002, head_dim=128, sigma=0.03, outliers_on=(KIND_K,)),
        KVConfig(name="c3_long_gqa_l32_h8_t32768", layers=32, heads=8, tokens=32768, dtype="bf16",
                 has_v=True, rank=256, rho=None, groups=4, split_kv=True, ratios=(3.0,),
                 encoders=("sketch",), bits=(1, 2, 3, 4), seed=1003, **base),
        KVConfig(name="c4_decode_sweep_16seq_l32_h8_t8192", layers=32, heads=8, tokens=8192, dtype="bf16",
                 has_v=True, rank=64, rho=None, groups=4, split_kv=True, ratios=(2.0, 2.5, 3.0),
                 encoders=("sketch",), batch=16, seed=1004, **base),
    ]
    return cfgs


CONFIGS = _mk()


def config(idx: int, **overrides) -> KVConfig:
    """Workload `idx` (0..4), optionally with fields replaced (e.g. a smaller `layers`)."""
    c = CONFIGS[idx]
    return replace(c, **overrides) if overrides else c


def bf16_bytes(cfg: KVConfig, kinds: int | None = None) -> int:
    """Bytes of one sequence's cache held in bf16 (the reference size the ratios divide)."""
    k = kinds if kinds is not None else (2 if cfg.has_v else 1)
    return cfg.layers * cfg.heads * cfg.tokens * cfg.head_dim * 2 * k


def _cfg_rng(cfg: KVConfig):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([cfg.seed])))


def _per_config_draws(cfg: KVConfig):
    """Outlier channels (once per config) and the per-layer decay rates."""
    rng = _cfg_rng(cfg)
    outl = np.sort(rng.choice(cfg.head_dim, 4, replace=False))
    if cfg.rho is not None:
        rho = np.full(cfg.layers, float(cfg.rho))
    else:
        rho = rng.uniform(8.0, 16.0, cfg.layers)
    return outl, rho


def _round_storage(x64: np.ndarray, dtype: str) -> np.ndarray:
    """Input rounding: float64 -> float32 (RNE) -> bf16 (RNE) for bf16 workloads."""
    x32 = x64.astype(np.float32)
    if dtype == "f32":
        return x32
    import torch
    t = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float32)
    return t.numpy()


def gen_layer_tensor(cfg: KVConfig, layer: int, kind: int, seq: int = 0) -> np.ndarray:
    """One layer-tensor X[h, t, d] as float32 holding storage-dtype values."""
    outl, rho = _per_config_draws(cfg)
    H, T, D, K = cfg.heads, cfg.tokens, cfg.head_dim, cfg.rank
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([cfg.seed, layer, kind, seq])))
    U = rng.standard_normal((T, K))
    U /= np.linalg.norm(U, axis=0, keepdims=True)
    V = rng.standard_normal((D, K))
    V /= np.linalg.norm(V, axis=0, keepdims=True)
    u = rng.uniform(0.0, 1.0, (H, K))
    S = np.exp(-np.arange(K) / rho[layer])[None, :] * (0.5 + u)          # H x K
    E = rng.standard_normal((H, T, D)) * cfg.sigma
    X = np.einsum("tk,hk,dk->htd", U, S, V, optimize=True) + E
    if kind in cfg.outliers_on:
        X[:, :, outl] *= 8.0
    return _round_storage(X, cfg.dtype)


def gen_cache_numpy(cfg: KVConfig, seq: int = 0, layers: range | None = None):
    """Whole cache as float32 arrays K, V of shape [L][H][T][D] (V is None without V)."""
    ls = range(cfg.layers) if layers is None else layers
    K = np.stack([gen_layer_tensor(cfg, l, KIND_K, seq) for l in ls])
    V = np.stack([gen_layer_tensor(cfg, l, KIND_V, seq) for l in ls]) if cfg.has_v else None
    return K, V


def gen_cache_torch(cfg: KVConfig, device, seq: int = 0):
    """Same recipe drawn with torch's generator on `device`, for the multi-GB workloads.

    Returns K, V as [L][H][T][D] tensors in the workload dtype (bf16 or float32).
    """
    import torch
    outl, rho = _per_config_draws(cfg)
    H, T, D, K, L = cfg.heads, cfg.tokens, cfg.head_dim, cfg.rank, cfg.layers
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    kinds = (KIND_K, KIND_V) if cfg.has_v else (KIND_K,)
    out = {k: torch.empty((L, H, T, D), dtype=dt, device=device) for k in kinds}
    outl_t = torch.as_tensor(outl, device=device)
    g = torch.Generator(device=device)
    for l in range(L):
        for k in kinds:
            g.manual_seed(((cfg.seed * 1_000_003 + l) * 7 + k) * 1_000_033 + seq)
            U = torch.randn((T, K), generator=g, device=device, dtype=torch.float32)
            U /= U.norm(dim=0, keepdim=True)
            V = torch.randn((D, K), generator=g, device=device, dtype=torch.float32)
            V /= V.norm(dim=0, keepdim=True)
            u = torch.rand((H, K), generator=g, device=device, dtype=torch.float32)
            S = torch.exp(-torch.arange(K, device=device, dtype=torch.float32) / float(rho[l]))[None] * (0.5 + u)
            X = torch.einsum("tk,hk,dk->htd", U, S, V)
            X += torch.randn((H, T, D), generator=g, device=device, dtype=torch.float32) * cfg.sigma
            if k in cfg.outliers_on:
                X[:, :, outl_t] *= 8.0
            out[k][l].copy_(X.to(dt))
    return out[KIND_K], out.get(KIND_V)


def budget_bytes(cfg: KVConfig, ratio: float) -> int:
    """Whole-stream byte budget for one sequence at compression ratio `ratio`."""
    return int(math.floor(bf16_bytes(cfg) / ratio))
