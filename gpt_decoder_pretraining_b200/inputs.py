"""Seeded synthetic inputs shared by the CUDA path, its tests, the benchmark and the oracle.

This module draws random numbers and rounds them to bf16; it holds none of the training step's
arithmetic.  Recipe:

* parameters: one flat buffer in packing order, N(0, 0.02²) from NumPy PCG64(seed 0), rounded to
  bf16 (round to nearest even) unless the config keeps fp32 parameters;
* token streams: PCG64(seed 1); for every row T+1 ids are drawn, tokens = ids[:T] and
  targets = ids[1:] (next-token prediction);  ids are uniform on [0, V) or a bounded Zipf(1.1)
  law P(id = k−1) ∝ k^−1.1, k = 1..V, drawn by inverse CDF (hot ids are the low ids);
* attention-only inputs: PCG64(seed 2), q, k, v ~ N(0, 1) in [B, H, T, Dh], rounded to bf16.

The text corpora the pages train on are not available; synthetic ids with the same vocabulary
size stand in for them (GEMM and attention cost do not depend on the ids).
"""
from __future__ import annotations

import numpy as np

PARAM_SEED = 0
TOKEN_SEED = 1
ATTN_SEED = 2
INIT_STD = 0.02


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), returned as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of float32 values that are already bf16-exact, as uint16."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def make_params(n_params: int, keep_fp32: bool = False, seed: int = PARAM_SEED, std: float = INIT_STD) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    p = rng.standard_normal(n_params, dtype=np.float32) * np.float32(std)
    return p if keep_fp32 else round_to_bf16(p)


def _zipf_ids(rng, n: int, vocab: int, s: float = 1.1) -> np.ndarray:
    k = np.arange(1, vocab + 1, dtype=np.float64)
    w = k ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(n)
    ids = np.searchsorted(cdf, u, side="right")
    return np.minimum(ids, vocab - 1).astype(np.int32)


def make_tokens(batch: int, seq_len: int, vocab: int, dist: str = "uniform", seed: int = TOKEN_SEED):
    """Return (tokens, targets), both int32 [batch, seq_len]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n = batch * (seq_len + 1)
    if dist == "uniform":
        ids = rng.integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)
    elif dist == "zipf1.1":
        ids = _zipf_ids(rng, n, vocab, 1.1)
    else:
        raise ValueError(dist)
    ids = ids.reshape(batch, seq_len + 1)
    return np.ascontiguousarray(ids[:, :-1]), np.ascontiguousarray(ids[:, 1:])


def make_attention_inputs(batch: int, heads: int, seq_len: int, head_dim: int, seed: int = ATTN_SEED):
    """q, k, v ~ N(0,1) rounded to bf16, float32 arrays [B, H, T, Dh]; plus dO of the same law."""
    rng = np.random.Generator(np.random.PCG64(seed))
    shape = (batch, heads, seq_len, head_dim)
    q, k, v, do = (round_to_bf16(rng.standard_normal(shape, dtype=np.float32)) for _ in range(4))
    return q, k, v, do


def make_config_inputs(cfg, seed_params: int = PARAM_SEED, seed_tokens: int = TOKEN_SEED):
    """Params (flat float32, bf16-exact unless cfg keeps fp32), tokens, targets for a GptConfig."""
    from .config import DTYPE_F32
    params = make_params(cfg.n_params, keep_fp32=(cfg.param_dtype == DTYPE_F32), seed=seed_params)
    tokens, targets = make_tokens(cfg.batch, cfg.seq_len, cfg.vocab, cfg.token_dist, seed=seed_tokens)
    return params, tokens, targets
