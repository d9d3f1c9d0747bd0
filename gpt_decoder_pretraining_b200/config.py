"""Model configurations, per-layer window patterns and the FLOP/parameter arithmetic.

The architecture is the nanochat GPT described in "nanochat User Guide" §10 (How It Works):
rotary embeddings, QK-norm, ReLU² MLPs, untied embedding/unembedding and a sliding-window
pattern.  "Introducing nanochat" (Pretraining section) states there are no biases and no norm
parameters, and prints the parameter count and FLOPs-per-token for the d20 model; the functions
below reproduce those printed figures exactly:

  params        = 2·V·d + L·(3d·d + d·d + F·d + d·F)           (= 2·V·d + 12·L·d² at F = 4d)
  flops / token = 6·(params − V·d) + 12·H·Dh·Σ_l T_eff(l)

with T_eff(l) = min(window_l, T).  The pages' formula predates windows and uses T for every layer;
using min(w, T) keeps the skipped work of a sliding-window layer out of the credited FLOPs.

This module is host-side bookkeeping only; it holds no step arithmetic.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence

DTYPE_BF16 = 0
DTYPE_F32 = 1

B200_DENSE_BF16_PEAK = 2.25e15  # nominal dense bf16 FLOP/s of one B200


def window_pattern(pattern: str, depth: int, short_window: int, seq_len: int) -> List[int]:
    """Expand a window pattern like "SSSL" over `depth` layers.

    Layer l uses pattern[l % len(pattern)]; 'L' is full causal attention (encoded as 0), 'S' is a
    sliding window of `short_window` keys including the query itself.  The last layer is always
    full ('L'), as the sliding-window pattern of nanochat keeps the final layer global.
    """
    pattern = pattern.upper()
    if not pattern or any(c not in "SL" for c in pattern):
        raise ValueError(f"bad window pattern {pattern!r}")
    out = []
    for l in range(depth):
        c = pattern[l % len(pattern)]
        if l == depth - 1:
            c = "L"
        out.append(0 if c == "L" else int(short_window))
    return out


@dataclass
class GptConfig:
    name: str
    depth: int
    d_model: int
    n_heads: int
    head_dim: int
    d_mlp: int
    vocab: int
    seq_len: int
    batch: int
    windows: List[int] = field(default_factory=list)  # per layer; 0 or >= seq_len = full causal
    param_dtype: int = DTYPE_BF16
    token_dist: str = "uniform"  # "uniform" or "zipf1.1"
    n_kv_heads: int = 0  # key/value heads of grouped-query attention; 0 = n_heads

    def __post_init__(self):
        if not self.windows:
            self.windows = [0] * self.depth
        if len(self.windows) != self.depth:
            raise ValueError("windows must have one entry per layer")
        if self.n_heads * self.head_dim != self.d_model:
            raise ValueError("n_heads * head_dim must equal d_model")
        if self.n_kv_heads and (self.n_kv_heads < 0 or self.n_heads % self.n_kv_heads):
            raise ValueError("n_heads must be a multiple of n_kv_heads")

    @property
    def kv_heads(self) -> int:
        return self.n_kv_heads if self.n_kv_heads > 0 else self.n_heads

    # ---- shapes ---------------------------------------------------------------------------
    @property
    def tokens(self) -> int:
        return self.batch * self.seq_len

    def effective_window(self, l: int) -> int:
        w = self.windows[l]
        return self.seq_len if (w <= 0 or w >= self.seq_len) else w

    def tensor_shapes(self):
        """(name, shape) in packing order: wte, per layer qkv/o/fc/proj, lm_head."""
        d, F, V = self.d_model, self.d_mlp, self.vocab
        shapes = [("wte", (V, d))]
        qkv = d + 2 * self.kv_heads * self.head_dim
        for l in range(self.depth):
            shapes += [
                (f"h{l}.w_qkv", (qkv, d)),
                (f"h{l}.w_o", (d, d)),
                (f"h{l}.w_fc", (F, d)),
                (f"h{l}.w_proj", (d, F)),
            ]
        shapes.append(("w_lm", (V, d)))
        return shapes

    # ---- counting (nanochat "Introducing nanochat", Pretraining log) -------------------------
    @property
    def n_params(self) -> int:
        n = 0
        for _, (a, b) in self.tensor_shapes():
            n += a * b
        return n

    def flops_per_token(self) -> int:
        """6·(N − V·d) + 12·H·Dh·Σ_l min(w_l, T): the pages' convention with windowed layers."""
        attn = sum(12 * self.n_heads * self.head_dim * self.effective_window(l) for l in range(self.depth))
        return 6 * (self.n_params - self.vocab * self.d_model) + attn

    def flops_per_step(self) -> int:
        return self.flops_per_token() * self.tokens

    def attention_executed_flops(self) -> float:
        """Causal-algorithmic attention FLOPs of one fwd+bwd (QKᵀ and PV, fwd ×1 + bwd ×2).

        Counts only the (query, key) pairs the mask keeps: Σ_t min(t+1, w) per head per row.
        """
        T = self.seq_len
        total = 0.0
        for l in range(self.depth):
            w = self.effective_window(l)
            keys = sum(min(t + 1, w) for t in range(T))
            total += 4.0 * self.head_dim * keys * self.n_heads * self.batch * 3  # fwd + 2x bwd
        return total

    def window_array(self) -> List[int]:
        return list(self.windows)


def _cfg(name, depth, d, heads, hd, F, V, T, B, windows=None, param_dtype=DTYPE_BF16, token_dist="uniform"):
    return GptConfig(name, depth, d, heads, hd, F, V, T, B, windows or [0] * depth, param_dtype, token_dist)


def preset(name: str) -> GptConfig:
    """Named configurations of the training step this library is measured on."""
    name = name.lower()
    if name == "smoke":
        return _cfg("smoke", 2, 64, 2, 32, 256, 2048, 128, 1, param_dtype=DTYPE_F32)
    if name == "d12":
        return _cfg("d12", 12, 768, 6, 128, 3072, 32768, 2048, 16)
    if name == "d20":
        return _cfg("d20", 20, 1280, 10, 128, 5120, 65536, 2048, 16,
                    windows=window_pattern("SSSL", 20, 1024, 2048))
    if name == "d24":
        return _cfg("d24", 24, 1536, 12, 128, 6144, 32768, 2048, 16, token_dist="zipf1.1")
    raise KeyError(name)


PRESETS = ("smoke", "d12", "d20", "d24")


def custom(depth: int, d_model: int, head_dim: int, vocab: int, seq_len: int, batch: int,
           windows: Optional[Sequence[int]] = None, d_mlp: Optional[int] = None,
           param_dtype: int = DTYPE_BF16, token_dist: str = "uniform", name: str = "custom",
           n_kv_heads: int = 0) -> GptConfig:
    """A config with nanochat's proportions (F = 4d) unless d_mlp is given."""
    return GptConfig(name, depth, d_model, d_model // head_dim, head_dim, d_mlp or 4 * d_model, vocab,
                     seq_len, batch, list(windows) if windows is not None else [0] * depth,
                     param_dtype, token_dist, n_kv_heads)
