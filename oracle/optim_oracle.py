"""Plain CPU oracle of the optimizer step that follows the training step (Muon + AdamW).

TEST INFRASTRUCTURE ONLY.  Only the tests may import this module.  It shares no code with the CUDA
path and nothing in the product calls it.

What the pages fix ("Introducing nanochat", Pretraining log):
  * the block matrices go to Muon, grouped by shape — at depth 20 eighty 1280×1280 matrices (q, k, v
    and the output projection of every layer, so W_qkv is three separate Muon matrices), twenty
    1280×5120 and twenty 5120×1280 (the MLP);
  * the embedding and the lm-head go to AdamW, whose learning rates are scaled by 1/√(d/768).

What they leave open, and the reading taken here (the published Muon method, restated):
  * Muon keeps a momentum buffer b ← μ·b + g and, with Nesterov, updates along u = g + μ·b;
  * u is orthogonalised by a fixed number of Newton–Schulz steps on X = u/‖u‖_F:
    X ← a·X + (b·A + c·A²)·X with A = X·Xᵀ, coefficients (a, b, c) passed in (the published quintic
    uses (3.4445, −4.7750, 2.0315) for 5 steps); a tall matrix is iterated transposed;
  * the update is W ← W − lr·√max(1, rows/cols)·X;
  * AdamW is the decoupled form: m ← β1·m + (1−β1)·g, v ← β2·v + (1−β2)·g²,
    W ← W·(1 − lr·wd) − lr·m̂/(√v̂ + ε) with m̂ = m/(1−β1^t), v̂ = v/(1−β2^t).
Every hyperparameter is an argument: the pages print none of their values.
"""
from __future__ import annotations

from typing import Dict, Tuple

import numpy as np

NS_QUINTIC = (3.4445, -4.7750, 2.0315)


# ------------------------------------------------------------------------------------------------
# Newton–Schulz orthogonalisation (Muon)
# ------------------------------------------------------------------------------------------------
def newton_schulz(g: np.ndarray, steps: int = 5, coeffs=NS_QUINTIC, eps: float = 1e-7) -> np.ndarray:
    """Approximate the orthogonal polar factor of g: X = g/‖g‖_F, then `steps` times
    X ← a·X + (b·A + c·A·A)·X with A = X·Xᵀ.  A matrix with more rows than columns is iterated as
    its transpose (so A is the smaller Gram matrix) and transposed back."""
    a, b, c = coeffs
    x = np.asarray(g, dtype=np.float64)
    tall = x.shape[0] > x.shape[1]
    if tall:
        x = x.T
    x = x / (np.linalg.norm(x) + eps)
    for _ in range(steps):
        gram = x @ x.T
        x = a * x + (b * gram + c * (gram @ gram)) @ x
    return x.T if tall else x


def newton_schulz_scalar(s: np.ndarray, steps: int = 5, coeffs=NS_QUINTIC) -> np.ndarray:
    """The same iteration on singular values: s ← a·s + b·s³ + c·s⁵ (s already normalised)."""
    a, b, c = coeffs
    s = np.asarray(s, dtype=np.float64)
    for _ in range(steps):
        s = a * s + b * s ** 3 + c * s ** 5
    return s


def muon_update(w: np.ndarray, g: np.ndarray, buf: np.ndarray, lr: float, momentum: float,
                nesterov: bool = True, steps: int = 5, coeffs=NS_QUINTIC) -> Tuple[np.ndarray, np.ndarray]:
    """One Muon step on one matrix: returns (new weight, new momentum buffer)."""
    buf = momentum * buf + g
    u = g + momentum * buf if nesterov else buf
    o = newton_schulz(u, steps, coeffs)
    scale = np.sqrt(max(1.0, w.shape[0] / w.shape[1]))
    return w - lr * scale * o, buf


# ------------------------------------------------------------------------------------------------
# AdamW
# ------------------------------------------------------------------------------------------------
def adamw_update(w: np.ndarray, g: np.ndarray, m: np.ndarray, v: np.ndarray, t: int, lr: float,
                 beta1: float, beta2: float, eps: float, weight_decay: float):
    """One decoupled AdamW step (t counts from 1): returns (new weight, m, v)."""
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    mhat = m / (1.0 - beta1 ** t)
    vhat = v / (1.0 - beta2 ** t)
    w = w * (1.0 - lr * weight_decay) - lr * mhat / (np.sqrt(vhat) + eps)
    return w, m, v


# ------------------------------------------------------------------------------------------------
# the whole optimizer step over the flat parameter packing
# ------------------------------------------------------------------------------------------------
def muon_matrices(cfg) -> Dict[str, Tuple[int, int, int]]:
    """Muon's matrices as (offset into the flat packing, rows, cols): per layer q, k, v (the three
    row blocks of W_qkv), o, fc, proj — the grouping the pages print."""
    d, F, V = cfg.d_model, cfg.d_mlp, cfg.vocab
    # with grouped key/value heads the k and v row blocks of W_qkv have kv_heads·Dh rows
    kv = getattr(cfg, "kv_heads", cfg.n_heads) * cfg.head_dim
    out = {}
    off = V * d
    for l in range(cfg.depth):
        out[f"h{l}.w_q"] = (off, d, d)
        out[f"h{l}.w_k"] = (off + d * d, kv, d)
        out[f"h{l}.w_v"] = (off + d * d + kv * d, kv, d)
        off += (d + 2 * kv) * d
        out[f"h{l}.w_o"] = (off, d, d)
        off += d * d
        out[f"h{l}.w_fc"] = (off, F, d)
        off += F * d
        out[f"h{l}.w_proj"] = (off, d, F)
        off += d * F
    return out


def adamw_tensors(cfg) -> Dict[str, Tuple[int, int, int]]:
    """AdamW's tensors as (offset, rows, cols): the embedding and the lm-head."""
    d, V = cfg.d_model, cfg.vocab
    n = int(sum(a * b for _, (a, b) in cfg.tensor_shapes()))
    return {"wte": (0, V, d), "w_lm": (n - V * d, V, d)}


def optimizer_step(cfg, params: np.ndarray, grads: np.ndarray, state: dict, t: int, hp: dict) -> np.ndarray:
    """Muon on the block matrices, AdamW (learning rates × 1/√(d/768)) on wte and W_lm.
    `state` holds per-tensor buffers and is updated in place; returns the new flat parameters.
    hp: muon_lr, muon_momentum, ns_steps, ns_coeffs, adam_lr_wte, adam_lr_lm, beta1, beta2, eps,
    weight_decay."""
    p = np.array(params, dtype=np.float64, copy=True)
    g = np.asarray(grads, dtype=np.float64)
    for name, (off, r, c) in muon_matrices(cfg).items():
        w = p[off:off + r * c].reshape(r, c)
        buf = state.setdefault(name, np.zeros((r, c)))
        w2, buf2 = muon_update(w, g[off:off + r * c].reshape(r, c), buf, hp["muon_lr"],
                               hp["muon_momentum"], True, hp["ns_steps"], hp["ns_coeffs"])
        p[off:off + r * c] = w2.ravel()
        state[name] = buf2
    scale = 1.0 / np.sqrt(cfg.d_model / 768.0)
    for name, (off, r, c) in adamw_tensors(cfg).items():
        lr = (hp["adam_lr_wte"] if name == "wte" else hp["adam_lr_lm"]) * scale
        m = state.setdefault(name + ".m", np.zeros(r * c))
        v = state.setdefault(name + ".v", np.zeros(r * c))
        w2, m2, v2 = adamw_update(p[off:off + r * c], g[off:off + r * c], m, v, t, lr,
                                  hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"])
        p[off:off + r * c] = w2
        state[name + ".m"], state[name + ".v"] = m2, v2
    return p
