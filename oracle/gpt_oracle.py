"""Plain CPU oracle of one GPT training step: forward, loss, and backward to parameter gradients.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline may import this module.  It shares no code with the CUDA path (it does not import the
``gpt_decoder_pretraining_b200`` package) and nothing in the product calls it.

What it computes (the nanochat architecture):
  * "nanochat User Guide" §10 How It Works: rotary positional embeddings, QK-norm, ReLU² MLPs,
    untied embedding/unembedding weights, a sliding-window attention pattern;
  * "Introducing nanochat", Pretraining section: no biases and no RMSNorm parameters; dims
    d = 1280, 10 heads of 128 at depth 20 (printed log);
  * "supa beginna nanochat" (discussion 677), Troubleshooting: the loss is
    F.cross_entropy(ignore_index=-1, reduction='mean');
  * the block order (pre-norm, QKV, RoPE + QK-norm, causal/window attention, output projection,
    second norm, 4× ReLU² MLP; final norm, lm-head, softmax cross-entropy) fixed by the
    step's specification.

Readings of points the pages leave open (each one stated where it is used):
  eps = 1e-6 inside RMSNorm and QK-norm; no norm right after the embedding; RoPE base 10000 with
  half-split pairs (i, i + Dh/2), angle t·10000^(−2i/Dh), (a, b) → (a cos − b sin, a sin + b cos),
  positions 0..T−1 per row; scores scaled by 1/√Dh; a window w keeps keys j ∈ [t−w+1, t]
  (w ≤ 0 or w ≥ T is full causal); targets equal to −1 are ignored and the loss is the mean over
  the others; when no target is valid the loss and every gradient are 0.

Everything is written as the textbook definition, one sequence at a time, with NumPy matmuls as
the only library primitive.  ``dtype`` selects float64 (finite-difference checks) or float32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, List, Optional

import numpy as np

EPS = 1e-6
ROPE_BASE = 10000.0


@dataclass
class OracleConfig:
    depth: int
    d_model: int
    n_heads: int
    head_dim: int
    d_mlp: int
    vocab: int
    seq_len: int
    batch: int
    windows: List[int]
    n_kv_heads: int = 0  # key/value heads (grouped-query attention); 0 means n_heads

    @property
    def kv_heads(self) -> int:
        return self.n_kv_heads if self.n_kv_heads > 0 else self.n_heads


def oracle_config(cfg) -> OracleConfig:
    """Copy the fields the oracle needs from any object that has them."""
    return OracleConfig(cfg.depth, cfg.d_model, cfg.n_heads, cfg.head_dim, cfg.d_mlp, cfg.vocab,
                        cfg.seq_len, cfg.batch, list(cfg.windows), int(getattr(cfg, "n_kv_heads", 0) or 0))


# ------------------------------------------------------------------------------------------------
# parameter packing: wte [V,d]; per layer W_qkv [d + 2·dkv, d] (rows q | k | v, dkv = kv_heads·Dh,
# = 3d without grouping), W_o [d,d], W_fc [F,d], W_proj [d,F]; W_lm [V,d]; every matrix row-major
# [out, in] and applied as y = x·Wᵀ.
# ------------------------------------------------------------------------------------------------
def qkv_rows(cfg: OracleConfig) -> int:
    return cfg.d_model + 2 * cfg.kv_heads * cfg.head_dim


def unpack(cfg: OracleConfig, flat: np.ndarray) -> Dict[str, np.ndarray]:
    d, F, V = cfg.d_model, cfg.d_mlp, cfg.vocab
    out = {}
    pos = 0

    def take(name, rows, cols):
        nonlocal pos
        out[name] = flat[pos:pos + rows * cols].reshape(rows, cols)
        pos += rows * cols

    take("wte", V, d)
    for l in range(cfg.depth):
        take(f"qkv{l}", qkv_rows(cfg), d)
        take(f"o{l}", d, d)
        take(f"fc{l}", F, d)
        take(f"proj{l}", d, F)
    take("lm", V, d)
    if pos != flat.size:
        raise ValueError(f"param buffer has {flat.size} elements, layout needs {pos}")
    return out


def n_params(cfg: OracleConfig) -> int:
    d, F, V = cfg.d_model, cfg.d_mlp, cfg.vocab
    return 2 * V * d + cfg.depth * (qkv_rows(cfg) * d + d * d + 2 * F * d)


# ------------------------------------------------------------------------------------------------
# building blocks
# ------------------------------------------------------------------------------------------------
def rmsnorm(x: np.ndarray):
    """y = x / sqrt(mean(x²) + eps) over the last axis; returns (y, rho) with rho = 1/sqrt(...)."""
    rho = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + EPS)
    return x * rho, rho


def rmsnorm_backward(dy: np.ndarray, y: np.ndarray, rho: np.ndarray) -> np.ndarray:
    """Chain rule of y = x·rho(x):  dx = rho·(dy − y·mean(y·dy))."""
    return rho * (dy - y * np.mean(y * dy, axis=-1, keepdims=True))


def rope_angles(seq_len: int, head_dim: int, dtype) -> (np.ndarray, np.ndarray):
    """cos/sin of φ[t, i] = t · base^(−2i/Dh), i < Dh/2, computed in float64."""
    half = head_dim // 2
    inv_freq = ROPE_BASE ** (-(2.0 * np.arange(half, dtype=np.float64)) / head_dim)
    phi = np.arange(seq_len, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.cos(phi).astype(dtype), np.sin(phi).astype(dtype)


def rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate the pairs (x_i, x_{i+Dh/2}) of x [T, H, Dh] by φ[t, i]."""
    half = x.shape[-1] // 2
    a, b = x[..., :half], x[..., half:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def rope_inverse(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate by −φ: the transpose of ``rope``, hence also its backward."""
    half = x.shape[-1] // 2
    a, b = x[..., :half], x[..., half:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([a * c + b * s, -a * s + b * c], axis=-1)


def attention_mask(seq_len: int, window: int) -> np.ndarray:
    """Boolean [T, T]: key j visible from query t iff t−w < j ≤ t (w ≤ 0 or ≥ T: j ≤ t)."""
    t = np.arange(seq_len)[:, None]
    j = np.arange(seq_len)[None, :]
    keep = j <= t
    if 0 < window < seq_len:
        keep &= j > t - window
    return keep


def softmax_rows(s: np.ndarray) -> np.ndarray:
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def logsumexp_rows(z: np.ndarray) -> np.ndarray:
    m = np.max(z, axis=-1)
    return m + np.log(np.sum(np.exp(z - m[:, None]), axis=-1))


def attention_forward(q: np.ndarray, k: np.ndarray, v: np.ndarray, window: int):
    """Causal (optionally windowed) softmax attention for one sequence: q [T, H, Dh], k and v
    [T, Hkv, Dh] with H a multiple of Hkv.  Query head h reads key/value head h // (H/Hkv) (grouped
    -query attention, consecutive query heads sharing one key/value head; Hkv = H is plain
    multi-head attention).

    Returns o [T, H, Dh], the probabilities p [H, T, T] and lse [H, T] (natural log of the
    row sums of exp(scores)).
    """
    T, H, Dh = q.shape
    group = H // k.shape[1]
    keep = attention_mask(T, window)
    scale = 1.0 / math.sqrt(Dh)
    o = np.zeros_like(q)
    p_all = np.zeros((H, T, T), dtype=q.dtype)
    lse = np.zeros((H, T), dtype=q.dtype)
    for h in range(H):
        g = h // group
        s = (q[:, h, :] @ k[:, g, :].T) * scale
        s = np.where(keep, s, -np.inf)
        p = softmax_rows(s)
        lse[h] = logsumexp_rows(s)
        p_all[h] = p
        o[:, h, :] = p @ v[:, g, :]
    return o, p_all, lse


def attention_backward(do: np.ndarray, q: np.ndarray, k: np.ndarray, v: np.ndarray, p: np.ndarray):
    """Gradients of attention_forward given dO [T, H, Dh] and the saved probabilities; the
    gradient of a shared key/value head sums over the query heads of its group."""
    T, H, Dh = q.shape
    group = H // k.shape[1]
    scale = 1.0 / math.sqrt(Dh)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for h in range(H):
        g = h // group
        ph = p[h]
        dv[:, g, :] += ph.T @ do[:, h, :]
        dp = do[:, h, :] @ v[:, g, :].T
        ds = ph * (dp - np.sum(dp * ph, axis=-1, keepdims=True))
        dq[:, h, :] = (ds @ k[:, g, :]) * scale
        dk[:, g, :] += (ds.T @ q[:, h, :]) * scale
    return dq, dk, dv


# ------------------------------------------------------------------------------------------------
# one sequence
# ------------------------------------------------------------------------------------------------
def forward_sequence(cfg: OracleConfig, P: Dict[str, np.ndarray], tok: np.ndarray, tgt: np.ndarray,
                     dtype=np.float64) -> dict:
    """Forward pass of one row; returns every intermediate the backward pass needs."""
    T, d, H, Dh = len(tok), cfg.d_model, cfg.n_heads, cfg.head_dim
    Hkv = cfg.kv_heads
    dkv = Hkv * Dh
    cos, sin = rope_angles(T, Dh, dtype)
    c = {"layers": []}
    x = P["wte"][tok].astype(dtype)
    c["x0"] = x
    for l in range(cfg.depth):
        L = {}
        r1, rho1 = rmsnorm(x)
        qkv = r1 @ P[f"qkv{l}"].T
        q = qkv[:, :d].reshape(T, H, Dh)
        k = qkv[:, d:d + dkv].reshape(T, Hkv, Dh)
        v = qkv[:, d + dkv:d + 2 * dkv].reshape(T, Hkv, Dh)
        qn, rq = rmsnorm(rope(q, cos, sin))
        kn, rk = rmsnorm(rope(k, cos, sin))
        o, p, lse = attention_forward(qn, kn, v, cfg.windows[l])
        of = o.reshape(T, d)
        x = x + of @ P[f"o{l}"].T
        r2, rho2 = rmsnorm(x)
        u = r2 @ P[f"fc{l}"].T
        a = np.maximum(u, 0.0)
        g = a * a
        x = x + g @ P[f"proj{l}"].T
        L.update(r1=r1, rho1=rho1, qn=qn, rq=rq, kn=kn, rk=rk, v=v, p=p, lse=lse, of=of, r2=r2,
                 rho2=rho2, a=a, g=g)
        c["layers"].append(L)
    xf, rhof = rmsnorm(x)
    z = xf @ P["lm"].T
    lse_z = logsumexp_rows(z)
    valid = tgt >= 0
    ell = np.where(valid, lse_z - z[np.arange(T), np.where(valid, tgt, 0)], 0.0)
    c.update(xL=x, xf=xf, rhof=rhof, z=z, lse_z=lse_z, ell=ell, valid=valid, cos=cos, sin=sin)
    return c


def backward_sequence(cfg: OracleConfig, P: Dict[str, np.ndarray], tok: np.ndarray, tgt: np.ndarray,
                      c: dict, weight: np.ndarray, G: Dict[str, np.ndarray]) -> np.ndarray:
    """Accumulate into G the gradient of Σ_t weight[t]·ℓ_t; returns dL/dx0 [T, d]."""
    T, d, H, Dh = len(tok), cfg.d_model, cfg.n_heads, cfg.head_dim
    # cross-entropy: dℓ_t/dz_t = softmax(z_t) − onehot(y_t)
    dz = softmax_rows(c["z"])
    rows = np.arange(T)
    dz[rows, np.where(c["valid"], tgt, 0)] -= 1.0
    dz *= (weight * c["valid"])[:, None]
    G["lm"] += dz.T @ c["xf"]
    dx = rmsnorm_backward(dz @ P["lm"], c["xf"], c["rhof"])
    for l in reversed(range(cfg.depth)):
        L = c["layers"][l]
        # MLP: x += relu(u)²·W_projᵀ,  u = r2·W_fcᵀ
        G[f"proj{l}"] += dx.T @ L["g"]
        dg = dx @ P[f"proj{l}"]
        du = dg * 2.0 * L["a"]
        G[f"fc{l}"] += du.T @ L["r2"]
        dx = dx + rmsnorm_backward(du @ P[f"fc{l}"], L["r2"], L["rho2"])
        # attention: x += o·W_oᵀ
        G[f"o{l}"] += dx.T @ L["of"]
        do = (dx @ P[f"o{l}"]).reshape(T, H, Dh)
        dqn, dkn, dv = attention_backward(do, L["qn"], L["kn"], L["v"], L["p"])
        dq = rope_inverse(rmsnorm_backward(dqn, L["qn"], L["rq"]), c["cos"], c["sin"])
        dk = rope_inverse(rmsnorm_backward(dkn, L["kn"], L["rk"]), c["cos"], c["sin"])
        dkv = cfg.kv_heads * Dh
        dqkv = np.concatenate([dq.reshape(T, d), dk.reshape(T, dkv), dv.reshape(T, dkv)], axis=1)
        G[f"qkv{l}"] += dqkv.T @ L["r1"]
        dx = dx + rmsnorm_backward(dqkv @ P[f"qkv{l}"], L["r1"], L["rho1"])
    np.add.at(G["wte"], tok, dx)
    return dx


# ------------------------------------------------------------------------------------------------
# whole step
# ------------------------------------------------------------------------------------------------
def step(cfg, params: np.ndarray, tokens: np.ndarray, targets: np.ndarray, dtype=np.float64,
         position_weights: Optional[np.ndarray] = None, keep: bool = False) -> dict:
    """Loss and flat parameter gradients of one training step over the batch.

    loss = Σ_valid ℓ / n_valid  (0 when n_valid = 0, with zero gradients).  ``position_weights``
    [B, T] replaces the 1/n_valid weights of the backward pass (used to differentiate single
    per-position losses).  Returns a dict with loss, grads (flat, same packing as params), the
    per-position losses ell [B, T], dx0 [B, T, d] and, if keep, the per-row caches.
    """
    cfg = cfg if isinstance(cfg, OracleConfig) else oracle_config(cfg)
    params = np.asarray(params, dtype=dtype)
    P = unpack(cfg, params)
    grads = np.zeros_like(params)
    G = unpack(cfg, grads)  # views into grads
    tokens = np.asarray(tokens).reshape(cfg.batch, cfg.seq_len)
    targets = np.asarray(targets).reshape(cfg.batch, cfg.seq_len)
    n_valid = int(np.sum(targets >= 0))
    ell = np.zeros(tokens.shape, dtype=dtype)
    dx0 = np.zeros(tokens.shape + (cfg.d_model,), dtype=dtype)
    caches = []
    for b in range(cfg.batch):
        c = forward_sequence(cfg, P, tokens[b], targets[b], dtype)
        ell[b] = c["ell"]
        if position_weights is not None:
            w = np.asarray(position_weights[b], dtype=dtype)
        else:
            w = np.full(cfg.seq_len, (1.0 / n_valid) if n_valid else 0.0, dtype=dtype)
        dx0[b] = backward_sequence(cfg, P, tokens[b], targets[b], c, w, G)
        if keep:
            caches.append(c)
    loss = float(np.sum(ell) / n_valid) if n_valid else 0.0
    out = dict(loss=loss, grads=grads, ell=ell, dx0=dx0, n_valid=n_valid)
    if keep:
        out["caches"] = caches
    return out


def forward_loss(cfg, params: np.ndarray, tokens: np.ndarray, targets: np.ndarray, dtype=np.float64) -> float:
    """Loss only (no backward): used by finite differences."""
    cfg = cfg if isinstance(cfg, OracleConfig) else oracle_config(cfg)
    P = unpack(cfg, np.asarray(params, dtype=dtype))
    tokens = np.asarray(tokens).reshape(cfg.batch, cfg.seq_len)
    targets = np.asarray(targets).reshape(cfg.batch, cfg.seq_len)
    n_valid = int(np.sum(targets >= 0))
    tot = 0.0
    for b in range(cfg.batch):
        tot += float(np.sum(forward_sequence(cfg, P, tokens[b], targets[b], dtype)["ell"]))
    return tot / n_valid if n_valid else 0.0


# ------------------------------------------------------------------------------------------------
# per-kernel reference functions (same definitions, exposed on their own for unit parity tests)
# ------------------------------------------------------------------------------------------------
def attention_batch_forward(q, k, v, window, dtype=np.float64):
    """q [B, H, T, Dh], k, v [B, Hkv, T, Dh] → o [B, H, T, Dh], lse [B, H, T]."""
    q, k, v = (np.asarray(a, dtype=dtype) for a in (q, k, v))
    B = q.shape[0]
    o = np.zeros_like(q)
    lse = np.zeros(q.shape[:3], dtype=dtype)
    for b in range(B):
        ob, _, lb = attention_forward(q[b].transpose(1, 0, 2), k[b].transpose(1, 0, 2),
                                      v[b].transpose(1, 0, 2), window)
        o[b] = ob.transpose(1, 0, 2)
        lse[b] = lb
    return o, lse


def attention_batch_backward(q, k, v, do, window, dtype=np.float64):
    """Gradients dq [B, H, T, Dh], dk, dv [B, Hkv, T, Dh] of Σ o·dO for attention_batch_forward."""
    q, k, v, do = (np.asarray(a, dtype=dtype) for a in (q, k, v, do))
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(q.shape[0]):
        qt, kt, vt = (a[b].transpose(1, 0, 2) for a in (q, k, v))
        _, p, _ = attention_forward(qt, kt, vt, window)
        a1, a2, a3 = attention_backward(do[b].transpose(1, 0, 2), qt, kt, vt, p)
        dq[b], dk[b], dv[b] = (a.transpose(1, 0, 2) for a in (a1, a2, a3))
    return dq, dk, dv
