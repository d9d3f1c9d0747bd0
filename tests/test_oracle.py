"""Pins of the CPU oracle against things other than itself (CPU only, no GPU).

* finite differences of its own loss (fp64, smoke config): pins the backward pass;
* closed forms: W_lm = 0 gives uniform logits, loss = ln V, zero gradients everywhere but dW_lm,
  and dW_lm = (1/V − onehot)ᵀ·x_f / n;
* invariants: probability rows sum to 1, RoPE is a norm-preserving group action, RoPE and QK-norm
  commute, a window ≥ T equals full causal attention, causality and window locality of the
  per-position loss gradients, batch linearity and row-permutation invariance;
* special cases that reduce to library routines: torch's rms_norm, linear (y = x·Wᵀ),
  scaled_dot_product_attention and cross_entropy, differentiated by autograd;
* the whole step rebuilt from those torch library ops (RoPE from its definition), every gradient
  from autograd, equal to the oracle to rounding;
* the figures the pages print (tests/golden/page_figures.txt) and the ≈ ln V initial loss.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from gpt_decoder_pretraining_b200.config import custom, preset
from gpt_decoder_pretraining_b200.inputs import make_config_inputs, make_params, make_tokens
from oracle import gpt_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.txt")


def golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            vals[k] = float(v)
    return vals


def tiny(depth=2, d=32, hd=16, V=64, T=12, B=2, windows=None, n_kv_heads=0):
    return custom(depth, d, hd, V, T, B, windows=windows, param_dtype=1, n_kv_heads=n_kv_heads)


def inputs_for(cfg, seed=0, std=0.3):
    p = make_params(cfg.n_params, keep_fp32=True, seed=seed, std=std).astype(np.float64)
    t, y = make_tokens(cfg.batch, cfg.seq_len, cfg.vocab, seed=seed + 1)
    return p, t, y


# -------------------------------------------------------------------------------------------------
def test_page_figures_config_arithmetic():
    g = golden()
    d20 = preset("d20")
    assert d20.n_params == g["d20_params"]
    assert O.n_params(O.oracle_config(d20)) == g["d20_params"]
    import dataclasses
    full = dataclasses.replace(d20, windows=[0] * 20)
    assert f"{full.flops_per_token():.6e}" == f"{g['d20_flops_per_token_T2048']:.6e}"
    t1024 = dataclasses.replace(d20, windows=[0] * 20, seq_len=1024)
    assert f"{t1024.flops_per_token():.6e}" == f"{g['d20_flops_per_token_T1024']:.6e}"
    d24 = preset("d24")
    assert round((d24.n_params - d24.vocab * d24.d_model) / 1e6, 1) == g["d24_scaling_params_millions"]
    # page-reported random-init losses sit at ln V (uniform guessing)
    assert abs(g["d20_step0_loss"] - math.log(65536)) < 1e-3
    assert abs(g["d24_step1_loss"] - math.log(32768)) < 2e-3


def _fd_check(cfg, p, t, y, coords_per_tensor=24, h=1e-4, rng_seed=5, extra=()):
    """4-point central differences of the loss at sampled coordinates; returns worst scaled error.

    h = 1e-4: ReLU² is only once continuously differentiable, so wider stencils that straddle
    u = 0 pick up an O(h) error; at 1e-4 the fp64 rounding error stays near 1e-9.
    """
    res = O.step(cfg, p, t, y, dtype=np.float64)
    g = res["grads"]
    oc = O.oracle_config(cfg)
    rng = np.random.default_rng(rng_seed)
    worst = 0.0
    off = 0
    for name, (a, b) in cfg.tensor_shapes():
        n = a * b
        gmax = np.max(np.abs(g[off:off + n])) + 1e-30
        idx = list(off + rng.choice(n, size=min(coords_per_tensor, n), replace=False))
        idx += [off + i for (nm, i) in extra if nm == name]
        for i in idx:
            vals = []
            for s in (2, 1, -1, -2):
                q = p.copy()
                q[i] += s * h
                vals.append(O.forward_loss(oc, q, t, y))
            fd = (-vals[0] + 8 * vals[1] - 8 * vals[2] + vals[3]) / (12 * h)
            worst = max(worst, abs(fd - g[i]) / gmax)
        off += n
    return worst


def test_finite_differences_smoke_fp64():
    cfg = preset("smoke")
    p, t, y = make_config_inputs(cfg)
    p = p.astype(np.float64)
    # a token id that repeats in the sequence: the scatter-add of the embedding grad must sum
    t = t.copy()
    t[0, 5] = t[0, 40] = t[0, 77]
    rep = int(t[0, 5])
    d = cfg.d_model
    extra = [("wte", rep * d + j) for j in range(0, d, 4)]
    # one attention head's W_q rows (head 1, a few full rows)
    extra += [("h1.w_qkv", (cfg.head_dim + r) * d + j) for r in (0, 7, 31) for j in range(0, d, 8)]
    worst = _fd_check(cfg, p, t, y, coords_per_tensor=16, extra=extra)
    assert worst < 1e-6, worst


def test_finite_differences_windowed_tiny():
    cfg = tiny(depth=2, windows=[3, 0])
    p, t, y = inputs_for(cfg)
    assert _fd_check(cfg, p, t, y, coords_per_tensor=40) < 1e-6


def test_zero_lm_head_closed_form():
    cfg = tiny(depth=2, windows=[4, 0])
    p, t, y = inputs_for(cfg)
    off = cfg.n_params - cfg.vocab * cfg.d_model
    p[off:] = 0.0
    r = O.step(cfg, p, t, y, keep=True)
    assert r["loss"] == pytest.approx(math.log(cfg.vocab), abs=1e-14)
    g = r["grads"]
    assert np.all(g[:off] == 0.0)
    n = t.size
    dW = np.zeros((cfg.vocab, cfg.d_model))
    for b in range(cfg.batch):
        xf = r["caches"][b]["xf"]
        sm = np.full((cfg.seq_len, cfg.vocab), 1.0 / cfg.vocab)
        sm[np.arange(cfg.seq_len), y[b]] -= 1.0
        dW += sm.T @ xf / n
    np.testing.assert_allclose(g[off:].reshape(cfg.vocab, cfg.d_model), dW, rtol=0, atol=1e-15)


def test_probability_rows_sum_to_one():
    cfg = tiny(depth=2, windows=[5, 0])
    p, t, y = inputs_for(cfg)
    r = O.step(cfg, p, t, y, keep=True)
    c = r["caches"][0]
    for L in c["layers"]:
        np.testing.assert_allclose(L["p"].sum(-1), 1.0, atol=1e-12)
        assert np.all(L["p"] >= 0)
    np.testing.assert_allclose(O.softmax_rows(c["z"]).sum(-1), 1.0, atol=1e-12)


def test_rope_invariants():
    rng = np.random.default_rng(0)
    T, H, Dh = 37, 3, 16
    x = rng.standard_normal((T, H, Dh))
    cos, sin = O.rope_angles(T, Dh, np.float64)
    y = O.rope(x, cos, sin)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)
    np.testing.assert_allclose(y[0], x[0], atol=0)  # position 0 is the identity
    np.testing.assert_allclose(O.rope_inverse(y, cos, sin), x, atol=1e-12)
    # composition: rotating a vector placed at position a by angle(b) equals angle(a+b)
    a, b = 5, 11
    c2, s2 = O.rope_angles(T, Dh, np.float64)
    xa = O.rope(x[a:a + 1], c2[a:a + 1], s2[a:a + 1])
    xab = O.rope(xa, c2[b:b + 1], s2[b:b + 1])
    np.testing.assert_allclose(xab, O.rope(x[a:a + 1], c2[a + b:a + b + 1], s2[a + b:a + b + 1]), atol=1e-12)
    # frequency of pair i is base^(-2i/Dh): position 1 rotates pair 0 by exactly 1 radian
    e = np.zeros((2, 1, Dh))
    e[:, 0, 0] = 1.0
    r = O.rope(e, cos[:2], sin[:2])
    assert r[1, 0, 0] == pytest.approx(math.cos(1.0)) and r[1, 0, Dh // 2] == pytest.approx(math.sin(1.0))


def test_qknorm_rope_commute():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((20, 2, 32)) * 3
    cos, sin = O.rope_angles(20, 32, np.float64)
    a, _ = O.rmsnorm(O.rope(x, cos, sin))
    b = O.rope(O.rmsnorm(x)[0], cos, sin)
    np.testing.assert_allclose(a, b, atol=1e-12)


def test_window_at_least_T_is_full_causal():
    cfg_full = tiny(depth=2, windows=[0, 0])
    p, t, y = inputs_for(cfg_full)
    r0 = O.step(cfg_full, p, t, y)
    for w in (cfg_full.seq_len, cfg_full.seq_len + 7):
        r1 = O.step(tiny(depth=2, windows=[w, w]), p, t, y)
        assert r1["loss"] == r0["loss"]
        assert np.array_equal(r1["grads"], r0["grads"])


def _dloss_s_dx0(cfg, p, t, y, s):
    w = np.zeros((cfg.batch, cfg.seq_len))
    w[0, s] = 1.0
    return O.step(cfg, p, t, y, position_weights=w)["dx0"][0]


def test_causality_and_window_locality():
    T = 12
    for win in (0, 3):
        cfg = tiny(depth=1, T=T, B=1, windows=[win])
        p, t, y = inputs_for(cfg)
        for s in (0, 5, 11):
            g = _dloss_s_dx0(cfg, p, t, y, s)
            norms = np.linalg.norm(g, axis=-1)
            assert np.all(norms[s + 1:] == 0.0)            # no position after s
            if win:
                assert np.all(norms[:max(0, s - win + 1)] == 0.0)  # nothing older than the window
            lo = max(0, s - win + 1) if win else 0
            assert np.all(norms[lo:s + 1] > 0.0)


def test_batch_linearity_and_permutation():
    cfg = tiny(depth=2, B=3, windows=[4, 0])
    p, t, y = inputs_for(cfg)
    y = y.copy()
    y[1, :5] = -1  # uneven valid counts
    r = O.step(cfg, p, t, y)
    n = int(np.sum(y >= 0))
    acc = np.zeros_like(p)
    loss = 0.0
    for b in range(cfg.batch):
        c1 = tiny(depth=2, B=1, windows=[4, 0])
        rb = O.step(c1, p, t[b:b + 1], y[b:b + 1])
        nb = rb["n_valid"]
        acc += rb["grads"] * nb / n
        loss += rb["loss"] * nb / n
    np.testing.assert_allclose(r["grads"], acc, atol=1e-12 * np.max(np.abs(acc)))
    assert r["loss"] == pytest.approx(loss, abs=1e-12)
    perm = [2, 0, 1]
    rp = O.step(cfg, p, t[perm], y[perm])
    np.testing.assert_allclose(rp["grads"], r["grads"], atol=1e-12 * np.max(np.abs(acc)))


def test_all_targets_ignored_gives_zero():
    cfg = tiny()
    p, t, y = inputs_for(cfg)
    r = O.step(cfg, p, t, np.full_like(y, -1))
    assert r["loss"] == 0.0 and not np.any(r["grads"])


def test_single_position_attention_is_v():
    rng = np.random.default_rng(2)
    q, k, v = (rng.standard_normal((1, 3, 8)) for _ in range(3))
    o, p, lse = O.attention_forward(q, k, v, 0)
    np.testing.assert_allclose(o, v, atol=1e-15)
    np.testing.assert_allclose(p, 1.0)


def test_depth0_is_softmax_regression_vs_torch_autograd():
    cfg = tiny(depth=0, T=9, B=2)
    p, t, y = inputs_for(cfg)
    y = y.copy()
    y[0, 2] = -1
    r = O.step(cfg, p, t, y)
    V, d = cfg.vocab, cfg.d_model
    wte = torch.tensor(p[:V * d].reshape(V, d), requires_grad=True)
    wlm = torch.tensor(p[V * d:].reshape(V, d), requires_grad=True)
    x = F.rms_norm(wte[torch.tensor(t)], (d,), eps=1e-6)
    z = F.linear(x, wlm)
    loss = F.cross_entropy(z.reshape(-1, V), torch.tensor(y).reshape(-1).long(), ignore_index=-1)
    loss.backward()
    assert r["loss"] == pytest.approx(loss.item(), abs=1e-13)
    np.testing.assert_allclose(r["grads"][:V * d], wte.grad.numpy().ravel(), atol=1e-14)
    np.testing.assert_allclose(r["grads"][V * d:], wlm.grad.numpy().ravel(), atol=1e-14)


@pytest.mark.parametrize("window", [0, 1, 4, 9, 40])
def test_attention_vs_torch_sdpa(window):
    rng = np.random.default_rng(3)
    B, H, T, Dh = 2, 3, 23, 16
    q, k, v, do = (rng.standard_normal((B, H, T, Dh)) for _ in range(4))
    o, lse = O.attention_batch_forward(q, k, v, window)
    dq, dk, dv = O.attention_batch_backward(q, k, v, do, window)
    keep = torch.tensor(O.attention_mask(T, window))
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    to = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=keep)
    to.backward(torch.tensor(do))
    np.testing.assert_allclose(o, to.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)
    s = torch.einsum("bhtd,bhjd->bhtj", torch.tensor(q), torch.tensor(k)) / math.sqrt(Dh)
    ref_lse = torch.logsumexp(s.masked_fill(~keep, -float("inf")), dim=-1)
    np.testing.assert_allclose(lse, ref_lse.numpy(), atol=1e-12)


def test_rmsnorm_vs_torch():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((7, 48)) * 2
    dy = rng.standard_normal((7, 48))
    y, rho = O.rmsnorm(x)
    tx = torch.tensor(x, requires_grad=True)
    ty = F.rms_norm(tx, (48,), eps=1e-6)
    ty.backward(torch.tensor(dy))
    np.testing.assert_allclose(y, ty.detach().numpy(), atol=1e-14)
    np.testing.assert_allclose(O.rmsnorm_backward(dy, y, rho), tx.grad.numpy(), atol=1e-13)


def test_init_loss_near_ln_v_smoke():
    cfg = preset("smoke")
    p, t, y = make_config_inputs(cfg)
    loss = O.forward_loss(cfg, p, t, y, dtype=np.float64)
    assert abs(loss - (math.log(cfg.vocab) + 0.0002 * cfg.d_model)) < 0.05


@pytest.mark.slow
def test_init_loss_near_ln_v_d12_one_row():
    import dataclasses
    cfg = dataclasses.replace(preset("d12"), batch=1, depth=2, windows=[0, 0])
    p, t, y = make_config_inputs(cfg)
    loss = O.forward_loss(cfg, p.astype(np.float32), t, y, dtype=np.float32)
    assert abs(loss - (math.log(cfg.vocab) + 0.0002 * cfg.d_model)) < 0.05


# -------------------------------------------------------------------------------------------------
# planted mistakes: each plausible slip in the oracle must make one of the pins above fail
# -------------------------------------------------------------------------------------------------
def _run_pins(monkeypatch_fn):
    cfg = tiny(depth=2, windows=[3, 0])
    p, t, y = inputs_for(cfg)
    try:
        fd = _fd_check(cfg, p, t, y, coords_per_tensor=12)
        fd_ok = fd < 1e-6
    except Exception:
        fd_ok = False
    ok = fd_ok
    try:
        test_attention_vs_torch_sdpa(4)
        test_rmsnorm_vs_torch()
        test_rope_invariants()
        test_depth0_is_softmax_regression_vs_torch_autograd()
        test_causality_and_window_locality()
    except AssertionError:
        ok = False
    return ok


@pytest.mark.parametrize("mistake", ["rms_bwd_term", "rope_bwd_sign", "relu2_factor", "attn_scale",
                                     "ds_rowsum", "eps_dropped", "window_off_by_one"])
def test_planted_mistakes_are_caught(monkeypatch, mistake):
    if mistake == "rms_bwd_term":
        monkeypatch.setattr(O, "rmsnorm_backward", lambda dy, y, rho: rho * dy)
    elif mistake == "rope_bwd_sign":
        monkeypatch.setattr(O, "rope_inverse", O.rope)
    elif mistake == "relu2_factor":
        orig = O.backward_sequence

        def bad(cfg, P, tok, tgt, c, weight, G):
            for L in c["layers"]:
                L["a"] = L["a"] * 0.5
            return orig(cfg, P, tok, tgt, c, weight, G)
        monkeypatch.setattr(O, "backward_sequence", bad)
    elif mistake == "attn_scale":
        orig_fwd = O.attention_forward

        def bad_fwd(q, k, v, window):
            return orig_fwd(q * math.sqrt(q.shape[-1]) ** 0.5, k, v, window)
        monkeypatch.setattr(O, "attention_forward", bad_fwd)
    elif mistake == "ds_rowsum":
        def bad_bwd(do, q, k, v, p):
            T, H, Dh = q.shape
            dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
            for h in range(H):
                ph = p[h]
                dv[:, h, :] = ph.T @ do[:, h, :]
                ds = ph * (do[:, h, :] @ v[:, h, :].T)
                dq[:, h, :] = ds @ k[:, h, :] / math.sqrt(Dh)
                dk[:, h, :] = ds.T @ q[:, h, :] / math.sqrt(Dh)
            return dq, dk, dv
        monkeypatch.setattr(O, "attention_backward", bad_bwd)
    elif mistake == "eps_dropped":
        monkeypatch.setattr(O, "EPS", 0.0)
    elif mistake == "window_off_by_one":
        def bad_mask(seq_len, window):
            t = np.arange(seq_len)[:, None]
            j = np.arange(seq_len)[None, :]
            keep = j <= t
            if 0 < window < seq_len:
                keep &= j >= t - window
            return keep
        monkeypatch.setattr(O, "attention_mask", bad_mask)
    assert not _run_pins(None)


def _torch_model_loss(cfg, flat, tokens, targets):
    """The architecture written with torch library ops only (embedding, rms_norm, linear, sdpa with a
    boolean mask, cross_entropy with ignore_index); autograd supplies every gradient."""
    d, H, Dh, T = cfg.d_model, cfg.n_heads, cfg.head_dim, cfg.seq_len
    ws, off = {}, 0
    for name, (a, b) in cfg.tensor_shapes():
        ws[name] = flat[off:off + a * b].view(a, b)
        off += a * b
    pos = torch.arange(T, dtype=torch.float64)
    inv = 10000.0 ** (-2.0 * torch.arange(Dh // 2, dtype=torch.float64) / Dh)
    ang = pos[:, None] * inv[None, :]
    cos, sin = torch.cos(ang), torch.sin(ang)

    def rotate(x):  # pairs (i, i + Dh/2), positions along dim −2
        a, b = x[..., :Dh // 2], x[..., Dh // 2:]
        return torch.cat([a * cos - b * sin, a * sin + b * cos], dim=-1)

    x = F.embedding(tokens, ws["wte"])
    B = tokens.shape[0]
    for l in range(cfg.depth):
        w = cfg.effective_window(l)
        i = torch.arange(T)
        keep = (i[None, :] <= i[:, None]) & (i[None, :] > i[:, None] - w)
        r = F.rms_norm(x, (d,), eps=1e-6)
        qkv = F.linear(r, ws[f"h{l}.w_qkv"])
        Hk = cfg.kv_heads
        qq, kk, vv = qkv.split([d, Hk * Dh, Hk * Dh], dim=-1)
        q = qq.view(B, T, H, Dh).transpose(1, 2)
        k, v = (t.view(B, T, Hk, Dh).transpose(1, 2) for t in (kk, vv))
        q = F.rms_norm(rotate(q), (Dh,), eps=1e-6)
        k = F.rms_norm(rotate(k), (Dh,), eps=1e-6)
        o = F.scaled_dot_product_attention(q, k, v, attn_mask=keep, enable_gqa=Hk != H)
        x = x + F.linear(o.transpose(1, 2).reshape(B, T, d), ws[f"h{l}.w_o"])
        u = F.linear(F.rms_norm(x, (d,), eps=1e-6), ws[f"h{l}.w_fc"])
        x = x + F.linear(torch.relu(u) ** 2, ws[f"h{l}.w_proj"])
    z = F.linear(F.rms_norm(x, (d,), eps=1e-6), ws["w_lm"])
    return F.cross_entropy(z.view(-1, cfg.vocab), targets.view(-1), ignore_index=-1, reduction="mean")


@pytest.mark.parametrize("windows,kv", [(None, 0), ([3, 0], 0), (None, 2), ([3, 0], 1)])
def test_whole_step_vs_torch_autograd(windows, kv):
    """Every gradient of the oracle's step equals torch autograd through library ops, to rounding;
    kv > 0: grouped-query attention with kv key/value heads (torch: sdpa with enable_gqa)."""
    cfg = tiny(depth=2, d=64, hd=16, V=64, T=12, B=2, windows=windows, n_kv_heads=kv)
    p, t, y = inputs_for(cfg, seed=5)
    y = y.copy()
    y[1, :3] = -1
    r = O.step(cfg, p, t, y, dtype=np.float64)
    flat = torch.tensor(p, requires_grad=True)
    loss = _torch_model_loss(cfg, flat, torch.tensor(t, dtype=torch.long), torch.tensor(y, dtype=torch.long))
    loss.backward()
    assert abs(r["loss"] - loss.item()) < 1e-12
    g = flat.grad.numpy()
    np.testing.assert_allclose(r["grads"], g, rtol=0, atol=1e-12 * max(1.0, np.abs(g).max()))


@pytest.mark.parametrize("kv", [1, 2])
def test_grouped_query_attention_equals_duplicated_heads(kv):
    """Grouped-query attention is multi-head attention whose consecutive query heads see copies of
    one key/value head: duplicating W_k and W_v row blocks gives the same loss, the same gradients
    of every other tensor, and key/value gradients that are the group sums of the duplicated ones."""
    g_cfg = tiny(depth=2, d=64, hd=16, V=64, T=10, B=2, windows=[4, 0], n_kv_heads=kv)
    m_cfg = tiny(depth=2, d=64, hd=16, V=64, T=10, B=2, windows=[4, 0])
    H, Dh, d = g_cfg.n_heads, g_cfg.head_dim, g_cfg.d_model
    G = H // kv
    p, t, y = inputs_for(g_cfg, seed=9)
    gP = O.unpack(O.oracle_config(g_cfg), p)
    mflat = np.zeros(m_cfg.n_params)
    mP = O.unpack(O.oracle_config(m_cfg), mflat)
    for name in gP:
        if not name.startswith("qkv"):
            mP[name][...] = gP[name]
            continue
        w = gP[name]
        mP[name][:d] = w[:d]
        for h in range(H):
            src = h // G
            mP[name][d + h * Dh:d + (h + 1) * Dh] = w[d + src * Dh:d + (src + 1) * Dh]
            mP[name][2 * d + h * Dh:2 * d + (h + 1) * Dh] = w[d + kv * Dh + src * Dh:d + kv * Dh + (src + 1) * Dh]
    rg = O.step(g_cfg, p, t, y)
    rm = O.step(m_cfg, mflat, t, y)
    assert abs(rg["loss"] - rm["loss"]) < 1e-12
    gG = O.unpack(O.oracle_config(g_cfg), rg["grads"])
    mG = O.unpack(O.oracle_config(m_cfg), rm["grads"])
    for name in gG:
        if not name.startswith("qkv"):
            np.testing.assert_allclose(gG[name], mG[name], atol=1e-13)
            continue
        np.testing.assert_allclose(gG[name][:d], mG[name][:d], atol=1e-13)
        for part in (1, 2):
            for g in range(kv):
                want = sum(mG[name][part * d + h * Dh:part * d + (h + 1) * Dh] for h in range(g * G, (g + 1) * G))
                got = gG[name][d + (part - 1) * kv * Dh + g * Dh:d + (part - 1) * kv * Dh + (g + 1) * Dh]
                np.testing.assert_allclose(got, want, atol=1e-13)
