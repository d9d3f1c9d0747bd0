"""Pins of the optimizer oracle (Muon + AdamW) against things other than itself (CPU only).

* Newton–Schulz acts on each singular value by the scalar quintic: a matrix built from a known SVD
  must come out with the same singular vectors and the scalar recursion applied to its normalised
  singular values;
* it is transpose-equivariant, and on rectangular inputs its output is near-orthogonal (singular
  values within the band the quintic is known to reach in 5 steps);
* AdamW closed forms: the first step from a zero state, and constant gradients (bias correction
  makes m̂ = g and v̂ = g² at every step);
* the parameter grouping and the AdamW learning-rate scale the pages print
  (tests/golden/page_figures.txt).
"""
import os

import numpy as np
import pytest

from gpt_decoder_pretraining_b200.config import custom, preset
from oracle import optim_oracle as Q

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.txt")


def golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            vals[k] = float(v)
    return vals


def _orthogonal(n, rng):
    q, r = np.linalg.qr(rng.standard_normal((n, n)))
    return q * np.sign(np.diag(r))


@pytest.mark.parametrize("shape", [(24, 16), (16, 24), (20, 20)])
def test_newton_schulz_acts_on_singular_values(shape):
    rng = np.random.default_rng(7)
    r, c = shape
    k = min(r, c)
    u, v = _orthogonal(r, rng)[:, :k], _orthogonal(c, rng)[:, :k]
    s = np.sort(rng.uniform(0.2, 3.0, k))[::-1]
    g = (u * s) @ v.T
    want = (u * Q.newton_schulz_scalar(s / np.linalg.norm(s))) @ v.T
    np.testing.assert_allclose(Q.newton_schulz(g, eps=0.0), want, atol=1e-12)


def test_newton_schulz_transpose_and_band():
    rng = np.random.default_rng(8)
    for shape in [(64, 32), (32, 64), (256, 64)]:
        g = rng.standard_normal(shape)
        x = Q.newton_schulz(g)
        np.testing.assert_allclose(Q.newton_schulz(g.T), x.T, atol=1e-12)
        sv = np.linalg.svd(x, compute_uv=False)
        assert sv.min() > 0.6 and sv.max() < 1.25, (shape, sv.min(), sv.max())


def test_adamw_first_step_closed_form():
    rng = np.random.default_rng(9)
    w, g = rng.standard_normal(50), rng.standard_normal(50)
    lr, wd, eps = 0.01, 0.1, 1e-8
    w1, m, v = Q.adamw_update(w, g, np.zeros(50), np.zeros(50), 1, lr, 0.8, 0.95, eps, wd)
    np.testing.assert_allclose(w1, w * (1 - lr * wd) - lr * g / (np.abs(g) + eps), atol=1e-15)
    np.testing.assert_allclose(m, 0.2 * g, atol=1e-15)
    np.testing.assert_allclose(v, 0.05 * g * g, atol=1e-15)


def test_adamw_constant_gradient_moves_by_lr_each_step():
    g = np.array([0.5, -2.0, 3.0])
    w = np.zeros(3)
    m = np.zeros(3)
    v = np.zeros(3)
    for t in range(1, 8):
        w_prev = w
        w, m, v = Q.adamw_update(w, g, m, v, t, 0.1, 0.9, 0.999, 0.0, 0.0)
        np.testing.assert_allclose(w - w_prev, -0.1 * np.sign(g), atol=1e-12)


def test_muon_without_momentum_is_scaled_polar_factor():
    rng = np.random.default_rng(10)
    w, g = rng.standard_normal((30, 10)), rng.standard_normal((30, 10))
    w1, buf = Q.muon_update(w, g, np.zeros_like(g), lr=0.02, momentum=0.0)
    np.testing.assert_allclose(buf, g, atol=0)
    np.testing.assert_allclose(w1, w - 0.02 * np.sqrt(3.0) * Q.newton_schulz(g), atol=1e-14)


def test_grouping_and_lr_scale_match_the_pages():
    gold = golden()
    cfg = preset("d20")
    shapes = {}
    for _, (off, r, c) in Q.muon_matrices(cfg).items():
        shapes[(r, c)] = shapes.get((r, c), 0) + 1
    # the printed shapes are [out, in] weight shapes, the packing's own layout
    assert shapes[(1280, 1280)] == gold["d20_muon_1280x1280"]
    assert shapes[(1280, 5120)] == gold["d20_muon_1280x5120"]
    assert shapes[(5120, 1280)] == gold["d20_muon_5120x1280"]
    assert abs(1.0 / np.sqrt(cfg.d_model / 768.0) - gold["d20_adamw_lr_scale"]) < 5e-7
    # Muon and AdamW together cover every parameter exactly once
    covered = np.zeros(cfg.n_params, dtype=np.int8)
    for _, (off, r, c) in list(Q.muon_matrices(cfg).items()) + list(Q.adamw_tensors(cfg).items()):
        covered[off:off + r * c] += 1
    assert np.all(covered == 1)


def test_optimizer_step_updates_every_tensor_once():
    cfg = custom(2, 32, 16, 64, 12, 2, param_dtype=1)
    rng = np.random.default_rng(11)
    p = rng.standard_normal(cfg.n_params)
    g = rng.standard_normal(cfg.n_params)
    hp = dict(muon_lr=0.02, muon_momentum=0.95, ns_steps=5, ns_coeffs=Q.NS_QUINTIC,
              adam_lr_wte=0.2, adam_lr_lm=0.004, beta1=0.8, beta2=0.95, eps=0.0, weight_decay=0.0)
    state = {}
    p1 = Q.optimizer_step(cfg, p, g, state, 1, hp)
    # the lm-head moves by its (scaled) lr on the first AdamW step, elementwise
    off, r, c = Q.adamw_tensors(cfg)["w_lm"]
    lr = 0.004 / np.sqrt(cfg.d_model / 768.0)
    np.testing.assert_allclose(p1[off:off + r * c] - p[off:off + r * c],
                               -lr * np.sign(g[off:off + r * c]), atol=1e-9)
    # a Muon matrix moves by lr·NS(g + μ·g) (Nesterov from a zero buffer)
    off, r, c = Q.muon_matrices(cfg)["h1.w_k"]
    step = (p1[off:off + r * c] - p[off:off + r * c]).reshape(r, c)
    np.testing.assert_allclose(step, -0.02 * Q.newton_schulz(1.95 * g[off:off + r * c].reshape(r, c)),
                               atol=1e-12)
