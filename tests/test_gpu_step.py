"""Step-level parity: gpt_step_fwd_bwd through the C ABI against the CPU oracle (needs a B200).

Tolerances (fixed by the step's specification): loss within 2e-2 absolute; every gradient
tensor with cosine similarity ≥ 0.999 and max |Δ| ≤ 5e-2 · max |g_oracle| of that tensor.
"""
import dataclasses

import numpy as np
import pytest
import torch

from gpt_decoder_pretraining_b200.config import custom, preset
from gpt_decoder_pretraining_b200.inputs import make_config_inputs
from oracle import gpt_oracle as O
from tests.gpu_util import cosine

pytestmark = pytest.mark.gpu

LOSS_TOL = 2e-2
GRAD_COS = 0.999
GRAD_REL = 5e-2


def setup_module(module):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def run_gpu(cfg, params, tokens, targets):
    from gpt_decoder_pretraining_b200.step import GptStep
    st = GptStep(cfg)
    if cfg.param_dtype == 1:
        p = torch.from_numpy(params.astype(np.float32)).cuda()
    else:
        p = torch.from_numpy(params.astype(np.float32)).cuda().to(torch.bfloat16)
    t = torch.from_numpy(tokens.astype(np.int32)).cuda()
    y = torch.from_numpy(targets.astype(np.int32)).cuda()
    loss, grads = st(p, t, y)
    torch.cuda.synchronize()
    assert st.status() == 0
    return float(loss.item()), grads.cpu().numpy().astype(np.float64), st


def compare(cfg, loss_gpu, g_gpu, ref):
    assert abs(loss_gpu - ref["loss"]) <= LOSS_TOL, (loss_gpu, ref["loss"])
    off = 0
    report = []
    for name, (a, b) in cfg.tensor_shapes():
        n = a * b
        g, r = g_gpu[off:off + n], ref["grads"][off:off + n]
        scale = np.max(np.abs(r))
        err = np.max(np.abs(g - r))
        c = cosine(g, r)
        report.append((name, c, err / max(scale, 1e-30)))
        assert c >= GRAD_COS, (name, c)
        assert err <= GRAD_REL * scale, (name, err, scale)
        off += n
    return report


def test_step_smoke_config():
    cfg = preset("smoke")
    params, tokens, targets = make_config_inputs(cfg)
    loss, g, _ = run_gpu(cfg, params, tokens, targets)
    ref = O.step(cfg, params.astype(np.float64), tokens, targets, dtype=np.float64)
    compare(cfg, loss, g, ref)


@pytest.mark.parametrize("T,windows,dh", [(100, [33, 0], 64), (129, [1, 200], 128), (64, [0, 0], 32),
                                          (192, [0, 50], 128), (128, [70, 0], 64)])
def test_step_small_bf16_configs(T, windows, dh):
    cfg = custom(2, 2 * dh, dh, 512, T, 2, windows=windows)
    params, tokens, targets = make_config_inputs(cfg)
    targets = targets.copy()
    targets[0, :7] = -1  # ignored positions
    loss, g, _ = run_gpu(cfg, params, tokens, targets)
    ref = O.step(cfg, params.astype(np.float64), tokens, targets, dtype=np.float64)
    compare(cfg, loss, g, ref)


@pytest.mark.parametrize("d,dh,kv,T,windows", [(256, 64, 2, 130, [40, 0]), (512, 128, 1, 200, [0, 77]),
                                                (384, 64, 3, 96, [0, 0])])
def test_step_grouped_query_attention(d, dh, kv, T, windows):
    """Grouped-query attention (kv key/value heads shared by consecutive query heads) through the
    whole step, against the oracle's grouped attention."""
    cfg = custom(2, d, dh, 512, T, 2, windows=windows, n_kv_heads=kv)
    params, tokens, targets = make_config_inputs(cfg)
    loss, g, _ = run_gpu(cfg, params, tokens, targets)
    ref = O.step(cfg, params.astype(np.float64), tokens, targets, dtype=np.float64)
    compare(cfg, loss, g, ref)


def test_step_all_targets_ignored():
    cfg = custom(1, 64, 32, 256, 16, 1)
    params, tokens, targets = make_config_inputs(cfg)
    loss, g, _ = run_gpu(cfg, params, tokens, np.full_like(targets, -1))
    assert loss == 0.0 and not np.any(g)


def test_step_is_bitwise_deterministic():
    cfg = custom(2, 128, 64, 512, 96, 2, windows=[40, 0])
    params, tokens, targets = make_config_inputs(cfg)
    l1, g1, _ = run_gpu(cfg, params, tokens, targets)
    l2, g2, _ = run_gpu(cfg, params, tokens, targets)
    assert l1 == l2 and np.array_equal(g1, g2)


def test_step_token_out_of_range_sets_status():
    from gpt_decoder_pretraining_b200.step import GptStep
    cfg = custom(1, 64, 32, 256, 16, 1)
    params, tokens, targets = make_config_inputs(cfg)
    tokens = tokens.copy()
    tokens[0, 3] = 999
    st = GptStep(cfg)
    p = torch.from_numpy(params).cuda().to(torch.bfloat16)
    st(p, torch.from_numpy(tokens).cuda(), torch.from_numpy(targets).cuda())
    assert st.status() == -6
    assert st.status() == 0  # reading clears the word


def test_step_accumulates_gradients_across_micro_batches():
    """accumulate = 1 adds this micro-batch's gradients to the buffer: two steps give exactly the
    fp32 sum of the two single-step gradients (each element is one fp32 addition)."""
    from gpt_decoder_pretraining_b200.step import GptStep
    cfg = custom(2, 128, 64, 512, 96, 2, windows=[40, 0])
    params, tokens, targets = make_config_inputs(cfg)
    tokens_b, targets_b = np.roll(tokens, 5, axis=1), np.roll(targets, 5, axis=1)
    st = GptStep(cfg)
    p = torch.from_numpy(params.astype(np.float32)).cuda().to(torch.bfloat16)
    as_t = lambda a: torch.from_numpy(np.ascontiguousarray(a).astype(np.int32)).cuda()  # noqa: E731
    _, g = st(p, as_t(tokens), as_t(targets))
    g_a = g.cpu().numpy().copy()
    _, g = st(p, as_t(tokens_b), as_t(targets_b))
    g_b = g.cpu().numpy().copy()
    acc = torch.zeros_like(g)
    st(p, as_t(tokens), as_t(targets), grads=acc)
    st(p, as_t(tokens_b), as_t(targets_b), grads=acc, accumulate=True)
    torch.cuda.synchronize()
    assert st.status() == 0
    assert np.array_equal(acc.cpu().numpy(), (g_a + g_b).astype(np.float32))


def test_step_graph_replay_matches_eager_launches():
    """The step captured as one CUDA graph (GptStep.capture) gives bitwise the eager step's loss and
    gradients, and a replay after the token buffers change computes the new batch."""
    from gpt_decoder_pretraining_b200.step import GptStep
    cfg = custom(2, 256, 128, 512, 256, 2, windows=[100, 0])
    params, tokens, targets = make_config_inputs(cfg)
    p = torch.from_numpy(params.astype(np.float32)).cuda().to(torch.bfloat16)
    t = torch.from_numpy(tokens.astype(np.int32)).cuda()
    y = torch.from_numpy(targets.astype(np.int32)).cuda()
    st = GptStep(cfg)
    graph = st.capture(p, t, y)
    assert graph.launches > 0
    loss_g, grads_g = graph.replay()
    torch.cuda.synchronize()
    loss_g, grads_g = loss_g.clone(), grads_g.clone()
    eager = GptStep(cfg)
    loss_e, grads_e = eager(p, t, y)
    torch.cuda.synchronize()
    assert torch.equal(loss_g, loss_e) and torch.equal(grads_g, grads_e)
    # new tokens in the captured buffers: the replay computes them
    t2 = torch.roll(t, 7, dims=1).contiguous()
    t.copy_(t2)
    loss_g2, grads_g2 = graph.replay()
    loss_e2, grads_e2 = eager(p, t2, y)
    torch.cuda.synchronize()
    assert torch.equal(loss_g2, loss_e2) and torch.equal(grads_g2, grads_e2)
    assert not torch.equal(loss_g2, loss_g)
