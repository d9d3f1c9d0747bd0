"""Forward-only inference with a key/value cache against the oracle (needs a B200).

The oracle's forward pass over a whole sequence gives the logits of every position and, per layer,
k̃ = RMS_Dh(RoPE(k)) and v.  Prefill of T positions must reproduce the logits of position T−1 and
the cache contents of positions 0..T−1; decoding tokens one at a time after a shorter prefill must
reproduce the logits of each new position — the same numbers the training step's forward computes,
within the bf16 tolerance of its activations.
"""
import numpy as np
import pytest
import torch

from gpt_decoder_pretraining_b200.config import custom
from gpt_decoder_pretraining_b200.inputs import make_config_inputs
from oracle import gpt_oracle as O
from tests.gpu_util import assert_close_rel

pytestmark = pytest.mark.gpu

CASES = [dict(depth=2, d=256, hd=64, kv=2, V=512, T=100, B=2, windows=[40, 0]),
         dict(depth=2, d=256, hd=128, kv=0, V=1024, T=130, B=3, windows=[0, 0])]


def setup_module(module):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _oracle_rows(cfg, params, tokens):
    oc = O.oracle_config(cfg)
    P = O.unpack(oc, params.astype(np.float64))
    return [O.forward_sequence(oc, P, tokens[b], np.zeros(tokens.shape[1], np.int64)) for b in range(tokens.shape[0])]


@pytest.mark.parametrize("case", CASES, ids=["gqa_window", "mha"])
def test_prefill_logits_and_cache(case):
    from gpt_decoder_pretraining_b200.step import GptInfer
    cfg = custom(case["depth"], case["d"], case["hd"], case["V"], case["T"], case["B"], windows=case["windows"],
                 n_kv_heads=case["kv"])
    params, tokens, _ = make_config_inputs(cfg)
    B, T = tokens.shape
    inf = GptInfer(cfg, max_batch=B + 1, max_len=T + 8)
    p = torch.from_numpy(params.astype(np.float32)).cuda().to(torch.bfloat16)
    logits = inf.prefill(p, torch.from_numpy(tokens).cuda())
    torch.cuda.synchronize()
    assert inf.status() == 0
    ref = _oracle_rows(cfg, params, tokens)
    got = logits.cpu().numpy().astype(np.float64)
    for b in range(B):
        assert_close_rel(got[b], ref[b]["z"][T - 1], rel=3e-2, cos=0.9995, what=f"logits row {b}")
    # cache: [depth][2][max_batch][Hkv][max_len][Dh]
    Hkv, Dh = cfg.kv_heads, cfg.head_dim
    cache = inf.kv_cache.float().cpu().numpy().astype(np.float64).reshape(cfg.depth, 2, B + 1, Hkv, T + 8, Dh)
    for l in range(cfg.depth):
        for b in range(B):
            L = ref[b]["layers"][l]
            k_ref = L["kn"].transpose(1, 0, 2)  # [Hkv, T, Dh]
            v_ref = L["v"].transpose(1, 0, 2)
            assert_close_rel(cache[l, 0, b, :, :T], k_ref, rel=2e-2, cos=0.9999, what=f"k̃ layer {l} row {b}")
            assert_close_rel(cache[l, 1, b, :, :T], v_ref, rel=3e-2, cos=0.9995, what=f"v layer {l} row {b}")


@pytest.mark.parametrize("case", CASES, ids=["gqa_window", "mha"])
def test_decode_matches_the_full_forward(case):
    from gpt_decoder_pretraining_b200.step import GptInfer
    cfg = custom(case["depth"], case["d"], case["hd"], case["V"], case["T"], case["B"], windows=case["windows"],
                 n_kv_heads=case["kv"])
    params, tokens, _ = make_config_inputs(cfg)
    B, T = tokens.shape
    n_new = 3
    inf = GptInfer(cfg, max_batch=B, max_len=T)
    p = torch.from_numpy(params.astype(np.float32)).cuda().to(torch.bfloat16)
    tt = torch.from_numpy(tokens).cuda()
    inf.prefill(p, tt[:, :T - n_new].contiguous())
    ref = _oracle_rows(cfg, params, tokens)
    for i in range(n_new):
        pos = T - n_new + i
        logits = inf.decode(p, tt[:, pos].contiguous(), pos)
        torch.cuda.synchronize()
        got = logits.cpu().numpy().astype(np.float64)
        for b in range(B):
            assert_close_rel(got[b], ref[b]["z"][pos], rel=3e-2, cos=0.9995, what=f"decode pos {pos} row {b}")
    assert inf.status() == 0
