"""gpt_attention_bwd_noalloc — the attention backward for callers that cannot allocate device
memory where they call it — checked against gpt_attention_bwd, the entry point that takes a
caller-allocated scratch buffer (needs a B200).

This file is collected last on purpose.  The first case runs two calls in a row on the shared
static scratch array; the second of them uses fewer rows, so the array still holds rows of the
first call beyond what the second one writes.  The test must pass both on its own in a fresh
process and after every other test.
"""
import numpy as np
import pytest
import torch

from tests.gpu_util import assert_close_rel, bf16_tensor, randn, to_np

pytestmark = pytest.mark.gpu

# (B, H, T, Dh, window): the second call has fewer rows than the first
CALLS = [(2, 3, 200, 128, 0), (1, 2, 97, 64, 33)]


def _inputs(B, H, T, Dh, seed):
    rng = np.random.default_rng(seed)
    q, k, v, do = (randn(rng, B, H, T, Dh) for _ in range(4))
    return [bf16_tensor(a) for a in (q, k, v, do)]


def _run(S, B, H, T, Dh, window, seed, noalloc):
    q, k, v, do = _inputs(B, H, T, Dh, seed)
    strides = (H * T * Dh, T * Dh, Dh)
    o = torch.zeros_like(q)
    lse = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
    S.attention_fwd(q, k, v, o, lse, window, strides, strides, B, H, T, Dh)
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if noalloc:
        S.attention_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, window, strides, strides, B, H, T, Dh,
                                status=st)
    else:
        delta = S.attention_bwd_scratch(B, H, T)
        S.attention_bwd(q, k, v, o, do, lse, delta, dq, dk, dv, window, strides, strides, B, H, T, Dh,
                        status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return [to_np(t) for t in (dq, dk, dv)]


def test_noalloc_attention_bwd_matches_allocating_entry_point():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gpt_decoder_pretraining_b200 import step as S
    refs = [_run(S, *c, seed=40 + i, noalloc=False) for i, c in enumerate(CALLS)]
    # two calls in a row on the shared array, then the same two again
    for _ in range(2):
        for i, c in enumerate(CALLS):
            got = _run(S, *c, seed=40 + i, noalloc=True)
            for name, g, r in zip(("dq", "dk", "dv"), got, refs[i]):
                assert np.all(np.isfinite(g)), name
                assert_close_rel(g, r, rel=3e-2, cos=0.999, what=f"{name} call {i}")


def test_noalloc_attention_bwd_rejects_more_rows_than_the_array_holds():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gpt_decoder_pretraining_b200 import step as S
    t = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(64, dtype=torch.float32, device="cuda")
    B, H, T, Dh = 1, 16, 65537, 64  # 2·1·16·65600 scratch values > 2^21
    with pytest.raises(S.GptError) as e:
        S.attention_bwd_noalloc(t, t, t, t, t, lse, t, t, t, 0, (H * T * Dh, T * Dh, Dh),
                                (H * T * Dh, T * Dh, Dh), B, H, T, Dh)
    assert e.value.status == -2
