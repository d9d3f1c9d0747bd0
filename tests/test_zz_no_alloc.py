"""gpt_attention_bwd_noalloc — the attention backward for callers that cannot allocate device
memory where they call it — checked against the oracle and against gpt_attention_bwd, the entry
point that takes a caller-allocated scratch buffer (needs a B200).

This file is collected last on purpose.  The calls run back to back on the one shared static
scratch array; each later call uses fewer rows than an earlier one, so the array still holds rows of
the earlier call beyond what the later one writes (the head_dim-32 call, which takes a different
kernel path with no extension rows, comes after a larger head_dim-128 call).  The test must pass
both on its own in a fresh process and after every other test.
"""
import math

import numpy as np
import pytest
import torch

from oracle import gpt_oracle as O
from tests.gpu_util import assert_close_rel, bf16_tensor, randn, to_np

pytestmark = pytest.mark.gpu

# (B, H, T, Dh, window): each call has fewer rows than the one before it
CALLS = [(2, 3, 200, 128, 0), (1, 2, 97, 64, 33), (1, 2, 77, 32, 9)]
# the largest shape the static array serves: B·H·⌈T/64⌉·64 = 1,048,576 rows of 8 bytes
LIMIT_CASE = (16384, 1, 64, 64, 0)


def _inputs(B, H, T, Dh, seed):
    rng = np.random.default_rng(seed)
    return [randn(rng, B, H, T, Dh) for _ in range(4)]


def _run(S, B, H, T, Dh, window, arrays, noalloc):
    q, k, v, do = (bf16_tensor(a) for a in arrays)
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


def test_noalloc_attention_bwd_matches_oracle_and_allocating_entry_point():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gpt_decoder_pretraining_b200 import step as S
    inputs = [_inputs(*c[:4], seed=40 + i) for i, c in enumerate(CALLS)]
    oracle = [O.attention_batch_backward(*inp[:3], inp[3], c[4]) for c, inp in zip(CALLS, inputs)]
    refs = [_run(S, *c, inp, noalloc=False) for c, inp in zip(CALLS, inputs)]
    # the calls in a row on the shared array, then all of them again
    for _ in range(2):
        for i, c in enumerate(CALLS):
            got = _run(S, *c, inputs[i], noalloc=True)
            floor = 2.0 ** -9 * math.sqrt(c[3])
            for name, g, r, o in zip(("dq", "dk", "dv"), got, refs[i], oracle[i]):
                assert np.all(np.isfinite(g)), name
                assert_close_rel(g, o, rel=3e-2, cos=0.999, what=f"{name} call {i} vs oracle", atol=floor)
                assert_close_rel(g, r, rel=3e-2, cos=0.999, what=f"{name} call {i} vs allocating entry")


def test_noalloc_attention_bwd_serves_its_largest_shape():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gpt_decoder_pretraining_b200 import step as S
    B, H, T, Dh, window = LIMIT_CASE
    assert B * H * ((T + 63) // 64 * 64) * 8 <= 4 * (1 << 21)
    arrays = _inputs(B, H, T, Dh, seed=77)
    ref = _run(S, B, H, T, Dh, window, arrays, noalloc=False)
    got = _run(S, B, H, T, Dh, window, arrays, noalloc=True)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert_close_rel(g, r, rel=3e-2, cos=0.999, what=f"{name} at the row limit")
    # spot-check two (b, h) slices against the oracle
    q, k, v, do = arrays
    for b in (0, B - 1):
        sl = slice(b, b + 1)
        o_ref = O.attention_batch_backward(q[sl], k[sl], v[sl], do[sl], window)
        for name, g, r in zip(("dq", "dk", "dv"), got, o_ref):
            assert_close_rel(g[sl], r, rel=3e-2, cos=0.999, what=f"{name} b={b}", atol=2.0 ** -9 * math.sqrt(Dh))
