"""Oracle parity of the attention kernels on the causal-attention sweep workload (needs a B200).

The sweep times attention alone on bf16 q, k, v, dO ~ N(0, 1) (not QK-normalised), 8 heads,
batch·heads·seq_len = 2^21, head_dim 64 and 128, seq_len 512, 2048 and 8192, full causal or a
1024-key window.  These tests run exactly that: the seeded sweep inputs, the whole batch through the
C ABI in the launch configuration the benchmark uses (forward with the measured key-norm bound,
backward with the stored dSᵀ), and compare the outputs element by element with the fp64 oracle on
a few (batch, head) slices — the first, one in the middle and the last — since the oracle's
T×T probabilities do not fit the whole batch.  Every other slice is checked for finiteness, and
both status words must stay 0.

A long-sequence test runs T = 32768 with a 1024-key window, where one batch's dS would exceed the
backward's dS bound, so dQ recomputes the scores: outputs are compared with the oracle on
sub-sequences that hold every key a checked output depends on.

Another test raises the norms of q and k until the fixed softmax shift ‖q‖·max‖k‖/√Dh exceeds 40
(where exp of the shifted scores may underflow in fp32): the forward must report
GPT_ERR_NUMERIC_RANGE instead of passing wrong values off as valid.
"""
import math

import numpy as np
import pytest
import torch

from gpt_decoder_pretraining_b200.inputs import make_attention_inputs, round_to_bf16
from oracle import gpt_oracle as O
from tests.gpu_util import assert_close_rel, bf16_tensor, to_np

pytestmark = pytest.mark.gpu

HEADS = 8
ROWS = 1 << 21
SWEEP = [(512, 64), (512, 128), (2048, 64), (2048, 128), (8192, 64), (8192, 128)]
WINDOWS = [0, 1024]

S = None


def setup_module(module):
    global S
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gpt_decoder_pretraining_b200 import step
    S = step
    S.lib()


def _slices(B):
    return sorted({(0, 0), (B // 2, 3), (B - 1, HEADS - 1)})


@pytest.mark.parametrize("T,Dh", SWEEP)
def test_sweep_shapes_match_oracle(T, Dh):
    B = ROWS // (HEADS * T)
    q, k, v, do = make_attention_inputs(B, HEADS, T, Dh)
    tq, tk, tv, tdo = (torch.from_numpy(a).cuda().to(torch.bfloat16) for a in (q, k, v, do))
    strides = (HEADS * T * Dh, T * Dh, Dh)
    delta = S.attention_bwd_scratch(B, HEADS, T)
    for window in WINDOWS:
        o = torch.zeros_like(tq)
        lse = torch.zeros(B, HEADS, T, dtype=torch.float32, device="cuda")
        dq, dk, dv = (torch.full_like(tq, float("nan")) for _ in range(3))
        st_f = torch.zeros(1, dtype=torch.int32, device="cuda")
        st_b = torch.zeros(1, dtype=torch.int32, device="cuda")
        S.attention_fwd(tq, tk, tv, o, lse, window, strides, strides, B, HEADS, T, Dh, status=st_f)
        S.attention_bwd(tq, tk, tv, o, tdo, lse, delta, dq, dk, dv, window, strides, strides, B, HEADS,
                        T, Dh, status=st_b)
        torch.cuda.synchronize()
        assert int(st_f.item()) == 0 and int(st_b.item()) == 0, (window, st_f.item(), st_b.item())
        for t in (o, lse, dq, dk, dv):
            assert bool(torch.isfinite(t).all())
        floor = 2.0 ** -9 * math.sqrt(Dh)
        for b, h in _slices(B):
            sl = (slice(b, b + 1), slice(h, h + 1))
            qs, ks, vs, dos = (a[sl].astype(np.float64) for a in (q, k, v, do))
            o_ref, lse_ref = O.attention_batch_forward(qs, ks, vs, window)
            dq_ref, dk_ref, dv_ref = O.attention_batch_backward(qs, ks, vs, dos, window)
            what = f"T={T} Dh={Dh} w={window} (b={b}, h={h})"
            assert_close_rel(to_np(o[sl]), o_ref, rel=2e-2, cos=0.9999, what="o " + what)
            np.testing.assert_allclose(to_np(lse[sl]), lse_ref, atol=2e-3, err_msg="lse " + what)
            assert_close_rel(to_np(dq[sl]), dq_ref, rel=3e-2, cos=0.999, what="dq " + what, atol=floor)
            assert_close_rel(to_np(dk[sl]), dk_ref, rel=3e-2, cos=0.999, what="dk " + what, atol=floor)
            assert_close_rel(to_np(dv[sl]), dv_ref, rel=3e-2, cos=0.999, what="dv " + what, atol=floor)
        del o, lse, dq, dk, dv


@pytest.mark.parametrize("Dh", [64, 128])
def test_scores_beyond_the_shift_bound_are_reported(Dh):
    B, H, T = 1, 2, 256
    rng = np.random.default_rng(21)
    # ‖q‖ ≈ ‖k‖ ≈ 4·√Dh, so ‖q‖·max‖k‖/√Dh ≈ 16·√Dh ≥ 128 > 40
    q, k, v = (round_to_bf16(rng.standard_normal((B, H, T, Dh)).astype(np.float32) * s)
               for s in (4.0, 4.0, 1.0))
    tq, tk, tv = (bf16_tensor(a) for a in (q, k, v))
    strides = (H * T * Dh, T * Dh, Dh)
    o = torch.zeros_like(tq)
    lse = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.attention_fwd(tq, tk, tv, o, lse, 0, strides, strides, B, H, T, Dh, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == -8
    # the same inputs scaled back below the bound are accepted and correct
    q2, k2 = (round_to_bf16((a / 4.0).astype(np.float32)) for a in (q, k))
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.attention_fwd(bf16_tensor(q2), bf16_tensor(k2), tv, o, lse, 0, strides, strides, B, H, T, Dh, status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    o_ref, _ = O.attention_batch_forward(q2, k2, v, 0)
    assert_close_rel(to_np(o), o_ref, rel=2e-2, cos=0.9999, what="o below the bound")


def test_long_sequence_backward_without_stored_ds():
    """T = 32768, H 8, Dh 128, window W = 1024: dS for one batch would be 16 GiB, above the 8 GiB
    bound, so the backward stores none and the dQ kernel recomputes the scores.  With a window, the
    outputs of query t depend only on positions (t − W, t], so the oracle on the sub-sequence
    [t0 − W + 1, t0 + R) reproduces o, LSE and dq of queries [t0, t0 + R) exactly, and dk, dv of keys
    [t0, t0 + R − W + 1), whose queries all lie in that range; the sub-sequence [0, R) needs no
    left margin.  Checked on the first and last head, R = 2W, at both ends of the sequence."""
    B, H, T, Dh, W = 1, HEADS, 32768, 128, 1024
    assert S.attention_bwd_scratch_bytes(B, H, T) == B * H * T * 8  # no dS held
    q, k, v, do = make_attention_inputs(B, H, T, Dh, seed=5)
    tq, tk, tv, tdo = (torch.from_numpy(a).cuda().to(torch.bfloat16) for a in (q, k, v, do))
    strides = (H * T * Dh, T * Dh, Dh)
    delta = S.attention_bwd_scratch(B, H, T)
    o = torch.zeros_like(tq)
    lse = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
    dq, dk, dv = (torch.full_like(tq, float("nan")) for _ in range(3))
    st_f = torch.zeros(1, dtype=torch.int32, device="cuda")
    st_b = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.attention_fwd(tq, tk, tv, o, lse, W, strides, strides, B, H, T, Dh, status=st_f)
    S.attention_bwd(tq, tk, tv, o, tdo, lse, delta, dq, dk, dv, W, strides, strides, B, H, T, Dh,
                    status=st_b)
    torch.cuda.synchronize()
    assert int(st_f.item()) == 0 and int(st_b.item()) == 0
    for t in (o, lse, dq, dk, dv):
        assert bool(torch.isfinite(t).all())
    R = 2 * W
    floor = 2.0 ** -9 * math.sqrt(Dh)
    for h in (0, H - 1):
        for t0 in (0, T - R):
            lo = max(0, t0 - W + 1)
            sl = (slice(0, 1), slice(h, h + 1), slice(lo, t0 + R))
            qs, ks, vs, dos = (a[sl].astype(np.float64) for a in (q, k, v, do))
            o_ref, lse_ref = O.attention_batch_forward(qs, ks, vs, W)
            dq_ref, dk_ref, dv_ref = O.attention_batch_backward(qs, ks, vs, dos, W)
            rq = slice(t0 - lo, t0 - lo + R)            # queries checked, within the sub-sequence
            rk = slice(t0 - lo, t0 - lo + R - W + 1)    # keys checked
            gq = (slice(0, 1), slice(h, h + 1), slice(t0, t0 + R))
            gk = (slice(0, 1), slice(h, h + 1), slice(t0, t0 + R - W + 1))
            what = f"T={T} w={W} h={h} t0={t0}"
            assert_close_rel(to_np(o[gq]), o_ref[:, :, rq], rel=2e-2, cos=0.9999, what="o " + what)
            np.testing.assert_allclose(to_np(lse[gq]), lse_ref[:, :, rq], atol=2e-3, err_msg="lse " + what)
            assert_close_rel(to_np(dq[gq]), dq_ref[:, :, rq], rel=3e-2, cos=0.999, what="dq " + what, atol=floor)
            assert_close_rel(to_np(dk[gk]), dk_ref[:, :, rk], rel=3e-2, cos=0.999, what="dk " + what, atol=floor)
            assert_close_rel(to_np(dv[gk]), dv_ref[:, :, rk], rel=3e-2, cos=0.999, what="dv " + what, atol=floor)
