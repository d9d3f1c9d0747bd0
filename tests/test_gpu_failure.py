"""Failure handling and approximations of the kernels, tested on a B200 without faulting it.

* Bounded waits: every mbarrier wait of the GEMM and attention kernels gives up after a limit that
  gpt_set_wait_limit sets.  A probe kernel waits on a barrier that nothing completes; then a GEMM
  and an attention forward/backward run with a limit of a few dozen cycles, so that their ordinary
  waits (a TMA load in flight) run out.  Each must come back with GPT_ERR_DEVICE_TIMEOUT in its
  status word and return (no trap, no hang), and the same context must then compute correct results
  at the default limit.
* The forward's FMA-pipe exponential (a fitted cubic for 2^f plus exponent insertion) against the
  exact 2^x, over the whole range the softmax uses.
"""
import math

import numpy as np
import pytest
import torch

from oracle import gpt_oracle as O
from tests.gpu_util import f32_accum_rel, assert_close_rel, bf16_tensor, randn, to_np

pytestmark = pytest.mark.gpu

TIMEOUT = -5
TINY_LIMIT = 64  # SM cycles: far below the latency of one TMA load

S = None


def setup_module(module):
    global S
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gpt_decoder_pretraining_b200 import step
    S = step
    S.lib()


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _gemm_case(seed=3, M=512, N=768, K=640):
    rng = np.random.default_rng(seed)
    A, B = randn(rng, M, K), randn(rng, N, K)
    return A, B, A @ B.T


def test_exp2_poly2_relative_error_bound():
    x = np.concatenate([np.linspace(-126.0, 1.0, 2_000_001), np.random.default_rng(0).uniform(-126, 1, 1 << 20)])
    x = x.astype(np.float32)
    tx = torch.from_numpy(x).cuda()
    ty = torch.empty_like(tx)
    S.debug_exp2_poly2(tx, ty)
    torch.cuda.synchronize()
    y = ty.cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    normal = x >= -125.0
    rel = np.abs(y[normal] - ref[normal]) / ref[normal]
    assert rel.max() <= 7.6e-5, rel.max()
    # next to the clamp at −126 the exponent insertion leaves the normal range: the result stays
    # within 2^-125 of the exact value (weights this small vanish in any softmax row sum)
    assert np.abs(y[~normal] - ref[~normal]).max() <= 2.0 ** -125
    # below the clamp the value of 2^-126 is returned
    lo = torch.tensor([-130.0, -200.0], dtype=torch.float32, device="cuda")
    ylo = torch.empty_like(lo)
    S.debug_exp2_poly2(lo, ylo)
    torch.cuda.synchronize()
    assert np.all(np.abs(ylo.cpu().numpy()) <= 2.0 ** -125)


def test_wait_probe_times_out_and_the_context_survives():
    st = _status()
    try:
        S.set_wait_limit(20000)
        S.debug_wait_probe(st)
        torch.cuda.synchronize()
    finally:
        S.set_wait_limit(0)
    assert int(st.item()) == TIMEOUT
    A, B, ref = _gemm_case()
    C = torch.zeros(ref.shape, dtype=torch.float32, device="cuda")
    st2 = _status()
    S.gemm(S.GEMM_NT, S.EPI_F32, bf16_tensor(A), bf16_tensor(B), C, *ref.shape, A.shape[1], status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    assert_close_rel(to_np(C), ref, rel=1e-5, cos=0.9999999, what="gemm after the probe")


@pytest.mark.parametrize("op", [0, 2])
def test_gemm_wait_timeout_returns_status_then_recovers(op):
    # one 256×256 tile with a long K: the epilogue warps wait for the accumulator through 512
    # k-steps, far longer than the time one mbarrier.try_wait may suspend before it reports "not yet"
    A, B, ref = _gemm_case(seed=4 + op, M=256, N=256, K=32768)
    M, N = ref.shape
    K = A.shape[1]
    tA = bf16_tensor(A if op == 0 else np.ascontiguousarray(A.T))   # TN takes A as [K, M]
    tB = bf16_tensor(B if op == 0 else np.ascontiguousarray(B.T))   # TN takes B as [K, N]
    C = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    st = _status()
    try:
        S.set_wait_limit(TINY_LIMIT)
        S.gemm(op, S.EPI_F32, tA, tB, C, M, N, K, status=st, scratch=None)
        torch.cuda.synchronize()
    finally:
        S.set_wait_limit(0)
    assert int(st.item()) == TIMEOUT
    st2 = _status()
    C.zero_()
    S.gemm(op, S.EPI_F32, tA, tB, C, M, N, K, status=st2, scratch=None)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    assert_close_rel(to_np(C), ref, rel=f32_accum_rel(K), cos=0.9999999, what="gemm after recovery")


def test_attention_wait_timeout_returns_status_then_recovers():
    B, H, T, Dh, window = 1, 2, 300, 128, 0
    rng = np.random.default_rng(9)
    q, k, v, do = (randn(rng, B, H, T, Dh) for _ in range(4))
    tq, tk, tv, tdo = (bf16_tensor(a) for a in (q, k, v, do))
    strides = (H * T * Dh, T * Dh, Dh)
    o = torch.zeros_like(tq)
    lse = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
    dq, dk, dv = (torch.zeros_like(tq) for _ in range(3))
    delta = S.attention_bwd_scratch(B, H, T)
    st_f, st_b = _status(), _status()
    try:
        S.set_wait_limit(TINY_LIMIT)
        S.attention_fwd(tq, tk, tv, o, lse, window, strides, strides, B, H, T, Dh, status=st_f)
        S.attention_bwd(tq, tk, tv, o, tdo, lse, delta, dq, dk, dv, window, strides, strides, B, H, T, Dh,
                        status=st_b)
        torch.cuda.synchronize()
    finally:
        S.set_wait_limit(0)
    assert int(st_f.item()) == TIMEOUT
    assert int(st_b.item()) == TIMEOUT
    # the same context, default limit: correct results
    st = _status()
    S.attention_fwd(tq, tk, tv, o, lse, window, strides, strides, B, H, T, Dh, status=st)
    S.attention_bwd(tq, tk, tv, o, tdo, lse, delta, dq, dk, dv, window, strides, strides, B, H, T, Dh,
                    status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    o_ref, lse_ref = O.attention_batch_forward(q, k, v, window)
    dq_ref, dk_ref, dv_ref = O.attention_batch_backward(q, k, v, do, window)
    assert_close_rel(to_np(o), o_ref, rel=2e-2, cos=0.9999, what="o")
    np.testing.assert_allclose(to_np(lse), lse_ref, atol=2e-3)
    floor = 2.0 ** -9 * math.sqrt(Dh)
    for name, g, r in (("dq", dq, dq_ref), ("dk", dk, dk_ref), ("dv", dv, dv_ref)):
        assert_close_rel(to_np(g), r, rel=3e-2, cos=0.999, what=name, atol=floor)
