"""Parity of the 8-bit path (needs a B200): gpt_quantize_e4m3 gives bit-identical codes and the same
dequantisation factor as the oracle (both decide every code in fp32), and gpt_gemm_e4m3 (tcgen05
kind::f8f6f4) matches the oracle's exact product of the decoded codes within the bf16 rounding of
its output, on ragged shapes and on a shape whose tail is split along K."""
import numpy as np
import pytest
import torch

from oracle import fp8_oracle as F8
from tests.gpu_util import assert_close_rel, bf16_tensor, randn, to_np

pytestmark = pytest.mark.gpu

S = None


def setup_module(module):
    global S
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gpt_decoder_pretraining_b200 import step
    S = step
    S.lib()


def _quantize(x):
    t = bf16_tensor(x)
    q = torch.empty(x.size, dtype=torch.uint8, device="cuda")
    dq = torch.zeros(1, dtype=torch.float32, device="cuda")
    S.quantize_e4m3(t, q, dq)
    return q.reshape(x.shape), dq


@pytest.mark.parametrize("n,scale", [(1 << 20, 1.0), (1000003, 0.01), (77, 300.0)])
def test_quantize_codes_bit_exact(n, scale):
    rng = np.random.default_rng(n)
    x = randn(rng, n, scale=scale)
    q, dq = _quantize(x)
    torch.cuda.synchronize()
    ref_q, ref_dq = F8.quantize_per_tensor(x.astype(np.float32))
    assert np.array_equal(q.cpu().numpy(), ref_q)
    assert np.float32(dq.item()) == ref_dq


@pytest.mark.parametrize("M,N,K", [(300, 200, 144), (1024, 768, 2048), (3000, 1704, 2560)])
def test_gemm_e4m3_matches_oracle(M, N, K):
    rng = np.random.default_rng(M + N + K)
    a = randn(rng, M, K)
    b = randn(rng, N, K, scale=0.05)
    qa, dqa = _quantize(a)
    qb, dqb = _quantize(b)
    C = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.gemm_e4m3(qa, qb, C, dqa, dqb, M, N, K, alpha=0.5, status=st)
    C2 = torch.zeros_like(C)
    S.gemm_e4m3(qa, qb, C2, dqa, dqb, M, N, K, alpha=0.5, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ra, rda = F8.quantize_per_tensor(a.astype(np.float32))
    rb, rdb = F8.quantize_per_tensor(b.astype(np.float32))
    ref = F8.gemm_e4m3(ra, rb, rda, rdb, alpha=0.5)
    assert_close_rel(to_np(C), ref, rel=8e-3, cos=0.99999, what="e4m3 gemm")
    assert torch.equal(C, C2)
    # and the 8-bit product approximates the bf16 one to the quantisation error
    assert_close_rel(to_np(C), 0.5 * a @ b.T, rel=0.15, cos=0.99, what="vs bf16 product")


def test_gemm_e4m3_rejects_rows_that_break_16_byte_alignment():
    # K = 136 one-byte codes per row: the row stride is not a multiple of 16 bytes (TMA)
    M, N, K = 64, 64, 136
    qa = torch.zeros(M, K, dtype=torch.uint8, device="cuda")
    qb = torch.zeros(N, K, dtype=torch.uint8, device="cuda")
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    C = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(S.GptError, match="UNSUPPORTED_SHAPE"):
        S.gemm_e4m3(qa, qb, C, one, one, M, N, K)
