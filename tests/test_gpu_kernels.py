"""Kernel-level parity of the CUDA path against the oracle's definitions (needs a B200).

Every call goes through the C ABI of libgptstep.so.  Inputs are seeded and bf16-exact; the
references are the oracle's functions (or, for the GEMM, the fp64 matrix product that defines it)
evaluated in float64 on the same values.  Sizes span several tiles and ragged tails.
"""
import math

import numpy as np
import pytest
import torch

from oracle import gpt_oracle as O
from tests.gpu_util import f32_accum_rel, assert_close_rel, bf16_tensor, cosine, randn, to_np

pytestmark = pytest.mark.gpu

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


# --------------------------------------------------------------------------------------------------
# GEMM: the three operand layouts and every epilogue
# --------------------------------------------------------------------------------------------------
GEMM_SHAPES = [(128, 64, 64), (296, 200, 200), (256, 520, 640), (136, 384, 96), (2048, 2560, 256)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
@pytest.mark.parametrize("op", [0, 1, 2])
def test_gemm_layouts_bf16_and_f32(op, M, N, K):
    rng = np.random.default_rng(M * 7 + N * 3 + K + op)
    A = randn(rng, *( (K, M) if op == 2 else (M, K) ))
    B = randn(rng, *( (N, K) if op == 0 else (K, N) ))
    ref = (A.T if op == 2 else A) @ (B.T if op == 0 else B)
    tA, tB = bf16_tensor(A), bf16_tensor(B)
    st = _status()
    C = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    S.gemm(op, S.EPI_BF16, tA, tB, C, M, N, K, status=st)
    Cf = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    S.gemm(op, S.EPI_F32, tA, tB, Cf, M, N, K, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_close_rel(to_np(C), ref, rel=8e-3, what="bf16 out")
    assert_close_rel(to_np(Cf), ref, rel=1e-5, cos=0.9999999, what="f32 out")


@pytest.mark.parametrize("M,N,K", [(300, 200, 200), (256, 520, 640)])
def test_gemm_epilogues(M, N, K):
    rng = np.random.default_rng(11)
    A, B = randn(rng, M, K), randn(rng, N, K)
    acc = A @ B.T
    tA, tB = bf16_tensor(A), bf16_tensor(B)
    # residual add in place
    X = randn(rng, M, N, scale=3.0)
    tX = bf16_tensor(X)
    S.gemm(0, S.EPI_RESID, tA, tB, tX, M, N, K)
    # ReLU²: h = max(acc, 0)²
    Ch = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    S.gemm(0, S.EPI_RELU2, tA, tB, Ch, M, N, K)
    # dReLU² from the saved h: acc·2·√h
    taux = bf16_tensor(np.maximum(randn(rng, M, N), 0) ** 2)
    aux = to_np(taux).astype(np.float64)
    Cd = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    S.gemm(0, S.EPI_DRELU2, tA, tB, Cd, M, N, K, aux=taux)
    # fp32 accumulate
    base = rng.standard_normal((M, N)).astype(np.float32)
    Cf = torch.from_numpy(base).cuda()
    S.gemm(0, S.EPI_F32_ADD, tA, tB, Cf, M, N, K)
    torch.cuda.synchronize()
    assert_close_rel(to_np(tX), X + acc, rel=8e-3, what="resid")
    r = np.maximum(acc, 0)
    assert_close_rel(to_np(Ch), r * r, rel=8e-3, what="relu2")
    assert_close_rel(to_np(Cd), acc * 2 * np.sqrt(aux), rel=8e-3, what="drelu2")
    assert_close_rel(to_np(Cf), base + acc, rel=1e-5, cos=0.9999999, what="f32 add")


# Shapes whose tile count leaves the last wave of CTA pairs partly empty, so that the GEMM splits
# the tail tiles along K: fewer tiles than CTA pairs (every tile in two pieces), a weight-gradient
# shape of 100 tiles (one whole wave, 26 tail tiles in two pieces), and 84 ragged tiles.
SK_SHAPES = [(1536, 1536, 16384, 2), (1280, 5120, 8192, 2), (3000, 1704, 2560, 0), (3000, 1704, 2560, 1)]


@pytest.mark.parametrize("M,N,K,op", SK_SHAPES)
def test_gemm_stream_k_tail_matches_fp64_and_is_reproducible(M, N, K, op):
    rng = np.random.default_rng(M + N + K + op)
    A = randn(rng, *((K, M) if op == 2 else (M, K)))
    B = randn(rng, *((N, K) if op == 0 else (K, N)))
    ref = (A.T if op == 2 else A) @ (B.T if op == 0 else B)
    tA, tB = bf16_tensor(A), bf16_tensor(B)
    st = _status()
    C1 = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    C2 = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    S.gemm(op, S.EPI_F32, tA, tB, C1, M, N, K, status=st)
    S.gemm(op, S.EPI_F32, tA, tB, C2, M, N, K, status=st)
    Cn = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    S.gemm(op, S.EPI_F32, tA, tB, Cn, M, N, K, status=st, scratch=None)  # every tile whole
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    tol = f32_accum_rel(K)
    assert_close_rel(to_np(C1), ref, rel=tol, cos=0.9999999, what="f32 split tail")
    assert torch.equal(C1, C2)  # bitwise reproducible
    assert_close_rel(to_np(Cn), ref, rel=tol, cos=0.9999999, what="f32 whole tiles")
    # both within tol of the fp64 product: they differ from each other only by fp32 summation order
    assert_close_rel(to_np(C1), to_np(Cn), rel=2 * tol, cos=0.9999999, what="split vs whole tiles")
    if op == 2:
        return
    # the element-wise epilogues on the same split schedule
    acc = ref
    X = randn(rng, M, N, scale=3.0)
    tX = bf16_tensor(X)
    S.gemm(op, S.EPI_RESID, tA, tB, tX, M, N, K, status=st)
    taux = bf16_tensor(np.maximum(randn(rng, M, N), 0) ** 2)
    aux = to_np(taux)
    Cd = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    S.gemm(op, S.EPI_DRELU2, tA, tB, Cd, M, N, K, aux=taux, status=st)
    Ch = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    S.gemm(op, S.EPI_RELU2, tA, tB, Ch, M, N, K, status=st)
    base = rng.standard_normal((M, N)).astype(np.float32)
    Cf = torch.from_numpy(base).cuda()
    S.gemm(op, S.EPI_F32_ADD, tA, tB, Cf, M, N, K, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_close_rel(to_np(tX), X + acc, rel=8e-3, what="resid")
    assert_close_rel(to_np(Cd), acc * 2 * np.sqrt(aux), rel=8e-3, what="drelu2")
    r = np.maximum(acc, 0)
    assert_close_rel(to_np(Ch), r * r, rel=8e-3, what="relu2")
    assert_close_rel(to_np(Cf), base + acc, rel=1e-5, cos=0.9999999, what="f32 add")


# the four weight gradients of one layer in one launch: small ragged sizes; the d20 layer shapes
# (75 + 25 + 100 + 100 tiles of 256 × 256, every tile whole at K = 4096); and 32 + 16 + 24 + 6 = 78
# tiles at K = 16384, one whole wave of 74 pairs and 4 tail tiles split along K
GROUP_CASES = [
    (512, [(296, 200), (136, 384), (520, 256), (64, 64)]),
    (4096, [(3840, 1280), (1280, 1280), (5120, 1280), (1280, 5120)]),
    (16384, [(2048, 1024), (1024, 1024), (1536, 1024), (768, 512)]),
]


@pytest.mark.parametrize("K,shapes", GROUP_CASES)
def test_gemm_group_tn_matches_fp64_and_single_products(K, shapes):
    rng = np.random.default_rng(K + len(shapes))
    probs, refs = [], []
    for M, N in shapes:
        A, B = randn(rng, K, M), randn(rng, K, N)
        refs.append(A.T @ B)
        probs.append((bf16_tensor(A), bf16_tensor(B), torch.full((M, N), float("nan"), device="cuda")))
    st = _status()
    S.gemm_group_tn(probs, K, S.EPI_F32, status=st)
    again = [torch.full_like(c, float("nan")) for _, _, c in probs]
    S.gemm_group_tn([(a, b, c) for (a, b, _), c in zip(probs, again)], K, S.EPI_F32, status=st)
    # accumulate form on a base
    bases = [rng.standard_normal(r.shape).astype(np.float32) for r in refs]
    accs = [torch.from_numpy(b).cuda() for b in bases]
    S.gemm_group_tn([(a, b, c) for (a, b, _), c in zip(probs, accs)], K, S.EPI_F32_ADD, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    tol = f32_accum_rel(K)
    for (a, b, c), c2, acc, base, ref, (M, N) in zip(probs, again, accs, bases, refs, shapes):
        assert_close_rel(to_np(c), ref, rel=tol, cos=0.9999999, what=f"grouped {M}x{N}")
        assert torch.equal(c, c2)  # bitwise reproducible
        assert_close_rel(to_np(acc), base + ref, rel=tol, cos=0.9999999, what=f"grouped add {M}x{N}")
        one = torch.zeros_like(c)
        S.gemm(2, S.EPI_F32, a, b, one, M, N, K, status=st)
        torch.cuda.synchronize()
        # the same products on their own differ only in fp32 summation order (split tiles)
        assert_close_rel(to_np(c), to_np(one), rel=2 * tol, cos=0.9999999, what=f"grouped vs single {M}x{N}")


def test_gemm_rejects_bad_arguments():
    t = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(S.GptError):
        S.gemm(0, S.EPI_BF16, t, t, t, 0, 64, 64)
    with pytest.raises(S.GptError):
        S.gemm(7, S.EPI_BF16, t, t, t, 64, 64, 64)
    with pytest.raises(S.GptError):
        S.gemm(0, 99, t, t, t, 64, 64, 64)


# --------------------------------------------------------------------------------------------------
# RMSNorm
# --------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("rows,d", [(1, 64), (77, 768), (300, 1536)])
def test_rmsnorm_fwd_bwd(rows, d):
    rng = np.random.default_rng(rows + d)
    x = randn(rng, rows, d, scale=2.0)
    dy = randn(rng, rows, d)
    g0 = rng.standard_normal((rows, d))
    y_ref, rho_ref = O.rmsnorm(x)
    tx = bf16_tensor(x)
    ty = torch.empty_like(tx)
    rho = torch.empty(rows, dtype=torch.float32, device="cuda")
    S.rmsnorm_fwd(tx, ty, rho)
    torch.cuda.synchronize()
    assert_close_rel(to_np(ty), y_ref, rel=8e-3, what="y")
    np.testing.assert_allclose(to_np(rho), rho_ref[:, 0], rtol=1e-5)
    # backward with y as stored by the forward (bf16) and accumulate into g0
    y_b = to_np(ty)
    ref = g0 + O.rmsnorm_backward(dy, y_b, to_np(rho)[:, None])
    gx = torch.from_numpy(g0.astype(np.float32)).cuda()
    gxb = torch.empty(rows, d, dtype=torch.bfloat16, device="cuda")
    S.rmsnorm_bwd(bf16_tensor(dy), ty, rho, gx, gxb, accumulate=True)
    gx2 = torch.zeros(rows, d, dtype=torch.float32, device="cuda")
    S.rmsnorm_bwd(torch.from_numpy(dy.astype(np.float32)).cuda(), ty, rho, gx2, None, accumulate=False)
    torch.cuda.synchronize()
    assert_close_rel(to_np(gx), ref, rel=1e-5, cos=0.9999999, what="gx")
    assert_close_rel(to_np(gxb), ref, rel=8e-3, what="gx bf16")
    assert_close_rel(to_np(gx2), ref - g0, rel=1e-5, cos=0.9999999, what="gx f32 dy")


# --------------------------------------------------------------------------------------------------
# RoPE + QK-norm
# --------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("B,T,H,Dh", [(1, 5, 2, 32), (2, 130, 3, 64), (1, 257, 2, 128)])
def test_rope_qknorm_fwd_bwd(B, T, H, Dh):
    rng = np.random.default_rng(B * 100 + T + Dh)
    d = H * Dh
    qkv = randn(rng, B * T, 3 * d, scale=1.5)
    dqkv = randn(rng, B * T, 3 * d)
    cs = torch.empty(T * Dh, dtype=torch.float32, device="cuda")
    S.rope_table(cs, T, Dh)
    tq = bf16_tensor(qkv)
    rq = torch.empty(B * T * H, dtype=torch.float32, device="cuda")
    rk = torch.empty_like(rq)
    S.rope_qknorm_fwd(tq, rq, rk, cs, B, T, H, Dh)
    torch.cuda.synchronize()
    cos, sin = O.rope_angles(T, Dh, np.float64)
    got = to_np(tq).reshape(B, T, 3, H, Dh)
    x = qkv.reshape(B, T, 3, H, Dh)
    for b in range(B):
        for part in range(2):
            ref, rho = O.rmsnorm(O.rope(x[b, :, part], cos, sin))
            assert_close_rel(got[b, :, part], ref, rel=1e-2, what=f"fwd part {part}")
            r_got = to_np(rq if part == 0 else rk).reshape(B, T, H)[b]
            np.testing.assert_allclose(r_got, rho[..., 0], rtol=2e-3)
        assert np.array_equal(got[b, :, 2], x[b, :, 2])  # v untouched
    # backward on the stored forward output
    td = bf16_tensor(dqkv)
    S.rope_qknorm_bwd(td, tq, rq, rk, cs, B, T, H, Dh)
    torch.cuda.synchronize()
    gd = to_np(td).reshape(B, T, 3, H, Dh)
    dx = dqkv.reshape(B, T, 3, H, Dh)
    for b in range(B):
        for part in range(2):
            yv = got[b, :, part]
            rho = to_np(rq if part == 0 else rk).reshape(B, T, H)[b][..., None]
            ref = O.rope_inverse(O.rmsnorm_backward(dx[b, :, part], yv, rho), cos, sin)
            assert_close_rel(gd[b, :, part], ref, rel=1e-2, what=f"bwd part {part}")


@pytest.mark.parametrize("B,T,H,Hkv,Dh", [(1, 130, 2, 2, 128), (2, 64, 3, 3, 64), (1, 96, 4, 4, 32),
                                          (2, 70, 4, 2, 64), (1, 130, 6, 1, 128)])
def test_qkv_proj_rope_matches_gemm_then_rope(B, T, H, Hkv, Dh):
    """The fused projection + RoPE + QK-norm equals the oracle's rope/rmsnorm of r·W_qkvᵀ; with
    grouped key/value heads (Hkv < H) the k and v blocks have Hkv heads."""
    rng = np.random.default_rng(B + T + H + Dh + Hkv)
    d, dkv = H * Dh, Hkv * Dh
    r = randn(rng, B * T, d)
    w = randn(rng, d + 2 * dkv, d, scale=0.05)
    cs = torch.empty(T * Dh, dtype=torch.float32, device="cuda")
    S.rope_table(cs, T, Dh)
    heads = torch.zeros(B * T * (d + 2 * dkv), dtype=torch.bfloat16, device="cuda")
    rq = torch.zeros(B * T * H, dtype=torch.float32, device="cuda")
    rk = torch.zeros(B * T * Hkv, dtype=torch.float32, device="cuda")
    S.qkv_proj_rope(bf16_tensor(r), bf16_tensor(w), heads, rq, rk, cs, B, T, H, Dh, H_kv=Hkv)
    torch.cuda.synchronize()
    qkv = r @ w.T
    cos, sin = O.rope_angles(T, Dh, np.float64)
    flat = to_np(heads)
    parts = [(0, H, qkv[:, :d]), (B * H * T * Dh, Hkv, qkv[:, d:d + dkv]),
             (B * (H + Hkv) * T * Dh, Hkv, qkv[:, d + dkv:])]
    for pi, (base, nh, src) in enumerate(parts):
        got = flat[base:base + B * nh * T * Dh].reshape(B, nh, T, Dh)
        x = src.reshape(B, T, nh, Dh)
        for b in range(B):
            if pi < 2:
                ref, rho = O.rmsnorm(O.rope(x[b], cos, sin))
                r_got = to_np(rq if pi == 0 else rk).reshape(B, T, nh)[b]
                np.testing.assert_allclose(r_got, rho[..., 0], rtol=2e-2)
            else:
                ref = x[b]
            assert_close_rel(got[b].transpose(1, 0, 2), ref, rel=2e-2, what=f"part {pi}")


# --------------------------------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------------------------------
ATTN_CASES = [(1, 1, 1, 64, 0), (2, 2, 63, 64, 0), (1, 2, 128, 32, 0), (2, 1, 77, 32, 9), (1, 3, 200, 128, 0), (2, 1, 200, 128, 17),
              (1, 2, 130, 64, 1), (1, 1, 257, 128, 64), (1, 2, 128, 128, 1000)]


@pytest.mark.parametrize("qk_norm", [True, False], ids=["qknorm", "raw"])
@pytest.mark.parametrize("B,H,T,Dh,window", ATTN_CASES)
def test_attention_fwd_bwd(B, H, T, Dh, window, qk_norm):
    """qk_norm: q and k RMS-normalised per head, as in the model; raw: N(0, 1) q and k as in the
    attention sweep, where the forward's softmax shift comes from the measured key norms."""
    rng = np.random.default_rng(B * 1000 + H * 100 + T + Dh + window)
    q, k, v, do = (randn(rng, B, H, T, Dh) for _ in range(4))
    if qk_norm:
        q = np.asarray([[O.rmsnorm(q[b, h])[0] for h in range(H)] for b in range(B)])
        k = np.asarray([[O.rmsnorm(k[b, h])[0] for h in range(H)] for b in range(B)])
        from gpt_decoder_pretraining_b200.inputs import round_to_bf16
        q = round_to_bf16(q.astype(np.float32)).astype(np.float64)
        k = round_to_bf16(k.astype(np.float32)).astype(np.float64)
    o_ref, lse_ref = O.attention_batch_forward(q, k, v, window)
    dq_ref, dk_ref, dv_ref = O.attention_batch_backward(q, k, v, do, window)
    tq, tk, tv, tdo = (bf16_tensor(a) for a in (q, k, v, do))
    strides = (H * T * Dh, T * Dh, Dh)
    to = torch.zeros(B, H, T, Dh, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
    st = _status()
    S.attention_fwd(tq, tk, tv, to, lse, window, strides, strides, B, H, T, Dh, status=st)
    # the same with the QK-norm bound instead of the measured key norms (valid for normalised k only)
    to_n = torch.zeros_like(to)
    lse_n = torch.zeros_like(lse)
    if qk_norm:
        S.attention_fwd(tq, tk, tv, to_n, lse_n, window, strides, strides, B, H, T, Dh, status=st,
                        qk_normalized=True)
    dq, dk, dv = (torch.zeros_like(tq) for _ in range(3))
    delta = S.attention_bwd_scratch(B, H, T)
    S.attention_bwd(tq, tk, tv, to, tdo, lse, delta, dq, dk, dv, window, strides, strides, B, H, T, Dh,
                    status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_close_rel(to_np(to), o_ref, rel=2e-2, cos=0.9999, what="o")
    np.testing.assert_allclose(to_np(lse), lse_ref, atol=2e-3)
    if qk_norm:
        assert_close_rel(to_np(to_n), o_ref, rel=2e-2, cos=0.9999, what="o (qk-norm bound)")
        np.testing.assert_allclose(to_np(lse_n), lse_ref, atol=2e-3)
    # Absolute floor: O is stored in bf16 (relative rounding 2^-9), so delta = rowsum(dO∘O) and
    # hence dS carry ~2^-9·|dO·v| ≈ 2^-9·√Dh of noise even where the exact dq is 0 (T = 1).
    floor = 2.0 ** -9 * math.sqrt(Dh)
    assert_close_rel(to_np(dq), dq_ref, rel=3e-2, cos=0.999, what="dq", atol=floor)
    assert_close_rel(to_np(dk), dk_ref, rel=3e-2, cos=0.999, what="dk", atol=floor)
    assert_close_rel(to_np(dv), dv_ref, rel=3e-2, cos=0.999, what="dv", atol=floor)


@pytest.mark.parametrize("B,H,Hkv,T,Dh,window", [(2, 4, 2, 150, 64, 0), (1, 6, 1, 257, 128, 64),
                                                (1, 8, 2, 300, 128, 0)])
def test_attention_grouped_query_heads(B, H, Hkv, T, Dh, window):
    """Query head h reads key/value head h / (H/Hkv); dk, dv sum over each group's query heads."""
    rng = np.random.default_rng(B + H + Hkv + T + Dh)
    q, do = (randn(rng, B, H, T, Dh) for _ in range(2))
    k, v = (randn(rng, B, Hkv, T, Dh) for _ in range(2))
    o_ref, lse_ref = O.attention_batch_forward(q, k, v, window)
    dq_ref, dk_ref, dv_ref = O.attention_batch_backward(q, k, v, do, window)
    tq, tk, tv, tdo = (bf16_tensor(a) for a in (q, k, v, do))
    sq, skv = (H * T * Dh, T * Dh, Dh), (Hkv * T * Dh, T * Dh, Dh)
    to = torch.zeros(B, H, T, Dh, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
    st = _status()
    S.attention_fwd(tq, tk, tv, to, lse, window, sq, sq, B, H, T, Dh, status=st, H_kv=Hkv, strides_kv=skv)
    dq = torch.zeros_like(tq)
    dk, dv = torch.zeros_like(tk), torch.zeros_like(tv)
    delta = S.attention_bwd_scratch(B, H, T)
    S.attention_bwd(tq, tk, tv, to, tdo, lse, delta, dq, dk, dv, window, sq, sq, B, H, T, Dh, status=st,
                    H_kv=Hkv, strides_kv=skv)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    floor = 2.0 ** -9 * math.sqrt(Dh)
    assert_close_rel(to_np(to), o_ref, rel=2e-2, cos=0.9999, what="o")
    np.testing.assert_allclose(to_np(lse), lse_ref, atol=2e-3)
    assert_close_rel(to_np(dq), dq_ref, rel=3e-2, cos=0.999, what="dq", atol=floor)
    assert_close_rel(to_np(dk), dk_ref, rel=3e-2, cos=0.999, what="dk", atol=floor)
    assert_close_rel(to_np(dv), dv_ref, rel=3e-2, cos=0.999, what="dv", atol=floor)


def test_attention_token_major_strides():
    """q/k/v read from a [B·T, 3·H·Dh] buffer and o written to [B·T, H·Dh], as the step does."""
    B, H, T, Dh, window = 2, 2, 96, 64, 40
    rng = np.random.default_rng(5)
    d = H * Dh
    qkv = randn(rng, B * T, 3 * d)
    tqkv = bf16_tensor(qkv)
    to = torch.zeros(B * T, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
    sq = (T * 3 * d, Dh, 3 * d)
    so = (T * d, Dh, d)
    S.attention_fwd(tqkv, tqkv[:, d:], tqkv[:, 2 * d:], to, lse, window, sq, so, B, H, T, Dh)
    torch.cuda.synchronize()
    x = qkv.reshape(B, T, 3, H, Dh).transpose(2, 0, 3, 1, 4)  # [3, B, H, T, Dh]
    o_ref, _ = O.attention_batch_forward(x[0], x[1], x[2], window)
    got = to_np(to).reshape(B, T, H, Dh).transpose(0, 2, 1, 3)
    assert_close_rel(got, o_ref, rel=2e-2, what="o token-major")


# --------------------------------------------------------------------------------------------------
# embedding
# --------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("V,d,M", [(512, 128, 3000), (64, 64, 40000), (2048, 1536, 700)])
def test_embedding_fwd_bwd_deterministic(V, d, M):
    """Zipf ids (long runs of the hot ids, runs crossing 64-token pieces, several sort segments)."""
    rng = np.random.default_rng(3)
    from gpt_decoder_pretraining_b200.inputs import _zipf_ids
    tok = _zipf_ids(rng, M, V)
    wte = randn(rng, V, d)
    gx = rng.standard_normal((M, d)).astype(np.float32)
    ttok = torch.from_numpy(tok).cuda()
    x = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    S.embedding_fwd(ttok, bf16_tensor(wte), x)
    scratch = torch.empty(S.embedding_bwd_scratch_bytes(M, d, V), dtype=torch.uint8, device="cuda")
    dw1 = torch.full((V, d), 7.0, dtype=torch.float32, device="cuda")
    dw2 = torch.empty((V, d), dtype=torch.float32, device="cuda")
    tg = torch.from_numpy(gx).cuda()
    S.embedding_bwd(ttok, tg, dw1, scratch)
    S.embedding_bwd(ttok, tg, dw2, scratch)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(x), wte[tok])
    ref = np.zeros((V, d))
    np.add.at(ref, tok, gx.astype(np.float64))
    assert_close_rel(to_np(dw1), ref, rel=1e-6, cos=0.9999999, what="dwte")
    assert torch.equal(dw1, dw2)  # bitwise reproducible


def test_embedding_out_of_range_is_flagged_not_faulted():
    V, d = 64, 64
    tok = torch.tensor([0, 5, 64, -3, 63], dtype=torch.int32, device="cuda")
    wte = torch.randn(V, d, device="cuda").to(torch.bfloat16)
    x = torch.empty(5, d, dtype=torch.bfloat16, device="cuda")
    st = _status()
    S.embedding_fwd(tok, wte, x, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == -6
    assert torch.equal(x[2], wte[63]) and torch.equal(x[3], wte[0])


# --------------------------------------------------------------------------------------------------
# fused lm-head + cross-entropy
# --------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("M,d,V,ignore", [(128, 64, 2048, 0), (300, 128, 1000 // 64 * 64 + 64, 7),
                                           (256, 64, 512, 256)])
def test_lmhead_ce(M, d, V, ignore):
    rng = np.random.default_rng(M + d + V)
    xf = randn(rng, M, d)
    w = randn(rng, V, d, scale=0.5)
    y = rng.integers(0, V, M).astype(np.int32)
    y[:ignore] = -1
    z = xf @ w.T
    lse_ref = O.logsumexp_rows(z)
    valid = y >= 0
    n = int(valid.sum())
    loss_ref = float(np.sum((lse_ref - z[np.arange(M), np.maximum(y, 0)])[valid]) / n) if n else 0.0
    dz = O.softmax_rows(z)
    dz[np.arange(M), np.maximum(y, 0)] -= 1.0
    dz *= (valid / max(n, 1))[:, None]
    txf, tw = bf16_tensor(xf), bf16_tensor(w)
    ty = torch.from_numpy(y).cuda()
    loss = torch.zeros(1, device="cuda")
    lse = torch.zeros(M, device="cuda")
    dx = torch.zeros(M, d, device="cuda")
    dW = torch.zeros(V, d, device="cuda")
    scratch = torch.empty(S.lmhead_ce_scratch_bytes(M, d, V), dtype=torch.uint8, device="cuda")
    S.lmhead_ce_fwd_bwd(txf, tw, ty, loss, lse, dx, dW, scratch)
    torch.cuda.synchronize()
    assert abs(loss.item() - loss_ref) < 2e-3
    np.testing.assert_allclose(to_np(lse), lse_ref, atol=2e-3)
    if n:
        assert_close_rel(to_np(dx), dz @ w, rel=2e-2, cos=0.9999, what="dx")
        assert_close_rel(to_np(dW), dz.T @ xf, rel=2e-2, cos=0.9999, what="dW")
    else:
        assert not torch.any(dx) and not torch.any(dW)
