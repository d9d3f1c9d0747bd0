"""Parity of the optimizer step (Muon + AdamW) and of the batched GEMM it uses, against the oracle
(needs a B200).  Every call goes through the C ABI.

* gpt_gemm_batched with the AXPBY epilogue against the fp64 products, for the three operand
  layouts, ragged sizes and a batch stride larger than one matrix;
* gpt_adamw_step against the oracle's AdamW over two steps (fp32 arithmetic: moments and weights
  within 1e-6 of their scale; the bf16 parameter copy is exactly the rounded master weight);
* gpt_muon_step against the oracle's Muon over two steps on wide, tall and square groups laid out
  as in the parameter packing: the momentum buffer within fp32 rounding, and the update direction
  within the tolerance of Newton–Schulz run in bf16 with fp32 accumulation (the method's published
  precision) against the fp64 oracle;
* gpt_optim_step over the whole packing of the smallest configuration and of a one-layer model of
  d12's widths, against the oracle's optimizer_step (the pages' grouping and AdamW scale).
"""
import numpy as np
import pytest
import torch

from gpt_decoder_pretraining_b200.config import custom, preset
from gpt_decoder_pretraining_b200.inputs import make_params, round_to_bf16
from oracle import optim_oracle as Q
from tests.gpu_util import assert_close_rel, bf16_tensor, cosine, randn, to_np

pytestmark = pytest.mark.gpu

S = None
HP = {"muon_lr": 0.02, "muon_momentum": 0.95, "ns_steps": 5, "ns_coeffs": Q.NS_QUINTIC,
      "adam_lr_wte": 0.2, "adam_lr_lm": 0.004, "beta1": 0.8, "beta2": 0.95, "eps": 1e-10,
      "weight_decay": 0.01}
# Newton–Schulz in bf16 against fp64: the update direction of every matrix
MUON_REL, MUON_COS = 4e-2, 0.999


def setup_module(module):
    global S
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gpt_decoder_pretraining_b200 import step
    S = step
    S.lib()


@pytest.mark.parametrize("op", [0, 1, 2])
def test_gemm_batched_axpby(op):
    rng = np.random.default_rng(70 + op)
    nb, M, N, K = 5, 296, 200, 136  # ragged against the 256-row tiles; M·2 bytes a 16-byte multiple (TN)
    a_shape = (K, M) if op == 2 else (M, K)
    b_shape = (N, K) if op == 0 else (K, N)
    pad = 64  # matrices further apart than their size
    A = randn(rng, nb, *a_shape)
    B = randn(rng, nb, *b_shape)
    X = randn(rng, nb, M, N)
    alpha, beta = -1.25, 0.75
    tA = torch.zeros(nb * (A[0].size + pad), dtype=torch.bfloat16, device="cuda")
    tB = torch.zeros(nb * (B[0].size + pad), dtype=torch.bfloat16, device="cuda")
    tX = torch.zeros(nb * (X[0].size + pad), dtype=torch.bfloat16, device="cuda")
    for i in range(nb):
        tA[i * (A[0].size + pad):i * (A[0].size + pad) + A[0].size] = bf16_tensor(A[i]).flatten()
        tB[i * (B[0].size + pad):i * (B[0].size + pad) + B[0].size] = bf16_tensor(B[i]).flatten()
        tX[i * (X[0].size + pad):i * (X[0].size + pad) + X[0].size] = bf16_tensor(X[i]).flatten()
    C = torch.zeros(nb, M, N, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.gemm_batched(op, 6, nb, M, N, K, tA, a_shape[1], A[0].size + pad, tB, b_shape[1], B[0].size + pad,
                   C, N, M * N, aux=tX, ldaux=N, aux_bstride=X[0].size + pad, alpha=alpha, beta=beta, status=st)
    Cp = torch.zeros(nb, M, N, dtype=torch.float32, device="cuda")
    S.gemm_batched(op, S.EPI_F32, nb, M, N, K, tA, a_shape[1], A[0].size + pad, tB, b_shape[1],
                   B[0].size + pad, Cp, N, M * N, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for i in range(nb):
        prod = (A[i].T if op == 2 else A[i]) @ (B[i].T if op == 0 else B[i])
        assert_close_rel(to_np(Cp[i]), prod, rel=1e-5, cos=0.9999999, what=f"f32 batch {i}")
        assert_close_rel(to_np(C[i]), alpha * prod + beta * X[i], rel=8e-3, what=f"axpby batch {i}")


def test_adamw_matches_oracle():
    rng = np.random.default_rng(5)
    n = (1 << 20) + 3
    w0 = make_params(n, keep_fp32=True).astype(np.float64)
    m0, v0 = np.zeros(n), np.zeros(n)
    tw = torch.from_numpy(w0.astype(np.float32)).cuda()
    tp = torch.zeros(n, dtype=torch.bfloat16, device="cuda")
    tm, tv = torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    w, m, v = w0, m0, v0
    for t in (1, 2):
        g = rng.standard_normal(n).astype(np.float32)
        S.adamw_step(tw, tp, torch.from_numpy(g).cuda(), tm, tv, t, 0.01, 0.9, 0.99, 1e-8, 0.1)
        w, m, v = Q.adamw_update(w, g.astype(np.float64), m, v, t, 0.01, 0.9, 0.99, 1e-8, 0.1)
    torch.cuda.synchronize()
    assert_close_rel(to_np(tm), m, rel=1e-6, cos=0.9999999, what="m")
    assert_close_rel(to_np(tv), v, rel=1e-6, cos=0.9999999, what="v")
    assert_close_rel(to_np(tw) - w0, w - w0, rel=1e-4, cos=0.99999, what="weight update")
    assert np.array_equal(tp.float().cpu().numpy(), round_to_bf16(tw.cpu().numpy()))


@pytest.mark.parametrize("rows,cols,groups,per", [(256, 256, 2, 3), (512, 128, 3, 1), (128, 384, 2, 1),
                                                   (64, 64, 2, 4)])
def test_muon_group_matches_oracle(rows, cols, groups, per):
    rng = np.random.default_rng(rows + cols + groups)
    mat = rows * cols
    gstride = per * mat + 4096  # other tensors between the groups, as in the packing
    total = groups * gstride
    w0 = make_params(total, keep_fp32=True).astype(np.float64)
    tw = torch.from_numpy(w0.astype(np.float32)).cuda()
    tp = torch.zeros(total, dtype=torch.bfloat16, device="cuda")
    tb = torch.zeros(total, device="cuda")
    ref_w = {i: w0[(i // per) * gstride + (i % per) * mat:][:mat].reshape(rows, cols) for i in range(groups * per)}
    ref_b = {i: np.zeros((rows, cols)) for i in ref_w}
    deltas = {}
    for step in range(2):
        g = (rng.standard_normal(total) * 0.1).astype(np.float32)
        before = to_np(tw)
        S.muon_step(tw, tp, torch.from_numpy(g).cuda(), tb, groups, per, gstride, rows, cols, 0.02, 0.95)
        torch.cuda.synchronize()
        after = to_np(tw)
        for i in ref_w:
            o = (i // per) * gstride + (i % per) * mat
            gi = g[o:o + mat].astype(np.float64).reshape(rows, cols)
            nw, ref_b[i] = Q.muon_update(ref_w[i], gi, ref_b[i], 0.02, 0.95, True, 5, Q.NS_QUINTIC)
            deltas[(step, i)] = (after[o:o + mat].reshape(rows, cols) - before[o:o + mat].reshape(rows, cols),
                                 nw - ref_w[i])
            ref_w[i] = ref_w[i] + (after[o:o + mat].reshape(rows, cols) - before[o:o + mat].reshape(rows, cols))
    for (step, i), (got, ref) in deltas.items():
        assert_close_rel(got, ref, rel=MUON_REL, cos=MUON_COS, what=f"muon update step {step} matrix {i}")
    bufs = to_np(tb)
    for i in ref_w:
        o = (i // per) * gstride + (i % per) * mat
        assert_close_rel(bufs[o:o + mat].reshape(rows, cols), ref_b[i], rel=1e-6, cos=0.9999999, what="buf")
    # the regions between the groups are untouched
    gap = np.concatenate([np.arange(k * gstride + per * mat, (k + 1) * gstride) for k in range(groups)])
    assert np.array_equal(to_np(tw)[gap], w0.astype(np.float32).astype(np.float64)[gap])
    assert np.array_equal(tp.float().cpu().numpy()[np.setdiff1d(np.arange(total), gap)],
                          round_to_bf16(tw.cpu().numpy())[np.setdiff1d(np.arange(total), gap)])


@pytest.mark.parametrize("which", ["smoke", "d12_layer", "gqa"])
def test_optim_step_matches_oracle(which):
    if which == "smoke":
        cfg = preset("smoke")
    elif which == "d12_layer":
        cfg = custom(1, 768, 128, 32768, 2048, 16, name="d12_layer")
    else:  # grouped key/value heads: k and v are their own Muon matrices of kv_heads·Dh rows
        cfg = custom(2, 256, 64, 1024, 64, 2, name="gqa", n_kv_heads=2)
    n = cfg.n_params
    rng = np.random.default_rng(11)
    w0 = make_params(n, keep_fp32=True).astype(np.float64)
    tw = torch.from_numpy(w0.astype(np.float32)).cuda()
    tp = torch.zeros(n, dtype=torch.float32 if cfg.param_dtype == 1 else torch.bfloat16, device="cuda")
    tm, tv = torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    state, ref = {}, w0
    for t in (1, 2):
        g = (rng.standard_normal(n) * 0.05).astype(np.float32)
        before = to_np(tw)
        S.optim_step(cfg, tw, tp, torch.from_numpy(g).cuda(), tm, tv, t, HP)
        torch.cuda.synchronize()
        after = to_np(tw)
        new_ref = Q.optimizer_step(cfg, before, g.astype(np.float64), state, t, HP)
        # per tensor: the update against the oracle's update from the same starting weights
        off = 0
        for name, (a, b) in cfg.tensor_shapes():
            sl = slice(off, off + a * b)
            off += a * b
            if name.endswith("w_qkv"):
                kvr = cfg.kv_heads * cfg.head_dim
                r0 = sl.start
                for j, rows in enumerate((cfg.d_model, kvr, kvr)):
                    s2 = slice(r0, r0 + rows * b)
                    r0 += rows * b
                    assert_close_rel(after[s2] - before[s2], new_ref[s2] - before[s2], rel=MUON_REL,
                                     cos=MUON_COS, what=f"{name}[{j}] t={t}")
            elif name in ("wte", "w_lm"):
                assert_close_rel(after[sl] - before[sl], new_ref[sl] - before[sl], rel=1e-4, cos=0.99999,
                                 what=f"{name} t={t}")
            else:
                assert_close_rel(after[sl] - before[sl], new_ref[sl] - before[sl], rel=MUON_REL,
                                 cos=MUON_COS, what=f"{name} t={t}")
        # continue both from the GPU's weights so that the second step compares like with like
        ref = after
    # the parameter copy the training step reads
    if cfg.param_dtype == 1:
        assert torch.equal(tp, tw)
    else:
        assert np.array_equal(tp.float().cpu().numpy(), round_to_bf16(tw.cpu().numpy()))
    # AdamW moments of the embedding (exact fp32 recurrences)
    V, d = cfg.vocab, cfg.d_model
    assert_close_rel(to_np(tv)[:V * d], state["wte.v"], rel=1e-5, cos=0.99999, what="wte v")


@pytest.mark.parametrize("world", [1, 2, 3])
def test_sharded_update_functions_cover_the_whole_step(world):
    """The per-rank update functions of the sharded optimizer (Muon on layers l ≡ r mod world, AdamW
    on row ranges), applied for every rank in turn on one GPU, give the same result as
    gpt_optim_step over the whole model (no collective is needed: the shards are disjoint)."""
    from gpt_decoder_pretraining_b200 import dp
    cfg = custom(4, 256, 64, 1024, 64, 2, name="shard")
    n = cfg.n_params
    rng = np.random.default_rng(3)
    w0 = make_params(n, keep_fp32=True)
    g = torch.from_numpy((rng.standard_normal(n) * 0.05).astype(np.float32)).cuda()
    ref_w, w = torch.from_numpy(w0).cuda(), torch.from_numpy(w0).cuda()
    ref_p, p = (torch.zeros(n, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    ref_m, ref_v, m, v = (torch.zeros(n, device="cuda") for _ in range(4))
    for t in (1, 2):
        S.optim_step(cfg, ref_w, ref_p, g, ref_m, ref_v, t, HP)
        ul, ur = dp.device_update_fns(cfg, w, p, g, m, v, HP, world)
        for r, sh in dp.optimizer_shards(cfg, world).items():
            if sh["layers"]:
                ul(sh["layers"], t)
            ur(*sh["rows"], t)
    torch.cuda.synchronize()
    assert torch.equal(w, ref_w)
    assert torch.equal(p, ref_p)
    assert torch.equal(m, ref_m) and torch.equal(v, ref_v)
