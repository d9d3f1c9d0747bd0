"""The C ABI on the host (no GPU): the library loads and exports every symbol the header
declares, the parameter packing agrees with the configs and the oracle, and argument errors come
back as status codes before anything touches a device."""
import ctypes
import os
import re

import numpy as np
import pytest

from gpt_decoder_pretraining_b200 import build as B
from gpt_decoder_pretraining_b200 import config as C
from gpt_decoder_pretraining_b200 import step as S
from oracle import gpt_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gptstep.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(S._LIB_PATH):
        B.build()
    return S.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gpt_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 20
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(S.EXPORTED)


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8):
        assert lib.gpt_strerror(code) and lib.gpt_strerror(code) != b"unknown status"
    assert lib.gpt_strerror(123) == b"unknown status"


@pytest.mark.parametrize("name", C.PRESETS)
def test_param_layout_matches_configs_and_oracle(lib, name):
    cfg = C.preset(name)
    offs, total = S.param_layout(cfg)
    assert total == cfg.n_params == O.n_params(O.oracle_config(cfg))
    pos, expect = 0, []
    for _, (a, b) in cfg.tensor_shapes():
        expect.append(pos)
        pos += a * b
    assert offs == expect
    assert all(o % 64 == 0 for o in offs)
    # the oracle unpacks the same flat buffer into the same tensors
    if name == "smoke":
        flat = np.arange(total, dtype=np.float64)
        P = O.unpack(O.oracle_config(cfg), flat)
        assert P["wte"][0, 0] == offs[0] and P["qkv0"][0, 0] == offs[1] and P["lm"][0, 0] == offs[-1]


def _create(lib, cfg):
    c, keep = S._cconfig(cfg)
    h = ctypes.c_void_p()
    return lib.gpt_step_create(ctypes.byref(c), ctypes.byref(h)), h, keep


def test_config_validation(lib):
    good = C.custom(2, 128, 64, 256, 32, 2)
    st, h, _ = _create(lib, good)
    assert st == 0
    lib.gpt_step_destroy(h)
    bad = [
        (C.custom(2, 96, 32, 256, 32, 2), -2),                 # d_model not a multiple of 64
        (C.custom(2, 128, 16, 256, 32, 2), -2),                # head_dim 16 unsupported
        (C.custom(2, 128, 64, 70000 // 64 * 64, 32, 2), -2),   # vocab above 65536
    ]
    for cfg, code in bad:
        assert _create(lib, cfg)[0] == code
    cfg = C.custom(2, 128, 64, 256, 32, 2)
    cfg.param_dtype = 7
    assert _create(lib, cfg)[0] == -1
    cfg = C.custom(2, 128, 64, 256, 32, 2)
    cfg.n_heads = 3  # n_heads·head_dim ≠ d_model
    assert _create(lib, cfg)[0] == -1


def test_workspace_sizes_grow_with_the_model(lib):
    sizes = []
    for name in C.PRESETS:
        st, h, _ = _create(lib, C.preset(name))
        assert st == 0
        n = ctypes.c_size_t()
        assert lib.gpt_step_workspace_bytes(h, ctypes.byref(n)) == 0
        sizes.append(n.value)
        lib.gpt_step_destroy(h)
    assert sizes[0] < sizes[1] < sizes[2] and sizes[3] > sizes[1]
    assert sizes[3] < 60e9  # d24 fits a 180 GB B200 with room to spare


def test_step_argument_errors_need_no_device(lib):
    st, h, _ = _create(lib, C.custom(1, 64, 32, 256, 16, 1))
    assert st == 0
    n = ctypes.c_size_t()
    lib.gpt_step_workspace_bytes(h, ctypes.byref(n))
    fake = 1 << 20  # never dereferenced: validation fails first
    call = lib.gpt_step_fwd_bwd
    assert call(h, None, fake, fake, fake, fake, fake, n.value, 0, None) == -1           # null params
    assert call(h, fake, fake, fake, fake, fake, fake, n.value, 2, None) == -1           # accumulate ∉ {0, 1}
    assert call(h, fake, fake, fake, fake, fake, fake, n.value - 1, 0, None) == -3       # too small
    assert call(h, fake + 8, fake, fake, fake, fake, fake, n.value, 0, None) == -2       # misaligned
    assert lib.gpt_step_status(None, fake, None) == -1
    lib.gpt_step_destroy(h)


def test_kernel_entry_points_reject_bad_arguments(lib):
    f = 1 << 20
    assert lib.gpt_gemm(0, 0, 0, 64, 64, f, 64, f, 64, f, 64, None, None, 0, None, None, None) == -1
    assert lib.gpt_gemm(5, 0, 64, 64, 64, f, 64, f, 64, f, 64, None, None, 0, None, None, None) == -1
    assert lib.gpt_gemm(0, 0, 64, 64, 64, f, 60, f, 64, f, 64, None, None, 0, None, None, None) == -1
    assert lib.gpt_gemm(0, 0, 64, 64, 64, f + 2, 64, f, 64, f, 64, None, None, 0, None, None, None) == -2
    # head_dim 48 is not supported; 3 query heads cannot share 2 key/value heads
    assert lib.gpt_attention_fwd(f, f, f, f, f, None, 1, 1, 1, 16, 48, 0, 48, 48, 48, 48, 48, 48, 48, 48, 48,
                                 None, None) == -2
    assert lib.gpt_attention_fwd(f, f, f, f, f, None, 1, 3, 2, 16, 64, 0, 64, 64, 64, 64, 64, 64, 64, 64, 64,
                                 None, None) == -1
    assert lib.gpt_rmsnorm_fwd(None, f, f, 4, 64, None) == -1
    assert lib.gpt_embedding_bwd(f, f, f, 16, 64, 70000, f, None) == -2
    # grouped weight gradients: 1..4 problems, fp32 epilogues only, each problem checked like gpt_gemm
    from gpt_decoder_pretraining_b200.step import GemmTnProblem
    probs = (GemmTnProblem * 5)(*[GemmTnProblem(64, 64, f, 64, f, 64, f, 64) for _ in range(5)])
    grp = lib.gpt_gemm_group_tn
    grp.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                    ctypes.c_void_p, ctypes.c_void_p]
    p0 = ctypes.addressof(probs)
    assert grp(0, p0, 64, 4, None, None, None) == -1      # no problem
    assert grp(5, p0, 64, 4, None, None, None) == -1      # more than four
    assert grp(2, p0, 64, 0, None, None, None) == -1      # bf16 epilogue
    assert grp(2, None, 64, 4, None, None, None) == -1
    probs[1] = GemmTnProblem(64, 64, f, 60, f, 64, f, 64)  # lda < M
    assert grp(2, p0, 64, 4, None, None, None) == -1
    probs[1] = GemmTnProblem(64, 64, f + 2, 64, f, 64, f, 64)  # misaligned A
    assert grp(2, p0, 64, 5, None, None, None) == -2


def test_multi_rank_timing_uses_the_slowest_rank():
    """bench.py with N>1 ranks: the job time is the max over ranks (gloo, 2 processes)."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, (ms, rate) in out:
        assert ms == [20.0, 7.0]  # max over ranks of [10+10r, 7-r]
        assert rate == pytest.approx(32768 * 2 / 0.020)


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    ms = bench.max_over_ranks([10.0 + 10.0 * rank, 7.0 - rank], world)
    rate = bench.whole_job_rate(32768, world, ms[0])
    dist.destroy_process_group()
    q.put((rank, (ms, rate)))


def test_data_parallel_average_equals_the_full_batch_step(bucketed=False):
    """Two gloo ranks each take the oracle step on one row; bench.average_gradients over the ranks
    gives the oracle gradient of the two-row batch (equal valid counts per rank)."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 30500 + (os.getpid() % 1000) + (500 if bucketed else 0)
    procs = [ctx.Process(target=_dp_rank_main, args=(r, 2, port, q, bucketed)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    from oracle import gpt_oracle as O
    from gpt_decoder_pretraining_b200.config import custom
    from gpt_decoder_pretraining_b200.inputs import make_params, make_tokens
    cfg = custom(2, 32, 16, 64, 12, 2, param_dtype=1)
    params = make_params(cfg.n_params, keep_fp32=True, std=0.3).astype(np.float64)
    tok, tgt = make_tokens(2, 12, 64, seed=1)
    full = O.step(cfg, params, tok, tgt)
    for r in range(2):
        np.testing.assert_allclose(out[r], full["grads"], rtol=0, atol=1e-12)


def _dp_rank_main(rank, world, port, q, bucketed=False):
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    import bench
    from oracle import gpt_oracle as O
    from gpt_decoder_pretraining_b200.config import custom
    from gpt_decoder_pretraining_b200.inputs import make_params, make_tokens
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    cfg1 = custom(2, 32, 16, 64, 12, 1, param_dtype=1)
    params = make_params(cfg1.n_params, keep_fp32=True, std=0.3).astype(np.float64)
    tok, tgt = make_tokens(2, 12, 64, seed=1)
    g = torch.from_numpy(O.step(cfg1, params, tok[rank:rank + 1], tgt[rank:rank + 1])["grads"])
    if bucketed:
        from gpt_decoder_pretraining_b200 import dp
        buckets = dp.grad_buckets(cfg1)
        order = []
        dp.average_in_buckets(g, buckets, world, wait=order.append)
        assert order == list(range(len(buckets)))
    else:
        bench.average_gradients(g, world)
    dist.destroy_process_group()
    q.put((rank, g.numpy()))


def _host_buckets(cfg):
    """Gradient buckets as the library defines them (host-only calls, no device)."""
    lib = S.lib()
    st, h, _keep = _create(lib, cfg)
    assert st == 0
    n = lib.gpt_step_grad_buckets(h)
    out = []
    for i in range(n):
        b, e = ctypes.c_size_t(), ctypes.c_size_t()
        assert lib.gpt_step_grad_bucket(h, i, ctypes.byref(b), ctypes.byref(e)) == 0
        out.append((b.value, e.value))
    lib.gpt_step_destroy(h)
    return out


@pytest.mark.parametrize("name", ["smoke", "d20"])
def test_gradient_buckets_tile_the_packing_in_backward_order(lib, name):
    from gpt_decoder_pretraining_b200 import dp
    cfg = C.preset(name)
    b = _host_buckets(cfg)
    assert b == dp.grad_buckets(cfg)
    offs, total = S.param_layout(cfg)
    assert len(b) == cfg.depth + 2
    assert b[0] == (offs[-1], total)                       # W_lm first
    assert b[-1] == (0, cfg.vocab * cfg.d_model)           # wte last
    for i in range(1, cfg.depth + 1):                      # layers from the last to the first
        l = cfg.depth - i
        assert b[i] == (offs[1 + 4 * l], offs[1 + 4 * l + 4] if l + 1 < cfg.depth else offs[-1])
    assert sum(e - s for s, e in b) == total and len({s for s, _ in b}) == len(b)


def test_bucketed_data_parallel_average_equals_the_full_batch_step():
    """The per-bucket exchange (the order and ranges the library reports) gives the same average."""
    test_data_parallel_average_equals_the_full_batch_step(bucketed=True)


def test_attention_backward_scratch_size(lib):
    """Per padded row 8 bytes (LSE·log2 e and delta in fp32), then dS for one chunk of batches:
    2·T bytes per padded row of the chunk, the chunk being as many batches as fit 8 GiB of dS (all
    of them at the training shapes; 8 of 32 at H 8 × T 8192; none at T 32768, where one batch's
    dS alone is 16 GiB and the dQ kernel recomputes the scores instead)."""
    f = lib.gpt_attention_bwd_scratch_bytes
    f.restype = ctypes.c_size_t
    cap = 8 << 30
    for B, H, T, nb in [(1, 1, 1, 1), (2, 3, 200, 2), (16, 12, 2048, 16), (4, 8, 130, 4),
                        (32, 8, 8192, 8), (9, 8, 8192, 8), (1, 8, 32768, 0), (3, 1, 65536, 1), (3, 2, 65536, 0)]:
        tpad = (T + 63) // 64 * 64
        rows = B * H * tpad
        assert nb * H * T * tpad * 2 <= cap < (nb + 1) * H * T * tpad * 2 or nb == B
        assert f(B, H, T) == rows * 8 + nb * H * T * tpad * 2, (B, H, T)
    assert f(0, 1, 1) == 0 and f(1, 1, 0) == 0


def test_noalloc_attention_backward_row_limit_needs_no_device(lib):
    """The allocation-free backward keeps 8 bytes per padded row in a static array of 2^21 floats
    (1,048,576 rows).  One 64-row pad beyond the largest accepted shape (B·H·⌈T/64⌉·64 =
    1,048,576) is refused with GPT_ERR_UNSUPPORTED_SHAPE before any CUDA call, so no device is
    needed here (the pointers are never dereferenced).  The accepted side runs in
    tests/test_zz_no_alloc.py."""
    f = 1 << 20
    call = lib.gpt_attention_bwd_noalloc
    assert (1 << 21) * 4 // 8 == 1048576 and 16384 * 64 == 1048576
    args = lambda B, H, T, Dh: (f, f, f, f, f, f, f, f, f, B, H, T, Dh, 0,  # noqa: E731
                                H * T * Dh, T * Dh, Dh, H * T * Dh, T * Dh, Dh, None, None)
    assert call(*args(16385, 1, 64, 64)) == -2          # 1,048,640 padded rows
    assert call(*args(1, 16385, 33, 128)) == -2         # T = 33 pads to 64 rows per (b, h)
    assert call(*args(1, 16, 65537 * 2, 64)) == -2
    assert call(*args(0, 1, 64, 64)) == -1


def test_sharded_optimizer_equals_the_whole_step():
    """Two gloo ranks split the optimizer step (layers by rank, table rows in halves) and exchange
    the results: both end with the parameters of the oracle's unsharded optimizer step."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 31500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_shard_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    from oracle import optim_oracle as Q
    cfg, params, grads, hp = _shard_case()
    state = {}
    ref = Q.optimizer_step(cfg, params, grads, state, 1, hp)
    ref = Q.optimizer_step(cfg, ref, grads * 0.5, state, 2, hp)
    for r in range(2):
        np.testing.assert_array_equal(out[r], ref)


def _shard_case():
    from gpt_decoder_pretraining_b200.config import custom
    cfg = custom(3, 64, 16, 96, 8, 1, param_dtype=1)
    rng = np.random.default_rng(4)
    params = rng.standard_normal(cfg.n_params) * 0.02
    grads = rng.standard_normal(cfg.n_params) * 0.1
    hp = {"muon_lr": 0.02, "muon_momentum": 0.95, "ns_steps": 5, "ns_coeffs": (3.4445, -4.7750, 2.0315),
          "adam_lr_wte": 0.2, "adam_lr_lm": 0.004, "beta1": 0.8, "beta2": 0.95, "eps": 1e-10,
          "weight_decay": 0.01}
    return cfg, params, grads, hp


def _shard_rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    from gpt_decoder_pretraining_b200 import dp
    from oracle import optim_oracle as Q
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    cfg, params, grads, hp = _shard_case()
    p = torch.from_numpy(params.copy())
    state = {}
    muon = Q.muon_matrices(cfg)
    adam = Q.adamw_tensors(cfg)
    d = cfg.d_model
    opt = dp.ShardedOptimizer(cfg, world, rank)

    def run(g, t):
        def update_layers(layers, t):
            for l in layers:
                for name, (off, r, c) in muon.items():
                    if not name.startswith(f"h{l}."):
                        continue
                    w = p.numpy()[off:off + r * c].reshape(r, c)
                    buf = state.setdefault(name, np.zeros((r, c)))
                    w2, state[name] = Q.muon_update(w, g[off:off + r * c].reshape(r, c), buf, hp["muon_lr"],
                                                    hp["muon_momentum"], True, hp["ns_steps"], hp["ns_coeffs"])
                    p.numpy()[off:off + r * c] = w2.ravel()

        def update_rows(r0, r1, t):
            scale = 1.0 / np.sqrt(d / 768.0)
            for name, (off, V, _) in adam.items():
                lr = (hp["adam_lr_wte"] if name == "wte" else hp["adam_lr_lm"]) * scale
                a, b = off + r0 * d, off + r1 * d
                m = state.setdefault(name + ".m", np.zeros(V * d))
                v = state.setdefault(name + ".v", np.zeros(V * d))
                w2, m2, v2 = Q.adamw_update(p.numpy()[a:b], g[a:b], m[r0 * d:r1 * d], v[r0 * d:r1 * d], t, lr,
                                            hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"])
                p.numpy()[a:b] = w2
                m[r0 * d:r1 * d], v[r0 * d:r1 * d] = m2, v2

        opt.step(p, t, update_layers, update_rows)

    run(grads, 1)
    run(grads * 0.5, 2)
    dist.destroy_process_group()
    q.put((rank, p.numpy().copy()))


def test_a_failed_rank_ends_the_others_exchange_with_an_error():
    """Rank 1 raises before its gradient exchange and exits; rank 0's bucketed average must end with
    an error (connection closed or the short process-group timeout), not wait for good."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 31700 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_failing_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert out[1] == "raised"
    assert out[0].startswith("error:"), out[0]


def _failing_rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    from gpt_decoder_pretraining_b200 import dp
    from gpt_decoder_pretraining_b200.config import custom
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    cfg = custom(2, 32, 16, 64, 12, 1, param_dtype=1)
    g = torch.ones(cfg.n_params, dtype=torch.float32)
    if rank == 1:
        try:
            raise RuntimeError("rank 1 fails before its exchange")
        except RuntimeError:
            q.put((rank, "raised"))
            q.close()
            q.join_thread()
            os._exit(0)  # leaves without destroying the process group, as a crashed rank would
    try:
        dp.average_in_buckets(g, dp.grad_buckets(cfg), world)
        q.put((rank, "completed"))
    except Exception as e:  # noqa: BLE001 - any error ends the wait, which is what is checked
        q.put((rank, "error: " + type(e).__name__))
    q.close()
    q.join_thread()
    os._exit(0)


def test_last_cuda_error_names_the_error_behind_gpt_err_cuda(lib):
    """gpt_last_cuda_error: the CUDA error name and text of this thread's last GPT_ERR_CUDA."""
    f = lib.gpt_last_cuda_error
    f.restype = ctypes.c_char_p
    msg = f().decode()
    assert msg.startswith("cuda") and ": " in msg
