"""ctypes binding of libgptstep.so (argument marshalling only; every computation runs in the
library's CUDA kernels).

The names mirror the C entry points of include/gptstep.h.  Tensors are torch tensors on the
current CUDA device; the library receives their data pointers and the current CUDA stream.  If the
shared library is missing, loading fails loudly: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from .config import DTYPE_F32, GptConfig

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgptstep.so")
_lib = None

GPT_OK = 0
STATUS_NAMES = {0: "GPT_OK", -1: "GPT_ERR_INVALID_ARG", -2: "GPT_ERR_UNSUPPORTED_SHAPE",
                -3: "GPT_ERR_WORKSPACE_TOO_SMALL", -4: "GPT_ERR_CUDA", -5: "GPT_ERR_DEVICE_TIMEOUT",
                -6: "GPT_ERR_TOKEN_OUT_OF_RANGE", -7: "GPT_ERR_NO_DEVICE",
                -8: "GPT_ERR_NUMERIC_RANGE"}
GEMM_NT, GEMM_NN, GEMM_TN = 0, 1, 2
PROFILE_CLASSES = ("gemm", "attn_fwd", "attn_bwd", "rmsnorm", "rope_qknorm", "embedding", "ce_reduce")
EPI_BF16, EPI_RESID, EPI_RELU2, EPI_DRELU2, EPI_F32, EPI_F32_ADD = 0, 1, 2, 3, 4, 5

EXPORTED = [
    "gpt_param_layout", "gpt_step_create", "gpt_step_destroy", "gpt_step_workspace_bytes",
    "gpt_step_fwd_bwd", "gpt_step_status", "gpt_strerror", "gpt_last_cuda_error", "gpt_step_last_launch_count",
    "gpt_step_set_profiling", "gpt_step_profile", "gpt_step_grad_buckets", "gpt_step_grad_bucket",
    "gpt_step_enable_grad_events", "gpt_step_wait_grad_bucket",
    "gpt_gemm", "gpt_gemm_scratch_bytes", "gpt_qkv_proj_rope", "gpt_rmsnorm_fwd", "gpt_rmsnorm_bwd", "gpt_rope_qknorm_fwd", "gpt_rope_qknorm_bwd",
    "gpt_rope_table", "gpt_attention_fwd", "gpt_attention_bwd", "gpt_attention_bwd_noalloc",
    "gpt_embedding_fwd",
    "gpt_attention_bwd_scratch_bytes", "gpt_embedding_bwd_scratch_bytes", "gpt_embedding_bwd", "gpt_lmhead_ce_scratch_bytes",
    "gpt_lmhead_ce_fwd_bwd", "gpt_set_wait_limit", "gpt_debug_wait_probe", "gpt_debug_exp2_poly2",
    "gpt_gemm_batched", "gpt_gemm_group_tn", "gpt_adamw_step", "gpt_muon_scratch_bytes", "gpt_muon_step",
    "gpt_optim_scratch_bytes", "gpt_optim_step", "gpt_gemm_e4m3", "gpt_quantize_e4m3",
    "gpt_infer_create", "gpt_infer_destroy", "gpt_infer_workspace_bytes", "gpt_infer_kv_cache_bytes",
    "gpt_prefill", "gpt_decode", "gpt_infer_status",
]


class OptimHparams(ctypes.Structure):
    """gpt_optim_hparams: Muon and AdamW hyperparameters (every value is the caller's)."""
    _fields_ = [("muon_lr", ctypes.c_float), ("muon_momentum", ctypes.c_float),
                ("muon_nesterov", ctypes.c_int32), ("ns_steps", ctypes.c_int32),
                ("ns_a", ctypes.c_float), ("ns_b", ctypes.c_float), ("ns_c", ctypes.c_float),
                ("adam_lr_wte", ctypes.c_float), ("adam_lr_lm", ctypes.c_float),
                ("beta1", ctypes.c_float), ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
                ("weight_decay", ctypes.c_float)]


class GptError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = f"{what}: {STATUS_NAMES.get(status, status)}"
        if status == -4 and _lib is not None:  # GPT_ERR_CUDA: add the CUDA error behind it
            msg += f" ({_lib.gpt_last_cuda_error().decode()})"
        super().__init__(msg)


class _Config(ctypes.Structure):
    _fields_ = [("depth", ctypes.c_int32), ("d_model", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("d_mlp", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("seq_len", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("window", ctypes.POINTER(ctypes.c_int32)), ("param_dtype", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32)]


def lib():
    """Load libgptstep.so (built in-tree by gpt_decoder_pretraining_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: build it with "
                              "`python -m gpt_decoder_pretraining_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        ll = ctypes.c_longlong
        L.gpt_param_layout.argtypes = [ctypes.POINTER(_Config), ctypes.POINTER(sz), ctypes.POINTER(sz)]
        L.gpt_step_create.argtypes = [ctypes.POINTER(_Config), ctypes.POINTER(vp)]
        L.gpt_step_destroy.argtypes = [vp]
        L.gpt_step_destroy.restype = None
        L.gpt_step_workspace_bytes.argtypes = [vp, ctypes.POINTER(sz)]
        L.gpt_step_fwd_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, sz, i32, vp]
        L.gpt_step_status.argtypes = [vp, vp, vp]
        L.gpt_strerror.argtypes = [i32]
        L.gpt_strerror.restype = ctypes.c_char_p
        L.gpt_last_cuda_error.argtypes = []
        L.gpt_last_cuda_error.restype = ctypes.c_char_p
        L.gpt_step_last_launch_count.argtypes = [vp]
        L.gpt_step_last_launch_count.restype = ctypes.c_int64
        L.gpt_step_set_profiling.argtypes = [vp, i32]
        L.gpt_step_profile.argtypes = [vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64),
                                       ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double), i32]
        L.gpt_step_grad_buckets.argtypes = [vp]
        L.gpt_step_grad_bucket.argtypes = [vp, i32, ctypes.POINTER(sz), ctypes.POINTER(sz)]
        L.gpt_step_enable_grad_events.argtypes = [vp, i32]
        L.gpt_step_wait_grad_bucket.argtypes = [vp, i32, vp]
        L.gpt_gemm.argtypes = [i32, i32, i32, i32, i32, vp, i32, vp, i32, vp, i32, vp, vp, i32, vp, vp, vp]
        L.gpt_gemm_scratch_bytes.argtypes = []
        L.gpt_gemm_scratch_bytes.restype = sz
        L.gpt_qkv_proj_rope.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]
        L.gpt_rmsnorm_fwd.argtypes = [vp, vp, vp, i32, i32, vp]
        L.gpt_rmsnorm_bwd.argtypes = [vp, i32, vp, vp, vp, vp, i32, i32, i32, vp]
        L.gpt_rope_qknorm_fwd.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, vp]
        L.gpt_rope_qknorm_bwd.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp]
        L.gpt_rope_table.argtypes = [vp, i32, i32, vp]
        L.gpt_attention_fwd.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                        ll, ll, ll, ll, ll, ll, ll, ll, ll, vp, vp]
        L.gpt_attention_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                        ll, ll, ll, ll, ll, ll, ll, ll, ll, vp, vp]
        L.gpt_attention_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                                ll, ll, ll, ll, ll, ll, vp, vp]
        L.gpt_embedding_fwd.argtypes = [vp, vp, vp, i32, i32, i32, vp, vp]
        L.gpt_attention_bwd_scratch_bytes.argtypes = [i32, i32, i32]
        L.gpt_attention_bwd_scratch_bytes.restype = sz
        L.gpt_embedding_bwd_scratch_bytes.argtypes = [i32, i32, i32]
        L.gpt_embedding_bwd_scratch_bytes.restype = sz
        L.gpt_embedding_bwd.argtypes = [vp, vp, vp, i32, i32, i32, vp, vp]
        L.gpt_lmhead_ce_scratch_bytes.argtypes = [i32, i32, i32]
        L.gpt_lmhead_ce_scratch_bytes.restype = sz
        L.gpt_lmhead_ce_fwd_bwd.argtypes = [vp, vp, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp]
        f32 = ctypes.c_float
        L.gpt_gemm_batched.argtypes = [i32, i32, i32, i32, i32, i32, vp, i32, ll, vp, i32, ll, vp, i32, ll,
                                       vp, i32, ll, f32, f32, vp, vp]
        L.gpt_gemm_group_tn.argtypes = [i32, vp, i32, i32, vp, vp, vp]
        L.gpt_adamw_step.argtypes = [vp, vp, i32, vp, vp, vp, ll, i32, f32, f32, f32, f32, f32, vp]
        L.gpt_muon_scratch_bytes.argtypes = [i32, i32, i32]
        L.gpt_muon_scratch_bytes.restype = sz
        L.gpt_muon_step.argtypes = [vp, vp, i32, vp, vp, i32, i32, ll, i32, i32, f32, f32, i32, i32,
                                    f32, f32, f32, vp, sz, vp, vp]
        L.gpt_optim_scratch_bytes.argtypes = [ctypes.POINTER(_Config)]
        L.gpt_optim_scratch_bytes.restype = sz
        L.gpt_optim_step.argtypes = [ctypes.POINTER(_Config), vp, vp, vp, vp, vp, i32,
                                     ctypes.POINTER(OptimHparams), vp, sz, vp, vp]
        L.gpt_gemm_e4m3.argtypes = [i32, i32, i32, vp, i32, vp, i32, vp, i32, vp, vp, f32, vp, vp, vp]
        L.gpt_quantize_e4m3.argtypes = [vp, ll, vp, vp, vp, vp]
        L.gpt_infer_create.argtypes = [ctypes.POINTER(_Config), i32, i32, ctypes.POINTER(vp)]
        L.gpt_infer_destroy.argtypes = [vp]
        L.gpt_infer_destroy.restype = None
        L.gpt_infer_workspace_bytes.argtypes = [vp, ctypes.POINTER(sz)]
        L.gpt_infer_kv_cache_bytes.argtypes = [vp]
        L.gpt_infer_kv_cache_bytes.restype = sz
        L.gpt_prefill.argtypes = [vp, vp, vp, i32, i32, vp, vp, vp, sz, vp]
        L.gpt_decode.argtypes = [vp, vp, vp, i32, i32, vp, vp, vp, sz, vp]
        L.gpt_infer_status.argtypes = [vp, vp, vp]
        L.gpt_set_wait_limit.argtypes = [ll]
        L.gpt_debug_wait_probe.argtypes = [vp, vp]
        L.gpt_debug_exp2_poly2.argtypes = [vp, vp, i32, vp]
        _lib = L
    return _lib


def _check(status: int, what: str):
    if status != GPT_OK:
        raise GptError(status, what)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


def _cconfig(cfg: GptConfig):
    win = (ctypes.c_int32 * max(1, cfg.depth))(*cfg.windows)
    c = _Config(cfg.depth, cfg.d_model, cfg.n_heads, cfg.head_dim, cfg.d_mlp, cfg.vocab, cfg.seq_len,
                cfg.batch, ctypes.cast(win, ctypes.POINTER(ctypes.c_int32)), cfg.param_dtype,
                int(getattr(cfg, "n_kv_heads", 0) or 0))
    return c, win


def param_layout(cfg: GptConfig):
    """(offsets, total) of the flat parameter packing, as the library defines it."""
    c, _keep = _cconfig(cfg)
    n = 2 + 4 * cfg.depth
    offs = (ctypes.c_size_t * n)()
    total = ctypes.c_size_t(0)
    _check(lib().gpt_param_layout(ctypes.byref(c), offs, ctypes.byref(total)), "gpt_param_layout")
    return list(offs), int(total.value)


class StepGraph:
    """A captured training step (GptStep.capture): replay() enqueues it on the current stream and
    returns (loss, grads), the buffers the captured step writes."""

    def __init__(self, graph, outputs, launches: int):
        self._g = graph
        self.outputs = outputs
        self.launches = launches  # kernel launches recorded in the graph

    def replay(self):
        self._g.replay()
        return self.outputs


class GptStep:
    """One training step on the GPU: ``loss, grads = step(params, tokens, targets)``."""

    def __init__(self, cfg: GptConfig, device=None):
        import torch
        self.cfg = cfg
        c, self._win = _cconfig(cfg)
        h = ctypes.c_void_p()
        _check(lib().gpt_step_create(ctypes.byref(c), ctypes.byref(h)), "gpt_step_create")
        self._h = h
        nbytes = ctypes.c_size_t(0)
        _check(lib().gpt_step_workspace_bytes(h, ctypes.byref(nbytes)), "gpt_step_workspace_bytes")
        self.workspace_bytes = int(nbytes.value)
        self.device = torch.device(device or "cuda")
        self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=self.device)
        self.offsets, self.n_params = param_layout(cfg)
        self.loss = torch.zeros(1, dtype=torch.float32, device=self.device)
        self.grads = torch.empty(self.n_params, dtype=torch.float32, device=self.device)

    def __del__(self):
        try:
            if getattr(self, "_h", None) is not None and _lib is not None:
                _lib.gpt_step_destroy(self._h)
                self._h = None
        except Exception:
            pass

    def __call__(self, params, tokens, targets, grads=None, loss=None, accumulate=False):
        """Enqueue one step on the current stream; returns (loss tensor [1], grads tensor).
        With ``accumulate`` the step's gradients are added to ``grads`` instead of replacing them."""
        grads = self.grads if grads is None else grads
        loss = self.loss if loss is None else loss
        want = "torch.float32" if self.cfg.param_dtype == DTYPE_F32 else "torch.bfloat16"
        if str(params.dtype) != want or params.numel() != self.n_params:
            raise ValueError(f"params must be {want}[{self.n_params}]")
        if tokens.dtype != targets.dtype or str(tokens.dtype) != "torch.int32":
            raise ValueError("tokens/targets must be int32")
        st = lib().gpt_step_fwd_bwd(self._h, params.data_ptr(), tokens.data_ptr(), targets.data_ptr(),
                                    loss.data_ptr(), grads.data_ptr(), self.workspace.data_ptr(),
                                    self.workspace_bytes, 1 if accumulate else 0, _stream())
        _check(st, "gpt_step_fwd_bwd")
        return loss, grads

    def capture(self, params, tokens, targets, grads=None, loss=None, accumulate=False):
        """Record one step with these buffers into a CUDA graph (one launch of the whole step instead
        of ~500 kernel launches from the host).  Returns a StepGraph; its replay() enqueues the step
        again on the current stream, reading whatever the same buffers then hold.  A plain step runs
        first, so that first-call work (kernel attributes) happens outside the capture."""
        import torch
        self(params, tokens, targets, grads, loss, accumulate)
        torch.cuda.synchronize(self.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            out = self(params, tokens, targets, grads, loss, accumulate)
        return StepGraph(g, out, self.last_launch_count())

    def grad_buckets(self):
        """[(begin, end)] element ranges of the gradient buckets, in the order the backward pass
        finishes them (W_lm, the layers from the last to the first, wte)."""
        out = []
        for i in range(int(lib().gpt_step_grad_buckets(self._h))):
            b, e = ctypes.c_size_t(), ctypes.c_size_t()
            _check(lib().gpt_step_grad_bucket(self._h, i, ctypes.byref(b), ctypes.byref(e)), "grad_bucket")
            out.append((int(b.value), int(e.value)))
        return out

    def enable_grad_events(self, on: bool = True):
        _check(lib().gpt_step_enable_grad_events(self._h, int(bool(on))), "enable_grad_events")

    def wait_grad_bucket(self, i: int, stream=None):
        """Make `stream` (default: the current stream) wait until bucket i of the last step is final."""
        import torch
        st = (stream or torch.cuda.current_stream()).cuda_stream
        _check(lib().gpt_step_wait_grad_bucket(self._h, i, st), "wait_grad_bucket")

    def status(self) -> int:
        return int(lib().gpt_step_status(self._h, self.workspace.data_ptr(), _stream()))

    def last_launch_count(self) -> int:
        return int(lib().gpt_step_last_launch_count(self._h))

    def set_profiling(self, on: bool):
        _check(lib().gpt_step_set_profiling(self._h, int(bool(on))), "gpt_step_set_profiling")

    def profile(self):
        """{class: (ms, calls, flops, bytes)} accumulated since the last read (see gpt_step_profile)."""
        n = len(PROFILE_CLASSES)
        ms = (ctypes.c_double * n)()
        calls = (ctypes.c_int64 * n)()
        fl = (ctypes.c_double * n)()
        by = (ctypes.c_double * n)()
        _check(lib().gpt_step_profile(self._h, ms, calls, fl, by, n), "gpt_step_profile")
        return {c: (ms[i], int(calls[i]), fl[i], by[i]) for i, c in enumerate(PROFILE_CLASSES)}


class GptInfer:
    """Forward-only inference with a KV cache: ``logits = infer.prefill(params, tokens)`` fills
    positions 0..T−1, ``logits = infer.decode(params, tokens, pos)`` one more position."""

    def __init__(self, cfg: GptConfig, max_batch: int, max_len: int, device=None):
        import torch
        self.cfg = cfg
        c, self._win = _cconfig(cfg)
        h = ctypes.c_void_p()
        _check(lib().gpt_infer_create(ctypes.byref(c), max_batch, max_len, ctypes.byref(h)), "gpt_infer_create")
        self._h = h
        nbytes = ctypes.c_size_t(0)
        _check(lib().gpt_infer_workspace_bytes(h, ctypes.byref(nbytes)), "gpt_infer_workspace_bytes")
        self.device = torch.device(device or "cuda")
        self.workspace = torch.empty(int(nbytes.value), dtype=torch.uint8, device=self.device)
        self.kv_cache = torch.zeros(int(lib().gpt_infer_kv_cache_bytes(h)) // 2, dtype=torch.bfloat16,
                                    device=self.device)
        self.logits = None

    def __del__(self):
        try:
            if getattr(self, "_h", None) is not None and _lib is not None:
                _lib.gpt_infer_destroy(self._h)
                self._h = None
        except Exception:
            pass

    def _out(self, batch):
        import torch
        if self.logits is None or self.logits.shape[0] != batch:
            self.logits = torch.empty(batch, self.cfg.vocab, dtype=torch.float32, device=self.device)
        return self.logits

    def prefill(self, params, tokens):
        B, T = tokens.shape
        out = self._out(B)
        _check(lib().gpt_prefill(self._h, params.data_ptr(), tokens.data_ptr(), B, T, out.data_ptr(),
                                 self.kv_cache.data_ptr(), self.workspace.data_ptr(), self.workspace.numel(),
                                 _stream()), "gpt_prefill")
        return out

    def decode(self, params, tokens, pos: int):
        B = tokens.numel()
        out = self._out(B)
        _check(lib().gpt_decode(self._h, params.data_ptr(), tokens.data_ptr(), B, pos, out.data_ptr(),
                                self.kv_cache.data_ptr(), self.workspace.data_ptr(), self.workspace.numel(),
                                _stream()), "gpt_decode")
        return out

    def status(self) -> int:
        return int(lib().gpt_infer_status(self._h, self.workspace.data_ptr(), _stream()))


# ------------------------------------------------------------------------------------------------
# kernel-level calls (tensors in, tensors out); used by the unit parity tests and the benchmark
# ------------------------------------------------------------------------------------------------
_gemm_scratch = {}


def gemm_scratch(device):
    """A device buffer for gpt_gemm's split-tile scratch, one per device, kept for reuse."""
    import torch
    dev = torch.device(device)
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    if key not in _gemm_scratch:
        _gemm_scratch[key] = torch.empty(int(lib().gpt_gemm_scratch_bytes()), dtype=torch.uint8, device=dev)
    return _gemm_scratch[key]


def gemm(op: int, epi: int, A, B, C, M: int, N: int, K: int, C2=None, aux=None, status=None,
         lda=None, ldb=None, ldc=None, scratch="auto"):
    """C (op) A·B as defined for gpt_gemm; row strides default to the tensors' last dimension.
    scratch: "auto" (a cached per-device buffer, so that a partly empty last wave may be split along
    K), None, or a tensor."""
    lda = lda or A.shape[-1]
    ldb = ldb or B.shape[-1]
    ldc = ldc or C.shape[-1]
    ldaux = aux.shape[-1] if aux is not None else 0
    if isinstance(scratch, str):
        scratch = gemm_scratch(C.device)
    _check(lib().gpt_gemm(op, epi, M, N, K, A.data_ptr(), lda, B.data_ptr(), ldb, C.data_ptr(), ldc,
                          _ptr(C2), _ptr(aux), ldaux, _ptr(scratch), _ptr(status), _stream()), "gpt_gemm")


class GemmTnProblem(ctypes.Structure):
    """gpt_gemm_tn_problem: C[M, N] (fp32) (+)= Aᵀ·B with A [K, M] and B [K, N] bf16."""
    _fields_ = [("M", ctypes.c_int), ("N", ctypes.c_int), ("A", ctypes.c_void_p), ("lda", ctypes.c_int),
                ("B", ctypes.c_void_p), ("ldb", ctypes.c_int), ("C", ctypes.c_void_p), ("ldc", ctypes.c_int)]


def gemm_group_tn(problems, K: int, epi: int, status=None, scratch="auto"):
    """gpt_gemm_group_tn over [(A, B, C), …]: C = Aᵀ·B (GPT_EPI_F32) or C += Aᵀ·B (GPT_EPI_F32_ADD),
    A [K, M], B [K, N] bf16 and C [M, N] fp32, row strides from the tensors' last dimension."""
    arr = (GemmTnProblem * max(1, len(problems)))()
    for i, (A, B, C) in enumerate(problems):
        arr[i] = GemmTnProblem(C.shape[0], C.shape[1], A.data_ptr(), A.shape[-1], B.data_ptr(), B.shape[-1],
                               C.data_ptr(), C.shape[-1])
    if isinstance(scratch, str):
        scratch = gemm_scratch(problems[0][2].device)
    _check(lib().gpt_gemm_group_tn(len(problems), ctypes.addressof(arr), K, epi, _ptr(scratch), _ptr(status),
                                   _stream()), "gpt_gemm_group_tn")


def qkv_proj_rope(r, w_qkv, heads, rho_q, rho_k, cs, B, T, H, Dh, status=None, H_kv=None):
    """gpt_qkv_proj_rope: QKV projection + RoPE + QK-norm, head-major q̃ [B][H][T][Dh] then k̃, v
    [B][H_kv][T][Dh]."""
    _check(lib().gpt_qkv_proj_rope(r.data_ptr(), w_qkv.data_ptr(), heads.data_ptr(), rho_q.data_ptr(),
                                   rho_k.data_ptr(), cs.data_ptr(), B, T, H, H_kv or H, Dh, _ptr(status),
                                   _stream()), "qkv_proj_rope")


def rmsnorm_fwd(x, y, rho):
    rows, d = x.shape
    _check(lib().gpt_rmsnorm_fwd(x.data_ptr(), y.data_ptr(), rho.data_ptr(), rows, d, _stream()), "rmsnorm_fwd")


def rmsnorm_bwd(dy, y, rho, gx, gx_bf16=None, accumulate=False):
    rows, d = y.shape
    dy_f32 = 1 if str(dy.dtype) == "torch.float32" else 0
    _check(lib().gpt_rmsnorm_bwd(dy.data_ptr(), dy_f32, y.data_ptr(), rho.data_ptr(), gx.data_ptr(),
                                 _ptr(gx_bf16), int(accumulate), rows, d, _stream()), "rmsnorm_bwd")


def rope_table(cs, T: int, Dh: int):
    _check(lib().gpt_rope_table(cs.data_ptr(), T, Dh, _stream()), "rope_table")


def rope_qknorm_fwd(qkv, rho_q, rho_k, cs, B, T, H, Dh):
    _check(lib().gpt_rope_qknorm_fwd(qkv.data_ptr(), rho_q.data_ptr(), rho_k.data_ptr(), cs.data_ptr(),
                                     B, T, H, Dh, _stream()), "rope_qknorm_fwd")


def rope_qknorm_bwd(dqkv, qkv, rho_q, rho_k, cs, B, T, H, Dh):
    _check(lib().gpt_rope_qknorm_bwd(dqkv.data_ptr(), qkv.data_ptr(), rho_q.data_ptr(), rho_k.data_ptr(),
                                     cs.data_ptr(), B, T, H, Dh, _stream()), "rope_qknorm_bwd")


def attention_fwd(q, k, v, o, lse, window: int, strides_qkv, strides_o, B, H, T, Dh, status=None,
                  kmax=None, qk_normalized=False, H_kv=None, strides_kv=None):
    """Causal/window attention forward.  Unless qk_normalized, a B·H_kv float scratch for the
    per-head key-norm bound is allocated here (or taken from `kmax`).  strides_qkv are q's (and, by
    default, k's and v's); H_kv / strides_kv describe grouped key/value heads."""
    import torch
    Hk = H_kv or H
    if not qk_normalized and kmax is None:
        kmax = torch.empty(B * Hk, dtype=torch.float32, device=q.device)
    _check(lib().gpt_attention_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                   _ptr(None if qk_normalized else kmax), B, H, Hk, T, Dh, window,
                                   *strides_qkv, *(strides_kv or strides_qkv), *strides_o, _ptr(status),
                                   _stream()), "attention_fwd")


def attention_bwd_scratch_bytes(B: int, H: int, T: int) -> int:
    return int(lib().gpt_attention_bwd_scratch_bytes(B, H, T))


def attention_bwd_scratch(B: int, H: int, T: int, device="cuda"):
    """A device buffer for gpt_attention_bwd's `delta` scratch."""
    import torch
    return torch.empty(attention_bwd_scratch_bytes(B, H, T) // 4, dtype=torch.float32, device=device)


def attention_bwd(q, k, v, o, do, lse, delta, dq, dk, dv, window: int, strides_qkv, strides_o, B, H, T,
                  Dh, status=None, H_kv=None, strides_kv=None):
    _check(lib().gpt_attention_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                   lse.data_ptr(), delta.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                   dv.data_ptr(), B, H, H_kv or H, T, Dh, window, *strides_qkv,
                                   *(strides_kv or strides_qkv), *strides_o, _ptr(status), _stream()),
           "attention_bwd")


def attention_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, window: int, strides_qkv, strides_o, B, H, T,
                          Dh, status=None):
    """gpt_attention_bwd_noalloc: the attention backward with its scratch held inside the library."""
    _check(lib().gpt_attention_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                           do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                           dv.data_ptr(), B, H, T, Dh, window, *strides_qkv, *strides_o,
                                           _ptr(status), _stream()), "attention_bwd_noalloc")


def embedding_fwd(tokens, wte, x, status=None):
    M = tokens.numel()
    V, d = wte.shape
    _check(lib().gpt_embedding_fwd(tokens.data_ptr(), wte.data_ptr(), x.data_ptr(), M, d, V, _ptr(status),
                                   _stream()), "embedding_fwd")


def embedding_bwd_scratch_bytes(M: int, d: int, V: int) -> int:
    return int(lib().gpt_embedding_bwd_scratch_bytes(M, d, V))


def embedding_bwd(tokens, gx, dwte, scratch):
    M = tokens.numel()
    V, d = dwte.shape
    _check(lib().gpt_embedding_bwd(tokens.data_ptr(), gx.data_ptr(), dwte.data_ptr(), M, d, V,
                                   scratch.data_ptr(), _stream()), "embedding_bwd")


def lmhead_ce_scratch_bytes(M: int, d: int, V: int) -> int:
    return int(lib().gpt_lmhead_ce_scratch_bytes(M, d, V))


def lmhead_ce_fwd_bwd(xf, wlm, targets, loss, lse, dx, dW, scratch, status=None):
    M, d = xf.shape
    V = wlm.shape[0]
    _check(lib().gpt_lmhead_ce_fwd_bwd(xf.data_ptr(), wlm.data_ptr(), targets.data_ptr(), M, d, V,
                                       loss.data_ptr(), lse.data_ptr(), dx.data_ptr(), dW.data_ptr(),
                                       scratch.data_ptr(), _ptr(status), _stream()), "lmhead_ce_fwd_bwd")


def gemm_batched(op: int, epi: int, batch: int, M: int, N: int, K: int, A, lda, a_bstride, B, ldb, b_bstride,
                 C, ldc, c_bstride, aux=None, ldaux=0, aux_bstride=0, alpha=1.0, beta=0.0, status=None):
    """gpt_gemm_batched (strides in elements)."""
    _check(lib().gpt_gemm_batched(op, epi, batch, M, N, K, A.data_ptr(), lda, a_bstride, B.data_ptr(), ldb,
                                  b_bstride, C.data_ptr(), ldc, c_bstride, _ptr(aux), ldaux, aux_bstride,
                                  float(alpha), float(beta), _ptr(status), _stream()), "gpt_gemm_batched")


def adamw_step(master, params, grads, m, v, t: int, lr, beta1, beta2, eps, weight_decay, param_dtype=None):
    """gpt_adamw_step over all elements of `master` (params may be None)."""
    pdt = param_dtype if param_dtype is not None else (
        DTYPE_F32 if params is None or str(params.dtype) == "torch.float32" else 0)
    _check(lib().gpt_adamw_step(master.data_ptr(), _ptr(params), pdt, grads.data_ptr(), m.data_ptr(),
                                v.data_ptr(), master.numel(), t, lr, beta1, beta2, eps, weight_decay,
                                _stream()), "gpt_adamw_step")


def muon_scratch_bytes(n: int, rows: int, cols: int) -> int:
    return int(lib().gpt_muon_scratch_bytes(n, rows, cols))


def muon_step(master, params, grads, buf, groups, per_group, group_stride, rows, cols, lr, momentum,
              nesterov=True, ns_steps=5, ns=(3.4445, -4.7750, 2.0315), scratch=None, status=None):
    """gpt_muon_step on a group of matrices laid out as in the flat parameter packing."""
    import torch
    pdt = DTYPE_F32 if params is None or str(params.dtype) == "torch.float32" else 0
    need = muon_scratch_bytes(groups * per_group, rows, cols)
    if scratch is None:
        scratch = torch.empty(need, dtype=torch.uint8, device=master.device)
    _check(lib().gpt_muon_step(master.data_ptr(), _ptr(params), pdt, grads.data_ptr(), buf.data_ptr(), groups,
                               per_group, group_stride, rows, cols, lr, momentum, int(bool(nesterov)),
                               ns_steps, ns[0], ns[1], ns[2], scratch.data_ptr(), scratch.numel(),
                               _ptr(status), _stream()), "gpt_muon_step")


def optim_scratch_bytes(cfg: GptConfig) -> int:
    c, _keep = _cconfig(cfg)
    return int(lib().gpt_optim_scratch_bytes(ctypes.byref(c)))


def optim_step(cfg: GptConfig, master, params, grads, state_m, state_v, t: int, hp: dict, scratch=None,
               status=None):
    """gpt_optim_step: Muon + AdamW over the whole flat packing (hp keys as gpt_optim_hparams)."""
    import torch
    c, _keep = _cconfig(cfg)
    h = OptimHparams(hp["muon_lr"], hp["muon_momentum"], int(hp.get("muon_nesterov", 1)), hp["ns_steps"],
                     hp["ns_coeffs"][0], hp["ns_coeffs"][1], hp["ns_coeffs"][2], hp["adam_lr_wte"],
                     hp["adam_lr_lm"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"])
    need = optim_scratch_bytes(cfg)
    if scratch is None:
        scratch = torch.empty(max(need, 256), dtype=torch.uint8, device=master.device)
    _check(lib().gpt_optim_step(ctypes.byref(c), master.data_ptr(), _ptr(params), grads.data_ptr(),
                                state_m.data_ptr(), state_v.data_ptr(), t, ctypes.byref(h),
                                scratch.data_ptr(), scratch.numel(), _ptr(status), _stream()), "gpt_optim_step")


def quantize_e4m3(x, q, dq, amax_scratch=None):
    """gpt_quantize_e4m3: x bf16 → q (uint8 codes), dq (device float [1]) with x ≈ q·dq."""
    import torch
    if amax_scratch is None:
        amax_scratch = torch.empty(1, dtype=torch.int32, device=x.device)
    _check(lib().gpt_quantize_e4m3(x.data_ptr(), x.numel(), q.data_ptr(), dq.data_ptr(),
                                   amax_scratch.data_ptr(), _stream()), "gpt_quantize_e4m3")


def gemm_e4m3(A, B, C, dq_a, dq_b, M: int, N: int, K: int, alpha=1.0, status=None, scratch="auto"):
    """gpt_gemm_e4m3: C (bf16) = alpha·dq_a·dq_b·A·Bᵀ on e4m3 codes A [M,K], B [N,K] (uint8)."""
    if isinstance(scratch, str):
        scratch = gemm_scratch(C.device)
    _check(lib().gpt_gemm_e4m3(M, N, K, A.data_ptr(), A.shape[-1], B.data_ptr(), B.shape[-1], C.data_ptr(),
                               C.shape[-1], dq_a.data_ptr(), dq_b.data_ptr(), float(alpha), _ptr(scratch),
                               _ptr(status), _stream()), "gpt_gemm_e4m3")


def set_wait_limit(cycles: int):
    """gpt_set_wait_limit: bound of every device-side wait on the current device (≤ 0: default)."""
    _check(lib().gpt_set_wait_limit(int(cycles)), "set_wait_limit")


def debug_wait_probe(status):
    """gpt_debug_wait_probe: a wait that nothing completes; *status receives the timeout code."""
    _check(lib().gpt_debug_wait_probe(status.data_ptr(), _stream()), "debug_wait_probe")


def debug_exp2_poly2(x, y):
    """gpt_debug_exp2_poly2: the attention forward's FMA-pipe 2^x on the fp32 array x."""
    _check(lib().gpt_debug_exp2_poly2(x.data_ptr(), y.data_ptr(), x.numel(), _stream()), "debug_exp2_poly2")


def flat_to_bf16_tensor(params_f32: np.ndarray, device="cuda"):
    """Upload bf16-exact float32 values as a torch bfloat16 tensor (exact)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(params_f32, dtype=np.float32)).to(device).to(torch.bfloat16)
