"""Data-parallel gradient exchange for the training step: one process per GPU, each running the
step on its own rows (weak scaling), and the gradient average over ranks — the one exchange step of
the path.  The pages train with 8 GPUs under torchrun ("Introducing nanochat") and with a sharded
optimizer whose ranks exchange gradients ("alpha-nanochat-d24", The run).

The exchange runs per bucket (W_lm, then each layer from the last to the first, then wte — the
order in which the backward pass finishes them) on a side stream: each bucket's all-reduce waits
only for the event the step records when that bucket is final, so the collectives of the early
buckets overlap the backward pass of the remaining layers.  The training stream then waits for the
side stream before anything reads the gradients.

Every rank holds the same number of valid targets per step, so the mean of the per-rank mean-loss
gradients is the gradient of the mean loss over the global batch.  NCCL averages inside the
collective (ReduceOp.AVG); other backends (the CPU tests use gloo) sum and divide.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple


def grad_buckets(cfg) -> List[Tuple[int, int]]:
    """Element ranges of the gradient buckets in backward order, from the parameter packing of a
    GptConfig (the same ranges gpt_step_grad_bucket reports): W_lm, layer depth−1 … layer 0, wte."""
    offs, pos = [], 0
    for _, (a, b) in cfg.tensor_shapes():
        offs.append(pos)
        pos += a * b
    L = cfg.depth
    out = [(offs[-1], pos)]
    for l in reversed(range(L)):
        out.append((offs[1 + 4 * l], offs[1 + 4 * l + 4] if l + 1 < L else offs[-1]))
    out.append((0, cfg.vocab * cfg.d_model))
    return out


def _average(t, world: int):
    import torch.distributed as dist
    if dist.get_backend() == "nccl":
        dist.all_reduce(t, op=dist.ReduceOp.AVG)
    else:
        dist.all_reduce(t)
        t /= world


def average_in_buckets(grads, buckets: Sequence[Tuple[int, int]], world: int,
                       wait: Optional[Callable[[int], None]] = None):
    """grads[b0:b1] ← mean over ranks, bucket by bucket in the given order; `wait(i)` (if given) is
    called before bucket i's collective is issued.  Every rank issues the same collectives in the
    same order."""
    if world <= 1:
        return grads
    for i, (b0, b1) in enumerate(buckets):
        if wait is not None:
            wait(i)
        _average(grads[b0:b1], world)
    return grads


class OverlappedGradAverage:
    """Per-bucket all-reduce of a GptStep's gradients on a side stream, overlapped with the
    backward pass.  Call `launch(grads)` right after the step is enqueued; the current stream waits
    for the exchange before it returns, so later work on that stream sees averaged gradients."""

    def __init__(self, step, world: int):
        import torch
        self.step = step
        self.world = world
        self.buckets: List[Tuple[int, int]] = step.grad_buckets()
        self.side = torch.cuda.Stream(device=step.device) if world > 1 else None
        if world > 1:
            step.enable_grad_events(True)

    def launch(self, grads):
        if self.world <= 1:
            return grads
        import torch
        main = torch.cuda.current_stream(self.step.device)
        # no wait on the whole training stream here: each collective waits only for its bucket
        with torch.cuda.stream(self.side):
            average_in_buckets(grads, self.buckets, self.world,
                               wait=lambda i: self.step.wait_grad_bucket(i, self.side))
        main.wait_stream(self.side)
        return grads


# ------------------------------------------------------------------------------------------------
# sharded optimizer step: every rank updates its share of the parameters, then the shares are
# exchanged so that every rank again holds all of them
# ------------------------------------------------------------------------------------------------
def optimizer_shards(cfg, world: int):
    """Which rank updates what.  Layer l's four block matrices (Muon needs whole matrices) belong
    to rank l mod world; the embedding and lm-head rows (AdamW is elementwise) are cut into world
    contiguous row ranges.  Returns {rank: {"layers": [l…], "rows": (r0, r1)}} with rows of the
    [V, d] tables."""
    V = cfg.vocab
    out = {}
    for r in range(world):
        r0 = (V * r) // world
        r1 = (V * (r + 1)) // world
        out[r] = {"layers": [l for l in range(cfg.depth) if l % world == r], "rows": (r0, r1)}
    return out


def _layer_ranges(cfg):
    offs, pos = [], 0
    for _, (a, b) in cfg.tensor_shapes():
        offs.append(pos)
        pos += a * b
    L = cfg.depth
    return [(offs[1 + 4 * l], offs[1 + 4 * l + 4] if l + 1 < L else offs[-1]) for l in range(L)], offs, pos


class ShardedOptimizer:
    """Data-parallel optimizer step with the work split over the ranks (as the sharded Muon/AdamW
    of the pages' two-rank run does): on averaged gradients, rank r runs Muon on the layers it
    owns and AdamW on its rows of wte and W_lm, then every layer is broadcast from its owner and the
    table rows are gathered, so all ranks end with identical parameters.  The update functions are
    the caller's: `update_layers(layers, t)` (Muon on those layers' matrices) and
    `update_rows(r0, r1, t)` (AdamW on rows r0..r1 of both tables); they act on `params` in
    place.  Every rank issues the same collectives in the same order."""

    def __init__(self, cfg, world: int, rank: int):
        self.cfg, self.world, self.rank = cfg, world, rank
        self.shards = optimizer_shards(cfg, world)
        self.layers, self.offs, self.total = _layer_ranges(cfg)

    def step(self, params, t: int, update_layers, update_rows):
        mine = self.shards[self.rank]
        if mine["layers"]:
            update_layers(mine["layers"], t)
        update_rows(*mine["rows"], t)
        if self.world <= 1:
            return params
        import torch.distributed as dist
        for l, (b0, b1) in enumerate(self.layers):
            dist.broadcast(params[b0:b1], src=l % self.world)
        d = self.cfg.d_model
        for base in (self.offs[0], self.offs[-1]):  # wte, then W_lm
            for r in range(self.world):
                r0, r1 = self.shards[r]["rows"]
                dist.broadcast(params[base + r0 * d:base + r1 * d], src=r)
        return params


def device_update_fns(cfg, master, params, grads, state_m, state_v, hp: dict, world: int,
                      scratch=None):
    """The update functions of ShardedOptimizer on the GPU, through the library's optimizer entry
    points: Muon (gpt_muon_step) on the owned layers' q, k, v, o (one group), W_fc and W_proj —
    the owned layers are `world` layers apart, which is the group stride — and AdamW
    (gpt_adamw_step) on row ranges of wte and W_lm with learning rates × 1/√(d/768).  Buffers are
    the full flat packing (master, grads, state fp32; params in the step's dtype)."""
    import numpy as np

    from . import step as S
    layers_rng, offs, total = _layer_ranges(cfg)
    d, F, V = cfg.d_model, cfg.d_mlp, cfg.vocab
    lstride = (layers_rng[1][0] - layers_rng[0][0]) if cfg.depth > 1 else 0
    qkv_rows = d + 2 * cfg.kv_heads * cfg.head_dim
    mu, lr = hp["muon_momentum"], hp["muon_lr"]
    ns = hp["ns_coeffs"]

    def sl(t, a, b):
        return None if t is None else t[a:b]

    def update_layers(layers, t):
        l0, n = layers[0], len(layers)
        gstride = world * lstride
        base = offs[1 + 4 * l0]
        end = total if l0 + (n - 1) * world + 1 >= cfg.depth else offs[1 + 4 * (l0 + (n - 1) * world + 1)]
        # q, k, v (row blocks of W_qkv: d rows, then kv rows twice) and W_o: the square d×d group
        # when q, k, v all have d rows; otherwise q and o share shape (d×d) and k, v another
        groups = []
        if qkv_rows == 3 * d:
            groups.append((0, 4, d, d))
        else:
            kvr = cfg.kv_heads * cfg.head_dim
            groups += [(0, 1, d, d), (d * d, 2, kvr, d), (qkv_rows * d, 1, d, d)]
        groups += [((qkv_rows + d) * d, 1, F, d), ((qkv_rows + d) * d + F * d, 1, d, F)]
        for rel, per, r, c in groups:
            a = base + rel
            S.muon_step(master[a:end], sl(params, a, end), grads[a:end], state_m[a:end], n, per, gstride, r, c,
                        lr, mu, bool(hp.get("muon_nesterov", 1)), hp["ns_steps"], ns, scratch=scratch)

    def update_rows(r0, r1, t):
        if r1 <= r0:
            return
        # the learning-rate scale in fp32, formed as gpt_optim_step forms it, so that both give
        # bitwise the same update
        scale = np.float32(1.0) / np.sqrt(np.float32(d) / np.float32(768.0))
        for base, lr_t in ((offs[0], hp["adam_lr_wte"]), (offs[-1], hp["adam_lr_lm"])):
            a, b = base + r0 * d, base + r1 * d
            lr32 = float(np.float32(lr_t) * scale)
            S.adamw_step(master[a:b], sl(params, a, b), grads[a:b], state_m[a:b], state_v[a:b], t,
                         lr32, hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"],
                         param_dtype=cfg.param_dtype)

    return update_layers, update_rows
