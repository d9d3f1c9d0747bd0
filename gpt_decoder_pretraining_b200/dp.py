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
