"""Benchmark of one GPT training step (forward + backward to parameter gradients) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config d24] [--impl ours|reference]

Prints ONE JSON line (rank 0).  Metric: training tokens/s of the fwd+bwd step and its MFU
(FLOPs/token × tokens/s ÷ 2.25e15, the nominal dense-bf16 peak of one B200), FLOPs/token by the
nanochat convention 6·(N − V·d) + 12·H·Dh·Σ_l min(w_l, T).

* `value`: whole-job tokens/s with inputs already resident in HBM, timed by CUDA events on the
  step's stream over K steps bracketed by barrier + synchronize, max over ranks.  Activations
  (tens of GB) exceed the 126 MB L2, so no flush is needed between steps.
* `e2e`: the same metric through the public API (GptStep) with the step's tokens/targets copied
  from pinned host memory and the loss copied back every step, inside the timed region.
* `roofline`: the GEMM class (the dominant kernel family) — algorithmic FLOPs ÷ its CUDA-event
  time, from separate profiled steps that record an event around every launch on the step's
  stream (kept out of the timed region) — against the measured sustained bf16 peak.
* `roofline`: `achieved` counts the method's GEMM FLOPs, 6·(N − V·d) per token; the lm-head logit
  recompute of the backward pass is reported separately as executed work (`executed_tflops`).
* `cpu_baseline`: the CPU oracle timed on this host on one row of the workload's sequence length
  (median of 3 runs; rank 0, N = 1).
* `also`: the second configuration the MFU target names (d20 by default), measured in the same run
  on the same GPU (N = 1 only).
* `--impl reference`: the oracle as it stands, one row of 512 tokens per step (a bounded sample
  that keeps K + W steps within minutes); its `config` states that sample.
* N > 1 (torchrun): data parallel with weak scaling — each rank runs the step on its own batch,
  then the fp32 gradients are averaged across ranks by one NCCL all-reduce per step (inside the
  timed region); the barrier and the max-reduction of the timings bracket the measurement.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from gpt_decoder_pretraining_b200.config import B200_DENSE_BF16_PEAK, preset  # noqa: E402
from gpt_decoder_pretraining_b200.inputs import make_params, make_tokens  # noqa: E402

METRIC = "training tokens/sec and MFU (% of B200 dense BF16) per fwd+bwd step, 1 GPU"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary, if any."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d.get(workload)
    except Exception:
        return None


def traffic_fields(workload: str):
    """roofline.traffic: DRAM bytes (read + write) per step of the GEMM family from the committed ncu
    launch list of this workload (null when there is none), with the algorithmic bytes beside it."""
    t = load_traffic(workload)
    if not t:
        return {"traffic": None}
    return {"traffic": t.get("dram_bytes_per_step"), "traffic_unit": "bytes per step",
            "traffic_algorithmic": t.get("algorithmic_bytes_per_step"), "traffic_source": t.get("source")}


# ------------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": ["no samples"]}
        # "under load": samples at or above half of the max power seen
        pmax = max(power) if power else 0
        loaded = [s for s, p in zip(sm, power) if p >= 0.5 * pmax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": pmax}


# ------------------------------------------------------------------------------------------------
# CPU oracle arm
# ------------------------------------------------------------------------------------------------
def cpu_sample_config(cfg, tokens: int):
    import dataclasses
    T = min(cfg.seq_len, tokens)
    wins = [w if (0 < w < T) else 0 for w in cfg.windows]
    return dataclasses.replace(cfg, batch=1, seq_len=T, windows=wins)


def time_oracle(cfg, sample_tokens: int, repeats: int = 1, warmup: int = 0, params=None):
    """Wall times of the oracle's fp32 fwd+bwd on one row of `sample_tokens` tokens."""
    from oracle import gpt_oracle as O
    scfg = cpu_sample_config(cfg, sample_tokens)
    p = params if params is not None else make_params(scfg.n_params, keep_fp32=(cfg.param_dtype == 1))
    t, y = make_tokens(1, scfg.seq_len, scfg.vocab, scfg.token_dist)
    times = []
    for i in range(warmup + repeats):
        t0 = time.perf_counter()
        O.step(scfg, p, t, y, dtype=np.float32)
        dt = time.perf_counter() - t0
        if i >= warmup:
            times.append(dt)
    return scfg, times


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def workload_config(cfg, world):
    """The `config` object both arms print: the workload, not the implementation."""
    return {"workload": f"{cfg.name} GPT fwd+bwd step", "model": cfg.name,
            "global_batch": cfg.batch * world, "seq_len": cfg.seq_len,
            "parallelism": f"dp{world}" if world > 1 else "none",
            "depth": cfg.depth, "d_model": cfg.d_model, "vocab": cfg.vocab,
            "windows": "SSSL w=1024" if any(cfg.windows) else "full causal",
            "l2": "inputs larger than L2 (activations ~tens of GB), no flush"}


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cores = cpu_cores()
    scfg, times = time_oracle(cfg, args.ref_sample_tokens, repeats=args.steps, warmup=args.warmup)
    per_step = statistics.median(times)
    value = scfg.seq_len / per_step
    mfu = cfg.flops_per_token() * value / B200_DENSE_BF16_PEAK
    sample = (f"one row of {scfg.seq_len} tokens of the {cfg.name} model (B=1), fp32 NumPy oracle "
              f"fwd+bwd, median of {args.steps} after {args.warmup} warm-up")
    # the model of the workload, timed on what one step of this arm processes: one row
    config = workload_config(scfg, 1)
    config.update(workload=f"{cfg.name} GPT fwd+bwd step", model=cfg.name,
                  timed_sample=f"B 1 x T {scfg.seq_len} per step (a bounded CPU sample of the "
                               f"B {cfg.batch * max(1, args.gpus)} x T {cfg.seq_len} workload)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic", "mfu": mfu,
        "config": config,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------------
# multi-rank bookkeeping and the data-parallel exchange
# ------------------------------------------------------------------------------------------------
def max_over_ranks(values, world, device="cpu"):
    """Element-wise maximum of per-rank timings (the slowest rank sets the job's time)."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def average_gradients(grads, world):
    """Data-parallel exchange: grads ← mean over ranks.  Every rank holds the same number of valid
    targets, so this is the gradient of the mean loss over the global batch.  NCCL averages in the
    collective itself; other backends (the CPU tests) sum and divide."""
    if world <= 1:
        return grads
    import torch.distributed as dist
    if dist.get_backend() == "nccl":
        dist.all_reduce(grads, op=dist.ReduceOp.AVG)
    else:
        dist.all_reduce(grads)
        grads /= world
    return grads


def whole_job_rate(units_per_rank_step, world, ms_per_step):
    """Units all ranks processed per second: every rank does units_per_rank_step per step."""
    return units_per_rank_step * world / (ms_per_step / 1e3)


# ------------------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------------------
def gemm_method_flops(cfg):
    """FLOPs of the step's dense contractions as the method defines them: 6·(N − V·d) per token
    (forward, data gradient and weight gradient of every projection, MLP and lm-head matrix).
    The lm-head logit recompute of the backward pass is executed work on top of this."""
    return 6.0 * (cfg.n_params - cfg.vocab * cfg.d_model) * cfg.tokens


def measure_step(args, cfg, dev, world, rank, barrier, exchange, with_e2e=True):
    """Warm up, time `args.steps` steps on device-resident inputs (CUDA events on the step's stream,
    barrier + synchronize on both sides), then per-kernel-class profile steps and, optionally, the
    same steps end to end through the public API with host buffers.  Returns a dict."""
    import torch
    from gpt_decoder_pretraining_b200.step import GptStep

    step = GptStep(cfg, device=dev)
    params_np = make_params(cfg.n_params, keep_fp32=(cfg.param_dtype == 1))
    params = torch.from_numpy(params_np).to(dev)
    if cfg.param_dtype == 0:
        params = params.to(torch.bfloat16)
    tok_np, tgt_np = make_tokens(cfg.batch, cfg.seq_len, cfg.vocab, cfg.token_dist, seed=1 + rank)
    tokens = torch.from_numpy(tok_np).to(dev)
    targets = torch.from_numpy(tgt_np).to(dev)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        _, grads = step(params, tokens, targets)
        exchange(grads)
    torch.cuda.synchronize(dev)
    st = step.status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up ({cfg.name})")
    loss0 = float(step.loss.item())

    # the step as one CUDA graph (its launches recorded once), unless disabled or not capturable
    graph = None
    if not getattr(args, "no_graph", False) and world == 1:
        try:
            graph = step.capture(params, tokens, targets)
            torch.cuda.synchronize(dev)
        except Exception as e:  # noqa: BLE001 - the eager launches below are the same kernels
            print(f"step graph not captured ({type(e).__name__}: {e}); timing eager launches",
                  file=sys.stderr)
            graph = None

    def run_step():
        if graph is not None:
            return graph.replay(), graph.launches
        out = step(params, tokens, targets)
        return out, step.last_launch_count()

    # ---------------- timed region (device-resident inputs) ----------------
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    clocks = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    launches = 0
    e0.record(stream)
    for _ in range(args.steps):
        (_, grads), n_launch = run_step()
        exchange(grads)
        launches += n_launch
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = e0.elapsed_time(e1) / args.steps
    clk = clocks.stop()

    # ---------------- per-kernel breakdown: separate steps with an event around every launch ----------------
    prof_steps = max(1, min(args.steps, 3))
    step.set_profiling(True)
    for _ in range(prof_steps):
        step(params, tokens, targets)
    torch.cuda.synchronize(dev)
    step.set_profiling(False)
    prof = step.profile()

    ms_e2e = None
    if with_e2e:
        # ---------------- end to end through the public API, host buffers ----------------
        tok_h = torch.from_numpy(tok_np).pin_memory()
        tgt_h = torch.from_numpy(tgt_np).pin_memory()
        loss_h = torch.zeros(1, dtype=torch.float32).pin_memory()
        # the graph reads tokens/targets from the buffers it was captured with: copy into those
        tok_d, tgt_d = (tokens, targets) if graph is not None else (torch.empty_like(tokens),
                                                                     torch.empty_like(targets))
        barrier()
        torch.cuda.synchronize(dev)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            tok_d.copy_(tok_h, non_blocking=True)
            tgt_d.copy_(tgt_h, non_blocking=True)
            if graph is not None:
                loss, grads = graph.replay()
            else:
                loss, grads = step(params, tok_d, tgt_d)
            exchange(grads)
            loss_h.copy_(loss, non_blocking=True)
        f1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        ms_e2e = f0.elapsed_time(f1) / args.steps
    ms, ms_e2e_m = max_over_ranks([ms, ms_e2e if ms_e2e is not None else 0.0], world, dev)
    kernels = {}
    for name, (kms, calls, fl, by) in prof.items():
        if calls == 0:
            continue
        ent = {"ms_per_step": kms / prof_steps, "calls_per_step": calls // prof_steps,
               "share": kms / (ms * prof_steps)}
        if fl:
            ent["tflops"] = fl / (kms / 1e3) / 1e12
        if by:
            ent["gbs"] = by / (kms / 1e3) / 1e9
        kernels[name] = ent
    out = {"ms": ms, "ms_e2e": ms_e2e_m if ms_e2e is not None else None, "clocks": clk,
           "launches": launches, "loss0": loss0, "prof": prof, "prof_steps": prof_steps,
           "step_launch": "one CUDA graph per step" if graph is not None else "kernel launches from the host",
           "kernels": kernels, "params_np": params_np,
           "h2d": int(tok_np.nbytes + tgt_np.nbytes)}
    del graph, step, params, tokens, targets, grads
    torch.cuda.empty_cache()
    return out


def muon_ns_flops(cfg, steps=5):
    """Newton–Schulz FLOPs of one Muon step over the model: per matrix (r ≤ c after transposing)
    and iteration X·Xᵀ (2r²c), A·A (2r³) and B·X (2r²c)."""
    def one(rows, cols):
        r, c = min(rows, cols), max(rows, cols)
        return steps * (4.0 * r * r * c + 2.0 * r ** 3)
    d, F = cfg.d_model, cfg.d_mlp
    return cfg.depth * (4 * one(d, d) + one(F, d) + one(d, F))


OPTIM_HP = {"muon_lr": 0.02, "muon_momentum": 0.95, "muon_nesterov": 1, "ns_steps": 5,
            "ns_coeffs": (3.4445, -4.7750, 2.0315), "adam_lr_wte": 0.2, "adam_lr_lm": 0.004,
            "beta1": 0.8, "beta2": 0.95, "eps": 1e-10, "weight_decay": 0.0}


def measure_optimizer(args, cfg, dev, params_np):
    """Time gpt_optim_step (Muon on the block matrices, AdamW on wte / W_lm) over the whole model,
    on fp32 master weights, fp32 gradients and optimizer state resident in HBM."""
    import torch
    from gpt_decoder_pretraining_b200 import step as S
    n = cfg.n_params
    master = torch.from_numpy(params_np.astype(np.float32)).to(dev)
    params = master.to(torch.bfloat16)
    g = torch.Generator(device=dev)
    g.manual_seed(3)
    grads = torch.randn(n, device=dev, generator=g) * 1e-3
    sm, sv = torch.zeros(n, device=dev), torch.zeros(n, device=dev)
    scratch = torch.empty(max(256, S.optim_scratch_bytes(cfg)), dtype=torch.uint8, device=dev)
    t = 1
    for _ in range(2):
        S.optim_step(cfg, master, params, grads, sm, sv, t, OPTIM_HP, scratch=scratch)
        t += 1
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    k = max(1, min(args.steps, 5))
    e0.record()
    for _ in range(k):
        S.optim_step(cfg, master, params, grads, sm, sv, t, OPTIM_HP, scratch=scratch)
        t += 1
    e1.record()
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / k
    adam_elems = 2 * cfg.vocab * cfg.d_model
    out = {"ms_per_step": ms, "steps": k,
           "what": "Muon (momentum, 5 Newton-Schulz steps in batched bf16 tcgen05 GEMMs, update) on every "
                   "block matrix + fused AdamW on wte and W_lm, fp32 master weights and state",
           "muon_ns_flops": muon_ns_flops(cfg), "adamw_bytes": 30.0 * adam_elems}
    del master, params, grads, sm, sv, scratch
    torch.cuda.empty_cache()
    return out


def run_ours(args, cfg):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def exchange(grads):
        average_gradients(grads, world)

    r = measure_step(args, cfg, dev, world, rank, barrier, exchange)
    ms, ms_e2e = r["ms"], r["ms_e2e"]
    tokens_step = cfg.batch * cfg.seq_len
    value = whole_job_rate(tokens_step, world, ms)
    value_e2e = whole_job_rate(tokens_step, world, ms_e2e)
    fpt = cfg.flops_per_token()
    mfu = fpt * value / (world * B200_DENSE_BF16_PEAK)

    peaks, peak_src = load_peaks()
    peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    g_ms, g_calls, g_fl, _ = r["prof"]["gemm"]
    g_ms_step = g_ms / r["prof_steps"]
    method = gemm_method_flops(cfg)
    achieved = (method / (g_ms_step / 1e3)) / 1e12 if g_ms > 0 else None
    executed = (g_fl / (g_ms / 1e3)) / 1e12 if g_ms > 0 else None
    workload = f"{cfg.name} GPT fwd+bwd step"
    line = {
        "metric": METRIC,
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,0.02) params, "
                                   f"{cfg.token_dist} token ids)",
        "mfu": mfu, "mfu_of_measured_sustained": fpt * value / (world * peak_sus * 1e12),
        "flops_per_token": fpt,
        "config": workload_config(cfg, world),
        "loss_first_step": r["loss0"],
        "e2e": {"value": value_e2e, "unit": "tokens/s",
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": 4},
        "gpu_launches": int(r["launches"]),
        "step_launch": r["step_launch"],
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_sus, "unit": "TFLOP/s",
                     "frac": (achieved / peak_sus) if achieved else None,
                     "peak_source": f"bf16_tflops_sustained of {peak_src}",
                     "kernel": "tcgen05 GEMM family (all projection, MLP and lm-head GEMMs)",
                     "achieved_basis": "6·(N − V·d)·B·T FLOP per step (the method's GEMM work) ÷ the "
                                       "family's summed CUDA-event time per step",
                     "gemm_method_flops_per_step": method,
                     "gemm_ms_per_step": g_ms_step,
                     "executed_tflops": executed,
                     "executed_basis": "all launched GEMM FLOPs, including the lm-head logit recompute "
                                       "of the backward pass (2·B·T·d·V per step)",
                     **traffic_fields(workload)},
        "kernels": r["kernels"],
        "clocks": r["clocks"],
    }
    if world == 1 and not args.no_optim:
        line["optimizer"] = measure_optimizer(args, cfg, torch.device("cuda", local), r["params_np"])
    # the other configuration the ≥ 45% MFU target names, measured in the same run
    if world == 1 and not args.no_also and cfg.name != args.also:
        import dataclasses
        acfg = preset(args.also)
        a_args = dataclasses.replace(args) if dataclasses.is_dataclass(args) else argparse.Namespace(**vars(args))
        a_args.steps = min(args.steps, 10)
        ra = measure_step(a_args, acfg, dev, world, rank, barrier, exchange, with_e2e=False)
        av = whole_job_rate(acfg.batch * acfg.seq_len, world, ra["ms"])
        ag_ms, _, ag_fl, _ = ra["prof"]["gemm"]
        ag_step = ag_ms / ra["prof_steps"]
        line["also"] = {acfg.name: {
            "workload": f"{acfg.name} GPT fwd+bwd step", "config": workload_config(acfg, world),
            "steps": a_args.steps, "warmup": args.warmup, "ms_per_step": ra["ms"], "tokens_per_s": av,
            "mfu": acfg.flops_per_token() * av / B200_DENSE_BF16_PEAK,
            "gemm_tflops_method": gemm_method_flops(acfg) / (ag_step / 1e3) / 1e12 if ag_ms > 0 else None,
            "kernels": ra["kernels"], "clocks": ra["clocks"], "loss_first_step": ra["loss0"]}}
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cores = cpu_cores()
        scfg, times = time_oracle(cfg, args.cpu_sample_tokens, repeats=args.cpu_repeats, warmup=0,
                                  params=r["params_np"])
        med = statistics.median(times)
        cv = scfg.seq_len / med
        line["cpu_baseline"] = {
            "value": cv, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"one row of {scfg.seq_len} tokens of the {cfg.name} model (B=1), fp32 NumPy "
                      f"oracle fwd+bwd, median of {len(times)} runs "
                      f"({', '.join(f'{t:.1f}' for t in times)} s)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------------------------------------
# single-kernel workloads (GEMM shapes of the step; the causal-attention sweep)
# ------------------------------------------------------------------------------------------------
def run_kernel(args):
    """Time one kernel-level call through the C ABI; prints one JSON line (not the step metric)."""
    import torch
    from gpt_decoder_pretraining_b200 import step as S
    from gpt_decoder_pretraining_b200.inputs import make_attention_inputs
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    peaks, src = load_peaks()
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    if args.kernel == "gemm":
        M, N, K = (int(x) for x in args.gemm_shape.split(","))
        op = {"nt": 0, "nn": 1, "tn": 2}[args.gemm_op]
        a_shape = (K, M) if op == 2 else (M, K)
        b_shape = (N, K) if op == 0 else (K, N)
        A = torch.randn(a_shape, device=dev, generator=g).to(torch.bfloat16)
        B = torch.randn(b_shape, device=dev, generator=g).to(torch.bfloat16)
        C = torch.empty(M, N, device=dev, dtype=torch.float32 if op == 2 else torch.bfloat16)
        epi = {"auto": S.EPI_F32 if op == 2 else S.EPI_BF16, "bf16": S.EPI_BF16, "resid": S.EPI_RESID,
               "relu2": S.EPI_RELU2, "drelu2": S.EPI_DRELU2, "f32": S.EPI_F32}[args.gemm_epi]
        if epi in (S.EPI_F32,) and C.dtype != torch.float32:
            C = torch.empty(M, N, device=dev, dtype=torch.float32)
        if epi not in (S.EPI_F32,) and C.dtype != torch.bfloat16:
            C = torch.zeros(M, N, device=dev, dtype=torch.bfloat16)
        aux = torch.rand(M, N, device=dev, generator=g).to(torch.bfloat16) if epi == S.EPI_DRELU2 else None
        scratch = None if args.no_stream_k else "auto"
        run = lambda: S.gemm(op, epi, A, B, C, M, N, K, aux=aux, scratch=scratch)  # noqa: E731
        flops = 2.0 * M * N * K
        unit_desc = f"GEMM {args.gemm_op} M={M} N={N} K={K}"
    elif args.kernel == "wgrad":
        # one layer's four weight gradients in one grouped launch: dW_proj [d, 4d], dW_fc [4d, d],
        # dW_o [d, d], dW_qkv [3d, d], all over K = tokens
        K, d = (int(x) for x in args.wgrad.split(","))
        shapes = [(d, 4 * d), (4 * d, d), (d, d), (3 * d, d)]
        probs = []
        for Mw, Nw in shapes:
            A = torch.randn(K, Mw, device=dev, generator=g).to(torch.bfloat16)
            B = torch.randn(K, Nw, device=dev, generator=g).to(torch.bfloat16)
            probs.append((A, B, torch.empty(Mw, Nw, device=dev)))
        scratch = None if args.no_stream_k else "auto"
        run = lambda: S.gemm_group_tn(probs, K, S.EPI_F32, scratch=scratch)  # noqa: E731
        flops = 2.0 * K * sum(Mw * Nw for Mw, Nw in shapes)
        unit_desc = f"grouped weight gradients K={K} d={d} (d x 4d, 4d x d, d x d, 3d x d)"
    elif args.kernel == "qkv":
        # QKV projection with the RoPE + QK-norm epilogue: r [M, d] · W_qkv [3d, d]ᵀ → q̃, k̃, v head-major
        M, d, H = (int(x) for x in args.qkv.split(","))
        Dh, T = d // H, 2048
        Bq = max(1, M // T)
        M = Bq * T
        r = torch.randn(M, d, device=dev, generator=g).to(torch.bfloat16)
        w = (torch.randn(3 * d, d, device=dev, generator=g) * 0.02).to(torch.bfloat16)
        heads = torch.empty(3 * M * d, device=dev, dtype=torch.bfloat16)
        rq = torch.empty(M * H, device=dev)
        rk = torch.empty(M * H, device=dev)
        cs = torch.empty(T * Dh, device=dev)
        S.rope_table(cs, T, Dh)
        run = lambda: S.qkv_proj_rope(r, w, heads, rq, rk, cs, Bq, T, H, Dh)  # noqa: E731
        flops = 2.0 * M * 3 * d * d
        unit_desc = f"QKV projection + RoPE + QK-norm M={M} d={d} H={H}"
    elif args.kernel == "rmsnorm":
        # RMSNorm forward and backward (bf16 dy, fp32 accumulate + bf16 copy) on [rows, d]
        rows, d = (int(x) for x in args.rows_d.split(","))
        x = torch.randn(rows, d, device=dev, generator=g).to(torch.bfloat16)
        y = torch.empty_like(x)
        rho = torch.empty(rows, device=dev)
        dy = torch.randn(rows, d, device=dev, generator=g).to(torch.bfloat16)
        gx = torch.zeros(rows, d, device=dev)
        gxb = torch.empty_like(x)
        if args.norm_pass == "fwd":
            run = lambda: S.rmsnorm_fwd(x, y, rho)  # noqa: E731
            nbytes = 4.0 * rows * d + 4.0 * rows
        else:
            S.rmsnorm_fwd(x, y, rho)
            run = lambda: S.rmsnorm_bwd(dy, y, rho, gx, gxb, accumulate=True)  # noqa: E731
            nbytes = 14.0 * rows * d + 4.0 * rows
        flops = None
        unit_desc = f"RMSNorm {args.norm_pass} rows={rows} d={d}"
    elif args.kernel == "embedding":
        # embedding backward (sort, fixed-order pieces, fix-up) on Zipf(1.1) ids
        from gpt_decoder_pretraining_b200.inputs import make_tokens as mk
        M, d, V = (int(x) for x in args.emb.split(","))
        tok_np, _ = mk(1, M, V, "zipf1.1")
        tok = torch.from_numpy(tok_np.reshape(-1)).to(dev)
        gx = torch.randn(M, d, device=dev, generator=g)
        dw = torch.empty(V, d, device=dev)
        scr = torch.empty(S.embedding_bwd_scratch_bytes(M, d, V), dtype=torch.uint8, device=dev)
        run = lambda: S.embedding_bwd(tok, gx, dw, scr)  # noqa: E731
        nbytes = 4.0 * M * d + 4.0 * V * d
        flops = None
        unit_desc = f"embedding bwd M={M} d={d} V={V} (Zipf ids)"
    else:
        T, Dh, W = (int(x) for x in args.attn.split(","))
        H = args.attn_heads
        Bt = max(1, args.attn_rows // (H * T))
        q, k, v, do = (torch.from_numpy(a).to(dev).to(torch.bfloat16)
                       for a in make_attention_inputs(Bt, H, T, Dh))
        o = torch.empty_like(q)
        lse = torch.empty(Bt, H, T, device=dev)
        strides = (H * T * Dh, T * Dh, Dh)
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        delta = S.attention_bwd_scratch(Bt, H, T, dev)
        Wf = W if 0 < W < T else T
        pairs = Wf * (Wf + 1) / 2 + (T - Wf) * Wf
        if args.attn_pass == "fwd":
            run = lambda: S.attention_fwd(q, k, v, o, lse, W, strides, strides, Bt, H, T, Dh)  # noqa: E731
            flops = 4.0 * Dh * pairs * H * Bt
        else:
            S.attention_fwd(q, k, v, o, lse, W, strides, strides, Bt, H, T, Dh)
            run = lambda: S.attention_bwd(q, k, v, o, do, lse, delta, dq, dk, dv, W, strides, strides,  # noqa: E731
                                          Bt, H, T, Dh)
            flops = 8.0 * Dh * pairs * H * Bt
        unit_desc = f"causal attention {args.attn_pass} B={Bt} H={H} T={T} Dh={Dh} window={W or 'full'}"
    for _ in range(max(3, args.warmup)):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    if flops is None:
        gbs = nbytes / (ms / 1e3) / 1e9
        peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        print(json.dumps({"kernel": unit_desc, "ms": ms, "gbs": gbs, "algorithmic_bytes": nbytes,
                          "peak_hbm_gbs": peak, "frac_of_hbm": gbs / peak, "peak_source": src,
                          "steps": args.steps}), flush=True)
        return 0
    tf = flops / (ms / 1e3) / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    print(json.dumps({"kernel": unit_desc, "ms": ms, "tflops": tf, "peak_burst_tflops": peak,
                      "frac_of_burst": tf / peak, "peak_source": src, "steps": args.steps}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="d24")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-sample-tokens", type=int, default=2048,
                    help="tokens of the one-row CPU oracle sample timed for cpu_baseline")
    ap.add_argument("--cpu-repeats", type=int, default=3, help="timed oracle runs (median reported)")
    ap.add_argument("--ref-sample-tokens", type=int, default=512,
                    help="tokens of the one-row oracle sample of each --impl reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--also", default="d20", help="second configuration measured in the same run")
    ap.add_argument("--no-also", action="store_true")
    ap.add_argument("--no-optim", action="store_true", help="skip the optimizer-step measurement")
    ap.add_argument("--no-graph", action="store_true", help="launch the step's kernels from the host "
                    "instead of replaying it as one CUDA graph")
    ap.add_argument("--rows-d", default="65536,1536", help="rmsnorm workload: rows,d")
    ap.add_argument("--norm-pass", default="fwd", choices=["fwd", "bwd"])
    ap.add_argument("--emb", default="32768,1536,32768", help="embedding workload: M,d,V")
    ap.add_argument("--qkv", default="8192,1536,12", help="QKV projection workload: tokens,d,heads")
    ap.add_argument("--wgrad", default="32768,1536", help="grouped weight-gradient workload: tokens,d")
    ap.add_argument("--kernel", choices=["gemm", "attention", "rmsnorm", "embedding", "qkv", "wgrad"], default=None,
                    help="time one kernel-level workload instead of the step")
    ap.add_argument("--gemm-shape", default="32768,6144,1536")
    ap.add_argument("--gemm-op", default="nt", choices=["nt", "nn", "tn"])
    ap.add_argument("--gemm-epi", default="auto", choices=["auto", "bf16", "resid", "relu2", "drelu2", "f32"])
    ap.add_argument("--no-stream-k", action="store_true", help="GEMM workload: every tile whole")
    ap.add_argument("--attn", default="2048,128,0", help="T,Dh,window (window 0 = full causal)")
    ap.add_argument("--attn-pass", default="fwd", choices=["fwd", "bwd"])
    ap.add_argument("--attn-rows", type=int, default=1 << 21, help="batch·heads·seq of the attention workload")
    ap.add_argument("--attn-heads", type=int, default=8)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.kernel:
        return run_kernel(args)
    cfg = preset(args.config)
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
