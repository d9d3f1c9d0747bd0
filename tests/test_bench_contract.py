"""The benchmark's output contract, checked on the CPU through its reference arm (which times the
oracle on the host and needs no GPU): one JSON line with the agreed keys, types and config."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_reference_arm_prints_one_contract_line():
    d = _run("--impl", "reference", "--config", "smoke", "--steps", "2", "--warmup", "1")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["vs_baseline"] is None
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    cfg = d["config"]
    assert cfg["workload"] == "smoke GPT fwd+bwd step" and cfg["model"] == "smoke"
    assert cfg["seq_len"] == 128 and cfg["global_batch"] == 1


def test_both_arms_name_the_same_workload():
    # the GPU arm builds its config with the same function the reference arm prints
    sys.path.insert(0, ROOT)
    import bench
    from gpt_decoder_pretraining_b200.config import preset
    cfg = preset("d24")
    c1 = bench.workload_config(cfg, 1)
    assert c1["workload"] == "d24 GPT fwd+bwd step" and c1["global_batch"] == 16
    assert c1["parallelism"] == "none"
    c8 = bench.workload_config(cfg, 8)
    assert c8["global_batch"] == 128 and c8["parallelism"] == "dp8"
