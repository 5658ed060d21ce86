"""The benchmark's reference arm (the fp64 oracle timed on the host) prints the JSON line
the driver reads, with the keys it needs; under several ranks only rank 0 runs and prints.
Host only: the tiny workload, a fraction of a second of oracle work per step; and the
algorithmic bytes behind the roofline object, against closed forms."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra, *args):
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--ref-step-seconds", "0.3", *args], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    return [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_reference_arm_prints_the_contract_line():
    lines = _run({}, "--steps", "2", "--warmup", "1")
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == "decode-attn tokens/s" and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 2, 1)
    assert d["scaling"] == "weak" and d["vs_baseline"] is None and d["data"] == "synthetic"
    assert d["config"]["workload"] == "tiny"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_runs_on_rank_zero_only():
    assert _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, "--steps", "1", "--warmup", "0") == []
    lines = _run({"RANK": "0", "WORLD_SIZE": "2", "LOCAL_RANK": "0"}, "--steps", "1", "--warmup", "0")
    assert len(lines) == 1 and json.loads(lines[0])["n_gpus"] == 2


def test_algorithmic_bytes_of_a_llama8b_step():
    """The roofline numerator: per decode launch, every cached row's K and V, q, the fp32
    output and the appended token read and written; per step, one read of the keys and the
    window queries plus the scores written, and the kept rows gathered. Closed forms for
    the LLaMA-3-8B shape (32 slots, G 4, d 128, bf16, L 8192, w 32, top-1024, 64 steps)."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    from workloads import get
    wl = get("llama8b")
    S, B, T = 32, 1024, 64
    work = bench.work_per_step(wl, np.full(S, B), 0)
    row = 2 * 128 * 2                                      # one row of K and V, bf16
    fixed = S * 4 * 128 * 2 + S * 4 * 128 * 4 + 2 * S * row
    assert work["decode_bytes"] == [(S * B + S * (t + 1)) * row + fixed for t in range(T)]
    assert sum(work["decode_bytes"]) / T == 17440768       # the figure the bench reports per launch
    assert work["compact_bytes"] == S * B * 2 * row + S * B * 4
    assert work["score_bytes"] == S * 8192 * 128 * 2 + S * 4 * 32 * 128 * 2 + S * 8192 * 4
    assert work["score_flops"] == 2.0 * S * 4 * 32 * 8192 * 128
