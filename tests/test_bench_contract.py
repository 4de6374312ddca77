"""bench.py's reference arm (the CPU oracle timed on the host cores) prints the
JSON line of the measurement contract: one line from rank 0, nothing from the
other ranks, every required key present.  Runs on the CPU in a few seconds."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

KEYS = ["impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
        "cpu_baseline", "e2e"]


def _json_lines(out):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


# the workload keys that the GPU arm's line carries too: both arms name the
# same configuration, so the two lines can be compared key for key
CONFIG_KEYS = ["workload", "T", "d_model", "d_latent", "experts", "top_k", "d_ff",
               "d_ff_shared", "expert_fmt", "bias", "outlier_rows", "parallelism",
               "cuda_graph", "block", "l2"]


def _check(line, steps, world=1):
    for k in KEYS:
        assert k in line, k
    assert line["impl"] == "reference" and line["steps"] == steps and line["value"] > 0
    c = line["config"]
    assert sorted(c) == sorted(CONFIG_KEYS)
    assert c["workload"] == "tiny_fp32" and c["T"] == 64 and c["experts"] == 16
    assert c["parallelism"] == f"replicas{world}"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    e = line["e2e"]
    assert e["value"] == line["value"] and e["unit"] == line["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config",
                        "tiny_fp32", "--steps", "2", "--warmup", "1"], cwd=ROOT,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check(lines[0], 2)


def test_reference_arm_under_two_ranks_prints_once():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node", "2", "--master-addr", "127.0.0.1", "--master-port",
                        str(port), "bench.py", "--impl", "reference", "--gpus", "2",
                        "--config", "tiny_fp32", "--steps", "1", "--warmup", "1"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check(lines[0], 1, world=2)
