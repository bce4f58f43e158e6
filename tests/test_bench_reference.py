"""bench.py's reference arm (the CPU oracle timed on the host cores) keeps the
JSON-line contract on the CPU: one line from rank 0, the required keys, at
least three warm-up steps, no GPU launches, and host-copy byte counts of 0.
Under torchrun with two gloo ranks only rank 0 prints."""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
        "cpu_baseline", "e2e", "gpu_launches"}


def _env():
    env = dict(os.environ)
    env.pop("RANK", None)
    env.pop("WORLD_SIZE", None)
    env["CUDA_VISIBLE_DEVICES"] = ""
    return env


def _json_lines(text):
    return [json.loads(line) for line in text.splitlines() if line.startswith("{")]


def _run(args, timeout=240):
    p = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, env=_env(),
                       capture_output=True, text=True, timeout=timeout)
    assert p.returncode == 0, p.stderr[-2000:]
    return _json_lines(p.stdout)


def _check_line(line, steps):
    assert KEYS <= set(line), KEYS - set(line)
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["steps"] == steps and line["warmup"] >= 3
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["vs_baseline"] is None and line["gpu_launches"] == 0
    assert line["config"]["workload"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == line["value"] and cb["unit"] == line["unit"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


@pytest.mark.parametrize("workload", ["tiny", "rope_write", "cow_copy"])
def test_reference_line(workload):
    lines = _run(["--impl", "reference", "--workload", workload, "--steps", "2", "--warmup", "1",
                  "--cpu-seconds", "0.2"])
    assert len(lines) == 1
    _check_line(lines[0], steps=2)


def test_reference_unavailable_for_graph_replay():
    lines = _run(["--impl", "reference", "--workload", "graph_decode", "--steps", "2"])
    assert len(lines) == 1 and lines[0]["impl"] == "reference" and lines[0]["unavailable"]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--gpus", "2", "--impl", "reference", "--workload", "tiny", "--steps", "2",
           "--warmup", "3", "--cpu-seconds", "0.2"]
    p = subprocess.run(cmd, cwd=ROOT, env=_env(), capture_output=True, text=True, timeout=240)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = _json_lines(p.stdout)
    assert len(lines) == 1
    _check_line(lines[0], steps=2)
    assert lines[0]["n_gpus"] == 2
