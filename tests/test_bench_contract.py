"""bench.py's output contract, checked on its CPU arm: `--impl reference` times the oracle
on this machine's cores and prints one JSON line with the keys every bench line carries,
plus the CPU-baseline and end-to-end objects that describe this run.  CPU only."""
import json
import os
import socket
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

COMMON_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
               "scaling", "vs_baseline", "dtype", "data", "config"}


def run_reference_arm(*extra):
    t0 = time.perf_counter()
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", *extra], cwd=ROOT,
                         capture_output=True, text=True, timeout=600, check=True).stdout
    wall = time.perf_counter() - t0
    lines = [ln for ln in out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out  # exactly one JSON line
    d = json.loads(lines[0])
    d["_wall_s"] = wall
    return d


def test_reference_arm_line():
    d = run_reference_arm("--steps", "1", "--warmup", "0")
    assert COMMON_KEYS <= set(d)
    assert d["impl"] == "reference"
    assert d["n_gpus"] == 1 and d["steps"] == 1
    assert d["warmup"] >= 3  # the timing rules' minimum, whatever was asked for
    assert d["higher_is_better"] is True and d["unit"] == "tokens/s"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"] == "mla_decode_b8_ctx131072_top2048"
    # the line reports the steps it ran: one request each (a fraction of a token), and
    # steps x ms_per_step fits inside the process's own wall time
    assert d["config"]["batch"] == 1
    f = d["config"]["tokens_per_step"]
    assert 0 < f <= 1
    assert abs(d["value"] - f / (d["ms_per_step"] / 1e3)) <= 1e-6 * d["value"]
    assert (d["steps"] + d["warmup"]) * d["ms_per_step"] / 1e3 <= d["_wall_s"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == d["value"] and cb["unit"] == d["unit"]
    st = cb["single_thread"]
    assert st["cores"] == 1 and st["value"] > 0 and st["kind"] == "oracle" and st["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_under_torchrun_prints_once():
    """Two ranks on this machine: rank 0 alone times the oracle and prints; rank 1 exits 0."""
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    out = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                          "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
                          "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600, check=True).stdout
    lines = [ln for ln in out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
