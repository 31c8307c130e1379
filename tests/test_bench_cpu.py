"""bench.py's reference arm on CPU: one JSON line with the contract's keys.

The reference arm times the fp64 oracle on the host cores; it needs no GPU, so
its launch, its JSON line and its argument checks are tested here.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True,
                          text=True, timeout=600, cwd=ROOT)


def test_reference_arm_prints_one_contract_line():
    r = _bench("--impl", "reference", "--workload", "gdn_decode_256x16", "--steps", "1", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["config"]["workload"] == "gdn_decode_256x16"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_warmup_below_three_is_rejected():
    r = _bench("--impl", "reference", "--workload", "gdn_decode_256x16", "--steps", "1", "--warmup", "1")
    assert r.returncode != 0 and "--warmup must be >= 3" in r.stderr


def test_reference_arm_under_torchrun_prints_one_line():
    """Launched the way multi-GPU runs are (torchrun, two ranks, 127.0.0.1), rank 0
    alone times the oracle and prints; the other rank exits 0 without work."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
                        "--impl", "reference", "--gpus", "2", "--workload", "gdn_decode_256x16", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0


def test_reference_arm_times_the_oracle_backward():
    """The backward workload's reference arm times the oracle's reverse mode on one sequence per step."""
    r = _bench("--impl", "reference", "--workload", "gdn_bwd_350m", "--steps", "1", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][0])
    assert d["config"]["workload"] == "gdn_bwd_350m" and d["value"] > 0
    assert "backward" in d["cpu_baseline"]["sample"]
