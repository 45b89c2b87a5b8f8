"""The benchmark's JSON contract, checked on the CPU through its reference arm (the oracle).

The GPU arm's line is checked by the GPU runs; here the fields every line must carry, their types,
and the multi-rank rule (rank 0 alone prints; the other ranks exit 0 without work).
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
REQUIRED = {"metric": str, "value": float, "unit": str, "n_gpus": int, "steps": int, "warmup": int,
            "ms_per_step": float, "higher_is_better": bool, "scaling": str, "dtype": str, "data": str,
            "config": dict, "cpu_baseline": dict, "e2e": dict}


def json_lines(out: str):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def check_line(d, n_gpus, steps, warmup):
    for k, t in REQUIRED.items():
        assert k in d, k
        assert isinstance(d[k], t), (k, type(d[k]))
    assert "vs_baseline" in d and d["vs_baseline"] is None
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (n_gpus, steps, warmup)
    assert d["scaling"] == "weak" and d["data"] == "synthetic" and "workload" in d["config"]
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["e2e"]["d2h_bytes_per_step"] == 0 and d["e2e"]["unit"] == d["unit"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3",
                        "--ref-budget-s", "2"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1
    check_line(lines[0], 1, 2, 3)


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_under_two_ranks_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(free_port()), "bench.py", "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "3", "--ref-budget-s", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1
    check_line(lines[0], 2, 1, 3)


def test_profile_commands_name_existing_probes():
    """Every ncu summary under profiles/ names the command that made it; each `--probe` it uses must be one
    that bench.py offers, so the command still runs as written."""
    import glob
    import re
    help_text = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--help"], capture_output=True,
                               text=True, check=True, timeout=120).stdout
    m = re.search(r"--probe \{([^}]*)\}", help_text)
    assert m, "bench.py --help lists no probe choices"
    offered = set(m.group(1).replace("\n", "").replace(" ", "").split(","))
    used = set()
    for path in glob.glob(os.path.join(ROOT, "profiles", "*")):
        with open(path, encoding="utf-8") as f:
            used |= set(re.findall(r"--probe ([a-z0-9_]+)", f.read()))
    assert used, "no profile names a probe"
    assert used <= offered, sorted(used - offered)
