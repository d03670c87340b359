"""The package's command-line runner, in each of its three forms, as a user
(and the committed profile commands) run it: exit status 0 and one JSON line
with the expected fields and consistent counts."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_cli(*args, timeout=600):
    p = subprocess.run([sys.executable, "-m", "minimax_scale_search_b200", *args], cwd=ROOT, capture_output=True,
                       text=True, timeout=timeout)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout[-2000:]
    return json.loads(lines[0])


def test_cli_selection_on_the_tiny_workload():
    out = run_cli("--workload", "1", "--repeat", "2")
    assert out["groups"] == 64 * 512 // 128 and out["E"] == 4
    assert len(out["ms"]) == 2 and all(t > 0 for t in out["ms"])
    c = out["counters"]
    assert c["nonfinite"] == 0 and c["finalists"] + c["fallback"] + c["trivial"] >= out["groups"]


def test_cli_general_spec_on_sweep_rows():
    out = run_cli("--workload", "3", "--rows", "16", "--qmin", "-4", "--qmax", "3", "--group-size", "64",
                  "--repeat", "1")
    assert out["groups"] == 16 * 16384 // 64
    assert (out["qmin"], out["qmax"], out["group_size"]) == (-4, 3, 64)
    assert out["groups_per_s"] > 0


def test_cli_secondary_kernels_once():
    out = run_cli("--ops")
    assert out["groups"] == 4096 * 16384 // 128
    for k in ("absmax", "objective", "gptq_export", "gptq_dequant_fp16", "gptq_dequant_fp32", "diagonals",
              "proxy_three_policies"):
        assert out["ms"][k] > 0, k
    assert set(out["proxy"]) == {"cliffquant", "pooled_wmse", "absmax"}
    assert all(v > 0 for v in out["proxy"].values())
