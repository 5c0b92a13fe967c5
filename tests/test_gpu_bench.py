"""The benchmark's own code paths on the GPU, run as the harness runs them.

Each test starts `bench.py` in a subprocess with a few steps and checks the
one JSON line it prints: the keys of the output contract, the roofline
object of the chain (and of the 64 x 1024^2 bank), the end-to-end leg, the
CPU-oracle baseline, and that the numbers are positive and consistent. The
data-parallel path runs under torchrun with one rank (the same code the
multi-GPU run uses, with one NCCL rank).
"""
import json
import os
import socket
import subprocess
import sys
import tempfile

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "e2e")


def _run(args, timeout=900):
    env = dict(os.environ, MUON_BENCH_CLOCKS_DIR=tempfile.mkdtemp(prefix="muon_bench_clocks_"))
    r = subprocess.run(args, cwd=ROOT, capture_output=True, text=True, timeout=timeout, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _check_common(d, steps):
    for k in KEYS:
        assert k in d, k
    assert d["steps"] == steps and d["value"] > 0 and d["ms_per_step"] > 0
    assert abs(d["value"] * d["ms_per_step"] / 1e3 - 1.0) < 0.05   # steps/s and ms/step agree
    assert d["config"]["workload"] == "gpt124m_matrix_bank"
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] == e["d2h_bytes_per_step"] == 169869312
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert 0 < r["frac"] < 1.2 and r["achieved"] == pytest.approx(r["frac"] * r["peak"])
    # a floor well under the ~0.5 of burst the chain reaches in short runs:
    # a regression of the Newton-Schulz kernel fails here, not only in a number
    assert r["frac"] > 0.35, r["frac"]
    assert r["flops_per_launch"] == pytest.approx(1.1421587866e12, rel=1e-9)
    assert d["gpu_launches"] == 4 * steps


def test_single_gpu_line():
    d = _run([sys.executable, "bench.py", "--steps", "5", "--warmup", "3", "--e2e-steps", "4"])
    _check_common(d, 5)
    assert d["n_gpus"] == 1 and d["dtype"] == "bf16"
    sq = d["roofline_square_1024x1024x64"]
    assert sq and 0 < sq["frac"] < 1.2 and sq["steps"] == 20
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and 0 < cpu["value"] < d["value"]
    assert "72 matrices" in cpu["sample"]
    # the chain plus the two passes make up the step
    b = d["breakdown_ms"]
    assert b["ns_chain"] + b["momentum_norm"] + b["update"] <= d["ms_per_step"] * 1.1
    assert d["roofline"]["launch_ms"] == pytest.approx(b["ns_chain"])
    assert len(d["step_ms_p10_p50_p90"]) == 3


def test_data_parallel_line_under_torchrun():
    d = _run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "1",
              "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
              "--gpus", "1", "--steps", "5", "--warmup", "3", "--e2e-steps", "4"])
    _check_common(d, 5)
    assert d["scaling"] == "strong" and d["config"]["parallelism"].startswith("dp1")
    assert d["sharded"]["load_max_over_mean"] == pytest.approx(1.0)


def test_reference_arm_times_the_oracle_on_the_whole_bank():
    d = _run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert d["impl"] == "reference" and d["dtype"] == "f64" and d["value"] > 0
    assert d["cpu_baseline"]["value"] == d["value"] and "72 matrices" in d["cpu_baseline"]["sample"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
