"""Host-side pieces of the benchmark (no GPU): the flop count behind the
roofline, the launch count and the config each JSON line carries."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import muon_inputs as mi  # noqa: E402
import oracle  # noqa: E402


@pytest.mark.parametrize("wid", sorted(mi.workloads()))
def test_roofline_flops_equal_the_oracle_count(wid):
    w = mi.workloads()[wid]
    k = len(w.hp["coeffs"])
    want = sum(b.count * oracle.ns_flops_algorithmic(b.rows, b.cols, k) for b in w.banks)
    assert bench._ns_flops(w) == pytest.approx(want, rel=1e-12)


def test_gpt_bank_chain_is_1p142_tflop():
    # 48 x 768^2 + 24 x 768x3072 (both orientations), five steps
    assert bench._ns_flops(mi.workloads()[bench.WORKLOAD_ID]) == pytest.approx(1.1421587866e12, rel=1e-9)


@pytest.mark.parametrize("wid", sorted(mi.workloads()))
def test_config_names_the_workload_and_its_cache_regime(wid):
    w = mi.workloads()[wid]
    c = bench._config(w)
    assert c["workload"] and c["banks"] and c["params"] == sum(b.count * b.rows * b.cols for b in w.banks)
    assert ("larger than L2" in c["l2"]) == (wid != 1)   # only the single 256x512 matrix fits in L2
    assert bench.launches_per_step(w) == 4


def test_traffic_is_null_once_the_kernel_sources_change(monkeypatch):
    sha = bench.kernel_source_sha16()
    monkeypatch.setitem(bench.NS_CHAIN_TRAFFIC, 2, {"bytes": 1.0e9, "source_sha16": sha,
                                                    "capture": "one chain launch"})
    assert bench.chain_traffic(2) == (1.0e9, "one chain launch")
    monkeypatch.setitem(bench.NS_CHAIN_TRAFFIC, 2, {"bytes": 1.0e9, "source_sha16": "0" * 16,
                                                    "capture": "one chain launch"})
    assert bench.chain_traffic(2)[0] is None
    assert bench.chain_traffic(77)[0] is None


def test_roofline_fraction_is_of_the_burst_peak():
    peaks = dict(hbm=6500.0, burst=1600.0, sustained=1400.0, src="measured")
    r = bench._roofline(800.0, peaks, 1.0e12, 1.25, None, "none")
    assert r["peak"] == 1600.0 and r["frac"] == 0.5
    assert r["frac_of_sustained"] == pytest.approx(800.0 / 1400.0)


def test_percentiles_nearest_rank():
    assert bench._percentiles([5.0, 1.0, 3.0, 2.0, 4.0]) == [1.0, 3.0, 5.0]
    assert bench._percentiles([2.0]) == [2.0, 2.0, 2.0]


def test_source_hash_ignores_comments():
    a = "int f(int x) {  // doubles\n  return 2 * x; /* twice */\n}\n"
    b = "// a header comment\nint f(int x) {\n\n  return 2 * x;\n}\n"
    assert bench.code_only(a) == bench.code_only(b)
    assert bench.code_only(a) != bench.code_only(a.replace("2 * x", "3 * x"))
    assert bench.chain_traffic(2)[0] is not None   # the stored capture describes these sources


def test_reference_arm_fits_its_budget(monkeypatch, capsys):
    """The reference arm times the whole bank each step when the requested
    steps fit its time budget, and otherwise the first matrices of each shape
    (scaled, labelled) so that the run still ends in a few minutes. A fake
    oracle timer stands in for the float64 oracle: 6 s per whole GPT bank,
    each matrix's share proportional to R C min(R, C)."""
    import json
    import types
    calls = []

    def fake(w, step=0, max_layers=None):
        def work(cap):
            return sum((sp.count if cap is None else min(sp.count, cap)) * sp.rows * sp.cols
                       * min(sp.rows, sp.cols) for sp in w.banks)
        t = 6.0 * work(max_layers) / work(None)
        calls.append((max_layers, t, f"sample {max_layers}"))
        return t, calls[-1][2]
    monkeypatch.setattr(bench, "_oracle_bank_time", fake)
    for steps, warmup, whole in ((20, 5, True), (200, 10, False)):
        calls.clear()
        bench.run_reference(types.SimpleNamespace(workload=2, steps=steps, warmup=warmup, gpus=1))
        line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
        assert line["steps"] == steps and line["impl"] == "reference"
        assert len(calls) == steps + max(warmup, 1)
        run_s = sum(c[1] for c in calls)
        assert run_s <= bench.REFERENCE_BUDGET_S, run_s
        assert (calls[-1][0] is None) == whole
        assert line["cpu_baseline"]["sample"].endswith(calls[-1][2])
