"""Host-side logic of bench.py that needs no GPU: the clock-record summary keeps only
the samples taken inside the timed window, and reports throttle reasons seen there."""
import bench

ROW = "{sm}, 1965, 900, Not Active, Not Active, Not Active, {cap}"


def _sampler(samples, window):
    c = bench.ClockSampler("0")
    c.lines = [(t, ROW.format(sm=sm, cap="Active" if cap else "Not Active")) for t, sm, cap in samples]
    c.window = window
    return c


def test_summary_uses_the_timed_window_only():
    c = _sampler([(0.9, 1965, False), (1.1, 1500, True), (1.2, 1400, True), (1.3, 1450, True), (2.5, 1965, False)],
                 [1.0, 1.4])
    s = c.summary()
    assert s["samples"] == 3 and s["timed_window_only"]
    assert s["sm_mhz"] == 1450 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_summary_falls_back_to_all_samples():
    c = _sampler([(0.9, 1965, False), (2.5, 1800, False)], [1.0, 1.4])
    s = c.summary()
    assert s["samples"] == 2 and not s["timed_window_only"] and s["reasons"] == []


def test_summary_without_samples():
    assert _sampler([], None).summary()["samples"] == 0


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the oracle on a bounded sample) needs no GPU."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "2",
                          "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == "llm_train_causal"
