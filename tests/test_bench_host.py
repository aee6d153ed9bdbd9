"""Host-side logic of bench.py that needs no GPU: the clock-record summary keeps only
the samples taken inside the timed window, and reports throttle reasons seen there."""
import bench

ROW = "{sm}, 1965, 900, Not Active, Not Active, Not Active, {cap}"


def _sampler(samples, window):
    c = bench.ClockSampler("0")
    c.samples = [bench.ClockSampler.parse_smi_line(t, ROW.format(sm=sm, cap="Active" if cap else "Not Active"))
                 for t, sm, cap in samples]
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


def test_smi_line_parsing():
    assert bench.ClockSampler.parse_smi_line(0.0, "garbage") is None
    t, sm, mx, r = bench.ClockSampler.parse_smi_line(1.0, "1500, 1965, 990.1, Active, Not Active, Not Active, Active")
    assert (sm, mx, r) == (1500.0, 1965.0, {"hw_slowdown", "sw_power_cap"})


def test_roofline_denominators():
    """The attention kernel's roofline uses its own mean launch time; the hardware
    peak at the sampled clock is 148 SMs x 8192 bf16 FLOP per clock."""
    import workloads
    w = workloads.WORKLOADS["llm_train_causal"]
    ms = w.flops / 1000e12 * 1e3          # a launch time giving exactly 1000 TFLOP/s
    r = bench.roofline(w, {"attn_fwd_sm100": ms}, 1965.0, w.name)
    assert r["bound"] == "tensor" and abs(r["achieved"] - 1000.0) < 1e-6
    assert abs(r["hw_peak_at_sampled_clock"] - 148 * 8192 * 1965e6 / 1e12) < 0.1
    assert abs(r["frac_of_datasheet_peak"] - 1000 / 2250) < 1e-4
    wv = workloads.WORKLOADS["vit_b16_batch"]
    rv = bench.roofline(wv, {"attn_fwd_sm100": 0.05}, None, wv.name)
    assert rv["bound"] == "hbm" and rv["unit"] == "GB/s"
    wf = workloads.WORKLOADS["fp8_rotated"]
    rf = bench.roofline(wf, {"attn_fwd_sm100": 1.0, "fp8_rotate_quantize": 0.1, "fp8_quantize": 0.05}, 1800.0,
                        wf.name)
    assert set(rf["prep"]) == {"fp8_rotate_quantize", "fp8_quantize"}
    assert rf["prep"]["fp8_quantize"]["algorithmic_bytes"] == 2 * 32 * 8192 * 128 * 3 + 4 * 2 * 32 * 64


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


def test_loop_steps_sizing():
    """Timed loops: the caller's count when given, else at least `minimum` steps
    and enough for the target duration (so short kernels still span several clock
    samples and the sustained loop reaches the power-capped regime)."""
    assert bench.loop_steps(7, 0.5, 10.0, 20) == 7
    assert bench.loop_steps(None, 0.55, 10.0, 20) == 20          # 20 x 0.55 ms >= 10 ms
    assert bench.loop_steps(None, 0.041, 10.0, 20) == 244        # ViT batch: ceil(10 / 0.041)
    assert bench.loop_steps(None, 0.55, 300.0, 500) == 546
    assert bench.loop_steps(None, 0.0, 10.0, 20) == 100000       # a zero estimate is floored, not divided by
    assert bench.loop_steps(0, 0.55, 300.0, 500) == 0             # an explicit 0 skips the loop


def test_sustained_denominator_fallback(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "HERE", str(tmp_path))
    assert bench.sustained_bf16_peak() == (1400.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"bf16_tflops": 1663.5, "bf16_tflops_sustained": 1410.5}')
    assert bench.sustained_bf16_peak() == (1410.5, "measured")
