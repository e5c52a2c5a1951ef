"""bench.py's JSON line on CPU: the algorithmic FLOP counts against closed forms, and the keys
and arithmetic of the reported line built from a synthetic per-kernel profile."""
import types

import pytest

import bench
import synthetic as S


def test_algorithmic_flops_closed_forms():
    spec = S.WORKLOADS["vitl16_1024_b8"].spec
    T, D, F = 4101, 1024, 4096
    f = bench.kernel_flops(spec, 8)
    assert f["attention"] == 4.0 * 8 * T * T * D                 # QK^T and PV, 2 FLOP per MAC each
    assert f["qkv_gemm"] == 2.0 * 8 * T * 3 * D * D
    assert f["fc1_gemm"] == f["fc2_gemm"] == 2.0 * 8 * T * D * F
    assert f["patch_gemm"] == 2.0 * 8 * 4096 * D * 3 * 16 * 16
    # per image: ViT-L/16@1024 GEMMs ~2483 GFLOP + attention ~1653 = ~4137; ViT-S/16@336 GEMMs
    # ~19.2 GFLOP + attention ~3.67
    assert bench.total_flops(spec, 1) == pytest.approx(4.137e12, rel=2e-3)
    assert spec.depth * bench.kernel_flops(spec, 1)["attention"] == pytest.approx(1653e9, rel=2e-3)
    s_spec = S.WORKLOADS["vits16_336_b64_outlier"].spec
    s_att = s_spec.depth * bench.kernel_flops(s_spec, 1)["attention"]
    assert s_att == pytest.approx(3.67e9, rel=1e-2)
    assert bench.total_flops(s_spec, 1) - s_att == pytest.approx(19.2e9, rel=1e-2)


def test_report_line_carries_the_contract_keys():
    wl = S.WORKLOADS["vitl16_1024_b8"]
    spec, B, steps = wl.spec, 8, 10
    args = types.SimpleNamespace(steps=steps, warmup=3)
    L = spec.depth * steps
    prof = {"attention": (9.65 * L / 10, L), "qkv_gemm": (1.6 * L / 10, L), "proj_gemm": (0.9 * L / 10, L),
            "fc1_gemm": (2.4 * L / 10, L), "fc2_gemm": (2.3 * L / 10, L), "final_ln": (0.06 * steps / 10, steps)}
    ms_total = 41.2 * steps
    peaks = {"hbm_gbs": 6548.0, "bf16_tflops": 1642.0, "bf16_tflops_sustained": 1397.0, "source": "measured"}
    enc = types.SimpleNamespace(w={}, wb=[])
    imgs = [types.SimpleNamespace(numel=lambda: B * 3 * 1024 * 1024)]
    e2e = {"value": 190.0, "unit": "images/s", "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 1}
    clk = {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": []}
    value = B * steps / (ms_total / 1000.0)
    line = bench.report(args, spec, wl, B, 1, prof, ms_total, value, e2e, 124, clk, peaks, imgs, enc)
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in line, k
    assert line["ms_per_step"] == pytest.approx(41.2)
    assert line["gpu_launches"] == 124 * steps
    r = line["roofline"]
    assert r["kernel"] == "attention" and r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(bench.kernel_flops(spec, B)["attention"] / 0.965e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1397.0)
    step_tflops = bench.total_flops(spec, B) / 41.2e-3 / 1e12
    assert line["tflops_per_gpu"] == pytest.approx(step_tflops)
    assert line["frac_of_bf16_peak"]["measured_sustained"] == pytest.approx(step_tflops / 1397.0)
    assert line["frac_of_bf16_peak"]["spec_dense_2250"] == pytest.approx(step_tflops / 2250.0)
    assert line["kernels"]["final_ln"]["gbs"] > 0


def test_cpu_baseline_decomposition_matches_a_full_oracle_run():
    """The CPU baseline times the oracle's per-image work outside the blocks once (the patch
    embedding on a strip, scaled by the patch count) plus one block counted depth times; on a
    small encoder that sum must agree with a full oracle forward to within timing noise."""
    import time
    import oracle as O
    spec = S.PRESETS["small_s16"]
    w = O.to_f64_weights(S.make_weights(spec, 3))
    im = S.make_images(spec, 1, 4)
    best_full = min(_timed(lambda: O.forward(im, w, spec)) for _ in range(3))
    est = []
    for _ in range(3):
        t_fixed, desc = bench.oracle_fixed_part(spec, w, im)
        est.append(t_fixed + spec.depth * bench.oracle_block_time(spec, w))
    assert "patch rows" in desc
    assert 0.33 * best_full <= min(est) <= 3.0 * best_full, (min(est), best_full)


def _timed(fn):
    import time
    t0 = time.perf_counter()
    fn()
    return time.perf_counter() - t0


def test_clock_sampler_summarises_only_the_timed_window(monkeypatch):
    """The sampler waits for nvidia-smi's first line, and mark() opens the window that stop()
    summarises: samples taken before the timed region (an idle clock) are left out, throttle
    reasons inside it are reported."""
    import io
    import time as _time
    pre = "0, 1965, 1965, 120.5, 0x0, Not Active, Not Active, Not Active, Not Active\n"
    inside = ["0, 1700, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active\n",
              "0, 1680, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active\n",
              "0, 1720, 1965, 940.0, 0x4, Not Active, Not Active, Not Active, Active\n"]

    class FakeProc:
        def __init__(self, *a, **k):
            self.stdout = io.StringIO(pre)
            self.alive = True

        def poll(self):
            return None if self.alive else 0

        def terminate(self):
            self.alive = False

        def wait(self, timeout=None):
            return 0

        def kill(self):
            self.alive = False

    monkeypatch.setattr(bench.subprocess, "Popen", FakeProc)
    cs = bench.ClockSampler(0)
    cs.start()
    t0 = _time.time()
    while not cs.lines and _time.time() - t0 < 2:
        _time.sleep(0.01)
    assert cs.lines == [pre.strip()]
    cs.mark()
    cs.lines.extend(x.strip() for x in inside)     # what the reader thread appends meanwhile
    clk = cs.stop()
    assert clk["samples"] == 3
    assert clk["sm_mhz"] == 1700.0 and clk["sm_max_mhz"] == 1965.0
    assert clk["reasons"] == ["sw_power_cap"]
    assert clk["power_w"] == 940.0
