"""bench.py's host-side bookkeeping on CPU: how exactly --steps steps are cut
into graph replays, the operand type reported per workload, and the JSON
fields summarize() derives from a measurement (units, roofline fractions,
the peak a long tensor-bound region is measured against, quantiles, e2e).
No GPU: the measurement is a hand-made result dictionary."""
import os
import sys
from types import SimpleNamespace

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402

PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}


@pytest.mark.parametrize("steps", [1, 3, 10, 20, 100, 200, 400, 997])
@pytest.mark.parametrize("pool", [1, 2, 4, 9, 16, 2944])
def test_segments_cover_exactly_the_steps(steps, pool):
    seg = bench.segment_len(steps, pool)
    assert 1 <= seg <= min(pool, 16)
    assert steps % seg == 0          # whole replays, exactly `steps` steps


def test_operand_type_per_workload():
    assert bench.arith_dtype("int4", 5) == "f16"
    assert bench.arith_dtype("int8", 5) == "f16"
    assert bench.arith_dtype("mxfp8", 4) == "f16"
    assert bench.arith_dtype("int4", 32) == "bf16"
    assert bench.arith_dtype("mxfp8", 128) == "bf16"
    assert bench.arith_dtype("bf16", 4) == "bf16"
    assert bench.kernel_of("mxfp8", 4) == "w4a16_stream_kernel"
    assert bench.kernel_of("mxfp8", 32) == "mxfp8_stream_kernel"
    assert bench.kernel_of("int4", 128) == "tc_gemm_kernel"


def fake_workload(name):
    fmt, M, layers, G = bench.WORKLOADS[name]
    step_bytes = sum(bench.layer_weight_bytes(fmt, K, N, G) for K, N in layers)
    step_flops = sum(2 * M * N * K for K, N in layers)
    return SimpleNamespace(name=name, fmt=fmt, M=M, layers=layers, G=G, step_bytes=step_bytes,
                           step_flops=step_flops, kernel=bench.kernel_of(fmt, M), pool=4)


def fake_result(step_us, layers, steps, e2e=False):
    per_layer = [step_us / layers] * layers
    res = {"elapsed_ms": step_us * steps / 1e3, "per_step_ms": [step_us / 1e3] * (steps // 4),
           "in_step_us": per_layer, "isolated_us": [v * 1.5 for v in per_layer],
           "cycle_steps": 4}
    if e2e:
        res.update({"e2e_steps": steps, "e2e_eager_ms": 2 * step_us * steps / 1e3,
                    "e2e_plain_ms": 3 * step_us * steps / 1e3,
                    "e2e_graph_ms": 1.5 * step_us * steps / 1e3, "h2d": 1000, "d2h": 2000})
    return res


def test_hbm_bound_summary():
    wl = fake_workload("mtp4_verify_int4")
    out = bench.summarize(wl, fake_result(50.0, 3, 200, e2e=True), 200, 1, PEAKS, "measured")
    tbps = wl.step_bytes / 50e-6 / 1e12
    assert out["unit"] == "TB/s" and out["value"] == pytest.approx(tbps, rel=1e-3)
    r = out["roofline"]
    assert r["bound"] == "hbm" and r["peak"] == PEAKS["hbm_gbs"]
    assert r["frac"] == pytest.approx(tbps * 1e3 / PEAKS["hbm_gbs"], rel=1e-3)
    # the per-layer in-step times add up to the step (each rounded to 1 ns)
    assert sum(r["in_step_us_per_layer"]) == pytest.approx(out["ms_per_step"] * 1e3, abs=3e-3)
    assert out["gpu_launches"] == 3 * 200
    assert out["step_ms_quantiles"]["median"] == pytest.approx(0.05)
    assert "replays of 4 steps" in out["step_ms_quantiles"]["over"]
    # e2e: the same metric with the host copies in the timed region
    assert out["e2e"]["value"] == pytest.approx(tbps / 2, rel=1e-3)
    assert out["e2e_plain"]["value"] == pytest.approx(tbps / 3, rel=1e-3)
    assert out["e2e"]["h2d_bytes_per_step"] == 1000 and out["e2e"]["d2h_bytes_per_step"] == 2000


def test_tensor_bound_peak_depends_on_the_timed_region():
    wl = fake_workload("prefill_int4")
    tflops = wl.step_flops / 1.5e-3 / 1e12
    # 200 steps of 1.5 ms: 0.3 s of back-to-back GEMMs -> the sustained peak
    long = bench.summarize(wl, fake_result(1500.0, 1, 200), 200, 1, PEAKS, "measured")["roofline"]
    assert long["peak"] == PEAKS["bf16_tflops_sustained"] and "sustained" in long["peak_source"]
    assert long["frac"] == pytest.approx(tflops / PEAKS["bf16_tflops_sustained"], rel=1e-3)
    assert long["frac_of_burst"] == pytest.approx(tflops / PEAKS["bf16_tflops"], rel=1e-3)
    # 20 steps: 30 ms -> the burst peak
    short = bench.summarize(wl, fake_result(1500.0, 1, 20), 20, 1, PEAKS, "measured")["roofline"]
    assert short["peak"] == PEAKS["bf16_tflops"] and "burst" in short["peak_source"]


def test_ridge_workloads_report_both_fractions():
    wl = fake_workload("c32_mtp3_int4")
    r = bench.summarize(wl, fake_result(110.0, 2, 200), 200, 1, PEAKS, "measured")["roofline"]
    f = r["fractions"]
    assert f["hbm"] == pytest.approx(wl.step_bytes / 110e-6 / 1e9 / PEAKS["hbm_gbs"], rel=1e-3)
    assert f["tensor"] == pytest.approx(wl.step_flops / 110e-6 / 1e12 / PEAKS["bf16_tflops"],
                                        rel=1e-3)


def test_whole_job_value_scales_with_ranks():
    wl = fake_workload("mxfp8_m4")
    one = bench.summarize(wl, fake_result(22.0, 1, 200), 200, 1, PEAKS, "measured")
    two = bench.summarize(wl, fake_result(22.0, 1, 200), 200, 2, PEAKS, "measured")
    assert two["value"] == pytest.approx(2 * one["value"], rel=1e-6)
