"""The JSON line of bench.py's own arm, assembled from synthetic measurements on the CPU: every mode
(both halves, --only prefill, --only decode) gives strict JSON with the contract's keys, and the
derived rates follow from the inputs."""
import json
import math

import pytest

import bench
import gqa_inputs as gi

PEAKS = {"bf16_tflops": 1637.6, "bf16_tflops_sustained": 1390.6, "hbm_gbs": 6449.7}
NAN = float("nan")
CONTRACT = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
            "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks",
            "impl")


def line_for(only, world=1, page=None, qkv=None, configs=None, dec_alone=(NAN, NAN), dec_rot=(NAN, NAN)):
    do_p, do_d = only in (None, "prefill"), only in (None, "decode")
    wp, wd = gi.BY_NAME[bench.PREFILL_WORKLOAD], gi.BY_NAME[bench.DECODE_WORKLOAD]
    fl = bench.prefill_flops(wp)
    pre_ms, attn_ms = 0.135, 0.118
    line = bench.build_line(
        world=world, K=30, W=5, only=only, do_p=do_p, do_d=do_d, wp=wp, wd=wd,
        value_tflops=world * fl / (pre_ms * 1e-3) / 1e12 if do_p else None,
        pre_mean=pre_ms if do_p else None, attn_mean=attn_ms if do_p else NAN,
        dec_mean=0.356 if do_d else 0.003, split_mean=0.345 if do_d else NAN, total_rows=954557, page=page,
        peaks=PEAKS, peak_src="measured",
        cpu_base={"value": 0.03, "unit": "TFLOP/s", "cores": 16, "kind": "oracle", "sample": "s"} if do_p else None,
        e2e_pre=1.3 if do_p else NAN, e2e_dec=0.4 if do_d else NAN, pre_io=(37748736, 29360128),
        dec_io=(459008, 458752), qkv_line=qkv, clocks={"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []},
        t_wall=0.05, configs=configs, dec_alone=dec_alone, dec_rot=dec_rot)
    text = json.dumps(bench.clean(line), allow_nan=False)   # strict JSON: no NaN or inf survives
    return json.loads(text)


def test_both_halves():
    d = line_for(None)
    for key in CONTRACT:
        assert key in d, key
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert math.isclose(r["achieved"], bench.prefill_flops(gi.BY_NAME[bench.PREFILL_WORKLOAD]) / 0.118e-3 / 1e12)
    assert math.isclose(r["frac"], r["achieved"] / PEAKS["bf16_tflops"])
    dr = d["decode"]["roofline"]
    assert dr["bound"] == "hbm" and math.isclose(dr["frac"], dr["achieved"] / PEAKS["hbm_gbs"])
    assert d["gpu_launches"] == (2 + 3) * 2 * 30 + (2 + 3) * 30   # headline + kernel-timing steps, e2e steps
    assert d["e2e"]["h2d_bytes_per_step"] == 37748736 and d["decode"]["e2e"]["d2h_bytes_per_step"] == 458752
    assert d["impl"] == "ours" and d["scaling"] == "weak"


def test_only_prefill_drops_the_decode_half():
    d = line_for("prefill")
    assert d["decode"] is None
    assert d["value"] > 0 and d["roofline"]["frac"] > 0
    assert d["gpu_launches"] == 2 * 2 * 30 + (2 + 3) * 30


def test_only_decode_carries_no_prefill_figures():
    d = line_for("decode")
    assert d["value"] is None and d["ms_per_step"] is None
    assert d["roofline"] is None and d["e2e"] is None and d["cpu_baseline"] is None
    assert d["decode"]["value"] > 0 and d["decode"]["roofline"]["frac"] > 0
    assert d["gpu_launches"] == 3 * 2 * 30


@pytest.mark.parametrize("world", [2, 8])
def test_whole_job_rates_scale_with_ranks(world):
    one, many = line_for(None), line_for(None, world=world)
    assert math.isclose(many["decode"]["value"], world * one["decode"]["value"])
    assert math.isclose(many["e2e"]["value"], world * one["e2e"]["value"])
    assert many["n_gpus"] == world


def test_paged_layout_is_named():
    d = line_for("decode", page=16)
    assert d["decode"]["layout"].startswith("paged: 16 rows per page")


def test_headline_is_the_largest_prefill_workload():
    prefill = [w for w in gi.WORKLOADS if w.kind == "prefill"]
    assert bench.PREFILL_WORKLOAD == max(prefill, key=bench.prefill_flops).name
    assert set(bench.CONFIG_WORKLOADS) | {bench.PREFILL_WORKLOAD} == {w.name for w in prefill}


def test_configs_carry_step_kernel_roofline_and_cpu_baseline():
    cb = {"value": 0.03, "unit": "TFLOP/s", "cores": 16, "kind": "oracle", "sample": "s"}
    times = {"qwen2-0.5b-prefill-L128": (0.02, 0.012), "qwen2-7b-prefill-L4096": (0.13, 0.115),
             "qwen2-72b-prefill-B4-L8192": (4.0, 3.8)}
    configs = {n: bench.config_entry(gi.BY_NAME[n], world=1, step_ms=a, attn_ms=b, peaks=PEAKS,
                                     peak_src="measured", cpu_base=cb) for n, (a, b) in times.items()}
    d = line_for(None, configs=configs)
    assert set(d["configs"]) == set(times) | {bench.PREFILL_WORKLOAD}
    for n, (a, b) in times.items():
        c = d["configs"][n]
        fl = bench.prefill_flops(gi.BY_NAME[n])
        assert c["ms_per_step"] == a and c["kernel_ms_per_launch"] == b
        assert math.isclose(c["roofline"]["frac"], fl / (b * 1e-3) / 1e12 / PEAKS["bf16_tflops"])
        assert math.isclose(c["step_frac"], fl / (a * 1e-3) / 1e12 / PEAKS["bf16_tflops"])
        assert c["cpu_baseline"]["kind"] == "oracle"
    head = d["configs"][bench.PREFILL_WORKLOAD]
    assert math.isclose(head["roofline"]["frac"], d["roofline"]["frac"])
    # two launches (rotation pass + attention) per step, two kinds of step, K steps, three more workloads
    assert d["gpu_launches"] == (2 + 3) * 2 * 30 + 3 * 2 * 2 * 30 + (2 + 3) * 30


def test_decode_alone_beside_the_in_step_decode():
    d = line_for(None, dec_alone=(0.345, 0.336))
    a = d["decode"]["alone"]
    allb = bench.decode_bytes(954557, gi.BY_NAME[bench.DECODE_WORKLOAD])
    assert math.isclose(a["split_frac"], allb / 0.336e-3 / 1e9 / PEAKS["hbm_gbs"])
    assert math.isclose(a["value"], allb / 0.345e-3 / 1e9)
    assert d["gpu_launches"] == (2 + 3) * 2 * 30 + 3 * 2 * 30 + (2 + 3) * 30
    assert line_for(None)["decode"]["alone"]["value"] is None   # not run: null, still strict JSON


def test_peak_is_sustained_only_for_long_power_capped_runs():
    capped = {"sm_mhz": 1605, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}
    assert bench.tensor_peak(PEAKS, capped, 0.4) == (PEAKS["bf16_tflops_sustained"], "sustained")
    assert bench.tensor_peak(PEAKS, capped, 0.01) == (PEAKS["bf16_tflops"], "burst")        # too short
    assert bench.tensor_peak(PEAKS, {"reasons": []}, 0.4) == (PEAKS["bf16_tflops"], "burst")  # no cap
    assert bench.tensor_peak(PEAKS, {"error": "nvml unavailable"}, 0.4) == (PEAKS["bf16_tflops"], "burst")
    w = gi.BY_NAME["qwen2-72b-prefill-B4-L8192"]
    c = bench.config_entry(w, world=1, step_ms=4.0, attn_ms=3.75, peaks=PEAKS, peak_src="measured", cpu_base=None,
                           clocks=capped, wall_s=0.25)
    ach = bench.prefill_flops(w) / 3.75e-3 / 1e12
    r = c["roofline"]
    assert r["peak"] == PEAKS["bf16_tflops_sustained"] and math.isclose(r["frac"], ach / r["peak"])
    assert math.isclose(r["frac_of_burst"], ach / PEAKS["bf16_tflops"])
    assert "sustained" in r["peak_source"]


def test_rotated_cache_decode_beside_the_in_step_decode():
    d = line_for(None, dec_rot=(0.33, 0.315))
    r = d["decode"]["rotated_cache"]
    allb = bench.decode_bytes(954557, gi.BY_NAME[bench.DECODE_WORKLOAD])
    assert abs(r["split_frac"] - allb / (0.315e-3) / 1e9 / PEAKS["hbm_gbs"]) < 1e-9
    assert abs(r["value"] - allb / (0.33e-3) / 1e9) < 1e-6
    # its K steps of prefill + decode count among the line's launches
    assert d["gpu_launches"] == line_for(None)["gpu_launches"] + (2 + 3) * 30
    assert line_for(None)["decode"]["rotated_cache"]["value"] is None
