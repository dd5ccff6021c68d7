"""The benchmark's JSON line carries every key of the reporting contract, with
the roofline and end-to-end objects filled from the measured inputs (host
only: a fake measurement through compose_line)."""
import types

import bench
import moe_inputs


def _line(world=1):
    cfg = moe_inputs.PREFILL
    res = {"peaks": bench.load_peaks(), "stage_ms": [0.02, 0.02, 1.40, 1.00, 0.10],
           "step_quantiles": {"p25": 2.5, "p50": 2.55, "p75": 2.6}, "n_active": 252,
           "clocks": {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]},
           "decode": None}
    args = types.SimpleNamespace(steps=100, warmup=5)
    return bench.compose_line(args, cfg, world, res, 2.6, 2.65), cfg


def test_required_keys_and_types():
    line, cfg = _line()
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in line, k
    assert line["n_gpus"] == 1 and line["steps"] == 100 and line["warmup"] == 5
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["vs_baseline"] is None and line["dtype"] == "bf16"
    assert line["config"]["workload"] == "prefill"
    # route + 3 map kernels + gate/up + W_down fp16 copy + down + combine
    assert line["gpu_launches"] == 800
    # value: routed-expert FLOPs of one step over the step time
    flops = 2.0 * cfg.m * cfg.top_k * 3 * cfg.hidden * cfg.inter
    assert abs(line["value"] - flops / 2.6e-3 / 1e12) < 1e-6 * line["value"]


def test_roofline_and_e2e_objects():
    line, cfg = _line()
    r = line["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in r, k
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    # achieved = the gate/up kernel's algorithmic bytes over its measured time
    assert abs(r["achieved"] - bench.gate_up_bytes(cfg, 252) / 1.40e-3 / 1e9) < 1e-6 * r["achieved"]
    e = line["e2e"]
    assert e["h2d_bytes_per_step"] == cfg.m * cfg.hidden * 2 + cfg.m * cfg.n_experts * 4
    assert e["d2h_bytes_per_step"] == cfg.m * cfg.hidden * 4
    assert e["unit"] == line["unit"]


def test_two_replicas_double_the_value():
    one, _ = _line(1)
    two, _ = _line(2)
    assert abs(two["value"] - 2 * one["value"]) < 1e-9 * two["value"]
    assert two["n_gpus"] == 2


def test_tensor_bound_layer_objects():
    """The skewed and long layers get their own lines: routed TFLOP/s against
    both bf16 peaks, the stage split, the gate/up tensor roofline, e2e."""
    cfg = moe_inputs.PREFILL
    peaks = bench.load_peaks()
    lay = {"stage_ms": [0.015, 0.02, 0.69, 0.54, 0.10], "n_active": 8, "ms": 1.37,
           "e2e_ms": 1.5, "step_quantiles": {"p25": 1.36, "p50": 1.37, "p75": 1.38}}
    res = {"peaks": peaks, "stage_ms": [0.02, 0.02, 1.40, 1.00, 0.10], "n_active": 252,
           "step_quantiles": None, "clocks": None, "decode": None,
           "layers": {"skewed": lay, "long": dict(lay, n_active=128)}}
    args = types.SimpleNamespace(steps=10, warmup=5)
    line = bench.compose_line(args, cfg, 1, res, 2.6, 2.65, {"skewed": (1.4, 1.6)})
    sk = line["skewed"]
    flops = 2.0 * cfg.m * cfg.top_k * 3 * cfg.hidden * cfg.inter
    assert abs(sk["TFLOP/s"] - flops / 1.4e-3 / 1e12) < 1e-6 * sk["TFLOP/s"]  # max-over-ranks time
    assert abs(sk["frac_of_bf16_burst"] - sk["TFLOP/s"] / peaks["bf16_tflops"]) < 1e-12
    r = sk["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    gu = 2.0 * cfg.m * cfg.top_k * cfg.hidden * 2 * cfg.inter
    assert abs(r["achieved"] - gu / 0.69e-3 / 1e12) < 1e-6 * r["achieved"]
    assert sk["e2e"]["unit"] == "TFLOP/s" and sk["stage_ms"]["down_scatter"] == 0.54
    lg = line["long"]
    lcfg = moe_inputs.LONG
    assert lg["e2e"]["h2d_bytes_per_step"] == (lcfg.m * lcfg.top_k * lcfg.hidden * 2
                                              + lcfg.m * lcfg.n_experts * 4)
    assert line["gpu_launches"] == 10 * 8 * 3  # 8 library kernels per step of each layer


def test_gate_up_bytes_count_the_activation_once():
    cfg = moe_inputs.PREFILL
    rows = cfg.m * cfg.top_k
    want = 252 * 2 * cfg.inter * cfg.hidden * 2 + cfg.m * cfg.hidden * 2 + rows * cfg.inter * 2
    assert bench.gate_up_bytes(cfg, 252) == want
