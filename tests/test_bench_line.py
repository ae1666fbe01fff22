"""The benchmark's JSON line on CPU: bench.assemble_line builds it from the
timings the GPU legs return; this checks the keys and derived numbers the
measurement contract asks for, with stage timings shaped like a real run."""
import argparse
import json

import bench


def _tr(world=1):
    fwd_flops, step_flops = bench.train_flops(bench.I.spec(bench.TRAIN_CFG))
    ms = 1.42
    return dict(
        ms=ms, value=bench.weak_scaling_value(step_flops, ms, world) / 1e12,
        fwd_ms=0.40, bwd_ms=1.02, fwd_tflops=680.0, bwd_tflops=675.0,
        launches=11 * 100, clocks={"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []},
        spec=bench.I.spec(bench.TRAIN_CFG), step_flops=step_flops, fwd_flops=fwd_flops,
        # api.timing_read: name -> (launches, total ms)
        stages={"prefix_scan": (20, 0.52), "operands": (20, 0.79), "fwd_tc": (20, 6.5),
                "bwd_pre": (20, 0.31), "bwd_keyblock": (100, 65.4), "bwd_dq": (20, 4.6),
                "bwd_finalize": (40, 1.8), "reverse_scan": (20, 0.63), "decode": (0, 0.0)},
        e2e={"value": 384.0, "unit": "TFLOP/s", "h2d_bytes_per_step": 117440512,
             "d2h_bytes_per_step": 83886080})


def test_line_has_the_contract_keys():
    args = argparse.Namespace(steps=100, warmup=3)
    peaks = dict(hbm_gbs=6549.4, bf16_tflops=1657.1, bf16_tflops_sustained=1394.4,
                 sm_max_mhz=1965.0, source="measured")
    dec = {"decode_gbs": 5200.0, "tokens_per_s": 15100.0}
    line = bench.assemble_line(args, 1, _tr(), dec, peaks)
    json.dumps(line)  # serialisable
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "gpu_launches", "clocks", "e2e", "decode"):
        assert key in line, key
    assert line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s"
    assert line["scaling"] == "weak" and line["vs_baseline"] is None
    assert line["higher_is_better"] is True and line["dtype"] == "bf16"
    assert line["config"]["workload"] and "l2" in line["config"]
    # value: the step's causal FLOPs over its time
    _, step_flops = bench.train_flops(bench.I.spec(bench.TRAIN_CFG))
    assert abs(line["value"] - step_flops / 1.42e-3 / 1e12) < 1e-9
    roof = line["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in roof, key
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    # the timed region ran at the maximum clock: the burst peak applies
    assert roof["peak"] == peaks["bf16_tflops"]
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-12
    assert abs(line["frac_bf16_peak"] - line["value"] / peaks["bf16_tflops"]) < 1e-12
    assert abs(roof["frac_of_sustained"] - roof["achieved"] / 1394.4) < 1e-12
    assert abs(line["frac_bf16_nominal"] - line["value"] / 2250.0) < 1e-12
    # the key block does 2 x the forward's FLOPs per launch
    fwd_flops = _tr()["fwd_flops"]
    assert abs(roof["achieved"] - 2 * fwd_flops / (0.654e-3) / 1e12) < 1e-6
    assert roof["traffic"] == bench.BWD_KEY_TRAFFIC_BYTES
    # stages without launches are left out; the others carry per-launch times
    assert "decode" not in line["stages"]
    assert abs(line["stages"]["bwd_finalize"]["ms_per_launch"] - 0.045) < 1e-12
    for key in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert key in line["e2e"], key


def test_weak_scaling_counts_every_rank():
    line1 = bench.assemble_line(argparse.Namespace(steps=10, warmup=3), 1, _tr(1), None,
                                dict(hbm_gbs=1.0, bf16_tflops=1.0, bf16_tflops_sustained=1.0,
                                     source="fallback"))
    line4 = bench.assemble_line(argparse.Namespace(steps=10, warmup=3), 4, _tr(4), None,
                                dict(hbm_gbs=1.0, bf16_tflops=1.0, bf16_tflops_sustained=1.0,
                                     source="fallback"))
    assert abs(line4["value"] - 4 * line1["value"]) < 1e-6
    assert line4["config"]["parallelism"] == "replicas x4"
    assert "decode" not in line1


def test_config_flops_count_visible_pairs():
    s3 = bench.I.spec(3)
    assert bench.config_fwd_flops(s3, [s3.T]) == bench.train_flops(s3)[0]
    # config 4: windowed pairs of every packed sequence
    s4 = bench.I.spec(4)
    lengths = bench.I.varlen_lengths(s4)
    W = s4.window
    pairs = sum(min(n, W) * (min(n, W) + 1) // 2 + max(0, n - W) * W for n in lengths)
    assert bench.config_fwd_flops(s4, lengths) == 2.0 * pairs * s4.HQ * (s4.K + s4.V)


def test_line_carries_the_other_configs():
    cfgs = {"config2": {"tflops": 400.0, "ms_per_step": 0.02},
            "config4": {"error": "RuntimeError: x"}}
    line = bench.assemble_line(argparse.Namespace(steps=10, warmup=3), 1, _tr(), None,
                               dict(hbm_gbs=1.0, bf16_tflops=1.0, bf16_tflops_sustained=1.0,
                                    source="fallback"), cfgs)
    assert line["configs"] == cfgs
    assert "configs" not in bench.assemble_line(
        argparse.Namespace(steps=10, warmup=3), 1, _tr(), None,
        dict(hbm_gbs=1.0, bf16_tflops=1.0, bf16_tflops_sustained=1.0, source="fallback"))


def test_decode_bytes_of_the_decode_workload():
    """HBM bytes of one decode step at B=32, T_kv=32768, HQ=32, H=8,
    K=V=128, C=64: k_tilde 8.590 GB + v 2.147 GB + r_cache 0.268 GB plus the
    per-row q, p_curr, o and lse."""
    s = bench.I.spec(5)
    kt = 32 * 32768 * 32 * 128 * 2
    v = 32 * 32768 * 8 * 128 * 2
    rc = 32 * (32768 // 64) * 32 * 128 * 4
    small = 32 * 32 * (128 * 2 + 128 * 4 + 128 * 2 + 4)
    assert (kt, v, rc) == (8589934592, 2147483648, 268435456)
    assert bench.decode_bytes(s, 32768) == kt + v + rc + small


def test_sustained_peak_below_the_maximum_clock():
    """A timed region whose median SM clock sat below the maximum (the power
    cap holding it down) takes the sustained peak."""
    args = argparse.Namespace(steps=100, warmup=3)
    peaks = dict(hbm_gbs=6549.4, bf16_tflops=1657.1, bf16_tflops_sustained=1394.4,
                 sm_max_mhz=1965.0, source="measured")
    tr = _tr()
    tr["clocks"] = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    line = bench.assemble_line(args, 1, tr, None, peaks)
    assert line["roofline"]["peak"] == peaks["bf16_tflops_sustained"]
    assert line["frac_bf16_peak_of"] == "bf16_tflops_sustained"


def test_e2e_names_the_bounding_stream():
    r = bench.e2e_record(1, 9.6e11, 4.79, 117440512, 83886080,
                         {"h2d": 4.5, "compute": 1.4, "d2h": 3.2})
    assert r["limit"] == "h2d" and abs(r["h2d_gbs"] - 117440512 / 4.5e-3 / 1e9) < 1e-9
    assert abs(r["value"] - 9.6e11 / 4.79e-3 / 1e12) < 1e-9
