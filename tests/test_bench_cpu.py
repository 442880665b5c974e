"""The benchmark's output contract, checked on the CPU: the GPU leg's JSON line
carries every key the contract asks for (built from stand-in measurements),
and the reference arm (the oracle on the host) prints a complete line."""
import contextlib
import io
import json

import bench


class _T:
    def __init__(self, nwords):
        self.nwords = nwords


def _work():
    return [{"name": "qkv", "M": 27648, "K": 9216, "N": n, "t": _T(51_000_000), "bytes": 204_000_000,
             "flops": 2 * 27648 * 9216 * n, "key": (2, 0)} for n in (8, 16)]


def test_gpu_line_has_every_contract_key():
    args = bench.parse_args([])
    calls, name = bench.workload_calls(args, 0)
    line = bench.bench_line(
        world=1, args=args, cfg_name=name, work=_work(), calls=calls, value=2285.0, total_ms=72.0, tflops=169.0,
        achieved=2285.0, peak=6539.5, peak_src="measured", bytes_step=3_300_000_000,
        cpu={"value": 0.15, "unit": "GB/s", "cores": 16, "kind": "oracle", "sample": "rows"},
        e2e={"value": 2088.0, "unit": "GB/s", "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 2},
        kernels_per_step=16, dense=None, clocks={"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []},
        enc_bytes=10, enc_ms=1.0, enc_first_ms=2.0, detail=[])
    json.dumps(line)
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e",
              "gpu_launches", "clocks"):
        assert k in line, k
    assert line["config"]["workload"] == "opt66b_layer"
    assert set(line["roofline"]) >= {"bound", "achieved", "peak", "unit", "frac", "traffic"}
    assert line["roofline"]["bound"] == "hbm" and abs(line["roofline"]["frac"] - 2285.0 / 6539.5) < 1e-4
    assert set(line["e2e"]) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
    assert line["gpu_launches"] == 16 * args.steps
    assert line["higher_is_better"] is True and line["unit"] == "GB/s"


def test_reference_arm_prints_a_complete_line():
    args = bench.parse_args(["--impl", "reference", "--workload", "single_1024", "--steps", "1", "--warmup", "1"])
    calls, name = bench.workload_calls(args, 0)
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(args, calls, name, 0, 1)
    line = json.loads(out.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["config"]["workload"] == "single_1024"
    assert set(line["cpu_baseline"]) >= {"value", "unit", "cores", "kind", "sample"}
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
