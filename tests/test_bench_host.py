"""Host logic of bench.py, without a GPU: the cross-rank timing reduction
over a real 2-process gloo group, and the shape of the JSON line."""
import io
import json
import os
import socket
import sys
import types
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 5.0], "cpu")
        out[rank] = res
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == [2.0, 10.0, 5.0]


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks([3.0, 4.5], "cpu") == [3.0, 4.5]


@pytest.mark.parametrize("world", [1, 2])
def test_report_line_has_the_contract_keys(world):
    args = types.SimpleNamespace(steps=5, warmup=3, no_cpu_baseline=True, cpu_seconds=1.0)
    kern = {"mx_quantize": 0.45, "gemm_fwd": 0.8, "gemm_dgrad": 1.0, "qc_fp8": 0.02,
            "qc_mxfp4": 0.02, "qc_nvfp4": 0.02, "mx_dequantize": 0.44}
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.report(args, world, total_ms=15.0, kern_ms=kern, e2e_dt=0.2, h2d=10, d2h=20,
                     clocks={"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": []})
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "e2e", "gpu_launches", "clocks", "gemm"):
        assert key in line, key
    assert line["n_gpus"] == world and line["scaling"] == "weak"
    assert line["roofline"]["bound"] in ("hbm", "tensor")
    # whole-job throughput: every rank moves the same bytes
    qd_bytes = sum(bench.algorithmic_bytes()[k] for k in ("mx_quantize", "mx_dequantize")) + \
        3 * bench.algorithmic_bytes()["quantize_cache"]
    per_gpu = qd_bytes / ((0.45 + 0.44 + 0.06) * 1e-3) / 1e9
    assert abs(line["value"] - world * per_gpu) / (world * per_gpu) < 1e-3


def _smi_line(ts, sm, watts, mask):
    import datetime

    stamp = datetime.datetime.fromtimestamp(ts).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return "%s, %s, 1965, %s, 0x%016x" % (stamp, sm, watts, mask)


def test_clock_summary_takes_only_the_timed_region():
    # idle samples at the boost clock before and after the region, power-capped
    # ones inside it: the summary must describe the region alone
    t0 = 1_800_000_000.0
    clk = bench.ClockSampler(0)
    clk.lines = ([_smi_line(t0 - 0.2 + 0.02 * i, 1965, 300.0, 0x1) for i in range(10)] +
                 [_smi_line(t0 + 0.01 + 0.02 * i, 1500 + i, 990.0, 0x4) for i in range(5)] +
                 [_smi_line(t0 + 0.2 + 0.02 * i, 1965, "[N/A]", 0x0) for i in range(10)] +
                 ["garbage", ""])
    s = clk.summary(t0, t0 + 0.1)
    assert s["samples"] == 5 and s["window"] == "timed region"
    assert s["sm_mhz"] == 1502 and s["sm_min_mhz"] == 1500 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["power_w_median"] == 990.0
    # no sample inside the region: every sample, and the summary says so
    s = clk.summary(t0 + 5.0, t0 + 5.001)
    assert s["samples"] == 25 and s["window"].startswith("whole sampler run")
    assert s["sm_mhz"] == 1965 and s["power_w_median"] == 300.0
    assert bench.ClockSampler(0).summary(t0, t0 + 1)["reasons"] == ["unavailable"]


def test_reference_arm_line():
    # the oracle arm: W untimed and K timed steps on rank 0, nothing elsewhere
    args = types.SimpleNamespace(steps=2, warmup=3)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args, 1, 2)
    assert buf.getvalue() == ""
    with redirect_stdout(buf):
        bench.run_reference(args, 0, 1)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["steps"] == 2 and line["warmup"] == 3 and line["ms_per_step"] > 0
    assert line["value"] > 0 and line["unit"] == "GB/s" and line["higher_is_better"] is True
    cb = line["cpu_baseline"]
    assert cb["value"] == line["value"] and cb["kind"] == "oracle" and cb["cores"] == 1
    assert cb["sample"] and line["config"]["workload"] == bench.WORKLOAD
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
