"""Host-side logic of bench.py, on the CPU: the whole-job aggregation over
ranks (world size 2, gloo), the roofline bookkeeping and the clock parser.
The layer itself has no collective: ranks are independent replicas, and the
only cross-rank traffic is the control-plane max/sum done here."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from routing_dispatch_expert_sigmoid_b200.workloads import WORKLOADS  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist = bench.init_dist(world, "gloo")
    ms, units = bench.aggregate(10.0 + 5.0 * rank, 1000 * (rank + 1), dist)
    bench.barrier(dist)
    q.put((rank, ms, units))
    dist.destroy_process_group()


def test_aggregate_max_time_sum_units_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the slowest rank's time and the job's total units
    assert [r[1] for r in res] == [15.0, 15.0]
    assert [r[2] for r in res] == [3000, 3000]


def test_aggregate_single_process():
    assert bench.aggregate(7.5, 42, None) == (7.5, 42)


def test_launch_count_and_algorithmic_work():
    w = WORKLOADS["mixtral_prefill"]
    assert bench.launches_per_layer(w) == 9
    assert bench.launches_per_layer(WORKLOADS["dsv3_prefill"]) == 11
    # decode batches: split-K router + fused gating/ranking instead of 5 launches
    assert bench.launches_per_layer(WORKLOADS["mixtral_decode"]) == 6
    # decode-sized shared expert: gate, up, SwiGLU and down, split along K
    assert bench.launches_per_layer(WORKLOADS["dsv3_decode"]) == 10
    assert bench.launches_per_layer(WORKLOADS["tiny_f32"]) == 9
    a = bench.algorithmic(w, R=16384, touched=8)
    assert a["up_flops"] == 4 * 16384 * 4096 * 14336
    assert a["layer_flops"] == 2 * 8192 * 4096 * 8 + 6 * 4096 * 14336 * 16384
    assert a["layer_bytes"] == 8 * 3 * 4096 * 14336 * 2 + 4096 * 8 * 2 + 2 * 8192 * 4096 * 2


def test_traffic_only_for_the_profiled_kernel_source(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    import hashlib
    h = hashlib.sha256(b"kernel v1").hexdigest()
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "k5_up_swiglu_demo.md").write_text(
        f"dram_bytes_per_launch: 1.5e+09\nkernel_source_sha256: {h}\n")
    monkeypatch.setattr(bench, "PROFILES", str(prof))
    monkeypatch.setattr(bench, "GEMM_SRC", str(src))
    assert bench.traffic_from_profile("demo") == 1.5e9
    src.write_text("kernel v2")  # the kernel changed since the counters were taken
    assert bench.traffic_from_profile("demo") is None
    assert bench.traffic_from_profile("missing") is None


def test_clock_summary_parses_reasons():
    c = bench.ClockSampler(0)
    import tempfile
    c.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
    c.file.write("0, 1920, 1965, 900.1, 0x4, Not Active, Not Active, Not Active, Active, 1000.00\n"
                 "0, 1900, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active, 1000.00\n"
                 "0, 600, 1965, 100.0, 0x0, Not Active, Not Active, Not Active, Not Active, 1000.00\n")
    c.file.flush()
    s = c.summary()
    assert s["sm_mhz"] == pytest.approx(1910.0) and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
    assert s["power_limit_w"] == 1000.0 and s["power_max_w"] == 950.0


def test_algorithmic_bytes_with_fp8_weights():
    w = WORKLOADS["mixtral_decode"]
    b = bench.algorithmic(w, R=128, touched=8)
    q = bench.algorithmic(w, R=128, touched=8, fp8=True)
    d, f = w.d, w.f
    assert q["up_bytes"] == 8 * 2 * (d * f + 4 * f) + 128 * d * 2 + 128 * f * 2
    assert q["up_flops"] == b["up_flops"]
    # one byte per expert weight plus the column scales; router, x and out unchanged
    assert b["layer_bytes"] - q["layer_bytes"] == 8 * (3 * d * f - 4 * (2 * f + d))


def test_layer_roofline_takes_the_slower_bound():
    alg = {"layer_flops": 2.25e12, "layer_bytes": 8e9}   # 1 ms at either nominal peak
    assert abs(bench.layer_roofline_ms(alg, bench.NOMINAL_PEAKS) - 1.0) < 1e-12
    alg = {"layer_flops": 4.5e12, "layer_bytes": 8e9}    # flops bound: 2 ms
    assert abs(bench.layer_roofline_ms(alg, bench.NOMINAL_PEAKS) - 2.0) < 1e-12
    alg = {"layer_flops": 2.25e12, "layer_bytes": 24e9}  # bytes bound: 3 ms
    assert abs(bench.layer_roofline_ms(alg, bench.NOMINAL_PEAKS) - 3.0) < 1e-12


PEAKS = {"hbm_gbs": 6548.8, "bf16_tflops": 1661.1, "bf16_tflops_sustained": 1383.9}
# stage means of a Mixtral-shaped prefill run (T=8192, 16384 kept rows) on B200
STAGES_MS = {"route": 0.0736, "dispatch": 0.0412, "up_swiglu": 2.7638, "down": 1.385,
             "shared": 0.0028, "combine": 0.0854}


def test_kernel_roofline_uses_the_burst_peak_whatever_the_clock_reasons():
    """The compute peak is the measured burst figure, the one the layer
    fraction uses too; a power-cap sample does not switch it.  Up projection:
    4.R.d.f = 3.848 TFLOP in 2.7638 ms = 1392 TFLOP/s = 0.838 of 1661.1."""
    w = WORKLOADS["mixtral_prefill"]
    alg = bench.algorithmic(w, R=16384, touched=8)
    for reasons in ([], ["sw_power_cap"]):
        clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": reasons}
        k = bench.stage_rooflines(w, alg, STAGES_MS, PEAKS, "measured", clocks, "x", 74.5,
                                  profiled=False)
        up = k["up_swiglu"]
        assert up["bound"] == "tensor" and up["peak"] == 1661.1
        assert up["frac"] == pytest.approx(0.8382, abs=1e-4)
        assert up["frac"] == pytest.approx(up["work_per_launch"] / (up["ms_per_launch"] * 1e-3)
                                           / 1e12 / up["peak"], abs=1e-4)
        # no compute-bound kernel of this run reads above its own peak
        assert all(o["frac"] <= 1.0 for o in k.values() if o["bound"] != "hbm")


def test_frac_at_sampled_clock_scales_the_compute_peak_only():
    clocks = {"sm_mhz": 1320.0, "sm_max_mhz": 1965.0, "samples": 20}
    t = bench.kernel_roofline(0.6 * 1661.1e9, 1e6, 1.0, PEAKS, "measured", clocks=clocks)
    assert t["bound"] == "tensor" and t["frac"] == pytest.approx(0.6)
    assert t["frac_at_sampled_clock"] == pytest.approx(0.6 * 1965.0 / 1320.0, abs=1e-4)
    h = bench.kernel_roofline(0, 6548.8e6, 1.0, PEAKS, "measured", clocks=clocks)
    assert h["bound"] == "hbm" and h["frac"] == pytest.approx(1.0)
    assert "frac_at_sampled_clock" not in h  # HBM bandwidth does not follow the SM clock


def test_frac_at_sampled_clock_needs_enough_samples_and_stays_below_one():
    few = {"sm_mhz": 1320.0, "sm_max_mhz": 1965.0, "samples": 4}
    t = bench.kernel_roofline(0.6 * 1661.1e9, 1e6, 1.0, PEAKS, "measured", clocks=few)
    assert t["frac_at_sampled_clock"] is None and "too few" in t["sampled_clock_note"]
    many = dict(few, samples=20)
    t = bench.kernel_roofline(0.9 * 1661.1e9, 1e6, 1.0, PEAKS, "measured", clocks=many)
    assert t["frac"] == pytest.approx(0.9)
    assert t["frac_at_sampled_clock"] is None  # 0.9 x 1965 / 1320 > 1: a missed clock
    assert "not reported" in t["sampled_clock_note"]


def test_combine_reports_both_byte_counts(monkeypatch):
    w = WORKLOADS["mixtral_prefill"]
    alg = bench.algorithmic(w, R=16384, touched=8)
    assert alg["combine_bytes"] == (16384 + 8192) * 4096 * 2
    # y16 rows: fp16 values plus one exponent byte per 32 columns
    assert alg["combine_bytes_actual"] == (16384 * (4096 * 2 + 128) + 8192 * 4096 * 2
                                           + 8192 * 2 * 8)
    monkeypatch.setenv("MOE_Y16", "0")  # fp32 rows
    a32 = bench.algorithmic(w, R=16384, touched=8)
    assert a32["combine_bytes_actual"] == 16384 * 4096 * 4 + 8192 * 4096 * 2 + 8192 * 2 * 8
    assert a32["down_bytes"] - alg["down_bytes"] == 16384 * (4096 * 2 - 128)
    monkeypatch.delenv("MOE_Y16")
    k = bench.stage_rooflines(w, alg, STAGES_MS, PEAKS, "measured", {}, "x", 74.5,
                              profiled=False)
    c = k["combine"]
    assert c["frac"] == pytest.approx(alg["combine_bytes"] / 0.0854e-3 / 1e9 / 6548.8, abs=1e-4)
    assert c["frac_on_actual_bytes"] > c["frac"]


def test_tiny_fp32_ffn_is_alu_bound():
    w = WORKLOADS["tiny_f32"]
    alg = bench.algorithmic(w, R=369, touched=8)
    st = dict(STAGES_MS, up_swiglu=0.058)
    alu = bench.alu_peak_tflops(148, 1965.0)
    assert alu == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)
    k = bench.stage_rooflines(w, alg, st, PEAKS, "measured", {}, "x", alu, profiled=False)
    assert k["up_swiglu"]["bound"] == "alu" and "down" not in k
