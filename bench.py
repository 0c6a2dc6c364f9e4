#!/usr/bin/env python
"""MoE-layer tokens/s on B200: prefill and decode regimes of the Mixtral-8x7B
shaped layer (d=4096, E=8, top-2, f=14336, bf16, Zipf(0.5) router bias).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one moe_layer call over one batch (router, gating, capacity,
dispatch, grouped SwiGLU expert FFN, combine), inputs resident in HBM.  Time
is taken on the device with CUDA events around K back-to-back steps, between
a barrier and a synchronize on both sides; with N GPUs (torchrun, one process
per GPU) every rank runs its own replica of the layer on its own batch and
the time is the max over ranks (weak scaling, no collective on the data path).

Extra keys of the JSON line:
  layer_roofline_frac          max(F / bf16 peak, B / HBM peak) of the whole layer
                               over its measured time, against the measured
                               peaks (MEASURED_PEAKS.json, burst figures);
  layer_roofline_frac_nominal  the same against nominal B200 peaks (8 TB/s,
                               2.25 PFLOP/s dense bf16);
  roofline     the up-projection + SwiGLU grouped GEMM (the dominant kernel):
               algorithmic FLOPs or bytes per launch (work_per_launch) over its
               mean launch time (ms_per_launch), from CUDA events recorded on the
               launching stream at its boundaries inside the timed steps; bound
               by whichever of its FLOPs at the measured burst bf16 peak or its
               bytes at the measured copy bandwidth takes longer (the same peaks
               as layer_roofline_frac).  Compute-bound kernels also carry
               frac_at_sampled_clock: achieved over the peak scaled by the
               median sampled SM clock over the maximum clock (null, with
               sampled_clock_note, under 8 samples or when it would exceed 1:
               the snapshots then missed the clock the kernel ran at);
  kernels      the same for the dispatch (K4), up projection (K5), down
               projection (K6) and combine (K7) stages;
  e2e          the same metric through the C ABI with host buffers: per step a
               pinned-host -> device copy of x and a device -> pinned-host copy
               of the layer output are inside the timed region, double-buffered
               on two copy streams so that they overlap the neighbouring steps'
               layers (serial_value: the same with copies and layer in one
               stream, one after the other);
  cpu_baseline the CPU oracle as it stands, on a bounded sample of the same
               workload, on the host cores (rank 0, N=1 only);
  clocks       nvidia-smi samples taken during the timed region;
  decode       the same layer at decode size (T=64), same keys;
  fp8_weights  the decode-size layer with e4m3 expert weights and per-column
               scales (quantised before timing), same keys;
  configs      every other workload of the layer definition (tiny fp32,
               Qwen3-, DeepSeek-V3- (decode and prefill) and GPT-OSS-shaped
               layers, and the DeepSeek-V3-shaped decode layer with e4m3 expert
               weights), same keys, each timed on its own inputs after the
               previous one's memory was freed.
`--impl reference` times the CPU oracle alone on the same workload (the
reference arm: there is no other implementation of this layer to run).
"""
from __future__ import annotations

import argparse
import csv
import gc
import hashlib
import io
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from routing_dispatch_expert_sigmoid_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Nominal B200 figures, the second denominator of the layer roofline: 8 TB/s
# HBM3e and 2.25 PFLOP/s dense bf16.
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def layer_roofline_ms(alg: dict, peaks: dict) -> float:
    """max(F / bf16 peak, B / HBM peak) of the whole layer, in ms."""
    return max(alg["layer_flops"] / (peaks["bf16_tflops"] * 1e12),
               alg["layer_bytes"] / (peaks["hbm_gbs"] * 1e9)) * 1e3
PROFILES = os.path.join(ROOT, "profiles")
GEMM_SRC = os.path.join(ROOT, "routing_dispatch_expert_sigmoid_b200", "csrc",
                        "grouped_gemm_sm100.cu")
PERMUTE_SRC = os.path.join(ROOT, "routing_dispatch_expert_sigmoid_b200", "csrc", "permute.cu")
F8_SRC = os.path.join(ROOT, "routing_dispatch_expert_sigmoid_b200", "csrc", "grouped_gemm_f8.cu")


def w_is_decode(workload: str) -> bool:
    """Decode-sized legs with fp8 weights run on the kind::f8f6f4 engine."""
    return "decode" in workload
METRIC = "MoE-layer tokens/sec on 1 B200 (decode & prefill); % of roofline"
PREFILL, DECODE = "mixtral_prefill", "mixtral_decode"
L2_BYTES = 126 * 2 ** 20


# ---------------------------------------------------------------------------
# process group / ranks
# ---------------------------------------------------------------------------
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init_dist(world: int, backend: str):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_max(value: float, dist) -> float:
    """Max over ranks (control plane only)."""
    if dist is None:
        return value
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(local_ms: float, local_units: int, dist) -> tuple[float, int]:
    """(max elapsed ms over ranks, total units over ranks) -- whole-job numbers."""
    ms = reduce_max(local_ms, dist)
    if dist is None:
        return ms, local_units
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([local_units], dtype=torch.int64, device=dev)
    dist.all_reduce(t)
    return ms, int(t.item())


def barrier(dist):
    if dist is not None:
        dist.barrier()


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
                "enforced.power.limit")


MIN_CLOCK_SAMPLES = 8  # before a clock-scaled fraction is reported


class ClockSampler:
    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={CLOCK_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.file,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self) -> dict:
        if self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.file.flush()
        with open(self.file.name) as fh:
            rows = [r for r in csv.reader(io.StringIO(fh.read())) if len(r) >= 9]
        os.unlink(self.file.name)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, pw, lim, reasons = [], [], [], [], set()
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                pw.append(float(r[3]))
            except ValueError:
                continue
            try:  # the enforced power limit, read (never set) alongside the clocks
                lim.append(float(r[9]))
            except (IndexError, ValueError):
                pass
            for name, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": sorted(reasons), "samples": 0}
        hot = [s for s, p in zip(sm, pw) if p > 0.3 * max(pw)] or sm
        out = {"sm_mhz": statistics.median(hot), "sm_max_mhz": max(mx),
               "reasons": sorted(reasons), "samples": len(sm), "power_max_w": max(pw)}
        if lim:
            out["power_limit_w"] = statistics.median(lim)
        return out


# ---------------------------------------------------------------------------
# the layer on the GPU
# ---------------------------------------------------------------------------
def peaks() -> tuple[dict, str]:
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as fh:
            return json.load(fh), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def small_batch_routing(w) -> bool:
    """Decode-sized bf16 batches (E % 8 == 0, T <= 128) route with two launches:
    the split-K router and one fused gating/ranking kernel."""
    return (w.dtype == "bf16" and w.E % 8 == 0 and 1 <= w.T <= 128
            and not os.environ.get("MOE_SMALL_ROUTE", "1").startswith("0"))


def shared_split_k(w) -> bool:
    """Whether the layer splits its shared expert along K (a decode-sized
    batch: at most two 128-row tiles, 256-column output tiles, splits that
    divide the 64-deep K blocks, at most one wave of 148 CTAs)."""
    if w.f_shared <= 0 or w.dtype != "bf16":
        return False
    row_tiles = (w.T + 127) // 128
    if row_tiles > 2 or w.d % 64 or w.f_shared % 64:
        return False
    kb, tiles = w.d // 64, row_tiles * ((w.f_shared + 255) // 256)
    s_up = max(s for s in range(1, min(16, kb) + 1) if kb % s == 0 and s * tiles <= 148)
    return s_up >= 2


def launches_per_layer(w) -> int:
    """Kernel launches of one moe_layer call (see the C ABI's launch order)."""
    # router, gating, hist+scan+rank -- or the two small-batch launches
    routing = 2 if small_batch_routing(w) else 1 + 1 + 3
    n = routing + 1 + 2 + 1  # + dispatch, 2 FFN passes, combine
    if w.f_shared > 0:  # two FFN passes, or gate, up, SwiGLU and down split along K
        n += 4 if shared_split_k(w) else 2
    return n


def algorithmic(w, R: int, touched: int, fp8: bool = False) -> dict:
    """Algorithmic work of the layer and of its stages.  With fp8 expert
    weights each weight is one byte plus its column's fp32 scale; the router
    stays in the layer dtype.  Stage bytes count each tensor a stage must read
    or write once: K4 reads and writes the R dispatched rows, K5 reads the
    touched experts' W1 and W3 and the R rows and writes h, K6 reads W2 and h
    and writes the fp32 expert outputs, K7 -- in the measurement's definition
    -- reads R expert rows and writes T output rows in the layer dtype."""
    s = w.elem_bytes
    ws = 1 if fp8 else s                              # bytes per expert weight
    sc = 4 if fp8 else 0                              # bytes per column scale
    hs = s                                            # h: bf16 (or fp32 for fp32 layers)
    # expert output rows between the down projection and the combine: fp32,
    # or (bf16 layers, bf16 weights) the compact y16 form -- fp16 values and
    # one exponent byte per 32-column block
    ys = w.d * 2 + (w.d + 31) // 32 if y16_rows(w, fp8) else w.d * 4
    return {
        "layer_flops": 2 * w.T * w.d * w.E + 6 * w.d * w.f * R + 6 * w.d * w.f_shared * w.T,
        "layer_bytes": (touched * (3 * w.d * w.f * ws + (2 * w.f + w.d) * sc)
                        + 3 * w.d * w.f_shared * ws + (2 * w.f_shared + w.d) * sc * (w.f_shared > 0)
                        + w.d * w.E * s + 2 * w.T * w.d * s),
        "up_flops": 4 * R * w.d * w.f,
        "up_bytes": touched * 2 * (w.d * w.f * ws + w.f * sc) + R * w.d * s + R * w.f * hs,
        "down_flops": 2 * R * w.f * w.d,
        "down_bytes": touched * (w.f * w.d * ws + w.d * sc) + R * w.f * hs + R * ys,
        "dispatch_bytes": 2 * R * w.d * s,
        "combine_bytes": (R + w.T) * w.d * s,
        # what the combine actually moves: the expert rows (fp32 or y16), the
        # output rows, the fp32 shared-expert rows, and each slot's row index
        # and weight
        "combine_bytes_actual": (R * ys + w.T * w.d * s + (w.f_shared > 0) * w.T * w.d * 4
                                 + w.T * w.k_max * 8),
    }


def y16_rows(w, fp8: bool = False) -> bool:
    """Whether moe_layer passes the routed experts' outputs to the combine in
    the compact y16 form: bf16 layers with bf16 expert weights, unless
    MOE_Y16=0 or the down projection is forced onto the swap-AB engine."""
    eng = os.environ.get("MOE_GEMM_ENGINE", "")
    return (w.dtype == "bf16" and not fp8 and not os.environ.get("MOE_Y16", "1").startswith("0")
            and not eng.startswith("sw"))


def profile_summary(path: str, src: str):
    """DRAM bytes per launch from a committed ncu summary, when that summary
    was taken on the current source of the kernel; else None."""
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_hash = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", text)
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not (m_hash and m_bytes):
        return None
    cur = hashlib.sha256(open(src, "rb").read()).hexdigest()
    return float(m_bytes.group(1)) if cur == m_hash.group(1) else None


def traffic_from_profile(workload: str, kernel: str = "k5_up_swiglu"):
    """DRAM bytes per launch of a stage's kernel from profiles/<kernel>_<workload>.md
    (workload names ending in _fp8: the legs with e4m3 expert weights)."""
    if kernel.startswith(("k4", "k7")):
        src = PERMUTE_SRC
    elif workload.endswith("_fp8") and w_is_decode(workload):
        src = F8_SRC
    else:
        src = GEMM_SRC
    return profile_summary(os.path.join(PROFILES, f"{kernel}_{workload}.md"), src)


def alu_peak_tflops(sms: int, sm_max_mhz: float) -> float:
    """fp32 FMA peak of the CUDA cores: SMs x 128 fp32 lanes x 2 flops x clock."""
    return sms * 128 * 2 * sm_max_mhz * 1e6 / 1e12


def roofline_obj(kind: str, achieved: float, peak: float, unit: str, traffic, peak_src: str,
                 work: float, ms: float, clocks: dict | None = None) -> dict:
    o = {"bound": kind, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
         "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": peak_src,
         "work_per_launch": work, "ms_per_launch": round(ms, 5)}
    # the tensor and ALU peaks scale with the SM clock; HBM bandwidth does not.
    # nvidia-smi gives clock snapshots, which swing by hundreds of MHz under
    # the power cap: the scaled fraction needs enough of them, and one above
    # 1 says the snapshots missed the clock the kernel ran at
    if kind in ("tensor", "alu") and clocks and clocks.get("sm_mhz") and clocks.get("sm_max_mhz"):
        o["sm_mhz"] = clocks["sm_mhz"]
        n = clocks.get("samples", 0)
        v = achieved / (peak * clocks["sm_mhz"] / clocks["sm_max_mhz"])
        if n < MIN_CLOCK_SAMPLES:
            o["frac_at_sampled_clock"] = None
            o["sampled_clock_note"] = f"{n} clock samples in the timed region: too few"
        elif v > 1.0:
            o["frac_at_sampled_clock"] = None
            o["sampled_clock_note"] = ("the median sampled clock is below the clock the kernel "
                                       "ran at (snapshots under the power cap): not reported")
        else:
            o["frac_at_sampled_clock"] = round(v, 4)
    return o


def kernel_roofline(flops: float, nbytes: float, ms: float, pk: dict, pk_src: str, traffic=None,
                    clocks: dict | None = None, alu_peak: float | None = None) -> dict:
    """Roofline of one kernel from its algorithmic work and its mean launch
    time: bound by whichever of its FLOPs at the compute peak (bf16 tensor
    cores, measured burst figure; or, for fp32 CUDA-core work, the ALU peak)
    or its bytes at the measured copy bandwidth takes longer."""
    peak_tf = alu_peak if alu_peak else pk["bf16_tflops"]
    t_flops = flops / (peak_tf * 1e12)
    t_bytes = nbytes / (pk["hbm_gbs"] * 1e9)
    if flops and t_flops >= t_bytes:
        kind = "alu" if alu_peak else "tensor"
        src = ("fp32 FMA peak: SMs x 128 lanes x 2 x max SM clock" if alu_peak
               else f"{pk_src} bf16 burst (cuBLAS)")
        return roofline_obj(kind, flops / (ms * 1e-3) / 1e12, round(peak_tf, 1), "TFLOP/s",
                            traffic, src, flops, ms, clocks)
    return roofline_obj("hbm", nbytes / (ms * 1e-3) / 1e9, pk["hbm_gbs"], "GB/s", traffic,
                        f"{pk_src} copy bandwidth", nbytes, ms, clocks)


def stage_rooflines(w, alg: dict, stage_ms: dict, pk: dict, pk_src: str, clocks: dict,
                    workload: str, alu_peak: float, profiled: bool = True) -> dict:
    """Roofline objects of the dispatch (K4), up projection (K5), down
    projection (K6) and combine (K7) stages, from their event-timed means."""
    tr = (lambda k: traffic_from_profile(workload, k)) if profiled else (lambda k: None)
    out = {}
    if w.dtype == "f32":  # one fp32 CUDA-core FFN kernel runs both projections
        out["up_swiglu"] = kernel_roofline(
            alg["up_flops"] + alg["down_flops"], alg["up_bytes"] + alg["down_bytes"],
            stage_ms["up_swiglu"], pk, pk_src, None, clocks, alu_peak)
    else:
        out["up_swiglu"] = kernel_roofline(alg["up_flops"], alg["up_bytes"], stage_ms["up_swiglu"],
                                           pk, pk_src, tr("k5_up_swiglu"), clocks)
        out["down"] = kernel_roofline(alg["down_flops"], alg["down_bytes"], stage_ms["down"], pk,
                                      pk_src, tr("k6_down"), clocks)
    out["dispatch"] = kernel_roofline(0, alg["dispatch_bytes"], stage_ms["dispatch"], pk, pk_src,
                                      tr("k4_dispatch"), clocks)
    comb = kernel_roofline(0, alg["combine_bytes"], stage_ms["combine"], pk, pk_src,
                           tr("k7_combine"), clocks)
    act = alg["combine_bytes_actual"] / (stage_ms["combine"] * 1e-3) / 1e9
    comb["actual_bytes_per_launch"] = alg["combine_bytes_actual"]
    comb["frac_on_actual_bytes"] = round(act / pk["hbm_gbs"], 4)
    comb["note"] = ("bytes per the layer definition, (R+T) rows in the layer dtype; "
                    "frac_on_actual_bytes counts what the kernel moves: the expert rows "
                    + ("in y16 form (fp16 + a block exponent)" if y16_rows(w) else "in fp32")
                    + ", the output rows, the slots' rows and weights")
    out["combine"] = comb
    return out


class Layer:
    def __init__(self, name: str, dev, seed: int, T: int = 0, fp8: bool = False, E: int = 0):
        from routing_dispatch_expert_sigmoid_b200 import ops
        self.ops = ops
        self.w = WORKLOADS[name] if T <= 0 else WORKLOADS[name].scaled(T=T)
        if E > 0:
            self.w = self.w.scaled(E=E)
        self.inp = make_inputs(self.w, seed, device=dev)
        self.cfg = ops.config(self.w)
        self.ws = ops.workspace(self.cfg, ops.WS_LAYER, device=dev)
        self.rb = ops.route_buffers(self.cfg, device=dev)
        self.out = torch.empty_like(self.inp["x"])
        self.fp8 = None
        if fp8:  # weight preparation, outside any timed region
            i = self.inp
            self.fp8 = (ops.fp8_weight_set(i["W1"], i["W3"], i["W2"]),
                        ops.fp8_weight_set(i["Ws1"], i["Ws3"], i["Ws2"]) if self.w.f_shared
                        else None)
            for k in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2"):
                i[k] = None  # the bf16 copies are not used by this layer
            torch.cuda.empty_cache()

    def args(self, x=None, out=None):
        i = self.inp
        return (self.cfg, i["x"] if x is None else x, i["Wr"], i["logit_bias"], i["sel_bias"],
                i["k_per_token"], i["W1"], i["W3"], i["W2"], i["Ws1"], i["Ws3"], i["Ws2"],
                self.out if out is None else out, self.rb, self.ws)

    def step(self, x=None, out=None):
        if self.fp8:
            self._fp8_layer(x, out, None)
        else:
            self.ops.moe_layer(*self.args(x, out))

    def timed_step(self, events):
        if self.fp8:
            self._fp8_layer(None, None, events)
        else:
            self.ops.moe_layer_timed(*self.args(), events)

    def _fp8_layer(self, x, out, events):
        i = self.inp
        self.ops.moe_layer_fp8(self.cfg, i["x"] if x is None else x, i["Wr"], i["logit_bias"],
                               i["sel_bias"], i["k_per_token"], self.fp8[0], self.fp8[1],
                               self.out if out is None else out, self.rb, self.ws, events=events)


def run_device(layer: Layer, steps: int, warmup: int, dist, gpu_index: int) -> dict:
    """K device-timed steps of moe_layer, the call a user makes (the layer
    time); then K more steps of moe_layer_timed, whose events on the
    launching stream between the stages give the per-stage times.  The
    events are kept out of the first loop: each costs the stream a few
    microseconds, which a layer called without them does not pay."""
    nst = len(layer.ops.STAGES)
    for _ in range(warmup):
        layer.step()
    layer.ops.moe_check_errors()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nst)] for _ in range(steps)]
    for row in evs:  # create the events before the timed region
        for e in row:
            e.record()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t2, t3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(dist)
    torch.cuda.synchronize()
    with ClockSampler(gpu_index) as clk:
        t0.record()
        for k in range(steps):
            layer.step()
        t1.record()
        torch.cuda.synchronize()
    barrier(dist)
    torch.cuda.synchronize()
    layer.ops.moe_check_errors()
    ms = t0.elapsed_time(t1)
    # the stage-timed pass (same steps, outside the timed region)
    t2.record()
    for k in range(steps):
        layer.timed_step(evs[k])
    t3.record()
    torch.cuda.synchronize()
    layer.ops.moe_check_errors()
    stage_ms = {}
    for i in range(1, nst):
        stage_ms[layer.ops.STAGES[i]] = statistics.mean(
            evs[k][i - 1].elapsed_time(evs[k][i]) for k in range(steps))
    R = int(layer.rb["offsets"][-1].item())
    touched = int((layer.rb["kept"] > 0).sum().item())
    counts = layer.rb["counts"].double()
    return {"ms": ms, "stage_ms": stage_ms, "staged_ms": t2.elapsed_time(t3), "R": R,
            "touched": touched,
            "load_max_over_mean": float(counts.max() / counts.mean()),
            "n_dropped": int(layer.rb["n_dropped"].item()), "clocks": clk.summary()}


def run_e2e(layer: Layer, steps: int, warmup: int, dist) -> dict:
    """Host buffers through the C ABI, double-buffered the way a serving loop
    runs: every step copies its x from pinned host memory and its output back
    to pinned host memory, on two copy streams, so that the input copy of step
    i+1 and the output copy of step i-1 overlap the layer of step i.  The timed
    region runs from before the first input copy to after the last output
    copy."""
    x_host = layer.inp["x"].cpu().pin_memory()
    out_host = [torch.empty_like(x_host).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(layer.inp["x"]) for _ in range(2)]
    out_dev = [torch.empty_like(layer.out) for _ in range(2)]
    comp = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    x_free = [torch.cuda.Event() for _ in range(2)]     # the layer is done with x_dev[b]
    out_ready = [torch.cuda.Event() for _ in range(2)]
    out_free = [torch.cuda.Event() for _ in range(2)]   # out_dev[b] has been copied out

    def load(b):
        with torch.cuda.stream(h2d):
            h2d.wait_event(x_free[b])
            x_dev[b].copy_(x_host, non_blocking=True)
            in_ready[b].record(h2d)

    def run(n):
        h2d.wait_stream(comp)
        d2h.wait_stream(comp)
        load(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                load(1 - b)
            comp.wait_event(in_ready[b])
            comp.wait_event(out_free[b])
            layer.step(x_dev[b], out_dev[b])
            x_free[b].record(comp)
            out_ready[b].record(comp)
            with torch.cuda.stream(d2h):
                d2h.wait_event(out_ready[b])
                out_host[b].copy_(out_dev[b], non_blocking=True)
                out_free[b].record(d2h)
        comp.wait_stream(d2h)

    def serial(n):  # the same copies and layer, one after the other on one stream
        for _ in range(n):
            x_dev[0].copy_(x_host, non_blocking=True)
            layer.step(x_dev[0], out_dev[0])
            out_host[0].copy_(out_dev[0], non_blocking=True)

    ms = {}
    for kind, fn in (("overlapped", run), ("serial", serial)):
        fn(max(warmup, 2))
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        barrier(dist)
        t0.record(comp)
        fn(steps)
        t1.record(comp)
        torch.cuda.synchronize()
        barrier(dist)
        ms[kind] = t0.elapsed_time(t1)
    nbytes = x_host.numel() * x_host.element_size()
    return {"ms": ms["overlapped"], "ms_serial": ms["serial"], "h2d": nbytes,
            "d2h": out_host[0].numel() * out_host[0].element_size()}


# ---------------------------------------------------------------------------
# the CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------
def oracle_tokens_per_s(name: str, n_tok: int, reps: int = 1, dev=None) -> dict:
    import numpy as np

    import oracle
    from routing_dispatch_expert_sigmoid_b200.workloads import to_numpy
    w = WORKLOADS[name]
    gen_dev = dev if dev is not None else ("cuda" if torch.cuda.is_available() else "cpu")
    inp = make_inputs(w, 0, device=gen_dev)
    h = {k: to_numpy(v) for k, v in inp.items()}
    del inp
    n_tok = min(n_tok, w.T)
    times = []
    for r in range(reps):
        lo = (r * n_tok) % max(w.T - n_tok + 1, 1)
        sl = slice(lo, lo + n_tok)
        t0 = time.perf_counter()
        oracle.layer(h["x"][sl], h["Wr"], h["W1"], h["W3"], h["W2"], k_max=w.k_max,
                     gating_mode=w.gating, capacity_factor=float(np.float32(w.capacity_factor)),
                     logit_bias=h["logit_bias"], sel_bias=h["sel_bias"],
                     k_per_token=None if h["k_per_token"] is None else h["k_per_token"][sl],
                     n_groups=w.n_groups, topk_groups=w.topk_groups,
                     group_score_topk=w.group_score_topk, routed_scale=w.routed_scale,
                     Ws1=h["Ws1"], Ws3=h["Ws3"], Ws2=h["Ws2"])
        times.append(time.perf_counter() - t0)
    threads = int(os.environ.get("OMP_NUM_THREADS", len(os.sched_getaffinity(0))))
    # the oracle parallelises the FFN over tokens: it keeps min(tokens, threads) cores busy
    return {"tokens": n_tok, "times": times, "cores": min(threads, n_tok)}


def cpu_sample_tokens(name: str, budget_s: float) -> int:
    """Tokens the oracle processes in about budget_s on all host cores, from a
    probe of one token per core."""
    cores = len(os.sched_getaffinity(0))
    probe = oracle_tokens_per_s(name, cores)
    per_tok = max(probe["times"][0] / cores, 1e-4)
    return max(1, min(int(budget_s / per_tok), WORKLOADS[name].T))


# ---------------------------------------------------------------------------
# one measured leg: a workload, timed, with its rooflines
# ---------------------------------------------------------------------------
# The workloads of the layer definition besides the Mixtral-shaped legs, each
# measured by the default run and reported under "configs".
OTHER_CONFIGS = ("tiny_f32", "qwen3_prefill", "dsv3_decode", "dsv3_decode:fp8", "dsv3_prefill",
                 "gptoss_sub")


def describe(w) -> str:
    return (f"{w.name}: T={w.T}, d={w.d}, E={w.E}, top-{w.k_max}"
            + (f" (k_t in {w.k_min}..{w.k_max})" if w.k_min else "") + f", f={w.f}"
            + (f", shared f={w.f_shared}" if w.f_shared else "")
            + f", {w.gating}, capacity factor {w.capacity_factor or 'none'}, {w.dtype}")


def measure_leg(name: str, steps: int, warmup: int, dist, local_rank: int, dev, pk: dict,
                pk_src: str, sms: int, T: int = 0, fp8: bool = False, e2e: bool = False,
                profiled: bool = True, E: int = 0) -> tuple[dict, dict]:
    """Time one workload; returns (the leg's JSON object, raw numbers)."""
    layer = Layer(name, dev, seed=int(os.environ.get("RANK", "0")), T=T, fp8=fp8, E=E)
    w = layer.w
    r = run_device(layer, steps, warmup, dist, local_rank)
    e2e_r = run_e2e(layer, steps, warmup, dist) if e2e else None
    ms_max, tokens = aggregate(r["ms"], w.T * steps, dist)
    alg = algorithmic(w, r["R"], r["touched"], fp8=fp8)
    clocks = r["clocks"]
    alu = alu_peak_tflops(sms, clocks.get("sm_max_mhz") or 1965.0)
    kern = stage_rooflines(w, alg, r["stage_ms"], pk, pk_src, clocks,
                           w.name + ("_fp8" if fp8 else ""), alu, profiled and T <= 0 and E <= 0)
    roof_ms = layer_roofline_ms(alg, pk)
    step_ms = ms_max / steps
    obj = {
        "workload": describe(w) + (", e4m3 expert weights with per-column fp32 scales"
                                   if fp8 else ""),
        "steps": steps, "value": round(tokens / (ms_max * 1e-3), 1), "unit": "tokens/s",
        "ms_per_step": round(step_ms, 4),
        "stage_ms": {k: round(v, 4) for k, v in r["stage_ms"].items()},
        # the per-step time of the stage-timed pass (its events included)
        "ms_per_step_stage_timed": round(r["staged_ms"] / steps, 4),
        "layer_roofline_ms": round(roof_ms, 4),
        "layer_roofline_frac": round(roof_ms / step_ms, 4),
        "layer_roofline_frac_nominal": round(layer_roofline_ms(alg, NOMINAL_PEAKS) / step_ms, 4),
        # the dominant kernel: the up projection with SwiGLU (K5)
        "roofline": kern["up_swiglu"],
        "kernels": kern,
        "kept_rows": r["R"], "experts_touched": r["touched"],
        "load_max_over_mean": round(r["load_max_over_mean"], 3), "n_dropped": r["n_dropped"],
        # the device-timed loop, the stage-timed pass and (e2e) its two loops
        "gpu_launches": launches_per_layer(w) * steps * (4 if e2e else 2),
        "clocks": clocks,
    }
    raw = {"w": w, "ms_max": ms_max, "tokens": tokens, "e2e": e2e_r}
    if e2e_r is not None:
        raw["e2e_ms"] = aggregate(e2e_r["ms"], w.T * steps, dist)[0]
        raw["e2e_serial_ms"] = aggregate(e2e_r["ms_serial"], w.T * steps, dist)[0]
    del layer
    gc.collect()
    torch.cuda.empty_cache()
    return obj, raw


# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--workload", default=PREFILL, choices=sorted(WORKLOADS),
                    help="workload of the main (prefill) leg")
    ap.add_argument("--T", type=int, default=0, help="override the main leg's token count")
    ap.add_argument("--E", type=int, default=0,
                    help="override the main leg's expert count (a smaller case for profiling)")
    ap.add_argument("--decode-workload", default=DECODE,
                    choices=sorted(WORKLOADS) + ["none"], help="workload of the decode leg")
    ap.add_argument("--fp8-workload", default=DECODE, choices=sorted(WORKLOADS) + ["none"],
                    help="workload of the leg with fp8 expert weights")
    ap.add_argument("--configs", default=",".join(OTHER_CONFIGS),
                    help="comma-separated further workloads to measure ('none': no others)")
    a = ap.parse_args()
    rank, local_rank, world = dist_env()
    warmup = max(a.warmup, 3)

    if a.impl == "reference":
        if rank != 0:
            return 0
        cores = len(os.sched_getaffinity(0))
        n_tok = max(cores, cpu_sample_tokens(PREFILL, a.cpu_budget_s / max(a.steps + warmup, 1)))
        r = oracle_tokens_per_s(PREFILL, n_tok, reps=a.steps + warmup)
        timed = r["times"][warmup:]
        total_s = sum(timed)
        value = n_tok * len(timed) / total_s
        sample = (f"{n_tok} consecutive tokens of the {PREFILL} batch per step "
                  f"(router, gating, dispatch layout, expert FFN and combine in fp64)")
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
            "n_gpus": a.gpus, "steps": a.steps, "warmup": warmup,
            "ms_per_step": round(1e3 * total_s / len(timed), 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{PREFILL} (T={WORKLOADS[PREFILL].T}, d=4096, E=8, top-2, "
                                   "f=14336), CPU oracle on a sample of the batch"},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": r["cores"],
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }), flush=True)
        return 0

    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = init_dist(world, "nccl")
    pk, pk_src = peaks()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    leg = dict(dist=dist, local_rank=local_rank, dev=dev, pk=pk, pk_src=pk_src, sms=sms)

    main_obj, main_raw = measure_leg(a.workload, a.steps, warmup, T=a.T, E=a.E,
                                     e2e=not a.no_e2e, **leg)
    w = main_raw["w"]
    dec_obj = None
    if a.decode_workload != "none":
        dec_obj, _ = measure_leg(a.decode_workload, max(a.steps, 50), warmup, **leg)
    fp8_obj = None
    if a.fp8_workload != "none":
        fp8_obj, _ = measure_leg(a.fp8_workload, max(a.steps, 50), warmup, fp8=True, **leg)
    configs = {}
    for entry in [c for c in a.configs.split(",") if c and c != "none"]:
        name, _, kind = entry.partition(":")  # "<workload>:fp8": e4m3 expert weights
        wc = WORKLOADS[name]
        steps = max(a.steps, 50) if wc.T <= 256 else a.steps
        configs[name + ("_fp8" if kind == "fp8" else "")], _ = measure_leg(
            name, steps, warmup, fp8=kind == "fp8", **leg)

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        n_tok = cpu_sample_tokens(a.workload, a.cpu_budget_s)
        r = oracle_tokens_per_s(a.workload, n_tok, dev=dev)
        cpu = {"value": round(n_tok / r["times"][0], 3), "unit": "tokens/s", "cores": r["cores"],
               "kind": "oracle",
               "sample": f"{n_tok} tokens of the {a.workload} batch, whole layer in fp64 "
                         f"({r['times'][0]:.1f} s)"}

    if rank == 0:
        ms_max, tokens = main_raw["ms_max"], main_raw["tokens"]
        e2e = main_raw["e2e"]
        line = {
            "metric": METRIC, "value": round(tokens / (ms_max * 1e-3), 1), "unit": "tokens/s",
            "n_gpus": world, "steps": a.steps, "warmup": warmup,
            "ms_per_step": round(ms_max / a.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded normal inputs and weights of the stated shapes)",
            "config": {
                "workload": describe(w),
                "global_batch_tokens": w.T * world, "parallelism": f"replicas x{world}",
                "l2": "inputs larger than L2 (expert weights > 126 MB L2); no flush",
                "kept_rows": main_obj["kept_rows"], "experts_touched": main_obj["experts_touched"],
                "load_max_over_mean": main_obj["load_max_over_mean"],
                "n_dropped": main_obj["n_dropped"],
            },
            "stage_ms": main_obj["stage_ms"],
            "ms_per_step_stage_timed": main_obj["ms_per_step_stage_timed"],
            "layer_roofline_ms": main_obj["layer_roofline_ms"],
            "layer_roofline_frac": main_obj["layer_roofline_frac"],
            "layer_roofline_frac_nominal": main_obj["layer_roofline_frac_nominal"],
            "roofline": main_obj["roofline"],
            "kernels": main_obj["kernels"],
            "decode": dec_obj,
            "fp8_weights": fp8_obj,
            "configs": configs,
            "e2e": None if e2e is None else {
                "value": round(tokens / (main_raw["e2e_ms"] * 1e-3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "copies": "pinned host buffers; each step's input and output copies run on two "
                          "copy streams, overlapping the neighbouring steps' layers",
                "serial_value": round(tokens / (main_raw["e2e_serial_ms"] * 1e-3), 1)},
            "gpu_launches": (main_obj["gpu_launches"]
                             + sum(o["gpu_launches"] for o in (dec_obj, fp8_obj) if o)
                             + sum(o["gpu_launches"] for o in configs.values())),
            "clocks": main_obj["clocks"],
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
