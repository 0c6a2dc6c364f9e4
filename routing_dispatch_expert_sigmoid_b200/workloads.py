"""Workload shapes and seeded synthetic inputs for the MoE layer.

This module holds no arithmetic of the layer itself: it only names the layer
shapes and draws the random tensors that both the CUDA library and the CPU
oracle consume.  Draw order (one torch.Generator per call, seeded):
x, Wr, logit-bias permutation, W1, W3, W2, Ws1, Ws3, Ws2, sel_bias, k_t.

Distributions: x ~ N(0, 1); Wr, W1, W3, Ws1, Ws3 ~ N(0, 1/d); W2 ~ N(0, 1/f);
Ws2 ~ N(0, 1/f_shared); values are drawn in fp32 and rounded to nearest-even
into the layer's storage type.  The per-expert logit bias that creates hot
experts is the log of a Zipf law over a random ranking of the experts,
b_e = -s * ln(rank_e), rank a seeded permutation of 1..E; the DeepSeek-V3
shaped layer's selection bias is N(0, 0.05^2); the fine-grained GPT-OSS shaped
layer draws each token's k uniformly from {8, ..., 16}.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k_max: int
    f: int
    f_shared: int = 0
    dtype: str = "bf16"              # "f32" or "bf16" (storage of x, weights, outputs)
    gating: str = "topk_softmax"     # "topk_softmax" | "softmax_topk_renorm" | "sigmoid_grouped"
    capacity_factor: float = 0.0     # <= 0: no capacity limit
    zipf_s: float = 0.0              # log-Zipf logit bias exponent; 0: no logit bias
    n_groups: int = 1
    topk_groups: int = 1
    group_score_topk: int = 1
    routed_scale: float = 1.0
    k_min: int = 0                   # > 0: per-token k drawn from U{k_min..k_max}
    sel_bias_std: float = 0.0        # > 0: per-expert selection bias N(0, std^2)
    regime: str = ""

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


# Zipf exponent scale for the Qwen3-shaped layer: s = 1.2 * QWEN3_ZIPF_ALPHA gives
# a max/mean expert-load ratio near 3 on seed 0 (tests/golden/calibrate_qwen3_zipf.py
# recomputes it with the oracle's router and counts).
QWEN3_ZIPF_ALPHA = 0.14

WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_f32", T=256, d=256, E=8, k_max=2, f=512, dtype="f32",
                 capacity_factor=1.25, zipf_s=1.0, regime="correctness"),
        Workload("mixtral_decode", T=64, d=4096, E=8, k_max=2, f=14336, zipf_s=0.5,
                 regime="decode"),
        Workload("mixtral_prefill", T=8192, d=4096, E=8, k_max=2, f=14336, zipf_s=0.5,
                 regime="prefill"),
        Workload("qwen3_prefill", T=16384, d=2048, E=128, k_max=8, f=768,
                 gating="softmax_topk_renorm", capacity_factor=1.0,
                 zipf_s=1.2 * QWEN3_ZIPF_ALPHA, regime="prefill"),
        Workload("dsv3_decode", T=128, d=7168, E=256, k_max=8, f=2048, f_shared=2048,
                 gating="sigmoid_grouped", n_groups=8, topk_groups=4, group_score_topk=2,
                 routed_scale=2.5, sel_bias_std=0.05, regime="decode"),
        Workload("dsv3_prefill", T=4096, d=7168, E=256, k_max=8, f=2048, f_shared=2048,
                 gating="sigmoid_grouped", n_groups=8, topk_groups=4, group_score_topk=2,
                 routed_scale=2.5, sel_bias_std=0.05, regime="prefill"),
        Workload("gptoss_sub", T=8192, d=2880, E=512, k_max=16, k_min=8, f=720, zipf_s=1.0,
                 regime="prefill"),
    ]
}


def _normal(g, shape, std, dtype, device):
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        v.mul_(std)
    return v.to(dtype)


def _expert_stack(g, E, rows, cols, std, dtype, device):
    out = torch.empty((E, rows, cols), dtype=dtype, device=device)
    for e in range(E):  # one expert at a time: no fp32 copy of the whole stack
        out[e] = _normal(g, (rows, cols), std, dtype, device)
    return out


def make_inputs(w: Workload, seed: int = 0, device="cpu") -> dict:
    """Seeded synthetic inputs of workload w, as torch tensors on `device`."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    inp = {}
    inp["x"] = _normal(g, (w.T, w.d), 1.0, dt, dev)
    inp["Wr"] = _normal(g, (w.d, w.E), 1.0 / math.sqrt(w.d), dt, dev)
    if w.zipf_s > 0:
        rank = torch.randperm(w.E, generator=g, device=dev).to(torch.float64) + 1.0
        inp["logit_bias"] = (-w.zipf_s * torch.log(rank)).to(torch.float32)
    else:
        inp["logit_bias"] = None
    inp["W1"] = _expert_stack(g, w.E, w.d, w.f, 1.0 / math.sqrt(w.d), dt, dev)
    inp["W3"] = _expert_stack(g, w.E, w.d, w.f, 1.0 / math.sqrt(w.d), dt, dev)
    inp["W2"] = _expert_stack(g, w.E, w.f, w.d, 1.0 / math.sqrt(w.f), dt, dev)
    if w.f_shared > 0:
        inp["Ws1"] = _normal(g, (w.d, w.f_shared), 1.0 / math.sqrt(w.d), dt, dev)
        inp["Ws3"] = _normal(g, (w.d, w.f_shared), 1.0 / math.sqrt(w.d), dt, dev)
        inp["Ws2"] = _normal(g, (w.f_shared, w.d), 1.0 / math.sqrt(w.f_shared), dt, dev)
    else:
        inp["Ws1"] = inp["Ws3"] = inp["Ws2"] = None
    if w.sel_bias_std > 0:
        inp["sel_bias"] = _normal(g, (w.E,), w.sel_bias_std, torch.float32, dev)
    else:
        inp["sel_bias"] = None
    if w.k_min > 0:
        inp["k_per_token"] = torch.randint(w.k_min, w.k_max + 1, (w.T,), generator=g,
                                           device=dev, dtype=torch.int32)
    else:
        inp["k_per_token"] = None
    return inp


def to_numpy(t):
    """Host numpy view of a tensor for the oracle: float32 as is, bf16 as uint16 bits."""
    if t is None:
        return None
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    return t.numpy()
