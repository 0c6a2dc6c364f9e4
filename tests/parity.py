"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same seeded inputs, compare.

Tolerances (written here once, used by every test):
  - routing indices, counts, kept, offsets, slot_row, row_src, n_dropped and
    the dispatched rows: bit-exact, with the oracle fed the GPU's fp32 logits;
  - router logits: max-abs error <= 1e-4 x RMS of the fp64 logits;
  - gate weights: |w_gpu - w_oracle| <= 1e-5 (fp32 softmax/sigmoid sums vs fp64);
  - layer / FFN outputs: max-abs error <= 2e-2 x RMS(reference) and relative
    Frobenius error <= 5e-3 (bf16 storage, fp32 accumulation).  The max-abs
    bound is on the error beyond the rounding of the result to its storage
    type: elementwise |got - ref| <= 2e-2 x RMS(ref) + half an ulp of the
    storage type at ref.  A correctly rounded bf16 copy of the exact output
    is already off by up to 2^-8 of |ref| just above a power of two, which
    exceeds 2e-2 x RMS on heavy-tailed outputs (2.1% measured on a case with
    many dropped tokens); the Frobenius bound is applied as stated.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from routing_dispatch_expert_sigmoid_b200 import ops
from routing_dispatch_expert_sigmoid_b200.workloads import Workload, make_inputs, to_numpy

LOGIT_TOL = 1e-4
W_TOL = 1e-5
OUT_MAXABS = 2e-2
OUT_FROB = 5e-3


def f64(t):
    """A device/host tensor (any float dtype) as a float64 numpy array."""
    return t.detach().to(torch.float64).cpu().numpy()


def assert_logits_close(gpu_logits, ref64):
    err = np.abs(f64(gpu_logits) - ref64).max() if ref64.size else 0.0
    rms = np.sqrt(np.mean(ref64 ** 2)) if ref64.size else 1.0
    assert err <= LOGIT_TOL * rms, f"logits max-abs {err:.3e} > {LOGIT_TOL} x RMS {rms:.3e}"


def half_ulp(ref, storage):
    """Half an ulp of the storage type (bf16: 8 significant bits, fp32: 24) at |ref|."""
    bits = {"bf16": 8, "f32": 24}[storage]
    e = np.floor(np.log2(np.maximum(np.abs(ref), np.finfo(np.float64).tiny)))
    return np.exp2(e - bits)


# (what, max-abs beyond rounding / RMS, raw max-abs / RMS, relative Frobenius,
# elements) of every output comparison of the session, printed at its end
MARGINS: list = []


def assert_out_close(got, ref, what="output", storage="bf16"):
    got = got if isinstance(got, np.ndarray) else f64(got)
    if ref.size == 0:
        return
    diff = got - ref
    rms = np.sqrt(np.mean(ref ** 2))
    excess = (np.abs(diff) - half_ulp(ref, storage)).max()
    raw = np.abs(diff).max()
    frob = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    MARGINS.append((what, excess / rms, raw / rms, frob, int(ref.size)))
    msg = (f"{what}: max-abs beyond {storage} rounding / RMS {excess / rms:.3e} (bound "
           f"{OUT_MAXABS}; raw max-abs/RMS {raw / rms:.3e}), "
           f"relative Frobenius {frob:.3e} (bound {OUT_FROB})")
    assert excess <= OUT_MAXABS * rms and frob <= OUT_FROB, msg
    return excess / rms, frob


def storage(w: Workload) -> str:
    return "f32" if w.dtype == "f32" else "bf16"


def oracle_cf(w: Workload) -> float:
    # The ABI carries the capacity factor as fp32; the oracle takes the same value.
    return float(np.float32(w.capacity_factor)) if w.capacity_factor > 0 else 0.0


def oracle_gating_kw(w: Workload, inp) -> dict:
    return dict(sel_bias=to_numpy(inp["sel_bias"]), k_per_token=to_numpy(inp["k_per_token"]),
                n_groups=w.n_groups, topk_groups=w.topk_groups,
                group_score_topk=w.group_score_topk, routed_scale=w.routed_scale)


def gpu_inputs(w: Workload, seed: int, dev, host_inputs=None):
    """Seeded inputs on the device (drawn on the host when host_inputs is given)."""
    if host_inputs is not None:
        return {k: (None if v is None else v.to(dev)) for k, v in host_inputs.items()}
    return make_inputs(w, seed, device=dev)


def run_route(w: Workload, inp, T=None):
    cfg = ops.config(w, T)
    out = ops.route_buffers(cfg)
    ws = ops.workspace(cfg, ops.WS_ROUTE)
    ops.moe_route(cfg, inp["x"], inp["Wr"], inp["logit_bias"], inp["sel_bias"],
                  inp["k_per_token"], out, ws)
    ops.moe_check_errors()
    return cfg, out


def check_routing_bit_exact(w: Workload, inp, out):
    """Oracle gating on the GPU's fp32 logits, oracle capacity/dispatch layout,
    compared element by element.  Returns the oracle's routing."""
    l32 = out["logits"].cpu().numpy()
    idx, wts = oracle.gating(l32, w.k_max, w.gating, **oracle_gating_kw(w, inp))
    got_idx = out["topk_idx"].cpu().numpy()
    bad = np.argwhere(got_idx != idx)
    assert bad.size == 0, f"topk_idx differs at {bad[:5].tolist()} (of {len(bad)})"
    np.testing.assert_allclose(out["topk_w"].cpu().numpy(), wts, rtol=0, atol=W_TOL)
    lay = oracle.capacity_dispatch(idx, w.E, oracle_cf(w))
    R = int(lay["offsets"][-1])
    for key in ("counts", "kept", "offsets"):
        assert (out[key].cpu().numpy() == lay[key]).all(), key
    assert (out["slot_row"].cpu().numpy() == lay["slot_row"]).all(), "slot_row"
    assert (out["row_src"][:R].cpu().numpy() == lay["row_src"]).all(), "row_src"
    assert int(out["n_dropped"].item()) == lay["n_dropped"], "n_dropped"
    return dict(topk_idx=idx, topk_w=wts, **lay)


def run_layer(w: Workload, inp, T=None, route_out=True):
    cfg = ops.config(w, T)
    ws = ops.workspace(cfg, ops.WS_LAYER)
    out = torch.empty_like(inp["x"])
    rb = ops.route_buffers(cfg) if route_out else None
    ops.moe_layer(cfg, inp["x"], inp["Wr"], inp["logit_bias"], inp["sel_bias"],
                  inp["k_per_token"], inp["W1"], inp["W3"], inp["W2"], inp["Ws1"], inp["Ws3"],
                  inp["Ws2"], out, rb, ws)
    ops.moe_check_errors()
    return out, rb


def oracle_layer_on_tokens(inp, routing, tokens, chunk_bytes=4 << 30):
    """fp64 layer output on the listed tokens, given the oracle's routing.

    Copies to the host only the weights of the experts the listed tokens use,
    at most about chunk_bytes of them at a time: the oracle runs once per
    chunk of experts with the slots of the other experts masked out (the
    shared expert in the first chunk only), and the fp64 chunk outputs are
    added.  That regroups the oracle's fp64 sum over a token's slots, which
    moves the result by a few fp64 ulps -- nothing next to the tolerances."""
    idx = routing["topk_idx"]
    sr = routing["slot_row"]
    toks = np.asarray(tokens, np.int32)
    used = sorted({int(e) for t in tokens for j, e in enumerate(idx[t]) if sr[t, j] >= 0})
    x = to_numpy(inp["x"])
    sh = [to_numpy(inp[k]) for k in ("Ws1", "Ws3", "Ws2")]
    per_expert = sum(inp[k][0].numel() * inp[k].element_size() for k in ("W1", "W3", "W2"))
    step = max(1, int(chunk_bytes // max(per_expert, 1)))
    chunks = [used[i:i + step] for i in range(0, len(used), step)] or [[]]
    total = None
    for ci, chunk in enumerate(chunks):
        remap = np.full(max(int(idx.max()) + 1, 1), -1, np.int32)
        remap[chunk] = np.arange(len(chunk), dtype=np.int32)
        W = {}
        for key in ("W1", "W3", "W2"):
            src = inp[key]
            if not chunk:
                W[key] = to_numpy(src[:1])
            else:
                sel = torch.tensor(chunk, device=src.device, dtype=torch.long)
                W[key] = to_numpy(src.index_select(0, sel))
        sub_idx = np.where(idx >= 0, remap[np.maximum(idx, 0)], -1).astype(np.int32)
        # slots of experts outside this chunk take no part in this pass
        sub_sr = np.where(sub_idx >= 0, sr, -1).astype(np.int32)
        part = oracle.layer_tokens(toks, x, W["W1"], W["W3"], W["W2"], sub_idx,
                                   routing["topk_w"], sub_sr, *(sh if ci == 0 else (None,) * 3))
        total = part if total is None else total + part
        del W
    return total
