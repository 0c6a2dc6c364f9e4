"""moe_route_static_scratch: routing for callers that cannot give the library
device memory (a plugin interface that carries only inputs and outputs, a
runtime whose HBM is fully planned in advance, a path that must not call an
allocator).  Its scratch is a fixed 1 MiB device array inside libmoe.so.

The GPU test calls it through the C ABI twice in a row, on different inputs,
and checks each result against moe_route (the workspace entry point) on the
same inputs: indices, counts and layout bit for bit, logits within the router
tolerance.  The second call also shows that the array's leftover contents
from the first call do not leak into the next result.  This file is collected
last so that a failure here cannot hide the result of any other test.
"""
import ctypes

import pytest
import torch

from parity import LOGIT_TOL, f64
from routing_dispatch_expert_sigmoid_b200 import ops
from routing_dispatch_expert_sigmoid_b200.workloads import WORKLOADS, make_inputs

CASES = [
    # capacity drops, renormalised softmax
    WORKLOADS["qwen3_prefill"].scaled(T=3000, d=256, E=128, f=64),
    # variable k, 512 experts, several chunks of the capacity step
    WORKLOADS["gptoss_sub"].scaled(T=2500, d=256, f=64),
    # sigmoid scores, selection bias, group-limited routing
    WORKLOADS["dsv3_decode"].scaled(d=512, f=64, f_shared=64),
    # decode-sized Mixtral-shaped routing: 8 experts, split-K router partials
    WORKLOADS["mixtral_decode"].scaled(d=512, f=64),
    # the split-K partials at their 768 KiB limit: 96 tokens x 1024 experts x
    # 4 bytes x 2 slices
    WORKLOADS["qwen3_prefill"].scaled(T=96, d=1024, E=1024, f=64),
]


def _route_both(w, seed, dev):
    inp = make_inputs(w, seed, device=dev)
    cfg = ops.config(w)
    ref = ops.route_buffers(cfg)
    ws = ops.workspace(cfg, ops.WS_ROUTE)
    ops.moe_route(cfg, inp["x"], inp["Wr"], inp["logit_bias"], inp["sel_bias"],
                  inp["k_per_token"], ref, ws)
    got = ops.route_buffers(cfg)
    for b in got.values():  # poison the outputs: every element must be written
        b.fill_(-7)
    ops.moe_route_static_scratch(cfg, inp["x"], inp["Wr"], inp["logit_bias"], inp["sel_bias"],
                                 inp["k_per_token"], got)
    ops.moe_check_errors()
    return ref, got


def _same(ref, got, R):
    for key in ("topk_idx", "counts", "kept", "offsets", "slot_row", "n_dropped"):
        assert torch.equal(ref[key], got[key]), key
    assert torch.equal(ref["row_src"][:R], got["row_src"][:R]), "row_src"
    assert torch.equal(ref["topk_w"], got["topk_w"]), "topk_w"
    lref, lgot = f64(ref["logits"]), f64(got["logits"])
    rms = (lref ** 2).mean() ** 0.5
    assert abs(lgot - lref).max() <= LOGIT_TOL * rms


@pytest.mark.gpu
def test_static_scratch_route_matches_workspace_route_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    for w in CASES:
        for seed in (11, 12):  # two calls in a row on different inputs
            ref, got = _route_both(w, seed, dev)
            _same(ref, got, int(ref["offsets"][-1].item()))


def test_static_scratch_rejects_configs_beyond_its_size():
    """Host-side check: nothing is enqueued, no device is touched."""
    w = WORKLOADS["gptoss_sub"].scaled(T=200000, E=1024, k_max=16)  # needs ~25 MiB
    cfg = ops.config(w)
    fake = ctypes.c_void_p(0x7F0000000000)
    out = ops.MoeRouteOut(*([0x7F0000000000] * 9))
    st = ops.lib().moe_route_static_scratch(ctypes.byref(cfg), fake, fake, None, None, None,
                                            ctypes.byref(out), None)
    assert st == -3 and "workspace" in ops.moe_status_string(st).lower()


def test_budget_case_fills_the_partial_logit_budget():
    """Host-side: the last case's routing scratch is the split-K partial
    logits at their 768 KiB limit plus the 256-byte ticket word."""
    cfg = ops.config(CASES[-1])
    assert ops.moe_workspace_size(cfg, ops.WS_ROUTE) == (768 << 10) + 256
