"""moe_layer inside a CUDA graph.

The layer neither allocates, frees nor synchronises, so a caller can capture
one call into a CUDA graph and replay it: the launch chain is then submitted
by one graph launch, which is what a decode loop wants (the "MoE-Prism"
summary, section 2.B, treats the routing budget k as a runtime knob: one graph
per k).  A replay must give exactly the eager result, also after the inputs
are overwritten in place between replays.
"""
import pytest
import torch

from routing_dispatch_expert_sigmoid_b200 import ops
from routing_dispatch_expert_sigmoid_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

CASES = {
    # decode-sized batch: split-K router and fused gating/ranking kernel
    "mixtral_decode": WORKLOADS["mixtral_decode"].scaled(T=16, d=512, f=1024),
    # separate routing kernels, shared expert
    "dsv3_prefill": WORKLOADS["dsv3_prefill"].scaled(T=300, d=256, E=64, f=136, f_shared=72),
}

_ARGS = ("x", "Wr", "logit_bias", "sel_bias", "k_per_token", "W1", "W3", "W2", "Ws1", "Ws3",
         "Ws2")


def _layer(cfg, inp, out, rb, ws):
    ops.moe_layer(cfg, *[inp[k] for k in _ARGS], out, rb, ws)


@pytest.mark.parametrize("name", list(CASES))
def test_graph_replay_matches_eager(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    w = CASES[name]
    inp = make_inputs(w, 0, device=dev)
    nxt = make_inputs(w, 1, device=dev)  # second batch of tokens, same weights
    cfg = ops.config(w)
    ws = ops.workspace(cfg, ops.WS_LAYER)

    def eager(x):
        out = torch.empty_like(x)
        _layer(cfg, dict(inp, x=x), out, None, ws)
        ops.moe_check_errors()
        return out

    want0, want1 = eager(inp["x"].clone()), eager(nxt["x"].clone())

    x_static = inp["x"].clone()
    out = torch.empty_like(x_static)
    rb = ops.route_buffers(cfg)
    args = dict(inp, x=x_static)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up off the capture
        _layer(cfg, args, out, rb, ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _layer(cfg, args, out, rb, ws)
    out.fill_(0)
    g.replay()
    torch.cuda.synchronize()
    ops.moe_check_errors()
    assert torch.equal(out, want0)
    x_static.copy_(nxt["x"])  # new tokens in place, same graph
    g.replay()
    torch.cuda.synchronize()
    ops.moe_check_errors()
    assert torch.equal(out, want1)
    del g
