"""CUDA path vs the CPU oracle, element by element, on seeded inputs.

Small cases: every gating mode, both dtypes, several tiles of every kernel,
ragged tails in T, d, f and the expert groups, variable k, capacity drops,
shared expert.  Each step is checked on its own through its C-ABI entry point
(moe_route, moe_dispatch, moe_expert_ffn, moe_combine) and then as a whole
(moe_layer).  Tolerances are those of tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import (assert_logits_close, assert_out_close, check_routing_bit_exact, f64,
                    gpu_inputs, oracle_gating_kw, oracle_layer_on_tokens, run_layer, run_route,
                    storage)
from routing_dispatch_expert_sigmoid_b200 import ops
from routing_dispatch_expert_sigmoid_b200.workloads import WORKLOADS, make_inputs, to_numpy

pytestmark = pytest.mark.gpu

# Scaled-down layers of every workload family: same gating, k, groups, dtype;
# dimensions cross tile edges (128-row M tiles, 128/256-column N tiles, 64-deep
# K steps) with ragged tails.
SMALL = {
    "tiny_f32": WORKLOADS["tiny_f32"],
    "mixtral_small": WORKLOADS["mixtral_prefill"].scaled(T=300, d=256, f=384),
    # a handful of rows per expert
    "qwen3_decode_small": WORKLOADS["qwen3_prefill"].scaled(T=50, d=192, E=16, k_max=4, f=200),
    "qwen3_small": WORKLOADS["qwen3_prefill"].scaled(T=257, d=192, E=16, k_max=4, f=200),
    "dsv3_small": WORKLOADS["dsv3_prefill"].scaled(T=130, d=256, E=64, f=136, f_shared=72),
    "gptoss_small": WORKLOADS["gptoss_sub"].scaled(T=211, d=200, E=32, k_max=6, k_min=2, f=72),
    "mixtral_decode_small": WORKLOADS["mixtral_decode"].scaled(T=5, d=512, f=1024),
    # more rows per expert on average than the small cases
    "qwen3_medium": WORKLOADS["qwen3_prefill"].scaled(T=1100, d=192, E=16, k_max=4, f=200),
    "dsv3_medium": WORKLOADS["dsv3_prefill"].scaled(T=1200, d=256, E=64, f=136, f_shared=72),
}


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()
    return torch.device("cuda:0")


def _host_inputs(w, seed=0):
    return make_inputs(w, seed, device="cpu")


@pytest.mark.parametrize("name", list(SMALL))
def test_route_bit_exact_and_logits(name, dev):
    w = SMALL[name]
    hin = _host_inputs(w)
    inp = gpu_inputs(w, 0, dev, hin)
    cfg, out = run_route(w, inp)
    ref = oracle.router_logits(to_numpy(hin["x"]), to_numpy(hin["Wr"]),
                               to_numpy(hin["logit_bias"]))
    assert_logits_close(out["logits"], ref)
    check_routing_bit_exact(w, hin, out)


# The router GEMM on CTA pairs (default for E >= 512 and T >= 2048; forced on
# here): ragged T and E across the 256-row and 256-column tile edges, every
# gating mode, with and without the logit bias.
PAIR_ROUTER = {
    "gptoss_like": WORKLOADS["gptoss_sub"].scaled(T=600, d=200, E=512, k_max=16, k_min=8, f=64),
    "qwen3_like_ragged": WORKLOADS["qwen3_prefill"].scaled(T=257, d=136, E=136, k_max=8, f=64),
    "dsv3_like": WORKLOADS["dsv3_prefill"].scaled(T=300, d=256, E=256, f=64, f_shared=64),
    "mixtral_like_e8": WORKLOADS["mixtral_prefill"].scaled(T=513, d=128, f=64),
}


@pytest.mark.parametrize("name", list(PAIR_ROUTER))
def test_pair_router_bit_exact_and_logits(name, dev):
    import os
    old = os.environ.get("MOE_ROUTER_PAIR")
    os.environ["MOE_ROUTER_PAIR"] = "1"
    try:
        w = PAIR_ROUTER[name]
        hin = _host_inputs(w, seed=7)
        inp = gpu_inputs(w, 7, dev, hin)
        cfg, out = run_route(w, inp)
        ref = oracle.router_logits(to_numpy(hin["x"]), to_numpy(hin["Wr"]),
                                   to_numpy(hin["logit_bias"]))
        assert_logits_close(out["logits"], ref)
        check_routing_bit_exact(w, hin, out)
    finally:
        if old is None:
            os.environ.pop("MOE_ROUTER_PAIR", None)
        else:
            os.environ["MOE_ROUTER_PAIR"] = old


# The CUDA-core router (fp32 layers, and bf16 layers whose E is not a multiple
# of 8): one warp per token for short batches with at most 16 experts, the
# tiled kernel beyond 2048 tokens or 16 experts.
SIMT_ROUTER = {
    "bf16_e12_warp": WORKLOADS["qwen3_prefill"].scaled(T=300, d=200, E=12, k_max=3, f=64),
    "bf16_e12_tiled": WORKLOADS["qwen3_prefill"].scaled(T=2100, d=200, E=12, k_max=3, f=64),
    "bf16_e20_tiled": WORKLOADS["qwen3_prefill"].scaled(T=300, d=136, E=20, k_max=3, f=64),
    "f32_e8_tiled": WORKLOADS["tiny_f32"].scaled(T=2049),
}


@pytest.mark.parametrize("name", list(SIMT_ROUTER))
def test_simt_router_bit_exact_and_logits(name, dev):
    w = SIMT_ROUTER[name]
    hin = _host_inputs(w, seed=6)
    inp = gpu_inputs(w, 6, dev, hin)
    cfg, out = run_route(w, inp)
    ref = oracle.router_logits(to_numpy(hin["x"]), to_numpy(hin["Wr"]),
                               to_numpy(hin["logit_bias"]))
    assert_logits_close(out["logits"], ref)
    check_routing_bit_exact(w, hin, out)


@pytest.mark.parametrize("name", list(SMALL))
def test_dispatch_bit_exact(name, dev):
    w = SMALL[name]
    hin = _host_inputs(w)
    inp = gpu_inputs(w, 0, dev, hin)
    cfg, out = run_route(w, inp)
    lay = check_routing_bit_exact(w, hin, out)
    R = int(lay["offsets"][-1])
    x_perm = torch.full((w.T * w.k_max, w.d), float("nan"), dtype=inp["x"].dtype, device=dev)
    ops.moe_dispatch(cfg, inp["x"], out["offsets"], out["row_src"], x_perm)
    ops.moe_check_errors()
    ref = oracle.dispatch(to_numpy(hin["x"]), lay["row_src"], w.k_max)
    assert (to_numpy(x_perm[:R]) == ref).all()


@pytest.mark.parametrize("name", list(SMALL))
def test_expert_ffn_matches_oracle(name, dev):
    """Grouped FFN alone, on the oracle's dispatched rows and layout."""
    w = SMALL[name]
    hin = _host_inputs(w)
    inp = gpu_inputs(w, 0, dev, hin)
    cfg, out = run_route(w, inp)
    lay = check_routing_bit_exact(w, hin, out)
    R = int(lay["offsets"][-1])
    xp = oracle.dispatch(to_numpy(hin["x"]), lay["row_src"], w.k_max)
    x_perm = torch.zeros((w.T * w.k_max, w.d), dtype=inp["x"].dtype)
    x_perm[:R] = hin["x"][torch.from_numpy(lay["row_src"] // w.k_max).long()]
    assert (to_numpy(x_perm[:R]) == xp).all()
    x_perm = x_perm.to(dev)
    y_perm = torch.zeros(x_perm.shape, dtype=torch.float32, device=dev)
    ws = ops.workspace(cfg, ops.WS_EXPERT_FFN)
    offs = torch.from_numpy(lay["offsets"]).to(dev)
    ops.moe_expert_ffn(cfg, x_perm, offs, inp["W1"], inp["W3"], inp["W2"], y_perm, ws)
    ops.moe_check_errors()
    ref = oracle.grouped_ffn(xp, lay["offsets"], to_numpy(hin["W1"]), to_numpy(hin["W3"]),
                             to_numpy(hin["W2"]))
    assert_out_close(f64(y_perm[:R]), ref, "y_perm", "f32")


@pytest.mark.parametrize("name", list(SMALL))
def test_combine_matches_oracle(name, dev):
    """Combine alone, on seeded synthetic expert outputs and the oracle's layout."""
    w = SMALL[name]
    hin = _host_inputs(w)
    cfg = ops.config(w)
    l32 = oracle.router_logits(to_numpy(hin["x"]), to_numpy(hin["Wr"]),
                               to_numpy(hin["logit_bias"])).astype(np.float32)
    idx, wts = oracle.gating(l32, w.k_max, w.gating, **oracle_gating_kw(w, hin))
    lay = oracle.capacity_dispatch(idx, w.E, float(np.float32(w.capacity_factor)))
    dt = hin["x"].dtype
    g = torch.Generator().manual_seed(1)
    # expert outputs are fp32 rows; the layer output is rounded once to dt
    y_perm = torch.randn((w.T * w.k_max, w.d), generator=g)
    shared = torch.randn((w.T, w.d), generator=g) if w.f_shared else None
    out = torch.empty((w.T, w.d), dtype=dt, device=dev)
    ops.moe_combine(cfg, y_perm.to(dev), torch.from_numpy(lay["slot_row"]).to(dev),
                    torch.from_numpy(wts.astype(np.float32)).to(dev),
                    None if shared is None else shared.to(dev), out)
    ops.moe_check_errors()
    ref = oracle.combine_rows(wts.astype(np.float32).astype(np.float64), lay["slot_row"],
                              to_numpy(y_perm), to_numpy(shared))
    assert_out_close(f64(out), ref, "combine", storage(w))


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_matches_oracle(name, dev):
    w = SMALL[name]
    hin = _host_inputs(w)
    inp = gpu_inputs(w, 0, dev, hin)
    out, rb = run_layer(w, inp)
    routing = check_routing_bit_exact(w, hin, rb)
    ref = oracle_layer_on_tokens(hin, routing, list(range(w.T)))
    assert_out_close(f64(out), ref, "layer out", storage(w))
    # the layer without caller routing buffers gives the same output
    out2, _ = run_layer(w, inp, route_out=False)
    assert torch.equal(out, out2)


# ---------------------------------------------------------------------------
# Edge cases
# ---------------------------------------------------------------------------
def _layer_vs_oracle(w, hin, dev):
    inp = gpu_inputs(w, 0, dev, hin)
    out, rb = run_layer(w, inp)
    routing = check_routing_bit_exact(w, hin, rb)
    ref = oracle_layer_on_tokens(hin, routing, list(range(w.T)))
    assert_out_close(f64(out), ref, "layer out", storage(w))
    return rb


@pytest.mark.parametrize("T", [1, 2, 127, 129])
def test_token_counts_across_tile_edges(T, dev):
    w = SMALL["mixtral_small"].scaled(T=T)
    _layer_vs_oracle(w, _host_inputs(w, seed=T), dev)


def test_all_equal_logits_tie_to_lower_index(dev):
    w = SMALL["qwen3_small"].scaled(zipf_s=0.0, capacity_factor=0.0)
    hin = _host_inputs(w)
    hin["Wr"] = torch.zeros_like(hin["Wr"])
    rb = _layer_vs_oracle(w, hin, dev)
    assert (rb["topk_idx"].cpu() == torch.arange(w.k_max, dtype=torch.int32)).all()


def test_one_expert_takes_every_token_and_others_idle(dev):
    w = SMALL["mixtral_small"].scaled(T=260, k_max=1, zipf_s=0.0)
    hin = _host_inputs(w)
    hin["logit_bias"] = torch.tensor([0, 0, 0, 50.0, 0, 0, 0, 0])
    rb = _layer_vs_oracle(w, hin, dev)
    counts = rb["counts"].cpu().numpy()
    assert counts[3] == w.T and counts.sum() == w.T


def test_heavy_drops_small_capacity(dev):
    w = SMALL["qwen3_small"].scaled(capacity_factor=0.3)
    rb = _layer_vs_oracle(w, _host_inputs(w), dev)
    assert int(rb["n_dropped"].item()) > 0


def test_single_expert_dense(dev):
    w = SMALL["mixtral_small"].scaled(E=1, k_max=1, T=77)
    _layer_vs_oracle(w, _host_inputs(w), dev)


def test_k_equals_E_uniform(dev):
    w = SMALL["mixtral_small"].scaled(E=8, k_max=8, T=40, zipf_s=0.0)
    hin = _host_inputs(w)
    hin["Wr"] = torch.zeros_like(hin["Wr"])
    _layer_vs_oracle(w, hin, dev)


def test_empty_batch(dev):
    w = SMALL["dsv3_small"].scaled(T=0)
    cfg = ops.config(w)
    inp = make_inputs(w.scaled(T=1), 0, device=dev)
    x = inp["x"][:0]
    ws = ops.workspace(cfg, ops.WS_LAYER)
    out = torch.empty((0, w.d), dtype=x.dtype, device=dev)
    ops.moe_layer(cfg, inp["x"], inp["Wr"], None, inp["sel_bias"], None, inp["W1"], inp["W3"],
                  inp["W2"], inp["Ws1"], inp["Ws3"], inp["Ws2"], out, None, ws)
    ops.moe_check_errors()


# Decode-sized batches (bf16, E % 8 == 0, T <= 128) route with the split-K
# router and the fused gating/ranking kernel; T = 129 is the first batch on
# the separate kernels.  Cases: one token; the largest batch with a ragged last
# K slice (d = 448 is 7 steps of 64); 512 experts with variable k and padded
# slots; 1024 experts with k = 32 (4096 slots ranked by one CTA) and capacity
# drops; a small capacity factor; a shared expert whose projections are both
# split along K (7 up splits, 4 down splits added by the combine).
SMALL_BATCH = {
    "t1_mixtral": WORKLOADS["mixtral_decode"].scaled(T=1, d=512, f=128),
    "t128_dsv3_ragged_k": WORKLOADS["dsv3_decode"].scaled(T=128, d=448, f=64, f_shared=64),
    "t129_dsv3": WORKLOADS["dsv3_decode"].scaled(T=129, d=448, f=64, f_shared=64),
    "gptoss_e512_var_k": WORKLOADS["gptoss_sub"].scaled(T=100, d=200, f=72),
    "e1024_k32_drops": WORKLOADS["qwen3_prefill"].scaled(T=128, d=128, E=1024, k_max=32, f=64),
    "qwen3_cf_half": WORKLOADS["qwen3_prefill"].scaled(T=96, d=192, E=16, k_max=4, f=64,
                                                       capacity_factor=0.5),
    "t64_dsv3_shared_split": WORKLOADS["dsv3_decode"].scaled(T=64, d=448, f=64, f_shared=256),
}


@pytest.mark.parametrize("name", list(SMALL_BATCH))
def test_small_batch_route_bit_exact(name, dev):
    w = SMALL_BATCH[name]
    hin = _host_inputs(w, seed=3)
    inp = gpu_inputs(w, 3, dev, hin)
    cfg, out = run_route(w, inp)
    ref = oracle.router_logits(to_numpy(hin["x"]), to_numpy(hin["Wr"]),
                               to_numpy(hin["logit_bias"]))
    assert_logits_close(out["logits"], ref)
    check_routing_bit_exact(w, hin, out)


@pytest.mark.parametrize("name", list(SMALL_BATCH))
def test_small_batch_layer(name, dev):
    w = SMALL_BATCH[name]
    _layer_vs_oracle(w, _host_inputs(w, seed=4), dev)


@pytest.mark.parametrize("E", [64, 256])
@pytest.mark.parametrize("T", [512, 128])
def test_sigmoid_grouped_near_ties_bit_exact(T, E, dev):
    """Logits on a fine grid with many exact and one-ulp ties in the biased
    scores: selection must follow the specified sigmoid bit for bit (T = 128
    goes through the fused small-batch routing kernel; E = 256 makes groups
    of 32 experts, whose scores the warp computes by reductions)."""
    w = SMALL["dsv3_small"].scaled(T=T, E=E)
    hin = _host_inputs(w)
    cfg = ops.config(w)
    g = torch.Generator().manual_seed(5)
    # logits from a coarse grid -> many equal sigmoid values; bias on a grid too
    logits = (torch.randint(-8, 9, (w.T, w.E), generator=g).float() / 8.0)
    sel_bias = (torch.randint(-4, 5, (w.E,), generator=g).float() / 64.0)
    l_dev = logits.to(dev)
    out = ops.route_buffers(cfg)
    # route with Wr = 0 and the grid as logit bias would tie every token; instead
    # drive the gating through a router whose logits are exactly the grid:
    # x = identity rows (T <= d is not required: use d >= E and one-hot x).
    assert w.d >= w.E
    x = torch.zeros((w.T, w.d))
    Wr = torch.zeros((w.d, w.E))
    Wr[: w.E, :] = torch.eye(w.E)
    # x[t, :E] = logits[t] makes x.Wr = logits exactly (values are bf16-exact)
    x[:, : w.E] = logits
    hin2 = dict(hin, x=x.to(torch.bfloat16), Wr=Wr.to(torch.bfloat16), sel_bias=sel_bias,
                logit_bias=None)
    inp = gpu_inputs(w, 0, dev, hin2)
    ws = ops.workspace(cfg, ops.WS_ROUTE)
    ops.moe_route(cfg, inp["x"], inp["Wr"], None, inp["sel_bias"], None, out, ws)
    ops.moe_check_errors()
    assert torch.equal(out["logits"], l_dev)
    check_routing_bit_exact(w, hin2, out)


# ---------------------------------------------------------------------------
# Every grouped-GEMM engine (single-CTA, CTA-pair and swap-AB tiles) on every shape
# ---------------------------------------------------------------------------
@pytest.fixture(params=["single", "narrow", "pair", "swap", "mixed"])
def gemm_engine(request):
    import os
    old = os.environ.get("MOE_GEMM_ENGINE")
    os.environ["MOE_GEMM_ENGINE"] = request.param
    yield request.param
    if old is None:
        os.environ.pop("MOE_GEMM_ENGINE", None)
    else:
        os.environ["MOE_GEMM_ENGINE"] = old


BF16_SMALL = [n for n, w in SMALL.items() if w.dtype == "bf16"]


@pytest.mark.parametrize("name", BF16_SMALL)
def test_expert_ffn_each_engine(name, gemm_engine, dev):
    test_expert_ffn_matches_oracle(name, dev)


@pytest.mark.parametrize("name", BF16_SMALL)
def test_layer_each_engine(name, gemm_engine, dev):
    test_layer_matches_oracle(name, dev)


@pytest.mark.parametrize("T", [1, 15, 17, 255, 257, 600])
def test_tile_row_edges(T, gemm_engine, dev):
    w = SMALL["mixtral_small"].scaled(T=T)
    _layer_vs_oracle(w, _host_inputs(w, seed=T), dev)


# group sizes around every tile edge: empty, a few rows, the 16-row steps of a
# swap-AB tile, the 32-row boxes, full 128-row chunks with and without a
# remainder
GROUP_SIZES = [0, 1, 15, 16, 17, 31, 33, 127, 128, 129, 0, 255, 256, 300, 5]


def test_expert_ffn_group_size_edges(gemm_engine, dev):
    """moe_expert_ffn on hand-made expert groups (ragged K and N), every engine."""
    E, d, f = len(GROUP_SIZES), 200, 200
    offsets = np.concatenate([[0], np.cumsum(GROUP_SIZES)]).astype(np.int32)
    R = int(offsets[-1])
    w = WORKLOADS["qwen3_prefill"].scaled(T=R, d=d, E=E, k_max=1, f=f)
    cfg = ops.config(w)
    hin = _host_inputs(w, seed=5)
    xp = torch.randn(R, d, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    y = torch.zeros((R, d), dtype=torch.float32, device=dev)
    ops.moe_expert_ffn(cfg, xp.to(dev), torch.from_numpy(offsets).to(dev), hin["W1"].to(dev),
                       hin["W3"].to(dev), hin["W2"].to(dev), y,
                       ops.workspace(cfg, ops.WS_EXPERT_FFN))
    ops.moe_check_errors()
    ref = oracle.grouped_ffn(to_numpy(xp), offsets, to_numpy(hin["W1"]), to_numpy(hin["W3"]),
                             to_numpy(hin["W2"]))
    assert_out_close(f64(y), ref, "y_perm, group sizes across tile edges", "f32")


@pytest.fixture
def fp32_expert_rows():
    """MOE_Y16=0: the down projection writes fp32 rows instead of the compact
    y16 form (fp16 values with a power-of-two exponent per 32-column block)."""
    import os
    old = os.environ.get("MOE_Y16")
    os.environ["MOE_Y16"] = "0"
    yield
    if old is None:
        os.environ.pop("MOE_Y16", None)
    else:
        os.environ["MOE_Y16"] = old


@pytest.mark.parametrize("name", BF16_SMALL)
def test_layer_with_fp32_expert_rows(name, fp32_expert_rows, dev):
    test_layer_matches_oracle(name, dev)


@pytest.fixture(params=[("0", None), ("2", None), ("1", "255"), ("1", "1")],
                ids=["no-swap", "swap-remainders", "light-below-256", "light-1-row"])
def pair_swap(request):
    """MOE_GEMM_ENGINE=pair with MOE_PAIR_SWAP=0 (no swap-AB tiles: small
    groups padded to 256-row pair tiles), 2 (every group's partial last
    256-row chunk as a swap-AB pair tile too), or the default mode with the
    light list's row limit (MOE_PAIR_SWAP_ROWS) at its extremes; the default
    limit runs in every other pair test."""
    import os
    keys = ("MOE_GEMM_ENGINE", "MOE_PAIR_SWAP", "MOE_PAIR_SWAP_ROWS")
    old = {k: os.environ.get(k) for k in keys}
    os.environ["MOE_GEMM_ENGINE"] = "pair"
    os.environ["MOE_PAIR_SWAP"] = request.param[0]
    if request.param[1] is None:
        os.environ.pop("MOE_PAIR_SWAP_ROWS", None)
    else:
        os.environ["MOE_PAIR_SWAP_ROWS"] = request.param[1]
    yield request.param
    for k, v in old.items():
        if v is None:
            os.environ.pop(k, None)
        else:
            os.environ[k] = v


@pytest.mark.parametrize("name", BF16_SMALL)
def test_layer_pair_with_swap_tiles(name, pair_swap, dev):
    test_layer_matches_oracle(name, dev)


def test_expert_ffn_group_size_edges_pair_with_swap(pair_swap, dev):
    test_expert_ffn_group_size_edges("pair", dev)


@pytest.mark.parametrize("name", BF16_SMALL)
def test_expert_ffn_pair_with_swap_tiles(name, pair_swap, dev):
    test_expert_ffn_matches_oracle(name, dev)


@pytest.fixture(params=["1", "2"])
def pair_kps(request):
    """k-blocks per ring stage of the CTA-pair engine (the default picks 2
    only for K of 32 k-blocks or more, so small shapes would test 1 alone)."""
    import os
    keys = ("MOE_GEMM_ENGINE", "MOE_PAIR_KPS")
    old = {k: os.environ.get(k) for k in keys}
    os.environ["MOE_GEMM_ENGINE"] = "pair"
    os.environ["MOE_PAIR_KPS"] = request.param
    yield request.param
    for k, v in old.items():
        if v is None:
            os.environ.pop(k, None)
        else:
            os.environ[k] = v


# qwen3_small has d = 192: three k-blocks, so two per stage leaves a ragged last stage
@pytest.mark.parametrize("name", ["mixtral_small", "qwen3_small", "dsv3_small", "gptoss_small",
                                  "qwen3_medium"])
def test_layer_pair_kblocks_per_stage(name, pair_kps, dev):
    test_layer_matches_oracle(name, dev)


def test_expert_ffn_group_size_edges_pair_kblocks_per_stage(pair_kps, dev):
    test_expert_ffn_group_size_edges("pair", dev)


@pytest.fixture(params=["1", "2", "3"])
def l2_hints(request):
    """MOE_L2_HINTS=1|2|3: the GEMMs' TMA loads carry L2 eviction hints (the
    CTA-pair engine's three policies)."""
    import os
    old = os.environ.get("MOE_L2_HINTS")
    os.environ["MOE_L2_HINTS"] = request.param
    yield
    if old is None:
        os.environ.pop("MOE_L2_HINTS", None)
    else:
        os.environ["MOE_L2_HINTS"] = old


@pytest.mark.parametrize("name", ["mixtral_small", "qwen3_medium", "dsv3_medium", "gptoss_small"])
def test_layer_with_l2_hints(name, l2_hints, gemm_engine, dev):
    test_layer_matches_oracle(name, dev)


@pytest.fixture(params=["MOE_MIXED_SPLIT", "MOE_MIXED_PHASED", "MOE_MIXED_LIGHT_EVICT"])
def mixed_deal(request):
    """Deal variants of the mixed engine: heavy and light lists as two
    launches, heavy tiles before light ones, evict-first light weights."""
    import os
    keys = (request.param, "MOE_GEMM_ENGINE")
    old = {k: os.environ.get(k) for k in keys}
    os.environ[request.param] = "1"
    os.environ["MOE_GEMM_ENGINE"] = "mixed"
    yield request.param
    for k, v in old.items():
        if v is None:
            os.environ.pop(k, None)
        else:
            os.environ[k] = v


@pytest.mark.parametrize("name", ["mixtral_small", "qwen3_medium", "dsv3_medium", "gptoss_small"])
def test_layer_mixed_deal_variants(name, mixed_deal, dev):
    test_layer_matches_oracle(name, dev)


def test_expert_ffn_group_size_edges_mixed_deal_variants(mixed_deal, dev):
    test_expert_ffn_group_size_edges("mixed", dev)


# moe_layer dispatches long batches (T >= 1024) walking tokens: each row of x
# is read once and stored to every kept row of the token.  Ragged d (rows not
# a whole number of 4 KB chunks), capacity drops, variable k.
TOKEN_DISPATCH = {
    "qwen3_drops_ragged_d": WORKLOADS["qwen3_prefill"].scaled(T=1100, d=200, E=16, k_max=4,
                                                              f=64),
    "gptoss_variable_k": WORKLOADS["gptoss_sub"].scaled(T=1500, d=136, E=64, k_max=8, k_min=2,
                                                        f=64),
    "mixtral_wide_rows": WORKLOADS["mixtral_prefill"].scaled(T=1024, d=2056, f=64),
}


@pytest.mark.parametrize("by_row", ["0", "1"], ids=["by-token", "by-row"])
@pytest.mark.parametrize("name", list(TOKEN_DISPATCH))
def test_layer_dispatch_walks(name, by_row, dev):
    import os
    old = os.environ.get("MOE_DISPATCH_BY_ROW")
    os.environ["MOE_DISPATCH_BY_ROW"] = by_row
    try:
        w = TOKEN_DISPATCH[name]
        _layer_vs_oracle(w, _host_inputs(w, seed=11), dev)
    finally:
        if old is None:
            os.environ.pop("MOE_DISPATCH_BY_ROW", None)
        else:
            os.environ["MOE_DISPATCH_BY_ROW"] = old


@pytest.mark.parametrize("name", ["mixtral_small", "qwen3_medium", "dsv3_medium", "gptoss_small"])
def test_layer_combine_one_vector_per_lane(name, dev):
    """MOE_COMBINE_VPL=1: the y16 combine with one 16-byte vector per lane
    per row (two for top-2; without a shared expert the defaults take four
    for top-2 and two for top-8, with one the same one)."""
    import os
    old = os.environ.get("MOE_COMBINE_VPL")
    os.environ["MOE_COMBINE_VPL"] = "1"
    try:
        test_layer_matches_oracle(name, dev)
    finally:
        if old is None:
            os.environ.pop("MOE_COMBINE_VPL", None)
        else:
            os.environ["MOE_COMBINE_VPL"] = old


@pytest.mark.parametrize("name", ["mixtral_small", "qwen3_medium", "dsv3_medium", "gptoss_small",
                                  "mixtral_decode_small"])
def test_layer_same_with_and_without_dependent_launch(name, dev):
    """MOE_PDL=0 launches every kernel in plain stream order; by default each
    launch overlaps the previous kernel's tail, and every kernel waits for
    its predecessor before it touches memory.  The outputs and routing must
    be the same bit for bit."""
    import os
    w = SMALL[name]
    hin = _host_inputs(w, seed=5)
    inp = gpu_inputs(w, 0, dev, hin)
    old = os.environ.get("MOE_PDL")
    try:
        os.environ["MOE_PDL"] = "0"
        plain, rb0 = run_layer(w, inp)
        os.environ.pop("MOE_PDL", None)
        pdl, rb1 = run_layer(w, inp)
    finally:
        if old is None:
            os.environ.pop("MOE_PDL", None)
        else:
            os.environ["MOE_PDL"] = old
    assert torch.equal(plain, pdl)
    for k in ("logits", "topk_idx", "topk_w", "slot_row", "offsets"):
        assert torch.equal(rb0[k], rb1[k]), k
    R = int(rb0["offsets"][-1])  # row_src holds the kept rows only
    assert torch.equal(rb0["row_src"][:R], rb1["row_src"][:R])


@pytest.fixture
def fused_dispatch():
    import os
    old = os.environ.get("MOE_FUSED_DISPATCH")
    os.environ["MOE_FUSED_DISPATCH"] = "1"
    yield
    if old is None:
        os.environ.pop("MOE_FUSED_DISPATCH", None)
    else:
        os.environ["MOE_FUSED_DISPATCH"] = old


@pytest.mark.parametrize("name", BF16_SMALL)
def test_layer_with_dispatch_fused_into_gemm(name, fused_dispatch, dev):
    """The layer with the up projection gathering token rows itself (TMA gather4)."""
    test_layer_matches_oracle(name, dev)


@pytest.mark.parametrize("name", ["mixtral_small", "dsv3_small", "gptoss_small"])
def test_fused_dispatch_each_engine(name, fused_dispatch, gemm_engine, dev):
    test_layer_matches_oracle(name, dev)


# ---------------------------------------------------------------------------
# Gate weights applied by the down projection's epilogue (combine only sums)
# ---------------------------------------------------------------------------
@pytest.fixture
def weights_in_gemm():
    import os
    old = os.environ.get("MOE_WEIGHTS_IN_GEMM")
    os.environ["MOE_WEIGHTS_IN_GEMM"] = "1"
    yield
    if old is None:
        os.environ.pop("MOE_WEIGHTS_IN_GEMM", None)
    else:
        os.environ["MOE_WEIGHTS_IN_GEMM"] = old


@pytest.mark.parametrize("name", BF16_SMALL)
def test_layer_with_weights_in_gemm(name, weights_in_gemm, dev):
    test_layer_matches_oracle(name, dev)


@pytest.mark.parametrize("name", ["mixtral_small", "dsv3_small", "qwen3_small",
                                  "mixtral_decode_small"])
def test_weights_in_gemm_each_engine(name, weights_in_gemm, gemm_engine, dev):
    test_layer_matches_oracle(name, dev)


@pytest.mark.parametrize("name", ["t128_dsv3_ragged_k", "e1024_k32_drops"])
def test_small_batch_layer_with_weights_in_gemm(name, weights_in_gemm, dev):
    test_small_batch_layer(name, dev)
