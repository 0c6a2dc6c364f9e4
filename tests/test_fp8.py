"""FP8 expert weights on the GPU against the oracle.

The experts' matrices are e4m3 codes with one fp32 scale per output column
("LLM MoE Expert Parallel 生产实战", sections 5 and 10: fp8 serving with the
router head left in precision).  Checks:
  - the library's quantiser gives the oracle's codes and scales bit for bit;
  - the layer and the expert FFN on fp8 weights match the oracle run on its
    own quantisation of the same bf16 weights (dequantised exactly in fp64),
    within the output tolerances of tests/parity.py; the routing is bit-exact
    as for bf16 weights.
Shapes cross tile edges with ragged tails in N (f or d = 16 mod 32) and K.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import (assert_out_close, check_routing_bit_exact, f64, gpu_inputs, run_route,
                    storage)
from routing_dispatch_expert_sigmoid_b200 import ops
from routing_dispatch_expert_sigmoid_b200.workloads import WORKLOADS, make_inputs, to_numpy

pytestmark = pytest.mark.gpu

CASES = {
    "mixtral_small": WORKLOADS["mixtral_prefill"].scaled(T=300, d=256, f=384),
    "mixtral_decode_small": WORKLOADS["mixtral_decode"].scaled(T=5, d=512, f=1024),
    # N of both projections 16 mod 32 (ragged scale chunk), K = 400 not a multiple of 64
    "ragged_n_k": WORKLOADS["mixtral_prefill"].scaled(T=200, d=272, f=400),
    "qwen3_small": WORKLOADS["qwen3_prefill"].scaled(T=257, d=192, E=16, k_max=4, f=208),
    "dsv3_small": WORKLOADS["dsv3_prefill"].scaled(T=130, d=256, E=64, f=144, f_shared=80),
    # decode-sized batch: the shared expert split along K (8 up, 2 down splits)
    "dsv3_decode_shared_split": WORKLOADS["dsv3_decode"].scaled(T=100, d=512, E=64, f=144,
                                                                f_shared=128),
    "gptoss_small": WORKLOADS["gptoss_sub"].scaled(T=211, d=208, E=32, k_max=6, k_min=2, f=80),
    # capacity drops (a quarter of the slots kept), renormalised softmax
    "qwen3_heavy_drops": WORKLOADS["qwen3_prefill"].scaled(T=150, d=192, E=16, k_max=4, f=208,
                                                           capacity_factor=0.25),
    # one expert, k = 1: the dense FFN on fp8 weights
    "single_expert": WORKLOADS["mixtral_prefill"].scaled(T=77, d=256, E=1, k_max=1, f=384,
                                                         zipf_s=0.0),
    # decode-sized layers (the kind::f8f6f4 engine by default): N of both
    # projections 16 mod 128 and K not a multiple of the 128-deep k-block
    "f8_decode_ragged": WORKLOADS["mixtral_decode"].scaled(T=40, d=272, f=400),
    # one hot expert holding several 64-row tiles
    "f8_decode_hot_expert": WORKLOADS["mixtral_decode"].scaled(T=128, d=256, f=320, zipf_s=3.0),
    # 256 experts, a row or two each, group-limited sigmoid routing
    "f8_decode_many_experts": WORKLOADS["dsv3_decode"].scaled(T=64, d=384, E=256, f=144,
                                                              f_shared=0),
}


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()
    return torch.device("cuda:0")


@pytest.fixture(params=["default", "single", "narrow", "swap"])
def fp8_engine(request):
    """default: swap-AB for decode-sized groups, single-CTA tiles otherwise;
    the others force one engine on every GEMM of the layer."""
    import os
    old = os.environ.get("MOE_GEMM_ENGINE")
    if request.param == "default":
        os.environ.pop("MOE_GEMM_ENGINE", None)
    else:
        os.environ["MOE_GEMM_ENGINE"] = request.param
    yield request.param
    if old is None:
        os.environ.pop("MOE_GEMM_ENGINE", None)
    else:
        os.environ["MOE_GEMM_ENGINE"] = old


def _oracle_set(hin, keys):
    """The oracle's quantisation of host bf16 weights, dequantised in fp64."""
    out = {}
    for k in keys:
        W = to_numpy(hin[k])
        q, s = oracle.quantize_fp8(W if W.ndim == 3 else W[None])
        out[k] = (q, s, oracle.dequantize_fp8(q, s))
    return out


def _assert_same_quantisation(gpu_set, oracle_set, names):
    for k in names:
        q, s, _ = oracle_set[k]
        gq = gpu_set["W" + k[-1]].cpu().numpy()  # a set's keys: W1 W3 W2 s1 s3 s2
        gs = gpu_set["s" + k[-1]].cpu().numpy()
        gq, gs = (gq, gs) if gq.ndim == 3 else (gq[None], gs[None])
        gq = gq.swapaxes(1, 2)  # the library stores the codes K-contiguous
        assert (gq == q).all(), f"{k}: codes differ at {np.argwhere(gq != q)[:3].tolist()}"
        assert (gs == s).all(), f"{k}: scales differ"


def test_quantizer_matches_oracle_bit_for_bit(dev):
    g = torch.Generator().manual_seed(31)
    W = torch.randn(3, 112, 48, generator=g) * torch.rand(3, 1, 48, generator=g) * 4
    W[0, :, 7] = 0                            # all-zero column: scale 1, codes 0
    W[1, 3, 9] = 3e4                          # one large weight dominates its column
    W[2, :, 11] = 1e-39                       # subnormal in fp32 and bf16
    Wb = W.to(torch.bfloat16)
    q, s = ops.moe_quantize_fp8(Wb.to(dev))
    oq, os_ = oracle.quantize_fp8(to_numpy(Wb))
    # the library stores the codes transposed ([G, N, K]); the values must match
    assert q.shape == (3, 48, 112)
    assert (q.cpu().numpy().swapaxes(1, 2) == oq).all() and (s.cpu().numpy() == os_).all()
    # a 2-D matrix is one group
    q2, s2 = ops.moe_quantize_fp8(Wb[1].to(dev))
    assert (q2.cpu().numpy().T == oq[1]).all() and (s2.cpu().numpy() == os_[1]).all()


@pytest.mark.parametrize("name", list(CASES))
def test_fp8_layer_matches_oracle(name, fp8_engine, dev):
    w = CASES[name]
    hin = make_inputs(w, 0, device="cpu")
    inp = gpu_inputs(w, 0, dev, hin)
    experts = ops.fp8_weight_set(inp["W1"], inp["W3"], inp["W2"])
    shared = (ops.fp8_weight_set(inp["Ws1"], inp["Ws3"], inp["Ws2"]) if w.f_shared else None)
    ref_sets = _oracle_set(hin, ("W1", "W3", "W2"))
    _assert_same_quantisation(experts, ref_sets, ("W1", "W3", "W2"))
    cfg = ops.config(w)
    ws = ops.workspace(cfg, ops.WS_LAYER)
    out = torch.empty_like(inp["x"])
    rb = ops.route_buffers(cfg)
    ops.moe_layer_fp8(cfg, inp["x"], inp["Wr"], inp["logit_bias"], inp["sel_bias"],
                      inp["k_per_token"], experts, shared, out, rb, ws)
    ops.moe_check_errors()
    routing = check_routing_bit_exact(w, hin, rb)
    sh = [None] * 3
    if w.f_shared:
        sets = _oracle_set(hin, ("Ws1", "Ws3", "Ws2"))
        _assert_same_quantisation(shared, sets, ("Ws1", "Ws3", "Ws2"))
        sh = [sets[k][2][0] for k in ("Ws1", "Ws3", "Ws2")]
    ref = oracle.layer_tokens(np.arange(w.T, dtype=np.int32), to_numpy(hin["x"]),
                              ref_sets["W1"][2], ref_sets["W3"][2], ref_sets["W2"][2],
                              routing["topk_idx"], routing["topk_w"], routing["slot_row"], *sh)
    assert_out_close(f64(out), ref, "fp8 layer out", storage(w))


@pytest.mark.parametrize("name", ["mixtral_small", "ragged_n_k", "gptoss_small"])
def test_fp8_expert_ffn_matches_oracle(name, dev):
    """Grouped FFN alone on fp8 weights, on the oracle's dispatched rows and layout."""
    w = CASES[name]
    hin = make_inputs(w, 1, device="cpu")
    inp = gpu_inputs(w, 1, dev, hin)
    cfg, out = run_route(w, inp)
    lay = check_routing_bit_exact(w, hin, out)
    R = int(lay["offsets"][-1])
    xp = oracle.dispatch(to_numpy(hin["x"]), lay["row_src"], w.k_max)
    x_perm = torch.zeros((w.T * w.k_max, w.d), dtype=inp["x"].dtype)
    x_perm[:R] = hin["x"][torch.from_numpy(lay["row_src"] // w.k_max).long()]
    assert (to_numpy(x_perm[:R]) == xp).all()
    x_perm = x_perm.to(dev)
    experts = ops.fp8_weight_set(inp["W1"], inp["W3"], inp["W2"])
    sets = _oracle_set(hin, ("W1", "W3", "W2"))
    _assert_same_quantisation(experts, sets, ("W1", "W3", "W2"))
    y = torch.zeros((w.T * w.k_max, w.d), dtype=torch.float32, device=dev)
    offs = torch.from_numpy(lay["offsets"]).to(dev)
    ops.moe_expert_ffn_fp8(cfg, x_perm, offs, experts, y, ops.workspace(cfg, ops.WS_EXPERT_FFN))
    ops.moe_check_errors()
    ref = oracle.grouped_ffn(xp, lay["offsets"], sets["W1"][2], sets["W3"][2], sets["W2"][2])
    assert_out_close(f64(y[:R]), ref, "fp8 expert FFN", "f32")


@pytest.mark.parametrize("T", [192, 64])
def test_fp8_every_code_through_the_ffn(T, fp8_engine, dev):
    """Codes drawn uniformly from every finite e4m3 code (subnormals, both
    zeros and the largest magnitude included) with random column scales: the
    widening to bf16 in shared memory, or the tensor cores' own e4m3 inputs
    (T = 64: 21 rows per expert, the kind::f8f6f4 engine), must give each
    code's exact value."""
    w = WORKLOADS["mixtral_prefill"].scaled(T=T, d=256, E=3, k_max=1, f=384)
    cfg = ops.config(w)
    g = np.random.default_rng(41)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    sets = {}
    for k, (K, N) in (("W1", (w.d, w.f)), ("W3", (w.d, w.f)), ("W2", (w.f, w.d))):
        q = g.choice(finite, size=(w.E, K, N)).astype(np.uint8)
        sc = (g.uniform(0.5, 2.0, (w.E, N)) / (448 * np.sqrt(K))).astype(np.float32)
        sets[k] = (q, sc)
    gpu = {}
    for k, (q, sc) in sets.items():  # the library takes the codes K-contiguous
        gpu[k] = torch.from_numpy(np.ascontiguousarray(q.swapaxes(1, 2))).to(dev)
        gpu["s" + k[-1]] = torch.from_numpy(sc).to(dev)
    offsets = np.array([0, T // 4, T // 4, T], np.int32)  # an empty expert in the middle
    xb = torch.randn(T, w.d, generator=torch.Generator().manual_seed(42)).to(torch.bfloat16)
    y = torch.zeros((T, w.d), dtype=torch.float32, device=dev)
    ops.moe_expert_ffn_fp8(cfg, xb.to(dev), torch.from_numpy(offsets).to(dev), gpu, y,
                           ops.workspace(cfg, ops.WS_EXPERT_FFN))
    ops.moe_check_errors()
    deq = {k: oracle.dequantize_fp8(q, sc) for k, (q, sc) in sets.items()}
    ref = oracle.grouped_ffn(to_numpy(xb), offsets, deq["W1"], deq["W3"], deq["W2"])
    assert_out_close(f64(y), ref, "fp8 FFN over every code", "f32")


def test_fp8_empty_batch_is_a_no_op(dev):
    w = CASES["dsv3_small"]
    inp = make_inputs(w.scaled(T=1), 0, device=dev)
    cfg = ops.config(w, T=0)
    experts = ops.fp8_weight_set(inp["W1"], inp["W3"], inp["W2"])
    shared = ops.fp8_weight_set(inp["Ws1"], inp["Ws3"], inp["Ws2"])
    out = torch.empty((0, w.d), dtype=inp["x"].dtype, device=dev)
    ops.moe_layer_fp8(cfg, inp["x"][:0], inp["Wr"], None, inp["sel_bias"], None, experts, shared,
                      out, None, ops.workspace(cfg, ops.WS_LAYER))
    ops.moe_check_errors()


@pytest.mark.parametrize("name", ["mixtral_decode_small", "dsv3_small", "qwen3_heavy_drops"])
def test_fp8_layer_with_weights_in_gemm(name, fp8_engine, dev):
    """Gate weights applied by the down projection's epilogue on fp8 weights."""
    import os
    old = os.environ.get("MOE_WEIGHTS_IN_GEMM")
    os.environ["MOE_WEIGHTS_IN_GEMM"] = "1"
    try:
        test_fp8_layer_matches_oracle(name, fp8_engine, dev)
    finally:
        if old is None:
            os.environ.pop("MOE_WEIGHTS_IN_GEMM", None)
        else:
            os.environ["MOE_WEIGHTS_IN_GEMM"] = old


@pytest.mark.parametrize("name", ["mixtral_decode_small", "f8_decode_ragged",
                                  "f8_decode_many_experts"])
def test_fp8_layer_with_code_prefetch(name, dev):
    """MOE_F8_PREFETCH=3: the kind::f8f6f4 engine prefetches code tiles into L2."""
    import os
    old = os.environ.get("MOE_F8_PREFETCH")
    os.environ["MOE_F8_PREFETCH"] = "3"
    try:
        test_fp8_layer_matches_oracle(name, "default", dev)
    finally:
        if old is None:
            os.environ.pop("MOE_F8_PREFETCH", None)
        else:
            os.environ["MOE_F8_PREFETCH"] = old


@pytest.mark.parametrize("name", ["mixtral_decode_small", "f8_decode_ragged",
                                  "f8_decode_hot_expert", "f8_decode_many_experts"])
def test_fp8_layer_with_rotated_k_order(name, dev):
    """MOE_F8_KSTAGGER=1: each CTA of the kind::f8f6f4 engine walks the
    k-blocks of its tiles from its own starting block."""
    import os
    old = os.environ.get("MOE_F8_KSTAGGER")
    os.environ["MOE_F8_KSTAGGER"] = "1"
    try:
        test_fp8_layer_matches_oracle(name, "default", dev)
    finally:
        if old is None:
            os.environ.pop("MOE_F8_KSTAGGER", None)
        else:
            os.environ["MOE_F8_KSTAGGER"] = old
