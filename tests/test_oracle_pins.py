"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these compares the oracle with itself: each check is a hand-derived
worked example (tests/golden), a closed form, an invariant of the definition,
brute force over a tiny input, or a special case that reduces to a library
routine (torch fp64 matmul).  They run on the CPU only.
"""
import itertools
import json
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from routing_dispatch_expert_sigmoid_b200.workloads import WORKLOADS, make_inputs, to_numpy

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return json.load(fh)


# --------------------------------------------------------------------------
# Specified fp32 exp / sigmoid (Cody-Waite reduction + degree-7 Taylor)
# --------------------------------------------------------------------------
def _round_to_f32(fr: Fraction) -> float:
    """Exact round-to-nearest-even of a positive rational to binary32."""
    assert fr > 0
    e = math.floor(math.log2(fr.numerator) - math.log2(fr.denominator))
    while Fraction(2) ** e > fr:
        e -= 1
    while Fraction(2) ** (e + 1) <= fr:
        e += 1
    scale = Fraction(2) ** (23 - e)
    m = fr * scale
    lo = m.numerator // m.denominator
    rem = m - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return float(Fraction(lo) / scale)


def _ln2_fraction() -> Fraction:
    getcontext().prec = 60
    return Fraction(Decimal(2).ln())


def test_spec_exp_constants_are_the_rounded_definitions():
    c = oracle.spec_constants().astype(np.float64)
    ln2 = _ln2_fraction()
    assert c[0] == _round_to_f32(1 / ln2)                      # LOG2E
    assert Fraction(c[1]) == Fraction(2839, 4096)               # LN2_HI: ln 2 to 12 bits
    assert abs(Fraction(c[1]) - ln2) < Fraction(1, 4096)
    assert c[2] == _round_to_f32(ln2 - Fraction(2839, 4096))    # LN2_LO
    for k in range(8):
        assert c[3 + k] == _round_to_f32(Fraction(1, math.factorial(k))), k


def _ulp32(v):
    v = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(v, np.finfo(np.float32).tiny)))
    return np.exp2(e - 23)


def test_spec_exp_within_one_ulp_of_exp():
    rng = np.random.default_rng(0)
    z = np.concatenate([np.linspace(-87.0, 87.0, 400001), rng.uniform(-87, 87, 200000),
                        rng.uniform(-1, 1, 200000), [0.0, 1.0, -1.0, 0.5, -0.5]])
    z = z.astype(np.float32)
    got = oracle.spec_expf(z).astype(np.float64)
    ref = np.exp(z.astype(np.float64))
    err_ulp = np.abs(got - ref) / _ulp32(ref)
    assert err_ulp.max() <= 1.0, err_ulp.max()
    assert oracle.spec_expf(np.float32([0.0]))[0] == 1.0


def test_spec_exp_clamps_to_normal_range():
    big = oracle.spec_expf(np.float32([200.0, 87.0]))
    assert big[0] == big[1] and np.isfinite(big[0])
    small = oracle.spec_expf(np.float32([-200.0, -87.0]))
    assert small[0] == small[1] and small[0] > 0


def test_spec_sigmoid_within_three_ulp_and_symmetric():
    z = np.linspace(-30, 30, 300001).astype(np.float32)
    got = oracle.spec_sigmoidf(z).astype(np.float64)
    zd = z.astype(np.float64)
    ref = 1.0 / (1.0 + np.exp(-zd))
    err = np.abs(got - ref) / _ulp32(ref)
    assert err.max() <= 3.0, err.max()
    assert oracle.spec_sigmoidf(np.float32([0.0]))[0] == 0.5
    # sigma(z) + sigma(-z) = 1 up to rounding
    s = got + oracle.spec_sigmoidf(-z).astype(np.float64)
    assert np.abs(s - 1.0).max() < 3e-7


# --------------------------------------------------------------------------
# Gating
# --------------------------------------------------------------------------
@pytest.mark.parametrize("case", _load("gating_worked_example.json")["cases"],
                         ids=lambda c: c["name"])
def test_gating_worked_examples(case):
    logits = np.float32([[math.log(a) for a in case["logits_ln"]]])
    kw = {}
    if case["mode"] == "sigmoid_grouped":
        kw = dict(sel_bias=np.float32(case["sel_bias"]), n_groups=case["n_groups"],
                  topk_groups=case["topk_groups"], group_score_topk=case["group_score_topk"],
                  routed_scale=case["routed_scale"])
    idx, w = oracle.gating(logits, case["k"], case["mode"], **kw)
    assert idx[0].tolist() == case["expect_idx"]
    np.testing.assert_allclose(w[0], case["expect_w"], rtol=2e-6)


def _rank_select(key, k):
    """Slot j holds the expert whose rank is j, rank(e) = #{e' ahead of e}."""
    E = len(key)
    rank = [sum(1 for q in range(E) if key[q] > key[e] or (key[q] == key[e] and q < e))
            for e in range(E)]
    return [rank.index(j) for j in range(k)]


@pytest.mark.parametrize("mode", ["topk_softmax", "softmax_topk_renorm"])
def test_gating_brute_force_with_ties(mode):
    rng = np.random.default_rng(1)
    for E in (1, 2, 5, 8):
        for k in range(1, E + 1):
            logits = rng.integers(-1, 2, size=(64, E)).astype(np.float32)
            idx, w = oracle.gating(logits, k, mode)
            for t in range(64):
                assert idx[t].tolist() == _rank_select(logits[t].tolist(), k)
                # softmax weights: sum to 1, ratios are exp of logit gaps
                assert abs(w[t].sum() - 1.0) < 1e-12
                l = logits[t, idx[t]].astype(np.float64)
                np.testing.assert_allclose(w[t] / w[t, 0], np.exp(l - l[0]), rtol=1e-12)


def test_gating_variable_k_pads():
    rng = np.random.default_rng(2)
    logits = rng.standard_normal((50, 12)).astype(np.float32)
    kt = rng.integers(1, 7, size=50).astype(np.int32)
    idx, w = oracle.gating(logits, 6, "topk_softmax", k_per_token=kt)
    for t in range(50):
        assert idx[t, : kt[t]].tolist() == _rank_select(logits[t].tolist(), int(kt[t]))
        assert (idx[t, kt[t]:] == -1).all() and (w[t, kt[t]:] == 0).all()
        assert abs(w[t].sum() - 1.0) < 1e-12


def _grouped_brute(l32, bias, n_groups, topk_groups, k, scale):
    """Group-limited selection by enumeration over every set of kept groups."""
    E = l32.size
    gs = E // n_groups
    s = oracle.spec_sigmoidf(l32)
    u = (s + bias).astype(np.float32)
    # score of a group: the largest fp32 sum over pairs of its members
    score = []
    for g in range(n_groups):
        mem = u[g * gs:(g + 1) * gs]
        score.append(max(np.float32(mem[i]) + np.float32(mem[j])
                         for i in range(gs) for j in range(gs) if i != j))
    chosen = None
    for sub in itertools.combinations(range(n_groups), topk_groups):
        rest = [g for g in range(n_groups) if g not in sub]
        if all(score[a] > score[b] or (score[a] == score[b] and a < b)
               for a in sub for b in rest):
            assert chosen is None
            chosen = sub
    cand = [e for e in range(E) if e // gs in chosen]
    keys = [float(u[e]) if e in cand else -np.inf for e in range(E)]
    sel = _rank_select(keys, k)
    ssum = sum(float(s[e]) for e in sel)
    return sel, [scale * float(s[e]) / ssum for e in sel]


def test_gating_grouped_brute_force():
    rng = np.random.default_rng(3)
    for trial in range(300):
        E, n_groups = 16, 8
        l32 = rng.integers(-2, 3, size=E).astype(np.float32) * np.float32(0.5)
        bias = (rng.integers(-2, 3, size=E) * 0.125).astype(np.float32)
        topk_groups = int(rng.integers(1, n_groups + 1))
        k = int(rng.integers(1, 2 * topk_groups + 1))
        idx, w = oracle.gating(l32[None], k, "sigmoid_grouped", sel_bias=bias,
                               n_groups=n_groups, topk_groups=topk_groups,
                               group_score_topk=2, routed_scale=2.5)
        sel, ww = _grouped_brute(l32, bias, n_groups, topk_groups, k, 2.5)
        assert idx[0].tolist() == sel, trial
        np.testing.assert_allclose(w[0], ww, rtol=1e-12)
        assert abs(w[0].sum() - 2.5) < 1e-12


# --------------------------------------------------------------------------
# Capacity, histogram, prefix sum, dispatch layout
# --------------------------------------------------------------------------
@pytest.mark.parametrize("case", _load("capacity_worked_example.json")["cases"],
                         ids=lambda c: c["name"])
def test_capacity_worked_examples(case):
    r = oracle.capacity_dispatch(np.int32(case["topk_idx"]), case["E"], case["capacity_factor"])
    assert r["capacity"] == case["capacity"]
    for key in ("counts", "kept", "offsets", "slot_row", "row_src"):
        assert np.asarray(r[key]).tolist() == case[key], key
    assert r["n_dropped"] == case["n_dropped"]


def _check_layout(idx, E, cf, r):
    T, k_max = idx.shape
    sum_k = int((idx >= 0).sum())
    C = math.ceil(cf * sum_k / E) if cf > 0 else None
    # sum of counts = sum of k_t; kept = min(count, C); sum kept = sum k - drops
    assert r["counts"].sum() == sum_k
    exp_kept = r["counts"] if C is None else np.minimum(r["counts"], C)
    assert (r["kept"] == exp_kept).all()
    assert r["kept"].sum() == sum_k - r["n_dropped"]
    assert (np.diff(r["offsets"]) == r["kept"]).all() and r["offsets"][0] == 0
    R = int(r["offsets"][E])
    # the kept set of expert e is its first C assignments in (token, slot) order
    seen = np.zeros(E, np.int64)
    kept_slots = []
    for t in range(T):
        for j in range(k_max):
            e = idx[t, j]
            if e < 0:
                assert r["slot_row"][t, j] == -1
                continue
            keep = C is None or seen[e] < C
            seen[e] += 1
            assert (r["slot_row"][t, j] >= 0) == keep
            if keep:
                kept_slots.append(t * k_max + j)
    # row_src is a bijection onto kept slots, inverse of slot_row, sorted by
    # (expert, token, slot)
    assert sorted(r["row_src"].tolist()) == sorted(kept_slots) and len(r["row_src"]) == R
    for row, a in enumerate(r["row_src"]):
        assert r["slot_row"].ravel()[a] == row
    keys = [(idx.ravel()[a], a) for a in r["row_src"]]
    assert keys == sorted(keys)


@pytest.mark.parametrize("T,E,k,cf", [(1, 1, 1, 0.0), (7, 4, 2, 1.0), (100, 8, 2, 1.25),
                                      (300, 16, 4, 0.5), (64, 64, 8, 1.0), (33, 5, 5, 2.0)])
def test_capacity_invariants_random(T, E, k, cf):
    rng = np.random.default_rng(T * 131 + E)
    p = rng.dirichlet(np.ones(E) * 0.3)
    idx = np.empty((T, k), np.int32)
    for t in range(T):
        idx[t] = rng.choice(E, size=k, replace=False, p=p)
    r = oracle.capacity_dispatch(idx, E, cf)
    _check_layout(idx, E, cf, r)


def test_capacity_variable_k_and_empty():
    rng = np.random.default_rng(5)
    idx = np.full((40, 6), -1, np.int32)
    for t in range(40):
        kt = int(rng.integers(1, 7))
        idx[t, :kt] = rng.choice(10, size=kt, replace=False)
    for cf in (0.0, 0.7, 1.0):
        _check_layout(idx, 10, cf, oracle.capacity_dispatch(idx, 10, cf))
    empty = oracle.capacity_dispatch(np.zeros((0, 2), np.int32), 4, 1.0)
    assert empty["offsets"].tolist() == [0, 0, 0, 0, 0] and empty["n_dropped"] == 0


def test_dispatch_inverse_restores_token_rows():
    rng = np.random.default_rng(6)
    T, d, E, k = 50, 24, 6, 3
    x = rng.standard_normal((T, d)).astype(np.float32)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    r = oracle.capacity_dispatch(idx, E, 1.0)
    xp = oracle.dispatch(x, r["row_src"], k)
    for t in range(T):
        for j in range(k):
            row = r["slot_row"][t, j]
            if row >= 0:
                assert (xp[row] == x[t]).all()
    # bf16 bit patterns are copied unchanged
    xb = rng.integers(0, 2 ** 16, size=(T, d)).astype(np.uint16)
    xpb = oracle.dispatch(xb, r["row_src"], k)
    assert (xpb == xb[r["row_src"] // k]).all()


# --------------------------------------------------------------------------
# Router, FFN and the whole layer: special cases with a closed form
# --------------------------------------------------------------------------
def _t64(a):
    if a.dtype == np.uint16:
        a = (a.astype(np.uint32) << 16).view(np.float32)
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.float64)


def _dense_swiglu(x, W1, W3, W2):
    x, W1, W3, W2 = (_t64(a) for a in (x, W1, W3, W2))
    return (torch.nn.functional.silu(x @ W1) * (x @ W3) @ W2).numpy()


def test_router_logits_match_fp64_matmul():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((37, 48)).astype(np.float32)
    Wr = rng.standard_normal((48, 11)).astype(np.float32)
    b = rng.standard_normal(11).astype(np.float32)
    got = oracle.router_logits(x, Wr, b)
    ref = (_t64(x) @ _t64(Wr)).numpy() + b.astype(np.float64)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    xb = to_numpy(torch.from_numpy(x).to(torch.bfloat16))
    Wb = to_numpy(torch.from_numpy(Wr).to(torch.bfloat16))
    np.testing.assert_allclose(oracle.router_logits(xb, Wb), (_t64(xb) @ _t64(Wb)).numpy(),
                               rtol=1e-12, atol=1e-12)


def test_expert_ffn_matches_fp64_library_swiglu():
    rng = np.random.default_rng(8)
    n, d, f = 9, 20, 36          # d != f: a transposed operand cannot pass
    x = rng.standard_normal((n, d)).astype(np.float32)
    W1, W3 = (rng.standard_normal((d, f)).astype(np.float32) / 4 for _ in range(2))
    W2 = rng.standard_normal((f, d)).astype(np.float32) / 6
    np.testing.assert_allclose(oracle.expert_ffn(x, W1, W3, W2), _dense_swiglu(x, W1, W3, W2),
                               rtol=1e-11, atol=1e-12)


def _small_inputs(dtype, T, d, E, k, f, seed, fs=0):
    w = WORKLOADS["tiny_f32"].scaled(T=T, d=d, E=E, k_max=k, f=f, dtype=dtype, f_shared=fs,
                                     zipf_s=0.0, capacity_factor=0.0)
    return w, {key: to_numpy(v) for key, v in make_inputs(w, seed).items()}


@pytest.mark.parametrize("mode", ["topk_softmax", "softmax_topk_renorm"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_identical_experts_reduce_to_dense_ffn(mode, dtype):
    w, inp = _small_inputs(dtype, T=40, d=32, E=6, k=3, f=48, seed=9)
    W1 = np.repeat(inp["W1"][:1], w.E, 0)
    W3 = np.repeat(inp["W3"][:1], w.E, 0)
    W2 = np.repeat(inp["W2"][:1], w.E, 0)
    r = oracle.layer(inp["x"], inp["Wr"], W1, W3, W2, k_max=w.k_max, gating_mode=mode)
    dense = _dense_swiglu(inp["x"], W1[0], W3[0], W2[0])
    np.testing.assert_allclose(r["out"], dense, rtol=1e-10, atol=1e-12)


def test_grouped_sigmoid_identical_experts_give_scaled_ffn_plus_shared():
    w, inp = _small_inputs("bf16", T=30, d=32, E=16, k=4, f=40, seed=10, fs=24)
    W1 = np.repeat(inp["W1"][:1], w.E, 0)
    W3 = np.repeat(inp["W3"][:1], w.E, 0)
    W2 = np.repeat(inp["W2"][:1], w.E, 0)
    bias = np.random.default_rng(0).normal(0, 0.05, w.E).astype(np.float32)
    r = oracle.layer(inp["x"], inp["Wr"], W1, W3, W2, k_max=4, gating_mode="sigmoid_grouped",
                     sel_bias=bias, n_groups=4, topk_groups=2, group_score_topk=2,
                     routed_scale=2.5, Ws1=inp["Ws1"], Ws3=inp["Ws3"], Ws2=inp["Ws2"])
    ref = 2.5 * _dense_swiglu(inp["x"], W1[0], W3[0], W2[0]) + _dense_swiglu(
        inp["x"], inp["Ws1"], inp["Ws3"], inp["Ws2"])
    np.testing.assert_allclose(r["out"], ref, rtol=1e-10, atol=1e-12)


def test_k_equals_E_with_uniform_gates_is_mean_of_experts():
    w, inp = _small_inputs("f32", T=12, d=16, E=5, k=5, f=24, seed=11)
    Wr = np.zeros_like(inp["Wr"])             # equal logits: every expert, weight 1/E
    r = oracle.layer(inp["x"], Wr, inp["W1"], inp["W3"], inp["W2"], k_max=5)
    assert (np.sort(r["topk_idx"], axis=1) == np.arange(5)).all()
    np.testing.assert_allclose(r["topk_w"], 0.2, rtol=1e-15)
    mean = sum(_dense_swiglu(inp["x"], inp["W1"][e], inp["W3"][e], inp["W2"][e])
               for e in range(5)) / 5
    np.testing.assert_allclose(r["out"], mean, rtol=1e-10, atol=1e-12)


def test_sub_experts_sum_to_parent_expert():
    """Disjoint neuron partitions: 4 sub-experts at equal gates g = g * parent FFN."""
    rng = np.random.default_rng(12)
    T, d, f = 10, 16, 32
    x = rng.standard_normal((T, d)).astype(np.float32)
    P1, P3 = (rng.standard_normal((d, f)).astype(np.float32) / 4 for _ in range(2))
    P2 = rng.standard_normal((f, d)).astype(np.float32) / 5
    fq = f // 4
    W1 = np.stack([P1[:, q * fq:(q + 1) * fq] for q in range(4)])
    W3 = np.stack([P3[:, q * fq:(q + 1) * fq] for q in range(4)])
    W2 = np.stack([P2[q * fq:(q + 1) * fq, :] for q in range(4)])
    r = oracle.layer(x, np.zeros((d, 4), np.float32), W1, W3, W2, k_max=4)
    np.testing.assert_allclose(r["out"], 0.25 * _dense_swiglu(x, P1, P3, P2), rtol=1e-10,
                               atol=1e-12)


def test_zero_input_and_single_expert():
    w, inp = _small_inputs("f32", T=8, d=16, E=1, k=1, f=24, seed=13)
    r = oracle.layer(np.zeros_like(inp["x"]), inp["Wr"], inp["W1"], inp["W3"], inp["W2"],
                     k_max=1)
    assert (r["out"] == 0).all()
    r = oracle.layer(inp["x"], inp["Wr"], inp["W1"], inp["W3"], inp["W2"], k_max=1)
    np.testing.assert_allclose(r["out"], _dense_swiglu(inp["x"], inp["W1"][0], inp["W3"][0],
                                                       inp["W2"][0]), rtol=1e-10, atol=1e-12)


def test_dropped_slots_contribute_nothing():
    w, inp = _small_inputs("f32", T=64, d=16, E=4, k=2, f=20, seed=14)
    r = oracle.layer(inp["x"], inp["Wr"], inp["W1"], inp["W3"], inp["W2"], k_max=2,
                     capacity_factor=0.5, logit_bias=np.float32([3, 0, 0, 0]))
    assert r["n_dropped"] > 0
    for t in range(w.T):
        ref = np.zeros(w.d)
        for j in range(2):
            if r["slot_row"][t, j] >= 0:
                e = r["topk_idx"][t, j]
                ref += r["topk_w"][t, j] * _dense_swiglu(inp["x"][t:t + 1], inp["W1"][e],
                                                         inp["W3"][e], inp["W2"][e])[0]
        np.testing.assert_allclose(r["out"][t], ref, rtol=1e-10, atol=1e-12)


def test_combine_worked_example():
    g = _load("combine_worked_example.json")
    y = np.float32(g["y_perm"])
    sr = np.int32(g["slot_row"])
    w = np.float64(g["topk_w"])
    assert oracle.combine_rows(w, sr, y).tolist() == g["expect_no_shared"]
    assert oracle.combine_rows(w, sr, y, np.float32(g["shared"])).tolist() == \
        g["expect_with_shared"]
    km = (sr >= 0).astype(np.int32)
    ys = np.where(km[..., None] > 0, y[np.maximum(sr, 0)], 0).astype(np.float64)
    assert oracle.combine(w, km, ys).tolist() == g["expect_no_shared"]


# --------------------------------------------------------------------------
# FP8 expert weights: e4m3 codes, per-output-column scales
# --------------------------------------------------------------------------
def _bf16_bits(a) -> np.ndarray:
    return to_numpy(torch.as_tensor(np.asarray(a, np.float32)).to(torch.bfloat16))


def test_e4m3_decode_known_codes():
    """Values fixed by the format: bias 7, 3 fraction bits, subnormals m*2^-9,
    the all-ones exponent-and-fraction code is NaN, no infinity."""
    code = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
            0x38: 1.0, 0x39: 1.125, 0x3C: 1.5, 0x40: 2.0, 0x77: 240.0, 0x78: 256.0,
            0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0}
    v = oracle.e4m3_decode(np.array(list(code), np.uint8))
    assert v.tolist() == list(code.values())
    assert np.isnan(oracle.e4m3_decode(np.uint8([0x7F, 0xFF]))).all()
    neg0 = oracle.e4m3_decode(np.uint8([0x80]))[0]
    assert neg0 == 0.0 and math.copysign(1.0, neg0) == -1.0
    pos = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    assert (np.diff(pos) > 0).all()                      # codes 0..126 increase
    assert (oracle.e4m3_decode(np.arange(0x80, 0xFF, dtype=np.uint8)) == -pos).all()


def test_e4m3_encode_round_trip_ties_and_saturation():
    c = np.arange(256, dtype=np.uint8)
    v = oracle.e4m3_decode(c)
    fin = ~np.isnan(v)
    assert (oracle.e4m3_encode(v[fin].astype(np.float32)) == c[fin]).all()
    pos = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mid = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)  # exact in float32
    got = oracle.e4m3_encode(mid).astype(int)
    lower = np.arange(0x7E)
    assert (got == np.where(lower % 2 == 0, lower, lower + 1)).all()  # ties to even
    up = np.nextafter(mid, np.float32(np.inf))
    dn = np.nextafter(mid, np.float32(0))
    assert (oracle.e4m3_encode(up).astype(int) == lower + 1).all()
    assert (oracle.e4m3_encode(dn).astype(int) == lower).all()
    sat = oracle.e4m3_encode(np.float32([449, 464, 1e6, 3e38, -500, -np.inf, np.inf]))
    assert sat.tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7E]
    assert oracle.e4m3_encode(np.float32([np.nan]))[0] == 0x7F
    assert oracle.e4m3_encode(np.float32([-0.0]))[0] == 0x80


def test_e4m3_encode_matches_library_conversion_in_range():
    """Inside the finite range, round-to-nearest-even to e4m3 is what torch's
    float8_e4m3fn conversion does (out of range it saturates here, NaN there)."""
    g = torch.Generator().manual_seed(21)
    x = torch.cat([torch.randn(200000, generator=g) * s for s in (1e-3, 0.05, 1.0, 60.0)])
    x = x[x.abs() < 448]
    lib = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (oracle.e4m3_encode(x.numpy()) == lib).all()


def test_quantize_fp8_per_column_scales_and_error_bound():
    rng = np.random.default_rng(22)
    G, K, N = 3, 40, 24
    W = rng.standard_normal((G, K, N)).astype(np.float32) * rng.uniform(0.01, 3, (G, 1, N))
    W[1, :, 5] = 0.0                                       # an all-zero column
    Wb = _bf16_bits(W)
    q, s = oracle.quantize_fp8(Wb)
    Wf = torch.from_numpy(Wb.astype(np.int32) << 16).view(torch.float32).numpy()
    amax = np.abs(Wf).max(axis=1)
    exp_s = np.where(amax > 0, (amax / np.float32(448)).astype(np.float32), np.float32(1))
    assert (s == exp_s).all()
    assert (q[1, :, 5] == 0).all() and s[1, 5] == 1.0
    # the largest magnitude of every column maps to the largest code
    kmax = np.abs(Wf).argmax(axis=1)
    top = np.take_along_axis(q, kmax[:, None, :], axis=1)[:, 0, :]
    nz = amax > 0
    assert ((top[nz] & 0x7F) == 0x7E).all()
    # dequantised weights are within half a grid step of the weight
    deq = oracle.dequantize_fp8(q, s)
    qv = Wf / s[:, None, :]
    step = np.where(np.abs(qv) < 2.0 ** -6, 2.0 ** -9,
                    2.0 ** (np.floor(np.log2(np.maximum(np.abs(qv), 1e-30))) - 3))
    assert (np.abs(deq - Wf) <= 0.5 * step * s[:, None, :] * (1 + 1e-6)).all()


def test_fp8_layer_equals_layer_on_representable_weights():
    """Weights that are e4m3 values times a power-of-two column scale with the
    column maximum at 448 * scale quantise exactly, so the layer on the
    dequantised fp64 weights equals the layer on the bf16 weights."""
    w, inp = _small_inputs("bf16", T=20, d=32, E=4, k=2, f=48, seed=23, fs=16)
    rng = np.random.default_rng(24)
    grid = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))

    def representable(shape):
        v = rng.choice(np.concatenate([grid, -grid]), size=shape)
        G, K, N = shape
        v[:, 0, :] = 448.0                              # column maximum
        scale = 2.0 ** rng.integers(-12, -6, size=(G, 1, N))
        return _bf16_bits(v * scale)

    Wq = {k: representable(inp[k].shape) for k in ("W1", "W3", "W2")}
    Sq = {k: representable((1,) + inp[k].shape) for k in ("Ws1", "Ws3", "Ws2")}
    deq = {k: oracle.dequantize_fp8(*oracle.quantize_fp8(v)) for k, v in Wq.items()}
    sdeq = {k: oracle.dequantize_fp8(*oracle.quantize_fp8(v))[0] for k, v in Sq.items()}
    for k, v in Wq.items():  # the quantisation is exact
        assert (deq[k] == torch.from_numpy(v.astype(np.int32) << 16).view(torch.float32)
                .numpy()).all()
    r = oracle.layer(inp["x"], inp["Wr"], Wq["W1"], Wq["W3"], Wq["W2"], k_max=2,
                     Ws1=Sq["Ws1"][0], Ws3=Sq["Ws3"][0], Ws2=Sq["Ws2"][0])
    tok = np.arange(w.T)
    got = oracle.layer_tokens(tok, inp["x"], deq["W1"], deq["W3"], deq["W2"], r["topk_idx"],
                              r["topk_w"], r["slot_row"], sdeq["Ws1"], sdeq["Ws3"],
                              sdeq["Ws2"])
    assert (got == r["out"]).all()
