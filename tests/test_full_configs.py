"""Every workload at its full size, through moe_layer (the call bench.py times).

Routing, counts, drops and the dispatch layout are compared bit for bit over
all tokens (oracle fed the GPU's fp32 logits).  Logits are checked on a sample
of tokens against fp64, and layer outputs on a sample of tokens (first, last,
and seeded random ones) against the oracle, which only needs the weights of
the experts those tokens use.
"""
import gc

import numpy as np
import pytest
import torch

import oracle
from parity import (assert_logits_close, assert_out_close, check_routing_bit_exact, f64,
                    oracle_layer_on_tokens, run_layer, storage)
from routing_dispatch_expert_sigmoid_b200 import ops
from routing_dispatch_expert_sigmoid_b200.workloads import WORKLOADS, make_inputs, to_numpy

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()
    return torch.device("cuda:0")


def _sample(T, n, seed=0):
    rng = np.random.default_rng(seed)
    pick = {0, T - 1} | set(rng.integers(0, T, size=max(n - 2, 0)).tolist())
    return sorted(pick)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_full_size_workload(name, dev):
    w = WORKLOADS[name]
    inp = make_inputs(w, seed=0, device=dev)
    out, rb = run_layer(w, inp)
    hin = {k: (None if v is None else v) for k, v in inp.items()}
    routing = check_routing_bit_exact(w, {"sel_bias": hin["sel_bias"],
                                          "k_per_token": hin["k_per_token"]}, rb)
    toks = _sample(w.T, 8 if w.T > 8 else w.T)
    sel = torch.tensor(toks, device=dev, dtype=torch.long)
    ref_logits = oracle.router_logits(to_numpy(inp["x"].index_select(0, sel)),
                                      to_numpy(inp["Wr"]), to_numpy(inp["logit_bias"]))
    assert_logits_close(rb["logits"].index_select(0, sel), ref_logits)
    ref = oracle_layer_on_tokens(inp, routing, toks)
    assert_out_close(f64(out.index_select(0, sel)), ref, f"{name} sampled outputs", storage(w))
    # the kept-row count matches the stated drop policy
    assert int(rb["offsets"][-1].item()) == int(rb["counts"].sum().item()) - int(
        rb["n_dropped"].item())
    del inp, out, rb
    gc.collect()
    torch.cuda.empty_cache()
