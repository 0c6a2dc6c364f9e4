"""Every workload at its full size, through moe_layer (the call bench.py times).

Routing, counts, drops and the dispatch layout are compared bit for bit over
all tokens (oracle fed the GPU's fp32 logits).  Layer outputs are compared
element by element with the oracle on a set of tokens that touches every tile
the expert GEMMs compute: the tokens that own the first and the last row of
every 128-row tile of every expert (the single-CTA engine's tiles; the
CTA-pair engine's 256-row tiles are pairs of them, the swap-AB engine's row
boxes lie inside them), plus the first and last token of the batch.  Each
such token's output row spans every column tile of both projections, so
every (expert, row tile, column tile) of the layer holds a checked row at
each of its row edges.  Decode-sized batches are checked on every token.
Router logits are checked against fp64 on the same tokens.  The oracle needs
only the weights of the experts those tokens use, which it reads a few GB at
a time.
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

TILE_ROWS = 128
ALL_TOKENS_UP_TO = 256  # decode-sized batches: every token


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ops.lib()
    return torch.device("cuda:0")


def tile_edge_tokens(offsets, row_src, k_max, T, tile_rows=TILE_ROWS):
    """Tokens owning the first and last row of every tile_rows-row tile of
    every expert's rows offsets[e] .. offsets[e+1]-1, plus tokens 0 and T-1."""
    rows = []
    for e in range(len(offsets) - 1):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        for r0 in range(lo, hi, tile_rows):
            rows += [r0, min(r0 + tile_rows, hi) - 1]
    toks = {0, T - 1}
    if rows:
        toks |= set((np.asarray(row_src)[np.asarray(rows)] // k_max).tolist())
    return sorted(toks)


def test_tile_edge_tokens_cover_every_tile():
    # 3 experts with 300, 0 and 129 rows, k_max = 2, rows taken in order
    offsets = np.array([0, 300, 300, 429])
    row_src = np.arange(429) * 2 + 1  # row r serves slot 2r+1, token r
    toks = tile_edge_tokens(offsets, row_src, 2, 1000)
    assert toks == [0, 127, 128, 255, 256, 299, 300, 427, 428, 999]


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(WORKLOADS))
def test_full_size_workload(name, dev):
    w = WORKLOADS[name]
    inp = make_inputs(w, seed=0, device=dev)
    out, rb = run_layer(w, inp)
    routing = check_routing_bit_exact(w, {"sel_bias": inp["sel_bias"],
                                          "k_per_token": inp["k_per_token"]}, rb)
    # the kept-row count matches the stated drop policy
    assert int(rb["offsets"][-1].item()) == int(rb["counts"].sum().item()) - int(
        rb["n_dropped"].item())
    if w.T <= ALL_TOKENS_UP_TO:
        toks = list(range(w.T))
    else:
        toks = tile_edge_tokens(routing["offsets"], routing["row_src"], w.k_max, w.T)
    print(f"{name}: checking {len(toks)} of {w.T} tokens")
    sel = torch.tensor(toks, device=dev, dtype=torch.long)
    ref_logits = oracle.router_logits(to_numpy(inp["x"].index_select(0, sel)),
                                      to_numpy(inp["Wr"]), to_numpy(inp["logit_bias"]))
    assert_logits_close(rb["logits"].index_select(0, sel), ref_logits)
    ref = oracle_layer_on_tokens(inp, routing, toks)
    assert_out_close(f64(out.index_select(0, sel)), ref,
                     f"{name} full size, {len(toks)} tokens on every tile edge", storage(w))
    del inp, out, rb
    gc.collect()
    torch.cuda.empty_cache()
