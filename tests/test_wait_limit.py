"""A pipeline wait that runs out ends the GEMM with an error flag, not a hang.

Every wait of the tensor-core GEMMs (data landing in shared memory, a free
accumulator, ...) is bounded in time.  MOE_WAIT_LIMIT_NS lowers that bound for
the single-CTA and swap-AB engines; at 0 ns the first wait that does not
succeed at once gives up.  The CTA then records bit 1 in the device error
word, stops its other roles, lets the copies and MMAs it already issued land,
frees its tensor memory and returns.  The test routes a small decode-sized
layer normally (up projection on the swap-AB engine, down projection on the
single-CTA engine), runs the expert FFN with a 0 ns limit, and checks that
moe_check_errors reports exactly that flag; then, in the same process, the
same FFN and the whole layer with the default limit match the oracle.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

import oracle
from parity import assert_out_close, check_routing_bit_exact, f64, gpu_inputs, run_layer, \
    run_route, oracle_layer_on_tokens, storage
from routing_dispatch_expert_sigmoid_b200 import ops
from routing_dispatch_expert_sigmoid_b200.workloads import WORKLOADS, make_inputs, to_numpy

pytestmark = pytest.mark.gpu

MOE_ERR_DEVICE_CHECK = -6
FLAG_WAIT = 2


def _check_errors_raw():
    flags = ctypes.c_uint32(0)
    st = ops.lib().moe_check_errors(ops._stream(None), ctypes.byref(flags))
    return st, flags.value


def test_wait_limit_stops_and_next_call_is_correct(cuda_device):
    dev = cuda_device
    # 64 tokens x top-2 over 8 experts: 16 rows per expert on average, so the up
    # projection runs on the swap-AB engine and the down projection single-CTA
    w = WORKLOADS["mixtral_decode"].scaled(T=64, d=512, f=640)
    hin = make_inputs(w, seed=11, device="cpu")
    inp = gpu_inputs(w, 11, dev, hin)
    cfg, rb = run_route(w, inp)  # default limit
    lay = check_routing_bit_exact(w, hin, rb)
    R = int(lay["offsets"][-1])
    x_perm = torch.zeros((w.T * w.k_max, w.d), dtype=inp["x"].dtype, device=dev)
    ops.moe_dispatch(cfg, inp["x"], rb["offsets"], rb["row_src"], x_perm)
    y_perm = torch.zeros((w.T * w.k_max, w.d), dtype=torch.float32, device=dev)
    ws = ops.workspace(cfg, ops.WS_EXPERT_FFN)
    assert _check_errors_raw() == (0, 0)

    old = os.environ.get("MOE_WAIT_LIMIT_NS")
    os.environ["MOE_WAIT_LIMIT_NS"] = "0"
    try:
        ops.moe_expert_ffn(cfg, x_perm, rb["offsets"], inp["W1"], inp["W3"], inp["W2"], y_perm,
                           ws)
        st, flags = _check_errors_raw()
    finally:
        if old is None:
            os.environ.pop("MOE_WAIT_LIMIT_NS", None)
        else:
            os.environ["MOE_WAIT_LIMIT_NS"] = old
    assert st == MOE_ERR_DEVICE_CHECK and flags == FLAG_WAIT, (st, flags)
    # the flags were cleared by the read, and the context is usable
    assert _check_errors_raw() == (0, 0)

    # default limit again: the same FFN and the whole layer match the oracle
    ops.moe_expert_ffn(cfg, x_perm, rb["offsets"], inp["W1"], inp["W3"], inp["W2"], y_perm, ws)
    ops.moe_check_errors()
    xp = oracle.dispatch(to_numpy(hin["x"]), lay["row_src"], w.k_max)
    ref = oracle.grouped_ffn(xp, lay["offsets"], to_numpy(hin["W1"]), to_numpy(hin["W3"]),
                             to_numpy(hin["W2"]))
    assert_out_close(f64(y_perm[:R]), ref, "y_perm after a stopped call", "f32")
    out, rb2 = run_layer(w, inp)
    routing = check_routing_bit_exact(w, hin, rb2)
    toks = list(range(w.T))
    ref_out = oracle_layer_on_tokens(inp, routing, toks)
    assert_out_close(f64(out), ref_out, "layer after a stopped call", storage(w))
