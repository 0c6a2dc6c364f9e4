"""Thin ctypes binding of libmoe.so (include/moe.h): argument marshalling only.

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: torch tensors supply device pointers and the current
CUDA stream, the library does the work.  There is no fallback: if libmoe.so
is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .workloads import Workload

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_F32, MOE_BF16 = 0, 1
GATING = {"topk_softmax": 0, "softmax_topk_renorm": 1, "sigmoid_grouped": 2}
WS_ROUTE, WS_EXPERT_FFN, WS_LAYER = 0, 1, 2


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {moe_status_string(status)} ({status})")
        self.status = status


class MoeConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k_max", ctypes.c_int32), ("f", ctypes.c_int32), ("f_shared", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("gating", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("n_groups", ctypes.c_int32),
                ("topk_groups", ctypes.c_int32), ("group_score_topk", ctypes.c_int32),
                ("routed_scale", ctypes.c_float)]


class MoeRouteOut(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in
                ("logits", "topk_idx", "topk_w", "counts", "kept", "offsets", "slot_row",
                 "row_src", "n_dropped")]


EP_MAX_RANKS = 8


class MoeEpRanks(ctypes.Structure):
    _fields_ = [("rank", ctypes.c_int32), ("n_ranks", ctypes.c_int32),
                ("counts_all", ctypes.c_void_p),
                ("recv_rows", ctypes.c_void_p * EP_MAX_RANKS),
                ("y_back", ctypes.c_void_p * EP_MAX_RANKS)]


class MoeFp8Weights(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in ("W1", "W3", "W2", "s1", "s3", "s2")]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so (built by routing_dispatch_expert_sigmoid_b200/build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmoe.so not built ({LIB_PATH}); run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        cfgp = ctypes.POINTER(MoeConfig)
        outp = ctypes.POINTER(MoeRouteOut)
        L.moe_workspace_size.argtypes = [cfgp, I, ctypes.POINTER(S)]
        L.moe_route.argtypes = [cfgp, P, P, P, P, P, outp, P, S, P]
        L.moe_route_static_scratch.argtypes = [cfgp, P, P, P, P, P, outp, P]
        L.moe_dispatch.argtypes = [cfgp, P, P, P, P, P]
        L.moe_expert_ffn.argtypes = [cfgp, P, P, P, P, P, P, P, S, P]
        L.moe_combine.argtypes = [cfgp, P, P, P, P, P, P]
        L.moe_layer.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, P, outp, P, S, P]
        L.moe_layer_timed.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, P, outp, P, S, P,
                                      ctypes.POINTER(ctypes.c_void_p), I]
        fp8p = ctypes.POINTER(MoeFp8Weights)
        L.moe_quantize_fp8.argtypes = [P, I, I, I, P, P, P]
        L.moe_expert_ffn_fp8.argtypes = [cfgp, P, P, fp8p, P, P, S, P]
        L.moe_layer_fp8.argtypes = [cfgp, P, P, P, P, P, fp8p, fp8p, P, outp, P, S, P,
                                    ctypes.POINTER(ctypes.c_void_p), I]
        epp = ctypes.POINTER(MoeEpRanks)
        L.moe_ep_plan.argtypes = [cfgp, epp, P, P, P]
        L.moe_ep_dispatch.argtypes = [cfgp, epp, P, P, P, P, P, P]
        L.moe_ep_return.argtypes = [cfgp, epp, P, P, P]
        L.moe_ep_plan_host.argtypes = [I, I, I, P, P, P, P, P, I]
        L.moe_check_errors.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
        L.moe_status_string.argtypes = [I]
        L.moe_status_string.restype = ctypes.c_char_p
        for fn in ("moe_workspace_size", "moe_route", "moe_route_static_scratch", "moe_dispatch",
                   "moe_expert_ffn",
                   "moe_combine", "moe_layer", "moe_layer_timed", "moe_check_errors",
                   "moe_quantize_fp8", "moe_expert_ffn_fp8", "moe_layer_fp8", "moe_ep_plan",
                   "moe_ep_dispatch", "moe_ep_return", "moe_ep_plan_host"):
            getattr(L, fn).restype = I
        _lib = L
    return _lib


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != 0:
        raise MoeError(status, what)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def config(w: Workload, T: int | None = None) -> MoeConfig:
    """The moe_config of a workload (optionally with another token count)."""
    return MoeConfig(T=w.T if T is None else T, d=w.d, E=w.E, k_max=w.k_max, f=w.f,
                     f_shared=w.f_shared, dtype=MOE_F32 if w.dtype == "f32" else MOE_BF16,
                     gating=GATING[w.gating], capacity_factor=w.capacity_factor,
                     n_groups=w.n_groups, topk_groups=w.topk_groups,
                     group_score_topk=w.group_score_topk, routed_scale=w.routed_scale)


def moe_workspace_size(cfg: MoeConfig, kind: int = WS_LAYER) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_workspace_size(ctypes.byref(cfg), kind, ctypes.byref(n)),
           "moe_workspace_size")
    return int(n.value)


def workspace(cfg: MoeConfig, kind: int = WS_LAYER, device="cuda") -> torch.Tensor:
    """A caller-owned workspace of the size moe_workspace_size asks for."""
    return torch.empty(max(moe_workspace_size(cfg, kind), 1), dtype=torch.uint8, device=device)


def route_buffers(cfg: MoeConfig, device="cuda") -> dict:
    """Caller-owned routing output tensors for moe_route / moe_layer."""
    T, E, k = cfg.T, cfg.E, cfg.k_max
    i32 = dict(dtype=torch.int32, device=device)
    return dict(logits=torch.empty((T, E), dtype=torch.float32, device=device),
                topk_idx=torch.empty((T, k), **i32), topk_w=torch.empty((T, k), dtype=torch.float32,
                                                                        device=device),
                counts=torch.empty(E, **i32), kept=torch.empty(E, **i32),
                offsets=torch.empty(E + 1, **i32), slot_row=torch.empty((T, k), **i32),
                row_src=torch.empty(max(T * k, 1), **i32), n_dropped=torch.empty(1, **i32))


def _route_struct(b: dict) -> MoeRouteOut:
    return MoeRouteOut(*[b[name].data_ptr() for name, _ in MoeRouteOut._fields_])


def moe_route(cfg, x, Wr, logit_bias, sel_bias, k_per_token, out: dict, ws, stream=None):
    r = _route_struct(out)
    _check(lib().moe_route(ctypes.byref(cfg), _p(x), _p(Wr), _p(logit_bias), _p(sel_bias),
                           _p(k_per_token), ctypes.byref(r), _p(ws),
                           0 if ws is None else ws.numel(), _stream(stream)), "moe_route")


def moe_route_static_scratch(cfg, x, Wr, logit_bias, sel_bias, k_per_token, out: dict,
                             stream=None):
    """moe_route for callers that cannot provide a workspace: the library's
    fixed device scratch is used instead (see include/moe.h)."""
    r = _route_struct(out)
    _check(lib().moe_route_static_scratch(ctypes.byref(cfg), _p(x), _p(Wr), _p(logit_bias),
                                          _p(sel_bias), _p(k_per_token), ctypes.byref(r),
                                          _stream(stream)), "moe_route_static_scratch")


def moe_dispatch(cfg, x, offsets, row_src, x_perm, stream=None):
    _check(lib().moe_dispatch(ctypes.byref(cfg), _p(x), _p(offsets), _p(row_src), _p(x_perm),
                              _stream(stream)), "moe_dispatch")


def moe_expert_ffn(cfg, x_perm, offsets, W1, W3, W2, y_perm, ws, stream=None):
    _check(lib().moe_expert_ffn(ctypes.byref(cfg), _p(x_perm), _p(offsets), _p(W1), _p(W3),
                                _p(W2), _p(y_perm), _p(ws), 0 if ws is None else ws.numel(),
                                _stream(stream)), "moe_expert_ffn")


def moe_combine(cfg, y_perm, slot_row, topk_w, shared_y, out, stream=None):
    _check(lib().moe_combine(ctypes.byref(cfg), _p(y_perm), _p(slot_row), _p(topk_w),
                             _p(shared_y), _p(out), _stream(stream)), "moe_combine")


def moe_layer(cfg, x, Wr, logit_bias, sel_bias, k_per_token, W1, W3, W2, Ws1, Ws3, Ws2, out,
              route_out: dict | None, ws, stream=None):
    r = None if route_out is None else ctypes.byref(_route_struct(route_out))
    _check(lib().moe_layer(ctypes.byref(cfg), _p(x), _p(Wr), _p(logit_bias), _p(sel_bias),
                           _p(k_per_token), _p(W1), _p(W3), _p(W2), _p(Ws1), _p(Ws3), _p(Ws2),
                           _p(out), r, _p(ws), 0 if ws is None else ws.numel(), _stream(stream)),
           "moe_layer")


STAGES = ("start", "route", "dispatch", "up_swiglu", "down", "shared", "combine")


def moe_layer_timed(cfg, x, Wr, logit_bias, sel_bias, k_per_token, W1, W3, W2, Ws1, Ws3, Ws2,
                    out, route_out: dict | None, ws, events, stream=None):
    """moe_layer that records events[i] (torch.cuda.Event, len(STAGES)) at stage boundary i."""
    r = None if route_out is None else ctypes.byref(_route_struct(route_out))
    handles = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(lib().moe_layer_timed(ctypes.byref(cfg), _p(x), _p(Wr), _p(logit_bias), _p(sel_bias),
                                 _p(k_per_token), _p(W1), _p(W3), _p(W2), _p(Ws1), _p(Ws3),
                                 _p(Ws2), _p(out), r, _p(ws), 0 if ws is None else ws.numel(),
                                 _stream(stream), handles, len(events)), "moe_layer_timed")


def moe_check_errors(stream=None) -> int:
    """Synchronise the stream and return the device error flags (raises if any)."""
    flags = ctypes.c_uint32(0)
    st = lib().moe_check_errors(_stream(stream), ctypes.byref(flags))
    if st not in (0, -6):
        _check(st, "moe_check_errors")
    if flags.value:
        raise MoeError(st, f"moe_check_errors: device flags {flags.value:#x}")
    return 0


# ---- fp8 expert weights -----------------------------------------------------
def moe_quantize_fp8(W: torch.Tensor, stream=None):
    """W [G, K, N] (or [K, N]) bf16 -> (codes uint8 [G, N, K] (or [N, K]),
    scales fp32 [G, N] (or [N])), computed by the library."""
    Wg = W if W.dim() == 3 else W.unsqueeze(0)
    G, K, N = Wg.shape
    q = torch.empty((G, N, K), dtype=torch.uint8, device=W.device)
    sc = torch.empty((G, N), dtype=torch.float32, device=W.device)
    _check(lib().moe_quantize_fp8(_p(Wg), G, K, N, _p(q), _p(sc), _stream(stream)),
           "moe_quantize_fp8")
    if W.dim() == 2:
        return q[0], sc[0]
    return q, sc


def fp8_weight_set(W1, W3, W2, stream=None) -> dict:
    """Quantise one set of expert matrices (routed [E, ...] or shared [d, f])."""
    out = {}
    for name, W in (("W1", W1), ("W3", W3), ("W2", W2)):
        q, sc = moe_quantize_fp8(W, stream)
        out[name], out["s" + name[1]] = q, sc
    return out


def _fp8_struct(ws: dict | None):
    if ws is None:
        return None
    return MoeFp8Weights(*[ws[k].data_ptr() for k in ("W1", "W3", "W2", "s1", "s3", "s2")])


def moe_expert_ffn_fp8(cfg, x_perm, offsets, weights: dict, y_perm, ws, stream=None):
    wq = _fp8_struct(weights)
    _check(lib().moe_expert_ffn_fp8(ctypes.byref(cfg), _p(x_perm), _p(offsets), ctypes.byref(wq),
                                    _p(y_perm), _p(ws), 0 if ws is None else ws.numel(),
                                    _stream(stream)), "moe_expert_ffn_fp8")


def moe_layer_fp8(cfg, x, Wr, logit_bias, sel_bias, k_per_token, experts: dict,
                  shared: dict | None, out, route_out: dict | None, ws, events=None,
                  stream=None):
    """moe_layer with fp8 expert weights (dicts from fp8_weight_set); events as
    in moe_layer_timed, or None."""
    r = None if route_out is None else ctypes.byref(_route_struct(route_out))
    we, wsh = _fp8_struct(experts), _fp8_struct(shared)
    n = 0 if events is None else len(events)
    handles = None if events is None else (ctypes.c_void_p * n)(
        *[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(lib().moe_layer_fp8(ctypes.byref(cfg), _p(x), _p(Wr), _p(logit_bias), _p(sel_bias),
                               _p(k_per_token), ctypes.byref(we),
                               None if wsh is None else ctypes.byref(wsh), _p(out), r, _p(ws),
                               0 if ws is None else ws.numel(), _stream(stream), handles, n),
           "moe_layer_fp8")


# ---- expert parallelism -----------------------------------------------------
def ep_ranks(rank: int, n_ranks: int, counts_all, recv_rows, y_back) -> MoeEpRanks:
    """The moe_ep_ranks of one rank: counts_all [n_ranks, E] int32 on its
    device, and every rank's receive and return buffers (device tensors)."""
    ep = MoeEpRanks()
    ep.rank, ep.n_ranks = rank, n_ranks
    ep.counts_all = counts_all.data_ptr()
    for r in range(n_ranks):
        ep.recv_rows[r] = recv_rows[r].data_ptr()
        ep.y_back[r] = y_back[r].data_ptr()
    return ep


def moe_ep_plan(cfg, ep: MoeEpRanks, recv_offsets, send_base, stream=None):
    _check(lib().moe_ep_plan(ctypes.byref(cfg), ctypes.byref(ep), _p(recv_offsets),
                             _p(send_base), _stream(stream)), "moe_ep_plan")


def moe_ep_dispatch(cfg, ep: MoeEpRanks, x, offsets, row_src, topk_idx, send_base, stream=None):
    _check(lib().moe_ep_dispatch(ctypes.byref(cfg), ctypes.byref(ep), _p(x), _p(offsets),
                                 _p(row_src), _p(topk_idx), _p(send_base), _stream(stream)),
           "moe_ep_dispatch")


def moe_ep_return(cfg, ep: MoeEpRanks, y_recv, recv_offsets, stream=None):
    _check(lib().moe_ep_return(ctypes.byref(cfg), ctypes.byref(ep), _p(y_recv),
                               _p(recv_offsets), _stream(stream)), "moe_ep_return")


def moe_ep_plan_host(n_ranks: int, E: int, rank: int, counts_all, max_recv: int):
    """Host mirror of the plan: (recv_offsets, send_base, recv_src, recv_src_row)
    as int32 numpy arrays, from counts_all [n_ranks, E] (numpy)."""
    import numpy as np
    C = np.ascontiguousarray(counts_all, dtype=np.int32)
    e_loc = E // max(n_ranks, 1)
    ro = np.zeros(e_loc + 1, np.int32)
    sb = np.zeros(E, np.int32)
    rs = np.zeros(max(max_recv, 1), np.int32)
    rr = np.zeros(max(max_recv, 1), np.int32)
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(lib().moe_ep_plan_host(n_ranks, E, rank, ptr(C), ptr(ro), ptr(sb), ptr(rs), ptr(rr),
                                  max_recv), "moe_ep_plan_host")
    R = int(ro[-1])
    return ro, sb, rs[:R], rr[:R]
