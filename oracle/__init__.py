"""CPU oracle of one Mixture-of-Experts layer (test infrastructure only).

Only tests/, the smoke check in __graft_entry__ and the CPU-baseline /
reference leg of bench.py may import this package.  The product library never
does, and the two implementations share no code.

Each function is a thin numpy <-> C marshaller around oracle/moe_oracle.c,
where the arithmetic and its citations live.  Floating tensors are passed as
numpy arrays of float32, or of uint16 holding bf16 bit patterns (dtype="bf16");
the FFN and layer functions also take float64 weights (dequantised fp8).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

F32, BF16, F64 = 0, 1, 2
TOPK_SOFTMAX, SOFTMAX_TOPK_RENORM, SIGMOID_GROUPED = 0, 1, 2
GATING = {"topk_softmax": TOPK_SOFTMAX, "softmax_topk_renorm": SOFTMAX_TOPK_RENORM,
          "sigmoid_grouped": SIGMOID_GROUPED}

_lib = None


def lib():
    global _lib
    if _lib is None:
        # MOE_ORACLE_LIB points the tests that plant mistakes at a mutated copy.
        path = os.environ.get("MOE_ORACLE_LIB") or _build.LIB
        if path == _build.LIB and not os.path.exists(path):
            _build.build()
        _lib = ctypes.CDLL(path)
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.c_double


def _declare(L):
    L.oracle_router_logits.argtypes = [_I, _I, _I, _P, _P, _I, _P, _P]
    L.oracle_router_logits.restype = None
    L.oracle_spec_expf_n.argtypes = [_I, _P, _P]
    L.oracle_spec_sigmoidf_n.argtypes = [_I, _P, _P]
    L.oracle_spec_constants.argtypes = [_P]
    L.oracle_gating.argtypes = [_I, _I, _I, _I, _I, _I, _I, _D, _P, _P, _P, _P, _P]
    L.oracle_gating.restype = _I
    L.oracle_capacity_dispatch.argtypes = [_I, _I, _I, _D, _P, _P, _P, _P, _P, _P, _P]
    L.oracle_capacity_dispatch.restype = ctypes.c_longlong
    L.oracle_dispatch.argtypes = [_I, _I, _I, _I, _P, _P, _P]
    L.oracle_expert_ffn.argtypes = [_I, _I, _I, _P, _I, _P, _P, _P, _I, _P]
    L.oracle_combine.argtypes = [_I, _I, _I, _P, _P, _P, _P, _P]
    L.oracle_combine_rows.argtypes = [_I, _I, _I, _P, _P, _P, _P, _I, _P]
    L.oracle_layer_tokens.argtypes = [_I, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P,
                                      _I, _I, _P, _P, _P, _P]
    L.oracle_e4m3_decode_n.argtypes = [ctypes.c_longlong, _P, _P]
    L.oracle_e4m3_encode_n.argtypes = [ctypes.c_longlong, _P, _P]
    L.oracle_quantize_fp8.argtypes = [_I, _I, _I, _P, _P, _P]


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _dt(a) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float64:
        return F64
    raise TypeError(f"oracle tensors are float32, uint16 (bf16 bits) or float64, got {a.dtype}")


# --------------------------------------------------------------------------
def router_logits(x, Wr, logit_bias=None) -> np.ndarray:
    """fp64 logits[T,E] = x[T,d] . Wr[d,E] (+ logit_bias[E])."""
    x = np.ascontiguousarray(x)
    Wr = np.ascontiguousarray(Wr)
    assert x.dtype == Wr.dtype
    T, d = x.shape
    E = Wr.shape[1]
    out = np.empty((T, E), np.float64)
    lb = None if logit_bias is None else _c(logit_bias, np.float32)
    lib().oracle_router_logits(T, d, E, _ptr(x), _ptr(Wr), _dt(x), _ptr(lb), _ptr(out))
    return out


def spec_expf(z) -> np.ndarray:
    z = _c(z, np.float32).ravel()
    out = np.empty_like(z)
    lib().oracle_spec_expf_n(z.size, _ptr(z), _ptr(out))
    return out


def spec_sigmoidf(z) -> np.ndarray:
    z = _c(z, np.float32).ravel()
    out = np.empty_like(z)
    lib().oracle_spec_sigmoidf_n(z.size, _ptr(z), _ptr(out))
    return out


def spec_constants() -> np.ndarray:
    out = np.empty(11, np.float32)
    lib().oracle_spec_constants(_ptr(out))
    return out


def gating(logits32, k_max, mode="topk_softmax", *, sel_bias=None, k_per_token=None,
           n_groups=1, topk_groups=1, group_score_topk=1, routed_scale=1.0):
    """Top-k selection on fp32 logits. Returns (topk_idx int32 [T,k_max], topk_w f64)."""
    l32 = _c(logits32, np.float32)
    T, E = l32.shape
    idx = np.empty((T, k_max), np.int32)
    w = np.empty((T, k_max), np.float64)
    sb = None if sel_bias is None else _c(sel_bias, np.float32)
    kt = None if k_per_token is None else _c(k_per_token, np.int32)
    m = GATING[mode] if isinstance(mode, str) else int(mode)
    rc = lib().oracle_gating(T, E, k_max, m, n_groups, topk_groups, group_score_topk,
                             float(routed_scale), _ptr(l32), _ptr(sb), _ptr(kt), _ptr(idx),
                             _ptr(w))
    if rc != 0:
        raise ValueError("oracle_gating rejected its arguments")
    return idx, w


def capacity_dispatch(topk_idx, E, capacity_factor=0.0):
    """Counts, capacity, drops and the expert-contiguous row layout."""
    idx = _c(topk_idx, np.int32)
    T, k_max = idx.shape
    counts = np.empty(E, np.int32)
    kept = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    slot_row = np.empty((T, k_max), np.int32)
    row_src = np.full(max(T * k_max, 1), -1, np.int32)
    cap = ctypes.c_longlong(0)
    dropped = lib().oracle_capacity_dispatch(T, E, k_max, float(capacity_factor), _ptr(idx),
                                             _ptr(counts), _ptr(kept), _ptr(offsets),
                                             _ptr(slot_row), _ptr(row_src), ctypes.byref(cap))
    if dropped < 0:
        raise ValueError("oracle_capacity_dispatch: expert index out of range")
    R = int(offsets[E])
    return dict(counts=counts, kept=kept, offsets=offsets, slot_row=slot_row,
                row_src=row_src[:R].copy(), n_dropped=int(dropped), capacity=int(cap.value))


def dispatch(x, row_src, k_max):
    """x_perm[r] = x[row_src[r] // k_max] (values copied as stored)."""
    x = np.ascontiguousarray(x)
    rs = _c(row_src, np.int32)
    R = rs.size
    T, d = x.shape
    out = np.empty((R, d), x.dtype)
    lib().oracle_dispatch(R, k_max, d, x.itemsize, _ptr(rs), _ptr(x), _ptr(out))
    return out


def expert_ffn(x, W1e, W3e, W2e) -> np.ndarray:
    """fp64 y = (silu(x.W1e) * (x.W3e)) . W2e for every row of x."""
    x = np.ascontiguousarray(x)
    W1e, W3e, W2e = (np.ascontiguousarray(a) for a in (W1e, W3e, W2e))
    assert W1e.dtype == W3e.dtype == W2e.dtype
    n, d = x.shape
    f = W1e.shape[1]
    assert W1e.shape == (d, f) and W3e.shape == (d, f) and W2e.shape == (f, d)
    y = np.empty((n, d), np.float64)
    lib().oracle_expert_ffn(n, d, f, _ptr(x), _dt(x), _ptr(W1e), _ptr(W3e), _ptr(W2e),
                            _dt(W1e), _ptr(y))
    return y


def grouped_ffn(x_perm, offsets, W1, W3, W2) -> np.ndarray:
    """fp64 y_perm[r] = FFN_e(x_perm[r]) for rows offsets[e] <= r < offsets[e+1]."""
    E = W1.shape[0]
    R = int(offsets[E])
    y = np.zeros((R, x_perm.shape[1]), np.float64)
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b > a:
            y[a:b] = expert_ffn(x_perm[a:b], W1[e], W3[e], W2[e])
    return y


def combine(w, kept_mask, y_slot, shared=None) -> np.ndarray:
    """fp64 out[t] = sum_j kept * w[t,j] * y_slot[t,j] (+ shared[t])."""
    w = _c(w, np.float64)
    n, k_max = w.shape
    d = y_slot.shape[-1]
    km = _c(kept_mask, np.int32)
    ys = _c(y_slot, np.float64)
    sh = None if shared is None else _c(shared, np.float64)
    out = np.empty((n, d), np.float64)
    lib().oracle_combine(n, k_max, d, _ptr(w), _ptr(km), _ptr(ys), _ptr(sh), _ptr(out))
    return out


def combine_rows(topk_w, slot_row, y_perm, shared=None) -> np.ndarray:
    """fp64 out[t] = sum_j w[t,j] * y_perm[slot_row[t,j]] over kept slots (+ shared[t])."""
    w = _c(topk_w, np.float64)
    T, k_max = w.shape
    y_perm = np.ascontiguousarray(y_perm)
    d = y_perm.shape[1]
    sr = _c(slot_row, np.int32)
    if shared is not None:
        shared = np.ascontiguousarray(shared)
        assert shared.dtype == y_perm.dtype
    out = np.empty((T, d), np.float64)
    lib().oracle_combine_rows(T, k_max, d, _ptr(w), _ptr(sr), _ptr(y_perm), _ptr(shared),
                              _dt(y_perm), _ptr(out))
    return out


def layer_tokens(tokens, x, W1, W3, W2, topk_idx, topk_w, slot_row, Ws1=None, Ws3=None,
                 Ws2=None) -> np.ndarray:
    """fp64 layer output for the listed tokens, given a routing."""
    tok = _c(tokens, np.int32)
    x = np.ascontiguousarray(x)
    W1, W3, W2 = (np.ascontiguousarray(a) for a in (W1, W3, W2))
    E, d, f = W1.shape
    k_max = topk_idx.shape[1]
    fs = 0 if Ws1 is None else Ws1.shape[1]
    if Ws1 is not None:
        Ws1, Ws3, Ws2 = (np.ascontiguousarray(a) for a in (Ws1, Ws3, Ws2))
    out = np.empty((tok.size, d), np.float64)
    if Ws1 is not None:
        assert Ws1.dtype == W1.dtype, "routed and shared weights share one storage type"
    lib().oracle_layer_tokens(tok.size, _ptr(tok), d, E, k_max, f, fs, _ptr(x), _ptr(W1),
                              _ptr(W3), _ptr(W2), _ptr(Ws1), _ptr(Ws3), _ptr(Ws2), _dt(x), _dt(W1),
                              _ptr(_c(topk_idx, np.int32)), _ptr(_c(topk_w, np.float64)),
                              _ptr(_c(slot_row, np.int32)), _ptr(out))
    return out


def layer(x, Wr, W1, W3, W2, *, k_max, gating_mode="topk_softmax", capacity_factor=0.0,
          logit_bias=None, sel_bias=None, k_per_token=None, n_groups=1, topk_groups=1,
          group_score_topk=1, routed_scale=1.0, Ws1=None, Ws3=None, Ws2=None,
          logits32=None):
    """The whole layer: router -> gating -> capacity/dispatch layout -> FFN -> combine.

    Selection is decided on fp32 logits: the fp64 router logits rounded to
    fp32, unless logits32 (e.g. another implementation's fp32 logits) is given.
    """
    logits = router_logits(x, Wr, logit_bias)
    l32 = logits.astype(np.float32) if logits32 is None else _c(logits32, np.float32)
    idx, w = gating(l32, k_max, gating_mode, sel_bias=sel_bias, k_per_token=k_per_token,
                    n_groups=n_groups, topk_groups=topk_groups,
                    group_score_topk=group_score_topk, routed_scale=routed_scale)
    E = Wr.shape[1]
    disp = capacity_dispatch(idx, E, capacity_factor)
    T = x.shape[0]
    out = layer_tokens(np.arange(T, dtype=np.int32), x, W1, W3, W2, idx, w, disp["slot_row"],
                       Ws1, Ws3, Ws2)
    return dict(logits=logits, topk_idx=idx, topk_w=w, out=out, **disp)


# --------------------------------------------------------------------------
# FP8 expert weights ("LLM MoE Expert Parallel 生产实战", sections 5 and 10:
# DeepSeek-V3 served with fp8 quantisation, router head kept in precision).
# e4m3 codes with one fp32 scale per output column of each expert matrix.
def e4m3_decode(codes) -> np.ndarray:
    """The value of every e4m3 code (NaN for the two NaN codes), as float64."""
    c = _c(codes, np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().oracle_e4m3_decode_n(c.size, _ptr(c), _ptr(out))
    return out


def e4m3_encode(values) -> np.ndarray:
    """Nearest e4m3 code of every float32 value, ties to even, saturating at 448."""
    v = _c(values, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().oracle_e4m3_encode_n(v.size, _ptr(v), _ptr(out))
    return out


def quantize_fp8(W):
    """W: [G, K, N] bf16 bits (uint16).  Returns (codes uint8 [G, K, N],
    scales float32 [G, N]): per output column s = max|W| / 448 in fp32 (1 for
    an all-zero column) and codes e4m3(W / s) of the fp32 quotient."""
    W = _c(W, np.uint16)
    G, K, N = W.shape
    q = np.empty((G, K, N), np.uint8)
    s = np.empty((G, N), np.float32)
    lib().oracle_quantize_fp8(G, K, N, _ptr(W), _ptr(q), _ptr(s))
    return q, s


def dequantize_fp8(q, s) -> np.ndarray:
    """The weights the quantised layer computes with: e4m3_decode(q) * s per
    output column, exact in float64 ([G, K, N])."""
    return e4m3_decode(q) * np.asarray(s, np.float64)[:, None, :]
