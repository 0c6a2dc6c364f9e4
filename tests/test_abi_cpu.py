"""The C ABI without a GPU: the library loads, exports every entry point that
include/moe.h declares, sizes workspaces, and rejects bad arguments on the
host before touching the device.  Nothing here launches a kernel.
"""
import ctypes
import math
import os
import re
import struct
from fractions import Fraction

import pytest

from routing_dispatch_expert_sigmoid_b200 import ops
from routing_dispatch_expert_sigmoid_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 8, names
    L = ops.lib()
    for n in names:
        assert hasattr(L, n), f"libmoe.so does not export {n}"
    assert {"moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_layer"} <= set(names)


def test_status_strings():
    for st in range(-6, 1):
        s = ops.moe_status_string(st)
        assert s.startswith("MOE_")
    assert "unknown" in ops.moe_status_string(42)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workspace_sizes(name):
    w = WORKLOADS[name]
    cfg = ops.config(w)
    s = w.elem_bytes
    slots = w.T * w.k_max
    layer = ops.moe_workspace_size(cfg, ops.WS_LAYER)
    # x_perm, h and y_perm are the dominant regions
    assert layer >= slots * (2 * w.d + w.f) * s
    assert ops.moe_workspace_size(cfg, ops.WS_EXPERT_FFN) >= slots * w.f * s
    assert 0 < ops.moe_workspace_size(cfg, ops.WS_ROUTE) < layer
    for kind in (ops.WS_ROUTE, ops.WS_EXPERT_FFN, ops.WS_LAYER):
        assert ops.moe_workspace_size(cfg, kind) % 256 == 0


def _status(fn, *args):
    return getattr(ops.lib(), fn)(*args)


def _cfg(**kw):
    c = ops.config(WORKLOADS["dsv3_decode"])
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("kw,expect", [
    (dict(k_max=300), -1), (dict(k_max=0), -1), (dict(E=0), -1), (dict(E=2048), -1),
    (dict(T=-1), -1), (dict(d=0), -1), (dict(dtype=7), -2), (dict(gating=9), -2),
    (dict(d=7164), -4), (dict(f=2044), -4), (dict(n_groups=7), -1), (dict(n_groups=64), -1),
    (dict(topk_groups=9), -1), (dict(group_score_topk=33), -1), (dict(group_score_topk=9), -2),
    (dict(topk_groups=1, k_max=33), -1),
])
def test_config_validation(kw, expect):
    c = _cfg(**kw)
    n = ctypes.c_size_t(0)
    assert ops.lib().moe_workspace_size(ctypes.byref(c), ops.WS_LAYER, ctypes.byref(n)) == expect


FAKE = 0x7f0000000000  # 16-byte aligned, never dereferenced: validation fails first


def _route_out(ptr=FAKE):
    return ops.MoeRouteOut(*([ptr] * 9))


def test_null_and_misaligned_pointers_rejected_before_launch():
    c = _cfg()
    L = ops.lib()
    r = _route_out()
    P = ctypes.c_void_p
    ws = ctypes.c_size_t(1 << 40)
    # null x
    assert L.moe_route(ctypes.byref(c), None, P(FAKE), None, None, None, ctypes.byref(r), P(FAKE),
                       ws, None) == -1
    # misaligned x
    assert L.moe_route(ctypes.byref(c), P(FAKE + 8), P(FAKE), None, None, None, ctypes.byref(r),
                       P(FAKE), ws, None) == -4
    # misaligned k_per_token (int32 array: 4-byte rule)
    assert L.moe_route(ctypes.byref(c), P(FAKE), P(FAKE), None, None, P(FAKE + 2),
                       ctypes.byref(r), P(FAKE), ws, None) == -4
    # a null routing output
    bad = _route_out()
    bad.offsets = None
    assert L.moe_route(ctypes.byref(c), P(FAKE), P(FAKE), None, None, None, ctypes.byref(bad),
                       P(FAKE), ws, None) == -1
    assert L.moe_dispatch(ctypes.byref(c), P(FAKE), None, P(FAKE), P(FAKE), None) == -1
    assert L.moe_combine(ctypes.byref(c), P(FAKE), P(FAKE), P(FAKE), P(FAKE + 4), P(FAKE),
                         None) == -4
    # shared expert weights are required when f_shared > 0
    args = [P(FAKE)] * 5 + [P(FAKE)] * 3 + [None, P(FAKE), P(FAKE), P(FAKE)]
    assert L.moe_layer(ctypes.byref(c), P(FAKE), P(FAKE), None, None, None, P(FAKE), P(FAKE),
                       P(FAKE), None, P(FAKE), P(FAKE), P(FAKE), None, P(FAKE), ws, None) == -1
    del args


def test_workspace_too_small_rejected():
    c = _cfg()
    L = ops.lib()
    P = ctypes.c_void_p
    need = ops.moe_workspace_size(c, ops.WS_LAYER)
    small = ctypes.c_size_t(need - 1)
    assert L.moe_layer(ctypes.byref(c), P(FAKE), P(FAKE), None, None, None, P(FAKE), P(FAKE),
                       P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), None, P(FAKE), small,
                       None) == -3
    assert L.moe_layer(ctypes.byref(c), P(FAKE), P(FAKE), None, None, None, P(FAKE), P(FAKE),
                       P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), None, None,
                       ctypes.c_size_t(need), None) == -3
    r = _route_out()
    need_r = ops.moe_workspace_size(c, ops.WS_ROUTE)
    assert L.moe_route(ctypes.byref(c), P(FAKE), P(FAKE), None, None, None, ctypes.byref(r),
                       P(FAKE), ctypes.c_size_t(need_r - 256), None) == -3


def test_empty_batch_is_a_noop_without_pointers():
    c = _cfg(T=0)
    L = ops.lib()
    assert L.moe_layer(ctypes.byref(c), None, None, None, None, None, None, None, None, None,
                       None, None, None, None, None, ctypes.c_size_t(0), None) == 0


def _exact_f32(fr: Fraction) -> int:
    """binary32 bits of a positive rational, rounded to nearest even."""
    e = math.floor(math.log2(fr.numerator) - math.log2(fr.denominator))
    while Fraction(2) ** e > fr:
        e -= 1
    while Fraction(2) ** (e + 1) <= fr:
        e += 1
    m = fr * Fraction(2) ** (23 - e)
    lo = m.numerator // m.denominator
    rem = m - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2):
        lo += 1
    return struct.unpack("<I", struct.pack("<f", float(Fraction(lo) * Fraction(2) ** (e - 23))))[0]


def test_gpu_sigmoid_constants_are_the_rounded_definitions():
    """The GPU's specified exp takes its constants from their definitions."""
    from decimal import Decimal, getcontext
    getcontext().prec = 60
    ln2 = Fraction(Decimal(2).ln())
    src = open(os.path.join(ROOT, "routing_dispatch_expert_sigmoid_b200", "csrc", "gating.cuh")).read()
    lits = dict(re.findall(r"const float (k\w+) = ([0-9.e+-]+)f;", src))

    def bits(name):
        return struct.unpack("<I", struct.pack("<f", float(lits[name])))[0]

    assert bits("kLog2e") == _exact_f32(1 / ln2)
    assert Fraction(float(lits["kLn2Hi"])) == Fraction(2839, 4096)
    assert bits("kLn2Lo") == _exact_f32(ln2 - Fraction(2839, 4096))
    for k in range(3, 8):
        assert bits(f"kC{k}") == _exact_f32(Fraction(1, math.factorial(k))), k


# ---- fp8 expert weights: host-side checks (nothing reaches the device) -------
_FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced: rejected first


def _fp8_set(**kw):
    v = dict(W1=_FAKE, W3=_FAKE, W2=_FAKE, s1=_FAKE, s3=_FAKE, s2=_FAKE)
    v.update(kw)
    return ops.MoeFp8Weights(*[v[k] for k in ("W1", "W3", "W2", "s1", "s3", "s2")])


@pytest.mark.parametrize("kw,expect", [
    (dict(dtype=ops.MOE_F32), -2),   # fp8 weights need bf16 activations
    (dict(d=7160), -4),              # d a multiple of 8 but not of 16
    (dict(f=2040), -4),
    (dict(f_shared=2040), -4),
])
def test_fp8_layer_config_checks(kw, expect):
    c = _cfg(**kw)
    w = _fp8_set()
    st = ops.lib().moe_layer_fp8(ctypes.byref(c), _FAKE, _FAKE, None, None, None, ctypes.byref(w),
                                 ctypes.byref(w), _FAKE, None, _FAKE, 1 << 40, None, None, 0)
    assert st == expect


def test_fp8_layer_argument_checks():
    c = _cfg()
    w = _fp8_set()
    lib = ops.lib()
    args = lambda we, ws, ev=None, n=0: (ctypes.byref(c), _FAKE, _FAKE, None, None, None, we, ws,
                                         _FAKE, None, _FAKE, 1 << 40, None, ev, n)
    assert lib.moe_layer_fp8(*args(None, ctypes.byref(w))) == -1           # no experts
    assert lib.moe_layer_fp8(*args(ctypes.byref(w), None)) == -1           # shared expert missing
    assert lib.moe_layer_fp8(*args(ctypes.byref(w), ctypes.byref(w), None, 3)) == -1  # events
    bad = _fp8_set(s2=_FAKE + 4)                                            # scales need 16 B
    assert lib.moe_layer_fp8(*args(ctypes.byref(bad), ctypes.byref(w))) == -4
    bad = _fp8_set(W3=0)
    assert lib.moe_layer_fp8(*args(ctypes.byref(bad), ctypes.byref(w))) == -1
    assert lib.moe_expert_ffn_fp8(ctypes.byref(c), _FAKE, _FAKE, None, _FAKE, _FAKE, 1 << 40,
                                  None) == -1


def test_fp8_quantize_checks():
    lib = ops.lib()
    assert lib.moe_quantize_fp8(_FAKE, 2, 64, 24, _FAKE, _FAKE, None) == -4   # N % 16
    assert lib.moe_quantize_fp8(_FAKE, 2, 40, 32, _FAKE, _FAKE, None) == -4   # K % 16
    assert lib.moe_quantize_fp8(_FAKE, -1, 64, 32, _FAKE, _FAKE, None) == -1
    assert lib.moe_quantize_fp8(_FAKE, 0, 64, 32, _FAKE, _FAKE, None) == 0    # nothing to do
    assert lib.moe_quantize_fp8(_FAKE + 8, 2, 64, 32, _FAKE, _FAKE, None) == -4


def test_fp8_widening_bit_formula_gives_every_code():
    """The GEMM widens four e4m3 codes (one 32-bit word) to bf16 by moving
    bits: signs cleared, each pair's bytes placed 16 bits apart and multiplied
    by 16 (exponent and fraction land in the bf16 field), one multiply by
    2^120, then the signs or-ed back in.  Emulated here for every finite code
    in every byte position against the oracle's decoding (the GPU tests cover
    the hardware's multiply)."""
    import numpy as np

    import oracle
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint64)
    ref = oracle.e4m3_decode(codes.astype(np.uint8))
    other = np.uint64(0x38)  # the code of 1.0 in the other byte positions
    for pos in range(4):
        words = np.full(codes.shape, 0, np.uint64)
        for q in range(4):
            words |= (codes if q == pos else other) << np.uint64(8 * q)
        mag = words & np.uint64(0x7F7F7F7F)
        byte = (mag >> np.uint64(8 * pos)) & np.uint64(0xFF)
        field = (byte * np.uint64(16)) & np.uint64(0xFFFF)   # this half's 16 bits
        sign = (words >> np.uint64(8 * pos + 7)) & np.uint64(1)
        val = (field.astype(np.uint32) << 16).view(np.float32).astype(np.float64) * 2.0 ** 120
        val = np.where(sign == 1, -val, val)
        assert (val == ref).all(), pos
        assert (np.signbit(val) == np.signbit(ref)).all(), pos


def _shared_split_bytes(w):
    """The decode-sized shared-expert split's scratch, from its rule: T <= 256
    (at most two 128-row tiles), d and f_shared multiples of 64, 256-column
    tiles, splits dividing the 64-deep K steps within one wave of 148 CTAs
    (at most 16); used when the up projection splits at least twice."""
    if w.f_shared <= 0 or w.dtype != "bf16":
        return 0
    rt = (w.T + 127) // 128
    if rt > 2 or w.d % 64 or w.f_shared % 64:
        return 0

    def splits(kb, tiles):
        return max(s for s in range(1, min(16, kb) + 1) if kb % s == 0 and s * tiles <= 148)

    s_up = splits(w.d // 64, rt * ((w.f_shared + 255) // 256))
    s_dn = splits(w.f_shared // 64, rt * ((w.d + 255) // 256))
    if s_up < 2:
        return 0
    b = 2 * s_up * w.T * w.f_shared * 4 + (s_dn * w.T * w.d * 4 if s_dn > 1 else 0)
    return (b + 255) // 256 * 256


@pytest.mark.parametrize("w", [
    WORKLOADS["dsv3_decode"],                                            # 16 up, 4 down splits
    WORKLOADS["dsv3_decode"].scaled(T=200, d=448, f=64, f_shared=256),   # two row tiles
    WORKLOADS["dsv3_decode"].scaled(T=300),                              # three tiles: unsplit
    WORKLOADS["dsv3_decode"].scaled(f_shared=2040),                      # not in 64-steps
    WORKLOADS["dsv3_prefill"],                                           # prefill: unsplit
], ids=["dsv3_decode", "t200", "t300", "fsh2040", "prefill"])
def test_shared_split_workspace_follows_its_rule(w, monkeypatch):
    """The layer workspace holds the shared expert's split-K partial sums
    exactly when the split rule (mirrored by bench.py's launch count) applies."""
    cfg = ops.config(w)
    with_split = ops.moe_workspace_size(cfg, ops.WS_LAYER)
    monkeypatch.setenv("MOE_SHARED_SPLIT", "0")
    without = ops.moe_workspace_size(cfg, ops.WS_LAYER)
    assert with_split - without == _shared_split_bytes(w)
    import bench
    assert bench.shared_split_k(w) == (_shared_split_bytes(w) > 0)
