"""ctypes binding of the C oracle (oracle/exactmoe_oracle.c).

TEST INFRASTRUCTURE ONLY: only tests/, __graft_entry__ and bench.py's
CPU-baseline/reference legs may import this module. It compiles the C file
with gcc on first use (or when the source is newer than the library) into
oracle/libexactmoe_oracle.so; it imports nothing from the CUDA package and
nothing from the numpy oracle. Arrays cross as BF16 bit patterns, int32 and
float64; every function mirrors the numpy oracle's function of the same name
so the two can be checked against each other.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "exactmoe_oracle.c")
LIB = os.path.join(HERE, "libexactmoe_oracle.so")
CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-std=c99", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile the C oracle unless an up-to-date library is present."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".%d.tmp" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"])
        os.replace(tmp, LIB)
    return LIB


_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        sig = {
            "eo_quantize_pack": (_I, [_P, _I, _I, _P, _P]),
            "eo_dequantize": (None, [_P, _P, _I, _I, _P]),
            "eo_router_logits": (None, [_P, _P, _I, _I, _I, _P]),
            "eo_route_topk": (_I, [_P, _P, _I, _I, _I, _I, _P, _P]),
            "eo_group_tokens": (_I, [_P, _I, _I, _I, _P, _P, _P, _P]),
            "eo_grouped_ffn": (_I, [_P, _I, _P, _P, _I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P]),
            "eo_combine": (None, [_P, _P, _P, _P, _I, _I, _I, _P]),
            "eo_layer_per_token": (_I, [_P, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P]),
            "eo_moe_layer": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                  _P]),
            "eo_threads": (_I, []),
            "eo_set_threads": (None, [_I]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def to_bits(v) -> np.ndarray:
    """BF16 bit patterns of BF16-representable values."""
    return (np.asarray(v, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def from_bits(b) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def threads() -> int:
    return int(lib().eo_threads())


def set_threads(n: int) -> None:
    lib().eo_set_threads(int(n))


# ------------------------------------------------------------------ A1

def quantize_pack(w):
    """BF16 weights [N][K] -> (packed uint8 [N][K/2], scale bits uint16 [N][K/128])."""
    wb = _c(to_bits(w), np.uint16)
    N, K = wb.shape
    packed = np.zeros((N, K // 2), dtype=np.uint8)
    scales = np.zeros((N, K // 128), dtype=np.uint16)
    if lib().eo_quantize_pack(_ptr(wb), N, K, _ptr(packed), _ptr(scales)) != 0:
        raise ValueError("K must be a multiple of 128")
    return packed, scales


def dequantize_packed(packed, scale_bits):
    p = _c(packed, np.uint8)
    s = _c(scale_bits, np.uint16)
    N, KB = p.shape
    out = np.zeros((N, KB * 2))
    lib().eo_dequantize(_ptr(p), _ptr(s), N, KB * 2, _ptr(out))
    return out


def quantize_pack_bits(wb):
    """quantize_pack of BF16 bit patterns (uint16 [N][K]) without a float copy."""
    wb = _c(wb, np.uint16)
    N, K = wb.shape
    packed = np.zeros((N, K // 2), dtype=np.uint8)
    scales = np.zeros((N, K // 128), dtype=np.uint16)
    if lib().eo_quantize_pack(_ptr(wb), N, K, _ptr(packed), _ptr(scales)) != 0:
        raise ValueError("K must be a multiple of 128")
    return packed, scales


def pack_experts(gate, up, down, bits: bool = False):
    """Quantise + pack [E][N][K] weights: (gq, gs, uq, us, dq, ds). The
    weights are BF16-valued floats, or BF16 bit patterns (uint16) with bits."""
    out = []
    for m in (gate, up, down):
        qs = [quantize_pack_bits(m[e]) if bits else quantize_pack(m[e]) for e in range(m.shape[0])]
        out.append(np.ascontiguousarray(np.stack([q for q, _ in qs])))
        out.append(np.ascontiguousarray(np.stack([s for _, s in qs])))
    return tuple(out)


# ------------------------------------------------------------------ A2, A3

def router_logits(x, wr):
    xb, wb = _c(to_bits(x), np.uint16), _c(to_bits(wr), np.uint16)
    T, H = xb.shape
    E = wb.shape[0]
    out = np.zeros((T, E), dtype=np.uint16)
    lib().eo_router_logits(_ptr(xb), _ptr(wb), T, H, E, _ptr(out))
    return from_bits(out)


def route_topk(logits, k: int, bias=None, renorm: bool = False):
    lb = _c(to_bits(logits), np.uint16)
    T, E = lb.shape
    b = None if bias is None else _c(bias, np.float32)
    ids = np.zeros((T, k), dtype=np.int32)
    w = np.zeros((T, k))
    if lib().eo_route_topk(_ptr(lb), _ptr(b), T, E, k, int(renorm), _ptr(ids), _ptr(w)) != 0:
        raise ValueError("need 1 <= k <= E")
    return ids, w


# ------------------------------------------------------------------ A4

def group_tokens(ids, E: int):
    d = _c(ids, np.int32)
    T, k = d.shape
    counts = np.zeros(E, dtype=np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    sp = np.zeros(T * k, dtype=np.int32)
    pp = np.zeros(T * k, dtype=np.int32)
    if lib().eo_group_tokens(_ptr(d), T, k, E, _ptr(counts), _ptr(offsets), _ptr(sp), _ptr(pp)) != 0:
        raise ValueError("expert id out of range")
    return counts, offsets, sp, pp


# ------------------------------------------------------------------ A5, A6, A7

def _packs(packs):
    gq, gs, uq, us, dq, ds = (_c(a, t) for a, t in zip(packs, (np.uint8, np.uint16) * 3))
    E, I, HB = gq.shape
    return (gq, gs, uq, us, dq, ds), E, HB * 2, I


def grouped_ffn(x, packs, sorted_pair, offsets, k: int):
    """h [P][I] (BF16 values) and y [P][H] (float64) in sorted order."""
    (gq, gs, uq, us, dq, ds), E, H, I = _packs(packs)
    xb = _c(to_bits(x), np.uint16)
    sp, off = _c(sorted_pair, np.int32), _c(offsets, np.int32)
    P = int(off[-1])
    h = np.zeros((P, I))
    y = np.zeros((P, H))
    st = lib().eo_grouped_ffn(_ptr(xb), xb.shape[0], _ptr(sp), _ptr(off), k, _ptr(gq), _ptr(gs), _ptr(uq),
                              _ptr(us), _ptr(dq), _ptr(ds), E, H, I, _ptr(h), _ptr(y))
    if st != 0:
        raise RuntimeError("eo_grouped_ffn failed (%d)" % st)
    return h, y


def combine(y_sorted, w, pair_pos, residual=None):
    y = _c(y_sorted, np.float64)
    ww = _c(w, np.float64)
    T, k = ww.shape
    H = y.shape[1]
    pp = _c(pair_pos, np.int32)
    rb = None if residual is None else _c(to_bits(residual), np.uint16)
    out = np.zeros((T, H), dtype=np.uint16)
    lib().eo_combine(_ptr(y), _ptr(ww), _ptr(pp), _ptr(rb), T, k, H, _ptr(out))
    return from_bits(out)


def layer_per_token(x, packs, ids, w, residual=None):
    (gq, gs, uq, us, dq, ds), E, H, I = _packs(packs)
    xb = _c(to_bits(x), np.uint16)
    d = _c(ids, np.int32)
    ww = _c(w, np.float64)
    T, k = d.shape
    rb = None if residual is None else _c(to_bits(residual), np.uint16)
    out = np.zeros((T, H), dtype=np.uint16)
    st = lib().eo_layer_per_token(_ptr(xb), _ptr(d), _ptr(ww), T, k, _ptr(gq), _ptr(gs), _ptr(uq), _ptr(us),
                                  _ptr(dq), _ptr(ds), E, H, I, _ptr(rb), _ptr(out))
    if st != 0:
        raise RuntimeError("eo_layer_per_token failed (%d)" % st)
    return from_bits(out)


def moe_layer(x, wr, packs, k: int, bias=None, renorm: bool = False, residual: bool = False):
    """Router -> top-k -> grouping -> grouped FFN -> combine: (out, logits, ids, w)."""
    (gq, gs, uq, us, dq, ds), E, H, I = _packs(packs)
    xb = _c(to_bits(x), np.uint16)
    wb = _c(to_bits(wr), np.uint16)
    T = xb.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    logits = np.zeros((T, E), dtype=np.uint16)
    ids = np.zeros((T, k), dtype=np.int32)
    w = np.zeros((T, k))
    out = np.zeros((T, H), dtype=np.uint16)
    st = lib().eo_moe_layer(_ptr(xb), _ptr(wb), T, H, I, E, k, _ptr(b), int(renorm), int(residual), _ptr(gq),
                            _ptr(gs), _ptr(uq), _ptr(us), _ptr(dq), _ptr(ds), _ptr(logits), _ptr(ids), _ptr(w),
                            _ptr(out))
    if st != 0:
        raise RuntimeError("eo_moe_layer failed (%d)" % st)
    return from_bits(out), from_bits(logits), ids, w
