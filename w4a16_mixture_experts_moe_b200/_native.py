"""ctypes binding of libexactmoe.so: the C ABI of include/exactmoe.h, same names.

Argument marshalling only. Pointer arguments accept a torch tensor (its
data_ptr), a plain int address, or None (NULL). Stream arguments accept a
torch.cuda.Stream, a raw cudaStream_t int, or None (torch's current stream).
A non-zero status raises MoeError with the library's message. There is no
fallback: if the library is missing the import of this module fails.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libexactmoe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m w4a16_mixture_experts_moe_b200.build` "
        "(the MoE layer has no CPU or Python fallback)")

lib = C.CDLL(LIB_PATH)

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_SHAPE, MOE_ERR_CUDA, MOE_ERR_CAPACITY, MOE_ERR_DEVICE, MOE_ERR_UNSUPPORTED = range(7)
MOE_DEVERR_NONE, MOE_DEVERR_EXPERT_ID, MOE_DEVERR_NOT_RESIDENT, MOE_DEVERR_TIMEOUT, MOE_DEVERR_RANGE = range(5)
MOE_RENORM, MOE_LOGITS_GIVEN, MOE_IDS_GIVEN = 1, 2, 4
MOE_PATH_AUTO, MOE_PATH_GEMV, MOE_PATH_TC, MOE_PATH_SEQUENTIAL = 0, 1, 2, 3
MOE_SLOT_SKIP = -2
MOE_FFN_X_F16 = 0x100

_p = C.c_void_p
_i = C.c_int
_i64 = C.c_int64
_sz = C.c_size_t


class moe_record_layout(C.Structure):
    _fields_ = [("gate_q", _i64), ("up_q", _i64), ("down_q", _i64),
                ("gate_s", _i64), ("up_s", _i64), ("down_s", _i64), ("bytes", _i64)]


class moe_bf16_layout(C.Structure):
    _fields_ = [("gate", _i64), ("up", _i64), ("down", _i64), ("bytes", _i64)]


class moe_pool_info(C.Structure):
    _fields_ = [("layers", C.c_int32), ("E", C.c_int32), ("H", C.c_int32), ("I", C.c_int32),
                ("record_bytes", _i64)]


# name -> (restype, argtypes); kept in the order of include/exactmoe.h
SIGNATURES = {
    "moe_last_error": (C.c_char_p, []),
    "moe_abi_version": (_i, []),
    "moe_launch_counter": (C.c_uint64, []),
    "moe_expert_record_layout": (_i, [_i, _i, C.POINTER(moe_record_layout)]),
    "moe_quantize_pack": (_i, [_p, _i, _i, _i, _p, _i64, _p, _i64, _p]),
    "moe_route_topk": (_i, [_p, _p, _i, _i, _i, _i, _p, _i, _p, _p, _p, _p]),
    "moe_route_topk_x16": (_i, [_p, _p, _i, _i, _i, _i, _p, _i, _p, _p, _p, _p, _p, _p]),
    "moe_group_workspace_size": (_sz, [_i, _i, _i]),
    "moe_group_tokens": (_i, [_p, _i, _i, _i, _p, _p, _p, _p, _p, _sz, _p]),
    "moe_group_tokens_noalloc": (_i, [_p, _i, _i, _i, _p, _p, _p, _p, _p]),
    "moe_ffn_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "moe_grouped_w4a16_ffn": (_i, [_p, _p, _p, _p, _i64, _p, _i, _i, _i, _i, _i, _i, _i, _p, _p, _sz, _p]),
    "moe_bf16_record_layout": (_i, [_i, _i, C.POINTER(moe_bf16_layout)]),
    "moe_bf16_ffn_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "moe_grouped_bf16_ffn": (_i, [_p, _p, _p, _p, _i64, _i, _i, _i, _i, _i, _p, _p, _sz, _p]),
    "moe_debug_stall_next_tc_ffn": (_i, [_i]),
    "moe_combine": (_i, [_p, _p, _p, _p, _i, _i, _i, _p, _p]),
    "moe_read_device_error": (_i, [_p, _p, C.POINTER(C.c_int32)]),
    "slot_cache_create": (_i, [C.POINTER(_p), _i, _i, _i, _i64, _p, _p, _p]),
    "slot_cache_lookup": (_i, [_p, _i, _p, _i, _p, _p, C.POINTER(_i)]),
    "slot_cache_fill": (_i, [_p, _i, _p, _i, _p, _p]),
    "slot_cache_release": (_i, [_p, _i, _p]),
    "slot_cache_plan_waves": (_i, [_p, _i, _p, _i, _p, _p, C.POINTER(_i)]),
    "slot_cache_stats": (_i, [_p, C.POINTER(C.c_uint64), C.POINTER(C.c_uint64), C.POINTER(C.c_uint64)]),
    "slot_cache_inject_fill_failure": (_i, [_p, _i]),
    "slot_cache_destroy": (None, [_p]),
    "moe_pool_save": (_i, [C.c_char_p, C.POINTER(moe_pool_info), _p]),
    "moe_pool_file_info": (_i, [C.c_char_p, C.POINTER(moe_pool_info)]),
    "moe_pool_load": (_i, [C.c_char_p, _p, _sz, C.POINTER(moe_pool_info)]),
}

for _name, (_res, _args) in SIGNATURES.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class MoeError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"[status {status}] {message}")
        self.status = status


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _addr(arr):
    return C.cast(arr, C.c_void_p).value


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int):
    if status != MOE_OK:
        raise MoeError(status, lib.moe_last_error().decode())


def moe_last_error() -> str:
    return lib.moe_last_error().decode()


def moe_abi_version() -> int:
    return lib.moe_abi_version()


def moe_launch_counter() -> int:
    return lib.moe_launch_counter()


def moe_expert_record_layout(H: int, I: int) -> dict:
    out = moe_record_layout()
    _check(lib.moe_expert_record_layout(H, I, C.byref(out)))
    return {f: getattr(out, f) for f, _ in moe_record_layout._fields_}


def moe_quantize_pack(w, E, N, K, packed, packed_stride, scales, scales_stride, stream=None):
    _check(lib.moe_quantize_pack(_ptr(w), E, N, K, _ptr(packed), packed_stride, _ptr(scales), scales_stride,
                                 _stream(stream)))


def moe_route_topk(x, w_router, T, H, E, k, bias, flags, logits, topk_ids, topk_w, stream=None):
    _check(lib.moe_route_topk(_ptr(x), _ptr(w_router), T, H, E, k, _ptr(bias), flags, _ptr(logits),
                              _ptr(topk_ids), _ptr(topk_w), _stream(stream)))


def moe_route_topk_x16(x, w_router, T, H, E, k, bias, flags, logits, topk_ids, topk_w, x16, err=None, stream=None):
    _check(lib.moe_route_topk_x16(_ptr(x), _ptr(w_router), T, H, E, k, _ptr(bias), flags, _ptr(logits),
                                  _ptr(topk_ids), _ptr(topk_w), _ptr(x16), _ptr(err), _stream(stream)))


def moe_group_workspace_size(T, k, E) -> int:
    return lib.moe_group_workspace_size(T, k, E)


def moe_group_tokens(topk_ids, T, k, E, counts, offsets, sorted_pair, pair_pos, ws, ws_bytes, stream=None):
    _check(lib.moe_group_tokens(_ptr(topk_ids), T, k, E, _ptr(counts), _ptr(offsets), _ptr(sorted_pair),
                                _ptr(pair_pos), _ptr(ws), ws_bytes, _stream(stream)))


def moe_group_tokens_noalloc(topk_ids, T, k, E, counts, offsets, sorted_pair, pair_pos, stream=None):
    """moe_group_tokens with the library's fixed scratch (no workspace); see include/exactmoe.h."""
    _check(lib.moe_group_tokens_noalloc(_ptr(topk_ids), T, k, E, _ptr(counts), _ptr(offsets), _ptr(sorted_pair),
                                        _ptr(pair_pos), _stream(stream)))


MOE_NOALLOC_MAX_PAIRS = 65536


def moe_ffn_workspace_size(T, k, E, H, I, path=MOE_PATH_AUTO) -> int:
    return lib.moe_ffn_workspace_size(T, k, E, H, I, path)


def moe_grouped_w4a16_ffn(x, sorted_pair, offsets, bank, record_bytes, expert_slot, n_slots, T, k, E, H, I, path,
                          y, ws, ws_bytes, stream=None):
    _check(lib.moe_grouped_w4a16_ffn(_ptr(x), _ptr(sorted_pair), _ptr(offsets), _ptr(bank), record_bytes,
                                     _ptr(expert_slot), n_slots, T, k, E, H, I, path, _ptr(y), _ptr(ws), ws_bytes,
                                     _stream(stream)))


def moe_bf16_record_layout(H: int, I: int) -> dict:
    out = moe_bf16_layout()
    _check(lib.moe_bf16_record_layout(H, I, C.byref(out)))
    return {f: getattr(out, f) for f, _ in moe_bf16_layout._fields_}


def moe_bf16_ffn_workspace_size(T, k, E, H, I) -> int:
    return lib.moe_bf16_ffn_workspace_size(T, k, E, H, I)


def moe_grouped_bf16_ffn(x, sorted_pair, offsets, bank, record_bytes, T, k, E, H, I, y, ws, ws_bytes,
                         stream=None):
    _check(lib.moe_grouped_bf16_ffn(_ptr(x), _ptr(sorted_pair), _ptr(offsets), _ptr(bank), record_bytes, T, k, E,
                                    H, I, _ptr(y), _ptr(ws), ws_bytes, _stream(stream)))


def moe_debug_stall_next_tc_ffn(calls: int):
    """Test hook: the next `calls` tensor-core FFN launches time out on purpose."""
    _check(lib.moe_debug_stall_next_tc_ffn(calls))


def moe_combine(y, topk_w, pair_pos, residual, T, k, H, out, stream=None):
    _check(lib.moe_combine(_ptr(y), _ptr(topk_w), _ptr(pair_pos), _ptr(residual), T, k, H, _ptr(out),
                           _stream(stream)))


def moe_read_device_error(ws, stream=None) -> int:
    """Synchronises, returns the device error code of the workspace and clears it."""
    code = C.c_int32(0)
    st = lib.moe_read_device_error(_ptr(ws), _stream(stream), C.byref(code))
    if st not in (MOE_OK, MOE_ERR_DEVICE):
        _check(st)
    return code.value


class SlotCache:
    """Owner of a moe_slot_cache handle; methods map 1:1 onto slot_cache_*."""

    def __init__(self, layers, E, slots, record_bytes, pinned_pool, device_slots, expert_slot):
        h = C.c_void_p()
        _check(lib.slot_cache_create(C.byref(h), layers, E, slots, record_bytes, _ptr(pinned_pool),
                                     _ptr(device_slots), _ptr(expert_slot)))
        self.h = h
        self.E = E

    def lookup(self, layer, ids):
        """ids: sequence of ints. Returns (slot_of_id list, miss_ids list)."""
        n = len(ids)
        arr = (C.c_int32 * max(n, 1))(*ids)
        slot = (C.c_int32 * max(n, 1))()
        miss = (C.c_int32 * max(n, 1))()
        nm = C.c_int(0)
        _check(lib.slot_cache_lookup(self.h, layer, _addr(arr), n, _addr(slot), _addr(miss), C.byref(nm)))
        return list(slot[:n]), list(miss[:nm.value])

    def fill(self, layer, miss_ids, side=None, compute=None):
        n = len(miss_ids)
        arr = (C.c_int32 * max(n, 1))(*miss_ids)
        _check(lib.slot_cache_fill(self.h, layer, _addr(arr), n, _stream(side), _stream(compute)))

    def release(self, layer, compute=None):
        _check(lib.slot_cache_release(self.h, layer, _stream(compute)))

    def plan_waves(self, layer, ids):
        """ids: sequence of ints. Returns the waves as lists of distinct ids."""
        n = len(ids)
        arr = (C.c_int32 * max(n, 1))(*ids)
        wid = (C.c_int32 * max(n, 1))()
        wst = (C.c_int32 * (n + 1))()
        nw = C.c_int(0)
        _check(lib.slot_cache_plan_waves(self.h, layer, _addr(arr), n, _addr(wid), _addr(wst), C.byref(nw)))
        return [list(wid[wst[w]:wst[w + 1]]) for w in range(nw.value)]

    def stats(self):
        h, m, b = C.c_uint64(), C.c_uint64(), C.c_uint64()
        _check(lib.slot_cache_stats(self.h, C.byref(h), C.byref(m), C.byref(b)))
        return {"hits": h.value, "misses": m.value, "h2d_bytes": b.value}

    def inject_fill_failure(self, count):
        _check(lib.slot_cache_inject_fill_failure(self.h, count))

    def close(self):
        if self.h:
            lib.slot_cache_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _info_dict(info):
    return {f: getattr(info, f) for f, _ in moe_pool_info._fields_}


def moe_pool_save(path, layers, E, H, I, record_bytes, pool):
    """Writes the host pool (a tensor, numpy array via its address, or int) to path."""
    info = moe_pool_info(layers, E, H, I, record_bytes)
    addr = pool if isinstance(pool, int) else (pool.ctypes.data if hasattr(pool, "ctypes") else pool.data_ptr())
    _check(lib.moe_pool_save(os.fsencode(path), C.byref(info), addr))


def moe_pool_file_info(path) -> dict:
    info = moe_pool_info()
    _check(lib.moe_pool_file_info(os.fsencode(path), C.byref(info)))
    return _info_dict(info)


def moe_pool_load(path, pool, capacity) -> dict:
    """Reads path's records into the host buffer `pool` of `capacity` bytes."""
    info = moe_pool_info()
    addr = pool if isinstance(pool, int) else (pool.ctypes.data if hasattr(pool, "ctypes") else pool.data_ptr())
    _check(lib.moe_pool_load(os.fsencode(path), addr, capacity, C.byref(info)))
    return _info_dict(info)
