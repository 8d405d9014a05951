"""The C-ABI library loads on a machine without a GPU, exports every entry
point include/*.h declares, and rejects bad arguments before touching CUDA.
The slot cache's host bookkeeping (LRU, capacity, rollback on an injected
fill failure) runs here too: lookups touch no device memory."""
import ctypes as C
import glob
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_ ]*[\s\*]+\**([a-z_][a-z0-9_]*)\s*\(", src, re.M):
            names.append(m.group(1))
    return sorted(set(names))


@pytest.fixture(scope="module")
def native():
    from w4a16_mixture_experts_moe_b200 import build
    build.build()
    from w4a16_mixture_experts_moe_b200 import _native
    return _native


def test_header_declares_the_boundary():
    names = _declared_functions()
    for want in ["moe_quantize_pack", "moe_route_topk", "moe_group_tokens", "moe_grouped_w4a16_ffn",
                 "moe_combine", "slot_cache_lookup", "slot_cache_fill"]:
        assert want in names


def test_library_exports_every_declared_symbol(native):
    lib = C.CDLL(native.LIB_PATH)
    names = _declared_functions()
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert set(names) <= set(native.SIGNATURES), set(names) - set(native.SIGNATURES)


def test_record_layout(native):
    L = native.moe_expert_record_layout(2048, 1024)
    assert L["bytes"] == 3 * 1024 * 2048 // 2 + 3 * (1024 * 2048 // 128) * 2 == 3244032
    assert all(v % 256 == 0 for v in L.values())
    with pytest.raises(native.MoeError) as ei:
        native.moe_expert_record_layout(2048, 1000)
    assert ei.value.status == 2


def test_argument_checks_run_before_any_cuda_call(native):
    lib = native.lib
    assert lib.moe_quantize_pack(16, 1, 1, 100, 16, 0, 16, 0, None) == native.MOE_ERR_SHAPE
    assert b"K=100" in lib.moe_last_error()
    assert lib.moe_route_topk(16, 16, 4, 256, 300, 2, None, 0, 16, 16, 16, None) == native.MOE_ERR_SHAPE
    assert lib.moe_route_topk(16, 16, 4, 256, 8, 9, None, 0, 16, 16, 16, None) == native.MOE_ERR_SHAPE
    assert lib.moe_route_topk(16, 16, 4, 256, 8, 2, None, 64, 16, 16, 16, None) == native.MOE_ERR_INVALID_ARG
    assert lib.moe_group_tokens(16, 4, 2, 8, 16, 16, 16, 16, 256, 1, None) == native.MOE_ERR_INVALID_ARG
    assert lib.moe_grouped_w4a16_ffn(16, 16, 16, 256, 3244032, None, 64, 4, 8, 64, 2048, 1000, 0,
                                     16, 256, 1 << 20, None) == native.MOE_ERR_SHAPE
    assert lib.moe_grouped_w4a16_ffn(16, 16, 16, 256, 1000, None, 64, 4, 8, 64, 2048, 1024, 0,
                                     16, 256, 1 << 20, None) == native.MOE_ERR_INVALID_ARG
    assert lib.moe_grouped_w4a16_ffn(16, 16, 16, 256, 3244032, None, 64, 4, 8, 64, 2048, 1024, 7,
                                     16, 256, 1 << 20, None) == native.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(16, 16, 16, None, 4, 40, 2048, 16, None) == native.MOE_ERR_SHAPE
    # T == 0 is a no-op that launches nothing
    assert lib.moe_combine(None, None, None, None, 0, 2, 2048, None, None) == native.MOE_OK
    assert lib.moe_route_topk(None, None, 0, 2048, 64, 8, None, 0, None, None, None, None) == native.MOE_OK
    # the FP16-copy variant needs x and x16 (also with given logits) and H a multiple of 8
    assert lib.moe_route_topk_x16(16, 16, 4, 2048, 64, 8, None, 0, 16, 16, 16, None, None, None) == \
        native.MOE_ERR_INVALID_ARG
    assert lib.moe_route_topk_x16(None, 16, 4, 2048, 64, 8, None, 2, 16, 16, 16, 16, None, None) == \
        native.MOE_ERR_INVALID_ARG
    assert lib.moe_route_topk_x16(16, 16, 4, 2044, 64, 8, None, 0, 16, 16, 16, 16, None, None) == \
        native.MOE_ERR_SHAPE
    assert lib.moe_route_topk_x16(16, 16, 4, 2048, 64, 8, None, 0, 16, 16, 16, 24, None, None) == \
        native.MOE_ERR_INVALID_ARG  # x16 not 16-byte aligned
    assert lib.moe_route_topk_x16(None, None, 0, 2048, 64, 8, None, 0, None, None, None, None, None, None) == \
        native.MOE_OK
    # the FP16-input flag is stripped before the path check, an unknown bit is not
    assert lib.moe_grouped_w4a16_ffn(16, 16, 16, 256, 3244032, None, 64, 4, 8, 64, 2048, 1024, 0x100 | 7,
                                     16, 256, 1 << 20, None) == native.MOE_ERR_INVALID_ARG
    assert native.moe_ffn_workspace_size(16, 8, 64, 2048, 1024, 0x100 | 1) == \
        native.moe_ffn_workspace_size(16, 8, 64, 2048, 1024, 1)


def test_slot_cache_lru_matches_oracle(native):
    """The library's host LRU against the oracle's slot-cache policy."""
    import synth
    from oracle import exactmoe_oracle as o
    E, S, k, steps = 64, 16, 8, 200
    c = native.SlotCache(1, E, S, 256, None, None, None)   # no memory: simulates the policy
    model = o.SlotCacheLRU(E, S)
    routing = synth.drawn_routing(0, E, k, steps)
    for s in range(steps):
        ids = [int(v) for v in routing[s]]
        got = c.lookup(0, ids)
        slots, loaded, _ = model.lookup(ids)
        assert got == (slots, loaded), s
        c.fill(0, got[1], side=0, compute=0)         # simulated: counts the copies
        # every id maps to a distinct slot this step
        assert len(set(got[0])) == len(ids)
    st = c.stats()
    assert (st["hits"], st["misses"]) == (model.hits, model.misses)
    assert st["h2d_bytes"] == model.h2d_bytes(256)
    # keep-probability 0.5 routing over 16 slots: a fair share of hits
    assert 0.3 < st["hits"] / (st["hits"] + st["misses"]) < 0.9
    c.close()


def test_slot_cache_capacity_duplicates_and_resident_mode(native):
    c = native.SlotCache(2, 8, 2, 256, None, None, None)
    with pytest.raises(native.MoeError) as ei:
        c.lookup(0, [0, 1, 2])
    assert ei.value.status == native.MOE_ERR_CAPACITY
    slots, miss = c.lookup(1, [5, 5, 5])
    assert len(set(slots)) == 1 and miss == [5]
    c.close()
    r = native.SlotCache(1, 8, 8, 256, None, None, None)
    slots, miss = r.lookup(0, [3, 1])
    assert slots == [3, 1] and miss == [3, 1]          # first touch loads
    r.fill(0, miss, side=0, compute=0)
    slots, miss = r.lookup(0, [3, 1, 7])
    assert slots == [3, 1, 7] and miss == [7]
    assert r.stats() == {"hits": 0, "misses": 0, "h2d_bytes": 2 * 256}   # accounting bypassed; first loads copied
    r.close()


def test_slot_cache_injected_fill_failure_rolls_back(native):
    c = native.SlotCache(1, 8, 4, 256, None, None, None)
    _, miss = c.lookup(0, [1, 2])
    c.inject_fill_failure(1)
    with pytest.raises(native.MoeError) as ei:
        c.fill(0, miss, side=0, compute=0)
    assert ei.value.status == native.MOE_ERR_CUDA and "injected" in str(ei.value)
    # the failed experts are not resident: the next lookup misses them again
    _, miss2 = c.lookup(0, [1, 2])
    assert sorted(miss2) == [1, 2]
    with pytest.raises(native.MoeError):
        c.fill(0, [5], side=0, compute=0)                 # never assigned by a lookup
    c.close()


def test_slot_cache_lookup_without_fill_is_undone(native):
    # a lookup whose misses were never copied must not leave them "resident":
    # the next lookup misses them again rather than reading stale slot bytes
    c = native.SlotCache(1, 8, 4, 256, None, None, None)
    _, miss = c.lookup(0, [1, 2])
    assert miss == [1, 2]
    _, miss = c.lookup(0, [1, 2])                         # no fill in between
    assert miss == [1, 2]
    c.fill(0, miss, side=0, compute=0)
    _, miss = c.lookup(0, [1, 2, 3])
    assert miss == [3]
    st = c.stats()
    assert st["hits"] == 2 and st["h2d_bytes"] == 2 * 256   # the unfilled lookup copied nothing
    c.close()


def test_slot_cache_needs_all_memories_or_none(native):
    with pytest.raises(native.MoeError) as ei:
        native.SlotCache(1, 8, 4, 256, None, 0x2000, None)
    assert ei.value.status == native.MOE_ERR_INVALID_ARG


def test_slot_cache_waves_match_oracle(native):
    """Steps needing more experts than slots run in waves: the library's plan
    and each wave's lookup match the oracle's policy (simulation mode)."""
    import synth
    from oracle import exactmoe_oracle as o
    E, S, k, T, steps = 64, 16, 8, 4, 60
    c = native.SlotCache(1, E, S, 256, None, None, None)
    model = o.SlotCacheLRU(E, S)
    rng = np.random.default_rng(17)
    waves_seen = 0
    for s in range(steps):
        ids = [int(v) for v in rng.integers(0, E, size=T * k)] if s % 3 else \
              [int(v) for v in synth.drawn_routing(0, E, k, steps)[s]]
        waves = c.plan_waves(0, ids)
        assert waves == model.plan_waves(ids), s
        waves_seen += len(waves)
        for w in waves:
            got = c.lookup(0, w)
            slots, loaded, _ = model.lookup(w)
            assert got == (slots, loaded), s
            c.fill(0, got[1], side=0, compute=0)
    st = c.stats()
    assert (st["hits"], st["misses"], st["h2d_bytes"]) == (model.hits, model.misses, model.h2d_bytes(256))
    assert waves_seen > steps                       # some steps needed more than one wave
    c.close()
