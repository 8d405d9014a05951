"""Pins for the CPU oracle, each against something other than the oracle itself.

Sources of truth used here: the hand-derived worked example in
tests/golden/quant_pack_worked_example.json, torch's BF16 conversion and
scipy's softmax (library routines), brute force on tiny inputs (nearest
quantisation level, top-k by explicit ranking, grouping by counting), a
closed-form combine, and the E=1/k=1 layer reducing to a dense SwiGLU written
with torch's linear/silu. Each pin is chosen so that a plausible slip in the
oracle (wrong divisor, rounding mode, nibble slot, tie-break, sort order,
token/expert index, transposed operand) fails at least one test.
"""
import itertools
import json
import os

import numpy as np
import pytest
import scipy.special
import torch

from oracle import exactmoe_oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quant_pack_worked_example.json")


def _bf16_values(rng, shape, std):
    v = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * np.float32(std))
    return v.to(torch.bfloat16).float().double().numpy()


# ---------------------------------------------------------------- BF16 rounding

def test_round_to_bf16_matches_torch_on_fp32_values():
    rng = np.random.default_rng(0)
    parts = [
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),   # subnormal range
        np.clip(rng.standard_normal(2000) * 1e38, -3.3e38, 3.3e38).astype(np.float32),  # near overflow
    ]
    # exact ties: a BF16 value plus half a BF16 ulp
    base = torch.from_numpy(rng.standard_normal(2000).astype(np.float32)).to(torch.bfloat16).float().numpy()
    ulp = np.ldexp(1.0, np.frexp(base.astype(np.float64))[1] - 8)
    parts.append((base.astype(np.float64) + ulp / 2).astype(np.float32))
    parts.append(np.array([0.0, -0.0, np.inf, -np.inf], dtype=np.float32))
    x = np.concatenate(parts)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().double().numpy()
    got = o.round_to_bf16(x.astype(np.float64))
    assert np.array_equal(got, ref)
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(o.f64_to_bf16_bits(ref), bits)
    assert np.array_equal(o.bf16_bits_to_f64(bits), ref)


# ---------------------------------------------------------------- quantiser

def _golden_rows():
    g = json.load(open(GOLDEN))
    w = np.zeros((len(g["rows"]), g["K"]))
    for r, row in enumerate(g["rows"]):
        for k, v in row["nonzero"].items():
            w[r, int(k)] = v
    return g, w


def test_worked_example_codes_scales_and_bytes():
    g, w = _golden_rows()
    q, s = o.quantize_group128(w)
    packed, sbits = o.quantize_pack(w)
    for r, row in enumerate(g["rows"]):
        assert list(q[r, :16]) == row["q_first16"]
        assert "%04x" % sbits[r, 0] == row["scale_bits"]
        assert packed[r, :8].tobytes().hex() == row["packed_first8_hex"]
        assert packed[r, 8:].tobytes().hex() == g["rest_of_row_byte_hex"] * 56
    assert np.array_equal(o.unpack_rows(packed), q)


def test_roundtrip_error_within_half_scale():
    rng = np.random.default_rng(1)
    w = _bf16_values(rng, (64, 512), 0.02)
    w[3, 128:256] = 0.0                                     # all-zero group
    w[5, :128] = 0.0
    w[5, 17] = -0.05                                        # one-hot group
    q, s = o.quantize_group128(w)
    deq = o.dequantize(q, s)
    bound = np.repeat(s, 128, axis=1) / 2
    assert np.all(np.abs(w - deq) <= bound * (1 + 2.0 ** -20))
    assert np.all((q >= -8) & (q <= 7))
    assert s[3, 1] == 0 and np.all(q[3, 128:256] == 0)
    assert q[5, 17] == -7 and np.count_nonzero(q[5, :128]) == 1


def test_codes_are_nearest_level_by_brute_force():
    rng = np.random.default_rng(2)
    w = _bf16_values(rng, (16, 256), 0.02)
    q, s = o.quantize_group128(w)
    levels = np.arange(-8, 8, dtype=np.float64)
    sfull = np.repeat(s, 128, axis=1)
    for n in range(w.shape[0]):
        for k in range(w.shape[1]):
            d = np.abs(w[n, k] - levels * sfull[n, k])
            best = levels[d == d.min()]
            want = best[0] if best.size == 1 else best[np.abs(best) % 2 == 0][0]   # tie: even
            assert q[n, k] == want, (n, k, w[n, k], sfull[n, k])


def test_scale_is_absmax_over_seven_rounded_to_bf16():
    rng = np.random.default_rng(3)
    w = _bf16_values(rng, (8, 384), 0.02)
    _, s = o.quantize_group128(w)
    absmax = np.abs(w).reshape(8, 3, 128).max(axis=2)
    ref = torch.from_numpy((absmax.astype(np.float32) / np.float32(7.0))).to(torch.bfloat16).double().numpy()
    assert np.array_equal(s, ref)


def test_packed_slot_positions_one_code_at_a_time():
    # A single non-default code at k lands in exactly one nibble: byte
    # (k//8)*4 + slot//2, high half iff slot is odd, slot = (k%8)//2 + 4*(k%2).
    for k in range(16):
        q = np.zeros((1, 16), dtype=np.int8)
        q[0, k] = 7                                             # u = 15
        b = o.pack_rows(q)[0]
        slot = (k % 8) // 2 + 4 * (k % 2)
        byte = (k // 8) * 4 + slot // 2
        expect = np.full(8, 0x88, dtype=np.uint8)
        expect[byte] = 0x8F if slot % 2 == 0 else 0xF8
        assert np.array_equal(b, expect), k


# ---------------------------------------------------------------- router / top-k

def test_router_logits_match_library_matmul():
    rng = np.random.default_rng(4)
    x = _bf16_values(rng, (5, 256), 1.0)
    wr = _bf16_values(rng, (8, 256), 0.02)
    ref = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(wr)).to(torch.bfloat16).double().numpy()
    got = o.router_logits(x, wr)
    # fp64 sum then one BF16 rounding vs fp64 sum -> fp64->bf16 in torch: same value
    assert np.array_equal(got, ref)


def test_router_logits_hand_computed():
    # integer-valued operands make every product and sum exact, so the values
    # below are worked by hand; E = 3 and H = 4 differ, so a transposed router
    # fails on shape, and each row of W picks out a different combination of x
    x = np.array([[1.0, -2.0, 3.0, 0.5],
                  [0.0, 1.0, 1.0, 1.0]])
    wr = np.array([[1.0, 1.0, 1.0, 1.0],       # sum of x
                   [2.0, 0.0, -1.0, 4.0],      # 2*x0 - x2 + 4*x3
                   [0.25, 0.0, 0.0, -8.0]])    # x0/4 - 8*x3
    want = np.array([[2.5, 1.0, -3.75],
                     [3.0, 3.0, -8.0]])
    assert np.array_equal(o.router_logits(x, wr), want)
    # the one rounding to BF16 (8 significant bits), ties to even: 257 and 259
    # lie halfway between neighbours 2 apart and go to 256 and 260; 257.5 is
    # just above the midpoint and goes to 258
    ones = np.ones((3, 1))
    xs = np.array([[257.0], [259.0], [257.5]])
    assert list(o.router_logits(xs, ones)[:, 0]) == [256.0, 260.0, 258.0]


def test_weights_for_given_ids():
    # probabilities of given ids are the full softmax at those ids, in the
    # order given (scipy); for the top-k ids they equal route_topk's weights;
    # renormalised ones sum to one
    rng = np.random.default_rng(9)
    T, E, k = 6, 10, 3
    logits = o.round_to_bf16(rng.standard_normal((T, E)))
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)])
    p = scipy.special.softmax(logits, axis=1)
    w = o.weights_for_ids(logits, ids)
    assert np.allclose(w, np.take_along_axis(p, ids, axis=1), rtol=1e-14, atol=0)
    wn = o.weights_for_ids(logits, ids, renorm=True)
    assert np.allclose(wn.sum(axis=1), 1.0, rtol=1e-14)
    assert np.allclose(wn, w / w.sum(axis=1, keepdims=True), rtol=1e-14)
    top, wt = o.route_topk(logits, k)
    assert np.array_equal(o.weights_for_ids(logits, top), wt)


def _brute_topk(key_row, k):
    E = len(key_row)
    keyv = [(-np.inf if np.isnan(v) else float(v)) for v in key_row]
    rank = [sum(1 for b in range(E) if keyv[b] > keyv[a] or (keyv[b] == keyv[a] and b < a)) for a in range(E)]
    chosen = sorted([a for a in range(E) if rank[a] < k], key=lambda a: rank[a])
    return chosen


@pytest.mark.parametrize("E,k", [(4, 1), (6, 2), (8, 3), (8, 8), (64, 8)])
def test_topk_matches_brute_force_rank(E, k):
    rng = np.random.default_rng(5 + E + k)
    T = 40
    logits = o.round_to_bf16(rng.standard_normal((T, E)) * 0.5)
    logits[0, :] = 0.0                                      # all tied
    logits[1, :] = logits[1, 0]
    logits[2, 1::2] = -0.0                                  # -0 and +0 tie
    logits[2, 0::2] = 0.0
    logits[3, E // 2] = np.nan                              # NaN never beats a number
    ids, _ = o.route_topk(logits, k)
    for t in range(T):
        assert list(ids[t]) == _brute_topk(o.routing_keys(logits)[t], k), t


def test_topk_with_bias_and_weights_against_scipy_softmax():
    rng = np.random.default_rng(6)
    T, E, k = 32, 16, 4
    logits = o.round_to_bf16(rng.standard_normal((T, E)))
    bias = np.log(np.arange(1, E + 1, dtype=np.float64) ** -1.2 / np.sum(np.arange(1, E + 1) ** -1.2)).astype(np.float32)
    ids, w = o.route_topk(logits, k, bias)
    keys = logits.astype(np.float32) + bias
    p = scipy.special.softmax(keys.astype(np.float64), axis=1)
    for t in range(T):
        assert list(ids[t]) == _brute_topk(keys[t], k)
        assert np.allclose(w[t], p[t, ids[t]], rtol=1e-14, atol=0)
    _, wn = o.route_topk(logits, k, bias, renorm=True)
    assert np.allclose(wn.sum(axis=1), 1.0, rtol=1e-14)
    assert np.all(w.sum(axis=1) < 1.0)


# ---------------------------------------------------------------- grouping

def test_grouping_by_counting():
    rng = np.random.default_rng(7)
    T, k, E = 37, 3, 9
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    ids[:5] = [0, 1, 2]                                     # dense expert 0..2, leaves gaps
    counts, offsets, sorted_pair, pair_pos = o.group_tokens(ids, E)
    flat = ids.reshape(-1)
    want_sorted = [p for e in range(E) for p in range(T * k) if flat[p] == e]
    assert list(sorted_pair) == want_sorted
    assert [int((flat == e).sum()) for e in range(E)] == list(counts)
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert all(offsets[e + 1] - offsets[e] == counts[e] for e in range(E))
    assert all(sorted_pair[pair_pos[p]] == p for p in range(T * k))
    with pytest.raises(ValueError):
        o.group_tokens(np.array([[0, E]]), E)


def test_grouping_empty_and_all_in_one():
    counts, offsets, sp, pp = o.group_tokens(np.zeros((0, 2), np.int32), 4)
    assert list(counts) == [0] * 4 and list(offsets) == [0] * 5 and sp.size == 0
    counts, offsets, sp, pp = o.group_tokens(np.full((6, 1), 2, np.int32), 4)
    assert list(counts) == [0, 0, 6, 0] and list(sp) == list(range(6))


# ---------------------------------------------------------------- FFN / layer

def _tiny_experts(rng, E, H, I):
    gate = np.stack([_bf16_values(rng, (I, H), 0.05) for _ in range(E)])
    up = np.stack([_bf16_values(rng, (I, H), 0.05) for _ in range(E)])
    down = np.stack([_bf16_values(rng, (H, I), 0.05) for _ in range(E)])
    return o.PackedExperts.from_bf16(gate, up, down)


def test_single_expert_top1_equals_dense_swiglu():
    rng = np.random.default_rng(8)
    T, H, I = 9, 256, 128
    ex = _tiny_experts(rng, 1, H, I)
    x = _bf16_values(rng, (T, H), 1.0)
    res = _bf16_values(rng, (T, H), 1.0)
    wr = _bf16_values(rng, (1, H), 0.02)
    out, logits, ids, w = o.moe_layer(x, wr, ex, 1, residual=res)
    assert np.all(ids == 0) and np.all(w == 1.0)
    wg, wu, wd = (torch.from_numpy(m) for m in ex.dequantized(0))
    xt = torch.from_numpy(x)
    F = torch.nn.functional
    h = (F.silu(F.linear(xt, wg)) * F.linear(xt, wu)).to(torch.bfloat16).double()
    ref = (torch.from_numpy(res) + F.linear(h, wd)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(out, ref)


def test_bf16_experts_top1_equals_dense_swiglu():
    # the BF16 baseline's experts are used unquantised: with one expert and
    # k = 1 the layer is a dense SwiGLU on the raw weights (torch), h rounded
    # to BF16, the output rounded to BF16
    rng = np.random.default_rng(21)
    T, H, I = 5, 256, 128
    x = _bf16_values(rng, (T, H), 1.0)
    wg, wu = _bf16_values(rng, (I, H), 0.05), _bf16_values(rng, (I, H), 0.05)
    wd = _bf16_values(rng, (H, I), 0.05)
    ex = o.Bf16Experts(lambda e: (wg, wu, wd), 1, H, I)
    ids = np.zeros((T, 1), dtype=np.int32)
    out = o.moe_layer_grouped(x, ex, ids, np.ones((T, 1)))
    xt = torch.from_numpy(x)
    g = torch.nn.functional.linear(xt, torch.from_numpy(wg))
    u = torch.nn.functional.linear(xt, torch.from_numpy(wu))
    h = (torch.nn.functional.silu(g) * u).to(torch.bfloat16).double()
    ref = torch.nn.functional.linear(h, torch.from_numpy(wd)).to(torch.bfloat16).double().numpy()
    assert np.mean(out == ref) > 0.99 and np.allclose(out, ref, rtol=2.0 ** -7, atol=1e-6)
    # and it differs from the quantised experts' layer on the same weights
    q = o.LazyQuantizedExperts(lambda e: (wg, wu, wd), 1, H, I)
    assert not np.array_equal(out, o.moe_layer_grouped(x, q, ids, np.ones((T, 1))))


def test_per_token_loop_equals_grouped_form():
    rng = np.random.default_rng(9)
    T, H, I, E, k = 24, 256, 128, 6, 2
    ex = _tiny_experts(rng, E, H, I)
    x = _bf16_values(rng, (T, H), 1.0)
    wr = _bf16_values(rng, (E, H), 0.02)
    logits = o.router_logits(x, wr)
    ids, w = o.route_topk(logits, k)
    ids[0] = [5, 4]                                         # experts out of index order
    a = o.moe_layer_grouped(x, ex, ids, w, residual=x)
    b = o.moe_layer_per_token(x, ex, ids, w, residual=x)
    # same math, different summation shapes: at most one BF16 ulp apart
    assert np.allclose(a, b, rtol=2.0 ** -7, atol=1e-6)
    assert np.mean(a == b) > 0.99


def test_combine_closed_form():
    T, k, H = 3, 2, 4
    ids = np.array([[1, 0], [0, 1], [1, 1]], dtype=np.int32)
    _, _, sorted_pair, pair_pos = o.group_tokens(ids, 2)
    # y row for pair p = constant (p + 1); weights 0.25 and 0.5
    y = np.zeros((T * k, H))
    for p in range(T * k):
        y[pair_pos[p]] = p + 1
    w = np.tile([0.25, 0.5], (T, 1))
    res = np.ones((T, H))
    out = o.combine(y, w, pair_pos, res)
    for t in range(T):
        assert np.all(out[t] == 1 + 0.25 * (2 * t + 1) + 0.5 * (2 * t + 2))


def test_combine_dropped_pair_equals_zero_weight():
    # a pair with pair_pos = -1 contributes exactly what a weight of 0 would
    rng = np.random.default_rng(5)
    T, k, H = 4, 3, 8
    y = rng.standard_normal((T * k, H))
    w = rng.random((T, k))
    pos = rng.permutation(T * k).astype(np.int64)
    res = rng.standard_normal((T, H))
    dropped = pos.copy()
    dropped[[1, 7]] = -1                     # pairs (0, 1) and (2, 1)
    w0 = w.copy()
    w0[0, 1] = 0.0
    w0[2, 1] = 0.0
    assert np.array_equal(o.combine(y, w, dropped, res), o.combine(y, w0, pos, res))



# ---------------------------------------------------------------- slot cache (A8)

LRU_GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "slot_cache_lru_trace.json")


def test_slot_cache_hand_worked_trace():
    g = json.load(open(LRU_GOLDEN))
    c = o.SlotCacheLRU(g["E"], g["slots"])
    for st in g["steps"]:
        if st.get("capacity_error"):
            with pytest.raises(o.SlotCapacityError):
                c.lookup(st["ids"])
        else:
            slots, loaded, evicted = c.lookup(st["ids"])
            assert slots == st["slot_of_ids"], st
            assert loaded == st["loaded"], st
            assert evicted == st["evicted"], st
        assert (c.hits, c.misses) == (st["hits"], st["misses"]), st
    r = g["resident"]
    c = o.SlotCacheLRU(r["E"], r["slots"])
    for st in r["steps"]:
        slots, loaded, evicted = c.lookup(st["ids"])
        assert (slots, loaded, evicted) == (st["slot_of_ids"], st["loaded"], [])
    assert (c.hits, c.misses, c.loads) == (r["hits"], r["misses"], r["loads"])
    assert c.h2d_bytes(1000) == 1000 * r["loads"]


def test_slot_cache_waves_hand_worked():
    g = json.load(open(LRU_GOLDEN))["waves"]
    c = o.SlotCacheLRU(g["E"], g["slots"])
    for st in g["steps"]:
        waves = c.plan_waves(st["ids"])
        assert waves == st["waves"], st
        for w, want in zip(waves, st["per_wave"]):
            slots, loaded, evicted = c.lookup(w)
            assert (slots, loaded, evicted) == (want["slot_of_ids"], want["loaded"], want["evicted"]), st
        assert (c.hits, c.misses) == (st["hits"], st["misses"]), st


def test_slot_cache_waves_cover_each_expert_once():
    # the waves of a step are a partition of its distinct ids, none larger
    # than the cache, held ids first; with S >= distinct there is one wave
    rng = np.random.default_rng(8)
    c = o.SlotCacheLRU(20, 4)
    for _ in range(100):
        ids = [int(v) for v in rng.integers(0, 20, size=rng.integers(1, 13))]
        held = {v for v in ids if c.slot_of(v) is not None}
        waves = c.plan_waves(ids)
        flat = [v for w in waves for v in w]
        assert sorted(flat) == sorted(set(ids)) and all(1 <= len(w) <= 4 for w in waves)
        assert set(flat[:len(held)]) == held
        for w in waves:
            c.lookup(w)
    assert o.SlotCacheLRU(20, 16).plan_waves([3, 1, 3, 7]) == [[3, 1, 7]]


@pytest.mark.parametrize("S", [1, 2, 3, 5, 8])
def test_slot_cache_one_id_per_step_equals_library_lru(S):
    # with one expert per step the policy is a plain LRU cache of S entries:
    # its hit count equals that of functools.lru_cache(maxsize=S) on the
    # same sequence of keys
    import functools
    rng = np.random.default_rng(S)
    seq = [int(v) for v in rng.integers(0, 9, size=400)]

    @functools.lru_cache(maxsize=S)
    def touch(e):
        return e

    c = o.SlotCacheLRU(9, S)
    for e in seq:
        touch(e)
        c.lookup([e])
    info = touch.cache_info()
    assert (c.hits, c.misses) == (info.hits, info.misses)


def test_slot_cache_cyclic_sweep_never_hits_and_invariants_hold():
    # a cyclic sweep over S + 1 experts defeats LRU completely (each expert
    # is evicted just before it comes back); S experts fit and always hit
    S = 4
    c = o.SlotCacheLRU(16, S)
    for r in range(5):
        for e in range(S + 1):
            c.lookup([e])
    assert c.hits == 0 and c.misses == 5 * (S + 1)
    c = o.SlotCacheLRU(16, S)
    for r in range(5):
        c.lookup(list(range(S)))
    assert (c.hits, c.misses) == (4 * S, S)
    # random multi-id steps: every id is held afterwards in distinct slots, an
    # evicted expert was not needed by the step, and the counters add up
    rng = np.random.default_rng(3)
    c = o.SlotCacheLRU(12, 5)
    lookups = 0
    for _ in range(300):
        ids = [int(v) for v in rng.integers(0, 12, size=rng.integers(1, 7))]
        if len(set(ids)) > 5:
            with pytest.raises(o.SlotCapacityError):
                c.lookup(ids)
            continue
        slots, loaded, evicted = c.lookup(ids)
        lookups += len(set(ids))
        held = {e: c.slot_of(e) for e in set(ids)}
        assert all(held[e] == s for e, s in zip(ids, slots))
        assert len(set(held.values())) == len(held)
        assert not set(evicted) & set(ids)
        assert set(loaded) <= set(ids)
    assert c.hits + c.misses == lookups
