"""Pins for the C oracle (oracle/exactmoe_oracle.c), and cross-checks of the
two oracles, which were written independently from the same definitions.

The pins mirror those of the numpy oracle: the hand-derived worked example
(tests/golden), the round-trip bound |w - q s| <= s/2, torch's BF16 rounding
of a library matmul, brute-force top-k ranking and scipy's softmax, grouping
by counting, a closed-form combine, and the E=1/k=1 layer reducing to a dense
SwiGLU written with torch. The cross-checks then ask the two oracles to agree
bit for bit on every integer and BF16 result, and to 1e-12 relative on fp64
ones, on random layers.
"""
import json
import os

import numpy as np
import pytest
import scipy.special
import torch

from oracle import c_oracle as c
from oracle import exactmoe_oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quant_pack_worked_example.json")


def _bf16_values(rng, shape, std):
    v = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * np.float32(std))
    return v.to(torch.bfloat16).float().double().numpy()


def _codes(packed):
    """int4 codes of packed rows, decoded here from the layout's definition."""
    p = np.asarray(packed, dtype=np.uint8)
    N, KB = p.shape
    q = np.zeros((N, KB * 2), dtype=np.int64)
    for k in range(KB * 2):
        j, i, h = k // 8, (k % 8) // 2, k % 2
        word = (p[:, 4 * j].astype(np.int64) | (p[:, 4 * j + 1].astype(np.int64) << 8) |
                (p[:, 4 * j + 2].astype(np.int64) << 16) | (p[:, 4 * j + 3].astype(np.int64) << 24))
        q[:, k] = ((word >> (4 * (i + 4 * h))) & 0xF) - 8
    return q


def test_builds_and_reports_threads():
    c.build()
    assert c.threads() >= 1


def test_worked_example_codes_scales_and_bytes():
    g = json.load(open(GOLDEN))
    w = np.zeros((len(g["rows"]), g["K"]))
    for r, row in enumerate(g["rows"]):
        for k, v in row["nonzero"].items():
            w[r, int(k)] = v
    packed, sbits = c.quantize_pack(w)
    q = _codes(packed)
    for r, row in enumerate(g["rows"]):
        assert list(q[r, :16]) == row["q_first16"]
        assert "%04x" % sbits[r, 0] == row["scale_bits"]
        assert packed[r, :8].tobytes().hex() == row["packed_first8_hex"]
        assert packed[r, 8:].tobytes().hex() == g["rest_of_row_byte_hex"] * 56


def test_roundtrip_error_within_half_scale_and_scale_definition():
    rng = np.random.default_rng(1)
    w = _bf16_values(rng, (32, 512), 0.02)
    w[3, 128:256] = 0.0
    packed, sbits = c.quantize_pack(w)
    s = c.from_bits(sbits)
    deq = c.dequantize_packed(packed, sbits)
    assert np.array_equal(deq, _codes(packed) * np.repeat(s, 128, axis=1))
    assert np.all(np.abs(w - deq) <= np.repeat(s, 128, axis=1) / 2 * (1 + 2.0 ** -20))
    absmax = np.abs(w).reshape(32, 4, 128).max(axis=2)
    ref = torch.from_numpy(absmax.astype(np.float32) / np.float32(7.0)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(s, ref)
    assert s[3, 1] == 0 and np.all(_codes(packed)[3, 128:256] == 0)


def test_codes_are_nearest_level_by_brute_force():
    rng = np.random.default_rng(2)
    w = _bf16_values(rng, (8, 256), 0.02)
    packed, sbits = c.quantize_pack(w)
    q, s = _codes(packed), np.repeat(c.from_bits(sbits), 128, axis=1)
    levels = np.arange(-8, 8, dtype=np.float64)
    for n in range(w.shape[0]):
        for k in range(w.shape[1]):
            d = np.abs(w[n, k] - levels * s[n, k])
            best = levels[d == d.min()]
            want = best[0] if best.size == 1 else best[np.abs(best) % 2 == 0][0]
            assert q[n, k] == want, (n, k)


def test_router_logits_match_library_matmul():
    rng = np.random.default_rng(4)
    x = _bf16_values(rng, (5, 256), 1.0)
    wr = _bf16_values(rng, (8, 256), 0.02)
    ref = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(wr)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(c.router_logits(x, wr), ref)


def _brute_topk(keys, k):
    E = len(keys)
    kv = [(-np.inf if np.isnan(v) else float(v)) for v in keys]
    rank = [sum(1 for b in range(E) if kv[b] > kv[a] or (kv[b] == kv[a] and b < a)) for a in range(E)]
    return sorted([a for a in range(E) if rank[a] < k], key=lambda a: rank[a])


@pytest.mark.parametrize("E,k", [(4, 1), (8, 3), (8, 8), (64, 8)])
def test_topk_brute_force_and_scipy_softmax(E, k):
    rng = np.random.default_rng(5 + E + k)
    T = 30
    logits = c.from_bits(c.to_bits(rng.standard_normal((T, E)) * 0.5))
    logits[0, :] = 0.0
    logits[2, 1::2] = -0.0
    logits[2, 0::2] = 0.0
    logits[3, E // 2] = np.nan
    bias = (rng.standard_normal(E) * 0.1).astype(np.float32)
    for b in (None, bias):
        ids, w = c.route_topk(logits, k, b)
        keys = logits.astype(np.float32) + (0 if b is None else b)
        keys = np.where(np.isnan(keys), np.float32(-np.inf), keys)
        p = scipy.special.softmax(keys.astype(np.float64), axis=1)
        for t in range(T):
            assert list(ids[t]) == _brute_topk(keys[t], k), t
            assert np.allclose(w[t], p[t, ids[t]], rtol=1e-14, atol=0)
    _, wn = c.route_topk(logits, k, bias, renorm=True)
    assert np.allclose(wn.sum(axis=1), 1.0, rtol=1e-14)


def test_grouping_by_counting():
    rng = np.random.default_rng(7)
    T, k, E = 37, 3, 9
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, sp, pp = c.group_tokens(ids, E)
    flat = ids.reshape(-1)
    assert list(sp) == [p for e in range(E) for p in range(T * k) if flat[p] == e]
    assert list(counts) == [int((flat == e).sum()) for e in range(E)]
    assert list(offsets) == [0] + list(np.cumsum(counts))
    assert all(sp[pp[p]] == p for p in range(T * k))
    counts, offsets, sp, _ = c.group_tokens(np.zeros((0, 2), np.int32), 4)
    assert list(counts) == [0] * 4 and list(offsets) == [0] * 5 and sp.size == 0
    with pytest.raises(ValueError):
        c.group_tokens(np.array([[0, E]]), E)


def test_combine_closed_form_and_dropped_pair():
    T, k, H = 3, 2, 4
    ids = np.array([[1, 0], [0, 1], [1, 1]], dtype=np.int32)
    _, _, _, pp = c.group_tokens(ids, 2)
    y = np.zeros((T * k, H))
    for p in range(T * k):
        y[pp[p]] = p + 1
    w = np.tile([0.25, 0.5], (T, 1))
    out = c.combine(y, w, pp, np.ones((T, H)))
    for t in range(T):
        assert np.all(out[t] == 1 + 0.25 * (2 * t + 1) + 0.5 * (2 * t + 2))
    dropped = pp.copy()
    dropped[1] = -1
    w0 = w.copy()
    w0[0, 1] = 0.0
    assert np.array_equal(c.combine(y, w, dropped, np.ones((T, H))), c.combine(y, w0, pp, np.ones((T, H))))


def _experts(rng, E, H, I):
    gate = np.stack([_bf16_values(rng, (I, H), 0.05) for _ in range(E)])
    up = np.stack([_bf16_values(rng, (I, H), 0.05) for _ in range(E)])
    down = np.stack([_bf16_values(rng, (H, I), 0.05) for _ in range(E)])
    return gate, up, down


def test_single_expert_top1_equals_dense_swiglu():
    rng = np.random.default_rng(8)
    T, H, I = 9, 256, 128
    gate, up, down = _experts(rng, 1, H, I)
    packs = c.pack_experts(gate, up, down)
    x = _bf16_values(rng, (T, H), 1.0)
    wr = _bf16_values(rng, (1, H), 0.02)
    out, _, ids, w = c.moe_layer(x, wr, packs, 1, residual=True)
    assert np.all(ids == 0) and np.all(w == 1.0)
    wg, wu, wd = (torch.from_numpy(c.dequantize_packed(packs[2 * m][0], packs[2 * m + 1][0])) for m in range(3))
    F = torch.nn.functional
    xt = torch.from_numpy(x)
    h = (F.silu(F.linear(xt, wg)) * F.linear(xt, wu)).to(torch.bfloat16).double()
    ref = (xt + F.linear(h, wd)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(out, ref)


def test_per_token_equals_grouped_and_thread_count_does_not_matter():
    rng = np.random.default_rng(9)
    T, H, I, E, k = 24, 256, 128, 6, 2
    packs = c.pack_experts(*_experts(rng, E, H, I))
    x = _bf16_values(rng, (T, H), 1.0)
    wr = _bf16_values(rng, (E, H), 0.02)
    out, logits, ids, w = c.moe_layer(x, wr, packs, k, residual=True)
    b = c.layer_per_token(x, packs, ids, w, residual=x)
    assert np.allclose(out, b, rtol=2.0 ** -7, atol=1e-6) and np.mean(out == b) > 0.99
    n = c.threads()
    try:
        c.set_threads(1)
        one = c.moe_layer(x, wr, packs, k, residual=True)[0]
    finally:
        c.set_threads(n)
    assert np.array_equal(one, out)


@pytest.mark.parametrize("T,E,H,I,k,renorm", [(13, 8, 256, 384, 2, False), (40, 16, 512, 256, 4, True)])
def test_c_and_numpy_oracles_agree(T, E, H, I, k, renorm):
    rng = np.random.default_rng(T * E + H)
    gate, up, down = _experts(rng, E, H, I)
    x = _bf16_values(rng, (T, H), 1.0)
    wr = _bf16_values(rng, (E, H), 0.05)
    bias = (rng.standard_normal(E) * 0.2).astype(np.float32)
    # A1: the same bytes
    packs = c.pack_experts(gate, up, down)
    ex = o.PackedExperts.from_bf16(gate, up, down)
    for m in range(3):
        assert np.array_equal(packs[2 * m], ex.m[m][0]) and np.array_equal(packs[2 * m + 1], ex.m[m][1])
    # A2-A4
    lc, ln = c.router_logits(x, wr), o.router_logits(x, wr)
    assert np.array_equal(lc, ln)
    ic, wc = c.route_topk(lc, k, bias, renorm)
    i_n, w_n = o.route_topk(ln, k, bias, renorm)
    assert np.array_equal(ic, i_n) and np.allclose(wc, w_n, rtol=1e-12, atol=0)
    gc, gn = c.group_tokens(ic, E), o.group_tokens(i_n, E)
    assert all(np.array_equal(a, b) for a, b in zip(gc, gn))
    # A5-A6: h to within one BF16 rounding of an fp64 sum, y to fp64 summation order
    hc, yc = c.grouped_ffn(x, packs, gc[2], gc[1], k)
    hn, yn = o.grouped_ffn(x, ex, gn[2], gn[1], k)
    assert np.mean(hc == hn) > 0.999 and np.allclose(hc, hn, rtol=2.0 ** -8, atol=0)
    same_h = np.all(hc == hn, axis=1)
    assert np.allclose(yc[same_h], yn[same_h], rtol=1e-9, atol=1e-12)
    # A7
    oc = c.combine(yn, w_n, gn[3], x)
    on = o.combine(yn, w_n, gn[3], x)
    assert np.array_equal(oc, on)


# ---------------------------------------------------------------- property checks (hypothesis)

from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=30, deadline=None)
@given(T=st.integers(0, 12), E=st.integers(1, 40), k=st.integers(1, 8), seed=st.integers(0, 2**31 - 1),
       renorm=st.booleans(), biased=st.booleans())
def test_property_routing_and_grouping_agree(T, E, k, seed, renorm, biased):
    k = min(k, E)
    rng = np.random.default_rng(seed)
    logits = c.from_bits(c.to_bits(rng.standard_normal((T, E))))
    if T and rng.random() < 0.3:
        logits[0, :] = logits[0, 0]                       # a fully tied row
    bias = (rng.standard_normal(E) * 0.3).astype(np.float32) if biased else None
    ic, wc = c.route_topk(logits, k, bias, renorm)
    i_n, w_n = o.route_topk(logits, k, bias, renorm)
    assert np.array_equal(ic, i_n)
    assert np.allclose(wc, w_n, rtol=1e-12, atol=0)
    for a, b in zip(c.group_tokens(ic, E), o.group_tokens(i_n, E)):
        assert np.array_equal(a, b)


@settings(max_examples=20, deadline=None)
@given(T=st.integers(1, 6), k=st.integers(1, 4), H=st.sampled_from([8, 64]), seed=st.integers(0, 2**31 - 1),
       res=st.booleans(), drop=st.booleans())
def test_property_combine_agrees(T, k, H, seed, res, drop):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((T * k, H))
    w = rng.random((T, k))
    pos = rng.permutation(T * k).astype(np.int32)
    if drop:
        pos[rng.integers(0, T * k)] = -1
    r = c.from_bits(c.to_bits(rng.standard_normal((T, H)))) if res else None
    assert np.array_equal(c.combine(y, w, pos, r), o.combine(y, w, pos, r))


@settings(max_examples=12, deadline=None)
@given(N=st.integers(1, 6), G=st.integers(1, 3), scale=st.sampled_from([1e-3, 0.02, 1.0, 300.0]),
       seed=st.integers(0, 2**31 - 1))
def test_property_quantiser_agrees_and_round_trips(N, G, scale, seed):
    rng = np.random.default_rng(seed)
    w = c.from_bits(c.to_bits(rng.standard_normal((N, 128 * G)) * scale))
    if rng.random() < 0.3:
        w[0, :128] = 0.0                                   # an all-zero group
    pc, sc_ = c.quantize_pack(w)
    pn, sn = o.quantize_pack(w)
    assert np.array_equal(pc, pn) and np.array_equal(sc_, sn)
    s = np.repeat(c.from_bits(sc_), 128, axis=1)
    assert np.all(np.abs(w - c.dequantize_packed(pc, sc_)) <= s / 2 * (1 + 2.0 ** -20))
