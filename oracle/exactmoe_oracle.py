"""CPU oracle for the fused grouped W4A16 routed-expert MoE layer.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module:
only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline/reference
legs may call it. It shares no code, table or constant generator with the
CUDA library; both sides implement the definitions below independently.

Source: "Every Expert Counts: ExactMoE for Memory-Efficient W4A16 Inference"
(A. Saab, arXiv 2608.15383):

* Abstract: only the routed experts are quantised, four-bit, symmetric, in
  groups of 128; router and activations stay BF16; exactness means that
  every chosen expert is run and top-k routing is left as it was.
* Figure 1 caption: the order of the steps. The BF16 router picks the
  experts, the tokens are gathered per chosen expert, fused grouped kernels
  run the active experts, and they read the packed codes and scales
  directly, with no FP16 copy of any expert.

The pages give no formula, pseudo-code or worked example, so each step below
is the plainest reading of those two passages (readings listed in the design
notes of the repository):

* quantiser (per row, per 128-wide K group): s = bf16_rn(absmax / 7) with the
  division in fp32; q = clamp(rint(w / s), -8, 7) with the division in fp32 and
  ties to even; an all-zero group has s = 0 and q = 0;
* packed layout: offset-binary u = q + 8; each row is K/8 little-endian 32-bit
  words; word j holds k in [8j, 8j+8); k = 8j + 2i + h (i in 0..3, h in 0..1)
  sits at bits [4(i+4h), 4(i+4h)+4). Scales are [N][K/128] BF16;
* router logits: fp64 sum of BF16 products, rounded to BF16;
* top-k: keys = fp32(logit) + fp32(bias), NaN -> -inf, k largest keys, ties to
  the lower expert index, listed by descending key then ascending index;
  weights are the full-softmax probabilities of the chosen experts (optionally
  renormalised over the k chosen);
* grouping: per-expert counts, exclusive prefix sum, and the stable
  permutation of flat pair indices p = t*k + j by expert;
* expert FFN (SwiGLU): g = x Wg^T, u = x Wu^T, h = bf16_rn(silu(g) * u),
  y = h Wd^T, where W = q * s dequantised exactly, sums in fp64; h is the
  expert's BF16 activation (A16), y is the expert's unrounded output that the
  combine weights (the pages do not store it, so it is not rounded);
* combine: out_t = bf16_rn(residual_t + sum_j w_tj * y_(t,j)) in j order.

Arithmetic is fp64 except where floating point decides an integer (the
quantiser's rint, the top-k comparison), which runs in fp32 like the kernels.
Parity of the whole layer against the trained BF16 model is not pinned by the
pages (their accuracy figures need trained weights and datasets).
"""
from __future__ import annotations

from functools import lru_cache

import numpy as np

GROUP = 128
QMIN, QMAX = -8, 7


# --------------------------------------------------------------------------
# BF16 helpers (definitions, not kernels)
# --------------------------------------------------------------------------

def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact value of BF16 bit patterns (uint16) as float64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def round_to_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest BF16 value, ties to even.

    BF16 keeps 8 significant bits and fp32's exponent range: for
    x = m * 2^e with 0.5 <= |m| < 1 the spacing is 2^(e-8), never finer
    than the subnormal spacing 2^-133. Results at or above 2^128 overflow
    to infinity. Single rounding from the exact fp64 value.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    ulp_exp = np.maximum(e - 8, -133)
    with np.errstate(over="ignore", invalid="ignore"):
        r = np.ldexp(np.rint(np.ldexp(x, -ulp_exp)), ulp_exp)
        r = np.where(np.isfinite(x) & (np.abs(r) >= 2.0 ** 128), np.copysign(np.inf, x), r)
    return r


def f64_to_bf16_bits(x) -> np.ndarray:
    """BF16 bit patterns of values that are already BF16-representable."""
    v = round_to_bf16(x).astype(np.float32)
    return (v.view(np.uint32) >> 16).astype(np.uint16)


# --------------------------------------------------------------------------
# Quantise + pack (Abstract: symmetric group-128 int4 on routed experts;
# Figure 1 caption: packing happens a single time, into the form the kernels read)
# --------------------------------------------------------------------------

def quantize_group128(w) -> tuple[np.ndarray, np.ndarray]:
    """Symmetric per-(row, 128-group) int4 quantisation.

    w: [N][K] BF16 values (as float64). Returns q int8 [N][K] in [-8, 7] and
    the stored scales s [N][K/128] as float64 BF16 values.
    """
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    g = w.astype(np.float32).reshape(N, K // GROUP, GROUP)
    absmax = np.max(np.abs(g), axis=2)                      # exact in fp32
    s32 = (absmax / np.float32(7.0)).astype(np.float32)     # IEEE fp32 divide
    s = round_to_bf16(s32.astype(np.float64))               # stored BF16 scale
    s_f32 = s.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = (g / s_f32[:, :, None]).astype(np.float32)  # fp32 divide
    q = np.clip(np.rint(ratio), QMIN, QMAX)                 # rint: ties to even
    q = np.where(s_f32[:, :, None] == 0, 0.0, q)
    return q.reshape(N, K).astype(np.int8), s


def dequantize(q, s) -> np.ndarray:
    """W = q * s, exact in float64 (4-bit times 8-bit significands)."""
    q = np.asarray(q, dtype=np.float64)
    N, K = q.shape
    return (q.reshape(N, K // GROUP, GROUP) * np.asarray(s, dtype=np.float64)[:, :, None]).reshape(N, K)


def pack_rows(q) -> np.ndarray:
    """int4 codes [N][K] -> packed bytes [N][K/2] in the interleaved word layout."""
    q = np.asarray(q)
    N, K = q.shape
    if K % 8:
        raise ValueError("K must be a multiple of 8")
    u = (q.astype(np.int32) + 8).astype(np.uint32)
    if np.any(u > 15):
        raise ValueError("codes outside [-8, 7]")
    u = u.reshape(N, K // 8, 4, 2)                          # [n][word][i][h], k = 8j+2i+h
    word = np.zeros((N, K // 8), dtype=np.uint32)
    for i in range(4):
        for h in range(2):
            word |= u[:, :, i, h] << np.uint32(4 * (i + 4 * h))
    return word.astype("<u4").view(np.uint8).reshape(N, K // 2)


def unpack_rows(packed) -> np.ndarray:
    """Inverse of pack_rows: packed bytes [N][K/2] -> int8 codes [N][K]."""
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    N, KB = p.shape
    word = p.view("<u4").astype(np.uint32).reshape(N, KB // 4)
    u = np.empty((N, KB // 4, 4, 2), dtype=np.int32)
    for i in range(4):
        for h in range(2):
            u[:, :, i, h] = (word >> np.uint32(4 * (i + 4 * h))) & np.uint32(0xF)
    return (u.reshape(N, KB * 2) - 8).astype(np.int8)


def quantize_pack(w) -> tuple[np.ndarray, np.ndarray]:
    """BF16 weights [N][K] -> (packed uint8 [N][K/2], scale bits uint16 [N][K/128])."""
    q, s = quantize_group128(w)
    return pack_rows(q), f64_to_bf16_bits(s)


def dequantize_packed(packed, scale_bits) -> np.ndarray:
    return dequantize(unpack_rows(packed), bf16_bits_to_f64(scale_bits))


# --------------------------------------------------------------------------
# Router (Abstract: the router stays BF16 and top-k routing is left as it
# was; Figure 1 caption: the model's own BF16 router picks the experts)
# --------------------------------------------------------------------------

def router_logits(x, w_router) -> np.ndarray:
    """logits[t][e] = bf16_rn(sum_h x[t][h] * Wr[e][h]); x [T][H], Wr [E][H]."""
    return round_to_bf16(np.asarray(x, np.float64) @ np.asarray(w_router, np.float64).T)


def routing_keys(logits, bias=None) -> np.ndarray:
    """fp32 selection keys: logit + bias, with NaN treated as -inf."""
    key = np.asarray(logits, dtype=np.float64).astype(np.float32)
    if bias is not None:
        key = (key + np.asarray(bias, dtype=np.float32)[None, :]).astype(np.float32)
    return np.where(np.isnan(key), np.float32(-np.inf), key)


def softmax_probs(logits, bias=None) -> np.ndarray:
    """Full softmax over all experts of the (biased) logits, in fp64."""
    lf = routing_keys(logits, bias).astype(np.float64)
    m = np.max(lf, axis=1, keepdims=True)
    e = np.exp(lf - m)
    return e / e.sum(axis=1, keepdims=True)


def route_topk(logits, k: int, bias=None, renorm: bool = False):
    """Top-k expert ids [T][k] (int32) and weights [T][k] (float64).

    Ids are the k largest fp32 keys, ties to the lower index, ordered by
    descending key then ascending index. Weights are the softmax
    probabilities of those ids, divided by their sum when renorm is set.
    """
    key = routing_keys(logits, bias)
    T, E = key.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    order = np.argsort(-key, axis=1, kind="stable")
    ids = order[:, :k].astype(np.int32)
    p = softmax_probs(logits, bias)
    w = np.take_along_axis(p, ids.astype(np.int64), axis=1)
    if renorm:
        w = w / w.sum(axis=1, keepdims=True)
    return ids, w


def weights_for_ids(logits, ids, bias=None, renorm: bool = False) -> np.ndarray:
    """Softmax probabilities of given expert ids (routing drawn elsewhere)."""
    p = softmax_probs(logits, bias)
    w = np.take_along_axis(p, np.asarray(ids, dtype=np.int64), axis=1)
    if renorm:
        w = w / w.sum(axis=1, keepdims=True)
    return w


# --------------------------------------------------------------------------
# Grouping (Figure 1 caption: the tokens are gathered per chosen expert)
# --------------------------------------------------------------------------

def group_tokens(ids, E: int):
    """counts [E], offsets [E+1], sorted_pair [T*k], pair_pos [T*k] (int32).

    sorted_pair lists flat pair indices p = t*k + j ordered by expert, and by
    p within an expert (stable). pair_pos is its inverse permutation.
    """
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert id out of range")
    counts = np.bincount(flat, minlength=E)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    sorted_pair = np.argsort(flat, kind="stable")
    pair_pos = np.empty_like(sorted_pair)
    pair_pos[sorted_pair] = np.arange(flat.size)
    return (counts.astype(np.int32), offsets.astype(np.int32),
            sorted_pair.astype(np.int32), pair_pos.astype(np.int32))


# --------------------------------------------------------------------------
# Expert FFN (Abstract: fused grouped MoE kernels over W4A16 experts)
# --------------------------------------------------------------------------

def silu(g):
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def swiglu_expert(xr, wg, wu, wd):
    """Rows xr [R][H] through one expert; W already dequantised (float64).

    Returns h [R][I] (BF16-rounded) and y [R][H] (float64).
    """
    xr = np.asarray(xr, dtype=np.float64)
    g = xr @ wg.T
    u = xr @ wu.T
    h = round_to_bf16(silu(g) * u)
    return h, h @ wd.T


class PackedExperts:
    """Packed experts of one layer: per matrix a packed [E][N][K/2] array and
    scale bits [E][N][K/128], dequantised lazily one expert at a time."""

    def __init__(self, gate_q, gate_s, up_q, up_s, down_q, down_s):
        self.m = ((gate_q, gate_s), (up_q, up_s), (down_q, down_s))
        self.E, self.I = gate_q.shape[0], gate_q.shape[1]
        self.H = down_q.shape[1]
        self._cache = lru_cache(maxsize=8)(self._deq)

    @classmethod
    def from_bf16(cls, gate, up, down):
        """Quantise + pack float64 BF16-valued weights [E][N][K] per matrix."""
        out = []
        for w in (gate, up, down):
            qs = [quantize_pack(w[e]) for e in range(w.shape[0])]
            out.append(np.stack([a for a, _ in qs]))
            out.append(np.stack([b for _, b in qs]))
        return cls(*out)

    def _deq(self, e: int):
        return tuple(dequantize_packed(q[e], s[e]) for q, s in self.m)

    def dequantized(self, e: int):
        """(Wg [I][H], Wu [I][H], Wd [H][I]) of expert e in float64."""
        return self._cache(int(e))


class LazyQuantizedExperts:
    """Experts quantised by this oracle on first use, from a function that
    returns expert e's BF16-valued (gate [I][H], up [I][H], down [H][I])."""

    def __init__(self, weights_of, E: int, H: int, I: int, cache: int = 80):
        self.weights_of, self.E, self.H, self.I = weights_of, E, H, I
        self._cache = lru_cache(maxsize=cache)(self._deq)

    def _deq(self, e: int):
        return tuple(dequantize_packed(*quantize_pack(w)) for w in self.weights_of(e))

    def packed(self, e: int):
        """(packed, scale bits) of gate, up, down of expert e."""
        return tuple(quantize_pack(w) for w in self.weights_of(e))

    def dequantized(self, e: int):
        return self._cache(int(e))


class Bf16Experts:
    """Unquantised experts, the pages' BF16 baseline (Abstract and Table 1
    compare the W4A16 model with the BF16 one): weights_of(e) returns expert
    e's BF16-valued (gate [I][H], up [I][H], down [H][I]), used as they are."""

    def __init__(self, weights_of, E: int, H: int, I: int):
        self.weights_of, self.E, self.H, self.I = weights_of, E, H, I

    def dequantized(self, e: int):
        return tuple(np.asarray(w, dtype=np.float64) for w in self.weights_of(int(e)))


def grouped_ffn(x, experts: PackedExperts, sorted_pair, offsets, k: int):
    """Grouped form: per expert, its rows in sorted order.

    Returns h [T*k][I] (BF16 values) and y [T*k][H] (float64) in sorted order.
    """
    x = np.asarray(x, dtype=np.float64)
    E = len(offsets) - 1
    P = int(offsets[-1])
    h_all = np.zeros((P, experts.I))
    y_all = np.zeros((P, experts.H))
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if lo == hi:
            continue
        wg, wu, wd = experts.dequantized(e)
        tok = np.asarray(sorted_pair[lo:hi]) // k
        h_all[lo:hi], y_all[lo:hi] = swiglu_expert(x[tok], wg, wu, wd)
    return h_all, y_all


def combine(y_sorted, w, pair_pos, residual=None) -> np.ndarray:
    """out[t] = bf16_rn(residual[t] + sum_j w[t][j] * y[pair_pos[t*k+j]]), j in order.

    A pair with pair_pos < 0 (dropped by the grouping because its expert id
    was out of range, which the library flags) contributes nothing.
    """
    w = np.asarray(w, dtype=np.float64)
    T, k = w.shape
    y = np.asarray(y_sorted, dtype=np.float64)
    pos = np.asarray(pair_pos, dtype=np.int64).reshape(T, k)
    acc = np.zeros((T, y.shape[1])) if residual is None else np.array(residual, dtype=np.float64)
    for j in range(k):
        keep = (pos[:, j] >= 0)[:, None]
        acc = acc + np.where(keep, w[:, j:j + 1] * y[np.maximum(pos[:, j], 0)], 0.0)
    return round_to_bf16(acc)


# --------------------------------------------------------------------------
# The whole layer, two independent forms
# --------------------------------------------------------------------------

def moe_layer_grouped(x, experts: PackedExperts, ids, w, residual=None):
    """histogram -> scan -> stable permutation -> per-expert FFN -> combine."""
    T, k = np.asarray(ids).shape
    counts, offsets, sorted_pair, pair_pos = group_tokens(ids, experts.E)
    _, y = grouped_ffn(x, experts, sorted_pair, offsets, k)
    return combine(y, w, pair_pos, residual)


def moe_layer_per_token(x, experts: PackedExperts, ids, w, residual=None):
    """For each token, for each chosen expert in j order: matrix-vector SwiGLU."""
    x = np.asarray(x, dtype=np.float64)
    ids = np.asarray(ids)
    w = np.asarray(w, dtype=np.float64)
    T, k = ids.shape
    out = np.zeros((T, experts.H))
    for t in range(T):
        acc = np.zeros(out.shape[1]) if residual is None else np.array(residual[t], dtype=np.float64)
        for j in range(k):
            wg, wu, wd = experts.dequantized(int(ids[t, j]))
            g = wg.dot(x[t])
            u = wu.dot(x[t])
            h = round_to_bf16(silu(g) * u)
            acc = acc + w[t, j] * wd.dot(h)
        out[t] = round_to_bf16(acc)
    return out


def moe_layer(x, w_router, experts: PackedExperts, k: int, bias=None,
              renorm: bool = False, residual=None):
    """Router -> top-k -> grouped FFN -> combine, all in the oracle."""
    logits = router_logits(x, w_router)
    ids, w = route_topk(logits, k, bias, renorm)
    return moe_layer_grouped(x, experts, ids, w, residual), logits, ids, w


# --------------------------------------------------------------------------
# Expert slot cache (Abstract: the experts live in pinned host memory and a
# slot cache of configurable size holds some of them on the GPU; Figure 1
# caption: a miss copies the expert's packed codes and scales; Figure 2
# caption: once the cache holds all experts no hit rate is counted; Table 1:
# hit rate and host-to-device traffic per slot count)
# --------------------------------------------------------------------------

class SlotCapacityError(ValueError):
    """A step needs more distinct experts than the cache has slots."""


class SlotCacheLRU:
    """Policy of one layer's slot cache, as plain bookkeeping.

    The pages name the cache and its counters but no replacement policy; the
    reading used here is least-recently-used:

    * a step's ids are de-duplicated (an expert chosen by several tokens of
      the step is one lookup) and handled in first-occurrence order;
    * an id already in a slot is a hit, and that slot counts as used by this
      step;
    * every other id is a miss: it takes the lowest-numbered empty slot if
      one exists, otherwise it evicts the expert whose slot was used least
      recently, never one used by this step, the lower slot number breaking
      ties; a miss is one whole expert record copied host -> device;
    * more distinct ids than slots is an error and changes nothing;
    * with at least as many slots as experts the cache is resident: expert e
      lives in slot e, the first use of an expert loads it, and hits and
      misses are not counted.

    `lookup` returns (slot of each id in the order given, ids loaded this
    step, experts evicted this step).
    """

    def __init__(self, E: int, slots: int):
        self.E, self.S = int(E), int(slots)
        self.resident = self.S >= self.E
        self.expert_in = [None] * self.S      # slot -> expert held
        self.last_use = [0] * self.S          # slot -> step that last used it
        self.step = 0
        self.hits = self.misses = self.loads = 0

    def slot_of(self, e: int):
        if self.resident:
            return e if self.expert_in[e] is not None else None
        for s in range(self.S):
            if self.expert_in[s] == e:
                return s
        return None

    def lookup(self, ids):
        ids = [int(v) for v in ids]
        if any(v < 0 or v >= self.E for v in ids):
            raise ValueError("expert id out of range")
        distinct = []
        for v in ids:
            if v not in distinct:
                distinct.append(v)
        if len(distinct) > self.S:
            raise SlotCapacityError(f"{len(distinct)} distinct experts > {self.S} slots")
        self.step += 1
        loaded, evicted = [], []
        if self.resident:
            for v in distinct:
                if self.expert_in[v] is None:
                    self.expert_in[v] = v
                    loaded.append(v)
            self.loads += len(loaded)
            return [v for v in ids], loaded, evicted
        in_use = set()
        for v in distinct:                      # hits first: their slots are protected
            s = self.slot_of(v)
            if s is not None:
                self.hits += 1
                self.last_use[s] = self.step
                in_use.add(s)
        for v in distinct:
            if self.slot_of(v) is not None:
                continue
            empty = [s for s in range(self.S) if self.expert_in[s] is None]
            if empty:
                s = empty[0]
            else:
                free = [s for s in range(self.S) if s not in in_use]
                s = min(free, key=lambda c: (self.last_use[c], c))
                evicted.append(self.expert_in[s])
            self.expert_in[s] = v
            self.last_use[s] = self.step
            in_use.add(s)
            self.misses += 1
            self.loads += 1
            loaded.append(v)
        return [self.slot_of(v) for v in ids], loaded, evicted

    def plan_waves(self, ids):
        """Cache-sized waves (Figure 1 caption: the active experts run in
        waves sized to the cache): the step's distinct ids in first-occurrence
        order, those already held in a slot first, cut into consecutive
        waves of at most S ids. Each wave is then one lookup."""
        distinct = []
        for v in (int(i) for i in ids):
            if v not in distinct:
                distinct.append(v)
        held = [v for v in distinct if self.slot_of(v) is not None]
        order = held + [v for v in distinct if v not in held]
        return [order[i:i + self.S] for i in range(0, len(order), self.S)]

    def h2d_bytes(self, record_bytes: int) -> int:
        """Host-to-device bytes moved so far: one record per load."""
        return self.loads * int(record_bytes)
