"""GPU parity of the whole layer (route -> group -> FFN -> combine through the
C ABI) against the oracle's own end-to-end layer on OLMoE-shaped synthetic
inputs, and of the slot-cache decode path against the resident path.

Routing is a floating-point decision on BF16 logits: the kernel's fp32 sum
and the oracle's fp64 sum can round a logit to neighbouring BF16 values, and
a near-tie at the k-th place can then pick a different (equally valid) expert.
Tokens whose ids differ are counted (a small bound) and checked for validity;
all other tokens must match the oracle within the BF16 bar.
"""
import functools

import numpy as np
import pytest
import torch

import synth
from oracle import exactmoe_oracle as o
from tests._util import assert_bf16_close, bf16_np, torch_weights_source

pytestmark = pytest.mark.gpu

H, I, E, K = 2048, 1024, 64, 8


@pytest.fixture(scope="module")
def M():
    import w4a16_mixture_experts_moe_b200 as m
    assert torch.cuda.is_available()
    return m


@functools.lru_cache(maxsize=2)
def _layer_weights(layer):
    return synth.expert_bank(layer, E, H, I), synth.router_weight(layer, E, H)


@functools.lru_cache(maxsize=2)
def _oracle_experts(layer):
    (g, u, d), _ = _layer_weights(layer)
    return o.LazyQuantizedExperts(torch_weights_source(g, u, d), E, H, I, cache=E)


def _gpu_bank(M, layer):
    from w4a16_mixture_experts_moe_b200.layer import ExpertBank
    (g, u, d), wr = _layer_weights(layer)
    bank = ExpertBank(E, H, I)
    bank.pack(g.cuda(), u.cuda(), d.cuda())
    return bank, wr.cuda()


def _compare(out_gpu, ids_gpu, out_ref, ids_ref, what, max_flip_frac=0.03):
    same = np.all(ids_gpu == ids_ref, axis=1)
    flips = int((~same).sum())
    assert flips <= max(1, int(max_flip_frac * len(same))), f"{what}: routing differs on {flips} tokens"
    assert_bf16_close(out_gpu[same], out_ref[same], what)
    return flips


def test_single_layer_T16_all_tokens(M):
    from w4a16_mixture_experts_moe_b200.layer import LayerBuffers, moe_layer_forward
    T = 16
    bank, wr = _gpu_bank(M, 0)
    x = synth.activations(T, H)
    buf = LayerBuffers(T, K, E, H, I)
    out = moe_layer_forward(x.cuda(), wr, bank, buf)
    assert M.moe_read_device_error(buf.ffn_ws) == 0 and M.moe_read_device_error(buf.group_ws) == 0
    ref, ref_logits, ref_ids, ref_w = o.moe_layer(x.double().numpy(), _layer_weights(0)[1].double().numpy(),
                                                  _oracle_experts(0), K)
    got_logits = bf16_np(buf.logits)
    ulp = np.ldexp(1.0, np.frexp(ref_logits)[1] - 8)
    assert np.all(np.abs(got_logits - ref_logits) <= ulp)
    _compare(bf16_np(out), buf.topk_ids.cpu().numpy(), ref, ref_ids, "layer T=16")


@pytest.mark.parametrize("T", [1, 4, 16, 64])
def test_two_layer_stack_with_residual(M, T):
    from w4a16_mixture_experts_moe_b200.layer import LayerBuffers, moe_layer_forward
    x = synth.activations(T, H, seed=11 + T)
    xs = x.cuda()
    xr = x.double().numpy()
    ok = np.ones(T, dtype=bool)
    for layer in range(2):
        bank, wr = _gpu_bank(M, layer)
        buf = LayerBuffers(T, K, E, H, I)
        nxt = torch.empty_like(xs)
        moe_layer_forward(xs, wr, bank, buf, residual=xs, out=nxt)
        ids_gpu = buf.topk_ids.cpu().numpy()
        ref, _, ref_ids, _ = o.moe_layer(xr, _layer_weights(layer)[1].double().numpy(), _oracle_experts(layer), K,
                                         residual=xr)
        ok &= np.all(ids_gpu == ref_ids, axis=1)
        xs, xr = nxt, ref
        del bank
    assert (~ok).sum() <= max(1, T // 20)
    assert_bf16_close(bf16_np(xs)[ok], xr[ok], f"stack T={T}")


def test_skewed_routing_T512_sampled(M):
    from w4a16_mixture_experts_moe_b200.layer import LayerBuffers, moe_layer_forward
    T = 512
    bank, wr = _gpu_bank(M, 0)
    x = synth.activations(T, H, seed=21)
    bias = torch.from_numpy(synth.zipf_log_bias(E)).cuda()
    buf = LayerBuffers(T, K, E, H, I)
    out = bf16_np(moe_layer_forward(x.cuda(), wr, bank, buf, bias=bias))
    counts = buf.counts.cpu().numpy()
    assert counts.max() >= 200 and (counts == 0).sum() >= 1      # hundreds on a few experts, some empty
    rng = np.random.default_rng(5)
    sample = np.sort(rng.choice(T, size=24, replace=False))
    ref, _, ref_ids, _ = o.moe_layer(x.double().numpy()[sample], _layer_weights(0)[1].double().numpy(),
                                     _oracle_experts(0), K, bias=synth.zipf_log_bias(E))
    _compare(out[sample], buf.topk_ids.cpu().numpy()[sample], ref, ref_ids, "skew T=512 sample")


def test_slot_cache_decode_matches_resident(M):
    """16 slots over 64 experts, 2 layers, 24 decode steps with drawn routing:
    outputs equal the all-resident bank's outputs bit for bit, and the cache's
    counters equal an independent count of first uses and reuses."""
    from w4a16_mixture_experts_moe_b200.layer import ExpertBank, LayerBuffers
    L, S, steps, T = 2, 16, 24, 1
    resident = [_gpu_bank(M, l) for l in range(L)]
    rec = resident[0][0].rec
    pool = torch.empty(L * E * rec, dtype=torch.uint8, pin_memory=True)
    for l in range(L):
        pool[l * E * rec:(l + 1) * E * rec].copy_(resident[l][0].buf.cpu())
    slots = torch.empty(L * S * rec, dtype=torch.uint8, device="cuda")
    table = torch.full((L, E), -1, dtype=torch.int32, device="cuda")
    cache = M.SlotCache(L, E, S, rec, pool, slots, table)
    side = torch.cuda.Stream()
    compute = torch.cuda.current_stream()
    routing = [synth.drawn_routing(l, E, K, steps) for l in range(L)]
    x = synth.activations(steps, H, seed=31).cuda()
    buf = LayerBuffers(T, K, E, H, I)
    for s in range(steps):
        for l in range(L):
            ids = [int(v) for v in routing[l][s]]
            _, miss = cache.lookup(l, ids)
            cache.fill(l, miss, side=side, compute=compute)
            xi = x[s:s + 1]
            outs = []
            for bank_ptr, rec_b, es, ns in ((resident[l][0].ptr, rec, None, E),
                                            (slots.data_ptr() + l * S * rec, rec, table[l], S)):
                buf.topk_ids.copy_(torch.tensor([ids], dtype=torch.int32))
                M.moe_route_topk(xi, resident[l][1], T, H, E, K, None, M.MOE_IDS_GIVEN, buf.logits, buf.topk_ids,
                                 buf.topk_w)
                M.moe_group_tokens(buf.topk_ids, T, K, E, buf.counts, buf.offsets, buf.sorted_pair, buf.pair_pos,
                                   buf.group_ws, buf.group_ws_bytes)
                M.moe_grouped_w4a16_ffn(xi, buf.sorted_pair, buf.offsets, bank_ptr, rec_b, es, ns, T, K, E, H, I,
                                        M.MOE_PATH_AUTO, buf.y, buf.ffn_ws, buf.ffn_ws_bytes)
                o_ = torch.empty(1, H, dtype=torch.bfloat16, device="cuda")
                M.moe_combine(buf.y, buf.topk_w, buf.pair_pos, xi, T, K, H, o_)
                outs.append(o_)
                assert M.moe_read_device_error(buf.ffn_ws) == 0
            cache.release(l, compute)
            assert torch.equal(outs[0], outs[1]), (s, l)
    st = cache.stats()
    seen_hits = seen_miss = 0
    for l in range(L):
        import tests.test_abi_exports as t
        model = t._LRUModel(E, S)
        for s in range(steps):
            model.lookup([int(v) for v in routing[l][s]])
        seen_hits += model.hits
        seen_miss += model.misses
    assert (st["hits"], st["misses"]) == (seen_hits, seen_miss)
    assert st["h2d_bytes"] == seen_miss * rec
    cache.close()


@pytest.mark.parametrize("T", [512, 2048, 8192])
def test_prefill_olmoe_tensor_core_sampled(M, T):
    """Prefill-sized OLMoE layer (AUTO picks the tcgen05 path: >= 32 rows per
    expert on average); every token is computed, a seeded sample is checked."""
    from w4a16_mixture_experts_moe_b200.layer import LayerBuffers, moe_layer_forward
    bank, wr = _gpu_bank(M, 0)
    x = synth.activations(T, H, seed=41)
    buf = LayerBuffers(T, K, E, H, I)
    out = bf16_np(moe_layer_forward(x.cuda(), wr, bank, buf))
    assert M.moe_read_device_error(buf.ffn_ws) == 0
    sample = np.sort(np.random.default_rng(T).choice(T, size=24, replace=False))
    ref, _, ref_ids, _ = o.moe_layer(x.double().numpy()[sample], _layer_weights(0)[1].double().numpy(),
                                     _oracle_experts(0), K)
    _compare(out[sample], buf.topk_ids.cpu().numpy()[sample], ref, ref_ids, f"prefill T={T} sample")


@pytest.mark.parametrize("T", [512, 8192])
def test_prefill_second_shape_sampled(M, T):
    """Hidden 4096, intermediate 14336, 8 experts, top-2 (tcgen05 path)."""
    from w4a16_mixture_experts_moe_b200.layer import ExpertBank, LayerBuffers, moe_layer_forward
    H2, I2, E2, K2 = 4096, 14336, 8, 2
    g, u, d = synth.expert_bank(0, E2, H2, I2)
    wr = synth.router_weight(0, E2, H2)
    bank = ExpertBank(E2, H2, I2)
    bank.pack(g.cuda(), u.cuda(), d.cuda())
    x = synth.activations(T, H2, seed=43)
    buf = LayerBuffers(T, K2, E2, H2, I2)
    out = bf16_np(moe_layer_forward(x.cuda(), wr.cuda(), bank, buf, flags=M.MOE_RENORM))
    assert M.moe_read_device_error(buf.ffn_ws) == 0
    del bank
    sample = np.sort(np.random.default_rng(7).choice(T, size=12, replace=False))
    experts = o.LazyQuantizedExperts(torch_weights_source(g, u, d), E2, H2, I2, cache=1)
    ref, _, ref_ids, _ = o.moe_layer(x.double().numpy()[sample], wr.double().numpy(), experts, K2, renorm=True)
    _compare(out[sample], buf.topk_ids.cpu().numpy()[sample], ref, ref_ids, f"second shape T={T} sample")
