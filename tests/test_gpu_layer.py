"""GPU parity of the whole layer (route -> group -> FFN -> combine through the
C ABI) against the oracle on OLMoE-shaped synthetic inputs, and of the
slot-cache decode path against the oracle's layer and slot-cache policy.

Routing is a floating-point decision on BF16 logits: the kernel's fp32 sum and
the oracle's fp64 sum may round a logit to neighbouring BF16 values, and a
near-tie at the k-th place then picks a different, equally valid expert. So
every check runs in three parts:

1. the GPU's logits are within one BF16 ulp of the oracle's fp64 logits plus
   the fp32 summation bound (H - 1) 2^-24 sum |x w|;
2. the oracle routes from the GPU's own logits: the top-k ids must then be
   identical and the weights equal to 1e-5 relative;
3. the oracle computes the layer from those ids and weights, and EVERY token
   of the GPU's output must meet the BF16 bar |d| <= 1e-2 + 1e-2 |ref|.

The number of tokens whose routing would differ had the oracle used its own
logits is returned for information only.
"""
import functools

import numpy as np
import pytest
import torch

import synth
from oracle import exactmoe_oracle as o
from tests._util import assert_bf16_close, assert_logits_close, bf16_np, torch_weights_source

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


def check_layer(x, wr, experts, k, gpu_logits, gpu_ids, gpu_w, gpu_out, what, bias=None, renorm=False,
                residual=None):
    """The three-part check above; x, wr, residual are float64 numpy arrays of
    BF16 values, the gpu_* arrays come back from the device. Returns the
    count of tokens whose routing from the oracle's own logits differs."""
    ref_logits = o.router_logits(x, wr)
    assert_logits_close(gpu_logits, ref_logits, x, wr, what)
    ids, w = o.route_topk(gpu_logits, k, bias, renorm)
    assert np.array_equal(gpu_ids, ids), f"{what}: top-k ids differ given identical logits"
    assert np.allclose(gpu_w, w, rtol=1e-5, atol=1e-8), f"{what}: routing weights"
    ref = o.moe_layer_grouped(x, experts, ids, w, residual)
    assert_bf16_close(gpu_out, ref, what)
    own_ids, _ = o.route_topk(ref_logits, k, bias, renorm)
    return int((~np.all(own_ids == gpu_ids, axis=1)).sum())


def _run_and_check(M, layer, x_cpu, buf, out, what, bias=None, renorm=False, residual=None, rows=None):
    """Check rows `rows` (all by default) of a layer the GPU already ran."""
    sel = slice(None) if rows is None else rows
    xr = x_cpu.double().numpy()[sel]
    return check_layer(xr, _layer_weights(layer)[1].double().numpy(), _oracle_experts(layer), K,
                       bf16_np(buf.logits)[sel], buf.topk_ids.cpu().numpy()[sel], buf.topk_w.cpu().numpy()[sel],
                       bf16_np(out)[sel], what, bias=bias, renorm=renorm,
                       residual=None if residual is None else residual.double().numpy()[sel])


def test_single_layer_T16_all_tokens(M):
    from w4a16_mixture_experts_moe_b200.layer import LayerBuffers, moe_layer_forward
    T = 16
    bank, wr = _gpu_bank(M, 0)
    x = synth.activations(T, H)
    buf = LayerBuffers(T, K, E, H, I)
    out = moe_layer_forward(x.cuda(), wr, bank, buf)
    assert M.moe_read_device_error(buf.ffn_ws) == 0 and M.moe_read_device_error(buf.group_ws) == 0
    flips = _run_and_check(M, 0, x, buf, out, "layer T=16")
    assert flips <= 2


@pytest.mark.parametrize("T", [1, 4, 16, 64])
def test_two_layer_stack_with_residual(M, T):
    """Each layer of the GPU's own trajectory (x_{l+1} = x_l + MoE(x_l)) is
    checked against the oracle's layer on the same input, every token."""
    from w4a16_mixture_experts_moe_b200.layer import LayerBuffers, moe_layer_forward
    x = synth.activations(T, H, seed=11 + T).cuda()
    for layer in range(2):
        bank, wr = _gpu_bank(M, layer)
        buf = LayerBuffers(T, K, E, H, I)
        nxt = torch.empty_like(x)
        moe_layer_forward(x, wr, bank, buf, residual=x, out=nxt)
        assert M.moe_read_device_error(buf.ffn_ws) == 0
        x_cpu = x.cpu()
        _run_and_check(M, layer, x_cpu, buf, nxt, f"stack T={T} layer {layer}", residual=x_cpu)
        x = nxt
        del bank


def test_skewed_routing_T512_all_tokens(M):
    from w4a16_mixture_experts_moe_b200.layer import LayerBuffers, moe_layer_forward
    T = 512
    bank, wr = _gpu_bank(M, 0)
    x = synth.activations(T, H, seed=21)
    bias = synth.zipf_log_bias(E)
    buf = LayerBuffers(T, K, E, H, I)
    out = moe_layer_forward(x.cuda(), wr, bank, buf, bias=torch.from_numpy(bias).cuda())
    assert M.moe_read_device_error(buf.ffn_ws) == 0
    counts = buf.counts.cpu().numpy()
    assert counts.max() >= 200 and (counts == 0).sum() >= 1      # hundreds on a few experts, some empty
    _run_and_check(M, 0, x, buf, out, "skew T=512", bias=bias)


def test_slot_cache_decode_matches_oracle(M):
    """16 slots over 64 experts, 2 layers, 24 decode steps at T = 1 with drawn
    routing. Each layer's output through the slot table is checked against the
    oracle's layer (ids given, weights from the GPU's logits), the lookups
    against the oracle's slot-cache policy (slot of every id, the ids loaded),
    and the cache's counters and bytes copied against the policy's counts. The
    all-resident bank must also give the same bits (same kernels, other
    addresses)."""
    from w4a16_mixture_experts_moe_b200.layer import LayerBuffers
    L, S, steps, T = 2, 16, 24, 1
    resident = [_gpu_bank(M, l) for l in range(L)]
    rec = resident[0][0].rec
    pool = torch.empty(L * E * rec, dtype=torch.uint8, pin_memory=True)
    for l in range(L):
        pool[l * E * rec:(l + 1) * E * rec].copy_(resident[l][0].buf.cpu())
    slots = torch.empty(L * S * rec, dtype=torch.uint8, device="cuda")
    table = torch.full((L, E), -1, dtype=torch.int32, device="cuda")
    cache = M.SlotCache(L, E, S, rec, pool, slots, table)
    policy = [o.SlotCacheLRU(E, S) for _ in range(L)]
    side = torch.cuda.Stream()
    compute = torch.cuda.current_stream()
    routing = [synth.drawn_routing(l, E, K, steps) for l in range(L)]
    x_all = synth.activations(steps, H, seed=31)
    x = x_all.cuda()
    buf = LayerBuffers(T, K, E, H, I)
    for s in range(steps):
        for l in range(L):
            ids = [int(v) for v in routing[l][s]]
            slot_of, miss = cache.lookup(l, ids)
            want_slots, want_loaded, _ = policy[l].lookup(ids)
            assert (slot_of, miss) == (want_slots, want_loaded), (s, l)
            cache.fill(l, miss, side=side, compute=compute)
            xi = x[s:s + 1]
            outs = []
            for bank_ptr, es, ns in ((slots.data_ptr() + l * S * rec, table[l], S), (resident[l][0].ptr, None, E)):
                buf.topk_ids.copy_(torch.tensor([ids], dtype=torch.int32))
                M.moe_route_topk(xi, resident[l][1], T, H, E, K, None, M.MOE_IDS_GIVEN, buf.logits, buf.topk_ids,
                                 buf.topk_w)
                M.moe_group_tokens(buf.topk_ids, T, K, E, buf.counts, buf.offsets, buf.sorted_pair, buf.pair_pos,
                                   buf.group_ws, buf.group_ws_bytes)
                M.moe_grouped_w4a16_ffn(xi, buf.sorted_pair, buf.offsets, bank_ptr, rec, es, ns, T, K, E, H, I,
                                        M.MOE_PATH_AUTO, buf.y, buf.ffn_ws, buf.ffn_ws_bytes)
                o_ = torch.empty(1, H, dtype=torch.bfloat16, device="cuda")
                M.moe_combine(buf.y, buf.topk_w, buf.pair_pos, xi, T, K, H, o_)
                outs.append(o_)
                assert M.moe_read_device_error(buf.ffn_ws) == 0
                if es is not None:
                    # the oracle's layer on the same token, ids given
                    xr = x_all[s:s + 1].double().numpy()
                    wr = _layer_weights(l)[1].double().numpy()
                    gl = bf16_np(buf.logits)
                    assert_logits_close(gl, o.router_logits(xr, wr), xr, wr, "slot path logits")
                    w = o.weights_for_ids(gl, np.array([ids]))
                    assert np.allclose(buf.topk_w.cpu().numpy(), w, rtol=1e-5, atol=1e-8)
                    ref = o.moe_layer_grouped(xr, _oracle_experts(l), np.array([ids]), w, residual=xr)
                    assert_bf16_close(bf16_np(o_), ref, f"slot path step {s} layer {l}")
            cache.release(l, compute)
            assert torch.equal(outs[0], outs[1]), (s, l)
    st = cache.stats()
    assert st["hits"] == sum(p.hits for p in policy)
    assert st["misses"] == sum(p.misses for p in policy)
    assert st["h2d_bytes"] == sum(p.h2d_bytes(rec) for p in policy)
    assert 0.3 < st["hits"] / (st["hits"] + st["misses"]) < 0.9
    cache.close()


@pytest.mark.parametrize("T", [512, 2048, 8192])
def test_prefill_olmoe_tensor_core_sampled(M, T):
    """Prefill-sized OLMoE layer (AUTO picks the tcgen05 path: >= 32 rows per
    expert on average); every token is computed, a seeded sample is checked."""
    from w4a16_mixture_experts_moe_b200.layer import LayerBuffers, moe_layer_forward
    bank, wr = _gpu_bank(M, 0)
    x = synth.activations(T, H, seed=41)
    buf = LayerBuffers(T, K, E, H, I)
    out = moe_layer_forward(x.cuda(), wr, bank, buf)
    assert M.moe_read_device_error(buf.ffn_ws) == 0
    sample = np.sort(np.random.default_rng(T).choice(T, size=24, replace=False))
    _run_and_check(M, 0, x, buf, out, f"prefill T={T} sample", rows=sample)


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
    out = moe_layer_forward(x.cuda(), wr.cuda(), bank, buf, flags=M.MOE_RENORM)
    assert M.moe_read_device_error(buf.ffn_ws) == 0
    del bank
    sample = np.sort(np.random.default_rng(7).choice(T, size=12, replace=False))
    experts = o.LazyQuantizedExperts(torch_weights_source(g, u, d), E2, H2, I2, cache=1)
    check_layer(x.double().numpy()[sample], wr.double().numpy(), experts, K2, bf16_np(buf.logits)[sample],
                buf.topk_ids.cpu().numpy()[sample], buf.topk_w.cpu().numpy()[sample], bf16_np(out)[sample],
                f"second shape T={T} sample", renorm=True)


def test_slot_cache_waves_match_oracle(M):
    """Steps that need more experts than the 16 slots run in cache-sized
    waves: 8 decode steps at T = 4 (about 27 distinct experts per step, two
    waves) and one 96-token pass that selects all 64 experts (four waves, on
    the tensor-core path). Every token of every step is checked against the
    oracle's layer (ids given, weights from the GPU's logits), the waves and
    lookups against the oracle's policy, the counters against its counts."""
    from w4a16_mixture_experts_moe_b200.layer import LayerBuffers
    S, layer = 16, 0
    bank, wr = _gpu_bank(M, layer)
    rec = bank.rec
    pool = bank.buf.cpu().pin_memory()
    del bank
    slots = torch.empty(S * rec, dtype=torch.uint8, device="cuda")
    table = torch.full((1, E), -1, dtype=torch.int32, device="cuda")
    cache = M.SlotCache(1, E, S, rec, pool, slots, table)
    policy = o.SlotCacheLRU(E, S)
    side = torch.cuda.Stream()
    compute = torch.cuda.current_stream()
    steps = [np.stack([synth.drawn_routing(layer, E, K, 8, stream=t)[s] for t in range(4)]) for s in range(8)]
    rng = np.random.default_rng(61)
    steps.append(np.stack([rng.choice(E, size=K, replace=False) for _ in range(96)]).astype(np.int32))
    assert len(set(steps[-1].reshape(-1))) == E
    total_waves = 0
    for s, ids in enumerate(steps):
        T = ids.shape[0]
        x_cpu = synth.activations(T, H, seed=70 + s)
        x = x_cpu.cuda()
        buf = LayerBuffers(T, K, E, H, I)
        buf.topk_ids.copy_(torch.from_numpy(ids.astype(np.int32)))
        M.moe_route_topk(x, wr, T, H, E, K, None, M.MOE_IDS_GIVEN, buf.logits, buf.topk_ids, buf.topk_w)
        M.moe_group_tokens(buf.topk_ids, T, K, E, buf.counts, buf.offsets, buf.sorted_pair, buf.pair_pos,
                           buf.group_ws, buf.group_ws_bytes)
        buf.y.fill_(float("nan"))              # every row must be written by exactly one wave
        flat = [int(v) for v in ids.reshape(-1)]
        waves = cache.plan_waves(0, flat)
        assert waves == policy.plan_waves(flat), s
        total_waves += len(waves)
        for w in waves:
            slot_of, miss = cache.lookup(0, w)
            want_slots, want_loaded, _ = policy.lookup(w)
            assert (slot_of, miss) == (want_slots, want_loaded), s
            cache.fill(0, miss, side=side, compute=compute)
            M.moe_grouped_w4a16_ffn(x, buf.sorted_pair, buf.offsets, slots.data_ptr(), rec, table[0], S, T, K, E,
                                    H, I, M.MOE_PATH_AUTO, buf.y, buf.ffn_ws, buf.ffn_ws_bytes)
            cache.release(0, compute)
        out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
        M.moe_combine(buf.y, buf.topk_w, buf.pair_pos, x, T, K, H, out)
        assert M.moe_read_device_error(buf.ffn_ws) == 0
        assert not torch.isnan(buf.y).any(), s
        xr = x_cpu.double().numpy()
        gl = bf16_np(buf.logits)
        wrn = wr.cpu().double().numpy()
        assert_logits_close(gl, o.router_logits(xr, wrn), xr, wrn, "waves logits")
        w = o.weights_for_ids(gl, ids)
        assert np.allclose(buf.topk_w.cpu().numpy(), w, rtol=1e-5, atol=1e-8)
        ref = o.moe_layer_grouped(xr, _oracle_experts(layer), ids, w, residual=xr)
        assert_bf16_close(bf16_np(out), ref, f"waves step {s} (T={T}, {len(waves)} waves)")
    assert total_waves >= 8 * 2 + 4
    st = cache.stats()
    assert (st["hits"], st["misses"], st["h2d_bytes"]) == (policy.hits, policy.misses, policy.h2d_bytes(rec))
    cache.close()


def test_packed_pool_file_round_trip_runs_the_layer(M, tmp_path):
    """Pack once on the GPU, save the records to a pool file, load them back
    into pinned host memory, copy them to a fresh device bank, and run the
    layer from it: the bank is byte-identical to the packed one, the output
    bit-identical to the output from the packed bank and within the BF16 bar
    of the oracle (Figure 1 caption: packing happens a single time)."""
    from w4a16_mixture_experts_moe_b200.layer import ExpertBank, LayerBuffers, moe_layer_forward
    T = 16
    bank, wr = _gpu_bank(M, 0)
    host = bank.buf.cpu()
    path = str(tmp_path / "olmoe_layer0.pool")
    M.moe_pool_save(path, 1, E, H, I, bank.rec, host)
    info = M.moe_pool_file_info(path)
    assert info == {"layers": 1, "E": E, "H": H, "I": I, "record_bytes": bank.rec}
    pinned = torch.empty(E * bank.rec, dtype=torch.uint8, pin_memory=True)
    M.moe_pool_load(path, pinned, pinned.numel())
    loaded = ExpertBank(E, H, I)
    loaded.buf.copy_(pinned)
    assert torch.equal(loaded.buf, bank.buf)
    x = synth.activations(T, H, seed=81)
    outs = []
    for b in (bank, loaded):
        buf = LayerBuffers(T, K, E, H, I)
        outs.append((moe_layer_forward(x.cuda(), wr, b, buf).clone(), buf))
        assert M.moe_read_device_error(buf.ffn_ws) == 0
    assert torch.equal(outs[0][0], outs[1][0])
    _run_and_check(M, 0, x, outs[1][1], outs[1][0], "layer from a loaded pool")
