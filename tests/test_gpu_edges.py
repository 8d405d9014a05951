"""GPU edge cases of the hot path, against the CPU oracle.

Empty batches on every entry point; all tokens routed to one expert (a group
that spans two 256-row tensor-core tiles, and many 8-token GEMV chunks); the
smallest dimensions (one 128-wide quantisation group, so some K-split warps
have no group); the largest expert count; the FP16 operand domain (weight
scales far below and above FP16's range, an activation at and beyond FP16's
largest value, an intermediate h beyond it). Bars as in test_gpu_parity.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import exactmoe_oracle as o
from tests._util import assert_bf16_close, torch_weights_source
from tests.test_gpu_parity import _ffn_gpu, _make_bank

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    import w4a16_mixture_experts_moe_b200 as m
    assert torch.cuda.is_available()
    return m


def test_empty_batch_is_a_no_op(M):
    E, k, H, I = 8, 2, 256, 256
    dev = dict(device="cuda")
    x = torch.zeros(1, H, dtype=torch.bfloat16, **dev)
    wr = synth.router_weight(0, E, H, device="cuda")
    logits = torch.full((1, E), 7.0, dtype=torch.bfloat16, **dev)
    ids = torch.full((1, k), 5, dtype=torch.int32, **dev)
    w = torch.full((1, k), 0.25, dtype=torch.float32, **dev)
    M.moe_route_topk(x, wr, 0, H, E, k, None, 0, logits, ids, w)
    torch.cuda.synchronize()
    assert torch.all(logits == 7.0) and torch.all(ids == 5) and torch.all(w == 0.25)

    counts = torch.full((E,), 9, dtype=torch.int32, **dev)
    offsets = torch.full((E + 1,), 9, dtype=torch.int32, **dev)
    sp = torch.full((1,), 9, dtype=torch.int32, **dev)
    pp = torch.full((1,), 9, dtype=torch.int32, **dev)
    gws = torch.zeros(M.moe_group_workspace_size(0, k, E), dtype=torch.uint8, **dev)
    M.moe_group_tokens(ids, 0, k, E, counts, offsets, sp, pp, gws, gws.numel())
    rc, ro, _, _ = o.group_tokens(np.zeros((0, k), dtype=np.int32), E)
    assert np.array_equal(counts.cpu().numpy(), rc) and np.array_equal(offsets.cpu().numpy(), ro)
    assert M.moe_read_device_error(gws) == 0

    gate = synth.normal_bf16((E, I, H), 0.02, 1)
    up = synth.normal_bf16((E, I, H), 0.02, 2)
    down = synth.normal_bf16((E, H, I), 0.02, 3)
    bank = _make_bank(M, gate, up, down)
    y = torch.full((1, H), 3.0, dtype=torch.float32, **dev)
    zero_off = torch.zeros(E + 1, dtype=torch.int32, **dev)
    for path in (M.MOE_PATH_GEMV, M.MOE_PATH_TC, M.MOE_PATH_AUTO):
        nb = M.moe_ffn_workspace_size(0, k, E, H, I, path)
        ws = torch.zeros(nb, dtype=torch.uint8, **dev)
        M.moe_grouped_w4a16_ffn(x, sp, zero_off, bank.ptr, bank.rec, None, E, 0, k, E, H, I, path, y, ws, nb)
        assert M.moe_read_device_error(ws) == 0
    assert torch.all(y == 3.0)

    out = torch.full((1, H), 2.0, dtype=torch.bfloat16, **dev)
    M.moe_combine(y, w, pp, None, 0, k, H, out)
    torch.cuda.synchronize()
    assert torch.all(out == 2.0)


def _ffn_case(M, path, E, H, I, T, k, ids, seed):
    gate = synth.normal_bf16((E, I, H), 0.02, 1000 + seed)
    up = synth.normal_bf16((E, I, H), 0.02, 2000 + seed)
    down = synth.normal_bf16((E, H, I), 0.02, 3000 + seed)
    x = synth.activations(T, H, seed=seed)
    bank = _make_bank(M, gate, up, down)
    P = {"gemv": M.MOE_PATH_GEMV, "tc": M.MOE_PATH_TC}[path]
    y, h, code = _ffn_gpu(M, bank, x, ids, k, P, E)
    assert code == 0
    experts = o.LazyQuantizedExperts(torch_weights_source(gate, up, down), E, H, I)
    _, offsets, sp, _ = o.group_tokens(ids, E)
    ref_h, ref_y = o.grouped_ffn(x.double().numpy(), experts, sp, offsets, k)
    assert_bf16_close(h, ref_h, "h")
    assert_bf16_close(y, ref_y, "y")


@pytest.mark.parametrize("path", ["gemv", "tc"])
def test_all_tokens_to_one_expert(M, path):
    # 300 rows in expert 2: two tensor-core token tiles (256 + 44), 38 GEMV chunks
    E, H, I, T, k = 4, 256, 256, 300, 1
    ids = np.full((T, k), 2, dtype=np.int32)
    _ffn_case(M, path, E, H, I, T, k, ids, seed=11)


@pytest.mark.parametrize("path", ["gemv", "tc"])
def test_smallest_dimensions(M, path):
    # H = I = 128: one quantisation group per row, so warps of a K split beyond
    # the first have no group of their own
    E, H, I, T, k = 3, 128, 128, 7, 2
    rng = np.random.default_rng(12)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    _ffn_case(M, path, E, H, I, T, k, ids, seed=12)


def test_largest_expert_count(M):
    E, H, I, T, k = 256, 256, 256, 5, 8
    rng = np.random.default_rng(13)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    _ffn_case(M, "gemv", E, H, I, T, k, ids, seed=13)


# ---------------------------------------------------------------- FP16 operand domain

@pytest.mark.parametrize("path", ["gemv", "tc"])
def test_extreme_weight_scales_are_exact(M, path):
    """Weight groups whose scales lie far outside FP16's comfortable range.
    Expert 0: gate/up scaled by 2^-12 (scales near 2^-19) and down by 2^-20
    (scales near 2^-27, below FP16's smallest subnormal). Expert 1: gate/up
    scaled by 2^22 (scales above 8188, where 8 s exceeds FP16's range). Both
    paths form the products exactly and sum them in fp32, so h must match the
    oracle to one BF16 ulp, and y must match the oracle's down projection of
    the GPU's own h to 1e-5 of the row's largest output."""
    E, H, I, T, k = 2, 256, 256, 8, 1
    gate = synth.normal_bf16((E, I, H), 0.02, 31).float()
    up = synth.normal_bf16((E, I, H), 0.02, 32).float()
    down = synth.normal_bf16((E, H, I), 0.02, 33).float()
    gate[0] *= 2.0 ** -12; up[0] *= 2.0 ** -12; down[0] *= 2.0 ** -20
    gate[1] *= 2.0 ** 22; up[1] *= 2.0 ** 22
    gate, up, down = (w.to(torch.bfloat16) for w in (gate, up, down))
    x = synth.activations(T, H, seed=34).float()
    x[:4] *= 1000.0                                 # tokens of expert 0
    x[4:] *= 2.0 ** -14                             # tokens of expert 1 (>= 2^-17 after scaling, mostly)
    x = x.to(torch.bfloat16)
    ids = np.array([[0]] * 4 + [[1]] * 4, dtype=np.int32)
    bank = _make_bank(M, gate, up, down)
    P = {"gemv": M.MOE_PATH_GEMV, "tc": M.MOE_PATH_TC}[path]
    y, h, code = _ffn_gpu(M, bank, x, ids, k, P, E)
    assert code == 0
    experts = o.LazyQuantizedExperts(torch_weights_source(gate, up, down), E, H, I)
    _, offsets, sp, _ = o.group_tokens(ids, E)
    xr = x.double().numpy()
    # the activations the kernels consume are FP16 copies: tokens whose
    # smallest non-zero |x| is below 2^-17 are rounded by design (documented
    # domain); compare on the exact FP16 values so the test isolates the weights
    x16 = x.to(torch.float16).double().numpy()
    ref_h, _ = o.grouped_ffn(x16, experts, sp, offsets, k)
    # h is the BF16 value (one ulp from the oracle's at most) held in FP16,
    # which rounds magnitudes below 2^-17 to a multiple of 2^-24 (documented)
    ulp = np.ldexp(1.0, np.frexp(np.abs(ref_h))[1] - 8) + 2.0 ** -25
    assert np.all(np.abs(h - ref_h) <= ulp), float(np.max(np.abs(h - ref_h) / ulp))
    ref_y = np.zeros_like(y)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        ref_y[lo:hi] = h[lo:hi] @ experts.dequantized(e)[2].T
    scale = np.max(np.abs(ref_y), axis=1, keepdims=True)
    assert np.all(scale > 0)
    assert np.all(np.abs(y - ref_y) <= 1e-5 * scale), float(np.max(np.abs(y - ref_y) / scale))
    assert np.max(np.abs(xr - x16)) < 2.0 ** -24   # the FP16 copy differs from x only below 2^-17


@pytest.mark.parametrize("path", ["gemv", "tc"])
def test_activation_beyond_fp16_range_is_flagged(M, path):
    E, H, I, T, k = 4, 256, 256, 6, 2
    gate = synth.normal_bf16((E, I, H), 0.02, 41).float()
    up = synth.normal_bf16((E, I, H), 0.02, 42).float()
    down = synth.normal_bf16((E, H, I), 0.02, 43)
    gate[:, :, 17] = 0.0
    up[:, :, 17] = 0.0
    bank = _make_bank(M, gate.to(torch.bfloat16), up.to(torch.bfloat16), down)
    ids = np.array([[t % E, (t + 1) % E] for t in range(T)], dtype=np.int32)
    P = {"gemv": M.MOE_PATH_GEMV, "tc": M.MOE_PATH_TC}[path]
    # at the edge: 65280 is the largest BF16 value FP16 holds; column 17 has
    # zero weights, so h stays small and the result is exact and unflagged
    x = synth.activations(T, H, seed=44).float()
    x[3, 17] = 65280.0
    x = x.to(torch.bfloat16)
    y, h, code = _ffn_gpu(M, bank, x, ids, k, P, E)
    assert code == 0
    experts = o.LazyQuantizedExperts(torch_weights_source(gate.to(torch.bfloat16), up.to(torch.bfloat16), down),
                                     E, H, I)
    _, offsets, sp, _ = o.group_tokens(ids, E)
    ref_h, ref_y = o.grouped_ffn(x.double().numpy(), experts, sp, offsets, k)
    assert_bf16_close(h, ref_h, "h at the FP16 edge")
    assert_bf16_close(y, ref_y, "y at the FP16 edge")
    # beyond it: 1e5 (BF16 99840) has no FP16 copy; the call reports it
    x = x.float()
    x[3, 17] = 1e5
    _, _, code = _ffn_gpu(M, bank, x.to(torch.bfloat16), ids, k, P, E)
    assert code == M.MOE_DEVERR_RANGE


@pytest.mark.parametrize("path", ["gemv", "tc"])
def test_intermediate_beyond_fp16_range_is_flagged(M, path):
    # token 2's activations are all 100 and expert 1's gate/up weights all
    # 0.5: g = u = 12800, h = 1.6e8, which the FP16 operand of the down pass
    # cannot hold
    E, H, I, T, k = 2, 256, 256, 4, 1
    gate = synth.normal_bf16((E, I, H), 0.02, 51).float()
    up = synth.normal_bf16((E, I, H), 0.02, 52).float()
    gate[1] = 0.5
    up[1] = 0.5
    down = synth.normal_bf16((E, H, I), 0.02, 53)
    bank = _make_bank(M, gate.to(torch.bfloat16), up.to(torch.bfloat16), down)
    x = synth.activations(T, H, seed=54).float()
    x[2] = 100.0
    ids = np.array([[0], [0], [1], [0]], dtype=np.int32)
    P = {"gemv": M.MOE_PATH_GEMV, "tc": M.MOE_PATH_TC}[path]
    _, _, code = _ffn_gpu(M, bank, x.to(torch.bfloat16), ids, k, P, E)
    assert code == M.MOE_DEVERR_RANGE
