"""GPU edge cases of the hot path, against the CPU oracle.

Empty batches on every entry point; all tokens routed to one expert (a group
that spans two 256-row tensor-core tiles, and many 8-token GEMV chunks); the
smallest dimensions (one 128-wide quantisation group, so some K-split warps
have no group); the largest expert count. Bars as in test_gpu_parity.
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
