"""GPU parity: every step of the CUDA path, called through the C ABI, against
the CPU oracle on the same seeded inputs.

Bars: packed codes, scales, top-k ids (given identical logits) and the
grouping are bit-exact; BF16 outputs satisfy |d| <= 1e-2 + 1e-2 |ref|; fp32
routing weights agree to 1e-5 relative (fp32 softmax vs the oracle's fp64).
"""
import json
import os

import numpy as np
import pytest
import torch

import synth
from oracle import exactmoe_oracle as o
from tests._util import assert_bf16_close, bf16_np, torch_weights_source

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quant_pack_worked_example.json")


@pytest.fixture(scope="module")
def M():
    import w4a16_mixture_experts_moe_b200 as m
    assert torch.cuda.is_available()
    return m


def _dev(t):
    return t.cuda()


def _gpu_quantize(M, w):
    """w [E][N][K] BF16 cpu -> (packed [E][N][K/2] u8, scale bits [E][N][K/128] u16) via the C ABI."""
    E, N, K = w.shape
    wd = w.cuda().contiguous()
    packed = torch.empty(E, N, K // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(E, N, K // 128, dtype=torch.int16, device="cuda")
    M.moe_quantize_pack(wd, E, N, K, packed, N * K // 2, scales, N * K // 128 * 2)
    torch.cuda.synchronize()
    return packed.cpu().numpy(), scales.cpu().numpy().view(np.uint16)


# ------------------------------------------------------------------ A1 quantise + pack

def test_quantize_pack_worked_example(M):
    g = json.load(open(GOLDEN))
    w = torch.zeros(1, len(g["rows"]), g["K"])
    for r, row in enumerate(g["rows"]):
        for k, v in row["nonzero"].items():
            w[0, r, int(k)] = v
    packed, sbits = _gpu_quantize(M, w.to(torch.bfloat16))
    for r, row in enumerate(g["rows"]):
        assert packed[0, r, :8].tobytes().hex() == row["packed_first8_hex"]
        assert packed[0, r, 8:].tobytes().hex() == g["rest_of_row_byte_hex"] * 56
        assert "%04x" % sbits[0, r, 0] == row["scale_bits"]


@pytest.mark.parametrize("E,N,K", [(3, 64, 512), (1, 1024, 2048), (1, 4096, 1024)])
def test_quantize_pack_bitexact(M, E, N, K):
    w = synth.normal_bf16((E, N, K), 0.02, 7 + N)
    w[0, 1, :128] = 0                                       # all-zero group
    w[0, 2, :128] = 0
    w[0, 2, 5] = 0.03125                                    # one-hot group
    w[0, 3, :128] = torch.tensor([3.5] + [((i % 14) - 6.5) * 0.5 for i in range(127)])  # s = 0.5, w/s on .5 ties
    packed, sbits = _gpu_quantize(M, w)
    for e in range(E):
        p_ref, s_ref = o.quantize_pack(w[e].double().numpy())
        assert np.array_equal(packed[e], p_ref)
        assert np.array_equal(sbits[e], s_ref)


# ------------------------------------------------------------------ A2/A3 router + top-k

def _route_gpu(M, x, wr, k, bias=None, flags=0, logits_in=None, ids_in=None):
    T, H = x.shape
    E = wr.shape[0]
    logits = logits_in.cuda() if logits_in is not None else torch.empty(T, E, dtype=torch.bfloat16, device="cuda")
    ids = ids_in.cuda() if ids_in is not None else torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    b = None if bias is None else torch.from_numpy(bias).cuda()
    M.moe_route_topk(x.cuda(), wr.cuda(), T, H, E, k, b, flags, logits, ids, w)
    torch.cuda.synchronize()
    return logits.cpu(), ids.cpu().numpy(), w.cpu().double().numpy()


@pytest.mark.parametrize("T,H,E,k,renorm,skew", [
    (37, 2048, 64, 8, False, False), (1, 2048, 64, 8, False, False), (29, 4096, 8, 2, False, False),
    (29, 4096, 8, 2, True, False), (64, 2048, 64, 8, False, True), (9, 256, 256, 32, True, False),
    (65, 2048, 64, 8, False, False), (300, 2048, 64, 8, True, True)])
def test_route_topk(M, T, H, E, k, renorm, skew):
    # T <= 64 runs 2 tokens per cluster, larger T 8 (both kernels covered)
    x = synth.activations(T, H, seed=3 + T)
    wr = synth.router_weight(0, E, H)
    bias = synth.zipf_log_bias(E) if skew else None
    flags = M.MOE_RENORM if renorm else 0
    logits, ids, w = _route_gpu(M, x, wr, k, bias, flags)
    ref_logits = o.router_logits(x.double().numpy(), wr.double().numpy())
    got_logits = bf16_np(logits)
    assert_bf16_close(got_logits, ref_logits, "logits")
    # one BF16 rounding of an fp32 sum taken in any order: at most one BF16 ulp
    # plus the fp32 summation bound (H - 1) 2^-24 sum |x w| from the fp64 sum
    ulp = np.ldexp(1.0, np.frexp(ref_logits)[1] - 8)
    fp32_sum_bound = (H - 1) * 2.0 ** -24 * (np.abs(x.double().numpy()) @ np.abs(wr.double().numpy()).T)
    assert np.all(np.abs(got_logits - ref_logits) <= ulp + fp32_sum_bound)
    # top-k given identical logits: bit-exact ids
    ref_ids, ref_w = o.route_topk(got_logits, k, bias, renorm)
    assert np.array_equal(ids, ref_ids)
    np.testing.assert_allclose(w, ref_w, rtol=1e-5, atol=1e-7)


def test_route_topk_ties_nan_and_given(M):
    T, E, k = 8, 64, 8
    lg = np.zeros((T, E))
    lg[1] = 1.0
    lg[2, ::3] = 0.5
    lg[3, 10] = np.nan
    lg[3, 11:20] = 2.0
    lg[4, 1::2] = -0.0
    lg[5] = np.round(np.linspace(-1, 1, E) * 4) / 4            # many equal keys
    lg[6] = -np.inf
    lg[6, 63] = 0.0
    lg_t = torch.from_numpy(lg).to(torch.bfloat16)
    x = torch.zeros(T, 128, dtype=torch.bfloat16)
    wr = torch.zeros(E, 128, dtype=torch.bfloat16)
    _, ids, w = _route_gpu(M, x, wr, k, flags=M.MOE_LOGITS_GIVEN, logits_in=lg_t)
    ref_ids, ref_w = o.route_topk(bf16_np(lg_t), k)
    assert np.array_equal(ids, ref_ids)
    np.testing.assert_allclose(w, ref_w, rtol=1e-5, atol=1e-7)
    # ids given: only the weights of those ids
    given = torch.from_numpy(np.stack([np.arange(k) * 7 % E for _ in range(T)]).astype(np.int32))
    _, ids2, w2 = _route_gpu(M, x, wr, k, flags=M.MOE_LOGITS_GIVEN | M.MOE_IDS_GIVEN | M.MOE_RENORM,
                             logits_in=lg_t, ids_in=given)
    assert np.array_equal(ids2, given.numpy())
    np.testing.assert_allclose(w2, o.weights_for_ids(bf16_np(lg_t), given.numpy(), renorm=True), rtol=1e-5, atol=1e-7)


# ------------------------------------------------------------------ A4 grouping

def _group_gpu(M, ids, E):
    T, k = ids.shape
    d = torch.from_numpy(ids.astype(np.int32)).cuda()
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sp = torch.full((max(T * k, 1),), -7, dtype=torch.int32, device="cuda")
    pp = torch.full((max(T * k, 1),), -7, dtype=torch.int32, device="cuda")
    nb = M.moe_group_workspace_size(T, k, E)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    M.moe_group_tokens(d, T, k, E, counts, offsets, sp, pp, ws, nb)
    code = M.moe_read_device_error(ws)
    return counts.cpu().numpy(), offsets.cpu().numpy(), sp.cpu().numpy()[:T * k], pp.cpu().numpy()[:T * k], code


@pytest.mark.parametrize("T,k,E,skew", [(1, 8, 64, False), (16, 8, 64, False), (128, 8, 64, False),
                                        (129, 8, 64, False), (8192, 8, 64, False), (512, 8, 64, True),
                                        (2048, 2, 8, False), (100, 32, 256, False), (0, 8, 64, False)])
def test_group_tokens_bitexact(M, T, k, E, skew):
    rng = np.random.default_rng(T * 31 + k)
    if skew:
        p = np.exp(synth.zipf_log_bias(E).astype(np.float64))
        p = p / p.sum()
        ids = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)])
    else:
        ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]) if T else np.zeros((0, k))
    ids = ids.astype(np.int32).reshape(T, k)
    counts, offsets, sp, pp, code = _group_gpu(M, ids, E)
    rc, ro, rsp, rpp = o.group_tokens(ids, E)
    assert code == 0
    assert np.array_equal(counts, rc) and np.array_equal(offsets, ro)
    assert np.array_equal(sp, rsp) and np.array_equal(pp, rpp)


def test_group_tokens_flags_bad_ids(M):
    ids = np.array([[0, 1], [2, 99], [3, -1]], dtype=np.int32)
    counts, offsets, sp, pp, code = _group_gpu(M, ids, 8)
    assert code == M.MOE_DEVERR_EXPERT_ID
    assert offsets[-1] == 4 and pp[3] == -1 and pp[5] == -1
    assert list(sp[:4]) == [0, 1, 2, 4]


# ------------------------------------------------------------------ A5/A6 grouped FFN

def _make_bank(M, gate, up, down):
    from w4a16_mixture_experts_moe_b200.layer import ExpertBank
    E, I, H = gate.shape
    bank = ExpertBank(E, H, I)
    bank.pack(gate.cuda(), up.cuda(), down.cuda())
    torch.cuda.synchronize()
    return bank


def _ffn_gpu(M, bank, x, ids, k, path, E, expert_slot=None, n_slots=None, x16=None):
    """x16: an FP16 copy of x passed with MOE_FFN_X_F16 instead of x."""
    T, H = x.shape
    I = bank.I
    d = torch.from_numpy(ids.astype(np.int32)).cuda()
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sp = torch.empty(T * k, dtype=torch.int32, device="cuda")
    pp = torch.empty(T * k, dtype=torch.int32, device="cuda")
    gws = torch.zeros(M.moe_group_workspace_size(T, k, E), dtype=torch.uint8, device="cuda")
    M.moe_group_tokens(d, T, k, E, counts, offsets, sp, pp, gws, gws.numel())
    y = torch.full((T * k, H), float("nan"), dtype=torch.float32, device="cuda")
    nb = M.moe_ffn_workspace_size(T, k, E, H, I, path)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    es = None if expert_slot is None else torch.tensor(expert_slot, dtype=torch.int32, device="cuda")
    x_in, p_in = (x.cuda(), path) if x16 is None else (x16.cuda(), path | M.MOE_FFN_X_F16)
    M.moe_grouped_w4a16_ffn(x_in, sp, offsets, bank.ptr, bank.rec, es, bank.n if n_slots is None else n_slots,
                            T, k, E, H, I, p_in, y, ws, nb)
    code = M.moe_read_device_error(ws)
    # h is internal: the BF16-rounded value held in FP16 (exact) on both paths
    h = ws[256:256 + T * k * I * 2].view(torch.float16).view(T * k, I)
    return y.cpu().double().numpy(), h.float().cpu().double().numpy(), code


@pytest.mark.parametrize("path", ["gemv", "tc", "seq"])
@pytest.mark.parametrize("E,H,I,T,k", [(5, 256, 384, 13, 2), (4, 512, 256, 40, 3), (64, 2048, 1024, 16, 8),
                                       (8, 4096, 1024, 9, 2), (4, 512, 256, 300, 2), (6, 384, 640, 700, 3),
                                       (64, 2048, 1024, 1, 8), (64, 2048, 1024, 64, 8),
                                       (8, 1024, 1024, 40, 2), (4, 1024, 2048, 100, 2), (256, 512, 256, 5, 8),
                                       (64, 2048, 1024, 4, 8)])
def test_grouped_ffn(M, path, E, H, I, T, k):
    """Both FFN paths, and the sequential per-expert reference, against the oracle
    (with fewer (token, expert) pairs than experts the GEMV grid is compact:
    one row per possible active expert)."""
    P = {"gemv": M.MOE_PATH_GEMV, "tc": M.MOE_PATH_TC, "seq": M.MOE_PATH_SEQUENTIAL}[path]
    rng = np.random.default_rng(E * H + T)
    gate = synth.normal_bf16((E, I, H), 0.02, 1000 + E)
    up = synth.normal_bf16((E, I, H), 0.02, 2000 + E)
    down = synth.normal_bf16((E, H, I), 0.02, 3000 + E)
    x = synth.activations(T, H, seed=5)
    ids = np.stack([rng.choice(E - 1, size=k, replace=False) for _ in range(T)]).astype(np.int32)  # expert E-1 empty
    bank = _make_bank(M, gate, up, down)
    y, h, code = _ffn_gpu(M, bank, x, ids, k, P, E)
    assert code == 0
    experts = o.LazyQuantizedExperts(torch_weights_source(gate, up, down), E, H, I)
    counts, offsets, sp, pp = o.group_tokens(ids, E)
    ref_h, ref_y = o.grouped_ffn(x.double().numpy(), experts, sp, offsets, k)
    assert_bf16_close(h, ref_h, "h")
    assert_bf16_close(y, ref_y, "y")


@pytest.mark.parametrize("path", ["gemv", "tc", "seq"])
@pytest.mark.parametrize("E,H,I,T,k", [(64, 2048, 1024, 16, 8), (4, 512, 256, 300, 2), (6, 384, 640, 70, 3)])
def test_grouped_ffn_fp16_input(M, path, E, H, I, T, k):
    """MOE_FFN_X_F16: the FFN fed the FP16 copy of x computes bit for bit what
    it computes from the BF16 x (the same FP16 operands, no conversion pass),
    and so meets the oracle's bar too."""
    P = {"gemv": M.MOE_PATH_GEMV, "tc": M.MOE_PATH_TC, "seq": M.MOE_PATH_SEQUENTIAL}[path]
    rng = np.random.default_rng(E * H + T + 7)
    gate = synth.normal_bf16((E, I, H), 0.02, 1100 + E)
    up = synth.normal_bf16((E, I, H), 0.02, 2100 + E)
    down = synth.normal_bf16((E, H, I), 0.02, 3100 + E)
    x = synth.activations(T, H, seed=15)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    bank = _make_bank(M, gate, up, down)
    y, h, code = _ffn_gpu(M, bank, x, ids, k, P, E)
    x16 = torch.from_numpy(x.double().numpy().astype(np.float16))  # numpy's RNE conversion, not the library's
    y16, h16, code16 = _ffn_gpu(M, bank, x, ids, k, P, E, x16=x16)
    assert code == 0 and code16 == 0
    assert np.array_equal(y16, y) and np.array_equal(h16, h)
    experts = o.LazyQuantizedExperts(torch_weights_source(gate, up, down), E, H, I)
    counts, offsets, sp, pp = o.group_tokens(ids, E)
    ref_h, ref_y = o.grouped_ffn(x.double().numpy(), experts, sp, offsets, k)
    assert_bf16_close(y16, ref_y, "y from the FP16 input")


@pytest.mark.parametrize("T,H,E,k,flags", [(1, 2048, 64, 8, 0), (16, 2048, 64, 8, 0), (64, 2048, 64, 8, 0),
                                           (37, 4096, 8, 2, 0), (100, 2048, 64, 8, 0), (300, 1024, 64, 8, 0),
                                           (16, 2048, 64, 8, 2), (100, 2048, 64, 8, 2)])
def test_route_topk_x16(M, T, H, E, k, flags):
    """moe_route_topk_x16 routes exactly as moe_route_topk and writes the FP16
    copy of x: fused into the decode router kernel for T <= 64, a conversion
    pass otherwise, and with given logits (flags 2) a conversion pass too."""
    x = synth.activations(T, H, seed=21 + T)
    wr = synth.router_weight(0, E, H)
    given = flags & M.MOE_LOGITS_GIVEN
    lg_in = torch.from_numpy(np.round(np.random.default_rng(T).normal(size=(T, E)) * 8) / 8).to(torch.bfloat16)
    ref_logits, ref_ids, ref_w = _route_gpu(M, x, wr, k, flags=flags, logits_in=lg_in if given else None)
    logits = lg_in.cuda() if given else torch.empty(T, E, dtype=torch.bfloat16, device="cuda")
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    x16 = torch.full((T, H), float("nan"), dtype=torch.float16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_route_topk_x16(x.cuda(), wr.cuda(), T, H, E, k, None, flags, logits, ids, w, x16, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(logits.cpu(), ref_logits)
    assert np.array_equal(ids.cpu().numpy(), ref_ids)
    assert np.array_equal(w.cpu().double().numpy(), ref_w)
    want = x.double().numpy().astype(np.float16)  # numpy's RNE conversion of the BF16 values
    assert np.array_equal(x16.cpu().numpy().view(np.uint16), want.view(np.uint16))


@pytest.mark.parametrize("T", [16, 100])
def test_route_topk_x16_flags_values_beyond_fp16(M, T):
    H, E, k = 2048, 64, 8
    x = synth.activations(T, H, seed=4)
    x[T // 2, 77] = 1.0e5                      # beyond FP16's largest finite value
    logits = torch.empty(T, E, dtype=torch.bfloat16, device="cuda")
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    x16 = torch.empty(T, H, dtype=torch.float16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_route_topk_x16(x.cuda(), synth.router_weight(0, E, H).cuda(), T, H, E, k, None, 0, logits, ids, w, x16,
                         err)
    torch.cuda.synchronize()
    assert int(err.item()) == M.MOE_DEVERR_RANGE


@pytest.mark.parametrize("E,H,I,T,k", [(5, 256, 384, 13, 2), (64, 2048, 1024, 16, 8), (8, 4096, 1024, 9, 2),
                                       (4, 512, 256, 300, 2), (64, 2048, 1024, 1, 8)])
def test_grouped_bf16_ffn(M, E, H, I, T, k):
    """The BF16 baseline: unquantised experts through moe_grouped_bf16_ffn
    against the oracle's grouped FFN on the same BF16 weights."""
    from w4a16_mixture_experts_moe_b200.layer import Bf16Bank
    rng = np.random.default_rng(E * H + T + 1)
    gate = synth.normal_bf16((E, I, H), 0.02, 1100 + E)
    up = synth.normal_bf16((E, I, H), 0.02, 2100 + E)
    down = synth.normal_bf16((E, H, I), 0.02, 3100 + E)
    x = synth.activations(T, H, seed=6)
    ids = np.stack([rng.choice(E - 1, size=k, replace=False) for _ in range(T)]).astype(np.int32)  # expert E-1 empty
    bank = Bf16Bank(E, H, I)
    bank.load(gate.cuda(), up.cuda(), down.cuda())
    d = torch.from_numpy(ids).cuda()
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sp = torch.empty(T * k, dtype=torch.int32, device="cuda")
    pp = torch.empty(T * k, dtype=torch.int32, device="cuda")
    gws = torch.zeros(M.moe_group_workspace_size(T, k, E), dtype=torch.uint8, device="cuda")
    M.moe_group_tokens(d, T, k, E, counts, offsets, sp, pp, gws, gws.numel())
    y = torch.full((T * k, H), float("nan"), dtype=torch.float32, device="cuda")
    nb = M.moe_bf16_ffn_workspace_size(T, k, E, H, I)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    M.moe_grouped_bf16_ffn(x.cuda(), sp, offsets, bank.ptr, bank.rec, T, k, E, H, I, y, ws, nb)
    torch.cuda.synchronize()
    h = ws[256:256 + T * k * I * 2].view(torch.bfloat16).view(T * k, I).double().cpu().numpy()
    experts = o.Bf16Experts(torch_weights_source(gate, up, down), E, H, I)
    _, o_off, o_sp, _ = o.group_tokens(ids, E)
    ref_h, ref_y = o.grouped_ffn(x.double().numpy(), experts, o_sp, o_off, k)
    assert_bf16_close(h, ref_h, "bf16 h")
    assert_bf16_close(y.cpu().double().numpy(), ref_y, "bf16 y")


def test_grouped_ffn_not_resident_is_flagged(M):
    E, H, I, T, k = 4, 256, 256, 6, 2
    gate = synth.normal_bf16((E, I, H), 0.02, 1)
    up = synth.normal_bf16((E, I, H), 0.02, 2)
    down = synth.normal_bf16((E, H, I), 0.02, 3)
    bank = _make_bank(M, gate, up, down)
    ids = np.array([[0, 1]] * T, dtype=np.int32)
    _, _, code = _ffn_gpu(M, bank, synth.activations(T, H), ids, k, M.MOE_PATH_GEMV, E,
                          expert_slot=[0, -1, 2, 3], n_slots=4)
    assert code == M.MOE_DEVERR_NOT_RESIDENT


# ------------------------------------------------------------------ A7 combine

@pytest.mark.parametrize("T,k,H,res,drop", [(16, 8, 2048, True, False), (5, 2, 4096, False, False),
                                            (1, 8, 2048, True, False), (7, 4, 2048, True, True)])
def test_combine(M, T, k, H, res, drop):
    rng = np.random.default_rng(T + k)
    y = synth.normal_bf16((T * k, H), 0.5, 77).float() * 1.001   # fp32 values with low bits set
    w = torch.from_numpy(rng.random((T, k)).astype(np.float32))
    perm = rng.permutation(T * k).astype(np.int32)
    if drop:                                                       # dropped pairs contribute nothing
        perm[[0, 5, 13]] = -1
    pp = torch.from_numpy(perm)
    r = synth.activations(T, H, seed=78) if res else None
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    M.moe_combine(y.cuda(), w.cuda(), pp.cuda(), None if r is None else r.cuda(), T, k, H, out)
    torch.cuda.synchronize()
    ref = o.combine(y.double().numpy(), w.double().numpy(), pp.numpy(), None if r is None else r.double().numpy())
    assert y.dtype == torch.float32
    assert_bf16_close(bf16_np(out), ref, "combine")
    assert np.mean(bf16_np(out) == ref) > 0.99   # one final rounding on both sides


def test_tc_pipeline_wait_times_out_and_reports(M):
    """Failure detection without a fault: the producers of one tensor-core FFN
    call never publish a stage, every bounded wait runs out (~2 s), the kernels
    drain and return, MOE_DEVERR_TIMEOUT is read back, and the next call on the
    same context is correct again."""
    import time
    E, H, I, T, k = 4, 256, 256, 160, 2
    gate = synth.normal_bf16((E, I, H), 0.02, 11)
    up = synth.normal_bf16((E, I, H), 0.02, 12)
    down = synth.normal_bf16((E, H, I), 0.02, 13)
    bank = _make_bank(M, gate, up, down)
    x = synth.activations(T, H, seed=14)
    ids = np.stack([np.arange(k) + (t % (E - 1)) for t in range(T)]).astype(np.int32) % E
    M.moe_debug_stall_next_tc_ffn(1)
    t0 = time.time()
    _, _, code = _ffn_gpu(M, bank, x, ids, k, M.MOE_PATH_TC, E)
    assert code == M.MOE_DEVERR_TIMEOUT
    assert time.time() - t0 < 30
    y, _, code = _ffn_gpu(M, bank, x, ids, k, M.MOE_PATH_TC, E)
    assert code == 0
    experts = o.LazyQuantizedExperts(torch_weights_source(gate, up, down), E, H, I)
    _, offsets, sp, _ = o.group_tokens(ids, E)
    _, ref_y = o.grouped_ffn(x.double().numpy(), experts, sp, offsets, k)
    assert_bf16_close(y, ref_y, "y after timeout")
