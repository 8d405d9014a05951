"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch

ATOL = 1e-2
RTOL = 1e-2


def bf16_np(t: torch.Tensor) -> np.ndarray:
    """BF16 tensor (any device) -> exact float64 numpy array."""
    return t.detach().float().cpu().double().numpy()


def assert_bf16_close(got, ref, what=""):
    """|got - ref| <= 1e-2 + 1e-2 |ref| elementwise (the stated BF16 bar)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    bad = ~(np.abs(got - ref) <= ATOL + RTOL * np.abs(ref))
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first "
                             f"{[(tuple(i), got[tuple(i)], ref[tuple(i)]) for i in idx]}")
    return float(np.max(np.abs(got - ref))) if got.size else 0.0


def torch_weights_source(gate, up, down):
    """Oracle expert source over CPU BF16 tensors [E][N][K]."""
    def weights_of(e):
        return gate[e].double().numpy(), up[e].double().numpy(), down[e].double().numpy()
    return weights_of


def assert_logits_close(got, ref, x, wr, what=""):
    """Router logits: one BF16 rounding of an fp32 sum taken in any order is
    within one BF16 ulp of the fp64 oracle's rounded sum plus the fp32
    summation bound (H - 1) 2^-24 sum_h |x w| (which matters near zero,
    where a BF16 ulp is tiny and the fp32 sum cancels)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    wr = np.asarray(wr, dtype=np.float64)
    ulp = np.ldexp(1.0, np.frexp(ref)[1] - 8)
    bound = ulp + (x.shape[1] - 1) * 2.0 ** -24 * (np.abs(x) @ np.abs(wr).T)
    bad = ~(np.abs(got - ref) <= bound)
    assert not bad.any(), f"{what}: {int(bad.sum())} logits beyond one BF16 ulp + the fp32 summation bound"
