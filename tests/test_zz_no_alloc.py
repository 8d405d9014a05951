"""The grouping entry point that allocates nothing, checked on the GPU.

Some callers cannot call cudaMalloc: code running under CUDA stream capture,
or inside a framework that owns all device memory and hands out no scratch.
moe_group_tokens_noalloc serves them with a fixed scratch array inside the
library. This test calls it through the C ABI twice in a row (a single-chunk
and a multi-chunk size, so the second call reuses scratch the first one
left behind) and checks that its outputs equal moe_group_tokens' with a
caller-provided workspace. Integer outputs: the comparison is exact. The file
name sorts last so a run that stops at the first failure has already run
every other test.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _outputs(T, k, E):
    d = dict(dtype=torch.int32, device="cuda")
    return (torch.full((E,), -5, **d), torch.full((E + 1,), -5, **d), torch.full((T * k,), -5, **d),
            torch.full((T * k,), -5, **d))


@pytest.fixture(scope="module")
def M():
    import w4a16_mixture_experts_moe_b200 as m
    assert torch.cuda.is_available()
    return m


def test_noalloc_grouping_matches_workspace_grouping_twice(M):
    rng = np.random.default_rng(2024)
    for T, k, E in [(16, 8, 64), (3000, 8, 64)]:           # second call: several chunks
        ids_np = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        ids = torch.from_numpy(ids_np).cuda()
        ref = _outputs(T, k, E)
        ws = torch.empty(M.moe_group_workspace_size(T, k, E), dtype=torch.uint8, device="cuda")
        M.moe_group_tokens(ids, T, k, E, *ref, ws, ws.numel())
        got = _outputs(T, k, E)
        M.moe_group_tokens_noalloc(ids, T, k, E, *got)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)


def test_noalloc_rejects_sizes_beyond_its_limit(M):
    T, k = M.MOE_NOALLOC_MAX_PAIRS // 8 + 1, 8
    with pytest.raises(M.MoeError) as ei:
        M.moe_group_tokens_noalloc(0, T, k, 64, 0, 0, 0, 0)
    assert ei.value.status == 2 and "scratch limit" in str(ei.value)
