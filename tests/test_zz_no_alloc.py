"""moe_permute_noalloc: the dispatch permutation for callers that cannot
allocate device memory (for example a serving engine whose memory is all
pre-assigned to fixed pools, or a plugin host that gives the library no
allocator). Its scratch lives in a fixed device array owned by the library,
so its results must be identical to moe_permute's, which takes a caller
workspace, on consecutive calls that reuse that array.

This file is collected last so that a stop-at-first-failure run has already
run every other test if it fails.
"""
import numpy as np
import pytest
import torch

from fine_grained_sparse_fp32_b200 import _build, kmoe

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _build.build()
    kmoe.load()


def _rows(seed, N, K, E, skew):
    rng = np.random.default_rng(seed)
    if skew:
        p = 1.0 / np.arange(1, E + 1) ** 1.1
        p = p[rng.permutation(E)]
        p /= p.sum()
        return np.stack([rng.choice(E, size=K, replace=False, p=p) for _ in range(N)]).astype(np.int32)
    return np.argsort(rng.random((N, E)), axis=1)[:, :K].astype(np.int32)


def test_noalloc_permute_equals_workspace_permute_on_two_calls_in_a_row():
    E, K = 384, 6
    # a large call, then a smaller one that reads back only what it wrote
    for seed, N, skew in ((1, 65536, True), (2, 5000, False)):
        idx = torch.from_numpy(_rows(seed, N, K, E, skew)).cuda()
        ref = kmoe.moe_permute(idx, E)
        got = kmoe.moe_permute_noalloc(idx, E)
        torch.cuda.synchronize()
        for r, g in zip(ref, got):
            assert torch.equal(r, g)        # integer outputs: bit-exact, as for moe_permute
        assert int(got[0].sum()) == N * K


def test_noalloc_permute_rejects_sizes_beyond_its_fixed_scratch():
    idx = torch.zeros((65537, 6), dtype=torch.int32, device="cuda")
    with pytest.raises(kmoe.KmoeError) as exc:
        kmoe.moe_permute_noalloc(idx, 1024)
    assert exc.value.status == kmoe.KMOE_ERR_UNSUPPORTED
    assert "fixed array" in str(exc.value)
