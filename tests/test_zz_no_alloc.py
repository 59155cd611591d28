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

import oracle
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


def _spread_rows(seed, N, K, E):
    """K distinct experts per token: a random start plus K evenly spaced offsets (cheap at large N)."""
    base = np.random.default_rng(seed).integers(0, E, size=(N, 1))
    return ((base + np.arange(K)[None, :] * (E // K)) % E).astype(np.int32)


@pytest.mark.parametrize("N,E,K", [(65536, 1024, 8),    # ceil(N/256) * E == 262144: the array exactly full
                                   (32, 384, 6), (256, 384, 6),   # single-CTA sizes (no scratch used)
                                   (257, 384, 6)])               # the first size that uses chunk histograms
def test_noalloc_permute_matches_the_oracle_directly(N, E, K):
    idx = _spread_rows(N + E, N, K, E)
    got = kmoe.moe_permute_noalloc(torch.from_numpy(idx).cuda(), E)
    ref = kmoe.moe_permute(torch.from_numpy(idx).cuda(), E)
    torch.cuda.synchronize()
    for want, g, r in zip(oracle.permute(idx, E), got, ref):
        np.testing.assert_array_equal(g.cpu().numpy().reshape(np.shape(want)), want)
        assert torch.equal(g, r)


def test_noalloc_permute_zero_tokens_writes_zero_counts_and_offsets():
    E = 384
    counts = torch.full((E,), 7, dtype=torch.int32, device="cuda")
    offsets = torch.full((E + 1,), 7, dtype=torch.int32, device="cuda")
    kmoe.moe_permute_noalloc(torch.empty((0, 6), dtype=torch.int32, device="cuda"), E, counts=counts, offsets=offsets)
    torch.cuda.synchronize()
    assert int(counts.abs().sum()) == 0 and int(offsets.abs().sum()) == 0
