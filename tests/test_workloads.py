"""CPU checks of the synthetic workloads' recipes (no GPU, no oracle).

The skewed-routing workload asks for about half of all routed slots on the
10 % most popular experts (38 of 384) and about 20 experts with no token. The
recipe adds a Zipf(1.1) popularity times SKEW_BETA to the correction bias; this
checks the resulting shares on simulated logits with the statistics of the
layer's router (x ~ N(0, 1) against router rows ~ N(0, 0.02) over d = 2560:
each logit ~ N(0, 2560 * 0.02^2), independent across experts to first order).
The GPU parity test checks the same shares on the real router's logits.
"""
import numpy as np
import pytest

from fine_grained_sparse_fp32_b200.inputs import CONFIGS, SKEW_BETA, SKEW_EMPTY


def _shares(beta, seed, N=20000):
    cfg = CONFIGS["skew"]
    E, K = cfg.E, cfg.K
    rng = np.random.default_rng(seed)
    logits = rng.normal(0.0, np.sqrt(cfg.d) * 0.02, size=(N, E))
    rank = rng.permutation(E) + 1.0
    bias = rng.uniform(-0.1, 0.1, E) - beta * 1.1 * np.log(rank)
    bias[rng.permutation(E)[:SKEW_EMPTY]] = -30.0
    idx = np.argpartition(-(logits + bias[None, :]), K, axis=1)[:, :K]
    counts = np.bincount(idx.ravel(), minlength=E)
    return np.sort(counts)[::-1][:38].sum() / (N * K), int((counts == 0).sum())


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_skew_recipe_puts_half_the_slots_on_ten_percent_of_experts(seed):
    top, empty = _shares(SKEW_BETA, seed)
    assert 0.45 <= top <= 0.55
    assert empty >= SKEW_EMPTY


def test_skew_recipe_is_not_far_more_skewed_than_asked():
    # a steeper popularity (the earlier 0.62) concentrates ~80 % of slots on the top 10 %
    assert _shares(0.62, 1)[0] > 0.75 > _shares(SKEW_BETA, 1)[0]
