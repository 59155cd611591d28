"""Pins for the CPU oracle: each check ties it to something other than itself.

- E4M3 decoding: all 256 codes against torch.float8_e4m3fn.
- Router: numpy float64 matmul.
- Top-k: brute-force enumeration of all K-subsets, and Python's sort for ties.
- Mixture weights: exact sigmoid values and the unbiased-logit rule under a
  bias that forces the selection.
- Permutation: Python's stable sort of (expert, token) pairs.
- Expert FFN and combine: a hand-computed d = I = 1 layer, numpy float64 SwiGLU
  on a non-square expert, and the closed forms (x = 0, zero routed down
  projection, identical experts).
- FP8 block scales: the E4M3 layer equals the FP32 layer on the decoded weights,
  and closed forms on weights whose every code is 1.0 with a distinct scale per
  128 x 128 block (several blocks along both axes, non-square), for both the
  BF16-activation and the FP8-activation expert.
- Shapes: the weight counts printed on the pages.
"""
import itertools
import ctypes
import math
import os

import numpy as np
import pytest
import torch

import oracle
from fine_grained_sparse_fp32_b200.inputs import CONFIGS, LayerConfig, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def test_e4m3_all_codes_match_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle.e4m3_to_double(c)
        if np.isnan(ref[c]):
            assert np.isnan(got), c
        else:
            assert got == ref[c], (c, got, ref[c])
    assert oracle.e4m3_to_double(0x7E) == 448.0
    assert oracle.e4m3_to_double(0x01) == 2.0 ** -9


def test_router_matches_numpy_float64():
    inp = make_inputs(CONFIGS["tiny"], seed=0)
    l = oracle.router_logits(inp["x"], "f32", inp["w_router"], nthreads=2)
    ref = inp["x"].double().numpy() @ inp["w_router"].double().numpy().T
    np.testing.assert_allclose(l, ref, rtol=1e-12, atol=1e-12)


def test_router_bf16_input_widened_exactly():
    cfg = LayerConfig("t", 4, 256, 16, 6, 128, "bf16", "bf16")
    inp = make_inputs(cfg, seed=3)
    l = oracle.router_logits(inp["x"], "bf16", inp["w_router"])
    ref = inp["x"].double().numpy() @ inp["w_router"].double().numpy().T
    np.testing.assert_allclose(l, ref, rtol=1e-12, atol=1e-12)


def test_topk_matches_bruteforce_subsets():
    rng = np.random.default_rng(1)
    E, K, N = 10, 6, 200
    logits = rng.normal(size=(N, E))
    bias = rng.uniform(-0.5, 0.5, size=E).astype(np.float32)
    idx, g, margin = oracle.select(logits, bias, K)
    s = logits + bias.astype(np.float64)
    for t in range(N):
        best = max(itertools.combinations(range(E), K), key=lambda c: sum(s[t, list(c)]))
        assert set(idx[t]) == set(best)
        assert all(s[t, idx[t, k]] >= s[t, idx[t, k + 1]] for k in range(K - 1))
        rest = sorted(set(range(E)) - set(best), key=lambda e: -s[t, e])
        assert margin[t] == pytest.approx(s[t, idx[t, K - 1]] - s[t, rest[0]], abs=1e-15)
        for k in range(K):
            assert g[t, k] == pytest.approx(_sig(logits[t, idx[t, k]]), rel=1e-15)


def test_topk_ties_go_to_lower_index():
    E, K = 12, 6
    rng = np.random.default_rng(2)
    for _ in range(50):
        logits = rng.integers(-2, 3, size=(1, E)).astype(np.float64)  # many exact ties
        bias = np.zeros(E, dtype=np.float32)
        idx, _, margin = oracle.select(logits, bias, K)
        order = sorted(range(E), key=lambda e: (-logits[0, e], e))
        assert list(idx[0]) == order[:K]
        assert margin[0] == logits[0, order[K - 1]] - logits[0, order[K]]


def test_mixture_weights_use_unbiased_logits_without_renormalising():
    E, K = 16, 6
    logits = np.zeros((2, E))
    logits[0, :] = -1.0
    logits[0, [3, 5, 7, 9, 11, 13]] = [0.0, math.log(3.0), 0.0, math.log(3.0), 0.0, 0.0]
    logits[1, :] = 2.0                       # best unbiased logits sit on 0..5 ...
    logits[1, [3, 5, 7, 9, 11, 13]] = 0.0
    bias = np.zeros(E, dtype=np.float32)
    bias[[3, 5, 7, 9, 11, 13]] = 30.0       # ... but the bias forces these six
    idx, g, _ = oracle.select(logits, bias, K)
    for t in range(2):
        assert sorted(idx[t]) == [3, 5, 7, 9, 11, 13]
    # sigmoid(0) = 1/2 and sigmoid(ln 3) = 3/4, from the unbiased logits
    assert sorted(g[0]) == pytest.approx([0.5, 0.5, 0.5, 0.5, 0.75, 0.75], abs=1e-15)
    assert list(g[1]) == [0.5] * 6
    assert abs(g[0].sum() - 1.0) > 1.0       # not renormalised to one


def test_softmax_score_closed_form_on_the_forced_six():
    """Softmax over the selected experts ("Kolibri 1 Deep Dive", routing formulation)
    on a forced selection: unbiased logits (0, ln3, 0, ln3, 0, 0) have exponentials
    1, 3, 1, 3, 1, 1 (sum 10), so the weights are 1/10 and 3/10."""
    E, K = 16, 6
    logits = np.full((1, E), 5.0)            # the best unbiased logits are elsewhere ...
    logits[0, [3, 5, 7, 9, 11, 13]] = [0.0, math.log(3.0), 0.0, math.log(3.0), 0.0, 0.0]
    bias = np.zeros(E, dtype=np.float32)
    bias[[3, 5, 7, 9, 11, 13]] = 30.0        # ... the bias forces these six
    idx, g, _ = oracle.select(logits, bias, K, score="softmax")
    assert sorted(idx[0]) == [3, 5, 7, 9, 11, 13]
    by_e = dict(zip(idx[0].tolist(), g[0].tolist()))
    for e in (3, 7, 11, 13):
        assert by_e[e] == pytest.approx(0.1, abs=1e-15)
    for e in (5, 9):
        assert by_e[e] == pytest.approx(0.3, abs=1e-15)


def test_softmax_score_keeps_selection_and_is_a_distribution():
    rng = np.random.default_rng(5)
    logits = rng.normal(0.0, 3.0, (50, 40))
    bias = rng.uniform(-0.1, 0.1, 40).astype(np.float32)
    i_sig, g_sig, m_sig = oracle.select(logits, bias, 6)
    i_soft, g_soft, m_soft = oracle.select(logits, bias, 6, score="softmax")
    np.testing.assert_array_equal(i_sig, i_soft)          # the score only changes the weights
    np.testing.assert_array_equal(m_sig, m_soft)
    assert np.all(g_soft > 0) and np.allclose(g_soft.sum(axis=1), 1.0, atol=1e-14)
    # two-expert special case against the logistic function: softmax(a, b)[0] = sigmoid(a - b)
    l2 = rng.normal(0.0, 2.0, (20, 2))
    i2, g2, _ = oracle.select(l2, np.zeros(2, dtype=np.float32), 2, score="softmax")
    first = np.take_along_axis(l2, i2, axis=1)
    np.testing.assert_allclose(g2[:, 0], 1.0 / (1.0 + np.exp(first[:, 1] - first[:, 0])), rtol=1e-13)


def _bf16_bits(a):
    return torch.tensor(np.asarray(a, dtype=np.float64)).to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bf16_values(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double().numpy()


def test_rmsnorm_closed_forms():
    """RMSNorm ("Inside Kolibri 1", section "The released stack"): a row of one repeated value c
    normalises to sign(c) * gamma; the row (3, 4) has mean square 12.5."""
    gamma = _bf16_bits([1.0, 1.0, 1.0, 1.0])
    x = oracle.rmsnorm_bf16(_bf16_bits([[2.5, 2.5, 2.5, 2.5], [-0.75, -0.75, -0.75, -0.75]]), gamma, 0.0)
    np.testing.assert_array_equal(_bf16_values(x), [[1, 1, 1, 1], [-1, -1, -1, -1]])
    g2 = _bf16_bits([1.0, 2.0])
    x2 = _bf16_values(oracle.rmsnorm_bf16(_bf16_bits([[3.0, 4.0]]), g2, 0.0))
    ref = torch.tensor([3.0 / math.sqrt(12.5), 2 * 4.0 / math.sqrt(12.5)]).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(x2[0], ref)


def test_rmsnorm_matches_torch_and_is_scale_invariant():
    rng = np.random.default_rng(11)
    h = _bf16_bits(rng.normal(0.0, 3.0, (16, 256)))
    gamma = _bf16_bits(rng.uniform(0.5, 1.5, 256))
    eps = 1e-6
    x = _bf16_values(oracle.rmsnorm_bf16(h, gamma, eps))
    hv, gv = _bf16_values(h), _bf16_values(gamma)
    ref = hv / np.sqrt((hv ** 2).mean(axis=1, keepdims=True) + eps) * gv
    ref_b = torch.tensor(ref).to(torch.bfloat16).double().numpy()   # one rounding from double
    assert (x != ref_b).mean() < 1e-3                                  # ties of a double -> float -> bf16 path aside
    assert np.abs(x - ref).max() <= 2.0 ** -8 * np.abs(ref).max()
    # scaling the row by 4 (exact in BF16) leaves the normalised row unchanged (eps = 0)
    x1 = oracle.rmsnorm_bf16(h, gamma, 0.0)
    x4 = oracle.rmsnorm_bf16(_bf16_bits(4.0 * hv), gamma, 0.0)
    np.testing.assert_array_equal(x1, x4)


def test_post_norm_residual_closed_form():
    """h_out = h + m / rms(m) * g_post: a constant m row adds sign(m) * g_post to h."""
    h = _bf16_bits([[0.5, -1.0, 2.0], [1.0, 1.0, 1.0]])
    gp = _bf16_bits([1.0, 2.0, 0.5])
    m = np.array([[3.0, 3.0, 3.0], [-0.25, -0.25, -0.25]])
    rows = np.array([0, 1], dtype=np.int32)
    out = np.empty_like(m)
    oracle.lib().oracle_post_residual(2, 3, 2, oracle._p(rows), oracle._p(h), oracle._p(m), oracle._p(gp),
                                      ctypes.c_double(0.0), oracle._p(out))
    np.testing.assert_allclose(out, [[1.5, 1.0, 2.5], [0.0, -1.0, 0.5]], atol=1e-15)


def test_permute_matches_stable_sort():
    rng = np.random.default_rng(4)
    for N, K, E in [(128, 6, 64), (1, 6, 6), (57, 6, 384), (300, 2, 5)]:
        idx = np.stack([rng.permutation(E)[:K] for _ in range(N)]).astype(np.int32)
        counts, offsets, perm, inv = oracle.permute(idx, E)
        pairs = sorted(((idx[t, k], t, k) for t in range(N) for k in range(K)), key=lambda p: (p[0], p[1]))
        assert [p[1] for p in pairs] == list(perm)
        for pos, (e, t, k) in enumerate(pairs):
            assert inv[t, k] == pos
        assert counts.sum() == N * K and offsets[0] == 0 and offsets[-1] == N * K
        assert np.all(np.diff(offsets) == counts)
        assert sorted(inv.ravel()) == list(range(N * K))          # bijection
        assert np.all(perm[inv] == np.arange(N)[:, None])          # perm o inv_pos = id


def test_permute_rejects_out_of_range():
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, 7]], dtype=np.int32), 4)


def _one_by_one_layer():
    cfg = LayerConfig("hand", 1, 1, 2, 1, 1, "f32", "f32")
    inp = {
        "cfg": cfg,
        "x": torch.tensor([[2.0]]),
        "w_router": torch.tensor([[0.5], [-0.25]]),
        "bias": torch.tensor([0.0, 0.0]),
        # experts 0, 1 routed; index 2 is the shared expert
        "w_gate": torch.tensor([1.0, 2.0, 0.5]).reshape(3, 1, 1),
        "w_up": torch.tensor([3.0, 1.0, -1.0]).reshape(3, 1, 1),
        "w_down": torch.tensor([-1.5, 4.0, 2.0]).reshape(3, 1, 1),
    }
    return inp


def test_hand_computed_one_by_one_layer():
    # logits: 0.5*2 = 1 and -0.25*2 = -0.5, so expert 0 is chosen, g = sigmoid(1).
    # expert 0: SiLU(1*2) * (3*2) = 2*sigmoid(2)*6 = 10.569564935734588; down: * -1.5
    # shared:   SiLU(0.5*2) * (-1*2) = -1.4621171572600098;         down: * 2
    # y = -2.9242343145200196 + 0.7310585786300049 * -15.854347403601881
    out = oracle.layer(_one_by_one_layer())
    assert list(out["idx"][0]) == [0]
    assert out["g"][0, 0] == pytest.approx(0.7310585786300049, abs=1e-15)
    assert out["y"][0, 0] == pytest.approx(-14.51469099250352, abs=1e-13)


def test_expert_ffn_matches_numpy_swiglu_non_square():
    cfg = CONFIGS["tiny"]
    inp = make_inputs(cfg, seed=5)
    toks = np.array([0, 17, 127], dtype=np.int32)
    exps = np.array([3, cfg.E, 63], dtype=np.int32)
    got = oracle.expert_outputs(inp, toks, exps)
    x = inp["x"].double().numpy()
    for p, (t, e) in enumerate(zip(toks, exps)):
        wg = inp["w_gate"][e].double().numpy()     # [I, d]
        wu = inp["w_up"][e].double().numpy()       # [I, d]
        wd = inp["w_down"][e].double().numpy()     # [d, I]
        a, b = wg @ x[t], wu @ x[t]
        h = a / (1.0 + np.exp(-a)) * b
        np.testing.assert_allclose(got[p], wd @ h, rtol=1e-10, atol=1e-13)


def test_zero_input_gives_zero_output():
    inp = make_inputs(CONFIGS["tiny"], seed=6)
    inp["x"] = torch.zeros_like(inp["x"])
    out = oracle.layer(inp, rows=np.arange(8))
    assert np.all(out["y"] == 0.0)


def test_zero_routed_down_projection_leaves_shared_expert():
    cfg = CONFIGS["tiny"]
    inp = make_inputs(cfg, seed=7)
    inp["w_down"][: cfg.E].zero_()
    rows = np.arange(0, cfg.N, 9, dtype=np.int32)
    out = oracle.layer(inp, rows=rows)
    shared = oracle.expert_outputs(inp, rows, np.full(len(rows), cfg.E))
    np.testing.assert_array_equal(out["y"], shared)


def test_identical_experts_closed_form():
    # every expert (routed and shared) is the same F: y = (1 + sum_k g_k) F(x)
    cfg = CONFIGS["tiny"]
    inp = make_inputs(cfg, seed=8)
    for name in ("w_gate", "w_up", "w_down"):
        inp[name][:] = inp[name][cfg.E].clone()
    rows = np.arange(0, cfg.N, 5, dtype=np.int32)
    out = oracle.layer(inp, rows=rows)
    f = oracle.expert_outputs(inp, rows, np.full(len(rows), cfg.E))
    scale = 1.0 + out["g"].sum(axis=1)
    np.testing.assert_allclose(out["y"], scale[:, None] * f, rtol=1e-12, atol=1e-15)
    assert np.all(out["g"] > 0) and np.all(out["g"] < 1)


def test_bias_forcing_selects_the_same_six_everywhere():
    cfg = CONFIGS["tiny"]
    inp = make_inputs(cfg, seed=9)
    forced = [2, 11, 19, 30, 41, 60]
    inp["bias"][forced] = 30.0
    l = oracle.router_logits(inp["x"], "f32", inp["w_router"])
    idx, g, _ = oracle.select(l, inp["bias"], cfg.K)
    for t in range(cfg.N):
        assert sorted(idx[t]) == forced
        np.testing.assert_allclose(g[t], 1.0 / (1.0 + np.exp(-l[t, idx[t]])), rtol=1e-15)


@pytest.mark.parametrize("d,I", [(256, 128), (384, 256)])
def test_fp8_layer_equals_f32_layer_on_decoded_weights(d, I):
    """At (384, 256) every matrix has several scale blocks along both axes and is not square."""
    cfg = LayerConfig("q", 16, d, 8, 6, I, "f32", "e4m3")
    q = make_inputs(cfg, seed=10)
    f = dict(q)
    f["cfg"] = LayerConfig("f", 16, d, 8, 6, I, "f32", "f32")
    for w, s in (("w_gate", "s_gate"), ("w_up", "s_up"), ("w_down", "s_down")):
        vals = q[w].view(torch.float8_e4m3fn).to(torch.float64)          # [G, R, C]
        sc = q[s].double().repeat_interleave(128, 1).repeat_interleave(128, 2)
        f[w] = (vals * sc).to(torch.float32)
    a = oracle.layer(q)["y"]
    b = oracle.layer(f)["y"]
    np.testing.assert_allclose(a, b, rtol=1e-6, atol=1e-6 * np.abs(b).max())
    # and the scales really vary from block to block
    assert q["s_gate"].std() > 0


def _golden_counts():
    vals = {}
    with open(os.path.join(GOLDEN, "kolibri_shape_counts.txt")) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                name, value, _ = line.split()
                vals[name] = float(value)
    return vals


def test_layer_shape_matches_printed_weight_counts():
    g = _golden_counts()
    cfg = CONFIGS["decode"]
    assert cfg.expert_weights == g["weights_per_expert"]
    assert cfg.E == g["routed_experts"] and cfg.K == g["top_k"]
    assert cfg.E + 1 == g["experts_total_per_block"]
    assert round((cfg.K + 1) * cfg.expert_weights / 1e5) / 10 == g["touched_per_token_per_block"] / 1e6
    assert round((cfg.E + 1) * cfg.expert_weights / 1e7) / 100 == g["all_experts_per_block"] / 1e9


# ------------------------------------------------ FP8 activations (1 x 128)
# "Inside Kolibri 1", section "The FP8 path is explicitly mixed precision":
# activations are quantised dynamically in groups of 1 x 128.

def _e4m3_values(codes):
    return np.array([oracle.e4m3_to_double(int(c)) for c in np.ravel(codes)]).reshape(np.shape(codes))


def test_float_to_e4m3_matches_torch_rounding():
    """Round to nearest even on the E4M3 grid, the same codes as torch's float8_e4m3fn cast."""
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.uniform(-448, 448, 4000), rng.normal(0, 1, 4000), rng.normal(0, 2 ** -7, 2000),
                        rng.uniform(-2 ** -6, 2 ** -6, 2000)]).astype(np.float32)
    ours = oracle.float_to_e4m3(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_float_to_e4m3_round_trips_midpoints_and_saturates():
    finite = [c for c in range(256) if (c & 0x7F) != 0x7F]
    for c in finite:                                   # every finite code decodes and re-encodes to itself
        assert int(oracle.float_to_e4m3(np.float32(oracle.e4m3_to_double(c)))) == c
    for c in range(0, 0x7E):                           # halfway between neighbours: the even mantissa wins
        lo, hi = oracle.e4m3_to_double(c), oracle.e4m3_to_double(c + 1)
        want = c if c % 2 == 0 else c + 1
        assert int(oracle.float_to_e4m3(np.float32((lo + hi) / 2))) == want
    assert oracle.float_to_e4m3(np.float32([470.0, -1e6, 448.0])).tolist() == [0x7E, 0xFE, 0x7E]


def test_quant_1x128_exact_groups_and_error_bound():
    rng = np.random.default_rng(12)
    # groups built as E4M3 values times 2^k with one element at +-448: quantised exactly, scale 2^k
    codes = rng.integers(0, 0x7E, size=(3, 384)).astype(np.uint8) | (rng.integers(0, 2, size=(3, 384)) << 7).astype(np.uint8)
    codes[:, ::128] = 0x7E
    k = rng.integers(-8, 3, size=(3, 3))
    vals = _e4m3_values(codes) * np.repeat(2.0 ** k, 128, axis=1)
    q, s = oracle.quant_1x128(_bf16_bits(vals))
    assert np.array_equal(s, (2.0 ** k).astype(np.float32))
    assert np.array_equal(_e4m3_values(q), _e4m3_values(codes))
    # random BF16 rows: each group's largest magnitude maps to +-448, every value within half an E4M3 step
    x = _bf16_bits(rng.normal(0, 1.5, size=(4, 256)))
    xv = _bf16_values(x)
    q, s = oracle.quant_1x128(x)
    deq = _e4m3_values(q) * np.repeat(s.astype(np.float64), 128, axis=1)
    for r in range(4):
        for g in range(2):
            seg = slice(128 * g, 128 * g + 128)
            j = int(np.argmax(np.abs(xv[r, seg])))
            assert int(q[r, seg][j]) & 0x7F == 0x7E
    bound = np.maximum(np.abs(xv) * 2.0 ** -4, np.repeat(s.astype(np.float64), 128, axis=1) * 2.0 ** -10)
    assert np.all(np.abs(deq - xv) <= bound * (1 + 1e-6))
    zq, zs = oracle.quant_1x128(_bf16_bits(np.zeros((1, 128))))
    assert zs.tolist() == [[1.0]] and not zq.any()


def _a8_layer(d=256, I=128, E=8, K=2, N=6, seed=3):
    cfg = LayerConfig("a8", N, d, E, K, I, "bf16", "e4m3")
    return make_inputs(cfg, seed=seed)


def test_layer_a8_routes_like_the_bf16_layer_and_stays_close():
    inp = _a8_layer()
    a8 = oracle.layer_a8(inp)
    ref = oracle.layer(inp)
    assert np.array_equal(a8["idx"], ref["idx"]) and np.allclose(a8["g"], ref["g"])
    err = np.abs(a8["y"] - ref["y"]).max(axis=1) / np.abs(ref["y"]).max(axis=1)
    # E4M3 activations carry 3 mantissa bits: a few percent, but not zero (quantisation is applied)
    assert np.all(err < 0.15) and np.all(err > 1e-4)
    zero = dict(inp, x=torch.zeros_like(inp["x"]))
    assert not oracle.layer_a8(zero)["y"].any()


def test_layer_a8_hand_computed_case():
    """d = I = 128, one routed and the shared expert, identical: W_g and W_u read column 0 only,
    W_d is all ones. Then g_i = u_i = a for every i, H = bf16(SiLU(a) a) in one 128-group (scale
    H / 448, every code 448), and each expert outputs 128 * 448 * fl32(H / 448) on every column."""
    d = I = 128
    cfg = LayerConfig("hand", 1, d, 1, 1, I, "bf16", "e4m3")
    a = 448.0 * 2.0 ** -8                              # exact in E4M3 with scale 2^-8
    x = torch.zeros((1, d), dtype=torch.bfloat16)
    x[0, 0] = a
    one = 0x38                                         # E4M3 code of 1.0
    wg = torch.zeros((2, I, d), dtype=torch.uint8)
    wg[:, :, 0] = one
    wd = torch.full((2, d, I), one, dtype=torch.uint8)
    ones = torch.ones((2, 1, 1), dtype=torch.float32)
    inp = {"cfg": cfg, "x": x, "w_router": torch.full((1, d), 0.5, dtype=torch.float32),
           "bias": torch.zeros(1, dtype=torch.float32), "w_gate": wg, "w_up": wg.clone(), "w_down": wd,
           "s_gate": ones, "s_up": ones.clone(), "s_down": ones.clone()}
    out = oracle.layer_a8(inp)
    h = float(_bf16_values(_bf16_bits([a / (1.0 + math.exp(-a)) * a]))[0])
    s_h = float(np.float32(h) / np.float32(448.0))
    f = 128 * 448.0 * s_h
    logit = a * 0.5
    g = 1.0 / (1.0 + math.exp(-logit))
    assert out["idx"].tolist() == [[0]]
    assert np.allclose(out["y"], (1.0 + g) * f, rtol=1e-12, atol=0)


# ------------------------------------------------ FP8 block-scale indexing
# "Inside Kolibri 1", FP8 section: one FP32 scale per 128 x 128 block, stored
# [G, rows / 128, cols / 128]. With every E4M3 code equal to 1.0 (0x38) each
# weight equals the scale of its block, and with x non-zero in one 128-column
# block only, every projection reduces to a closed form in the scales. Each
# block of each matrix of each expert gets its own scale, and the shapes have
# several blocks along both axes (gate/up [256, 384]: 2 x 3, down [384, 256]:
# 3 x 2), so reading a scale with rows and columns swapped, or from the wrong
# expert, changes the result.

def _blocky_layer(x_dtype, d=384, I=256, E=2):
    G = E + 1
    one = 0x38
    cfg = LayerConfig("blocky", 1, d, E, 1, I, x_dtype, "e4m3")

    def scales(rows, cols, base):
        n = G * (rows // 128) * (cols // 128)
        return torch.arange(base + 1, base + 1 + n, dtype=torch.float32).reshape(G, rows // 128, cols // 128) / 64

    return {"cfg": cfg, "w_router": torch.zeros((E, d), dtype=torch.float32),
            "bias": torch.tensor([0.0] * (E - 1) + [30.0], dtype=torch.float32),   # forces the last routed expert
            "w_gate": torch.full((G, I, d), one, dtype=torch.uint8), "w_up": torch.full((G, I, d), one, dtype=torch.uint8),
            "w_down": torch.full((G, d, I), one, dtype=torch.uint8),
            "s_gate": scales(I, d, 0), "s_up": scales(I, d, 40), "s_down": scales(d, I, 80)}


def _x_in_block(inp, kb, v, torch_dtype):
    d = inp["cfg"].d
    x = torch.zeros((1, d), dtype=torch.float32)
    x[0, 128 * kb:128 * (kb + 1)] = v
    return x.to(torch_dtype)


def _bf16_rne(v: float) -> float:
    """v rounded to 8 significant bits, ties to even (the BF16 grid; v normal and non-zero)."""
    m, e = math.frexp(v)
    return math.ldexp(round(math.ldexp(m, 8)), e - 8)


@pytest.mark.parametrize("kb", [1, 2])
def test_fp8_block_scales_closed_form_bf16_activations(kb):
    """F_g(x) with x = v on columns of block kb only: a_i = 128 v s_g[g, i/128, kb] (same for the
    up projection), h_i = SiLU(a_i) b_i, y_j = sum_ib s_d[g, j/128, ib] * sum_{i in ib} h_i."""
    inp = _blocky_layer("bf16")
    cfg = inp["cfg"]
    v = 1.0 / 32
    inp["x"] = _x_in_block(inp, kb, v, torch.bfloat16)
    sg, su, sd = (inp[k].double().numpy() for k in ("s_gate", "s_up", "s_down"))
    G = cfg.E + 1
    got = oracle.expert_outputs(inp, np.zeros(G, dtype=np.int32), np.arange(G, dtype=np.int32))
    for g in range(G):
        a = 128 * v * np.repeat(sg[g, :, kb], 128)
        b = 128 * v * np.repeat(su[g, :, kb], 128)
        h = a / (1.0 + np.exp(-a)) * b
        hb = h.reshape(cfg.I // 128, 128).sum(axis=1)
        want = np.repeat(sd[g] @ hb, 128)
        np.testing.assert_allclose(got[g], want, rtol=1e-13, atol=0)


@pytest.mark.parametrize("kb", [1, 2])
def test_fp8_block_scales_closed_form_fp8_activations(kb):
    """The same weights with FP8 activations: x's block kb quantises to scale fl32(v / 448) and
    codes 448, so a_i = fl32(v / 448) * s_g[g, i/128, kb] * 128 * 448; every 128-group of H is
    constant (one gate row block), so it quantises to scale fl32(bf16(h) / 448) and codes 448, and
    y_j = sum_ib s_h[ib] * s_d[g, j/128, ib] * 128 * 448. Routing is forced onto the last routed
    expert (bias +30, zero router weights: g = sigmoid(0) = 1/2), so y = F_shared + F_last / 2."""
    inp = _blocky_layer("bf16")
    cfg = inp["cfg"]
    v = 1.0 / 32
    inp["x"] = _x_in_block(inp, kb, v, torch.bfloat16)
    sg, su, sd = (inp[k].double().numpy() for k in ("s_gate", "s_up", "s_down"))
    s_x = float(np.float32(v) / np.float32(448.0))

    def expert(g):
        a = s_x * sg[g, :, kb] * 128 * 448         # one value per gate row block
        b = s_x * su[g, :, kb] * 128 * 448
        h = [_bf16_rne(float(ai / (1.0 + math.exp(-ai)) * bi)) for ai, bi in zip(a, b)]
        s_h = np.array([float(np.float32(hi) / np.float32(448.0)) for hi in h])
        return np.repeat(sd[g] @ (s_h * 128 * 448), 128)

    out = oracle.layer_a8(inp)
    last = cfg.E - 1
    assert out["idx"].tolist() == [[last]]
    np.testing.assert_allclose(out["y"][0], expert(cfg.E) + 0.5 * expert(last), rtol=1e-13, atol=0)
    G = cfg.E + 1
    per = oracle.expert_outputs_a8(inp, np.zeros(G, dtype=np.int32), np.arange(G, dtype=np.int32))
    for g in range(G):
        np.testing.assert_allclose(per[g], expert(g), rtol=1e-13, atol=0)
