"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Every test here needs a B200. Inputs are drawn on the device by the seeded
generator and copied to the host for the oracle; no oracle input or expected
value comes from the CUDA path.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from fine_grained_sparse_fp32_b200 import _build, kmoe
from fine_grained_sparse_fp32_b200.inputs import CONFIGS, LayerConfig, make_block_inputs, make_inputs, to_host
from parity import G_TOL, TOL, biased_scores, check_routing, frob_rel_err, row_rel_err

pytestmark = pytest.mark.gpu

NT = None  # oracle threads: all host cores


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _build.build()
    kmoe.load()


_CACHE = {}


def layer_inputs(name, N=None, seed=0):
    cfg = CONFIGS[name] if N is None else CONFIGS[name].with_tokens(N)
    key = (cfg, seed)
    if key not in _CACHE:
        if len(_CACHE) >= 2:
            _CACHE.clear()
            torch.cuda.empty_cache()
        dev = make_inputs(cfg, seed, device="cuda")
        _CACHE[key] = (dev, to_host(dev))
    return _CACHE[key]


def threads():
    return oracle.max_threads()


def expert_ref(host, tokens, experts):
    """The oracle's expert outputs under the config's activation precision."""
    f = oracle.expert_outputs_a8 if host["cfg"].w_dtype == "e4m3_a8" else oracle.expert_outputs
    return f(host, tokens, experts, nthreads=threads())


def layer_ref(host, rows=None, score="sigmoid"):
    f = oracle.layer_a8 if host["cfg"].w_dtype == "e4m3_a8" else oracle.layer
    return f(host, rows=rows, nthreads=threads(), score=score)


# ----------------------------------------------------------------- router
@pytest.mark.parametrize("name,N", [("tiny", None), ("decode", None), ("decode", 300), ("decode", 1),
                                    ("skew", 2048), ("decode", 513), ("prefill", None), ("skew", None)])
def test_router_topk_matches_oracle(name, N):
    dev, host = layer_inputs(name, N)
    cfg = host["cfg"]
    logits = torch.empty((cfg.N, cfg.E), dtype=torch.float32, device="cuda")
    idx, w = kmoe.moe_router_topk(dev["x"], dev["w_router"], dev["bias"], cfg.K, logits=logits)
    torch.cuda.synchronize()
    l_ora = oracle.router_logits(host["x"], cfg.x_dtype, host["w_router"], nthreads=threads())
    i_ora, g_ora, _ = oracle.select(l_ora, host["bias"], cfg.K)
    l_gpu = logits.cpu().double().numpy()
    assert np.abs(l_gpu - l_ora).max() <= 2e-5
    s = biased_scores(l_ora, host["bias"])
    idx_g = idx.cpu().numpy()
    _, differ = check_routing(idx_g, i_ora, s, cfg.K)
    w_g = w.cpu().double().numpy()
    for t in range(cfg.N):
        if t in differ:
            continue
        ora = dict(zip(i_ora[t].tolist(), g_ora[t].tolist()))
        for k in range(cfg.K):
            assert abs(w_g[t, k] - ora[int(idx_g[t, k])]) <= G_TOL


@pytest.mark.parametrize("name,N", [("decode", None), ("prefill", 1024), ("tiny", None)])
def test_router_topk_softmax_score_matches_oracle(name, N):
    """KMOE_SCORE_SOFTMAX: same selection, weights = softmax over the K chosen unbiased logits."""
    dev, host = layer_inputs(name, N)
    cfg = host["cfg"]
    idx, w = kmoe.moe_router_topk(dev["x"], dev["w_router"], dev["bias"], cfg.K, score="softmax")
    torch.cuda.synchronize()
    l_ora = oracle.router_logits(host["x"], cfg.x_dtype, host["w_router"], nthreads=threads())
    i_ora, g_ora, _ = oracle.select(l_ora, host["bias"], cfg.K, score="softmax")
    idx_g, w_g = idx.cpu().numpy(), w.cpu().double().numpy()
    _, differ = check_routing(idx_g, i_ora, biased_scores(l_ora, host["bias"]), cfg.K)
    assert np.allclose(w_g.sum(axis=1), 1.0, atol=1e-5)
    for t in range(cfg.N):
        if t in differ:
            continue
        ora = dict(zip(i_ora[t].tolist(), g_ora[t].tolist()))
        for k in range(cfg.K):
            assert abs(w_g[t, k] - ora[int(idx_g[t, k])]) <= G_TOL


# ---------------------------------------------------------------- permute
def _distinct_rows(rng, N, K, E, skew=False):
    if skew:
        p = 1.0 / np.arange(1, E + 1) ** 1.1
        p /= p.sum()
        return np.stack([rng.choice(E, size=K, replace=False, p=p) for _ in range(N)]).astype(np.int32)
    return np.argsort(rng.random((N, E)), axis=1)[:, :K].astype(np.int32)


@pytest.mark.parametrize("N,E,skew", [(1, 384, False), (31, 64, False), (32, 384, False), (256, 384, False),
                                      (257, 384, False), (1000, 64, True), (8192, 384, False),
                                      (65536, 384, True), (300, 6, False)])
def test_permute_is_bit_exact(N, E, skew):
    rng = np.random.default_rng(N + E)
    K = 6
    idx = _distinct_rows(rng, N, K, E, skew)
    counts, offsets, perm, inv = kmoe.moe_permute(torch.from_numpy(idx).cuda(), E)
    c_o, o_o, p_o, i_o = oracle.permute(idx, E)
    np.testing.assert_array_equal(counts.cpu().numpy(), c_o)
    np.testing.assert_array_equal(offsets.cpu().numpy(), o_o)
    np.testing.assert_array_equal(perm.cpu().numpy(), p_o)
    np.testing.assert_array_equal(inv.cpu().numpy(), i_o)


def test_permute_zero_tokens():
    counts, offsets, _, _ = kmoe.moe_permute(torch.empty((0, 6), dtype=torch.int32, device="cuda"), 384)
    assert counts.abs().sum().item() == 0 and offsets.abs().sum().item() == 0


def test_permute_all_tokens_on_the_same_experts():
    N, E, K = 4000, 384, 6
    idx = np.tile(np.array([383, 0, 17, 200, 5, 6], dtype=np.int32), (N, 1))
    counts, offsets, perm, inv = kmoe.moe_permute(torch.from_numpy(idx).cuda(), E)
    c_o, o_o, p_o, i_o = oracle.permute(idx, E)
    np.testing.assert_array_equal(perm.cpu().numpy(), p_o)
    np.testing.assert_array_equal(inv.cpu().numpy(), i_o)
    np.testing.assert_array_equal(counts.cpu().numpy(), c_o)


# ------------------------------------------------------------ grouped FFN
@pytest.mark.parametrize("name,N", [("tiny", None), ("decode", None), ("fp8_decode", None), ("decode", 200),
                                    ("fp8_decode", 130), ("fp8_decode", 1), ("fp8_decode", 255), ("prefill", 256), ("prefill", 300), ("prefill", 1000),
                                    ("fp8_prefill", 300), ("fp8_prefill", 777), ("fp8a8_decode", None),
                                    ("fp8a8_decode", 1), ("fp8a8_decode", 255), ("fp8a8_prefill", 256),
                                    ("fp8a8_prefill", 1000), ("fp8a8_prefill", 2500)])
def test_grouped_ffn_matches_oracle(name, N):
    dev, host = layer_inputs(name, N)
    cfg = host["cfg"]
    l_ora = oracle.router_logits(host["x"], cfg.x_dtype, host["w_router"], nthreads=threads())
    i_ora, _, _ = oracle.select(l_ora, host["bias"], cfg.K)
    counts, offsets, perm, inv = oracle.permute(i_ora, cfg.E)
    y_perm, y_shared = kmoe.moe_grouped_ffn(dev["x"], dev, torch.from_numpy(perm).cuda(),
                                            torch.from_numpy(offsets).cuda())
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, cfg.N * cfg.K - 1], rng.integers(0, cfg.N * cfg.K, 48)]))
    expert_of_row = np.searchsorted(offsets, rows, side="right") - 1
    ref = expert_ref(host, perm[rows], expert_of_row)
    got = y_perm[torch.from_numpy(rows).cuda().long()].float().cpu().numpy()
    assert row_rel_err(got, ref) <= TOL[cfg.w_dtype]
    toks = np.unique(np.concatenate([[0, cfg.N - 1], rng.integers(0, cfg.N, 16)]))
    ref_s = expert_ref(host, toks, np.full(len(toks), cfg.E))
    got_s = y_shared[torch.from_numpy(toks).cuda().long()].float().cpu().numpy()
    assert row_rel_err(got_s, ref_s) <= TOL[cfg.w_dtype]


@pytest.mark.parametrize("N", [32, 130])
def test_two_term_activations_keep_bf16_precision(N):
    """The two-term E4M3 form of x and H (error about 2^-8 of each value) keeps the E4M3-weight FFN
    within the BF16 tolerance of the oracle's exact-BF16-activation expert outputs, and closer to
    them than single-term FP8 activations on the same weights and tokens."""
    dev, host = layer_inputs("fp8_decode", N)
    cfg = host["cfg"]
    l_ora = oracle.router_logits(host["x"], cfg.x_dtype, host["w_router"], nthreads=threads())
    i_ora, _, _ = oracle.select(l_ora, host["bias"], cfg.K)
    _, offsets, perm, _ = oracle.permute(i_ora, cfg.E)
    y_perm, _ = kmoe.moe_grouped_ffn(dev["x"], dev, torch.from_numpy(perm).cuda(), torch.from_numpy(offsets).cuda())
    torch.cuda.synchronize()
    rows = np.arange(0, cfg.N * cfg.K, 3)
    ref = expert_ref(host, perm[rows], np.searchsorted(offsets, rows, side="right") - 1)
    err_two = row_rel_err(y_perm[torch.from_numpy(rows).cuda().long()].float().cpu().numpy(), ref)
    assert err_two <= TOL["bf16"]
    a8 = dict(dev, cfg=dataclasses.replace(cfg, w_dtype="e4m3_a8"))
    y8, _ = kmoe.moe_grouped_ffn(dev["x"], a8, torch.from_numpy(perm).cuda(), torch.from_numpy(offsets).cuda())
    torch.cuda.synchronize()
    err_a8 = row_rel_err(y8[torch.from_numpy(rows).cuda().long()].float().cpu().numpy(), ref)
    assert err_two < err_a8


@pytest.mark.parametrize("E,N,chunk", [(64, 200, 32), (16, 255, 64), (64, 40, 16)])
def test_two_term_fp8_ffn_chunk_sizes(E, N, chunk):
    """E4M3 weights with BF16 activations below 256 tokens take the FP8 tensor cores with two-term
    activations; with few experts the expected rows per expert N*K/E pick 16-, 32- or 64-row chunks
    (B operands of 32, 64 or 128 rows). Reduced layer (d = 512, I = 128) drawn on the host."""
    cfg = LayerConfig(f"two_term_{E}_{N}", N, 512, E, 6, 128, "bf16", "e4m3")
    avg = N * cfg.K // E
    assert chunk == (16 if avg <= 12 else 32 if avg <= 32 else 64)
    host = make_inputs(cfg, seed=5, device="cpu")
    dev = {k: (v.to("cuda") if torch.is_tensor(v) else v) for k, v in host.items()}
    l_ora = oracle.router_logits(host["x"], cfg.x_dtype, host["w_router"], nthreads=threads())
    i_ora, _, _ = oracle.select(l_ora, host["bias"], cfg.K)
    _, offsets, perm, _ = oracle.permute(i_ora, cfg.E)
    y_perm, y_shared = kmoe.moe_grouped_ffn(dev["x"], dev, torch.from_numpy(perm).cuda(),
                                            torch.from_numpy(offsets).cuda())
    torch.cuda.synchronize()
    rows = np.arange(cfg.N * cfg.K)
    ref = expert_ref(host, perm, np.searchsorted(offsets, rows, side="right") - 1)
    assert row_rel_err(y_perm.float().cpu().numpy(), ref) <= TOL["e4m3"]
    ref_s = expert_ref(host, np.arange(cfg.N), np.full(cfg.N, cfg.E))
    assert row_rel_err(y_shared.float().cpu().numpy(), ref_s) <= TOL["e4m3"]


@pytest.mark.parametrize("name,N", [("decode", 200), ("fp8_decode", 200), ("decode", 33), ("fp8a8_decode", 200),
                                    ("fp8a8_prefill", 600)])
def test_grouped_ffn_crowded_experts(name, N):
    """Every token on the same six experts: groups of N rows, several 32-row
    token chunks per expert on the small-batch path, and 378 empty groups."""
    dev, host = layer_inputs(name, N)
    cfg = host["cfg"]
    idx = np.tile(np.array([383, 0, 17, 200, 5, 6], dtype=np.int32), (cfg.N, 1))
    counts, offsets, perm, inv = oracle.permute(idx, cfg.E)
    y_perm, y_shared = kmoe.moe_grouped_ffn(dev["x"], dev, torch.from_numpy(perm).cuda(),
                                            torch.from_numpy(offsets).cuda())
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, cfg.N * cfg.K - 1], np.arange(0, cfg.N * cfg.K, 7)]))
    expert_of_row = np.searchsorted(offsets, rows, side="right") - 1
    ref = expert_ref(host, perm[rows], expert_of_row)
    got = y_perm[torch.from_numpy(rows).cuda().long()].float().cpu().numpy()
    assert row_rel_err(got, ref) <= TOL[cfg.w_dtype]
    toks = np.arange(cfg.N)
    ref_s = expert_ref(host, toks, np.full(len(toks), cfg.E))
    assert row_rel_err(y_shared.float().cpu().numpy(), ref_s) <= TOL[cfg.w_dtype]


@pytest.mark.parametrize("name", ["decode", "fp8_decode", "prefill", "fp8a8_decode", "fp8a8_prefill"])
def test_grouped_ffn_without_shared_expert(name):
    dev, host = layer_inputs(name, 40 if name != "prefill" else 300)
    cfg = host["cfg"]
    l_ora = oracle.router_logits(host["x"], cfg.x_dtype, host["w_router"], nthreads=threads())
    i_ora, _, _ = oracle.select(l_ora, host["bias"], cfg.K)
    counts, offsets, perm, inv = oracle.permute(i_ora, cfg.E)
    y_perm, y_shared = kmoe.moe_grouped_ffn(dev["x"], dev, torch.from_numpy(perm).cuda(),
                                            torch.from_numpy(offsets).cuda(), with_shared=False)
    torch.cuda.synchronize()
    assert y_shared is None
    rows = np.arange(0, cfg.N * cfg.K, 5)
    expert_of_row = np.searchsorted(offsets, rows, side="right") - 1
    ref = expert_ref(host, perm[rows], expert_of_row)
    got = y_perm[torch.from_numpy(rows).cuda().long()].float().cpu().numpy()
    assert row_rel_err(got, ref) <= TOL[cfg.w_dtype]


def test_fp8_small_batch_takes_activations_across_the_bf16_range():
    """The E4M3 small-batch path holds each 128-wide activation group as two scaled E4M3 terms:
    a group with one value of 1e6 (beyond the F16 range) among values near 1 stays within the
    tolerance of the float64 expert outputs."""
    dev, host = layer_inputs("fp8_decode", 8)
    cfg = host["cfg"]
    x = dev["x"].clone()
    x[3, 100] = 1.0e6
    hx = dict(host)
    hx["x"] = x.cpu()
    idx = np.tile(np.arange(cfg.K, dtype=np.int32), (cfg.N, 1))
    _, offsets, perm, _ = oracle.permute(idx, cfg.E)
    y_perm, _ = kmoe.moe_grouped_ffn(x, dev, torch.from_numpy(perm).cuda(), torch.from_numpy(offsets).cuda())
    torch.cuda.synchronize()
    rows = np.arange(cfg.N * cfg.K)
    expert_of_row = np.searchsorted(offsets, rows, side="right") - 1
    ref = expert_ref(hx, perm[rows], expert_of_row)
    got = y_perm.float().cpu().numpy()
    assert np.isfinite(got).all()
    assert row_rel_err(got, ref) <= TOL[cfg.w_dtype]


@pytest.mark.parametrize("N,d,with_shared,y_dtype", [(1, 2560, True, torch.bfloat16), (32, 2560, True, torch.bfloat16),
                                                       (777, 2560, False, torch.bfloat16), (300, 512, True, torch.float32),
                                                       (8192, 2560, True, torch.bfloat16)])
def test_combine_matches_float64(N, d, with_shared, y_dtype):
    """y[t] = y_shared[t] + sum_k g[t,k] y_perm[inv_pos[t,k]] against a float64 sum of the same BF16 inputs."""
    K = 6
    gen = torch.Generator(device="cuda").manual_seed(N + d)
    y_perm = torch.randn((N * K, d), generator=gen, device="cuda").bfloat16()
    y_sh = torch.randn((N, d), generator=gen, device="cuda").bfloat16() if with_shared else None
    w = torch.rand((N, K), generator=gen, device="cuda")
    inv = torch.randperm(N * K, generator=gen, device="cuda").int().reshape(N, K)
    y = kmoe.moe_combine(y_perm, y_sh, w, inv, y_dtype=y_dtype)
    torch.cuda.synchronize()
    yp, wv, iv = y_perm.double().cpu().numpy(), w.double().cpu().numpy(), inv.long().cpu().numpy()
    ref = np.einsum("tk,tkj->tj", wv, yp[iv])
    if with_shared:
        ref = ref + y_sh.double().cpu().numpy()
    got = y.double().cpu().numpy()
    tol = 1e-5 if y_dtype == torch.float32 else 2 ** -8
    assert np.abs(got - ref).max() <= tol * max(1.0, np.abs(ref).max())


# ----------------------------------------------------------- whole layer
def _forward_and_compare(name, N=None, rows=None, check_all_routing=True):
    dev, host = layer_inputs(name, N)
    cfg = host["cfg"]
    y_dtype = torch.float32 if cfg.x_dtype == "f32" else torch.bfloat16
    y, idx, w, counts = kmoe.moe_forward(dev["x"], dev, y_dtype=y_dtype, with_outputs=True)
    torch.cuda.synchronize()
    idx_g = idx.cpu().numpy()
    if rows is None:
        rows = np.arange(cfg.N, dtype=np.int32)
    ora = layer_ref(host, rows=rows)
    # routing on the compared rows (oracle logits recomputed for them)
    xr = host["x"][torch.from_numpy(rows).long()]
    l_rows = oracle.router_logits(xr, cfg.x_dtype, host["w_router"], nthreads=threads())
    s = biased_scores(l_rows, host["bias"])
    _, differ = check_routing(idx_g[rows], ora["idx"], s, cfg.K)
    keep = np.array([r not in differ for r in range(len(rows))])
    got = y[torch.from_numpy(rows).cuda().long()].float().cpu().numpy()
    err = row_rel_err(got[keep], ora["y"][keep])
    assert err <= TOL[cfg.w_dtype], (name, err, frob_rel_err(got[keep], ora["y"][keep]))
    if check_all_routing:
        l_all = oracle.router_logits(host["x"], cfg.x_dtype, host["w_router"], nthreads=threads())
        i_all, _, _ = oracle.select(l_all, host["bias"], cfg.K)
        _, differ_all = check_routing(idx_g, i_all, biased_scores(l_all, host["bias"]), cfg.K)
        # counts equal the oracle's counting sort of the GPU's own (validated) indices
        c_o, _, _, _ = oracle.permute(idx_g, cfg.E)
        np.testing.assert_array_equal(counts.cpu().numpy(), c_o)
    assert int(counts.sum().item()) == cfg.N * cfg.K
    return err


@pytest.mark.parametrize("name,N", [("tiny", None), ("decode", None), ("fp8_decode", None),
                                    ("prefill", 300), ("fp8_prefill", 259), ("decode", 1), ("fp8a8_decode", None),
                                    ("fp8a8_decode", 1), ("fp8a8_prefill", 259)])
def test_forward_matches_oracle_all_tokens(name, N):
    _forward_and_compare(name, N)


@pytest.mark.parametrize("name", ["prefill", "fp8_prefill", "fp8a8_prefill"])
def test_forward_full_size_sampled_tokens(name):
    cfg = CONFIGS[name]
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([[0, cfg.N - 1], rng.integers(0, cfg.N, 30)])).astype(np.int32)
    _forward_and_compare(name, rows=rows, check_all_routing=True)


def test_forward_skew_full_size():
    """The skewed layer (N = 65536) at full size: routing of every token against the oracle's
    router and selection, counts against the oracle's counting sort of the GPU's own (validated)
    indices, the workload's skew itself, and the outputs and mixture weights of 160 tokens that
    include tokens routed to the busiest expert and to the least busy non-empty one."""
    dev, host = layer_inputs("skew")
    cfg = host["cfg"]
    y, idx, w, counts = kmoe.moe_forward(dev["x"], dev, with_outputs=True)
    torch.cuda.synchronize()
    idx_g, w_g = idx.cpu().numpy(), w.cpu().double().numpy()
    l_all = oracle.router_logits(host["x"], cfg.x_dtype, host["w_router"], nthreads=threads())
    i_all, g_all, _ = oracle.select(l_all, host["bias"], cfg.K)
    _, differ = check_routing(idx_g, i_all, biased_scores(l_all, host["bias"]), cfg.K)
    c_gpu = counts.cpu().numpy()
    np.testing.assert_array_equal(c_gpu, oracle.permute(idx_g, cfg.E)[0])
    c_ora = np.bincount(i_all.ravel(), minlength=cfg.E)
    top = np.sort(c_ora)[::-1]
    assert 0.45 <= top[:38].sum() / (cfg.N * cfg.K) <= 0.55            # ~half the slots on 10 % of experts
    assert (c_ora == 0).sum() >= 20                                      # the empty groups exist
    heavy = int(np.argmax(c_ora))
    light = int(np.where(c_ora > 0, c_ora, np.iinfo(np.int64).max).argmin())
    rng = np.random.default_rng(2)
    on = lambda e: np.nonzero((i_all == e).any(axis=1))[0]
    rows = np.unique(np.concatenate([[0, cfg.N - 1], rng.choice(on(heavy), 64, replace=False), on(light)[:32],
                                     rng.integers(0, cfg.N, 64)])).astype(np.int32)
    assert len(rows) >= 128
    ora = oracle.layer(host, rows=rows, nthreads=threads())
    keep = np.array([r not in set(differ) for r in rows])
    got = y[torch.from_numpy(rows).cuda().long()].float().cpu().numpy()
    assert row_rel_err(got[keep], ora["y"][keep]) <= TOL[cfg.w_dtype]
    for j, t in enumerate(rows):
        if keep[j]:
            want = dict(zip(ora["idx"][j].tolist(), ora["g"][j].tolist()))
            for k in range(cfg.K):
                assert abs(w_g[t, k] - want[int(idx_g[t, k])]) <= G_TOL


@pytest.mark.parametrize("name,N", [("decode", None), ("prefill", 300), ("fp8_decode", 64), ("fp8a8_decode", 64)])
def test_forward_softmax_score_matches_oracle(name, N):
    dev, host = layer_inputs(name, N)
    cfg = host["cfg"]
    y, idx, w, counts = kmoe.moe_forward(dev["x"], dev, with_outputs=True, score="softmax")
    torch.cuda.synchronize()
    ora = layer_ref(host, score="softmax")
    l_all = oracle.router_logits(host["x"], cfg.x_dtype, host["w_router"], nthreads=threads())
    _, differ = check_routing(idx.cpu().numpy(), ora["idx"], biased_scores(l_all, host["bias"]), cfg.K)
    keep = np.array([t not in differ for t in range(cfg.N)])
    got = y.float().cpu().numpy()
    assert row_rel_err(got[keep], ora["y"][keep]) <= TOL[cfg.w_dtype]


def test_forward_is_deterministic():
    for name, N in (("decode", None), ("prefill", 300), ("fp8a8_decode", None), ("fp8a8_prefill", 300)):
        dev, _ = layer_inputs(name, N)
        a = kmoe.moe_forward(dev["x"], dev, with_outputs=True)
        b = kmoe.moe_forward(dev["x"], dev, with_outputs=True)
        for u, v in zip(a, b):
            assert torch.equal(u, v)


def test_device_status_is_clear_after_a_forward():
    for name, N in (("decode", None), ("prefill", 300), ("fp8a8_decode", None), ("fp8a8_prefill", 300)):
        dev, _ = layer_inputs(name, N)
        cfg = dev["cfg"]
        lay = kmoe.Layer(dev, cfg.N)
        lay.forward(dev["x"])
        assert kmoe.moe_device_status(lay.ws) == 0


def test_forward_zero_tokens():
    dev, _ = layer_inputs("decode")
    y = kmoe.moe_forward(dev["x"][:0], dev)
    assert y.shape == (0, 2560)


# ------------------------------------------------------- sandwich block
BLOCK_EPS = 1e-6
# The two sides route their own normalised inputs, which may differ by one
# BF16 ulp in a few elements (~1e-4 change of a logit at these weight scales).
BLOCK_TIE = 1e-3


def _bf16_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().astype(np.int32) & 0xFFFF


def _check_block(name, N, rows=None, score="sigmoid"):
    dev, host = layer_inputs(name, N)
    cfg = host["cfg"]
    blk = make_block_inputs(cfg, seed=11, device="cuda")
    hb = {k: v.cpu() for k, v in blk.items()}
    out, x, idx, w, counts = kmoe.moe_block_forward(blk["h"], dev, blk["gamma_pre"], blk["gamma_post"], BLOCK_EPS,
                                                    with_outputs=True, score=score)
    torch.cuda.synchronize()
    ora = oracle.block(host, hb["h"], hb["gamma_pre"], hb["gamma_post"], BLOCK_EPS, rows=rows, nthreads=threads(),
                       score=score)
    # pre-norm: BF16 bits equal except rare one-ulp flips of values on a rounding boundary
    xg, xo = _bf16_bits(x), ora["x"].astype(np.int32)
    diff = xg != xo
    assert diff.mean() <= 1e-3
    assert np.all(np.abs(xg[diff] - xo[diff]) == 1)
    rws = ora["rows"]
    l_all = oracle.router_logits(ora["x"][rws], "bf16", host["w_router"], nthreads=threads())
    _, differ = check_routing(idx.cpu().numpy()[rws], ora["idx"], biased_scores(l_all, host["bias"]), cfg.K,
                              margin=BLOCK_TIE)
    assert counts.sum().item() == cfg.N * cfg.K
    keep = np.array([t not in differ for t in range(len(rws))])
    got = out.float().cpu().numpy()[rws][keep]
    ref = ora["h_out"][keep]
    h = hb["h"].float().numpy()[rws][keep]
    # error against the size of the normalised MoE term, plus BF16 rounding of h_out
    n_max = np.abs(ref - h).max(axis=1)
    allow = TOL[cfg.w_dtype] * n_max + 2.0 ** -8 * np.abs(ref).max(axis=1)
    assert np.all(np.abs(got - ref).max(axis=1) <= allow)
    return out


@pytest.mark.parametrize("name,N", [("decode", None), ("decode", 1), ("decode", 300), ("fp8_decode", None),
                                    ("fp8_decode", 200), ("prefill", 1024), ("fp8a8_decode", None),
                                    ("fp8a8_prefill", 600)])
def test_block_forward_matches_oracle(name, N):
    _check_block(name, N)


def test_block_forward_full_prefill_sampled_rows():
    rows = np.random.default_rng(5).choice(8192, 192, replace=False).astype(np.int32)
    rows[:2] = [0, 8191]
    _check_block("prefill", None, rows=np.sort(rows))


def test_block_forward_softmax_score():
    _check_block("decode", 300, score="softmax")


def test_block_forward_in_place_equals_out_of_place():
    dev, _ = layer_inputs("decode", 300)
    cfg = dev["cfg"]
    blk = make_block_inputs(cfg, seed=3, device="cuda")
    lay = kmoe.Layer(dev, cfg.N, block=True)
    ref = lay.block_forward(blk["h"], blk["gamma_pre"], blk["gamma_post"], BLOCK_EPS)
    again = lay.block_forward(blk["h"], blk["gamma_pre"], blk["gamma_post"], BLOCK_EPS)
    h = blk["h"].clone()
    lay.block_forward(h, blk["gamma_pre"], blk["gamma_post"], BLOCK_EPS, h_out=h)
    torch.cuda.synchronize()
    assert torch.equal(ref, again)
    assert torch.equal(h, ref)
    assert kmoe.moe_device_status(lay.ws) == 0


def test_block_forward_zero_tokens():
    dev, _ = layer_inputs("decode")
    blk = make_block_inputs(dev["cfg"], seed=3, device="cuda")
    out = kmoe.moe_block_forward(blk["h"][:0], dev, blk["gamma_pre"], blk["gamma_post"], BLOCK_EPS)
    assert out.shape == (0, 2560)


# ------------------------------------------- FP8 activations: quantiser
@pytest.mark.parametrize("rows,cols,std", [(1, 128, 1.0), (33, 2560, 2.0), (300, 512, 1e-3), (7, 6144, 30.0)])
def test_quant_1x128_is_bit_exact(rows, cols, std):
    gen = torch.Generator(device="cuda")
    gen.manual_seed(rows * 7 + cols)
    x = torch.empty((rows, cols), device="cuda").normal_(0.0, std, generator=gen)
    x[0, :128] = 0.0                                   # an all-zero group
    if cols >= 256:                                    # one large value over tiny ones: subnormal codes
        x[0, 128:256] *= 1e-4
        x[0, 128] = 10.0 * std
    x = x.to(torch.bfloat16)
    codes, scales = kmoe.moe_quant_1x128(x)
    torch.cuda.synchronize()
    oc, os_ = oracle.quant_1x128(x.cpu())
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), os_.view(np.uint32))


# ------------------------------------------------------ failure path
@pytest.mark.parametrize("name,N", [("decode", None), ("fp8_decode", None), ("fp8a8_decode", None),
                                    ("prefill", 300), ("fp8_prefill", 300), ("fp8a8_prefill", 300)])
def test_a_wait_that_runs_out_reports_status_1_and_the_next_call_is_clean(name, N):
    """With a give-up limit of 100 SM cycles (below any load's latency) the FFN kernels' pipeline
    waits run out: the call leaves status 1 and returns; the GPU stays usable, and the next call
    with the default limit on the same workspace reports 0 and matches the oracle."""
    dev, host = layer_inputs(name, N)
    cfg = host["cfg"]
    l_ora = oracle.router_logits(host["x"], cfg.x_dtype, host["w_router"], nthreads=threads())
    i_ora, _, _ = oracle.select(l_ora, host["bias"], cfg.K)
    _, offsets, perm, _ = oracle.permute(i_ora, cfg.E)
    perm_d, off_d = torch.from_numpy(perm).cuda(), torch.from_numpy(offsets).cuda()
    ws = kmoe.workspace(cfg.N, cfg.d, cfg.E, cfg.K, cfg.I, kmoe.KMOE_BF16, kmoe.w_dtype_code(cfg.w_dtype))
    try:
        kmoe.moe_set_wait_limit(100)
        kmoe.moe_grouped_ffn(dev["x"], dev, perm_d, off_d, ws=ws)
        assert kmoe.moe_device_status(ws) == 1
    finally:
        kmoe.moe_set_wait_limit(0)
    y_perm, y_shared = kmoe.moe_grouped_ffn(dev["x"], dev, perm_d, off_d, ws=ws)
    assert kmoe.moe_device_status(ws) == 0
    rows = np.arange(0, cfg.N * cfg.K, 7)
    expert_of_row = np.searchsorted(offsets, rows, side="right") - 1
    got = y_perm[torch.from_numpy(rows).cuda().long()].float().cpu().numpy()
    assert row_rel_err(got, expert_ref(host, perm[rows], expert_of_row)) <= TOL[cfg.w_dtype]
    toks = np.arange(0, cfg.N, 5)
    got_s = y_shared[torch.from_numpy(toks).cuda().long()].float().cpu().numpy()
    assert row_rel_err(got_s, expert_ref(host, toks, np.full(len(toks), cfg.E))) <= TOL[cfg.w_dtype]
