"""The KMOE_DEBUG build (libkmoe_debug.so): the same kernels with index checks.

Its kernels check every dispatch index they read (token indices in
perm_token against N, expert offsets for a monotone partition of the N*K
rows) and, on a bad one, record status 3 in the workspace status word and use
a safe index (or skip the work) instead of reading outside a buffer. These
tests run it in a child process (KMOE_LIBRARY selects the library) on small
parity cases, where the status must stay 0 and the outputs match the oracle,
and on dispatch indices made invalid on purpose, which it must report.
"""
import os
import subprocess
import sys
import textwrap

import pytest
import torch

from fine_grained_sparse_fp32_b200 import _build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent('''
    import sys
    sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
    import numpy as np, torch
    import oracle
    from fine_grained_sparse_fp32_b200 import kmoe
    from fine_grained_sparse_fp32_b200.inputs import CONFIGS, make_inputs, to_host
    from parity import TOL, row_rel_err
    lib = kmoe.load()
    assert kmoe._lib is not None

    def case(name, N):
        cfg = CONFIGS[name].with_tokens(N)
        dev = make_inputs(cfg, seed=0, device="cuda")
        host = to_host(dev)
        l = oracle.router_logits(host["x"], cfg.x_dtype, host["w_router"], nthreads=oracle.max_threads())
        idx, _, _ = oracle.select(l, host["bias"], cfg.K)
        _, offsets, perm, _ = oracle.permute(idx, cfg.E)
        return cfg, dev, host, offsets, perm

    def ffn(cfg, dev, perm, offsets):
        ws = kmoe.workspace(cfg.N, cfg.d, cfg.E, cfg.K, cfg.I, kmoe.KMOE_BF16, kmoe.w_dtype_code(cfg.w_dtype))
        yp, ys = kmoe.moe_grouped_ffn(dev["x"], dev, torch.from_numpy(perm).cuda(), torch.from_numpy(offsets).cuda(),
                                      ws=ws)
        return yp, ys, kmoe.moe_device_status(ws)

    # valid dispatch: status 0 and parity (swap-AB BF16, FP8 tensor cores with two-term and with FP8
    # activations, tokens-as-M BF16)
    for name, N in (("decode", 32), ("fp8_decode", 32), ("fp8a8_decode", 32), ("prefill", 300)):
        cfg, dev, host, offsets, perm = case(name, N)
        yp, ys, st = ffn(cfg, dev, perm, offsets)
        assert st == 0, (name, st)
        rows = np.arange(0, cfg.N * cfg.K, 11)
        e = np.searchsorted(offsets, rows, side="right") - 1
        f = oracle.expert_outputs_a8 if cfg.w_dtype == "e4m3_a8" else oracle.expert_outputs
        ref = f(host, perm[rows], e, nthreads=oracle.max_threads())
        got = yp[torch.from_numpy(rows).cuda().long()].float().cpu().numpy()
        assert row_rel_err(got, ref) <= TOL[cfg.w_dtype], name
        y, idx, _, counts = kmoe.moe_forward(dev["x"], dev, with_outputs=True)
        torch.cuda.synchronize()
        assert int(counts.sum()) == cfg.N * cfg.K
        print("ok", name, N)

    # a token index past the batch (swap-AB path, where a row beyond N would only be read as zeros)
    cfg, dev, host, offsets, perm = case("decode", 32)
    bad = perm.copy(); bad[5] = cfg.N + 1000
    assert ffn(cfg, dev, bad, offsets)[2] == 3
    # the same on the FP8 tensor-core kernel (two-term activations)
    cfg8, dev8, host8, offsets8, perm8 = case("fp8_decode", 32)
    bad8 = perm8.copy(); bad8[7] = -5
    assert ffn(cfg8, dev8, bad8, offsets8)[2] == 3
    # offsets that are not a monotone partition: no unit runs, status 3 (both FFN kernels)
    bad_off = offsets.copy(); bad_off[10], bad_off[11] = bad_off[11] + 3, bad_off[10]
    assert ffn(cfg, dev, perm, bad_off)[2] == 3
    cfg, dev, host, offsets, perm = case("prefill", 300)
    bad_off = offsets.copy(); bad_off[-1] += 7
    assert ffn(cfg, dev, perm, bad_off)[2] == 3
    # and the library is still fine afterwards
    assert ffn(cfg, dev, perm, offsets)[2] == 0
    print("DEBUG-BUILD-OK")
''')


def test_debug_build_keeps_parity_and_reports_bad_dispatch_indices():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = _build.build(debug=True)
    env = dict(os.environ, KMOE_LIBRARY=lib)
    child = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", child], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "DEBUG-BUILD-OK" in r.stdout, r.stdout[-2000:] + r.stderr[-3000:]
