"""Python access to the CPU oracle (oracle/moe_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg. The product path (the CUDA library and its
binding) never imports it.

The C source is compiled with gcc on first use (or by the package build) into
oracle/liboracle.so; no CUDA toolchain is involved. All floating-point work is
done in double inside the C code; this wrapper only marshals arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16, E4M3 = 0, 1, 2
_DT = {"f32": F32, "bf16": BF16, "e4m3": E4M3, "e4m3_a8": E4M3}   # e4m3_a8: E4M3 weights, stored alike

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math: sums keep their order)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.oracle_e4m3_to_double.restype = ctypes.c_double
        _lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        _lib.oracle_float_to_e4m3.restype = ctypes.c_uint8
        _lib.oracle_float_to_e4m3.argtypes = [ctypes.c_float]
        _lib.oracle_permute.restype = ctypes.c_int
        _lib.oracle_max_threads.restype = ctypes.c_int
    return _lib


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def _p(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else ctypes.c_void_p(0)


def _bits(t):
    """A host array holding exactly the stored bits of a tensor (torch or numpy)."""
    try:
        import torch
        if torch.is_tensor(t):
            t = t.detach().cpu().contiguous()
            if t.dtype == torch.bfloat16:
                return t.view(torch.int16).numpy().view(np.uint16)
            return t.numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(t)


def e4m3_to_double(code: int) -> float:
    return float(lib().oracle_e4m3_to_double(ctypes.c_uint8(code)))


def router_logits(x, x_dtype: str, w_router, nthreads: int = 1) -> np.ndarray:
    xb = _bits(x)
    w = np.ascontiguousarray(_bits(w_router), dtype=np.float32)
    N, d = xb.shape
    E = w.shape[0]
    out = np.empty((N, E), dtype=np.float64)
    lib().oracle_router_logits(N, d, E, _p(xb), _DT[x_dtype], _p(w), _p(out), nthreads)
    return out


SCORES = {"sigmoid": 0, "softmax": 1}


def select(logits: np.ndarray, bias, K: int, score: str = "sigmoid"):
    """(idx [N,K] int32, g [N,K] double, margin [N] double) for given logits.

    score "sigmoid": g = sigmoid of the unbiased logit; "softmax": g = softmax
    over the K selected unbiased logits."""
    l = np.ascontiguousarray(logits, dtype=np.float64)
    b = np.ascontiguousarray(_bits(bias), dtype=np.float32)
    N, E = l.shape
    idx = np.empty((N, K), dtype=np.int32)
    g = np.empty((N, K), dtype=np.float64)
    margin = np.empty(N, dtype=np.float64)
    lib().oracle_select_score(N, E, K, _p(l), _p(b), SCORES[score], _p(idx), _p(g), _p(margin))
    return idx, g, margin


def permute(idx, E: int):
    """(counts [E], offsets [E+1], perm_token [N*K], inv_pos [N,K]) by counting sort."""
    ix = np.ascontiguousarray(idx, dtype=np.int32)
    N, K = ix.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    perm = np.empty(N * K, dtype=np.int32)
    inv = np.empty((N, K), dtype=np.int32)
    rc = lib().oracle_permute(N, K, E, _p(ix), _p(counts), _p(offsets), _p(perm), _p(inv))
    if rc != 0:
        raise ValueError("expert index out of range")
    return counts, offsets, perm, inv


def _weights(inp):
    cfg = inp["cfg"]
    wg, wu, wd = _bits(inp["w_gate"]), _bits(inp["w_up"]), _bits(inp["w_down"])
    if cfg.w_dtype in ("e4m3", "e4m3_a8"):
        sg, su, sd = (np.ascontiguousarray(_bits(inp[k]), dtype=np.float32) for k in ("s_gate", "s_up", "s_down"))
    else:
        sg = su = sd = None
    return wg, wu, wd, sg, su, sd


def expert_outputs(inp, tokens, experts, nthreads: int = 1) -> np.ndarray:
    """F_e(x_t) in double for each (t, e) pair; e == E is the shared expert."""
    cfg = inp["cfg"]
    xb = _bits(inp["x"])
    wg, wu, wd, sg, su, sd = _weights(inp)
    tok = np.ascontiguousarray(tokens, dtype=np.int32)
    ex = np.ascontiguousarray(experts, dtype=np.int32)
    out = np.empty((len(tok), cfg.d), dtype=np.float64)
    lib().oracle_expert_outputs(cfg.d, cfg.I, _p(xb), _DT[cfg.x_dtype], _DT[cfg.w_dtype],
                                _p(wg), _p(wu), _p(wd), _p(sg), _p(su), _p(sd),
                                len(tok), _p(tok), _p(ex), _p(out), nthreads)
    return out


def layer(inp, rows=None, nthreads: int = 1, score: str = "sigmoid"):
    """The whole layer for tokens `rows` (default: all), mixture weights by `score`.

    Returns dict(y [n,d] double, idx [n,K], g [n,K], margin [n])."""
    cfg = inp["cfg"]
    xb = _bits(inp["x"])
    N = xb.shape[0]
    rows = np.arange(N, dtype=np.int32) if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    wr = np.ascontiguousarray(_bits(inp["w_router"]), dtype=np.float32)
    b = np.ascontiguousarray(_bits(inp["bias"]), dtype=np.float32)
    wg, wu, wd, sg, su, sd = _weights(inp)
    n = len(rows)
    y = np.empty((n, cfg.d), dtype=np.float64)
    idx = np.empty((n, cfg.K), dtype=np.int32)
    g = np.empty((n, cfg.K), dtype=np.float64)
    margin = np.empty(n, dtype=np.float64)
    lib().oracle_layer_score(N, cfg.d, cfg.E, cfg.K, cfg.I, _p(xb), _DT[cfg.x_dtype], _p(wr), _p(b),
                             _p(wg), _p(wu), _p(wd), _p(sg), _p(su), _p(sd), _DT[cfg.w_dtype],
                             n, _p(rows), SCORES[score], _p(y), _p(idx), _p(g), _p(margin), nthreads)
    return {"y": y, "idx": idx, "g": g, "margin": margin, "rows": rows}


def rmsnorm_bf16(h, gamma, eps: float) -> np.ndarray:
    """x = bf16(h / sqrt(mean(h^2) + eps) * gamma) row by row, as uint16 BF16 bits."""
    hb = np.ascontiguousarray(_bits(h), dtype=np.uint16)
    gb = np.ascontiguousarray(_bits(gamma), dtype=np.uint16)
    N, d = hb.shape
    x = np.empty((N, d), dtype=np.uint16)
    lib().oracle_rmsnorm_bf16(N, d, _p(hb), _p(gb), ctypes.c_double(eps), _p(x))
    return x


def block(inp, h, gamma_pre, gamma_post, eps: float, rows=None, nthreads: int = 1, score: str = "sigmoid"):
    """The sandwich block around the layer for tokens `rows`: x = bf16(RMSNorm(h) * g_pre),
    m = layer(x), h_out = h + RMSNorm(m) * g_post. Returns dict(h_out, x, m, idx, g, margin)."""
    hb = np.ascontiguousarray(_bits(h), dtype=np.uint16)
    N, d = hb.shape
    x = rmsnorm_bf16(hb, gamma_pre, eps)
    layer_fn = layer_a8 if inp["cfg"].w_dtype == "e4m3_a8" else layer      # FP8 activations: the 1 x 128 layer
    ora = layer_fn(dict(inp, x=x), rows=rows, nthreads=nthreads, score=score)
    m = np.ascontiguousarray(ora["y"], dtype=np.float64)
    rws = ora["rows"]
    gp = np.ascontiguousarray(_bits(gamma_post), dtype=np.uint16)
    h_out = np.empty_like(m)
    lib().oracle_post_residual(N, d, len(rws), _p(rws), _p(hb), _p(m), _p(gp), ctypes.c_double(eps), _p(h_out))
    return {"h_out": h_out, "x": x, "m": m, "idx": ora["idx"], "g": ora["g"], "margin": ora["margin"], "rows": rws}


def float_to_e4m3(values) -> np.ndarray:
    """E4M3 codes (round to nearest even, saturated to +-448) of float32 values."""
    v = np.asarray(values, dtype=np.float32).ravel()
    return np.array([lib().oracle_float_to_e4m3(float(x)) for x in v], dtype=np.uint8).reshape(np.shape(values))


def quant_1x128(x):
    """Dynamic FP8 quantisation of BF16 rows in groups of 128 columns.

    Returns (codes uint8 [rows, cols], scales float32 [rows, cols / 128])."""
    xb = np.ascontiguousarray(_bits(x), dtype=np.uint16)
    rows, cols = xb.shape
    codes = np.empty((rows, cols), dtype=np.uint8)
    scales = np.empty((rows, cols // 128), dtype=np.float32)
    lib().oracle_quant_1x128(rows, cols, _p(xb), _p(codes), _p(scales))
    return codes, scales


def layer_a8(inp, rows=None, nthreads: int = 1, score: str = "sigmoid"):
    """The layer with E4M3 weights and activations quantised in 1 x 128 groups (x for
    gate/up, H for down); routing on x as stored. Returns dict(y, idx, g, margin, rows)."""
    cfg = inp["cfg"]
    if cfg.w_dtype not in ("e4m3", "e4m3_a8") or cfg.x_dtype != "bf16":
        raise ValueError("FP8 activations need BF16 x and E4M3 weights")
    xb = np.ascontiguousarray(_bits(inp["x"]), dtype=np.uint16)
    N = xb.shape[0]
    rows = np.arange(N, dtype=np.int32) if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    wr = np.ascontiguousarray(_bits(inp["w_router"]), dtype=np.float32)
    b = np.ascontiguousarray(_bits(inp["bias"]), dtype=np.float32)
    wg, wu, wd, sg, su, sd = _weights(inp)
    n = len(rows)
    y = np.empty((n, cfg.d), dtype=np.float64)
    idx = np.empty((n, cfg.K), dtype=np.int32)
    g = np.empty((n, cfg.K), dtype=np.float64)
    margin = np.empty(n, dtype=np.float64)
    lib().oracle_layer_a8(N, cfg.d, cfg.E, cfg.K, cfg.I, _p(xb), _p(wr), _p(b), _p(wg), _p(wu), _p(wd),
                          _p(sg), _p(su), _p(sd), n, _p(rows), SCORES[score], _p(y), _p(idx), _p(g), _p(margin),
                          nthreads)
    return {"y": y, "idx": idx, "g": g, "margin": margin, "rows": rows}


def expert_outputs_a8(inp, tokens, experts, nthreads: int = 1) -> np.ndarray:
    """F_e(x_t) in double with FP8 activations (x and H quantised in 1 x 128 groups) for each
    (t, e) pair; e == E is the shared expert. E4M3 weights and BF16 x only."""
    cfg = inp["cfg"]
    if cfg.w_dtype not in ("e4m3", "e4m3_a8") or cfg.x_dtype != "bf16":
        raise ValueError("FP8 activations need BF16 x and E4M3 weights")
    xb = np.ascontiguousarray(_bits(inp["x"]), dtype=np.uint16)
    wg, wu, wd, sg, su, sd = _weights(inp)
    tok = np.ascontiguousarray(tokens, dtype=np.int32)
    ex = np.ascontiguousarray(experts, dtype=np.int32)
    out = np.empty((len(tok), cfg.d), dtype=np.float64)
    lib().oracle_expert_outputs_a8(cfg.d, cfg.I, _p(xb), _p(wg), _p(wu), _p(wd), _p(sg), _p(su), _p(sd),
                                   len(tok), _p(tok), _p(ex), _p(out), nthreads)
    return out


__all__ = ["build", "lib", "max_threads", "e4m3_to_double", "router_logits", "select",
           "permute", "expert_outputs", "layer", "rmsnorm_bf16", "block", "float_to_e4m3", "quant_1x128",
           "layer_a8", "expert_outputs_a8", "F32", "BF16", "E4M3"]
