"""Thin Python binding of libkmoe.so (include/kmoe.h).

Argument marshalling only: every step of the layer runs in the CUDA library.
PyTorch supplies device memory and the current stream. There is no CPU
fallback: if the library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

from ._build import LIB

KMOE_OK, KMOE_ERR_INVALID_ARG, KMOE_ERR_UNSUPPORTED, KMOE_ERR_CUDA, KMOE_ERR_WORKSPACE, KMOE_ERR_DEVICE = range(6)
KMOE_F32, KMOE_BF16, KMOE_E4M3_B128, KMOE_E4M3_B128_A8 = 0, 1, 2, 3
SCORES = {"sigmoid": 0, "softmax": 1}     # kmoe_score

# Bytes at the head of a moe_grouped_ffn workspace: the status word, tickets
# and the grouped FFN's unit counters (include/kmoe.h).
FFN_STATUS_BYTES = (64 + 1088) * 4

EXPORTS = ["moe_workspace_size", "moe_router_topk", "moe_permute", "moe_permute_noalloc", "moe_grouped_ffn",
           "moe_combine", "moe_forward", "moe_block_workspace_size", "moe_block_forward", "moe_quant_1x128",
           "moe_device_status", "moe_set_wait_limit", "moe_last_error", "moe_abi_version"]


class KmoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"kmoe status {status}: {msg}")
        self.status = status


class Experts(ctypes.Structure):
    """kmoe_experts: one stack of SwiGLU experts."""
    _fields_ = [("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
                ("s_gate", ctypes.c_void_p), ("s_up", ctypes.c_void_p), ("s_down", ctypes.c_void_p),
                ("dtype", ctypes.c_int)]


_lib = None


def load(path: str | None = None):
    """Load libkmoe.so (or the library named by KMOE_LIBRARY, e.g. the KMOE_DEBUG build);
    raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or os.environ.get("KMOE_LIBRARY") or LIB
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is missing: build it with __graft_entry__.build()")
    lib = ctypes.CDLL(path)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.moe_workspace_size.restype = sz
    lib.moe_workspace_size.argtypes = [i, i, i, i, i, i, i]
    lib.moe_last_error.restype = ctypes.c_char_p
    lib.moe_abi_version.restype = i
    lib.moe_router_topk.argtypes = [vp, i, vp, vp, i, i, i, i, i, vp, vp, vp, vp, sz, vp]
    lib.moe_permute.argtypes = [vp, i, i, i, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_permute_noalloc.argtypes = [vp, i, i, i, vp, vp, vp, vp, vp]
    lib.moe_grouped_ffn.argtypes = [vp, i, i, i, i, i, i, vp, vp, ctypes.POINTER(Experts),
                                    ctypes.POINTER(Experts), vp, vp, vp, sz, vp]
    lib.moe_combine.argtypes = [vp, vp, i, vp, vp, i, i, i, vp, i, vp]
    lib.moe_forward.argtypes = [vp, i, i, i, i, i, i, i, vp, vp, ctypes.POINTER(Experts),
                                ctypes.POINTER(Experts), vp, i, vp, vp, vp, vp, sz, vp]
    lib.moe_block_workspace_size.restype = sz
    lib.moe_block_workspace_size.argtypes = [i, i, i, i, i, i]
    lib.moe_block_forward.argtypes = [vp, i, i, i, i, i, i, vp, vp, ctypes.c_float, vp, vp,
                                      ctypes.POINTER(Experts), ctypes.POINTER(Experts), vp, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_quant_1x128.argtypes = [vp, i, i, vp, vp, vp]
    lib.moe_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int), vp]
    lib.moe_set_wait_limit.argtypes = [ctypes.c_longlong]
    for f in ("moe_router_topk", "moe_permute", "moe_permute_noalloc", "moe_grouped_ffn", "moe_combine",
              "moe_forward", "moe_block_forward", "moe_quant_1x128", "moe_device_status", "moe_set_wait_limit"):
        getattr(lib, f).restype = i
    if lib.moe_abi_version() != 3:
        raise RuntimeError("libkmoe ABI version mismatch")
    _lib = lib
    return lib


def _check(status: int):
    if status != KMOE_OK:
        raise KmoeError(status, load().moe_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def dtype_code(t: torch.dtype) -> int:
    return {torch.float32: KMOE_F32, torch.bfloat16: KMOE_BF16}[t]


def w_dtype_code(name: str) -> int:
    return {"f32": KMOE_F32, "bf16": KMOE_BF16, "e4m3": KMOE_E4M3_B128, "e4m3_a8": KMOE_E4M3_B128_A8}[name]


def act_dtype_for(w_dtype: str) -> torch.dtype:
    """dtype of the grouped FFN outputs for a weight dtype (FP32 weights -> FP32)."""
    return torch.float32 if w_dtype == "f32" else torch.bfloat16


def experts_of(layer: dict, which: str = "routed") -> Experts:
    """kmoe_experts for a generator-layout layer: routed = experts 0..E-1, shared = index E."""
    cfg = layer["cfg"]
    e = cfg.E if which == "shared" else 0

    def at(name):
        t = layer.get(name)
        return None if t is None else ctypes.c_void_p(t[e].data_ptr() if which == "shared" else t.data_ptr())

    return Experts(at("w_gate"), at("w_up"), at("w_down"), at("s_gate"), at("s_up"), at("s_down"),
                   w_dtype_code(cfg.w_dtype))


def moe_workspace_size(N, d, E, K, I, x_dtype: int, w_dtype: int) -> int:
    return int(load().moe_workspace_size(N, d, E, K, I, x_dtype, w_dtype))


def workspace(N, d, E, K, I, x_dtype: int, w_dtype: int, device="cuda") -> torch.Tensor:
    n = moe_workspace_size(N, d, E, K, I, x_dtype, w_dtype)
    if n == 0:
        _check(KMOE_ERR_UNSUPPORTED)
    return torch.empty(n, dtype=torch.uint8, device=device)


def moe_router_topk(x, w_router, bias, K, logits=None, topk_idx=None, topk_w=None, ws=None, stream=None,
                    score="sigmoid"):
    N, d = x.shape
    E = w_router.shape[0]
    if topk_idx is None:
        topk_idx = torch.empty((N, K), dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty((N, K), dtype=torch.float32, device=x.device)
    if ws is None:   # logits (if not supplied) + status + the three BF16 router terms
        ws = torch.empty(((N * E * 4 + 255) // 256) * 256 + 256 + 3 * E * d * 2, dtype=torch.uint8,
                         device=x.device)
    _check(load().moe_router_topk(_ptr(x), dtype_code(x.dtype), _ptr(w_router), _ptr(bias), N, d, E, K,
                                  SCORES[score], _ptr(logits), _ptr(topk_idx), _ptr(topk_w), _ptr(ws),
                                  0 if ws is None else ws.numel(), _stream(stream)))
    return topk_idx, topk_w


def moe_permute(topk_idx, E, ws=None, stream=None):
    N, K = topk_idx.shape
    dev = topk_idx.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(N * K, 1), dtype=torch.int32, device=dev)
    inv = torch.empty((N, K), dtype=torch.int32, device=dev)
    if ws is None:
        ws = torch.empty(max(((N + 255) // 256) * E * 4, 16), dtype=torch.uint8, device=dev)
    _check(load().moe_permute(_ptr(topk_idx), N, K, E, _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv),
                              _ptr(ws), ws.numel(), _stream(stream)))
    return counts, offsets, perm[: N * K], inv


def moe_permute_noalloc(topk_idx, E, counts=None, offsets=None, perm=None, inv=None, stream=None):
    """moe_permute for callers that cannot hand the library a workspace.

    The library keeps the scratch in its own fixed 1 MiB device array, so the
    C call allocates nothing; the caller passes every output buffer (any left
    as None is allocated here by torch, for convenience in tests)."""
    N, K = topk_idx.shape
    dev = topk_idx.device
    counts = torch.empty(E, dtype=torch.int32, device=dev) if counts is None else counts
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev) if offsets is None else offsets
    perm = torch.empty(max(N * K, 1), dtype=torch.int32, device=dev) if perm is None else perm
    inv = torch.empty((N, K), dtype=torch.int32, device=dev) if inv is None else inv
    _check(load().moe_permute_noalloc(_ptr(topk_idx), N, K, E, _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv),
                                      _stream(stream)))
    return counts, offsets, perm[: N * K], inv


def moe_grouped_ffn(x, layer, perm_token, offsets, with_shared=True, ws=None, stream=None, out=None):
    cfg = layer["cfg"]
    N, d = x.shape
    I, E, K = cfg.I, cfg.E, cfg.K
    adt = act_dtype_for(cfg.w_dtype)
    if out is not None:
        y_perm, y_shared = out
    else:
        y_perm = torch.empty((N * K, d), dtype=adt, device=x.device)
        y_shared = torch.empty((N, d), dtype=adt, device=x.device) if with_shared else None
    if ws is None:
        ws = workspace(N, d, E, K, I, dtype_code(x.dtype), w_dtype_code(cfg.w_dtype), x.device)
    routed = experts_of(layer, "routed")
    shared = experts_of(layer, "shared") if with_shared else None
    _check(load().moe_grouped_ffn(_ptr(x), dtype_code(x.dtype), N, d, I, E, K, _ptr(perm_token), _ptr(offsets),
                                  ctypes.byref(routed), ctypes.byref(shared) if shared is not None else None,
                                  _ptr(y_perm), _ptr(y_shared), _ptr(ws), ws.numel(), _stream(stream)))
    return y_perm, y_shared


def moe_device_status(ws, stream=None) -> int:
    """Synchronises `stream` and returns the device status word of workspace `ws` (0 = ok)."""
    st = ctypes.c_int(-1)
    rc = load().moe_device_status(_ptr(ws), ctypes.byref(st), _stream(stream))
    if rc not in (KMOE_OK, KMOE_ERR_DEVICE):
        _check(rc)
    return st.value


def moe_set_wait_limit(cycles: int):
    """Give-up limit (SM cycles) of the FFN kernels' pipeline waits for this host thread; 0 = default."""
    _check(load().moe_set_wait_limit(int(cycles)))


def moe_combine(y_perm, y_shared, topk_w, inv_pos, y_dtype=torch.bfloat16, out=None, stream=None):
    N, K = topk_w.shape
    d = y_perm.shape[1]
    y = out if out is not None else torch.empty((N, d), dtype=y_dtype, device=y_perm.device)
    _check(load().moe_combine(_ptr(y_perm), _ptr(y_shared), dtype_code(y_perm.dtype), _ptr(topk_w), _ptr(inv_pos),
                              N, K, d, _ptr(y), dtype_code(y.dtype), _stream(stream)))
    return y


def moe_block_workspace_size(N, d, E, K, I, w_dtype: int) -> int:
    return int(load().moe_block_workspace_size(N, d, E, K, I, w_dtype))


class Layer:
    """Device-resident weights of one layer plus a reusable workspace.

    `forward(x)` is one moe_forward call and `block_forward(h, ...)` one
    moe_block_forward call (workspace sized for it when `block` is set);
    outputs are written into tensors owned here (or passed in)."""

    def __init__(self, layer: dict, max_tokens: int, y_dtype=torch.bfloat16, score: str = "sigmoid",
                 block: bool = False):
        self.layer = layer
        cfg = self.cfg = layer["cfg"]
        self.routed = experts_of(layer, "routed")
        self.shared = experts_of(layer, "shared")
        dev = layer["w_gate"].device
        self.x_code = w_dtype_code(cfg.x_dtype)
        if block:
            n = moe_block_workspace_size(max_tokens, cfg.d, cfg.E, cfg.K, cfg.I, w_dtype_code(cfg.w_dtype))
            if n == 0:
                _check(KMOE_ERR_UNSUPPORTED)
            self.ws = torch.empty(n, dtype=torch.uint8, device=dev)
        else:
            self.ws = workspace(max_tokens, cfg.d, cfg.E, cfg.K, cfg.I, self.x_code, w_dtype_code(cfg.w_dtype), dev)
        self.y_dtype = y_dtype
        self.max_tokens = max_tokens
        self.score = SCORES[score]

    def forward(self, x, y=None, topk_idx=None, topk_w=None, counts=None, stream=None):
        cfg = self.cfg
        N = x.shape[0]
        if N > self.max_tokens:
            raise ValueError("more tokens than the workspace was sized for")
        if y is None:
            y = torch.empty((N, cfg.d), dtype=self.y_dtype, device=x.device)
        L = self.layer
        _check(load().moe_forward(_ptr(x), dtype_code(x.dtype), N, cfg.d, cfg.E, cfg.K, cfg.I, self.score,
                                  _ptr(L["w_router"]), _ptr(L["bias"]), ctypes.byref(self.routed),
                                  ctypes.byref(self.shared), _ptr(y), dtype_code(y.dtype), _ptr(topk_idx),
                                  _ptr(topk_w), _ptr(counts), _ptr(self.ws), self.ws.numel(), _stream(stream)))
        return y

    def block_forward(self, h, gamma_pre, gamma_post, eps: float, h_out=None, topk_idx=None, topk_w=None,
                      counts=None, x_out=None, stream=None):
        """h_out = h + RMSNorm(layer(x)) * gamma_post with x = bf16(RMSNorm(h) * gamma_pre); h_out may
        be h; x_out (optional) receives x."""
        cfg = self.cfg
        N = h.shape[0]
        if N > self.max_tokens:
            raise ValueError("more tokens than the workspace was sized for")
        if h_out is None:
            h_out = torch.empty_like(h)
        L = self.layer
        _check(load().moe_block_forward(_ptr(h), N, cfg.d, cfg.E, cfg.K, cfg.I, self.score, _ptr(gamma_pre),
                                        _ptr(gamma_post), float(eps), _ptr(L["w_router"]), _ptr(L["bias"]),
                                        ctypes.byref(self.routed), ctypes.byref(self.shared), _ptr(h_out),
                                        _ptr(x_out), _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(self.ws),
                                        self.ws.numel(), _stream(stream)))
        return h_out


def moe_forward(x, layer, y_dtype=torch.bfloat16, with_outputs=False, stream=None, score="sigmoid"):
    """One whole-layer call; with_outputs also returns (topk_idx, topk_w, counts)."""
    cfg = layer["cfg"]
    N = x.shape[0]
    lay = Layer(layer, N, y_dtype, score)
    if not with_outputs:
        return lay.forward(x, stream=stream)
    idx = torch.empty((N, cfg.K), dtype=torch.int32, device=x.device)
    w = torch.empty((N, cfg.K), dtype=torch.float32, device=x.device)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=x.device)
    y = lay.forward(x, topk_idx=idx, topk_w=w, counts=counts, stream=stream)
    return y, idx, w, counts


def moe_block_forward(h, layer, gamma_pre, gamma_post, eps: float, with_outputs=False, stream=None,
                      score="sigmoid", h_out=None):
    """One sandwich-block call; with_outputs also returns (x, topk_idx, topk_w, counts)."""
    cfg = layer["cfg"]
    N = h.shape[0]
    lay = Layer(layer, N, torch.bfloat16, score, block=True)
    if not with_outputs:
        return lay.block_forward(h, gamma_pre, gamma_post, eps, h_out=h_out, stream=stream)
    idx = torch.empty((N, cfg.K), dtype=torch.int32, device=h.device)
    w = torch.empty((N, cfg.K), dtype=torch.float32, device=h.device)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=h.device)
    x = torch.empty_like(h)
    out = lay.block_forward(h, gamma_pre, gamma_post, eps, h_out=h_out, topk_idx=idx, topk_w=w, counts=counts,
                            x_out=x, stream=stream)
    return out, x, idx, w, counts


def moe_quant_1x128(x, codes=None, scales=None, stream=None):
    """E4M3 codes (uint8 [rows, cols]) and FP32 scales ([rows, cols / 128]) of BF16 x."""
    rows, cols = x.shape
    if codes is None:
        codes = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((rows, cols // 128), dtype=torch.float32, device=x.device)
    _check(load().moe_quant_1x128(_ptr(x), rows, cols, _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales
