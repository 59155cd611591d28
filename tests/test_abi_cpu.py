"""Host-side checks of the C ABI: the library loads, exports what the header
declares, sizes its workspace, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import pytest

from fine_grained_sparse_fp32_b200 import _build, kmoe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return kmoe.load()


def header_functions():
    src = open(os.path.join(ROOT, "include", "kmoe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_\w+)\s*\(", src)))


def test_header_declares_the_documented_entry_points():
    assert header_functions() == sorted(kmoe.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(_build.LIB)
    for name in header_functions():
        assert hasattr(raw, name), name


def test_abi_version(lib):
    assert lib.moe_abi_version() == 3


def test_workspace_size_grows_with_tokens(lib):
    a = kmoe.moe_workspace_size(32, 2560, 384, 6, 512, kmoe.KMOE_BF16, kmoe.KMOE_BF16)
    b = kmoe.moe_workspace_size(8192, 2560, 384, 6, 512, kmoe.KMOE_BF16, kmoe.KMOE_BF16)
    assert 0 < a < b
    # Y rows (N*K + N) * d * 2 bytes dominate at prefill
    assert b >= (8192 * 7) * 2560 * 2


@pytest.mark.parametrize("args", [
    (32, 2560, 384, 9, 512),     # K > 8
    (32, 2560, 4, 6, 512),       # E < K
    (32, 2500, 384, 6, 512),     # d not a multiple of 128
    (32, 2560, 384, 6, 500),     # I not a multiple of 128
    (-1, 2560, 384, 6, 512),     # negative N
    (32, 2560, 2048, 6, 512),    # E > 1024
])
def test_workspace_size_rejects_unsupported(lib, args):
    assert kmoe.moe_workspace_size(*args, kmoe.KMOE_BF16, kmoe.KMOE_BF16) == 0


def test_bad_arguments_fail_on_the_host(lib):
    vp = ctypes.c_void_p
    aligned = vp(1 << 20)
    # K = 9 is not compiled
    st = lib.moe_router_topk(aligned, kmoe.KMOE_BF16, aligned, aligned, 4, 2560, 384, 9, 0,
                             None, aligned, aligned, aligned, 1 << 20, None)
    assert st == kmoe.KMOE_ERR_UNSUPPORTED
    assert b"K=9" in lib.moe_last_error()
    # null x
    st = lib.moe_router_topk(None, kmoe.KMOE_BF16, aligned, aligned, 4, 2560, 384, 6, 0,
                             None, aligned, aligned, aligned, 1 << 20, None)
    assert st == kmoe.KMOE_ERR_INVALID_ARG
    # misaligned pointer
    st = lib.moe_router_topk(vp((1 << 20) + 4), kmoe.KMOE_BF16, aligned, aligned, 4, 2560, 384, 6, 0,
                             None, aligned, aligned, aligned, 1 << 20, None)
    assert st == kmoe.KMOE_ERR_INVALID_ARG and b"aligned" in lib.moe_last_error()
    # unknown activation dtype
    st = lib.moe_router_topk(aligned, 7, aligned, aligned, 4, 2560, 384, 6, 0,
                             None, aligned, aligned, aligned, 1 << 20, None)
    assert st == kmoe.KMOE_ERR_UNSUPPORTED
    # workspace too small
    st = lib.moe_router_topk(aligned, kmoe.KMOE_BF16, aligned, aligned, 4, 2560, 384, 6, 0,
                             None, aligned, aligned, aligned, 16, None)
    assert st == kmoe.KMOE_ERR_WORKSPACE


def test_unknown_score_function_is_rejected(lib):
    a = ctypes.c_void_p(1 << 20)
    st = lib.moe_router_topk(a, kmoe.KMOE_BF16, a, a, 4, 2560, 384, 6, 7, None, a, a, a, 1 << 20, None)
    assert st == kmoe.KMOE_ERR_INVALID_ARG and b"score" in lib.moe_last_error()


def test_forward_rejects_null_experts_and_mixed_dtypes(lib):
    vp = ctypes.c_void_p
    a = vp(1 << 20)
    ex = kmoe.Experts(a, a, a, None, None, None, kmoe.KMOE_BF16)
    fp8 = kmoe.Experts(a, a, a, None, None, None, kmoe.KMOE_E4M3_B128)   # scales missing
    args = lambda r, s: (a, kmoe.KMOE_BF16, 32, 2560, 384, 6, 512, 0, a, a, r, s, a, kmoe.KMOE_BF16,
                         None, None, None, a, 1 << 40, None)
    assert lib.moe_forward(*args(None, None)) == kmoe.KMOE_ERR_INVALID_ARG
    assert lib.moe_forward(*args(ctypes.byref(fp8), None)) == kmoe.KMOE_ERR_INVALID_ARG
    mixed = kmoe.Experts(a, a, a, a, a, a, kmoe.KMOE_E4M3_B128)
    assert lib.moe_forward(*args(ctypes.byref(ex), ctypes.byref(mixed))) == kmoe.KMOE_ERR_UNSUPPORTED


def test_zero_tokens_is_a_host_side_no_op(lib):
    a = ctypes.c_void_p(1 << 20)
    ex = kmoe.Experts(a, a, a, None, None, None, kmoe.KMOE_BF16)
    assert lib.moe_router_topk(None, kmoe.KMOE_BF16, None, None, 0, 2560, 384, 6, 0,
                               None, None, None, None, 0, None) == kmoe.KMOE_OK
    assert lib.moe_forward(None, kmoe.KMOE_BF16, 0, 2560, 384, 6, 512, 0, None, None, ctypes.byref(ex),
                           None, None, kmoe.KMOE_BF16, None, None, None, None, 0, None) == kmoe.KMOE_OK
    assert lib.moe_last_error() == b""


def test_block_workspace_adds_the_normalised_input(lib):
    for w in (kmoe.KMOE_BF16, kmoe.KMOE_E4M3_B128):
        base = lib.moe_workspace_size(64, 2560, 384, 6, 512, kmoe.KMOE_BF16, w)
        blk = lib.moe_block_workspace_size(64, 2560, 384, 6, 512, w)
        assert blk >= base + 64 * 2560 * 2
    assert lib.moe_block_workspace_size(64, 2560, 384, 6, 512, kmoe.KMOE_F32) == 0


def test_block_forward_checks_arguments_on_the_host(lib):
    vp = ctypes.c_void_p
    a = vp(1 << 20)
    bf = kmoe.Experts(a, a, a, None, None, None, kmoe.KMOE_BF16)
    f32 = kmoe.Experts(a, a, a, None, None, None, kmoe.KMOE_F32)

    def call(N=32, d=2560, K=6, g_pre=a, g_post=a, eps=1e-6, routed=bf, shared=bf, score=0):
        return lib.moe_block_forward(a, N, d, 384, K, 512, score, g_pre, g_post, eps, a, a, ctypes.byref(routed),
                                     ctypes.byref(shared) if shared is not None else None, a, None, None, None, None, a,
                                     1 << 40, None)

    assert call(routed=f32, shared=f32) == kmoe.KMOE_ERR_UNSUPPORTED and b"BF16" in lib.moe_last_error()
    assert call(eps=-1.0) == kmoe.KMOE_ERR_INVALID_ARG and b"eps" in lib.moe_last_error()
    assert call(eps=float("nan")) == kmoe.KMOE_ERR_INVALID_ARG
    assert call(g_pre=None) == kmoe.KMOE_ERR_INVALID_ARG and b"gamma_pre" in lib.moe_last_error()
    assert call(g_post=None) == kmoe.KMOE_ERR_INVALID_ARG and b"gamma_post" in lib.moe_last_error()
    assert call(score=5) == kmoe.KMOE_ERR_INVALID_ARG
    # K routed rows plus the shared row of d = 6144 do not fit the combine's staging buffer
    assert call(d=6144, K=8) == kmoe.KMOE_ERR_UNSUPPORTED and b"staging" in lib.moe_last_error()
    assert call(N=0, g_pre=None, g_post=None) == kmoe.KMOE_OK
    small = lib.moe_block_forward(a, 32, 2560, 384, 6, 512, 0, a, a, 1e-6, a, a, ctypes.byref(bf), None, a,
                                  None, None, None, None, a, 1024, None)
    assert small == kmoe.KMOE_ERR_WORKSPACE


def test_block_forward_needs_d_multiple_of_256(lib):
    a = ctypes.c_void_p(1 << 20)
    bf = kmoe.Experts(a, a, a, None, None, None, kmoe.KMOE_BF16)
    st = lib.moe_block_forward(a, 32, 2688, 384, 6, 512, 0, a, a, 1e-6, a, a, ctypes.byref(bf), ctypes.byref(bf), a,
                               None, None, None, None, a, 1 << 40, None)
    assert st == kmoe.KMOE_ERR_UNSUPPORTED and b"256" in lib.moe_last_error()


def test_quant_1x128_checks_arguments_on_the_host(lib):
    a = ctypes.c_void_p(1 << 20)
    assert lib.moe_quant_1x128(a, 4, 200, a, a, None) == kmoe.KMOE_ERR_UNSUPPORTED
    assert lib.moe_quant_1x128(a, -1, 128, a, a, None) == kmoe.KMOE_ERR_INVALID_ARG
    assert lib.moe_quant_1x128(a, 4, 128, None, a, None) == kmoe.KMOE_ERR_INVALID_ARG
    assert lib.moe_quant_1x128(None, 0, 128, None, None, None) == kmoe.KMOE_OK


def test_two_term_small_batches_are_sized_for_both_code_planes():
    """E4M3 weights with BF16 x below 256 tokens run with two-term activations: H's two code planes
    take the BF16 H's bytes, and H's scales plus x's high codes, low codes and scales come on top;
    from 256 tokens the workspace is the BF16-weight one."""
    d, E, K, I = 2560, 384, 6, 512
    for N in (1, 32, 255):
        e4 = kmoe.moe_workspace_size(N, d, E, K, I, kmoe.KMOE_BF16, kmoe.KMOE_E4M3_B128)
        bf = kmoe.moe_workspace_size(N, d, E, K, I, kmoe.KMOE_BF16, kmoe.KMOE_BF16)
        R = N * K + N
        expected = R * (I // 128) * 4 + 2 * N * d + N * (d // 128) * 4
        assert abs((e4 - bf) - expected) <= 4 * 256
    for N in (256, 4096):
        assert kmoe.moe_workspace_size(N, d, E, K, I, kmoe.KMOE_BF16, kmoe.KMOE_E4M3_B128) == \
            kmoe.moe_workspace_size(N, d, E, K, I, kmoe.KMOE_BF16, kmoe.KMOE_BF16)


def test_wait_limit_rejects_negative_and_restores_the_default(lib):
    assert lib.moe_set_wait_limit(-1) == kmoe.KMOE_ERR_INVALID_ARG
    assert lib.moe_set_wait_limit(1000) == kmoe.KMOE_OK
    assert lib.moe_set_wait_limit(0) == kmoe.KMOE_OK


def test_fp8_activation_mode_is_sized_and_checked_on_the_host(lib):
    """KMOE_E4M3_B128_A8: workspace sizes include the FP8 pieces, and FP32 x or a d that is not a
    multiple of 256 is rejected before anything is enqueued (no GPU needed)."""
    N, d, E, K, I = 32, 2560, 384, 6, 512
    a8 = kmoe.moe_workspace_size(N, d, E, K, I, kmoe.KMOE_BF16, kmoe.KMOE_E4M3_B128_A8)
    bf = kmoe.moe_workspace_size(N, d, E, K, I, kmoe.KMOE_BF16, kmoe.KMOE_BF16)
    # H as one-byte codes (instead of BF16) plus its scales, and x's codes and scales (each piece
    # 256-byte aligned)
    R = N * K + N
    expected = -R * I + R * (I // 128) * 4 + N * d + N * (d // 128) * 4
    assert a8 > 0 and abs((a8 - bf) - expected) <= 4 * 256
    assert kmoe.moe_block_workspace_size(N, d, E, K, I, kmoe.KMOE_E4M3_B128_A8) > 0
    aligned = ctypes.c_void_p(1 << 20)
    ex = kmoe.Experts(aligned, aligned, aligned, aligned, aligned, aligned, kmoe.KMOE_E4M3_B128_A8)
    for x_dtype, dd in ((kmoe.KMOE_F32, 2560), (kmoe.KMOE_BF16, 2688)):
        st = lib.moe_forward(aligned, x_dtype, N, dd, E, K, I, 0, aligned, aligned, ctypes.byref(ex), ctypes.byref(ex),
                             aligned, kmoe.KMOE_BF16, None, None, None, aligned, 1 << 40, None)
        assert st == kmoe.KMOE_ERR_UNSUPPORTED and b"FP8 activations" in lib.moe_last_error()
        st = lib.moe_grouped_ffn(aligned, x_dtype, N, dd, I, E, K, aligned, aligned, ctypes.byref(ex), None,
                                 aligned, None, aligned, 1 << 40, None)
        assert st == kmoe.KMOE_ERR_UNSUPPORTED
