"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import combine_moe_route_14_b200 as moe
from combine_moe_route_14_b200 import build as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "moe.h")
OK, INVALID, UNSUPPORTED = 0, 1, 2


@pytest.fixture(scope="module")
def lib():
    B.build()
    return moe.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_layer_calls():
    names = declared_functions()
    for n in ("moe_route", "moe_layout", "moe_dispatch", "moe_dispatch_by_token",
              "moe_expert_ffn", "moe_combine",
              "moe_layer_forward", "moe_router_logits", "moe_expert_gemm"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_declared_symbol():
    sig = set(moe._SIG)
    assert set(declared_functions()) <= sig


def _err(lib):
    return lib.moe_last_error_string().decode()


N = None


def test_route_rejects_bad_args(lib):
    assert lib.moe_route(N, 4, 8, 2, 0, 1, N, N, N) == INVALID          # null pointers
    assert lib.moe_route(N, 4, 8, 9, 0, 1, N, N, N) == INVALID          # k > E
    assert "k must be" in _err(lib)
    assert lib.moe_route(N, -1, 8, 2, 0, 1, N, N, N) == INVALID         # T < 0
    assert lib.moe_route(N, 4, 2048, 2, 0, 1, N, N, N) == UNSUPPORTED   # E > 1024
    assert lib.moe_route(N, 4, 64, 32, 0, 1, N, N, N) == UNSUPPORTED    # k > 16
    assert lib.moe_route(N, 4, 8, 2, 7, 1, N, N, N) == INVALID          # unknown score
    assert lib.moe_route(N, 0, 8, 2, 0, 1, N, N, N) == OK               # T == 0: no-op


def test_misaligned_pointer_is_rejected(lib):
    assert lib.moe_route(ctypes.c_void_p(0x1002), 4, 8, 2, 0, 1, ctypes.c_void_p(0x1000),
                         ctypes.c_void_p(0x1000), N) == INVALID
    assert "aligned" in _err(lib)
    assert lib.moe_dispatch(ctypes.c_void_p(0x1008), ctypes.c_void_p(0x2000), 4, 64, 2,
                            ctypes.c_void_p(0x3000), N) == INVALID


def test_dims_must_be_multiples_of_8(lib):
    assert lib.moe_dispatch(N, N, 4, 12, 2, N, N) == UNSUPPORTED
    assert lib.moe_combine(N, N, N, 4, 100, 2, N, N) == UNSUPPORTED
    assert lib.moe_expert_gemm(N, N, N, 8, 16, 12, 64, 0, N, N) == UNSUPPORTED
    assert lib.moe_expert_gemm(N, N, N, 8, 16, 64, 0, 0, N, N) == INVALID


def test_layout_rejects_short_workspace(lib):
    p = ctypes.c_void_p(0x10000)
    need = lib.moe_layout_workspace_size(8192, 256, 8)
    assert need > 0  # the multi-block scan needs look-back words
    assert lib.moe_layout(p, 8192, 256, 8, p, p, p, p, p, need - 1, N) == INVALID
    assert "workspace" in _err(lib)
    assert lib.moe_layout_workspace_size(16, 8, 2) == 0  # one-block path needs none


def test_layer_workspace_and_desc_checks(lib):
    d = moe.LayerDesc(4096, 4096, 8, 2, 14336, 0, 1, 0)
    ws = lib.moe_workspace_size(ctypes.byref(d))
    R = 4096 * 2
    assert ws >= R * 4096 * 2 * 2 + R * 14336 * 2  # Xe + Ye + H at least
    bad = moe.LayerDesc(4096, 4096, 8, 2, 14336, 0, 1, 0x10)  # unknown flag bits
    assert lib.moe_workspace_size(ctypes.byref(bad)) == 0
    # dispatch chunks live inside the fused FFN launch only
    lone = moe.LayerDesc(4096, 4096, 8, 2, 14336, 0, 1, moe.LAYER_FUSED_DISPATCH)
    assert lib.moe_workspace_size(ctypes.byref(lone)) == 0
    for ok in (moe.LAYER_PIPELINE, moe.LAYER_FUSED_COMBINE,
               moe.LAYER_FUSED_FFN | moe.LAYER_FUSED_COMBINE):
        good = moe.LayerDesc(4096, 4096, 8, 2, 14336, 0, 1, ok)
        assert lib.moe_workspace_size(ctypes.byref(good)) == ws  # one workspace serves all
    p = ctypes.c_void_p(0x10000)
    # both logits and Wr given
    assert lib.moe_layer_forward(ctypes.byref(d), p, p, p, p, p, p, N, N, N, p, ws, N) == INVALID
    # short workspace
    assert lib.moe_layer_forward(ctypes.byref(d), p, p, N, p, p, p, N, N, N, p, ws - 1,
                                 N) == INVALID
    assert lib.moe_layer_forward(N, p, p, N, p, p, p, N, N, N, p, ws, N) == INVALID


def test_launch_count(lib):
    # bf16: router, route (with the layout's ranking), dispatch, 2 GEMMs, combine
    d = moe.LayerDesc(4096, 4096, 8, 2, 14336, 0, 1, 0)
    assert lib.moe_kernel_launches_per_forward(ctypes.byref(d), 1) == 6
    assert lib.moe_kernel_launches_per_forward(ctypes.byref(d), 0) == 5
    # 256 experts: the separate layout (two kernels past 4096 slots)
    d4 = moe.LayerDesc(8192, 7168, 256, 8, 2048, 1, 1, 0)
    assert lib.moe_kernel_launches_per_forward(ctypes.byref(d4), 0) == 7
    # FP8: the separate layout kernel, absmax + dispatch
    assert lib.moe_kernel_launches_per_forward_fp8(ctypes.byref(d), 1) == 8
    assert lib.moe_kernel_launches_per_forward_fp8(ctypes.byref(d4), 0) == 8
    # gathering: the separate layout, no dispatch kernel
    dg = moe.LayerDesc(4096, 4096, 8, 2, 14336, 0, 1, moe.LAYER_GATHER_ON_LOAD)
    assert lib.moe_kernel_launches_per_forward(ctypes.byref(dg), 1) == 6
    assert lib.moe_kernel_launches_per_forward_fp8(ctypes.byref(dg), 1) == 8  # absmax + quantise
    # the pipeline: route, layout, one persistent FFN (dispatch, GEMMs, combine)
    dp = moe.LayerDesc(4096, 4096, 8, 2, 14336, 0, 1, moe.LAYER_PIPELINE)
    assert lib.moe_kernel_launches_per_forward(ctypes.byref(dp), 1) == 4
    # the layout's one-CTA path: up to 8192 slots with at most 32 experts, 4096 otherwise
    for T, E, one_cta in [(4096, 8, True), (4097, 8, False), (2048, 64, True), (2049, 64, False)]:
        dl = moe.LayerDesc(T, 256, E, 2, 256, 0, 1, moe.LAYER_GATHER_ON_LOAD)
        # router, route, layout (1 or 2), GEMM-1 (gathering), GEMM-2, combine
        assert lib.moe_kernel_launches_per_forward(ctypes.byref(dl), 1) == (6 if one_cta else 7)
        assert (lib.moe_layout_workspace_size(T, E, 2) == 0) == one_cta


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(moe, "_lib", None)
    monkeypatch.setattr(moe, "_LIB_PATH", str(tmp_path / "libmoe.so"))
    with pytest.raises(moe.MoeError):
        moe.load_library()


def test_fp8_calls_check_on_the_host(lib):
    p = ctypes.c_void_p(0x10000)
    # FP8 rows of codes must be 16-byte aligned: d, K, cols multiples of 16
    assert lib.moe_dispatch_fp8(p, p, 4, 72, 2, p, p, N) == UNSUPPORTED
    assert "multiple of 16" in _err(lib)
    assert lib.moe_expert_gemm_fp8(p, p, p, p, p, 8, 16, 64, 40, 1, p, N) == UNSUPPORTED
    assert lib.moe_quantize_experts_fp8(p, 8, 64, 24, p, p, N) == UNSUPPORTED
    assert lib.moe_expert_gemm_fp8(p, N, p, p, p, 8, 16, 64, 64, 1, p, N) == INVALID  # no a_scale
    assert lib.moe_quantize_experts_fp8(p, 0, 64, 64, p, p, N) == INVALID
    d = moe.LayerDesc(4096, 4096, 8, 2, 14336, 0, 1, 0)
    ws = lib.moe_workspace_size(ctypes.byref(d))
    assert lib.moe_layer_forward_fp8(ctypes.byref(d), p, p, N, p, N, p, p, N, N, N, p, ws,
                                     N) == INVALID                        # no w1_scale
    assert lib.moe_layer_forward_fp8(ctypes.byref(d), p, p, N, p, p, p, p, N, N, N, p, ws - 1,
                                     N) == INVALID                        # short workspace
    d72 = moe.LayerDesc(64, 72, 8, 2, 128, 0, 1, 0)
    ws72 = lib.moe_workspace_size(ctypes.byref(d72))
    assert lib.moe_layer_forward_fp8(ctypes.byref(d72), p, p, N, p, p, p, p, N, N, N, p, ws72,
                                     N) == UNSUPPORTED
    # the quantising dispatch adds one kernel (the absmax reduction)
    assert lib.moe_kernel_launches_per_forward_fp8(ctypes.byref(d), 1) == 8


def test_fused_ffn_checks_on_the_host(lib):
    p = ctypes.c_void_p(0x10000)
    need = lib.moe_expert_ffn_fused_workspace_size(8, 8192)
    assert need >= (8192 // 256 + 8) * 4
    assert lib.moe_expert_ffn_fused(p, p, p, p, 8, 8192, 4096, 14336, p, p, p, need - 1,
                                    N) == INVALID
    assert "workspace" in _err(lib)
    assert lib.moe_expert_ffn_fused_fp8(p, p, p, p, p, p, 8, 64, 72, 256, p, p, p, need,
                                        N) == UNSUPPORTED                 # d % 16 for FP8
    both = moe.LayerDesc(64, 128, 8, 2, 256, 0, 1,
                         moe.LAYER_GATHER_ON_LOAD | moe.LAYER_FUSED_FFN)
    ws = lib.moe_workspace_size(ctypes.byref(moe.LayerDesc(64, 128, 8, 2, 256, 0, 1, 0)))
    assert lib.moe_layer_forward(ctypes.byref(both), p, p, N, p, p, p, N, N, N, p, ws,
                                 N) == UNSUPPORTED
    fused = moe.LayerDesc(4096, 4096, 8, 2, 14336, 0, 1, moe.LAYER_FUSED_FFN)
    assert lib.moe_kernel_launches_per_forward(ctypes.byref(fused), 1) == 5  # one GEMM launch
    assert lib.moe_kernel_launches_per_forward_fp8(ctypes.byref(fused), 1) == 7


def test_host_batches_reject_bad_arguments(lib):
    d = moe.LayerDesc(64, 128, 8, 2, 256, 0, 1, 0)
    need = lib.moe_host_workspace_size(ctypes.byref(d), 1)
    assert need > lib.moe_workspace_size(ctypes.byref(d))  # two buffer sets on top
    p = ctypes.c_void_p(0x10000)
    arr = (ctypes.c_void_p * 2)(0x10000, 0x20000)
    zero = (ctypes.c_void_p * 2)(0x10000, 0)
    args = lambda n, X, L, Wr, Y, ws: (ctypes.byref(d), n, X, L, Wr, p, N, p, Y, p, ws, N)  # noqa
    assert lib.moe_layer_forward_host(*args(-1, arr, arr, N, arr, need)) == INVALID
    assert lib.moe_layer_forward_host(*args(2, arr, arr, p, arr, need)) == INVALID  # both routers
    assert lib.moe_layer_forward_host(*args(2, zero, arr, N, arr, need)) == INVALID  # NULL batch
    assert "batch 1" in _err(lib)
    assert lib.moe_layer_forward_host(*args(2, arr, arr, N, arr, need - 1)) == INVALID
    assert "workspace" in _err(lib)
    assert lib.moe_layer_forward_host(*args(0, N, N, N, N, 0)) == OK  # nothing to do


def test_workspace_holds_the_split_routers_partial_logits(lib):
    """At T <= 64 with up to 32 experts the layer's router writes one partial
    logit per 256-column slice (summed by the routing kernel), so the
    workspace holds slices * T * E floats there and not past either limit."""
    def ws(T, d, E):
        return lib.moe_workspace_size(ctypes.byref(moe.LayerDesc(T, d, E, 2, 256, 0, 1, 0)))
    part = 16 * 64 * 32 * 4  # d = 4096: 16 slices, 64 tokens, 32 experts
    # a 33rd expert adds a few hundred bytes of per-expert data but drops the partials
    assert part - 4096 < ws(64, 4096, 32) - ws(64, 4096, 33) <= part
    # a 65th token adds one token's buffers like a 64th does, but drops the
    # 16 * 64 * 8 floats of partials of an 8-expert layer
    step64 = ws(64, 4096, 8) - ws(63, 4096, 8)
    step65 = ws(65, 4096, 8) - ws(64, 4096, 8)
    assert abs((step64 - step65) - 16 * 64 * 8 * 4) <= 4096
