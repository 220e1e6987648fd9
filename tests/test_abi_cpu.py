"""The C-ABI library builds, loads without a GPU, exports every entry point include/gdn.h
declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "gdn.h")).read()
    return re.findall(r"GDN_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(_declared())
    for n in ("gdn_prefill_chunked", "gdn_decode_step", "gdn_gated_rmsnorm_silu",
              "nvfp4_quantize_act", "nvfp4_gemm"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import gated_deltanet_03_b200 as g
    lib = ctypes.CDLL(g.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(g.ABI_SYMBOLS) >= set(_declared())


def test_status_strings_and_version():
    import gated_deltanet_03_b200 as g
    assert g.LIB.gdn_version() >= 100
    assert g.status_string(0) == "ok"
    assert "timed out" in g.status_string(4)


def test_host_validation_rejects_bad_arguments_without_cuda():
    import gated_deltanet_03_b200 as g
    L = g.LIB
    P = None
    # Hv not a multiple of Hk
    assert L.gdn_prefill_chunked(P, P, P, P, P, P, P, P, 1, 8, 3, 4, 128, 128, 1.0, 1, 0, P, P, P, 0, P,
                                 0, P) == g.GDN_ERR_INVALID_ARG
    # several sequences without cu_seqlens
    assert L.gdn_prefill_chunked(P, P, P, P, P, P, P, P, 2, 8, 2, 4, 128, 128, 1.0, 1, 0, P, P, P, 0, P,
                                 0, P) == g.GDN_ERR_INVALID_ARG
    # more chunk slots than the prep grid's y dimension holds (T / 64 + num_seqs > 65535): refused
    # on the host, before any pointer is touched (the pointers are aligned placeholders)
    A = 1 << 20
    T_big = 64 * 65535
    assert L.gdn_prefill_chunked(A, A, A, A, A, A, A, P, 1, T_big, 16, 32, 128, 128, 1.0, 1, 0, P, P, A, 0,
                                 A, 1 << 40, P) == g.GDN_ERR_UNSUPPORTED
    # unsupported head size
    assert L.gdn_decode_step(P, P, P, P, P, P, P, 4, 1, 1, 96, 96, 1.0, 1, 0, P, P, 0,
                             P) == g.GDN_ERR_UNSUPPORTED
    # Dk != Dv
    assert L.gdn_decode_step(P, P, P, P, P, P, P, 4, 1, 1, 64, 128, 1.0, 1, 0, P, P, 0,
                             P) == g.GDN_ERR_UNSUPPORTED
    # null pointers with work to do
    assert L.gdn_decode_step(P, P, P, P, P, P, P, 4, 1, 1, 128, 128, 1.0, 1, 0, P, P, 0,
                             P) == g.GDN_ERR_INVALID_ARG
    # bad dtype code
    assert L.gdn_gated_rmsnorm_silu(P, P, P, 1e-6, 4, 2, 128, 7, P, 0, P) == g.GDN_ERR_INVALID_ARG
    # quantiser: K not a multiple of 32, non-positive global scale
    assert L.nvfp4_quantize_act(P, 0, 4, 48, 1.0, P, P, P) == g.GDN_ERR_UNSUPPORTED
    assert L.nvfp4_quantize_act(P, 0, 4, 64, 0.0, P, P, P) == g.GDN_ERR_INVALID_ARG
    assert L.nvfp4_quantize_act(P, 0, 4, 64, float("nan"), P, P, P) == g.GDN_ERR_INVALID_ARG
    # GEMM: N not a multiple of 16
    assert L.nvfp4_gemm(P, P, P, P, 1.0, 4, 24, 64, 0, P, P) == g.GDN_ERR_UNSUPPORTED
    # empty problems are no-ops
    assert L.nvfp4_gemm(P, P, P, P, 1.0, 0, 32, 64, 0, P, P) == g.GDN_OK
    assert L.gdn_decode_step(P, P, P, P, P, P, P, 0, 1, 1, 128, 128, 1.0, 1, 0, P, P, 0, P) == g.GDN_OK


def test_workspace_query_is_host_only():
    import gated_deltanet_03_b200 as g
    assert g.gdn_prefill_workspace_bytes(4096, 1, 16, 16, 128, 128) >= 0


@pytest.mark.parametrize("T,Hk,Hv,seg", [(32768, 16, 32, 57), (16384, 16, 32, 29), (4096, 16, 16, 8)])
def test_workspace_follows_the_segment_plan(T, Hk, Hv, seg):
    """The workspace holds one 82,944-byte item per (value head, chunk slot) and one
    196,608-byte segment item per (value head, segment slot), T / (64 L) + num_seqs slots for a
    segment length of L chunks. The host plans L from its cost model: 57 chunks at T = 32768 with
    32 value heads (288 output-pass CTAs, two whole waves on 148 SMs), 29 at T = 16384, 8 at
    T = 4096 with 16 heads."""
    import gated_deltanet_03_b200 as g
    expect = Hv * (T // 64 + 1) * 82944 + Hv * (T // (64 * seg) + 1) * 196608
    assert g.gdn_prefill_workspace_bytes(T, 1, Hk, Hv, 128, 128) == expect


def test_short_conv_host_validation():
    """Every case is rejected (or is a no-op) on the host, so nothing is launched; the fake
    addresses are never dereferenced."""
    import gated_deltanet_03_b200 as g
    L = g.LIB
    P = None
    X, W, Y, S = 0x10000, 0x20000, 0x30000, 0x40000
    parts3 = (ctypes.c_int32 * 3)(64, 64, 128)
    bad_sum = (ctypes.c_int32 * 3)(64, 64, 120)
    bad_mult = (ctypes.c_int32 * 3)(60, 68, 128)
    # width 5 is beyond the supported 1..4; channels not a multiple of 8
    assert L.gdn_short_conv1d_silu(X, 256, W, P, 1, 8, 256, 5, P, P, Y, P, 0, P) == g.GDN_ERR_UNSUPPORTED
    assert L.gdn_short_conv1d_silu(X, 256, W, P, 1, 8, 252, 4, P, P, Y, P, 0, P) == g.GDN_ERR_UNSUPPORTED
    # tokens not divisible into num_seqs equal runs without cu_seqlens; ldx < C; null output
    assert L.gdn_short_conv1d_silu(X, 256, W, P, 3, 8, 256, 4, P, P, Y, P, 0, P) == g.GDN_ERR_INVALID_ARG
    assert L.gdn_short_conv1d_silu(X, 128, W, P, 1, 8, 256, 4, P, P, Y, P, 0, P) == g.GDN_ERR_INVALID_ARG
    assert L.gdn_short_conv1d_silu(X, 256, W, P, 1, 8, 256, 4, P, P, P, P, 0, P) == g.GDN_ERR_INVALID_ARG
    # plane widths that do not sum to C or are not multiples of 8; too many planes
    assert L.gdn_short_conv1d_silu(X, 256, W, P, 1, 8, 256, 4, P, P, Y, bad_sum, 3, P) == g.GDN_ERR_INVALID_ARG
    assert L.gdn_short_conv1d_silu(X, 256, W, P, 1, 8, 256, 4, P, P, Y, bad_mult, 3, P) == g.GDN_ERR_INVALID_ARG
    assert L.gdn_short_conv1d_silu(X, 256, W, P, 1, 8, 256, 4, P, P, Y, parts3, 5, P) == g.GDN_ERR_INVALID_ARG
    # misaligned input; final state overlapping the input or the output
    assert L.gdn_short_conv1d_silu(X + 2, 256, W, P, 1, 8, 256, 4, P, P, Y, P, 0, P) == g.GDN_ERR_INVALID_ARG
    assert L.gdn_short_conv1d_silu(X, 256, W, P, 1, 8, 256, 4, P, X + 1024, Y, P, 0, P) == g.GDN_ERR_INVALID_ARG
    assert L.gdn_short_conv1d_silu(X, 256, W, P, 1, 8, 256, 4, P, Y, Y, parts3, 3, P) == g.GDN_ERR_INVALID_ARG
    # nothing to do: no tokens and no state requested; width 1 has no state
    assert L.gdn_short_conv1d_silu(P, 256, W, P, 1, 0, 256, 4, P, P, P, P, 0, P) == g.GDN_OK
    assert L.gdn_short_conv1d_silu(P, 256, W, P, 1, 0, 256, 1, P, S, P, P, 0, P) == g.GDN_OK
    # decode: missing or overlapping state, unsupported width, empty batch
    assert L.gdn_short_conv1d_silu_decode(X, 256, W, 4, 256, 4, P, Y, P, 0, P) == g.GDN_ERR_INVALID_ARG
    assert L.gdn_short_conv1d_silu_decode(X, 256, W, 4, 256, 4, Y, Y, P, 0, P) == g.GDN_ERR_INVALID_ARG
    assert L.gdn_short_conv1d_silu_decode(X, 256, W, 4, 256, 5, S, Y, P, 0, P) == g.GDN_ERR_UNSUPPORTED
    assert L.gdn_short_conv1d_silu_decode(X, 256, W, 0, 256, 4, S, Y, P, 0, P) == g.GDN_OK
