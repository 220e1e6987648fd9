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
