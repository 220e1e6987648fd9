"""The allocation-free prefill entry point, for callers that cannot allocate device memory
(it uses the library's fixed scratch array instead of a caller workspace), called through the
C ABI and checked against the regular entry point's results on two calls in a row, plus its
host-side rejection of sizes beyond the fixed scratch."""
import ctypes

import pytest
import torch

import workloads
from helpers import TOL_SCAN, rel_err, to_np, upload_scan_inputs

pytestmark = pytest.mark.gpu

GDN_ERR_WORKSPACE = 5


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_static_scratch_prefill_matches_regular_entry_point():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import gated_deltanet_03_b200 as g
    lib = g.LIB
    w = workloads.custom("noalloc", (150, 37, 300), 2, 4, 128, io="bf16", s0_std=0.1, seed=321)
    x = workloads.generate(w)
    d = upload_scan_inputs(x, True)
    N, T, D = w.num_seqs, w.T, w.D
    ref_o, ref_S = g.gdn_prefill_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                                         cu_seqlens=d["cu_seqlens"], initial_state=d["initial_state"],
                                         out_dtype=torch.float32)
    torch.cuda.synchronize()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        o = torch.full((T, w.Hv, D), float("nan"), dtype=torch.float32, device="cuda")
        S = torch.full((N, w.Hv, D, D), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.gdn_prefill_chunked_static_ws(
            _p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["a"]), _p(d["b"]), _p(d["A_log"]), _p(d["dt_bias"]),
            _p(d["cu_seqlens"]), N, T, w.Hk, w.Hv, D, D, 1.0, 1, g.GDN_BF16, _p(d["initial_state"]), _p(S),
            _p(o), g.GDN_F32, stream)
        assert st == 0, g.status_string(st)
        torch.cuda.synchronize()
        assert rel_err(to_np(o), to_np(ref_o)) <= TOL_SCAN
        assert rel_err(to_np(S), to_np(ref_S)) <= TOL_SCAN
    assert g.gdn_get_device_status() == 0
    # a size whose workspace exceeds the fixed scratch is rejected before any launch
    big_T = 1 << 20
    assert g.gdn_prefill_workspace_bytes(big_T, 1, w.Hk, w.Hv, D, D) > 32 << 20
    st = lib.gdn_prefill_chunked_static_ws(
        _p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["a"]), _p(d["b"]), _p(d["A_log"]), _p(d["dt_bias"]), None, 1,
        big_T, w.Hk, w.Hv, D, D, 1.0, 1, g.GDN_BF16, None, None, _p(ref_o), g.GDN_F32, stream)
    assert st == GDN_ERR_WORKSPACE
