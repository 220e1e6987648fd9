"""The fused prefill + gated tail (gdn_prefill_chunked_gated_nvfp4) against the two-call path
it stands for: prefill with bf16 o, then gated RMSNorm + NVFP4 encode of that o. The fused
output pass normalises and encodes the same bf16 o rows with the same arithmetic, so codes,
block scales, o and the final state must agree bit for bit. The two-call path itself is held to
the oracle by test_gpu_scan.py and test_gpu_tail.py."""
import numpy as np
import pytest
import torch

import workloads
from helpers import dev, upload_scan_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import gated_deltanet_03_b200 as lib
    return lib


def _run_both(g, w, gs=None):
    x = workloads.generate(w)
    inp = upload_scan_inputs(x, True)
    cu = inp.pop("cu_seqlens") if w.num_seqs > 1 else None
    inp.pop("cu_seqlens", None)
    S0 = inp.pop("initial_state")
    z = dev(x["z"], torch.bfloat16)
    nw = dev(x["norm_weight"], torch.float32)
    if gs is None:
        gs = 448.0 * 6.0 / 4.0
    o_ref, S_ref = g.gdn_prefill_chunked(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["A_log"],
                                         inp["dt_bias"], cu_seqlens=cu, initial_state=S0,
                                         out_dtype=torch.bfloat16)
    xq_ref, xs_ref = g.gdn_gated_rmsnorm_silu_nvfp4(o_ref, z, nw, gs)
    xq, xs, S, o = g.gdn_prefill_chunked_gated_nvfp4(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"],
                                                     inp["A_log"], inp["dt_bias"], z, nw, gs, cu_seqlens=cu,
                                                     initial_state=S0, write_o=True)
    xq2, xs2, _, o2 = g.gdn_prefill_chunked_gated_nvfp4(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"],
                                                        inp["A_log"], inp["dt_bias"], z, nw, gs, cu_seqlens=cu,
                                                        initial_state=S0)
    torch.cuda.synchronize()
    assert g.gdn_get_device_status() == 0
    assert o2 is None
    return dict(xq=(xq, xq_ref, xq2), xs=(xs, xs_ref, xs2), S=(S, S_ref), o=(o, o_ref))


def _check(r):
    for key in ("xq", "xs"):
        got, ref, got_no_o = (t.cpu().numpy() for t in r[key])
        np.testing.assert_array_equal(got, ref)
        np.testing.assert_array_equal(got_no_o, ref)
    np.testing.assert_array_equal(r["S"][0].cpu().numpy(), r["S"][1].cpu().numpy())
    np.testing.assert_array_equal(r["o"][0].view(torch.int16).cpu().numpy(),
                                  r["o"][1].view(torch.int16).cpu().numpy())


@pytest.mark.parametrize("seqlens,Hk,Hv", [
    ((300,), 2, 4),              # one sequence, ragged last chunk
    ((1, 63, 64, 65, 200), 2, 2),  # several sequences, lengths around the chunk size
    ((700, 129), 1, 3),          # GQA 1:3, several chunks per sequence
])
def test_fused_equals_two_call(g, seqlens, Hk, Hv):
    w = workloads.custom("fused_%d" % sum(seqlens), seqlens, Hk, Hv, 128, s0_std=0.1, seed=sum(seqlens))
    _check(_run_both(g, w))


def test_fused_equals_two_call_segmented(g):
    """Long enough that the chain is cut into segments (state / transition passes, combine)."""
    w = workloads.custom("fused_long", (6000, 2000), 2, 4, 128, s0_std=0.1, seed=11)
    _check(_run_both(g, w))


def test_fused_equals_two_call_benchmark_workload(g):
    _check(_run_both(g, workloads.PREFILL_1K, gs=448.0 * 6.0 / 3.0))


def test_fused_rejects_unsupported(g):
    w = workloads.custom("fused_small_d", (64,), 1, 1, 64, seed=3)
    x = workloads.generate(w)
    inp = upload_scan_inputs(x, True)
    z = dev(x["z"], torch.bfloat16)
    nw = dev(x["norm_weight"], torch.float32)
    with pytest.raises(g.GdnError) as e:
        g.gdn_prefill_chunked_gated_nvfp4(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["A_log"],
                                          inp["dt_bias"], z, nw, 1.0)
    assert e.value.status == g.GDN_ERR_UNSUPPORTED


@pytest.mark.parametrize("B,Hk,Hv", [(3, 1, 2), (256, 16, 32)])
def test_fused_decode_equals_decode_then_tail(g, B, Hk, Hv):
    """gdn_decode_step_gated_nvfp4 against gdn_decode_step (bf16 o) followed by
    gdn_gated_rmsnorm_silu_nvfp4 on that o: the same state, o, codes and block scales, bit for bit
    (the batched-decode shape and a small one)."""
    w = workloads.custom("fd", (1,) * B, Hk, Hv, 128, io="bf16", s0_std=0.1, seed=400 + B, kind="decode")
    x = workloads.generate(w)
    d = upload_scan_inputs(x, True)
    z = dev(x["z"], torch.bfloat16)
    nw = dev(x["norm_weight"], torch.float32)
    gs = 448.0 * 6.0 / 5.0
    st_ref = d["initial_state"].clone()
    o_ref = g.gdn_decode_step(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], st_ref)
    xq_ref, xs_ref = g.gdn_gated_rmsnorm_silu_nvfp4(o_ref, z, nw, gs)
    st = d["initial_state"].clone()
    o = torch.empty_like(o_ref)
    xq, xs, _ = g.gdn_decode_step_gated_nvfp4(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], st,
                                              z, nw, gs, o=o)
    torch.cuda.synchronize()
    assert g.gdn_get_device_status() == 0
    assert torch.equal(st, st_ref)
    assert torch.equal(o, o_ref)
    assert torch.equal(xq, xq_ref) and torch.equal(xs, xs_ref)
    # without the o output
    st2 = d["initial_state"].clone()
    xq2, xs2, _ = g.gdn_decode_step_gated_nvfp4(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                                                st2, z, nw, gs)
    assert torch.equal(xq2, xq_ref) and torch.equal(xs2, xs_ref) and torch.equal(st2, st_ref)
