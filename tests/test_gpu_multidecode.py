"""Multi-token decode (gdn_decode_verify / gdn_decode_commit) against the oracle: verifying T
draft tokens per sequence equals the token-by-token recurrence over those tokens from the
current state (outputs for every token, the state untouched); committing the first accepted[b]
tokens equals the recurrence over that prefix alone (zero accepted tokens leave the state bit
for bit)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import TOL_SCAN, TOL_SCAN_BF16_OUT, dev, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import gated_deltanet_03_b200 as lib
    return lib


def _setup(B, T, Hk, Hv, D, seed, io="bf16"):
    w = workloads.custom("verify_B%d_T%d" % (B, T), (T,) * B, Hk, Hv, D, io=io, s0_std=0.1, seed=seed)
    x = workloads.generate(w)
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    t = dict(q=dev(x["q"], dt).view(B, T, Hk, D), k=dev(x["k"], dt).view(B, T, Hk, D),
             v=dev(x["v"], dt).view(B, T, Hv, D), a=dev(x["a"], torch.float32).view(B, T, Hv),
             b=dev(x["b"], torch.float32).view(B, T, Hv), A_log=dev(x["A_log"], torch.float32),
             dt_bias=dev(x["dt_bias"], torch.float32))
    return x, t, dev(x["initial_state"], torch.float32)


def _prefix_oracle(x, B, T, m):
    """Oracle state after the first m[b] tokens of each sequence."""
    idx = np.concatenate([np.arange(b * T, b * T + int(m[b])) for b in range(B)]).astype(np.int64)
    cu = np.zeros(B + 1, dtype=np.int32)
    cu[1:] = np.cumsum(m)
    _, S = oracle.gdn_scan(x["q"][idx], x["k"][idx], x["v"][idx], x["a"][idx], x["b"][idx], x["A_log"],
                           x["dt_bias"], cu_seqlens=cu, initial_state=x["initial_state"])
    return S


@pytest.mark.parametrize("B,T,Hk,Hv,D,io", [(6, 5, 2, 4, 128, "bf16"), (3, 8, 1, 2, 64, "f32"),
                                             (4, 2, 2, 2, 16, "bf16")])
def test_verify_matches_recurrence(g, B, T, Hk, Hv, D, io):
    x, t, S = _setup(B, T, Hk, Hv, D, seed=B * 100 + T, io=io)
    S_before = S.clone()
    S_all = torch.empty_like(S)
    o = g.gdn_decode_verify(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], S,
                            final_state=S_all, out_dtype=torch.float32)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.gdn_scan(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                                   cu_seqlens=x["cu_seqlens"], initial_state=x["initial_state"])
    assert rel_err(to_np(o).reshape(o_ref.shape), o_ref) <= TOL_SCAN
    assert rel_err(to_np(S_all), S_ref) <= TOL_SCAN
    assert torch.equal(S, S_before)


@pytest.mark.parametrize("T,io,l2norm", [(2, "bf16", True), (3, "f32", True), (4, "bf16", True), (8, "bf16", True),
                                         (5, "f32", False)])
def test_verify_outputs_only_matches_recurrence(g, T, io, l2norm):
    """Verify without a final state (d = 128, 2..8 tokens: the chunk-form kernel): every output
    against the oracle's token-by-token recurrence, the state untouched, and against the
    token-by-token kernel (the same call with a final state)."""
    B, Hk, Hv, D = 9, 2, 4, 128
    x, t, S = _setup(B, T, Hk, Hv, D, seed=300 + T, io=io)
    scale = 1.0 if l2norm else 0.125
    if not l2norm:   # raw q and k: keep the products of unit scale
        for key in ("q", "k"):
            t[key] = t[key] / float(np.sqrt(D))
            x[key] = to_np(t[key].float()).reshape(x[key].shape)
    S_before = S.clone()
    o = g.gdn_decode_verify(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], S, scale=scale,
                            qk_l2norm=l2norm, out_dtype=torch.float32)
    S_all = torch.empty_like(S)
    o_seq = g.gdn_decode_verify(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], S, scale=scale,
                                qk_l2norm=l2norm, final_state=S_all, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert g.gdn_get_device_status() == 0
    assert torch.equal(S, S_before)
    o_ref, _ = oracle.gdn_scan(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                               cu_seqlens=x["cu_seqlens"], initial_state=x["initial_state"], scale=scale,
                               qk_l2norm=l2norm)
    assert rel_err(to_np(o).reshape(o_ref.shape), o_ref) <= TOL_SCAN
    assert rel_err(to_np(o), to_np(o_seq)) <= TOL_SCAN


def test_commit_takes_the_accepted_prefix(g):
    B, T, Hk, Hv, D = 7, 6, 2, 4, 128
    x, t, S = _setup(B, T, Hk, Hv, D, seed=77)
    S0 = S.clone()
    accepted_host = np.array([0, 1, 3, 6, 2, 9, -1], dtype=np.int32)   # 9 and -1 clamp to 6 and 0
    o = g.gdn_decode_verify(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], S)
    g.gdn_decode_commit(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], S,
                        dev(accepted_host, torch.int32))
    torch.cuda.synchronize()
    m = np.clip(accepted_host, 0, T)
    S_ref = _prefix_oracle(x, B, T, m)
    got = to_np(S)
    for b in range(B):
        if m[b] == 0:
            assert torch.equal(S[b], S0[b])
        else:
            assert rel_err(got[b], S_ref[b]) <= TOL_SCAN, b
    o_ref, _ = oracle.gdn_scan(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                               cu_seqlens=x["cu_seqlens"], initial_state=x["initial_state"])
    assert rel_err(to_np(o).reshape(o_ref.shape), o_ref) <= TOL_SCAN_BF16_OUT


def test_commit_all_equals_verify_final_state(g):
    B, T, Hk, Hv, D = 5, 4, 2, 2, 128
    _, t, S = _setup(B, T, Hk, Hv, D, seed=5)
    S_all = torch.empty_like(S)
    g.gdn_decode_verify(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], S, final_state=S_all)
    g.gdn_decode_commit(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], S,
                        torch.full((B,), T, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(S, S_all)


def test_verify_commit_batched_decode_size(g):
    """The batched-decode workload's shape (256 sequences, 16/32 heads, d = 128) with 4 draft
    tokens each: every output and every committed state against the oracle."""
    B, T, Hk, Hv, D = 256, 4, 16, 32, 128
    x, t, S = _setup(B, T, Hk, Hv, D, seed=1234)
    rng = np.random.default_rng(9)
    m = rng.integers(0, T + 1, size=B).astype(np.int32)
    o = g.gdn_decode_verify(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], S)
    g.gdn_decode_commit(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], S, dev(m, torch.int32))
    torch.cuda.synchronize()
    assert g.gdn_get_device_status() == 0
    o_ref, _ = oracle.gdn_scan(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                               cu_seqlens=x["cu_seqlens"], initial_state=x["initial_state"])
    assert rel_err(to_np(o).reshape(o_ref.shape), o_ref) <= TOL_SCAN_BF16_OUT
    S_ref = _prefix_oracle(x, B, T, m)
    assert rel_err(to_np(S), S_ref) <= TOL_SCAN


def test_verify_rejects_bad_arguments(g):
    _, t, S = _setup(2, 3, 1, 1, 128, seed=3)
    with pytest.raises(g.GdnError) as e:
        g.gdn_decode_verify(t["q"], t["k"], t["v"][:, :, :, :96].contiguous(), t["a"], t["b"], t["A_log"],
                            t["dt_bias"], S)
    assert e.value.status == g.GDN_ERR_UNSUPPORTED
