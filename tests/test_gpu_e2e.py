"""End-to-end parity of the whole layer path, per workload: the library's entry points called in
the order the benchmark calls them (scan -> gated RMSNorm * SiLU(z) -> NVFP4 encode -> NVFP4 W4A4
output projection), checked link by link against the oracle on the same seeded inputs, and the
projected output checked against the exact layer output.

"Red Lite dev15d - DeltaNet gated tail + Q4_K output projection", section "Field gate": every
normalised value and every projected output of the tail must agree between the two
implementations. The NVFP4 encode is a step function: a relative change of 1e-6 in o already
moves an E4M3 block scale across a rounding boundary somewhere in a 4096 x 2048 activation and
shifts the projected output by about 1e-2 of its largest value, so two correct implementations
whose scans differ in the last bits cannot be held to 1e-2 on the quantised output itself. The
chain is therefore checked where each link has a sharp bound:
  1. o (bf16) against the fp64 oracle scan: 2e-3 + 2^-8 (the bf16 storage rounding);
  2. the gated tail on that o against the oracle's tail: 1e-5 + 2^-8;
  3. the NVFP4 codes and block scales of that bf16 y against the oracle's encode of the same
     tensor: bit for bit; the fused tail and the fused prefill give the same bytes;
  4. the GEMM on those codes against the oracle's fp64 GEMM of the same codes: 1e-2;
  5. the projected output against the exact (unquantised, fp64) layer output: no further from
     it than the oracle pipeline's own output is (the W4A4 error, about 13 % here), within 2 % of
     that error in the Frobenius norm and 10 % in the largest element, and within 3e-2 of the
     oracle pipeline's output in the Frobenius norm (the oracle pipeline itself moves by 2.4e-2
     when o is perturbed by its 2e-3 bound).
Every row is checked for the tiny, 1024-wide prefill and batched-decode workloads; 256 sampled
rows (each sequence's last row among them) for the long and variable-length prefills."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import TOL_GEMM, TOL_SCAN_BF16_OUT, TOL_TAIL_BF16_OUT, dev, rel_err, to_np, upload_scan_inputs

pytestmark = pytest.mark.gpu

FRO_EXACT_FACTOR = 1.02
MAX_EXACT_FACTOR = 1.10
FRO_VS_ORACLE = 3e-2


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import gated_deltanet_03_b200 as lib
    return lib


def _fro(a):
    return float(np.sqrt(np.square(np.asarray(a, np.float64)).sum()))


def _oracle_scan(x):
    o_ref, S_ref = oracle.gdn_scan(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                                   cu_seqlens=x["cu_seqlens"], initial_state=x["initial_state"])
    return o_ref, S_ref


def _check_layer(g, x, o_ref, o_dev, z_dev, rows, bf16_io):
    """Links 1-5 for the rows `rows`, given the path's o on the device. Returns the fused-tail
    codes (for the fused prefill's bit-for-bit check) and the global scale used."""
    nw = dev(x["norm_weight"], torch.float32)
    M = o_dev.shape[0]
    # 1. the scan's output
    o_np = to_np(o_dev)
    tol_o = TOL_SCAN_BF16_OUT if o_dev.dtype == torch.bfloat16 else 2e-3
    assert rel_err(o_np[rows], o_ref[rows]) <= tol_o
    # activation global scale from the oracle pipeline's y over every row (the calibration pass),
    # shared by both sides
    o_in = workloads.round_bf16(o_ref.astype(np.float32)) if bf16_io else o_ref.astype(np.float32)
    y_ref_all = workloads.round_bf16(oracle.gated_rmsnorm_silu(o_in, x["z"], x["norm_weight"]).astype(np.float32))
    gx = np.float32(448.0 * 6.0 / max(float(np.abs(y_ref_all).max()), 1e-30))
    # 2. the gated tail on the path's own o
    y_dev = g.gdn_gated_rmsnorm_silu(o_dev, z_dev, nw, out_dtype=torch.bfloat16)
    y_np = to_np(y_dev)
    y_chk = oracle.gated_rmsnorm_silu(o_np[rows].astype(np.float32), x["z"][rows], x["norm_weight"])
    assert rel_err(y_np.reshape(M, -1)[rows], y_chk) <= TOL_TAIL_BF16_OUT
    # 3. encode: the standalone encoder and the fused tail against the oracle's encode of that y
    xq, xs = g.nvfp4_quantize_act(y_dev.reshape(M, -1), float(gx))
    xq_f, xs_f = g.gdn_gated_rmsnorm_silu_nvfp4(o_dev, z_dev, nw, float(gx))
    assert torch.equal(xq, xq_f) and torch.equal(xs, xs_f)
    xq_o, xs_o = oracle.nvfp4_quantize(y_np.reshape(M, -1)[rows], gx)
    np.testing.assert_array_equal(xq.cpu().numpy()[rows], xq_o)
    np.testing.assert_array_equal(xs.cpu().numpy()[rows], xs_o)
    # 4. the GEMM on those codes
    W = x["proj_weight"]
    gw = np.float32(448.0 * 6.0 / np.abs(W).max())
    wq, ws = g.nvfp4_quantize_act(dev(W, torch.bfloat16), float(gw))
    wq_o, ws_o = oracle.nvfp4_quantize(W, gw)
    np.testing.assert_array_equal(wq.cpu().numpy(), wq_o)
    Y = to_np(g.nvfp4_gemm(xq, xs, wq, ws, float(np.float32(1.0) / (gx * gw)), out_dtype=torch.float32))[rows]
    assert rel_err(Y, oracle.nvfp4_gemm(xq_o, xs_o, gx, wq_o, ws_o, gw)) <= TOL_GEMM
    # 5. against the exact layer output, beside the oracle pipeline's own quantised output
    y_ref = y_ref_all[rows]
    xq_r, xs_r = oracle.nvfp4_quantize(y_ref, gx)
    Y_ref = oracle.nvfp4_gemm(xq_r, xs_r, gx, wq_o, ws_o, gw)
    y_exact = oracle.gated_rmsnorm_silu(o_ref[rows].astype(np.float32), x["z"][rows], x["norm_weight"])
    Y_exact = y_exact @ W.astype(np.float64).T
    e_fro, e_fro_ref = _fro(Y - Y_exact) / _fro(Y_exact), _fro(Y_ref - Y_exact) / _fro(Y_exact)
    e_max, e_max_ref = rel_err(Y, Y_exact), rel_err(Y_ref, Y_exact)
    assert e_fro <= FRO_EXACT_FACTOR * e_fro_ref, (e_fro, e_fro_ref)
    assert e_max <= MAX_EXACT_FACTOR * e_max_ref, (e_max, e_max_ref)
    assert _fro(Y - Y_ref) / _fro(Y_ref) <= FRO_VS_ORACLE
    torch.cuda.synchronize()
    assert g.gdn_get_device_status() == 0
    return xq_f, xs_f, gx


def _prefill_e2e(g, w, x, rows):
    o_ref, _ = _oracle_scan(x)
    bf16 = w.io == "bf16"
    dt = torch.bfloat16 if bf16 else torch.float32
    d = upload_scan_inputs(x, bf16)
    cu = d["cu_seqlens"] if w.num_seqs > 1 else None
    z = dev(x["z"], dt)
    o, _ = g.gdn_prefill_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], cu_seqlens=cu,
                                 initial_state=d["initial_state"], out_dtype=dt)
    xq_f, xs_f, gx = _check_layer(g, x, o_ref, o, z, rows, bf16)
    if w.D == 128 and bf16:
        # the fused prefill (scan + gated tail + encode in its output pass): the same bytes
        xq, xs, _, _ = g.gdn_prefill_chunked_gated_nvfp4(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"],
                                                         d["dt_bias"], z, dev(x["norm_weight"], torch.float32),
                                                         float(gx), cu_seqlens=cu, initial_state=d["initial_state"])
        assert torch.equal(xq, xq_f) and torch.equal(xs, xs_f)


def test_e2e_tiny(g):
    """Tiny workload (T = 64, 2 heads, d = 16, fp32): out_proj 32 -> 16, every row."""
    w = workloads.TINY
    _prefill_e2e(g, w, workloads.generate(w), np.arange(w.T))


def test_e2e_prefill_1024_wide(g):
    """1024-wide layer (T = 4096, 16/16 heads): out_proj 2048 -> 1024, every row."""
    w = workloads.PREFILL_1K
    _prefill_e2e(g, w, workloads.generate(w), np.arange(w.T))


@pytest.mark.parametrize("wl", [workloads.PREFILL_LONG, workloads.VARLEN_8], ids=lambda w: w.name)
def test_e2e_long_and_varlen_sampled_rows(g, wl):
    """27B-class long prefill (T = 32768) and the variable-length batch: out_proj 4096 -> 2048
    on 256 sampled rows, each sequence's last row among them."""
    x = workloads.generate(wl)
    rng = np.random.default_rng(11)
    ends = np.asarray(x["cu_seqlens"][1:], np.int64) - 1
    rows = np.unique(np.concatenate([rng.integers(0, wl.T, size=256 - len(ends)), ends]))
    _prefill_e2e(g, wl, x, rows)


def test_e2e_batched_decode(g):
    """Batched decode (256 sequences, one token each, state [256, 32, 128, 128] in place):
    decode step -> gated tail + encode -> out_proj 4096 -> 2048 at M = 256, every row."""
    w = workloads.DECODE_B256
    x = workloads.generate(w)
    o_ref, S_ref = _oracle_scan(x)
    d = upload_scan_inputs(x, True)
    state = d["initial_state"].clone()
    o = g.gdn_decode_step(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], state)
    assert rel_err(to_np(state), S_ref) <= 2e-3
    _check_layer(g, x, o_ref, o, dev(x["z"], torch.bfloat16), np.arange(w.T), True)
