"""Parity of the scan kernels (decode, recurrent prefill, tensor-core chunked prefill) with
the CPU oracle on the same seeded inputs: element by element at sizes the oracle finishes
in seconds (several 64-token chunks and a ragged tail), and on sampled (sequence, head)
units at the full workload sizes, in the launch configuration the benchmark uses."""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import (TOL_SCAN, TOL_SCAN_BF16_OUT, oracle_unit, rel_err, to_np, upload_scan_inputs)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import gated_deltanet_03_b200 as lib
    return lib


def _run_prefill(g, x, w, out_dtype, pass_cu=True):
    d = upload_scan_inputs(x, w.io == "bf16")
    cu = d["cu_seqlens"] if (pass_cu or w.num_seqs > 1) else None
    o, S = g.gdn_prefill_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                                 cu_seqlens=cu, initial_state=d["initial_state"],
                                 out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert g.gdn_get_device_status() == 0
    return to_np(o), to_np(S)


def _full_oracle(x):
    return oracle.gdn_scan(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                           cu_seqlens=x["cu_seqlens"], initial_state=x["initial_state"])


@pytest.mark.parametrize("D", [16, 32, 64, 128])
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_prefill_small_all_head_sizes(g, D, io):
    w = workloads.custom("p", (150,), 2, 4, D, io=io, s0_std=0.1, seed=D)
    x = workloads.generate(w)
    o_ref, S_ref = _full_oracle(x)
    o, S = _run_prefill(g, x, w, torch.float32)
    assert rel_err(o, o_ref) <= TOL_SCAN
    assert rel_err(S, S_ref) <= TOL_SCAN


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 128, 200, 1000])
def test_prefill_chunked_lengths(g, T):
    w = workloads.custom("c", (T,), 2, 4, 128, io="bf16", s0_std=0.1 if T % 2 else 0.0, seed=100 + T)
    x = workloads.generate(w)
    o_ref, S_ref = _full_oracle(x)
    o, S = _run_prefill(g, x, w, torch.float32, pass_cu=bool(T % 3))
    assert rel_err(o, o_ref) <= TOL_SCAN, rel_err(o, o_ref)
    assert rel_err(S, S_ref) <= TOL_SCAN, rel_err(S, S_ref)


def test_prefill_bf16_output(g):
    w = workloads.custom("b", (300,), 2, 2, 128, io="bf16", seed=5)
    x = workloads.generate(w)
    o_ref, S_ref = _full_oracle(x)
    o, S = _run_prefill(g, x, w, torch.bfloat16)
    assert rel_err(o, o_ref) <= TOL_SCAN_BF16_OUT
    assert rel_err(S, S_ref) <= TOL_SCAN


def test_prefill_varlen_ragged(g):
    w = workloads.custom("v", (1, 64, 130, 7, 0, 77), 2, 4, 128, io="bf16", s0_std=0.1, seed=9)
    x = workloads.generate(w)
    o_ref, S_ref = _full_oracle(x)
    o, S = _run_prefill(g, x, w, torch.float32)
    assert rel_err(o, o_ref) <= TOL_SCAN
    assert rel_err(S, S_ref) <= TOL_SCAN
    # the empty sequence returns its initial state unchanged
    np.testing.assert_array_equal(S[4], x["initial_state"][4])


def _many_short_lengths(n, hi, seed):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, hi + 1, size=n)
    lens[::9] = 0          # every ninth sequence empty
    lens[5::11] = 64       # some exactly one chunk
    lens[7::13] = 1        # some a single token
    return tuple(int(x) for x in lens)


@pytest.mark.parametrize("seqlens", [
    _many_short_lengths(120, 100, 31),
    (2500,) + _many_short_lengths(40, 70, 32),
    _many_short_lengths(20, 70, 33) + (1500, 0, 700),
], ids=["120_short", "long_first_then_short", "short_then_long"])
def test_prefill_varlen_many_sequences(g, seqlens):
    """A packed batch of many sequences: most shorter than one 64-token chunk, empties and
    single tokens among them, and one to two long sequences that the batch's segment plan
    (sized from the mean length) cuts into several segments. Every sequence's chunk slots,
    segment bounds and initial state are checked against the oracle's per-sequence scan."""
    w = workloads.custom("m", seqlens, 2, 4, 128, io="bf16", s0_std=0.1, seed=len(seqlens))
    x = workloads.generate(w)
    o_ref, S_ref = _full_oracle(x)
    o, S = _run_prefill(g, x, w, torch.float32)
    assert rel_err(o, o_ref) <= TOL_SCAN, rel_err(o, o_ref)
    assert rel_err(S, S_ref) <= TOL_SCAN, rel_err(S, S_ref)
    for i, L in enumerate(seqlens):
        if L == 0:
            np.testing.assert_array_equal(S[i], x["initial_state"][i])


_DEGENERATE = ["alpha1_beta1", "alpha1_beta0", "same_key_beta1", "same_key", "strong_decay",
               "keys_in_4_directions"]


@pytest.mark.parametrize("case", _DEGENERATE)
def test_prefill_degenerate_gates(g, case):
    """The gates at their limits and keys that repeat: alpha -> 1 (A_log = -30, no decay),
    beta -> 1 (b = 20, each write replaces what the state held along k) or beta -> 0 (b = -20,
    no write), one key for every token, decay of about e^-80 per token (every chunk's exp(G)
    underflows), and keys drawn from four directions plus unit noise. Five 64-token chunks and
    a ragged tail, nonzero initial state."""
    w = workloads.custom("g", (300,), 2, 4, 128, io="bf16", s0_std=0.1, seed=300 + _DEGENERATE.index(case))
    x = workloads.generate(w)
    rng = np.random.default_rng(17)
    T, Hk = x["k"].shape[0], x["k"].shape[1]
    if case.startswith("alpha1"):
        x["A_log"][:] = -30.0
        x["b"][:] = 20.0 if case == "alpha1_beta1" else -20.0
    elif case.startswith("same_key"):
        x["k"][:] = workloads.round_bf16(np.broadcast_to(rng.standard_normal((1, Hk, 128)), x["k"].shape))
        if case == "same_key_beta1":
            x["A_log"][:] = -30.0
            x["b"][:] = 20.0
    elif case == "strong_decay":
        x["a"][:] = 5.0
        x["A_log"][:] = np.log(16.0)
    else:
        basis = rng.standard_normal((4, Hk, 128))
        pick = rng.integers(0, 4, size=T)
        x["k"][:] = workloads.round_bf16(basis[pick] + rng.standard_normal(x["k"].shape))
        x["A_log"][:] = -30.0
        x["b"][:] = 20.0
    o_ref, S_ref = _full_oracle(x)
    o, S = _run_prefill(g, x, w, torch.float32)
    assert rel_err(o, o_ref) <= TOL_SCAN, rel_err(o, o_ref)
    assert rel_err(S, S_ref) <= TOL_SCAN, rel_err(S, S_ref)


@pytest.mark.parametrize("T", [512, 4096])
@pytest.mark.parametrize("noise", [0.2, 0.05])
def test_prefill_concentrated_keys_overwrite(g, T, noise):
    """The overwrite regime ("Why Gated DeltaNet Survives 4-Bit Quantization", abstract,
    mechanism iii: each write replaces the state along the current key) with keys concentrated
    in four directions: key = one of four random directions + noise * N(0, 1), alpha -> 1
    (A_log = -30), beta -> 1 (b = 20), nonzero initial state. Nearly parallel keys make the
    state hold large components along their small differences, which is where a chunked form
    with a low-precision staging loses accuracy; the bound is the stated 2e-3 on fp32 o and S."""
    w = workloads.custom("ck", (T,), 2, 4, 128, io="bf16", s0_std=0.1, seed=700 + T + int(noise * 100))
    x = workloads.generate(w)
    rng = np.random.default_rng(23)
    Hk = x["k"].shape[1]
    basis = rng.standard_normal((4, Hk, 128))
    pick = rng.integers(0, 4, size=T)
    x["k"][:] = workloads.round_bf16(basis[pick] + noise * rng.standard_normal(x["k"].shape))
    x["A_log"][:] = -30.0
    x["b"][:] = 20.0
    o_ref, S_ref = _full_oracle(x)
    o, S = _run_prefill(g, x, w, torch.float32)
    assert rel_err(o, o_ref) <= TOL_SCAN, rel_err(o, o_ref)
    assert rel_err(S, S_ref) <= TOL_SCAN, rel_err(S, S_ref)


def test_prefill_empty_batch_copies_state(g):
    w = workloads.custom("e", (0,), 1, 1, 128, io="bf16", s0_std=0.1, seed=3)
    x = workloads.generate(w)
    o, S = _run_prefill(g, x, w, torch.float32)
    np.testing.assert_array_equal(S, x["initial_state"])


def test_prefill_scale_and_no_l2norm(g):
    """q scale and the caller-normalised mode (qk_l2norm = 0 on unit-norm inputs)."""
    w = workloads.custom("s", (96,), 1, 2, 64, io="f32", seed=21)
    x = workloads.generate(w)
    for key in ("q", "k"):
        x[key] = (x[key] / np.linalg.norm(x[key], axis=-1, keepdims=True)).astype(np.float32)
    o_ref, S_ref = oracle.gdn_scan(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                                   scale=0.25, qk_l2norm=False)
    d = upload_scan_inputs(x, False)
    o, S = g.gdn_prefill_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                                 scale=0.25, qk_l2norm=False)
    assert rel_err(to_np(o), o_ref) <= TOL_SCAN
    assert rel_err(to_np(S), S_ref) <= TOL_SCAN


@pytest.mark.parametrize("D", [16, 64, 128])
def test_decode_step_matches_oracle(g, D):
    B, Hk, Hv = 33, 2, 4
    w = workloads.custom("d", (1,) * B, Hk, Hv, D, io="bf16", s0_std=0.1, seed=40 + D, kind="decode")
    x = workloads.generate(w)
    o_ref, S_ref = _full_oracle(x)
    d = upload_scan_inputs(x, True)
    state = d["initial_state"].clone()
    o = g.gdn_decode_step(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], state,
                          out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert rel_err(to_np(o), o_ref) <= TOL_SCAN
    assert rel_err(to_np(state), S_ref) <= TOL_SCAN


def test_decode_equals_prefill_token_by_token(g):
    """T decode steps reproduce one prefill over the same T tokens."""
    w = workloads.custom("t", (40,), 1, 2, 128, io="bf16", s0_std=0.1, seed=77)
    x = workloads.generate(w)
    d = upload_scan_inputs(x, True)
    o_p, S_p = g.gdn_prefill_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                                     initial_state=d["initial_state"], out_dtype=torch.float32)
    state = d["initial_state"].clone()
    outs = []
    for t in range(40):
        outs.append(g.gdn_decode_step(d["q"][t:t + 1], d["k"][t:t + 1], d["v"][t:t + 1],
                                      d["a"][t:t + 1].contiguous(), d["b"][t:t + 1].contiguous(),
                                      d["A_log"], d["dt_bias"], state, out_dtype=torch.float32))
    o_d = torch.cat(outs)
    assert rel_err(to_np(o_d), to_np(o_p)) <= TOL_SCAN
    assert rel_err(to_np(state), to_np(S_p)) <= TOL_SCAN


# ------------------------------------------------------------- full-size workloads ----

def _sampled_units(w, x, units, o_gpu, S_gpu):
    with ThreadPoolExecutor(max_workers=len(units)) as ex:
        refs = list(ex.map(lambda u: oracle_unit(x, u[0], u[1], w.Hk, w.Hv), units))
    cu = x["cu_seqlens"]
    for (n, h), (o_ref, S_ref) in zip(units, refs):
        sl = slice(int(cu[n]), int(cu[n + 1]))
        e_o = rel_err(o_gpu[sl, h], o_ref)
        e_s = rel_err(S_gpu[n, h], S_ref)
        assert e_o <= TOL_SCAN_BF16_OUT, (n, h, e_o)
        assert e_s <= TOL_SCAN, (n, h, e_s)


@pytest.mark.parametrize("wl", [workloads.PREFILL_1K, workloads.PREFILL_LONG, workloads.VARLEN_8],
                         ids=lambda w: w.name)
def test_full_size_prefill_sampled(g, wl):
    x = workloads.generate(wl)
    o, S = _run_prefill(g, x, wl, torch.bfloat16)
    rng = np.random.default_rng(0)
    units = sorted({(int(rng.integers(wl.num_seqs)), int(rng.integers(wl.Hv))) for _ in range(4)})
    if wl.num_seqs > 1:   # include the shortest and the longest sequence
        lens = np.diff(x["cu_seqlens"])
        units += [(int(np.argmin(lens)), 0), (int(np.argmax(lens)), wl.Hv - 1)]
    _sampled_units(wl, x, units, o, S)


def test_full_size_decode(g):
    w = workloads.DECODE_B256
    x = workloads.generate(w)
    d = upload_scan_inputs(x, True)
    state = d["initial_state"].clone()
    o = g.gdn_decode_step(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], state)
    torch.cuda.synchronize()
    o_ref, S_ref = _full_oracle(x)
    assert rel_err(to_np(o), o_ref) <= TOL_SCAN_BF16_OUT
    assert rel_err(to_np(state), S_ref) <= TOL_SCAN


def test_tiny_workload(g):
    w = workloads.TINY
    x = workloads.generate(w)
    o_ref, S_ref = _full_oracle(x)
    o, S = _run_prefill(g, x, w, torch.float32)
    assert rel_err(o, o_ref) <= TOL_SCAN
    assert rel_err(S, S_ref) <= TOL_SCAN
