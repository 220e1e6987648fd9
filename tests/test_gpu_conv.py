"""The causal short convolution + SiLU (gdn_short_conv1d_silu, gdn_short_conv1d_silu_decode)
against the oracle, element by element: y within bf16 rounding, the carried state bit for bit
(it is a copy of inputs). Covers every width K, packed sequences with empty and one-token
members, a carried initial state (also updated in place), the q/k/v plane split, a strided
input, decode continuing a prefill, and the benchmark layer's full sizes."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import TOL_CONV_ATOL, TOL_CONV_RTOL, dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import gated_deltanet_03_b200 as lib
    return lib


def _close(got, ref, rows=4096):
    """Element-wise bound, taken over blocks of rows to keep host memory small at full size."""
    for r0 in range(0, got.shape[0], rows):
        gb = np.asarray(got[r0:r0 + rows], np.float64)
        rb = ref[r0:r0 + rows]
        err = np.abs(gb - rb)
        bound = TOL_CONV_RTOL * np.abs(rb) + TOL_CONV_ATOL
        worst = int(np.argmax(err - bound))
        assert (err <= bound).all(), ("conv", r0, np.unravel_index(worst, err.shape), gb.flat[worst],
                                      rb.flat[worst])


def _bits(t):
    return t.view(torch.int16).cpu().numpy()


def _bf16_bits(x):
    return dev(x, torch.bfloat16).view(torch.int16).cpu().numpy()


def _run(g, inp, cu=None, num_seqs=1, state_out=True, parts=None):
    x = dev(inp["x"], torch.bfloat16)
    w = dev(inp["weight"], torch.float32)
    s0 = None if inp["initial_state"] is None else dev(inp["initial_state"], torch.bfloat16)
    cu_d = None if cu is None else dev(cu, torch.int32)
    y, fs = g.gdn_short_conv1d_silu(x, w, cu_seqlens=cu_d, num_seqs=num_seqs, initial_state=s0,
                                    output_final_state=state_out, parts=parts)
    torch.cuda.synchronize()
    return y, fs


@pytest.mark.parametrize("K", [1, 2, 3, 4])
def test_conv_one_sequence_every_width(g, K):
    inp = workloads.conv_inputs(300, 264, K, seed=10 + K)
    y, fs = _run(g, inp)
    y_ref, f_ref = oracle.short_conv1d_silu(inp["x"], inp["weight"])
    _close(to_np(y), y_ref)
    if K > 1:
        np.testing.assert_array_equal(_bits(fs), _bf16_bits(f_ref))


@pytest.mark.parametrize("K", [2, 4])
def test_conv_packed_sequences_with_state(g, K):
    """Lengths 1, 1, 38, 0, 57, 203: sequences shorter than K - 1 keep part of the carried
    history in their final state; the empty one passes its history through unchanged."""
    cu = np.array([0, 1, 2, 40, 40, 97, 300], dtype=np.int32)
    inp = workloads.conv_inputs(300, 136, K, seed=20 + K, num_seqs=6, state=True)
    y, fs = _run(g, inp, cu=cu)
    y_ref, f_ref = oracle.short_conv1d_silu(inp["x"], inp["weight"], cu_seqlens=cu,
                                            initial_state=inp["initial_state"])
    _close(to_np(y), y_ref)
    np.testing.assert_array_equal(_bits(fs), _bf16_bits(f_ref))


def test_conv_equal_runs_without_cu_seqlens(g):
    inp = workloads.conv_inputs(4 * 75, 64, 4, seed=31, num_seqs=4, state=True)
    y, fs = _run(g, inp, num_seqs=4)
    cu = np.arange(0, 301, 75)
    y_ref, f_ref = oracle.short_conv1d_silu(inp["x"], inp["weight"], cu_seqlens=cu,
                                            initial_state=inp["initial_state"])
    _close(to_np(y), y_ref)
    np.testing.assert_array_equal(_bits(fs), _bf16_bits(f_ref))


def test_conv_state_in_place(g):
    cu = np.array([0, 2, 90, 91], dtype=np.int32)
    inp = workloads.conv_inputs(91, 128, 4, seed=41, num_seqs=3, state=True)
    x = dev(inp["x"], torch.bfloat16)
    w = dev(inp["weight"], torch.float32)
    st = dev(inp["initial_state"], torch.bfloat16)
    y, fs = g.gdn_short_conv1d_silu(x, w, cu_seqlens=dev(cu, torch.int32), initial_state=st, final_state=st)
    torch.cuda.synchronize()
    y_ref, f_ref = oracle.short_conv1d_silu(inp["x"], inp["weight"], cu_seqlens=cu,
                                            initial_state=inp["initial_state"])
    assert fs is st
    _close(to_np(y), y_ref)
    np.testing.assert_array_equal(_bits(st), _bf16_bits(f_ref))


def test_conv_planes_from_a_strided_projection(g):
    """x is the q|k|v column block of a wider projection output (z after it); y comes out as
    three contiguous planes [T, Hk*Dk], [T, Hk*Dk], [T, Hv*Dv]."""
    T, Hk, Hv, D = 333, 2, 4, 128
    C = 2 * Hk * D + Hv * D
    inp = workloads.conv_inputs(T, C + Hv * D, 4, seed=51)
    wide = dev(inp["x"], torch.bfloat16)
    x = wide[:, :C]
    w = dev(inp["weight"][:C], torch.float32)
    (q, k, v), _ = g.gdn_short_conv1d_silu(x, w, parts=(Hk * D, Hk * D, Hv * D))
    torch.cuda.synchronize()
    y_ref, _ = oracle.short_conv1d_silu(inp["x"][:, :C], inp["weight"][:C])
    _close(to_np(q), y_ref[:, :Hk * D])
    _close(to_np(k), y_ref[:, Hk * D:2 * Hk * D])
    _close(to_np(v), y_ref[:, 2 * Hk * D:])
    assert q.is_contiguous() and k.is_contiguous() and v.is_contiguous()


def test_conv_saturating_inputs(g):
    """Pre-activations far into both tails of SiLU (zero on the left, identity on the right)."""
    inp = workloads.conv_inputs(130, 64, 4, seed=61)
    inp["x"] = workloads.round_bf16(inp["x"] * np.float32(40.0))
    y, _ = _run(g, inp, state_out=False)
    y_ref, _ = oracle.short_conv1d_silu(inp["x"], inp["weight"])
    _close(to_np(y), y_ref)
    assert np.abs(y_ref).max() > 50.0 and (y_ref < -1e-6).any()


@pytest.mark.parametrize("K", [1, 4])
def test_conv_decode_continues_prefill(g, K):
    """A prefill of 7 tokens per sequence, then 5 decode steps from its final state, equals one
    pass over all 12 tokens; the state after the steps equals the oracle's final state."""
    B, C, T0, steps = 5, 192, 7, 5
    inp = workloads.conv_inputs(B * (T0 + steps), C, K, seed=70 + K)
    xs = inp["x"].reshape(B, T0 + steps, C)
    w = dev(inp["weight"], torch.float32)
    pre = np.ascontiguousarray(xs[:, :T0].reshape(B * T0, C))
    _, st = g.gdn_short_conv1d_silu(dev(pre, torch.bfloat16), w, num_seqs=B, output_final_state=True)
    if K == 1:
        st = torch.empty((B, 0, C), dtype=torch.bfloat16, device="cuda")
    ys = []
    for s in range(steps):
        ys.append(to_np(g.gdn_short_conv1d_silu_decode(dev(xs[:, T0 + s], torch.bfloat16), w, st)))
    torch.cuda.synchronize()
    cu = np.arange(0, B * (T0 + steps) + 1, T0 + steps)
    y_ref, f_ref = oracle.short_conv1d_silu(xs.reshape(-1, C), inp["weight"], cu_seqlens=cu)
    y_ref = y_ref.reshape(B, T0 + steps, C)
    for s in range(steps):
        _close(ys[s], y_ref[:, T0 + s])
    if K > 1:
        np.testing.assert_array_equal(_bits(st), _bf16_bits(f_ref))


def test_conv_decode_planes(g):
    B, Hk, Hv, D = 256, 2, 4, 128
    C = 2 * Hk * D + Hv * D
    inp = workloads.conv_inputs(B, C, 4, seed=81, num_seqs=B, state=True)
    st = dev(inp["initial_state"], torch.bfloat16)
    q, k, v = g.gdn_short_conv1d_silu_decode(dev(inp["x"], torch.bfloat16), dev(inp["weight"], torch.float32), st,
                                             parts=(Hk * D, Hk * D, Hv * D))
    torch.cuda.synchronize()
    y_ref, f_ref = oracle.short_conv1d_silu(inp["x"], inp["weight"], cu_seqlens=np.arange(B + 1),
                                            initial_state=inp["initial_state"])
    _close(np.concatenate([to_np(q), to_np(k), to_np(v)], axis=1), y_ref)
    np.testing.assert_array_equal(_bits(st), _bf16_bits(f_ref))


@pytest.mark.parametrize("T,Hk,Hv", [(4096, 16, 16), (32768, 16, 32)])
def test_conv_full_size_layer(g, T, Hk, Hv):
    """The convolution in front of the 1024-wide and the long prefill workloads (C = q + k + v
    channels, K = 4), every element against the oracle, in the plane layout the scan reads."""
    D = 128
    C = 2 * Hk * D + Hv * D
    inp = workloads.conv_inputs(T, C, 4, seed=90 + Hv, state=True)
    (q, k, v), fs = _run(g, inp, parts=(Hk * D, Hk * D, Hv * D))
    y_ref, f_ref = oracle.short_conv1d_silu(inp["x"], inp["weight"], initial_state=inp["initial_state"])
    _close(to_np(q), y_ref[:, :Hk * D])
    _close(to_np(k), y_ref[:, Hk * D:2 * Hk * D])
    _close(to_np(v), y_ref[:, 2 * Hk * D:])
    np.testing.assert_array_equal(_bits(fs), _bf16_bits(f_ref))
