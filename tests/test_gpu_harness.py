"""The error-propagation harness (gated_deltanet_03_b200.error_harness) and the NVFP4 decode
it relies on. Its GPU measurements are checked against the same measurements computed with
the oracle on the same seeded inputs (encode and decode in the oracle, the oracle's
recurrence and GEMM, its gate formula), and at full size against properties that hold at any
size: a flat noise level over the long-prefill sequence, and forgetting of a state impulse at
the rate the decay and the overwrite along random keys predict."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import gated_deltanet_03_b200 as lib
    return lib


@pytest.fixture(scope="module")
def h(g):
    from gated_deltanet_03_b200 import error_harness
    return error_harness


def _gs(x):
    return 448.0 * 6.0 / float(np.abs(x).max())


def _rel_rms(x, ref):
    return float(np.linalg.norm((np.asarray(x, np.float64) - ref).ravel()) / np.linalg.norm(np.asarray(ref).ravel()))


def test_dequantize_is_the_rounded_quotient(g):
    """Every decoded value is the correctly rounded fp32 quotient E2M1 * E4M3 / gs (half an ulp
    of the oracle's exact value), on heavy-tailed activations with all-zero blocks."""
    x = workloads.activations(300, 512, seed=41)
    gs = _gs(x)
    xq, xs = oracle.nvfp4_quantize(x, gs)
    ref = oracle.nvfp4_dequantize(xq, xs, gs)
    y = to_np(g.nvfp4_dequantize_act(dev(xq, torch.uint8), dev(xs, torch.uint8), gs))
    assert (np.abs(y - ref) <= 2.0 ** -24 * np.abs(ref)).all()
    assert ((ref == 0) == (y == 0)).all()
    yb = to_np(g.nvfp4_dequantize_act(dev(xq, torch.uint8), dev(xs, torch.uint8), gs, out_dtype=torch.bfloat16))
    assert (np.abs(yb - ref) <= 2.0 ** -8 * np.abs(ref)).all()


def test_roundtrip_equals_oracle_encode_decode(h):
    x = workloads.activations(64, 256, seed=42)
    xh, gs = h.nvfp4_roundtrip(dev(x, torch.bfloat16))
    ref = oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(x, gs), gs)
    assert (np.abs(to_np(xh) - ref) <= 2.0 ** -24 * np.abs(ref)).all()


def test_gate_compression_matches_oracle(h):
    M, K, Hv = 256, 512, 16
    rng = np.random.default_rng(7)
    x = workloads.round_bf16(rng.standard_normal((M, K)).astype(np.float32))
    w_a = workloads.round_bf16((rng.standard_normal((Hv, K)) / math.sqrt(K)).astype(np.float32))
    w_b = workloads.round_bf16((rng.standard_normal((Hv, K)) / math.sqrt(K)).astype(np.float32))
    _, A_spec, dt_spec = h.decay_spectrum(Hv)       # the fixed timescale spectrum (decay 1e-3 .. 0.999)
    A_log, dt_bias = A_spec.numpy().astype(np.float32), dt_spec.numpy().astype(np.float32)
    got = h.gate_compression(dev(x, torch.bfloat16), dev(w_a, torch.bfloat16), dev(w_b, torch.bfloat16),
                             dev(A_log, torch.float32), dev(dt_bias, torch.float32))
    # the same measurement with the oracle: encode, fp64 GEMM of the decoded operands, gates
    gx = _gs(x)
    xq, xs = oracle.nvfp4_quantize(x, gx)
    quant = []
    for w in (w_a, w_b):
        gw = _gs(w)
        wq, ws = oracle.nvfp4_quantize(w, gw)
        quant.append(oracle.nvfp4_gemm(xq, xs, gx, wq, ws, gw))
    exact_a, exact_b = x.astype(np.float64) @ w_a.T.astype(np.float64), x.astype(np.float64) @ w_b.T.astype(np.float64)

    def gates(a, b):
        al = np.empty_like(a)
        be = np.empty_like(b)
        for i in range(a.shape[0]):
            for j in range(Hv):
                _, al[i, j], be[i, j] = oracle.gates(float(a[i, j]), float(b[i, j]), float(A_log[j]),
                                                     float(dt_bias[j]))
        return al, be

    al, be = gates(exact_a, exact_b)
    alq, beq = gates(quant[0], quant[1])
    ref = {"preact_a": _rel_rms(quant[0], exact_a), "preact_b": _rel_rms(quant[1], exact_b),
           "alpha": _rel_rms(alq, al), "beta": _rel_rms(beq, be)}
    for key, val in ref.items():
        assert abs(got[key] - val) <= 1e-3 * val + 1e-7, (key, got[key], val)
    # mechanism ii: the sigmoid's slope is at most 1/4 and slow heads damp alpha's sensitivity by
    # sigma(a + dt_bias), so the gates carry a fraction of the pre-activations' error
    assert got["alpha"] < 0.25 * got["preact_a"] and got["beta"] < 0.5 * got["preact_b"], got


def test_noise_plateau_matches_oracle(h):
    w = workloads.custom("plateau_small", (1024,), 2, 2, 128, seed=21)
    x = workloads.generate(w)
    window = 256
    got = h.noise_plateau(dev(x["q"], torch.bfloat16), dev(x["k"], torch.bfloat16), dev(x["v"], torch.bfloat16),
                          dev(x["a"], torch.float32), dev(x["b"], torch.float32), dev(x["A_log"], torch.float32),
                          dev(x["dt_bias"], torch.float32), window=window)

    def noisy(a):
        a2 = a.reshape(a.shape[0], -1)
        gs = _gs(a2)
        return workloads.round_bf16(oracle.nvfp4_dequantize(*oracle.nvfp4_quantize(a2, gs), gs).astype(np.float32)
                                    ).reshape(a.shape)

    args = (x["a"], x["b"], x["A_log"], x["dt_bias"])
    o, S = oracle.gdn_scan(x["q"], x["k"], x["v"], *args)
    on, Sn = oracle.gdn_scan(noisy(x["q"]), noisy(x["k"]), noisy(x["v"]), *args)
    ref = [_rel_rms(on[i:i + window], o[i:i + window]) for i in range(0, 1024, window)]
    for gw, rw in zip(got["output_per_window"], ref):
        assert abs(gw - rw) <= 0.05 * rw, (gw, rw)
    assert abs(got["final_state"] - _rel_rms(Sn, S)) <= 0.05 * _rel_rms(Sn, S)


def test_impulse_response_matches_oracle(h):
    Hv, D, T = 4, 128, 256
    w = workloads.custom("impulse_small", (T,), 2, Hv, D, io="f32", seed=31)
    x = workloads.generate(w)
    alpha, A_log, dt_bias = h.decay_spectrum(Hv, lo=1e-3, hi=0.5)
    imp = np.random.default_rng(3).standard_normal((1, Hv, D, D)).astype(np.float32)
    steps = (8, 64, 256)
    got = h.impulse_response(dev(x["q"], torch.float32), dev(x["k"], torch.float32), dev(x["b"], torch.float32),
                             dev(A_log.numpy(), torch.float32), dev(dt_bias.numpy(), torch.float32),
                             dev(imp, torch.float32), steps)
    zeros_v = np.zeros((T, Hv, D), np.float32)
    zeros_a = np.zeros((T, Hv), np.float32)
    n0 = np.linalg.norm(imp.reshape(Hv, -1), axis=1)
    for si, t in enumerate(steps):
        _, S = oracle.gdn_scan(x["q"][:t], x["k"][:t], zeros_v[:t], zeros_a[:t], x["b"][:t],
                               A_log.numpy().astype(np.float32), dt_bias.numpy().astype(np.float32),
                               initial_state=imp)
        ref = np.linalg.norm(S.reshape(Hv, -1), axis=1) / n0
        for hh in range(Hv):
            if ref[hh] > 1e-25:
                assert abs(got["measured"][si][hh] - ref[hh]) <= 1e-3 * ref[hh], (t, hh)


def test_full_size_plateau_and_forgetting(h):
    """The long-prefill sequence (32768 tokens, 16/32 heads): the output error of the noisy run
    stays flat (last quarter within 1.5x of the first); a state impulse under a decay spectrum
    of 1e-3 .. 0.999 shrinks as the overwrite model predicts (within 2x at 1024 steps), and the
    slowest head forgets much faster than its decay gate alone (0.999^1024 = 0.36)."""
    rep = h._report()
    pl = rep["noise_plateau"]
    assert pl["last_over_first"] <= 1.5, pl
    im = rep["impulse_response"]
    i1024 = im["steps"].index(1024)
    meas, pred, gate = im["measured"][i1024], im["overwrite_model"][i1024], im["gate_only"][i1024]
    for hh in range(len(meas)):
        if pred[hh] > 1e-20:
            assert 0.5 * pred[hh] <= meas[hh] <= 2.0 * pred[hh], (hh, meas[hh], pred[hh])
    slow = int(np.argmax(im["alpha"]))
    assert meas[slow] < 0.25 * gate[slow]
    # mechanism ii under the fixed timescale spectrum: the gates keep a small part of the GEMM error
    gc = rep["gate_compression"]["timescale_spectrum"]
    assert gc["alpha"] < 0.25 * gc["preact_a"] and gc["beta"] < 0.5 * gc["preact_b"], gc
    assert gc["compression"] > 3.0, gc
