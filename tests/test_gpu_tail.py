"""Parity of the gated RMSNorm tail and the NVFP4 encoder with the oracle: the tail within
its fp32 tolerance, the encoder bit for bit (codes, nibble order and block scales), the
fused tail+encoder bit for bit against the two-call path, and the hardware E2M1 / E4M3
conversions against the oracle's round-to-nearest-even on every bf16 value and on the
rounding boundaries."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import TOL_TAIL, TOL_TAIL_BF16_OUT, dev, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import gated_deltanet_03_b200 as lib
    return lib


@pytest.mark.parametrize("D", [16, 32, 64, 128])
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_gated_rmsnorm(g, D, io):
    rng = np.random.default_rng(D)
    M, Hv = 67, 3
    o = rng.standard_normal((M, Hv, D)).astype(np.float32)
    z = rng.standard_normal((M, Hv, D)).astype(np.float32)
    if io == "bf16":
        o, z = workloads.round_bf16(o), workloads.round_bf16(z)
    w = rng.uniform(0.5, 1.5, D).astype(np.float32)
    y_ref = oracle.gated_rmsnorm_silu(o, z, w)
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    y = g.gdn_gated_rmsnorm_silu(dev(o, dt), dev(z, dt), dev(w, torch.float32), out_dtype=torch.float32)
    assert rel_err(to_np(y), y_ref) <= TOL_TAIL
    yb = g.gdn_gated_rmsnorm_silu(dev(o, dt), dev(z, dt), dev(w, torch.float32), out_dtype=torch.bfloat16)
    assert rel_err(to_np(yb), y_ref) <= TOL_TAIL_BF16_OUT


@pytest.mark.parametrize("M,K", [(1, 32), (257, 4096), (64, 2048), (3, 96)])
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_nvfp4_quantize_bit_exact(g, M, K, io):
    x = workloads.activations(M, K, seed=M * 7 + K, bf16=(io == "bf16"))
    gs = np.float32(448.0 * 6.0 / max(float(np.abs(x).max()), 1e-30))
    xq_ref, xs_ref = oracle.nvfp4_quantize(x, gs)
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    xq, xs = g.nvfp4_quantize_act(dev(x, dt), float(gs))
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)


def test_e2m1_hardware_rounding_every_bf16_value(g):
    """Blocks [6, v1..v15] with global scale 1: the block scale is exactly 1 (E4M3 0x38), so
    each code is E2M1(v) of the value itself. Every bf16 value with |v| <= 6 is covered."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    vals = vals[np.isfinite(vals) & (np.abs(vals) <= 6.0)]
    vals = np.concatenate([vals, np.zeros((-len(vals)) % 15, np.float32)])
    blocks = np.concatenate([np.full((len(vals) // 15, 1), 6.0, np.float32), vals.reshape(-1, 15)], axis=1)
    pad = (-blocks.shape[0]) % 2
    blocks = np.concatenate([blocks, np.full((pad, 16), 6.0, np.float32)])
    x = blocks.reshape(-1, 32)
    xq_ref, xs_ref = oracle.nvfp4_quantize(x, 1.0)
    assert np.all(xs_ref == 0x38)
    xq, xs = g.nvfp4_quantize_act(dev(x, torch.bfloat16), 1.0)
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)


def test_e2m1_and_e4m3_boundaries_fp32(g):
    """fp32 inputs at and next to every E2M1 decision point, and block maxima whose scale
    lands at and next to every E4M3 rounding midpoint."""
    pts = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32)
    near = np.concatenate([pts, np.nextafter(pts, np.float32(0)), np.nextafter(pts, np.float32(9))])
    near = np.concatenate([near, -near, np.float32([0.0, -0.0, 1e-30, -1e-30, 7.0, -100.0])])
    near = np.concatenate([near, np.zeros((-len(near)) % 15, np.float32)])
    blocks = np.concatenate([np.full((len(near) // 15, 1), 6.0, np.float32), near.reshape(-1, 15)], axis=1)
    # E4M3 midpoints: block max 6*m makes s = m exactly (global scale 1)
    e4 = np.sort(oracle.e4m3_decode(np.arange(1, 0x7F, dtype=np.uint8)))
    mids = ((e4[:-1].astype(np.float64) + e4[1:]) / 2).astype(np.float32)
    ms = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e4)), e4,
                         np.float32([500.0, 1e-6])])
    sblocks = np.zeros((len(ms), 16), np.float32)
    sblocks[:, 0] = ms * 6.0
    sblocks[:, 1] = -ms
    allb = np.concatenate([blocks, sblocks])
    allb = np.concatenate([allb, np.zeros(((-allb.shape[0]) % 2, 16), np.float32)])
    x = allb.reshape(-1, 32)
    xq_ref, xs_ref = oracle.nvfp4_quantize(x, 1.0)
    xq, xs = g.nvfp4_quantize_act(dev(x, torch.float32), 1.0)
    np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)


@pytest.mark.parametrize("D,Hv", [(128, 32), (128, 16), (16, 2)])
def test_fused_tail_equals_two_calls_and_oracle(g, D, Hv):
    rng = np.random.default_rng(D + Hv)
    M = 130
    o = workloads.round_bf16(rng.standard_normal((M, Hv, D)).astype(np.float32))
    z = workloads.round_bf16(rng.standard_normal((M, Hv, D)).astype(np.float32))
    w = rng.uniform(0.5, 1.5, D).astype(np.float32)
    y_ref = oracle.gated_rmsnorm_silu(o, z, w)
    gs = np.float32(448.0 * 6.0 / np.abs(y_ref).max())
    od, zd, wd = dev(o, torch.bfloat16), dev(z, torch.bfloat16), dev(w, torch.float32)
    xq_f, xs_f = g.gdn_gated_rmsnorm_silu_nvfp4(od, zd, wd, float(gs))
    y = g.gdn_gated_rmsnorm_silu(od, zd, wd, out_dtype=torch.bfloat16)
    xq_2, xs_2 = g.nvfp4_quantize_act(y, float(gs))
    np.testing.assert_array_equal(xq_f.cpu().numpy(), xq_2.cpu().numpy())
    np.testing.assert_array_equal(xs_f.cpu().numpy(), xs_2.cpu().numpy())
    # against the oracle: dequantised values of the fused output vs the oracle's encode of
    # its own (bf16-rounded) y agree to within one quantisation step of each block
    xq_r, xs_r = oracle.nvfp4_quantize(workloads.round_bf16(y_ref.astype(np.float32)), gs)
    d_gpu = oracle.nvfp4_dequantize(xq_f.cpu().numpy(), xs_f.cpu().numpy(), gs)
    d_ref = oracle.nvfp4_dequantize(xq_r, xs_r, gs)
    assert (xq_f.cpu().numpy() != xq_r).mean() < 0.01
    assert rel_err(d_gpu, d_ref) <= 0.25


def test_tail_zero_rows_and_zero_blocks(g):
    M, Hv, D = 4, 2, 128
    o = np.zeros((M, Hv, D), np.float32)
    z = np.ones((M, Hv, D), np.float32)
    w = np.ones(D, np.float32)
    xq, xs = g.gdn_gated_rmsnorm_silu_nvfp4(dev(o, torch.bfloat16), dev(z, torch.bfloat16),
                                            dev(w, torch.float32), 1.0)
    assert int(xs.abs().sum()) == 0 and int(xq.sum()) == 0


def test_nvfp4_block_scale_order_on_ties(g):
    """The encoder's block scale follows (amax / 6) * gs on the E4M3 tie cases of
    tests/golden/nvfp4_scale_order.txt, where another order of the same operations picks a
    different code; standalone encoder and fused tail both, bf16 and fp32 inputs."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_scale_order.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    for amax_s, gs_bits, want_s, _, _ in rows:
        amax = float(amax_s)
        gs = float(np.array([int(gs_bits, 16)], np.uint32).view(np.float32)[0])
        want = int(want_s, 16)
        x = np.zeros((4, 32), np.float32)
        x[:, 5] = amax
        x[:, 6] = -0.5 * amax
        x[:, 16 + 3] = -amax
        for dt in (torch.bfloat16, torch.float32):
            xq, xs = g.nvfp4_quantize_act(dev(x, dt), gs)
            xq_ref, xs_ref = oracle.nvfp4_quantize(x, np.float32(gs))
            assert (xs.cpu().numpy() == want).all()
            np.testing.assert_array_equal(xs.cpu().numpy(), xs_ref)
            np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)
