"""Parity of the block-scaled NVFP4 GEMM with the oracle (fp64 product of the dequantised
operands, both sides fed the same oracle-encoded codes and scales): within the stated
1e-2 max relative error, for ragged M, N and K tiles, the tiny K = 32 case, and the full
output-projection sizes (sampled rows)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import TOL_GEMM, dev, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import gated_deltanet_03_b200 as lib
    return lib


def _operands(M, N, K, seed):
    rng = np.random.default_rng(seed)
    A = workloads.activations(M, K, seed=seed)
    W = workloads.round_bf16(rng.standard_normal((N, K)).astype(np.float32) * 0.02)
    gsa = np.float32(448.0 * 6.0 / np.abs(A).max())
    gsw = np.float32(448.0 * 6.0 / np.abs(W).max())
    aq, as_ = oracle.nvfp4_quantize(A, gsa)
    wq, ws = oracle.nvfp4_quantize(W, gsw)
    return aq, as_, gsa, wq, ws, gsw


def _gpu(g, aq, as_, wq, ws, alpha, out_dtype):
    u8 = torch.uint8
    y = g.nvfp4_gemm(dev(aq, u8), dev(as_, u8), dev(wq, u8), dev(ws, u8), alpha, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert g.gdn_get_device_status() == 0
    return to_np(y)


@pytest.mark.parametrize("M,N,K", [(64, 16, 32), (128, 256, 256), (300, 272, 512), (1, 16, 96),
                                   (129, 512, 2048), (4096, 1024, 2048)])
def test_gemm_matches_oracle(g, M, N, K):
    aq, as_, gsa, wq, ws, gsw = _operands(M, N, K, seed=M + N + K)
    ref = oracle.nvfp4_gemm(aq, as_, gsa, wq, ws, gsw)
    alpha = float(np.float32(1.0) / (np.float32(gsa) * np.float32(gsw)))
    y32 = _gpu(g, aq, as_, wq, ws, alpha, torch.float32)
    assert rel_err(y32, ref) <= TOL_GEMM, rel_err(y32, ref)
    y16 = _gpu(g, aq, as_, wq, ws, alpha, torch.bfloat16)
    assert rel_err(y16, ref) <= TOL_GEMM


def test_gemm_exact_on_grid_values(g):
    """Codes whose products sum exactly in fp32: every element of y is exact."""
    rng = np.random.default_rng(5)
    M, N, K = 128, 256, 256
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    A = grid[rng.integers(0, 8, (M, K))] * np.where(rng.random((M, K)) < .5, -1, 1).astype(np.float32)
    B = grid[rng.integers(0, 8, (N, K))] * np.where(rng.random((N, K)) < .5, -1, 1).astype(np.float32)
    A.reshape(M, K // 16, 16)[:, :, 0] = 6.0
    B.reshape(N, K // 16, 16)[:, :, 0] = 6.0
    aq, as_ = oracle.nvfp4_quantize(A, 1.0)
    bq, bs = oracle.nvfp4_quantize(B, 1.0)
    y = _gpu(g, aq, as_, bq, bs, 1.0, torch.float32)
    np.testing.assert_array_equal(y, A.astype(np.float64) @ B.T.astype(np.float64))


@pytest.mark.parametrize("M,N,K", [(32768, 2048, 4096), (256, 2048, 4096)])
def test_gemm_full_size_sampled_rows(g, M, N, K):
    aq, as_, gsa, wq, ws, gsw = _operands(M, N, K, seed=11)
    alpha = float(np.float32(1.0) / (np.float32(gsa) * np.float32(gsw)))
    y = _gpu(g, aq, as_, wq, ws, alpha, torch.bfloat16)
    rows = np.random.default_rng(1).choice(M, size=min(M, 256), replace=False)
    rows = np.concatenate([rows, [0, M - 1]])
    ref = oracle.nvfp4_gemm(aq, as_, gsa, wq, ws, gsw, rows=rows)
    assert rel_err(y[rows], ref) <= TOL_GEMM


@pytest.mark.parametrize("M", [64, 300])
def test_fused_modules_colscale(g, M):
    """Several modules fused into one weight (as in a fused in_proj: q, k, v, z, a, b), each
    calibrated and quantised with its own global scale; the gate modules an order of magnitude
    smaller. With the per-column factor the fused GEMM matches the oracle module by module; with
    one factor for the whole output (the mismatch) the modules whose scale differs are off."""
    K = 512
    widths = (128, 128, 256, 256, 16, 16)
    mags = (0.02, 0.02, 0.02, 0.02, 0.001, 0.001)
    rng = np.random.default_rng(M)
    A = workloads.activations(M, K, seed=M + 1)
    gsa = np.float32(448.0 * 6.0 / np.abs(A).max())
    aq, as_ = oracle.nvfp4_quantize(A, gsa)
    wqs, wss, gsws, refs = [], [], [], []
    for n, mag in zip(widths, mags):
        W = workloads.round_bf16(rng.standard_normal((n, K)).astype(np.float32) * mag)
        gsw = np.float32(448.0 * 6.0 / np.abs(W).max())
        wq, ws = oracle.nvfp4_quantize(W, gsw)
        wqs.append(wq)
        wss.append(ws)
        gsws.append(gsw)
        refs.append(oracle.nvfp4_gemm(aq, as_, gsa, wq, ws, gsw))
    wq, ws, ref = np.concatenate(wqs), np.concatenate(wss), np.concatenate(refs, axis=1)
    u8 = torch.uint8
    ca = g.nvfp4_fused_col_alpha(widths, gsws, float(gsa))
    y = to_np(g.nvfp4_gemm_colscale(dev(aq, u8), dev(as_, u8), dev(wq, u8), dev(ws, u8), ca, out_dtype=torch.float32))
    torch.cuda.synchronize()
    assert g.gdn_get_device_status() == 0
    col = 0
    for n in widths:
        assert rel_err(y[:, col:col + n], ref[:, col:col + n]) <= TOL_GEMM
        col += n
    # one global scale (the first module's) for the fused output: the gate modules come out wrong
    alpha0 = float(np.float32(1.0) / (gsa * gsws[0]))
    y1 = _gpu(g, aq, as_, wq, ws, alpha0, torch.float32)
    gate = slice(sum(widths[:4]), sum(widths))
    assert rel_err(y1[:, gate], ref[:, gate]) > 100 * TOL_GEMM


@pytest.mark.parametrize("M,N,K", [(1, 128, 256), (200, 256, 768), (130, 512, 1024), (256, 2048, 4096), (4096, 2048, 4096),
                                   (10000, 2048, 4096)])
def test_q4k_gemm_matches_oracle(g, M, N, K):
    """The Q4_K output projection ("Red Lite dev15d - DeltaNet gated tail + Q4_K output
    projection", Q4_K implementation) against the fp64 product with the oracle's exact decode of
    the same synthetic weights: within the GEMM tolerance (the kernel rounds each decoded weight
    to bf16), for ragged M, the batched-decode shape (M = 256, 4096 -> 2048) and a prefill-sized
    M; bf16 and fp32 outputs. The small-M shapes run split over K in clusters of 2 (200 x 256 x
    768), 4 (130 x 512 x 1024) and 8 (256 x 2048 x 4096) CTAs; 4096 x 2048 x 4096 unsplit on
    128-wide tiles, and the ragged 10000 x 2048 x 4096 on 256-wide tiles (the large-M form)."""
    w = workloads.q4k_weights(N, K, seed=M + N + K)
    a = workloads.activations(M, K, seed=M * 3 + 1, heavy_tail=False)
    rows = np.arange(M) if M <= 256 else np.unique(np.concatenate([np.arange(0, M, 37), [M - 1]]))
    ref = oracle.q4k_gemm(a, w, K, rows=rows)
    aa, ww = dev(a, torch.bfloat16), dev(w, torch.uint8)
    y32 = to_np(g.q4k_gemm(aa, ww, out_dtype=torch.float32))
    yb = to_np(g.q4k_gemm(aa, ww, out_dtype=torch.bfloat16))
    torch.cuda.synchronize()
    assert g.gdn_get_device_status() == 0
    assert rel_err(y32[rows], ref) <= TOL_GEMM
    assert rel_err(yb[rows], ref) <= TOL_GEMM
