"""Shared test helpers: upload of workload inputs, the error metric, tolerances, and
per-unit oracle calls for sampled checks at full size."""
import numpy as np
import torch

import oracle

# Max relative error, || gpu - ref ||_inf / || ref ||_inf, per tensor.
# Scan (o and final state) with fp32 results: the stated 2e-3.
TOL_SCAN = 2e-3
# A bf16 result carries its own storage rounding on top: half an ulp of the largest
# element is 2^-8 of it, so the bound for bf16 outputs is 2e-3 + 2^-8.
TOL_SCAN_BF16_OUT = 2e-3 + 2.0 ** -8
# Gated RMSNorm in fp32 arithmetic (rsqrt, expf: a few ulp): 1e-5; bf16 output adds 2^-8.
TOL_TAIL = 1e-5
TOL_TAIL_BF16_OUT = 1e-5 + 2.0 ** -8
# Short convolution + SiLU, element by element: bf16 storage rounding of y (half an ulp, 2^-9
# relative) plus the fp32 sum of K products and the approximate exponential and reciprocal
# (about 1e-6 relative of the pre-activation): |got - ref| <= 2^-8 |ref| + 1e-5.
TOL_CONV_RTOL = 2.0 ** -8
TOL_CONV_ATOL = 1e-5
# NVFP4 GEMM against the fp64 product of the dequantised operands: the stated 1e-2.
TOL_GEMM = 1e-2


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max()
    if den == 0:
        return float(np.abs(got).max())
    return float(np.abs(got - ref).max() / den)


def dev(x, dtype, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dtype)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def upload_scan_inputs(x: dict, io_bf16: bool):
    dt = torch.bfloat16 if io_bf16 else torch.float32
    return dict(
        q=dev(x["q"], dt), k=dev(x["k"], dt), v=dev(x["v"], dt),
        a=dev(x["a"], torch.float32), b=dev(x["b"], torch.float32),
        A_log=dev(x["A_log"], torch.float32), dt_bias=dev(x["dt_bias"], torch.float32),
        cu_seqlens=dev(x["cu_seqlens"], torch.int32),
        initial_state=None if x["initial_state"] is None else dev(x["initial_state"], torch.float32),
    )


def oracle_unit(x: dict, n: int, h: int, Hk: int, Hv: int, scale: float = 1.0):
    """Oracle scan of one (sequence, value head) unit: returns (o [T_n, D], S [D, D])."""
    cu = x["cu_seqlens"]
    sl = slice(int(cu[n]), int(cu[n + 1]))
    hk = h // (Hv // Hk)
    S0 = None if x["initial_state"] is None else x["initial_state"][n:n + 1, h:h + 1]
    o, S = oracle.gdn_scan(x["q"][sl, hk:hk + 1], x["k"][sl, hk:hk + 1], x["v"][sl, h:h + 1],
                           x["a"][sl, h:h + 1], x["b"][sl, h:h + 1], x["A_log"][h:h + 1],
                           x["dt_bias"][h:h + 1], initial_state=S0, scale=scale, threads=1)
    return o[:, 0], S[0, 0]
