"""Error-propagation harness for the NVFP4 path.

"Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4 W4A4 for the Recurrent Half of a
Hybrid 27B LLM", abstract, mechanisms ii-iv: the gate parameterisations shrink the gate
projections' quantisation error, the delta-rule recurrence holds injected noise at a flat
level over long contexts and forgets a state impulse within hundreds of steps (each write
overwrites the state along the current key), so per-token quantisation cost does not
compound. This module injects NVFP4 error where the quantised model puts it and measures,
with the library's kernels on the GPU, how much of it reaches the gates, the outputs and the
state:

  gate_compression   the gate projections (a, b) as one NVFP4 W4A4 GEMM with per-module
                     global scales, against the unquantised product; relative error of the
                     pre-activations and of alpha = exp(-exp(A_log) softplus(a + dt_bias)) and
                     beta = sigmoid(b) computed from them.
  noise_plateau      the chunked scan on NVFP4-round-tripped q, k, v against the clean scan:
                     relative output error per window of positions, and of the final state.
  impulse_response   the trajectory of a state impulse: the recurrence is linear in the state,
                     so the impulse's own trajectory is the scan with zero values started from
                     the impulse; its Frobenius norm after t tokens, per head, under fixed gates
                     whose decay rates 1 - alpha span 1e-3 .. 0.999 across heads.

Every measurement is a relative root-mean-square error ||x~ - x||_2 / ||x||_2 over the stated
elements. The unquantised reference of a product is a float64 matmul; gates are evaluated in
float64 from the pre-activations. Run `python -m gated_deltanet_03_b200.error_harness` for a
JSON report at the workloads' sizes.
"""
from __future__ import annotations

import math

import torch

from . import (gdn_prefill_chunked, gdn_prefill_workspace_bytes, nvfp4_dequantize_act, nvfp4_fused_col_alpha,
               nvfp4_gemm_colscale,
               nvfp4_quantize_act)

E2M1_MAX = 6.0
E4M3_MAX = 448.0


def rel_rms(x: torch.Tensor, ref: torch.Tensor) -> float:
    x, ref = x.double(), ref.double()
    den = torch.linalg.vector_norm(ref)
    return float(torch.linalg.vector_norm(x - ref) / den) if den > 0 else float(torch.linalg.vector_norm(x))


def global_scale(x: torch.Tensor) -> float:
    """The calibrated per-tensor NVFP4 scale: the largest magnitude lands on 448 * 6."""
    amax = float(x.float().abs().max())
    return E4M3_MAX * E2M1_MAX / amax if amax > 0 else 1.0


def nvfp4_roundtrip(x: torch.Tensor, gs: float | None = None):
    """x [M, K] (bf16 or fp32) through the NVFP4 encoder and back: (x_hat fp32 [M, K], gs)."""
    gs = global_scale(x) if gs is None else gs
    xq, xs = nvfp4_quantize_act(x.contiguous(), gs)
    return nvfp4_dequantize_act(xq, xs, gs), gs


def gates_f64(a: torch.Tensor, b: torch.Tensor, A_log: torch.Tensor, dt_bias: torch.Tensor):
    """alpha, beta [.., Hv] in float64 from pre-activations [.., Hv]."""
    a, b = a.double(), b.double()
    g = -torch.exp(A_log.double()) * torch.nn.functional.softplus(a + dt_bias.double())
    return torch.exp(g), torch.sigmoid(b)


def gate_compression(x: torch.Tensor, w_a: torch.Tensor, w_b: torch.Tensor, A_log: torch.Tensor,
                     dt_bias: torch.Tensor) -> dict:
    """x [M, K] bf16 activations, w_a, w_b [Hv, K] bf16 gate projections (two modules, each with
    its own NVFP4 global scale, fused into one GEMM with per-column factors)."""
    Hv = w_a.shape[0]
    exact = x.double() @ torch.cat([w_a, w_b]).double().T                # [M, 2 Hv]
    gx = global_scale(x)
    xq, xs = nvfp4_quantize_act(x, gx)
    scales = [global_scale(w_a), global_scale(w_b)]
    wq_a, ws_a = nvfp4_quantize_act(w_a, scales[0])
    wq_b, ws_b = nvfp4_quantize_act(w_b, scales[1])
    col_alpha = nvfp4_fused_col_alpha((Hv, Hv), scales, gx, device=x.device)
    quant = nvfp4_gemm_colscale(xq, xs, torch.cat([wq_a, wq_b]), torch.cat([ws_a, ws_b]), col_alpha,
                                out_dtype=torch.float32)
    a, b = exact[:, :Hv], exact[:, Hv:]
    aq, bq = quant[:, :Hv], quant[:, Hv:]
    alpha, beta = gates_f64(a, b, A_log, dt_bias)
    alpha_q, beta_q = gates_f64(aq, bq, A_log, dt_bias)
    out = {"preact_a": rel_rms(aq, a), "preact_b": rel_rms(bq, b), "alpha": rel_rms(alpha_q, alpha),
           "beta": rel_rms(beta_q, beta)}
    out["preact"] = rel_rms(quant, exact)
    out["gates"] = rel_rms(torch.cat([alpha_q, beta_q], 1), torch.cat([alpha, beta], 1))
    out["compression"] = out["preact"] / out["gates"] if out["gates"] > 0 else math.inf
    return out


def _scan(q, k, v, a, b, A_log, dt_bias, S0=None):
    T, Hk, D = q.shape
    Hv = v.shape[1]
    ws = torch.empty((max(1, gdn_prefill_workspace_bytes(T, 1, Hk, Hv, D, D)),), dtype=torch.uint8,
                     device=q.device)
    S = torch.empty((1, Hv, D, D), dtype=torch.float32, device=q.device)
    o, S = gdn_prefill_chunked(q, k, v, a, b, A_log, dt_bias, initial_state=S0, final_state=S,
                               out_dtype=torch.float32, workspace=ws)
    return o, S


def noise_plateau(q, k, v, a, b, A_log, dt_bias, window: int = 1024) -> dict:
    """One sequence: q, k [T, Hk, D], v [T, Hv, D] bf16 (a, b, gates fp32). The noisy run takes
    q, k, v through the NVFP4 encoder and back (one global scale per tensor) and rounds them to
    bf16, the scan's input type."""
    T = q.shape[0]

    def noisy(x):
        xh, _ = nvfp4_roundtrip(x.reshape(T, -1))
        return xh.to(torch.bfloat16).reshape(x.shape)

    qn, kn, vn = noisy(q), noisy(k), noisy(v)
    o, S = _scan(q, k, v, a, b, A_log, dt_bias)
    on, Sn = _scan(qn, kn, vn, a, b, A_log, dt_bias)
    wins = [rel_rms(on[i:i + window], o[i:i + window]) for i in range(0, T, window)]
    quarter = max(1, len(wins) // 4)
    return {"input_q": rel_rms(qn, q), "input_k": rel_rms(kn, k), "input_v": rel_rms(vn, v),
            "window": window, "output_per_window": wins, "final_state": rel_rms(Sn, S),
            "first_quarter_mean": sum(wins[:quarter]) / quarter,
            "last_quarter_mean": sum(wins[-quarter:]) / quarter,
            "last_over_first": (sum(wins[-quarter:]) / quarter) / max(sum(wins[:quarter]) / quarter, 1e-30)}


def decay_spectrum(Hv: int, lo: float = 1e-3, hi: float = 0.999):
    """Fixed per-head gates (a = 0, A_log = 0) whose decay rates 1 - alpha are log-spaced from hi
    down to lo: returns (alpha [Hv], A_log [Hv], dt_bias [Hv]) with
    softplus(dt_bias) = -log(alpha)."""
    rates = torch.logspace(math.log10(hi), math.log10(lo), Hv, dtype=torch.float64)
    alpha = 1.0 - rates
    dt_bias = torch.log(torch.expm1(-torch.log(alpha)))
    return alpha, torch.zeros(Hv, dtype=torch.float64), dt_bias


def impulse_response(q, k, b, A_log, dt_bias, impulse, steps) -> dict:
    """||S_t||_F / ||S_0||_F per head after each t in `steps`, for the state trajectory from
    S_0 = impulse [1, Hv, D, D] with zero values (v = 0, a = 0). Also the prediction from the
    decay gates alone (prod alpha) and from the decay plus the overwrite along random unit
    keys, prod alpha_t sqrt(1 - (2 beta_t - beta_t^2) / D). Give q, k in fp32: the scan then
    runs the all-fp32 recurrent kernel, which follows the impulse down to fp32's range (the
    tensor-core path stages the state in fp16, too coarse for an impulse decayed by 1e4)."""
    Tmax, Hk, D = q.shape
    Hv = b.shape[1]
    dev = q.device
    a0 = torch.zeros((Tmax, Hv), dtype=torch.float32, device=dev)
    v0 = torch.zeros((Tmax, Hv, D), dtype=q.dtype, device=dev)
    n0 = torch.linalg.vector_norm(impulse.double().reshape(Hv, -1), dim=1)
    alpha, beta = gates_f64(a0, b, A_log, dt_bias)                     # [T, Hv]
    log_gate = torch.cumsum(torch.log(alpha), 0)
    log_pred = torch.cumsum(torch.log(alpha) + 0.5 * torch.log1p(-(2 * beta - beta * beta) / D), 0)
    out = {"steps": list(steps), "measured": [], "gate_only": [], "overwrite_model": []}
    for t in steps:
        _, S = _scan(q[:t].contiguous(), k[:t].contiguous(), v0[:t].contiguous(), a0[:t].contiguous(),
                     b[:t].contiguous(), A_log, dt_bias, S0=impulse)
        nt = torch.linalg.vector_norm(S.double().reshape(Hv, -1), dim=1)
        out["measured"].append((nt / n0).tolist())
        out["gate_only"].append(torch.exp(log_gate[t - 1]).tolist())
        out["overwrite_model"].append(torch.exp(log_pred[t - 1]).tolist())
    return out


def _report(seed: int = 2024) -> dict:
    """The three measurements at the workloads' sizes: the gate GEMM of the long-prefill layer
    (4096 tokens x 2048 -> 2 x 32 gates), the noise plateau over 32768 tokens (16/32 heads) and
    the impulse response over 4096 tokens with 32 heads spanning the decay spectrum."""
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev).manual_seed(seed)
    bf = torch.bfloat16

    def randn(*shape, std=1.0):
        return (torch.randn(shape, generator=gen, device=dev) * std)

    M, K, Hv, Hk, D = 4096, 2048, 32, 16, 128
    A_log = torch.log(torch.empty(Hv, device=dev).uniform_(1.0, 16.0, generator=gen))
    dt_bias = torch.zeros(Hv, device=dev)
    xg, wa, wb = randn(M, K).to(bf), randn(Hv, K, std=K ** -0.5).to(bf), randn(Hv, K, std=K ** -0.5).to(bf)
    # two gate parameterisations: the workloads' (A_log ~ U(log 1, log 16), dt_bias = 0) and the
    # fixed spectrum of timescales the walkthrough page reports (decay rates 1e-3 .. 0.999)
    _, A_spec, dt_spec = decay_spectrum(Hv)
    gates = {"workload_gates": gate_compression(xg, wa, wb, A_log, dt_bias),
             "timescale_spectrum": gate_compression(xg, wa, wb, A_spec.float().to(dev), dt_spec.float().to(dev))}

    T = 32768
    q, k = randn(T, Hk, D).to(bf), randn(T, Hk, D).to(bf)
    v = randn(T, Hv, D).to(bf)
    a, b = randn(T, Hv), randn(T, Hv)
    plateau = noise_plateau(q, k, v, a, b, A_log, dt_bias, window=2048)

    alpha, A0, dtb = decay_spectrum(Hv)
    Ti = 4096
    imp = randn(1, Hv, D, D)
    impulse = impulse_response(q[:Ti].float(), k[:Ti].float(), b[:Ti].contiguous(),
                               A0.float().to(dev), dtb.float().to(dev), imp, (16, 64, 256, 1024, 4096))
    impulse["alpha"] = alpha.tolist()
    return {"gate_compression": gates, "noise_plateau": plateau, "impulse_response": impulse}


if __name__ == "__main__":
    import json
    print(json.dumps(_report()))
