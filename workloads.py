"""Seeded synthetic inputs for the Gated DeltaNet hot path.

This module only draws random numbers and lays them out; it holds none of the method's
arithmetic. The CUDA path (through its binding) and the CPU oracle both take their inputs
from here, so both sides see the same bytes: values that the path reads in bf16 are
rounded to bf16 once, here, and the oracle gets their exact fp32 widening.

Workload recipe (shapes of the hybrid-model layers the pages describe: value heads of 128
flattened to 2048/4096 and projected to 1024/2048; d_model 1024 with 16+16 heads):
  q, k, v, z ~ N(0, 1); a, b ~ N(0, 1); A_log ~ U(log 1, log 16); dt_bias = 0;
  norm weight ~ U(0.5, 1.5); projection weight ~ N(0, 0.02) (standard deviation);
  initial states, where non-zero, ~ N(0, 0.1) (standard deviation).
Variable-length lengths are log-uniform in [1024, 65536], seeded. Short convolution: x ~ N(0, 1),
weight ~ N(0, 1/K), carried history ~ N(0, 1).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str               # "prefill" or "decode"
    seqlens: tuple          # per-sequence lengths (decode: B ones)
    Hk: int
    Hv: int
    D: int
    io: str                 # "bf16" or "f32": dtype of q, k, v, z, o, y
    s0_std: float           # 0 => zero initial state
    n_out: int              # output projection width (K = Hv * D in)
    seed: int

    @property
    def T(self) -> int:
        return int(sum(self.seqlens))

    @property
    def num_seqs(self) -> int:
        return len(self.seqlens)

    @property
    def K(self) -> int:
        return self.Hv * self.D


def _varlen_lengths(seed: int, n: int = 8, lo: int = 1024, hi: int = 65536):
    rng = np.random.default_rng(seed)
    u = rng.uniform(math.log(lo), math.log(hi), size=n)
    return tuple(int(round(math.exp(x))) for x in u)


# The five workloads: tiny oracle case, 1024-wide prefill, 27B-class long prefill,
# batched decode, variable-length packed prefill.
TINY = Workload("tiny_T64_h2_d16_f32", "prefill", (64,), 2, 2, 16, "f32", 0.0, 16, 1000)
PREFILL_1K = Workload("prefill_T4096_hk16_hv16_d128", "prefill", (4096,), 16, 16, 128, "bf16",
                      0.0, 1024, 1001)
PREFILL_LONG = Workload("prefill_T32768_hk16_hv32_d128", "prefill", (32768,), 16, 32, 128,
                        "bf16", 0.0, 2048, 1002)
DECODE_B256 = Workload("decode_B256_hk16_hv32_d128", "decode", (1,) * 256, 16, 32, 128, "bf16",
                       0.1, 2048, 1003)
VARLEN_8 = Workload("varlen_N8_hk16_hv32_d128", "prefill", _varlen_lengths(1004), 16, 32, 128,
                    "bf16", 0.1, 2048, 1004)

WORKLOADS = [TINY, PREFILL_1K, PREFILL_LONG, DECODE_B256, VARLEN_8]


def custom(name: str, seqlens, Hk: int, Hv: int, D: int, io: str = "bf16", s0_std: float = 0.0,
           n_out: int = 64, seed: int = 7, kind: str = "prefill") -> Workload:
    return Workload(name, kind, tuple(int(x) for x in seqlens), Hk, Hv, D, io, s0_std, n_out,
                    seed)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even) and widen them back to fp32."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.bfloat16).float().numpy()


def _normal(rng, shape, std=1.0):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def generate(w: Workload) -> dict:
    """All inputs of one workload as host numpy arrays (fp32 values; the ones the path reads
    in bf16 are already bf16-rounded). Keys: q, k, v, z, a, b, A_log, dt_bias, cu_seqlens,
    initial_state (or None), norm_weight, proj_weight [n_out, K]."""
    rng = np.random.default_rng(w.seed)
    T, Hk, Hv, D = w.T, w.Hk, w.Hv, w.D
    bf = w.io == "bf16"
    rnd = round_bf16 if bf else (lambda x: x)
    out = {}
    out["q"] = rnd(_normal(rng, (T, Hk, D)))
    out["k"] = rnd(_normal(rng, (T, Hk, D)))
    out["v"] = rnd(_normal(rng, (T, Hv, D)))
    out["z"] = rnd(_normal(rng, (T, Hv, D)))
    out["a"] = _normal(rng, (T, Hv))
    out["b"] = _normal(rng, (T, Hv))
    out["A_log"] = rng.uniform(math.log(1.0), math.log(16.0), size=(Hv,)).astype(np.float32)
    out["dt_bias"] = np.zeros((Hv,), dtype=np.float32)
    cu = np.zeros((w.num_seqs + 1,), dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(w.seqlens, dtype=np.int64))
    out["cu_seqlens"] = cu
    out["initial_state"] = (_normal(rng, (w.num_seqs, Hv, D, D), w.s0_std)
                            if w.s0_std > 0 else None)
    out["norm_weight"] = rng.uniform(0.5, 1.5, size=(D,)).astype(np.float32)
    out["proj_weight"] = round_bf16(_normal(rng, (w.n_out, w.K), 0.02))
    return out


def activations(M: int, K: int, seed: int, std: float = 1.0, heavy_tail: bool = True,
                bf16: bool = True) -> np.ndarray:
    """A synthetic activation matrix [M, K] for quantiser tests: Gaussian rows, with a few
    blocks scaled up or zeroed (heavy_tail) so that block scales span their range and the
    all-zero block case appears."""
    rng = np.random.default_rng(seed)
    x = _normal(rng, (M, K), std)
    if heavy_tail and K >= 16:
        nblk = M * (K // 16)
        xb = x.reshape(nblk, 16)
        pick = rng.integers(0, nblk, size=max(1, nblk // 16))
        xb[pick] *= np.float32(64.0)
        pick = rng.integers(0, nblk, size=max(1, nblk // 64))
        xb[pick] *= np.float32(1.0 / 256.0)
        pick = rng.integers(0, nblk, size=max(1, nblk // 97))
        xb[pick] = 0.0
        x = xb.reshape(M, K)
    return round_bf16(x) if bf16 else x


def q4k_weights(N: int, K: int, seed: int) -> np.ndarray:
    """Synthetic Q4_K weights [N, K/256*144] uint8 (the page's 144-byte blocks of 256 values):
    per block f16 d ~ |N(1e-4, 2e-5)| and dmin = 7.5 d U(0.5, 1.5) (so the values d*scale*q -
    dmin*min spread around zero with a standard deviation of about 0.02), 12 random bytes of
    6-bit scales / mins, 128 random bytes of 4-bit quants. Random bytes only; the packing is
    whatever the bytes say."""
    rng = np.random.default_rng(seed)
    nb = N * (K // 256)
    blocks = rng.integers(0, 256, size=(nb, 144), dtype=np.uint8)
    d = np.abs(rng.normal(1e-4, 2e-5, size=nb)).astype(np.float16)
    dmin = (d.astype(np.float32) * 7.5 * rng.uniform(0.5, 1.5, size=nb)).astype(np.float16)
    blocks[:, 0:2] = d.view(np.uint8).reshape(nb, 2)
    blocks[:, 2:4] = dmin.view(np.uint8).reshape(nb, 2)
    return blocks.reshape(N, (K // 256) * 144)


def conv_inputs(T: int, C: int, K: int, seed: int, num_seqs: int = 1, state: bool = False) -> dict:
    """Inputs of the causal short convolution: x [T, C] ~ N(0, 1) (bf16-rounded), weight [C, K]
    ~ N(0, 1/K) fp32 (so the pre-activation is about unit scale), and, with state, a carried
    input history [num_seqs, K - 1, C] ~ N(0, 1) (bf16-rounded)."""
    rng = np.random.default_rng(seed)
    out = {"x": round_bf16(_normal(rng, (T, C))),
           "weight": _normal(rng, (C, K), 1.0 / math.sqrt(K))}
    out["initial_state"] = round_bf16(_normal(rng, (num_seqs, K - 1, C))) if state else None
    return out
