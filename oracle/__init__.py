"""Oracle for the Gated DeltaNet hot path: plain, slow CPU code (fp64; fp32 with a fixed
order of operations for the NVFP4 encode).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of
``bench.py`` (``cpu_baseline`` and ``--impl reference``) may import this package. The
product path (``gated_deltanet_03_b200``) never imports it, and the two share no code.

The arithmetic lives in ``gdn_oracle.c``; this module only marshals numpy arrays into it
and splits independent units (sequence x value-head for the scan, rows for the tail) over
host threads. The one library step is the GEMM over dequantised operands, which is an
fp64 ``numpy`` matrix product.

Each function cites the passage it follows (page title, section):
  * scan and gates: "Why Gated DeltaNet Survives 4-Bit Quantization" (abstract,
    mechanisms ii and iii), with the gated delta rule of "Gated Delta Networks"
    (Yang, Kautz, Hatamizadeh, ICLR 2025) as the explicit formula;
  * gated tail: "Red Lite dev15d - DeltaNet gated tail" (Pinned graph semantics, 1-6);
  * NVFP4: "Why Gated DeltaNet Survives 4-Bit Quantization" (abstract, mechanism i:
    16-element block scaling), E2M1 values with E4M3 block scales and an fp32 global
    scale;
  * Q4_K weights: "Red Lite dev15d - DeltaNet gated tail + Q4_K output projection" (Q4_K
    implementation: 256-value blocks of 144 bytes);
  * short convolution: "A Node-by-Node White-Box Walkthrough of a Quantized Hybrid Gated
    DeltaNet Language Model" (Principais Contribuicoes, item 2: the short convolutions on the
    layer's path), read as the depthwise causal convolution of width K followed by SiLU.

Parity pins: every function here is checked by ``tests/test_oracle_pins.py`` against
closed forms, invariants, library routines or brute force. None is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

EPS_QK = 1e-6
EPS_NORM = 1e-6


def build(force: bool = False) -> str:
    """Compile ``gdn_oracle.c`` into ``liboracle.so`` (plain gcc, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-ffp-contract=off", "-fPIC",
                               "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    i32, i64, f32, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_double
    lib.oracle_gdn_scan.argtypes = [i32, P, i32, i32, i32, i32, P, P, P, P, P, P, P,
                                    f64, i32, f64, P, P, P, i32, i32]
    lib.oracle_gdn_scan.restype = ctypes.c_int
    lib.oracle_gates.argtypes = [f64, f64, f64, f64, P, P, P]
    lib.oracle_gates.restype = None
    lib.oracle_gated_rmsnorm_silu.argtypes = [i32, i32, i32, P, P, P, f64, P, i32, i32]
    lib.oracle_gated_rmsnorm_silu.restype = None
    lib.oracle_nvfp4_quantize.argtypes = [i32, i32, P, f32, P, P, i32, i32]
    lib.oracle_nvfp4_quantize.restype = None
    lib.oracle_nvfp4_dequantize.argtypes = [i32, i32, P, P, f32, P, i32, i32]
    lib.oracle_nvfp4_dequantize.restype = None
    lib.oracle_e2m1_encode_many.argtypes = [i64, P, P]
    lib.oracle_e4m3_encode_many.argtypes = [i64, P, P]
    lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e2m1_decode.restype = f32
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = f32
    lib.oracle_f16_decode.argtypes = [ctypes.c_uint16]
    lib.oracle_f16_decode.restype = f64
    lib.oracle_q4k_dequantize.argtypes = [i32, i32, P, P, i32, i32]
    lib.oracle_q4k_dequantize.restype = None
    _lib = lib
    return lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(np.asarray(a, dtype=dtype))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _split(n: int, parts: int):
    parts = max(1, min(parts, n))
    edges = [n * i // parts for i in range(parts + 1)]
    return [(edges[i], edges[i + 1]) for i in range(parts) if edges[i + 1] > edges[i]]


def gates(a: float, b: float, A_log: float, dt_bias: float):
    """(g, alpha, beta) for one token and head: g = -exp(A_log) softplus(a + dt_bias),
    alpha = exp(g), beta = sigmoid(b) ("Why Gated DeltaNet Survives 4-Bit Quantization",
    abstract, mechanism ii)."""
    lib = _load()
    out = [ctypes.c_double() for _ in range(3)]
    lib.oracle_gates(a, b, A_log, dt_bias, *[ctypes.byref(x) for x in out])
    return tuple(x.value for x in out)


def gdn_scan(q, k, v, a, b, A_log, dt_bias, cu_seqlens=None, initial_state=None,
             scale: float = 1.0, qk_l2norm: bool = True, eps: float = EPS_QK,
             units=None, threads: int | None = None):
    """Sequential gated delta rule (fp64), token by token.

    q, k: [T, Hk, Dk]; v: [T, Hv, Dv]; a, b: [T, Hv]; A_log, dt_bias: [Hv];
    cu_seqlens: [N+1] int (None = one sequence); initial_state: [N, Hv, Dv, Dk] or None.
    Returns (o [T, Hv, Dv] fp64, final_state [N, Hv, Dv, Dk] fp64).
    ``units`` (optional iterable of n*Hv + h) restricts the work to those units; the
    others are left as zeros in both outputs.
    """
    lib = _load()
    q, k, v = _c(q, np.float32), _c(k, np.float32), _c(v, np.float32)
    a, b = _c(a, np.float32), _c(b, np.float32)
    A_log, dt_bias = _c(A_log, np.float32), _c(dt_bias, np.float32)
    T, Hk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    if cu_seqlens is None:
        cu_seqlens = np.array([0, T], dtype=np.int32)
    cu = _c(cu_seqlens, np.int32)
    N = cu.shape[0] - 1
    S0 = None if initial_state is None else _c(initial_state, np.float64)
    S = np.zeros((N, Hv, Dv, Dk), dtype=np.float64)
    o = np.zeros((T, Hv, Dv), dtype=np.float64)
    if units is None:
        ranges = _split(N * Hv, threads or default_threads())
    else:
        ranges = [(u, u + 1) for u in sorted(set(int(u) for u in units))]

    def run(r):
        rc = lib.oracle_gdn_scan(N, _ptr(cu), Hk, Hv, Dk, Dv, _ptr(q), _ptr(k), _ptr(v),
                                 _ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias), float(scale),
                                 int(bool(qk_l2norm)), float(eps), _ptr(S0), _ptr(S), _ptr(o),
                                 r[0], r[1])
        if rc != 0:
            raise ValueError("oracle_gdn_scan: bad sizes")

    with ThreadPoolExecutor(max_workers=threads or default_threads()) as ex:
        list(ex.map(run, ranges))
    return o, S


def gated_rmsnorm_silu(o, z, weight, eps: float = EPS_NORM, threads: int | None = None):
    """y[m, h*D+i] = o[m,h,i] / sqrt(mean_i o[m,h,:]^2 + eps) * w[i] * SiLU(z[m,h,i]),
    fp64 ("Red Lite dev15d - DeltaNet gated tail", Pinned graph semantics, steps 1-5).
    o, z: [M, Hv, D]; weight: [D]. Returns y [M, Hv*D] fp64."""
    lib = _load()
    o, z, w = _c(o, np.float32), _c(z, np.float32), _c(weight, np.float32)
    M, Hv, D = o.shape
    y = np.zeros((M, Hv * D), dtype=np.float64)

    def run(r):
        lib.oracle_gated_rmsnorm_silu(M, Hv, D, _ptr(o), _ptr(z), _ptr(w), float(eps), _ptr(y),
                                      r[0], r[1])

    with ThreadPoolExecutor(max_workers=threads or default_threads()) as ex:
        list(ex.map(run, _split(M, threads or default_threads())))
    return y


def nvfp4_quantize(x, global_scale: float, threads: int | None = None):
    """NVFP4 encode of x [M, K] (fp32 values; K % 16 == 0) with the fp32 global encode
    scale: returns (xq [M, K/2] uint8, two E2M1 codes per byte, element 2j in the low
    nibble; xs [M, K/16] uint8 E4M3 block scales)."""
    lib = _load()
    x = _c(x, np.float32)
    M, K = x.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    xq = np.zeros((M, K // 2), dtype=np.uint8)
    xs = np.zeros((M, K // 16), dtype=np.uint8)

    def run(r):
        lib.oracle_nvfp4_quantize(M, K, _ptr(x), float(np.float32(global_scale)), _ptr(xq),
                                  _ptr(xs), r[0], r[1])

    with ThreadPoolExecutor(max_workers=threads or default_threads()) as ex:
        list(ex.map(run, _split(M, threads or default_threads())))
    return xq, xs


def nvfp4_dequantize(xq, xs, global_scale: float, threads: int | None = None):
    """x_hat = E2M1(code) * E4M3(block scale) / global_scale, fp64 [M, K]."""
    lib = _load()
    xq, xs = _c(xq, np.uint8), _c(xs, np.uint8)
    M, K = xq.shape[0], xq.shape[1] * 2
    out = np.zeros((M, K), dtype=np.float64)

    def run(r):
        lib.oracle_nvfp4_dequantize(M, K, _ptr(xq), _ptr(xs), float(np.float32(global_scale)),
                                    _ptr(out), r[0], r[1])

    with ThreadPoolExecutor(max_workers=threads or default_threads()) as ex:
        list(ex.map(run, _split(M, threads or default_threads())))
    return out


def nvfp4_gemm(aq, as_, gs_a: float, bq, bs, gs_b: float, rows=None):
    """Y = A_hat @ B_hat^T in fp64 over the dequantised NVFP4 operands (A [M, K], B [N, K],
    K contiguous). ``rows`` optionally selects rows of A. The product is a library fp64
    matrix multiply; the global scales are folded into the dequantisation."""
    if rows is not None:
        rows = np.asarray(rows)
        aq, as_ = np.asarray(aq)[rows], np.asarray(as_)[rows]
    A = nvfp4_dequantize(aq, as_, gs_a)
    B = nvfp4_dequantize(bq, bs, gs_b)
    return A @ B.T


def q4k_dequantize(w, K: int, threads: int | None = None):
    """Q4_K weights w [N, K/256*144] uint8 -> fp64 [N, K] (exact): "Red Lite dev15d - DeltaNet
    gated tail + Q4_K output projection", section "Q4_K implementation" (256-value blocks of
    144 bytes: f16 d, f16 dmin, 12 bytes of 6-bit scales / mins, 128 bytes of 4-bit quants;
    value = d * scale * q - dmin * min; bit positions as in gdn_oracle.c)."""
    lib = _load()
    w = _c(w, np.uint8)
    N = w.shape[0]
    if K % 256 or w.shape[1] != K // 256 * 144:
        raise ValueError("w must be [N, K/256*144] with K % 256 == 0")
    out = np.zeros((N, K), dtype=np.float64)

    def run(r):
        lib.oracle_q4k_dequantize(N, K, _ptr(w), _ptr(out), r[0], r[1])

    with ThreadPoolExecutor(max_workers=threads or default_threads()) as ex:
        list(ex.map(run, _split(N, threads or default_threads())))
    return out


def q4k_gemm(a, w, K: int, rows=None):
    """Y = A @ W^T in fp64 with W the dequantised Q4_K weights (A [M, K] fp32 values, W [N, K]);
    ``rows`` optionally selects rows of A. The product is a library fp64 matrix multiply."""
    a = np.asarray(a, dtype=np.float64)
    if rows is not None:
        a = a[np.asarray(rows)]
    return a @ q4k_dequantize(w, K).T


def f16_decode(h):
    """fp64 values of IEEE binary16 bit patterns."""
    lib = _load()
    h = np.asarray(h, dtype=np.uint16).ravel()
    return np.array([lib.oracle_f16_decode(int(x)) for x in h], dtype=np.float64)


def e2m1_encode(x):
    """E2M1 codes (round to nearest, ties to even code, saturating at 6, sign kept)."""
    lib = _load()
    x = _c(x, np.float32).ravel()
    out = np.zeros(x.shape, dtype=np.uint8)
    lib.oracle_e2m1_encode_many(x.size, _ptr(x), _ptr(out))
    return out


def e4m3_encode(x):
    """Non-negative E4M3 codes (round to nearest, ties to even code, saturating at 448)."""
    lib = _load()
    x = _c(x, np.float32).ravel()
    out = np.zeros(x.shape, dtype=np.uint8)
    lib.oracle_e4m3_encode_many(x.size, _ptr(x), _ptr(out))
    return out


def e2m1_decode(codes):
    lib = _load()
    return np.array([lib.oracle_e2m1_decode(int(c)) for c in np.asarray(codes).ravel()],
                    dtype=np.float32)


def e4m3_decode(codes):
    lib = _load()
    return np.array([lib.oracle_e4m3_decode(int(c)) for c in np.asarray(codes).ravel()],
                    dtype=np.float32)


def short_conv1d_silu(x, weight, cu_seqlens=None, initial_state=None):
    """Depthwise causal convolution of width K over each sequence, then SiLU, in fp64:
    y[t, c] = SiLU(sum_{j<K} weight[c, j] x[t - (K - 1) + j, c]), where inputs before a
    sequence's first token come from initial_state[n] ([K - 1, C], oldest first) or are zero.
    x [T, C]; weight [C, K]; cu_seqlens [N + 1] or None (one sequence).
    Returns (y [T, C] fp64, final_state [N, K - 1, C]: each sequence's last K - 1 inputs,
    continuing the initial state when the sequence is shorter)."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(weight, dtype=np.float64)
    T, C = x.shape
    K = w.shape[1]
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(cu_seqlens)
    N = len(cu) - 1
    y = np.zeros((T, C))
    final = np.zeros((N, K - 1, C))
    for n in range(N):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        hist = np.zeros((K - 1, C)) if initial_state is None else np.asarray(initial_state[n], dtype=np.float64)
        window = np.concatenate([hist, x[t0:t1]], axis=0)     # row K - 1 + i is token t0 + i
        for i in range(t1 - t0):
            acc = np.zeros(C)
            for j in range(K):
                acc += w[:, j] * window[i + j]
            y[t0 + i] = acc / (1.0 + np.exp(-acc))
        final[n] = window[len(window) - (K - 1):] if K > 1 else final[n]
    return y, final
