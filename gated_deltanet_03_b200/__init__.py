"""Python binding of the Gated DeltaNet B200 library (libgdn_b200.so, C ABI in include/gdn.h).

Argument marshalling only: every step of the path runs in the library's CUDA kernels.
PyTorch provides device memory (output tensors are allocated with torch) and the current
stream. There is no CPU fallback: if the library is missing, importing this package raises.

Functions keep the C names:
  gdn_prefill_chunked, gdn_prefill_chunked_gated_nvfp4, gdn_decode_step, gdn_decode_verify,
  gdn_decode_commit, gdn_gated_rmsnorm_silu,
  gdn_gated_rmsnorm_silu_nvfp4, nvfp4_quantize_act, nvfp4_dequantize_act, nvfp4_gemm,
  nvfp4_gemm_colscale, gdn_short_conv1d_silu, gdn_short_conv1d_silu_decode,
  gdn_prefill_workspace_bytes, gdn_get_device_status.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn_b200.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT, GDN_ERR_WORKSPACE = range(6)
GDN_BF16, GDN_F32 = 0, 1

# Exported C symbols, in the order include/gdn.h declares them.
ABI_SYMBOLS = (
    "gdn_prefill_chunked", "gdn_prefill_workspace_bytes", "gdn_prefill_chunked_gated_nvfp4", "gdn_decode_step",
    "gdn_decode_step_gated_nvfp4",
    "gdn_decode_verify", "gdn_decode_commit",
    "gdn_gated_rmsnorm_silu", "gdn_gated_rmsnorm_silu_nvfp4", "nvfp4_quantize_act", "nvfp4_dequantize_act",
    "nvfp4_gemm", "nvfp4_gemm_colscale", "nvfp4_fused_col_alpha", "q4k_gemm", "gdn_short_conv1d_silu", "gdn_short_conv1d_silu_decode",
    "gdn_prefill_chunked_static_ws", "gdn_get_device_status", "gdn_debug_set_wait", "gdn_status_string",
    "gdn_version",
)


class GdnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (fn, status_string(status), status))


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError("libgdn_b200.so is not built (run __graft_entry__.build() or "
                          "python gated_deltanet_03_b200/build.py)")
    lib = ctypes.CDLL(LIB_PATH)
    P, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    lib.gdn_prefill_chunked.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32,
                                        i32, P, P, P, i32, P, sz, P]
    lib.gdn_prefill_chunked_gated_nvfp4.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32,
                                                    i32, i32, P, P, P, P, P, f32, f32, P, P, P, sz, P]
    lib.gdn_prefill_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
    lib.gdn_prefill_workspace_bytes.restype = sz
    lib.gdn_decode_step.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, f32, i32, i32, P, P,
                                    i32, P]
    lib.gdn_decode_step_gated_nvfp4.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, f32, i32, i32, P, P, P,
                                                f32, f32, P, P, P, P]
    lib.gdn_decode_verify.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32, i32, P, P, P,
                                      i32, P]
    lib.gdn_decode_commit.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32, i32, P, P, P]
    lib.gdn_gated_rmsnorm_silu.argtypes = [P, P, P, f32, i32, i32, i32, i32, P, i32, P]
    lib.gdn_gated_rmsnorm_silu_nvfp4.argtypes = [P, P, P, f32, i32, i32, i32, i32, f32, P, P, P]
    lib.nvfp4_quantize_act.argtypes = [P, i32, i32, i32, f32, P, P, P]
    lib.nvfp4_dequantize_act.argtypes = [P, P, i32, i32, f32, i32, P, P]
    lib.nvfp4_gemm.argtypes = [P, P, P, P, f32, i32, i32, i32, i32, P, P]
    lib.nvfp4_gemm_colscale.argtypes = [P, P, P, P, P, i32, i32, i32, i32, P, P]
    lib.nvfp4_fused_col_alpha.argtypes = [P, P, i32, f32, P, P]
    lib.q4k_gemm.argtypes = [P, P, i32, i32, i32, i32, P, P]
    i64 = ctypes.c_int64
    lib.gdn_short_conv1d_silu.argtypes = [P, i64, P, P, i32, i32, i32, i32, P, P, P, P, i32, P]
    lib.gdn_short_conv1d_silu_decode.argtypes = [P, i64, P, i32, i32, i32, P, P, P, i32, P]
    lib.gdn_prefill_chunked_static_ws.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32,
                                                  i32, i32, P, P, P, i32, P]
    lib.gdn_get_device_status.argtypes = [P]
    lib.gdn_debug_set_wait.argtypes = [ctypes.c_uint64, ctypes.c_uint32]
    lib.gdn_status_string.argtypes = [i32]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_version.restype = i32
    for name in ("gdn_prefill_chunked", "gdn_prefill_chunked_gated_nvfp4", "gdn_prefill_chunked_static_ws", "gdn_decode_step",
                 "gdn_decode_step_gated_nvfp4", "gdn_decode_verify",
                 "gdn_decode_commit", "gdn_gated_rmsnorm_silu",
                 "gdn_gated_rmsnorm_silu_nvfp4", "nvfp4_quantize_act", "nvfp4_dequantize_act", "nvfp4_gemm",
                 "nvfp4_gemm_colscale", "nvfp4_fused_col_alpha", "q4k_gemm",
                 "gdn_short_conv1d_silu", "gdn_short_conv1d_silu_decode", "gdn_get_device_status", "gdn_debug_set_wait"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


LIB = _load()


def status_string(s: int) -> str:
    return LIB.gdn_status_string(int(s)).decode()


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError("unsupported dtype %s (bf16 or fp32)" % t.dtype)


def _dt_of(dtype) -> int:
    return GDN_BF16 if dtype == torch.bfloat16 else GDN_F32


def _check(name: str, status: int):
    if status != GDN_OK:
        raise GdnError(name, status)


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


_F32, _I32, _U8 = (torch.float32,), (torch.int32,), (torch.uint8,)
_IO = (torch.bfloat16, torch.float32)


def _args(device, **named):
    """Host-side checks before any launch, so that no kernel reads memory it was not given: a
    (dtypes, min_elems) pair after a tensor checks its dtype and that it holds at least the
    elements the call reads or writes (all tensors first), then every tensor must be a CUDA
    tensor on `device`."""
    given = [(name,) + (spec if isinstance(spec, tuple) else (spec, None, None)) for name, spec in named.items()]
    given = [x for x in given if x[1] is not None]
    for name, t, dtypes, need in given:
        if not isinstance(t, torch.Tensor):
            raise TypeError("%s must be a torch.Tensor" % name)
        if dtypes is not None and t.dtype not in dtypes:
            raise TypeError("%s must be %s (got %s)" % (name, " or ".join(map(str, dtypes)), t.dtype))
        if need is not None and t.numel() < need:
            raise ValueError("%s holds %d elements, the call needs %d" % (name, t.numel(), need))
    for name, t, _, _ in given:
        if t.device.type != "cuda":
            raise ValueError("%s must be a CUDA tensor (got %s)" % (name, t.device))
        if t.device != device:
            raise ValueError("%s is on %s, the call's other tensors on %s" % (name, t.device, device))


def gdn_prefill_workspace_bytes(T, num_seqs, Hk, Hv, Dk, Dv) -> int:
    return int(LIB.gdn_prefill_workspace_bytes(T, num_seqs, Hk, Hv, Dk, Dv))


def gdn_prefill_chunked(q, k, v, a, b, A_log, dt_bias, cu_seqlens=None, initial_state=None,
                        final_state=None, scale: float = 1.0, qk_l2norm: bool = True,
                        out_dtype=None, o=None, workspace=None, stream=None):
    """Gated delta rule over packed sequences. q, k [T, Hk, D]; v [T, Hv, D]; a, b [T, Hv] fp32;
    A_log, dt_bias [Hv] fp32; cu_seqlens int32 [N+1] on the device or None.
    Returns (o [T, Hv, D], final_state [N, Hv, D, D] fp32)."""
    T, Hk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    out_dtype = out_dtype or q.dtype
    _args(q.device, q=(q, _IO, None), k=(k, (q.dtype,), T * Hk * Dk), v=(v, (q.dtype,), T * Hv * Dv),
          a=(a, _F32, T * Hv), b=(b, _F32, T * Hv), A_log=(A_log, _F32, Hv), dt_bias=(dt_bias, _F32, Hv),
          cu_seqlens=(cu_seqlens, _I32, None), initial_state=(initial_state, _F32, N * Hv * Dv * Dk),
          final_state=(final_state, _F32, N * Hv * Dv * Dk), o=(o, _IO, T * Hv * Dv),
          workspace=(workspace, _U8, None))
    if o is None:
        o = torch.empty((T, Hv, Dv), dtype=out_dtype, device=q.device)
    if final_state is None:
        final_state = torch.empty((N, Hv, Dv, Dk), dtype=torch.float32, device=q.device)
    _contig(q, k, v, a, b, A_log, dt_bias, cu_seqlens, initial_state, final_state, o)
    ws_bytes = gdn_prefill_workspace_bytes(T, N, Hk, Hv, Dk, Dv)
    if ws_bytes and workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=q.device)
    st = LIB.gdn_prefill_chunked(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(A_log),
                                 _ptr(dt_bias), _ptr(cu_seqlens), N, T, Hk, Hv, Dk, Dv,
                                 float(scale), int(bool(qk_l2norm)), _dt(q), _ptr(initial_state),
                                 _ptr(final_state), _ptr(o), _dt(o), _ptr(workspace),
                                 0 if workspace is None else workspace.numel(), _stream(stream))
    _check("gdn_prefill_chunked", st)
    return o, final_state


def gdn_prefill_chunked_gated_nvfp4(q, k, v, a, b, A_log, dt_bias, z, norm_weight, global_scale: float,
                                    cu_seqlens=None, initial_state=None, final_state=None, scale: float = 1.0,
                                    qk_l2norm: bool = True, eps: float = 1e-6, o=None, write_o: bool = False,
                                    xq=None, xs=None, workspace=None, stream=None):
    """Prefill whose output pass also applies the gated RMSNorm and writes NVFP4 activations.
    q, k [T, Hk, 128] bf16; v, z [T, Hv, 128] bf16; norm_weight [128] fp32.
    Returns (xq [T, Hv*64] u8, xs [T, Hv*8] u8, final_state, o or None); o (bf16) is written only
    when given or when write_o is set."""
    T, Hk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    _args(q.device, q=(q, _IO, None), k=(k, (q.dtype,), T * Hk * Dk), v=(v, (q.dtype,), T * Hv * Dv),
          a=(a, _F32, T * Hv), b=(b, _F32, T * Hv), A_log=(A_log, _F32, Hv), dt_bias=(dt_bias, _F32, Hv),
          z=(z, (q.dtype,), T * Hv * Dv), norm_weight=(norm_weight, _F32, Dv),
          cu_seqlens=(cu_seqlens, _I32, None), initial_state=(initial_state, _F32, N * Hv * Dv * Dk),
          final_state=(final_state, _F32, N * Hv * Dv * Dk), o=(o, _IO, T * Hv * Dv),
          xq=(xq, _U8, T * Hv * Dv // 2), xs=(xs, _U8, T * Hv * Dv // 16), workspace=(workspace, _U8, None))
    if o is None and write_o:
        o = torch.empty((T, Hv, Dv), dtype=torch.bfloat16, device=q.device)
    if final_state is None:
        final_state = torch.empty((N, Hv, Dv, Dk), dtype=torch.float32, device=q.device)
    if xq is None:
        xq = torch.empty((T, Hv * Dv // 2), dtype=torch.uint8, device=q.device)
    if xs is None:
        xs = torch.empty((T, Hv * Dv // 16), dtype=torch.uint8, device=q.device)
    _contig(q, k, v, a, b, A_log, dt_bias, cu_seqlens, initial_state, final_state, o, z, norm_weight, xq, xs)
    ws_bytes = gdn_prefill_workspace_bytes(T, N, Hk, Hv, Dk, Dv)
    if ws_bytes and workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=q.device)
    st = LIB.gdn_prefill_chunked_gated_nvfp4(
        _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias), _ptr(cu_seqlens), N, T, Hk, Hv,
        Dk, Dv, float(scale), int(bool(qk_l2norm)), _dt(q), _ptr(initial_state), _ptr(final_state), _ptr(o),
        _ptr(z), _ptr(norm_weight), float(eps), float(global_scale), _ptr(xq), _ptr(xs), _ptr(workspace),
        0 if workspace is None else workspace.numel(), _stream(stream))
    _check("gdn_prefill_chunked_gated_nvfp4", st)
    return xq, xs, final_state, o


def gdn_decode_step(q, k, v, a, b, A_log, dt_bias, state, scale: float = 1.0,
                    qk_l2norm: bool = True, out_dtype=None, o=None, stream=None):
    """One token per sequence; `state` [B, Hv, D, D] fp32 is updated in place. Returns o."""
    B, Hk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    out_dtype = out_dtype or q.dtype
    _args(q.device, q=(q, _IO, None), k=(k, (q.dtype,), B * Hk * Dk), v=(v, (q.dtype,), B * Hv * Dv),
          a=(a, _F32, B * Hv), b=(b, _F32, B * Hv), A_log=(A_log, _F32, Hv), dt_bias=(dt_bias, _F32, Hv),
          state=(state, _F32, B * Hv * Dv * Dk), o=(o, _IO, B * Hv * Dv))
    if state is None:
        raise ValueError("state is required")
    if o is None:
        o = torch.empty((B, Hv, Dv), dtype=out_dtype, device=q.device)
    _contig(q, k, v, a, b, A_log, dt_bias, state, o)
    st = LIB.gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias),
                             B, Hk, Hv, Dk, Dv, float(scale), int(bool(qk_l2norm)), _dt(q),
                             _ptr(state), _ptr(o), _dt(o), _stream(stream))
    _check("gdn_decode_step", st)
    return o


def gdn_decode_step_gated_nvfp4(q, k, v, a, b, A_log, dt_bias, state, z, norm_weight, global_scale: float,
                                scale: float = 1.0, qk_l2norm: bool = True, eps: float = 1e-6, xq=None, xs=None,
                                o=None, stream=None):
    """One token per sequence (d = 128, bf16) with the gated RMSNorm and NVFP4 encode fused:
    `state` [B, Hv, 128, 128] fp32 is updated in place. Returns (xq [B, Hv*64], xs [B, Hv*8], o or None)."""
    B, Hk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    _args(q.device, q=(q, (torch.bfloat16,), None), k=(k, (torch.bfloat16,), B * Hk * Dk),
          v=(v, (torch.bfloat16,), B * Hv * Dv), a=(a, _F32, B * Hv), b=(b, _F32, B * Hv), A_log=(A_log, _F32, Hv),
          dt_bias=(dt_bias, _F32, Hv), state=(state, _F32, B * Hv * Dv * Dk), z=(z, (torch.bfloat16,), B * Hv * Dv),
          norm_weight=(norm_weight, _F32, Dv), xq=(xq, _U8, B * Hv * Dv // 2), xs=(xs, _U8, B * Hv * Dv // 16),
          o=(o, (torch.bfloat16,), B * Hv * Dv))
    if xq is None:
        xq = torch.empty((B, Hv * Dv // 2), dtype=torch.uint8, device=q.device)
    if xs is None:
        xs = torch.empty((B, Hv * Dv // 16), dtype=torch.uint8, device=q.device)
    _contig(q, k, v, a, b, A_log, dt_bias, state, z, norm_weight, xq, xs, o)
    st = LIB.gdn_decode_step_gated_nvfp4(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias),
                                         B, Hk, Hv, Dk, Dv, float(scale), int(bool(qk_l2norm)), _dt(q), _ptr(state),
                                         _ptr(z), _ptr(norm_weight), float(eps), float(global_scale), _ptr(xq),
                                         _ptr(xs), _ptr(o), _stream(stream))
    _check("gdn_decode_step_gated_nvfp4", st)
    return xq, xs, o


def gdn_decode_verify(q, k, v, a, b, A_log, dt_bias, state, scale: float = 1.0, qk_l2norm: bool = True,
                      final_state=None, out_dtype=None, o=None, stream=None):
    """T draft tokens per sequence: q, k [B, T, Hk, D], v [B, T, Hv, D], a, b [B, T, Hv];
    `state` [B, Hv, D, D] fp32 is only read. Returns o [B, T, Hv, D] (final_state, if given,
    receives the state after all T tokens)."""
    B, T, Hk, Dk = q.shape
    Hv, Dv = v.shape[2], v.shape[3]
    out_dtype = out_dtype or q.dtype
    _args(q.device, q=(q, _IO, None), k=(k, (q.dtype,), B * T * Hk * Dk), v=(v, (q.dtype,), B * T * Hv * Dv),
          a=(a, _F32, B * T * Hv), b=(b, _F32, B * T * Hv), A_log=(A_log, _F32, Hv), dt_bias=(dt_bias, _F32, Hv),
          state=(state, _F32, B * Hv * Dv * Dk), final_state=(final_state, _F32, B * Hv * Dv * Dk),
          o=(o, _IO, B * T * Hv * Dv))
    if state is None:
        raise ValueError("state is required")
    if o is None:
        o = torch.empty((B, T, Hv, Dv), dtype=out_dtype, device=q.device)
    _contig(q, k, v, a, b, A_log, dt_bias, state, final_state, o)
    st = LIB.gdn_decode_verify(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias),
                               B, T, Hk, Hv, Dk, Dv, float(scale), int(bool(qk_l2norm)), _dt(q), _ptr(state),
                               _ptr(final_state), _ptr(o), _dt(o), _stream(stream))
    _check("gdn_decode_verify", st)
    return o


def gdn_decode_commit(q, k, v, a, b, A_log, dt_bias, state, accepted, scale: float = 1.0,
                      qk_l2norm: bool = True, stream=None):
    """Advance `state` in place by the first accepted[b] (device int32 [B]) of each sequence's
    T draft tokens (the same tensors as the gdn_decode_verify call)."""
    B, T, Hk, Dk = q.shape
    Hv, Dv = v.shape[2], v.shape[3]
    _args(q.device, q=(q, _IO, None), k=(k, (q.dtype,), B * T * Hk * Dk), v=(v, (q.dtype,), B * T * Hv * Dv),
          a=(a, _F32, B * T * Hv), b=(b, _F32, B * T * Hv), A_log=(A_log, _F32, Hv), dt_bias=(dt_bias, _F32, Hv),
          state=(state, _F32, B * Hv * Dv * Dk), accepted=(accepted, _I32, B))
    if state is None or accepted is None:
        raise ValueError("state and accepted are required")
    _contig(q, k, v, a, b, A_log, dt_bias, state, accepted)
    st = LIB.gdn_decode_commit(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias),
                               B, T, Hk, Hv, Dk, Dv, float(scale), int(bool(qk_l2norm)), _dt(q), _ptr(accepted),
                               _ptr(state), _stream(stream))
    _check("gdn_decode_commit", st)
    return state


def gdn_gated_rmsnorm_silu(o, z, weight, eps: float = 1e-6, out_dtype=None, y=None, stream=None):
    """o, z [M, Hv, D] -> y [M, Hv * D]."""
    M, Hv, D = o.shape
    out_dtype = out_dtype or o.dtype
    _args(o.device, o=(o, _IO, None), z=(z, (o.dtype,), M * Hv * D), weight=(weight, _F32, D),
          y=(y, _IO, M * Hv * D))
    if y is None:
        y = torch.empty((M, Hv * D), dtype=out_dtype, device=o.device)
    _contig(o, z, weight, y)
    st = LIB.gdn_gated_rmsnorm_silu(_ptr(o), _ptr(z), _ptr(weight), float(eps), M, Hv, D, _dt(o),
                                    _ptr(y), _dt(y), _stream(stream))
    _check("gdn_gated_rmsnorm_silu", st)
    return y


def gdn_gated_rmsnorm_silu_nvfp4(o, z, weight, global_scale: float, eps: float = 1e-6,
                                 xq=None, xs=None, stream=None):
    """o, z [M, Hv, D] -> (xq [M, K/2] uint8, xs [M, K/16] uint8), K = Hv * D."""
    M, Hv, D = o.shape
    K = Hv * D
    _args(o.device, o=(o, _IO, None), z=(z, (o.dtype,), M * K), weight=(weight, _F32, D),
          xq=(xq, _U8, M * K // 2), xs=(xs, _U8, M * K // 16))
    if xq is None:
        xq = torch.empty((M, K // 2), dtype=torch.uint8, device=o.device)
    if xs is None:
        xs = torch.empty((M, K // 16), dtype=torch.uint8, device=o.device)
    _contig(o, z, weight, xq, xs)
    st = LIB.gdn_gated_rmsnorm_silu_nvfp4(_ptr(o), _ptr(z), _ptr(weight), float(eps), M, Hv, D, _dt(o),
                                          float(global_scale), _ptr(xq), _ptr(xs), _stream(stream))
    _check("gdn_gated_rmsnorm_silu_nvfp4", st)
    return xq, xs


def nvfp4_quantize_act(x, global_scale: float, xq=None, xs=None, stream=None):
    """x [M, K] bf16/fp32 -> (xq [M, K/2] uint8, xs [M, K/16] uint8)."""
    M, K = x.shape
    _args(x.device, x=(x, _IO, None), xq=(xq, _U8, M * K // 2), xs=(xs, _U8, M * K // 16))
    if xq is None:
        xq = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    if xs is None:
        xs = torch.empty((M, K // 16), dtype=torch.uint8, device=x.device)
    _contig(x, xq, xs)
    st = LIB.nvfp4_quantize_act(_ptr(x), _dt(x), M, K, float(global_scale), _ptr(xq), _ptr(xs),
                                _stream(stream))
    _check("nvfp4_quantize_act", st)
    return xq, xs


def nvfp4_dequantize_act(xq, xs, global_scale: float, out_dtype=torch.float32, y=None, stream=None):
    """(xq [M, K/2], xs [M, K/16]) -> y [M, K] = E2M1 * E4M3 / global_scale."""
    M, K = xq.shape[0], xq.shape[1] * 2
    _args(xq.device, xq=(xq, _U8, None), xs=(xs, _U8, M * K // 16), y=(y, _IO, M * K))
    if y is None:
        y = torch.empty((M, K), dtype=out_dtype, device=xq.device)
    _contig(xq, xs, y)
    st = LIB.nvfp4_dequantize_act(_ptr(xq), _ptr(xs), M, K, float(global_scale), _dt(y), _ptr(y), _stream(stream))
    _check("nvfp4_dequantize_act", st)
    return y


def nvfp4_gemm(aq, as_, bq, bs, alpha: float, out_dtype=torch.bfloat16, y=None, stream=None):
    """(aq [M, K/2], as [M, K/16]) x (bq [N, K/2], bs [N, K/16])^T * alpha -> y [M, N]."""
    M, K = aq.shape[0], aq.shape[1] * 2
    N = bq.shape[0]
    _args(aq.device, aq=(aq, _U8, None), as_=(as_, _U8, M * K // 16), bq=(bq, _U8, N * K // 2),
          bs=(bs, _U8, N * K // 16), y=(y, _IO, M * N))
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=aq.device)
    _contig(aq, as_, bq, bs, y)
    st = LIB.nvfp4_gemm(_ptr(aq), _ptr(as_), _ptr(bq), _ptr(bs), float(alpha), M, N, K, _dt(y), _ptr(y),
                        _stream(stream))
    _check("nvfp4_gemm", st)
    return y


def nvfp4_gemm_colscale(aq, as_, bq, bs, col_alpha, out_dtype=torch.bfloat16, y=None, stream=None):
    """nvfp4_gemm with a per-output-column factor col_alpha [N] fp32 (modules fused into one
    weight, each with its own global scale)."""
    M, K = aq.shape[0], aq.shape[1] * 2
    N = bq.shape[0]
    _args(aq.device, aq=(aq, _U8, None), as_=(as_, _U8, M * K // 16), bq=(bq, _U8, N * K // 2),
          bs=(bs, _U8, N * K // 16), col_alpha=(col_alpha, _F32, N), y=(y, _IO, M * N))
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=aq.device)
    _contig(aq, as_, bq, bs, col_alpha, y)
    st = LIB.nvfp4_gemm_colscale(_ptr(aq), _ptr(as_), _ptr(bq), _ptr(bs), _ptr(col_alpha), M, N, K, _dt(y), _ptr(y),
                                 _stream(stream))
    _check("nvfp4_gemm_colscale", st)
    return y


def nvfp4_fused_col_alpha(widths, module_scales, act_scale: float, col_alpha=None, device=None, stream=None):
    """col_alpha [sum(widths)] fp32 for a weight made of modules of the given output widths,
    module i quantised with global scale module_scales[i], activations with act_scale (computed
    by the library: 1 / (act_scale * module scale) per column)."""
    n = len(widths)
    wa = (ctypes.c_int32 * n)(*[int(w) for w in widths])
    sa = (ctypes.c_float * n)(*[float(s) for s in module_scales])
    N = sum(int(w) for w in widths)
    device = torch.device(device if device is not None else "cuda")
    _args(device, col_alpha=(col_alpha, _F32, N))
    if col_alpha is None:
        col_alpha = torch.empty((N,), dtype=torch.float32, device=device)
    _contig(col_alpha)
    st = LIB.nvfp4_fused_col_alpha(wa, sa, n, float(act_scale), _ptr(col_alpha), _stream(stream))
    _check("nvfp4_fused_col_alpha", st)
    return col_alpha


def q4k_gemm(a, w, out_dtype=torch.bfloat16, y=None, stream=None):
    """y [M, N] = a [M, K] (bf16) times the Q4_K weights w [N, K/256*144] (uint8) transposed."""
    M, K = a.shape
    N = w.shape[0]
    if w.dim() != 2 or K % 256 or w.shape[1] != K // 256 * 144:
        raise ValueError("w must be uint8 [N, K/256*144] with K % 256 == 0")
    _args(a.device, a=(a, (torch.bfloat16,), None), w=(w, _U8, N * (K // 256) * 144), y=(y, _IO, M * N))
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=a.device)
    _contig(a, w, y)
    st = LIB.q4k_gemm(_ptr(a), _ptr(w), M, N, K, _dt(y), _ptr(y), _stream(stream))
    _check("q4k_gemm", st)
    return y


def _conv_rows(x):
    """(rows, C, ldx) of a bf16 [rows, C] tensor whose rows may be strided (a column slice of a
    wider projection output)."""
    if x.dim() != 2 or x.dtype != torch.bfloat16 or (x.shape[1] > 1 and x.stride(1) != 1):
        raise ValueError("x must be bf16 [rows, C] with unit channel stride")
    return x.shape[0], x.shape[1], x.stride(0) if x.shape[0] > 1 else x.shape[1]


def _conv_planes(parts, rows, C, y, device):
    """Output buffer and the views of its planes ([rows, width] each, one after another)."""
    widths = [C] if parts is None else [int(p) for p in parts]
    if y is None:
        y = torch.empty((rows * C,), dtype=torch.bfloat16, device=device)
    _contig(y)
    arr = (ctypes.c_int32 * len(widths))(*widths)
    views, off = [], 0
    for wd in widths:
        views.append(y.view(-1)[off:off + rows * wd].view(rows, wd))
        off += rows * wd
    return y, arr, views


def gdn_short_conv1d_silu(x, weight, cu_seqlens=None, num_seqs=None, initial_state=None,
                          final_state=None, output_final_state=False, parts=None, y=None, stream=None):
    """Causal depthwise convolution (width K = weight.shape[1]) + SiLU over packed sequences.
    x bf16 [T, C] (rows may be strided); weight fp32 [C, K]; states bf16 [N, K - 1, C]
    (final_state may be initial_state: updated in place). parts: plane widths (e.g. q, k, v
    channel counts) -> the outputs are [T, width] views of one buffer. Returns (y or the list of
    plane views, final_state)."""
    T, C, ldx = _conv_rows(x)
    K = weight.shape[1]
    N = (cu_seqlens.numel() - 1) if cu_seqlens is not None else (num_seqs or 1)
    _args(x.device, x=x, weight=(weight, _F32, C * K), cu_seqlens=(cu_seqlens, _I32, None),
          initial_state=(initial_state, (torch.bfloat16,), N * (K - 1) * C),
          final_state=(final_state, (torch.bfloat16,), N * (K - 1) * C), y=(y, (torch.bfloat16,), T * C))
    if final_state is None and output_final_state:
        final_state = torch.empty((N, K - 1, C), dtype=torch.bfloat16, device=x.device)
    _contig(weight, cu_seqlens, initial_state, final_state)
    buf, arr, views = _conv_planes(parts, T, C, y, x.device)
    st = LIB.gdn_short_conv1d_silu(_ptr(x), ldx, _ptr(weight), _ptr(cu_seqlens), N, T, C, K, _ptr(initial_state),
                                   _ptr(final_state), _ptr(buf), arr, len(arr), _stream(stream))
    _check("gdn_short_conv1d_silu", st)
    return (views[0] if parts is None else views), final_state


def gdn_short_conv1d_silu_decode(x, weight, conv_state, parts=None, y=None, stream=None):
    """One token per sequence: x bf16 [B, C]; conv_state bf16 [B, K - 1, C] shifted in place.
    Returns y [B, C] (or the list of plane views)."""
    B, C, ldx = _conv_rows(x)
    K = weight.shape[1]
    _args(x.device, x=x, weight=(weight, _F32, C * K), conv_state=(conv_state, (torch.bfloat16,), B * (K - 1) * C),
          y=(y, (torch.bfloat16,), B * C))
    _contig(weight, conv_state)
    buf, arr, views = _conv_planes(parts, B, C, y, x.device)
    st = LIB.gdn_short_conv1d_silu_decode(_ptr(x), ldx, _ptr(weight), B, C, K, _ptr(conv_state), _ptr(buf), arr,
                                          len(arr), _stream(stream))
    _check("gdn_short_conv1d_silu_decode", st)
    return views[0] if parts is None else views


INJECT_SKIP_PREP_LOADS = 1


def gdn_debug_set_wait(wait_limit_ns: int = 0, inject_flags: int = 0) -> None:
    """Test support: bounded-wait limit (0 = the default 1 s) and the switches that make a wait
    run out with nothing in flight (INJECT_SKIP_PREP_LOADS) on the current device."""
    _check("gdn_debug_set_wait", LIB.gdn_debug_set_wait(int(wait_limit_ns), int(inject_flags)))


def gdn_get_device_status(stream=None) -> int:
    return int(LIB.gdn_get_device_status(_stream(stream)))
