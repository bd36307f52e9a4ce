"""Python binding of libqk.so -- argument marshalling only.

Two layers:

* ctypes functions with the C names (``qk_quantize_per_token``,
  ``qk_silu_mul_quant_per_token``, ``qk_w8a8_gemm``, ...) taking plain ints,
  device pointers and a stream handle, exactly as ``include/qk.h`` declares
  them (the ctypes binding shape follows "16. Deploying Custom Kernels",
  Python Bindings: sizes as ints, tensors as pointers, a status return);
* torch helpers (:func:`quantize_per_token`, :func:`silu_mul_quant_per_token`,
  :func:`w8a8_gemm`, :func:`linear`) that allocate outputs with torch, pass
  ``data_ptr()`` and the current stream, and raise :class:`QKError` on a
  non-zero status.

Every arithmetic step runs in the library's CUDA kernels; there is no CPU
fallback: a missing library or a non-CUDA tensor raises.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libqk.so")

ABI_VERSION = 12

QK_OK = 0
QK_ERR_INVALID_ARG = 1
QK_ERR_MISALIGNED = 2
QK_ERR_UNSUPPORTED = 3
QK_ERR_OVERFLOW_BOUND = 4
QK_ERR_CUDA = 5
QK_ERR_TIMEOUT = 6
QK_ERR_WORKSPACE = 7

QK_F32 = 0
QK_BF16 = 1

# QK_NOALLOC_SCRATCH_BYTES of include/qk.h: the size of the scratch array
# built into the library for qk_w8a8_gemm_noalloc (a host test checks that
# the two agree)
NOALLOC_SCRATCH_BYTES = 48 * 1024 * 1024 + 4096

# name -> (restype, argtypes), in include/qk.h order
_P = ctypes.c_void_p
_SIGNATURES = {
    "qk_abi_version": (ctypes.c_int, []),
    "qk_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "qk_quantize_per_token": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, _P, ctypes.c_int, _P, _P, _P]),
    "qk_silu_mul_quant_per_token": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, _P, _P, ctypes.c_int64,
                                                   ctypes.c_int, _P, _P, _P]),
    "qk_quantize_per_token_fp8": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, _P, ctypes.c_int, _P, _P, _P,
                                                 _P]),
    "qk_silu_mul_quant_per_token_fp8": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, _P, _P, ctypes.c_int64,
                                                       ctypes.c_int, _P, _P, _P, _P]),
    "qk_w8a8_gemm": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P, ctypes.c_int,
                                    ctypes.c_float, _P, _P, ctypes.c_int, _P, ctypes.c_size_t, _P]),
    "qk_fp8_gemm": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P, ctypes.c_float,
                                   _P, ctypes.c_int, _P]),
    "qk_quantize_per_token_asym": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, _P, ctypes.c_int, _P, _P, _P,
                                                  _P]),
    "qk_w8a8_moe_gemm": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        _P, _P, _P, _P, _P, ctypes.c_float, _P, ctypes.c_int, _P]),
    "qk_quantize_static": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, _P, ctypes.c_int, _P, _P, _P]),
    "qk_weight_row_sums": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, _P, _P, _P]),
    "qk_w8a8_gemm_asym": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P, _P, _P,
                                         ctypes.c_float, _P, _P, ctypes.c_int, _P, ctypes.c_size_t, _P]),
    "qk_w8a8_gemm_workspace_size": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "qk_w8a8_gemm_kernel": (ctypes.c_char_p, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int]),
    "qk_w8a8_linear": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, ctypes.c_int, _P, _P,
                                      ctypes.c_int, ctypes.c_float, _P, _P, ctypes.c_int, _P, ctypes.c_size_t,
                                      _P]),
    "qk_w8a8_linear_workspace_size": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "qk_w8a8_linear_fused": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, ctypes.c_int, _P, _P,
                                            ctypes.c_float, _P, _P, ctypes.c_int, _P, ctypes.c_size_t, _P]),
    "qk_w8a8_gemm_noalloc": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P,
                                            ctypes.c_int, ctypes.c_float, _P, _P, ctypes.c_int, _P]),
    "qk_device_status": (ctypes.c_int, [_P]),
    "qk_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_int, _P]),
    "qk_selftest_silu": (ctypes.c_int, [ctypes.c_uint32, ctypes.c_uint64, _P, _P, _P]),
    "qk_selftest_mma_rate": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_uint32,
                                            _P, _P]),
    "qk_selftest_mma_interference": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P]),
}

_lib: ctypes.CDLL | None = None


class QKError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        msg = status_string(status) if _lib is not None else str(status)
        super().__init__(f"{where}: qk status {status} ({msg})" if where else f"qk status {status} ({msg})")


def lib() -> ctypes.CDLL:
    """Load libqk.so and check its ABI number; raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m w8a8_int8_quantized_qk_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        got = L.qk_abi_version()
        if got != ABI_VERSION:
            raise RuntimeError(f"libqk.so ABI {got} != binding ABI {ABI_VERSION}: rebuild the library")
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().qk_status_string(status).decode()


# ---------------------------------------------------------------- C names
def qk_abi_version() -> int:
    return lib().qk_abi_version()


def qk_status_string(status: int) -> str:
    return status_string(status)


def qk_quantize_per_token(m, k, x, x_dtype, q, scale, stream) -> int:
    return lib().qk_quantize_per_token(m, k, x, x_dtype, q, scale, stream)


def qk_silu_mul_quant_per_token(m, k, gate, up, ld_in, in_dtype, q, scale, stream) -> int:
    return lib().qk_silu_mul_quant_per_token(m, k, gate, up, ld_in, in_dtype, q, scale, stream)


def qk_quantize_per_token_fp8(m, k, x, x_dtype, scale_ub, q, scale, stream) -> int:
    return lib().qk_quantize_per_token_fp8(m, k, x, x_dtype, scale_ub, q, scale, stream)


def qk_silu_mul_quant_per_token_fp8(m, k, gate, up, ld_in, in_dtype, scale_ub, q, scale, stream) -> int:
    return lib().qk_silu_mul_quant_per_token_fp8(m, k, gate, up, ld_in, in_dtype, scale_ub, q, scale,
                                                 stream)


def qk_w8a8_gemm(m, n, k, a, b, scale_a, scale_b, group_k, output_scale, c, out, out_dtype,
                 workspace, workspace_bytes, stream) -> int:
    return lib().qk_w8a8_gemm(m, n, k, a, b, scale_a, scale_b, group_k, output_scale, c, out,
                              out_dtype, workspace, workspace_bytes, stream)


def qk_fp8_gemm(m, n, k, a, b, scale_a, scale_b, output_scale, out, out_dtype, stream) -> int:
    return lib().qk_fp8_gemm(m, n, k, a, b, scale_a, scale_b, output_scale, out, out_dtype, stream)


def qk_quantize_per_token_asym(m, k, x, x_dtype, q, scale, zero_point, stream) -> int:
    return lib().qk_quantize_per_token_asym(m, k, x, x_dtype, q, scale, zero_point, stream)


def qk_w8a8_moe_gemm(num_experts, total_m, n, k, max_m_per_expert, expert_offsets, a, b, scale_a, scale_b,
                     output_scale, out, out_dtype, stream) -> int:
    return lib().qk_w8a8_moe_gemm(num_experts, total_m, n, k, max_m_per_expert, expert_offsets, a, b,
                                  scale_a, scale_b, output_scale, out, out_dtype, stream)


def qk_quantize_static(m, k, x, x_dtype, scale, q, stream) -> int:
    return lib().qk_quantize_static(m, k, x, x_dtype, scale, q, stream)


def qk_weight_row_sums(n, k, w, wsum, stream) -> int:
    return lib().qk_weight_row_sums(n, k, w, wsum, stream)


def qk_w8a8_gemm_asym(m, n, k, a, zero_point_a, b, wsum_b, scale_a, scale_b, output_scale, c, out,
                      out_dtype, workspace, workspace_bytes, stream) -> int:
    return lib().qk_w8a8_gemm_asym(m, n, k, a, zero_point_a, b, wsum_b, scale_a, scale_b, output_scale,
                                   c, out, out_dtype, workspace, workspace_bytes, stream)


def qk_w8a8_gemm_workspace_size(m, n, k, group_k) -> int:
    return lib().qk_w8a8_gemm_workspace_size(m, n, k, group_k)


def qk_w8a8_gemm_kernel(m, n, k, group_k, with_c) -> str:
    """The kernel, tile shape and split form qk_w8a8_gemm launches for this
    problem on the current device."""
    return lib().qk_w8a8_gemm_kernel(m, n, k, group_k, 1 if with_c else 0).decode()


def qk_w8a8_linear(m, n, k, x, x_dtype, b, scale_b, group_k, output_scale, scale_a_out, out, out_dtype,
                   workspace, workspace_bytes, stream) -> int:
    """The whole layer (quantise + GEMM + epilogue) with q and the scales in
    the workspace (see include/qk.h)."""
    return lib().qk_w8a8_linear(m, n, k, x, x_dtype, b, scale_b, group_k, output_scale, scale_a_out, out,
                                out_dtype, workspace, workspace_bytes, stream)


def qk_w8a8_linear_workspace_size(m, n, k, group_k) -> int:
    return lib().qk_w8a8_linear_workspace_size(m, n, k, group_k)


def qk_w8a8_linear_fused(m, n, k, x, x_dtype, b, scale_b, output_scale, scale_a_out, out, out_dtype,
                         workspace, workspace_bytes, stream) -> int:
    return lib().qk_w8a8_linear_fused(m, n, k, x, x_dtype, b, scale_b, output_scale, scale_a_out, out,
                                      out_dtype, workspace, workspace_bytes, stream)


def qk_w8a8_gemm_noalloc(m, n, k, a, b, scale_a, scale_b, group_k, output_scale, c, out, out_dtype,
                         stream) -> int:
    """qk_w8a8_gemm for callers that cannot allocate device memory: split-K
    scratch comes from an array built into the library (see include/qk.h)."""
    return lib().qk_w8a8_gemm_noalloc(m, n, k, a, b, scale_a, scale_b, group_k, output_scale, c, out,
                                      out_dtype, stream)


def qk_device_status(stream) -> int:
    return lib().qk_device_status(stream)


def qk_selftest_bounded_wait(timeout_us, stream) -> int:
    return lib().qk_selftest_bounded_wait(timeout_us, stream)


def qk_selftest_silu(first, count, mismatches, first_mismatch, stream) -> int:
    return lib().qk_selftest_silu(first, count, mismatches, first_mismatch, stream)


def qk_selftest_mma_rate(cta_group, n, iters, ctas, operand_seed, cycles, stream) -> int:
    return lib().qk_selftest_mma_rate(cta_group, n, iters, ctas, operand_seed, cycles, stream)


def qk_selftest_mma_interference(companion, groups, ctas, cycles, stream) -> int:
    return lib().qk_selftest_mma_interference(companion, groups, ctas, cycles, stream)


# ---------------------------------------------------------------- torch helpers
def _torch():
    import torch

    return torch


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p | None:
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return QK_BF16
    if t.dtype == torch.float32:
        return QK_F32
    raise TypeError(f"expected bfloat16 or float32, got {t.dtype}")


def _check(st: int, where: str) -> None:
    if st != QK_OK:
        raise QKError(st, where)


def _need_cuda(*ts) -> None:
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libqk works on CUDA tensors only (no CPU fallback)")


def quantize_per_token(x, q=None, scale=None, stream=None):
    """x [m, k] bf16/fp32 (CUDA, contiguous) -> (q int8 [m, k], scale fp32 [m])."""
    torch = _torch()
    _need_cuda(x)
    assert x.dim() == 2 and x.is_contiguous()
    m, k = x.shape
    q = torch.empty((m, k), dtype=torch.int8, device=x.device) if q is None else q
    scale = torch.empty((m,), dtype=torch.float32, device=x.device) if scale is None else scale
    _check(qk_quantize_per_token(m, k, _ptr(x), _dtype_code(x), _ptr(q), _ptr(scale), _stream(stream)),
           "qk_quantize_per_token")
    return q, scale


def silu_mul_quant_per_token(gate, up, q=None, scale=None, stream=None):
    """gate, up [m, k] (same dtype and row stride) -> (q int8 [m, k], scale fp32 [m]).
    gate/up may be the two halves of one [m, 2k] tensor (row stride 2k)."""
    torch = _torch()
    _need_cuda(gate, up)
    assert gate.shape == up.shape and gate.dtype == up.dtype and gate.dim() == 2
    assert gate.stride(1) == 1 and up.stride(1) == 1 and gate.stride(0) == up.stride(0)
    m, k = gate.shape
    q = torch.empty((m, k), dtype=torch.int8, device=gate.device) if q is None else q
    scale = torch.empty((m,), dtype=torch.float32, device=gate.device) if scale is None else scale
    _check(qk_silu_mul_quant_per_token(m, k, _ptr(gate), _ptr(up), gate.stride(0), _dtype_code(gate),
                                       _ptr(q), _ptr(scale), _stream(stream)),
           "qk_silu_mul_quant_per_token")
    return q, scale


def quantize_per_token_fp8(x, scale_ub=None, q=None, scale=None, stream=None):
    """x [m, k] bf16/fp32 -> (q e4m3 codes uint8 [m, k], scale fp32 [m]); scale_ub:
    optional one-element fp32 CUDA tensor bounding the scale."""
    torch = _torch()
    _need_cuda(x)
    assert x.dim() == 2 and x.is_contiguous()
    m, k = x.shape
    q = torch.empty((m, k), dtype=torch.uint8, device=x.device) if q is None else q
    scale = torch.empty((m,), dtype=torch.float32, device=x.device) if scale is None else scale
    _check(qk_quantize_per_token_fp8(m, k, _ptr(x), _dtype_code(x), _ptr(scale_ub), _ptr(q), _ptr(scale),
                                     _stream(stream)), "qk_quantize_per_token_fp8")
    return q, scale


def silu_mul_quant_per_token_fp8(gate, up, scale_ub=None, q=None, scale=None, stream=None):
    """gate, up [m, k] -> (q e4m3 codes uint8 [m, k], scale fp32 [m])."""
    torch = _torch()
    _need_cuda(gate, up)
    assert gate.shape == up.shape and gate.dtype == up.dtype and gate.dim() == 2
    assert gate.stride(1) == 1 and up.stride(1) == 1 and gate.stride(0) == up.stride(0)
    m, k = gate.shape
    q = torch.empty((m, k), dtype=torch.uint8, device=gate.device) if q is None else q
    scale = torch.empty((m,), dtype=torch.float32, device=gate.device) if scale is None else scale
    _check(qk_silu_mul_quant_per_token_fp8(m, k, _ptr(gate), _ptr(up), gate.stride(0), _dtype_code(gate),
                                           _ptr(scale_ub), _ptr(q), _ptr(scale), _stream(stream)),
           "qk_silu_mul_quant_per_token_fp8")
    return q, scale


def silu_mul_quant_packed(gu, stream=None):
    """gu [m, 2k]: gate = gu[:, :k], up = gu[:, k:]."""
    k = gu.shape[1] // 2
    return silu_mul_quant_per_token(gu[:, :k], gu[:, k:], stream=stream)


def w8a8_gemm(a, b, scale_a, scale_b, group_k: int = 0, output_scale: float = 1.0,
              out_dtype=None, want_out: bool = True, want_c: bool = False, out=None, c=None,
              workspace=None, stream=None):
    """a int8 [m, k], b int8 [n, k] -> (out [m, n] or None, c int32 [m, n] or None)."""
    torch = _torch()
    _need_cuda(a, b, scale_a, scale_b)
    m, k = a.shape
    n = b.shape[0]
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    if want_out and out is None:
        out = torch.empty((m, n), dtype=out_dtype, device=a.device)
    if want_c and c is None:
        c = torch.empty((m, n), dtype=torch.int32, device=a.device)
    need = qk_w8a8_gemm_workspace_size(m, n, k, group_k)
    if need and workspace is None:
        workspace = cached_workspace(need, a.device)
    code = _dtype_code(out) if out is not None else QK_BF16
    _check(qk_w8a8_gemm(m, n, k, _ptr(a), _ptr(b), _ptr(scale_a), _ptr(scale_b), group_k,
                        float(output_scale), _ptr(c), _ptr(out), code, _ptr(workspace),
                        0 if workspace is None else workspace.numel(), _stream(stream)),
           "qk_w8a8_gemm")
    return out, c


def fp8_gemm(a, b, scale_a, scale_b, output_scale: float = 1.0, out_dtype=None, out=None, stream=None):
    """a [m, k], b [n, k] e4m3 codes (uint8, CUDA) -> out [m, n] (bf16 by default)."""
    torch = _torch()
    _need_cuda(a, b, scale_a, scale_b)
    m, k = a.shape
    n = b.shape[0]
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    out = torch.empty((m, n), dtype=out_dtype, device=a.device) if out is None else out
    _check(qk_fp8_gemm(m, n, k, _ptr(a), _ptr(b), _ptr(scale_a), _ptr(scale_b), float(output_scale),
                       _ptr(out), _dtype_code(out), _stream(stream)), "qk_fp8_gemm")
    return out


def quantize_per_token_asym(x, stream=None):
    """x [m, k] bf16/fp32 -> (q int8 [m, k], scale fp32 [m], zero_point int32 [m])."""
    torch = _torch()
    _need_cuda(x)
    assert x.dim() == 2 and x.is_contiguous()
    m, k = x.shape
    q = torch.empty((m, k), dtype=torch.int8, device=x.device)
    scale = torch.empty((m,), dtype=torch.float32, device=x.device)
    zp = torch.empty((m,), dtype=torch.int32, device=x.device)
    _check(qk_quantize_per_token_asym(m, k, _ptr(x), _dtype_code(x), _ptr(q), _ptr(scale), _ptr(zp),
                                      _stream(stream)), "qk_quantize_per_token_asym")
    return q, scale, zp


def w8a8_moe_gemm(a, expert_offsets, b, scale_a, scale_b, max_m_per_expert: int, output_scale: float = 1.0,
                  out_dtype=None, stream=None):
    """a [total_m, k] int8 grouped by expert, expert_offsets int32 [E + 1] (CUDA),
    b [E, n, k] int8, scale_a [total_m], scale_b [E, n] -> out [total_m, n]."""
    torch = _torch()
    _need_cuda(a, b, scale_a, scale_b, expert_offsets)
    total_m, k = a.shape
    e, n, _ = b.shape
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    out = torch.empty((total_m, n), dtype=out_dtype, device=a.device)
    _check(qk_w8a8_moe_gemm(e, total_m, n, k, int(max_m_per_expert), _ptr(expert_offsets), _ptr(a), _ptr(b),
                            _ptr(scale_a), _ptr(scale_b), float(output_scale), _ptr(out), _dtype_code(out),
                            _stream(stream)), "qk_w8a8_moe_gemm")
    return out


def quantize_static(x, scale, stream=None):
    """x [m, k] bf16/fp32 -> q int8 [m, k] with the per-tensor scale (a one-element
    fp32 CUDA tensor)."""
    torch = _torch()
    _need_cuda(x, scale)
    assert x.dim() == 2 and x.is_contiguous()
    m, k = x.shape
    q = torch.empty((m, k), dtype=torch.int8, device=x.device)
    _check(qk_quantize_static(m, k, _ptr(x), _dtype_code(x), _ptr(scale), _ptr(q), _stream(stream)),
           "qk_quantize_static")
    return q


def weight_row_sums(w, stream=None):
    """w [n, k] int8 -> wsum int32 [n] (sum over k of each row)."""
    torch = _torch()
    _need_cuda(w)
    n, k = w.shape
    out = torch.empty((n,), dtype=torch.int32, device=w.device)
    _check(qk_weight_row_sums(n, k, _ptr(w), _ptr(out), _stream(stream)), "qk_weight_row_sums")
    return out


def w8a8_gemm_asym(a, zero_point_a, b, wsum_b, scale_a, scale_b, output_scale: float = 1.0,
                   out_dtype=None, want_out: bool = True, want_c: bool = False, workspace=None,
                   stream=None):
    """Asymmetric activations: (out [m, n] or None, c int32 [m, n] or None)."""
    torch = _torch()
    _need_cuda(a, b, zero_point_a, wsum_b)
    m, k = a.shape
    n = b.shape[0]
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    out = torch.empty((m, n), dtype=out_dtype, device=a.device) if want_out else None
    c = torch.empty((m, n), dtype=torch.int32, device=a.device) if want_c else None
    need = qk_w8a8_gemm_workspace_size(m, n, k, 0)
    if need and workspace is None:
        workspace = cached_workspace(need, a.device)
    code = _dtype_code(out) if out is not None else QK_BF16
    _check(qk_w8a8_gemm_asym(m, n, k, _ptr(a), _ptr(zero_point_a), _ptr(b), _ptr(wsum_b), _ptr(scale_a),
                             _ptr(scale_b), float(output_scale), _ptr(c), _ptr(out), code, _ptr(workspace),
                             0 if workspace is None else workspace.numel(), _stream(stream)),
           "qk_w8a8_gemm_asym")
    return out, c


_workspaces: dict = {}


def cached_workspace(nbytes: int, device):
    """A zero-filled workspace of at least `nbytes` on `device`, kept for reuse.
    The library leaves its counter header zero after every completed call, so
    the buffer can be shared by calls of any shape on one stream."""
    torch = _torch()
    key = torch.device(device).index
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros((max(nbytes, 1 << 20),), dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def w8a8_linear(x, w_q, sw, group_k: int = 0, output_scale: float = 1.0, out_dtype=None,
                want_scale: bool = False, workspace=None, stream=None):
    """qk_w8a8_linear: x [m, k] bf16/fp32 -> (out [m, n], per-token scales [m] or None).
    `workspace` (or a fresh zero-filled one) holds q and the scales between
    the two kernels."""
    torch = _torch()
    _need_cuda(x, w_q, sw)
    assert x.dim() == 2 and x.is_contiguous()
    m, k = x.shape
    n = w_q.shape[0]
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    out = torch.empty((m, n), dtype=out_dtype, device=x.device)
    sa = torch.empty((m,), dtype=torch.float32, device=x.device) if want_scale else None
    need = qk_w8a8_linear_workspace_size(m, n, k, group_k)
    if need and workspace is None:
        workspace = torch.zeros((need,), dtype=torch.uint8, device=x.device)
    _check(qk_w8a8_linear(m, n, k, _ptr(x), _dtype_code(x), _ptr(w_q), _ptr(sw), group_k,
                          float(output_scale), _ptr(sa), _ptr(out), _dtype_code(out), _ptr(workspace),
                          0 if workspace is None else workspace.numel(), _stream(stream)),
           "qk_w8a8_linear")
    return out, sa


def w8a8_linear_fused(x, w_q, sw, output_scale: float = 1.0, out_dtype=None, want_scale: bool = False,
                      workspace=None, stream=None):
    """qk_w8a8_linear_fused (decode shapes, one launch): x [m, k] -> (out [m, n],
    per-token scales [m] or None).  `workspace` (or a fresh zero-filled one)
    holds the flag words, q and the scales."""
    torch = _torch()
    _need_cuda(x, w_q, sw)
    assert x.dim() == 2 and x.is_contiguous()
    m, k = x.shape
    n = w_q.shape[0]
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    out = torch.empty((m, n), dtype=out_dtype, device=x.device)
    sa = torch.empty((m,), dtype=torch.float32, device=x.device) if want_scale else None
    need = qk_w8a8_linear_workspace_size(m, n, k, 0)
    if workspace is None:
        workspace = torch.zeros((max(need, 1),), dtype=torch.uint8, device=x.device)
    _check(qk_w8a8_linear_fused(m, n, k, _ptr(x), _dtype_code(x), _ptr(w_q), _ptr(sw), float(output_scale),
                                _ptr(sa), _ptr(out), _dtype_code(out), _ptr(workspace), workspace.numel(),
                                _stream(stream)),
           "qk_w8a8_linear_fused")
    return out, sa


def linear(x, w_q, sw, group_k: int = 0, output_scale: float = 1.0, out_dtype=None, stream=None):
    """The whole W8A8 linear layer: quantise x per token, INT8 GEMM, dequant
    (q and the scales in torch allocations, so concurrent calls on different
    streams do not share buffers)."""
    q, sa = quantize_per_token(x, stream=stream)
    out, _ = w8a8_gemm(q, w_q, sa, sw, group_k, output_scale, out_dtype, stream=stream)
    return out


def mlp_down(gate, up, w_q, sw, output_scale: float = 1.0, out_dtype=None, stream=None):
    """silu(gate) * up, quantised per token, then the INT8 down projection."""
    q, sa = silu_mul_quant_per_token(gate, up, stream=stream)
    out, _ = w8a8_gemm(q, w_q, sa, sw, 0, output_scale, out_dtype, stream=stream)
    return out


def device_status(stream=None) -> int:
    return qk_device_status(_stream(stream))


MMA_COMPANIONS = {0: "none", 1: "fp32 fma", 2: "fp32 mul", 3: "int32->fp32 cvt + logic", 4: "int32 mad",
                  5: "cvt + fp32 fma (group-128 epilogue mix)", 6: "fp32 -> bf16x2 pack"}


def mma_interference(groups: int = 4096, ctas: int | None = None, stream=None) -> dict:
    """qk_selftest_mma_interference for every companion loop: SM cycles per
    group of four 256x256x32 pair MMAs (512 at the full rate) while the other
    warps of the SM run that loop, and the clock the cycles imply."""
    torch = _torch()
    if ctas is None:
        ctas = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
        ctas -= ctas % 2
    cyc = torch.zeros((ctas,), dtype=torch.int64, device="cuda")
    s = _stream(stream)
    out = {}
    for c, name in MMA_COMPANIONS.items():
        _check(qk_selftest_mma_interference(c, groups, ctas, _ptr(cyc), s), "mma interference probe")
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        cur = torch.cuda.current_stream()
        e0.record(cur)
        _check(qk_selftest_mma_interference(c, groups, ctas, _ptr(cyc), s), "mma interference probe")
        e1.record(cur)
        torch.cuda.synchronize()
        cycles = float(cyc[::2].double().median().item())
        sec = e0.elapsed_time(e1) * 1e-3
        out[name] = {"cycles_per_group": cycles / groups, "clock_mhz_from_cycles": cycles / sec / 1e6}
    return out


def mma_rate(cta_group: int = 2, n: int = 256, iters: int = 16384, ctas: int | None = None,
             launches: int = 5, operand_seed: int = 0, stream=None) -> dict:
    """Time qk_selftest_mma_rate: `launches` back-to-back launches between
    CUDA events on the current stream, on zero operands (seed 0) or seeded
    random bytes.  Returns the INT8 rate (TOPS, 2 ops per multiply-add) and
    the issuing CTAs' median cycles per launch."""
    torch = _torch()
    if ctas is None:
        ctas = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
        ctas -= ctas % cta_group
    cyc = torch.zeros((ctas,), dtype=torch.int64, device="cuda")
    s = _stream(stream)
    _check(qk_selftest_mma_rate(cta_group, n, iters, ctas, operand_seed, _ptr(cyc), s), "mma rate probe")  # warm-up
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    e0.record(cur)
    for _ in range(launches):
        _check(qk_selftest_mma_rate(cta_group, n, iters, ctas, operand_seed, _ptr(cyc), s), "mma rate probe")
    e1.record(cur)
    torch.cuda.synchronize()
    sec = e0.elapsed_time(e1) * 1e-3 / launches
    macs = (ctas // cta_group) * iters * (128 * cta_group) * n * 32
    issuing = cyc[::cta_group].double()
    cycles = float(issuing.median().item())
    return {"tops": 2.0 * macs / sec / 1e12, "seconds_per_launch": sec, "cycles": cycles,
            "macs_per_clk_per_sm": macs / cta_group / (ctas // cta_group) / cycles if cycles > 0 else None,
            "clock_mhz_from_cycles": cycles / sec / 1e6, "cta_group": cta_group, "n": n, "iters": iters,
            "ctas": ctas, "operands": "zero" if operand_seed == 0 else f"random (seed {operand_seed})"}

