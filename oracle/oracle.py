"""CPU oracle for the W8A8 INT8 quantized linear layer -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg may import this module.  The product library never does, and the
oracle never imports the product package: the two share no code.

This module is a thin ctypes wrapper around ``qk_oracle.c`` (plain C, built
with ``gcc -O2 -ffp-contract=off``).  Every arithmetic step lives in the C
file; the functions here only allocate numpy arrays and pass pointers.

Which page each function follows:

* :func:`quantize_per_token` -- vLLM PR "fused silu_and_mul + dynamic per-token
  FP8 quantization", Purpose/Algorithm (scale from the token's own absmax,
  quantise with the inverse scale) and "write-int8-quantized-kernel", Inputs
  (per-token granularity, symmetric [-127, 127]).
* :func:`silu_mul_quant_per_token` -- the same PR, Algorithm Phase 1/Phase 2.
* :func:`gemm_s32` -- "write-int8-quantized-kernel" (INT32 accumulation is
  mandatory) and "KV-cache kernels" section 02 (int8 products go to int32).
* :func:`epilogue_per_channel` -- "KV-cache kernels" section 02
  (``acc * a_scale * b_scale``) and "16. Deploying Custom Kernels"
  (GemmConfig's scale_a, scale_b, output_scale).
* :func:`gemm_group` -- "KV-cache kernels" section 03 (per-group scales every
  64-128 channels); group partials in int32, fp32 accumulation across groups.
* :func:`quantize_per_token_fp8`, :func:`silu_mul_quant_per_token_fp8` -- the
  vLLM PR's own FP8 form (Purpose/Algorithm: float8_e4m3fn,
  scale = max(absmax, 1e-12) / fp8_max, optionally clamped by scale_ub).
* :func:`quantize_per_token_asym`, :func:`gemm_s32_asym` -- asymmetric
  per-token INT8 ("write-int8-quantized-kernel", Inputs: asymmetric maps
  [-128, 127] to an arbitrary range with a non-zero zero-point) and the
  GEMM with the zero-point correction.
* :func:`quantize_static` -- static per-tensor INT8 ("write-int8-quantized-
  kernel", Inputs: per-tensor granularity, scales computed offline).
* :func:`gemm_fp8` -- the FP8 x FP8 product with the exact accumulator
  (every e4m3 value is an integer multiple of 2^-9) and the per-channel
  epilogue.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qk_oracle.c")
_LIB = os.path.join(_HERE, "libqk_oracle.so")

QKO_F32 = 0
QKO_BF16 = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile ``qk_oracle.c`` into ``libqk_oracle.so`` next to it."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-pthread", "-Wall", "-Wextra", "-o", _LIB + ".tmp", _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def build_variant(out_path: str, defines: list[str]) -> str:
    """Compile a copy of the oracle with extra ``-D`` flags (used by tests that
    plant a mistake in the oracle to show that the pins catch it)."""
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
           *[f"-D{d}" for d in defines], "-o", out_path, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return out_path


def _declare(lib: ctypes.CDLL) -> ctypes.CDLL:
    P = ctypes.c_void_p
    i32, i64, f32 = ctypes.c_int, ctypes.c_int64, ctypes.c_float
    lib.qko_f32_to_bf16.argtypes = [f32]
    lib.qko_f32_to_bf16.restype = ctypes.c_uint16
    lib.qko_f32_to_bf16_array.argtypes = [P, P, i64]
    lib.qko_f32_to_bf16_array.restype = None
    lib.qko_exp.argtypes = [f32]
    lib.qko_exp.restype = f32
    lib.qko_silu.argtypes = [f32]
    lib.qko_silu.restype = f32
    lib.qko_quantize_row.argtypes = [P, i32, P, P]
    lib.qko_quantize_row.restype = None
    lib.qko_quantize_per_token.argtypes = [i32, i32, P, i32, P, P]
    lib.qko_quantize_per_token.restype = i32
    lib.qko_silu_mul_quant_per_token.argtypes = [i32, i32, P, P, i64, i32, P, P]
    lib.qko_silu_mul_quant_per_token.restype = i32
    lib.qko_gemm_s32.argtypes = [i32, i32, i32, P, P, P, i32]
    lib.qko_gemm_s32.restype = i32
    lib.qko_epilogue_per_channel.argtypes = [i32, i32, P, P, P, f32, P]
    lib.qko_epilogue_per_channel.restype = i32
    lib.qko_gemm_group.argtypes = [i32, i32, i32, i32, P, P, P, P, f32, P, P, i32]
    lib.qko_gemm_group.restype = i32
    lib.qko_e4m3_to_f32.argtypes = [ctypes.c_uint8]
    lib.qko_e4m3_to_f32.restype = f32
    lib.qko_f32_to_e4m3.argtypes = [f32]
    lib.qko_f32_to_e4m3.restype = ctypes.c_uint8
    lib.qko_f32_to_e4m3_array.argtypes = [P, P, i64]
    lib.qko_f32_to_e4m3_array.restype = None
    lib.qko_quantize_row_fp8.argtypes = [P, i32, P, P, P]
    lib.qko_quantize_row_fp8.restype = None
    lib.qko_quantize_per_token_fp8.argtypes = [i32, i32, P, i32, P, P, P]
    lib.qko_quantize_per_token_fp8.restype = i32
    lib.qko_silu_mul_quant_per_token_fp8.argtypes = [i32, i32, P, P, i64, i32, P, P, P]
    lib.qko_silu_mul_quant_per_token_fp8.restype = i32
    lib.qko_gemm_fp8.argtypes = [i32, i32, i32, P, P, P, P, f32, P, P, i32]
    lib.qko_gemm_fp8.restype = i32
    lib.qko_quantize_row_asym.argtypes = [P, i32, P, P, P]
    lib.qko_quantize_row_asym.restype = None
    lib.qko_quantize_per_token_asym.argtypes = [i32, i32, P, i32, P, P, P]
    lib.qko_quantize_per_token_asym.restype = i32
    lib.qko_weight_row_sums.argtypes = [i32, i32, P, P]
    lib.qko_weight_row_sums.restype = i32
    lib.qko_gemm_s32_asym.argtypes = [i32, i32, i32, P, P, P, P]
    lib.qko_gemm_s32_asym.restype = i32
    lib.qko_quantize_static.argtypes = [i32, i32, P, i32, f32, P]
    lib.qko_quantize_static.restype = i32
    return lib


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the oracle library (building it first if needed)."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    if _lib is None:
        _lib = _declare(ctypes.CDLL(build()))
    return _lib


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _dtype_code(x: np.ndarray) -> int:
    if x.dtype == np.float32:
        return QKO_F32
    if x.dtype == np.uint16:  # bf16 bit patterns
        return QKO_BF16
    raise TypeError(f"oracle inputs are float32 or bf16 bits (uint16), got {x.dtype}")


def _check(rc: int, what: str) -> None:
    if rc == 4:
        raise OverflowError(f"{what}: int32 accumulator bound exceeded")
    if rc != 0:
        raise ValueError(f"{what}: oracle returned {rc}")


class Oracle:
    """numpy front end of the C oracle; ``lib`` may be a planted-mistake build."""

    def __init__(self, lib: ctypes.CDLL | None = None, nthreads: int | None = None):
        self.lib = lib if lib is not None else load()
        self.nthreads = nthreads or (os.cpu_count() or 1)

    # -- scalar helpers -------------------------------------------------------
    def exp(self, t: float) -> float:
        return float(self.lib.qko_exp(ctypes.c_float(t)))

    def silu(self, g: float) -> float:
        return float(self.lib.qko_silu(ctypes.c_float(g)))

    def exp_array(self, t: np.ndarray) -> np.ndarray:
        f = self.lib.qko_exp
        return np.array([f(float(v)) for v in np.asarray(t, np.float32).ravel()],
                        np.float32).reshape(np.shape(t))

    def f32_to_bf16(self, x: np.ndarray) -> np.ndarray:
        x = np.ascontiguousarray(x, np.float32)
        out = np.empty(x.shape, np.uint16)
        self.lib.qko_f32_to_bf16_array(_ptr(x), _ptr(out), x.size)
        return out

    # -- the hot-path stages --------------------------------------------------
    def quantize_per_token(self, x: np.ndarray):
        """x [m, k] (float32 or bf16 bits) -> (q int8 [m, k], scale float32 [m])."""
        x = np.ascontiguousarray(x)
        m, k = x.shape
        q = np.empty((m, k), np.int8)
        s = np.empty((m,), np.float32)
        _check(self.lib.qko_quantize_per_token(m, k, _ptr(x), _dtype_code(x), _ptr(q), _ptr(s)),
               "quantize_per_token")
        return q, s

    def silu_mul_quant_per_token(self, gate: np.ndarray, up: np.ndarray):
        """gate, up [m, k] (same dtype) -> (q int8 [m, k], scale float32 [m])."""
        gate = np.ascontiguousarray(gate)
        up = np.ascontiguousarray(up)
        assert gate.shape == up.shape and gate.dtype == up.dtype
        m, k = gate.shape
        q = np.empty((m, k), np.int8)
        s = np.empty((m,), np.float32)
        _check(self.lib.qko_silu_mul_quant_per_token(m, k, _ptr(gate), _ptr(up), k,
                                                     _dtype_code(gate), _ptr(q), _ptr(s)),
               "silu_mul_quant_per_token")
        return q, s

    def silu_mul_quant_packed(self, gu: np.ndarray):
        """gu [m, 2k]: gate = gu[:, :k], up = gu[:, k:] (one buffer, ld = 2k)."""
        gu = np.ascontiguousarray(gu)
        m, k2 = gu.shape
        k = k2 // 2
        q = np.empty((m, k), np.int8)
        s = np.empty((m,), np.float32)
        base = gu.ctypes.data
        up = base + k * gu.itemsize
        _check(self.lib.qko_silu_mul_quant_per_token(m, k, ctypes.c_void_p(base),
                                                     ctypes.c_void_p(up), k2, _dtype_code(gu),
                                                     _ptr(q), _ptr(s)),
               "silu_mul_quant_per_token")
        return q, s

    def gemm_s32(self, a: np.ndarray, w: np.ndarray) -> np.ndarray:
        """a int8 [m, k], w int8 [n, k] -> acc int32 [m, n]."""
        a = np.ascontiguousarray(a, np.int8)
        w = np.ascontiguousarray(w, np.int8)
        m, k = a.shape
        n, k2 = w.shape
        assert k == k2
        acc = np.empty((m, n), np.int32)
        _check(self.lib.qko_gemm_s32(m, n, k, _ptr(a), _ptr(w), _ptr(acc), self.nthreads),
               "gemm_s32")
        return acc

    def epilogue_per_channel(self, acc: np.ndarray, sa: np.ndarray, sw: np.ndarray,
                             alpha: float = 1.0) -> np.ndarray:
        """acc int32 [m, n], sa [m], sw [n] -> fp32 [m, n]."""
        acc = np.ascontiguousarray(acc, np.int32)
        sa = np.ascontiguousarray(sa, np.float32)
        sw = np.ascontiguousarray(sw, np.float32)
        m, n = acc.shape
        out = np.empty((m, n), np.float32)
        _check(self.lib.qko_epilogue_per_channel(m, n, _ptr(acc), _ptr(sa), _ptr(sw),
                                                 ctypes.c_float(alpha), _ptr(out)),
               "epilogue_per_channel")
        return out

    def gemm_group(self, a: np.ndarray, w: np.ndarray, sa: np.ndarray, sw: np.ndarray,
                   group: int = 128, alpha: float = 1.0):
        """Per-group GEMM + epilogue -> (fp32 out [m, n], full-K int32 acc [m, n])."""
        a = np.ascontiguousarray(a, np.int8)
        w = np.ascontiguousarray(w, np.int8)
        sa = np.ascontiguousarray(sa, np.float32)
        sw = np.ascontiguousarray(sw, np.float32)
        m, k = a.shape
        n = w.shape[0]
        assert sw.shape == (n, k // group)
        out = np.empty((m, n), np.float32)
        acc = np.empty((m, n), np.int32)
        _check(self.lib.qko_gemm_group(m, n, k, group, _ptr(a), _ptr(w), _ptr(sa), _ptr(sw),
                                       ctypes.c_float(alpha), _ptr(out), _ptr(acc),
                                       self.nthreads),
               "gemm_group")
        return out, acc

    # -- whole linear layer (oracle composition of the stages) ---------------
    def linear(self, x: np.ndarray, w_q: np.ndarray, sw: np.ndarray, group_k: int = 0,
               alpha: float = 1.0):
        """quantise x per token, INT8 GEMM, dequant epilogue.
        Returns dict with q, sa, acc, out_f32, out_bf16 (bits)."""
        q, sa = self.quantize_per_token(x)
        return self.linear_from_q(q, sa, w_q, sw, group_k, alpha)

    def linear_from_q(self, q, sa, w_q, sw, group_k: int = 0, alpha: float = 1.0):
        if group_k:
            out, acc = self.gemm_group(q, w_q, sa, sw, group_k, alpha)
        else:
            acc = self.gemm_s32(q, w_q)
            out = self.epilogue_per_channel(acc, sa, sw, alpha)
        return {"q": q, "sa": sa, "acc": acc, "out_f32": out, "out_bf16": self.f32_to_bf16(out)}

    # -- FP8 (e4m3) variant ---------------------------------------------------
    def e4m3_to_f32(self, codes: np.ndarray) -> np.ndarray:
        f = self.lib.qko_e4m3_to_f32
        c = np.asarray(codes, np.uint8)
        return np.array([f(int(b)) for b in c.ravel()], np.float32).reshape(c.shape)

    def f32_to_e4m3(self, x: np.ndarray) -> np.ndarray:
        x = np.ascontiguousarray(x, np.float32)
        out = np.empty(x.shape, np.uint8)
        self.lib.qko_f32_to_e4m3_array(_ptr(x), _ptr(out), x.size)
        return out

    def _ub(self, scale_ub):
        if scale_ub is None:
            return None, ctypes.c_void_p(0)
        ub = np.array([scale_ub], np.float32)
        return ub, _ptr(ub)

    def quantize_per_token_fp8(self, x: np.ndarray, scale_ub: float | None = None):
        """x [m, k] (float32 or bf16 bits) -> (q e4m3 codes uint8 [m, k], scale float32 [m])."""
        x = np.ascontiguousarray(x)
        m, k = x.shape
        q = np.empty((m, k), np.uint8)
        s = np.empty((m,), np.float32)
        keep, ub = self._ub(scale_ub)
        _check(self.lib.qko_quantize_per_token_fp8(m, k, _ptr(x), _dtype_code(x), ub, _ptr(q),
                                                   _ptr(s)), "quantize_per_token_fp8")
        return q, s

    def silu_mul_quant_per_token_fp8(self, gate: np.ndarray, up: np.ndarray,
                                     scale_ub: float | None = None):
        """gate, up [m, k] (same dtype) -> (q e4m3 codes uint8 [m, k], scale float32 [m])."""
        gate = np.ascontiguousarray(gate)
        up = np.ascontiguousarray(up)
        assert gate.shape == up.shape and gate.dtype == up.dtype
        m, k = gate.shape
        q = np.empty((m, k), np.uint8)
        s = np.empty((m,), np.float32)
        keep, ub = self._ub(scale_ub)
        _check(self.lib.qko_silu_mul_quant_per_token_fp8(m, k, _ptr(gate), _ptr(up), k,
                                                         _dtype_code(gate), ub, _ptr(q), _ptr(s)),
               "silu_mul_quant_per_token_fp8")
        return q, s

    def gemm_fp8(self, a: np.ndarray, w: np.ndarray, sa: np.ndarray | None = None,
                 sw: np.ndarray | None = None, alpha: float = 1.0):
        """a [m, k], w [n, k] e4m3 codes -> (exact acc float64 [m, n], fp32 out [m, n] or None)."""
        a = np.ascontiguousarray(a, np.uint8)
        w = np.ascontiguousarray(w, np.uint8)
        m, k = a.shape
        n = w.shape[0]
        acc = np.empty((m, n), np.float64)
        out = None
        if sa is not None:
            sa = np.ascontiguousarray(sa, np.float32)
            sw = np.ascontiguousarray(sw, np.float32)
            out = np.empty((m, n), np.float32)
        _check(self.lib.qko_gemm_fp8(m, n, k, _ptr(a), _ptr(w),
                                     _ptr(sa) if sa is not None else ctypes.c_void_p(0),
                                     _ptr(sw) if sw is not None else ctypes.c_void_p(0),
                                     ctypes.c_float(alpha), _ptr(acc),
                                     _ptr(out) if out is not None else ctypes.c_void_p(0),
                                     self.nthreads), "gemm_fp8")
        return acc, out

    def linear_fp8_from_q(self, q, sa, w_q, sw, alpha: float = 1.0):
        acc, out = self.gemm_fp8(q, w_q, sa, sw, alpha)
        return {"q": q, "sa": sa, "acc": acc, "out_f32": out, "out_bf16": self.f32_to_bf16(out)}

    # -- asymmetric per-token INT8 --------------------------------------------
    def quantize_per_token_asym(self, x: np.ndarray):
        """x [m, k] -> (q int8 [m, k], scale float32 [m], zero-point int32 [m])."""
        x = np.ascontiguousarray(x)
        m, k = x.shape
        q = np.empty((m, k), np.int8)
        s = np.empty((m,), np.float32)
        z = np.empty((m,), np.int32)
        _check(self.lib.qko_quantize_per_token_asym(m, k, _ptr(x), _dtype_code(x), _ptr(q), _ptr(s),
                                                    _ptr(z)), "quantize_per_token_asym")
        return q, s, z

    def weight_row_sums(self, w: np.ndarray) -> np.ndarray:
        w = np.ascontiguousarray(w, np.int8)
        n, k = w.shape
        out = np.empty((n,), np.int32)
        _check(self.lib.qko_weight_row_sums(n, k, _ptr(w), _ptr(out)), "weight_row_sums")
        return out

    def gemm_s32_asym(self, a: np.ndarray, zp: np.ndarray, w: np.ndarray) -> np.ndarray:
        """sum_k (a[m, k] - zp[m]) * w[n, k] -> int32 [m, n]."""
        a = np.ascontiguousarray(a, np.int8)
        zp = np.ascontiguousarray(zp, np.int32)
        w = np.ascontiguousarray(w, np.int8)
        m, k = a.shape
        n = w.shape[0]
        acc = np.empty((m, n), np.int32)
        _check(self.lib.qko_gemm_s32_asym(m, n, k, _ptr(a), _ptr(zp), _ptr(w), _ptr(acc)),
               "gemm_s32_asym")
        return acc

    def linear_asym_from_q(self, q, sa, zp, w_q, sw, alpha: float = 1.0):
        acc = self.gemm_s32_asym(q, zp, w_q)
        out = self.epilogue_per_channel(acc, sa, sw, alpha)
        return {"acc": acc, "out_f32": out, "out_bf16": self.f32_to_bf16(out)}

    # -- static per-tensor INT8 -----------------------------------------------
    def quantize_static(self, x: np.ndarray, scale: float) -> np.ndarray:
        """x [m, k] -> q int8 [m, k] = clamp(rne(x / scale), -127, 127) (via 1 / scale)."""
        x = np.ascontiguousarray(x)
        m, k = x.shape
        q = np.empty((m, k), np.int8)
        _check(self.lib.qko_quantize_static(m, k, _ptr(x), _dtype_code(x), ctypes.c_float(scale),
                                            _ptr(q)), "quantize_static")
        return q
