"""Host-side tests of the C ABI (no GPU needed, nothing is launched).

* libqk.so loads and exports every function include/qk.h declares;
* the ABI number matches;
* argument checks reject bad calls before touching the device;
* the product package never imports the oracle, and has no CPU fallback.
"""
import ctypes
import os
import re

import pytest

from w8a8_int8_quantized_qk_b200 import build as qkbuild
from w8a8_int8_quantized_qk_b200 import qk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qk.h")
PKG = os.path.join(ROOT, "w8a8_int8_quantized_qk_b200")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qk_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    qkbuild.build()
    return qk.lib()


def test_header_declares_the_calls():
    names = header_functions()
    for n in ("qk_quantize_per_token", "qk_silu_mul_quant_per_token", "qk_w8a8_gemm",
              "qk_abi_version", "qk_status_string", "qk_device_status"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    raw = ctypes.CDLL(qk.LIB_PATH)
    for name in header_functions():
        assert hasattr(raw, name), name
        assert name in qk._SIGNATURES, f"binding lacks {name}"


def test_abi_version(L):
    hdr = open(HEADER).read()
    assert int(re.search(r"#define QK_ABI_VERSION (\d+)", hdr).group(1)) == qk.ABI_VERSION
    assert qk.qk_abi_version() == qk.ABI_VERSION


def test_noalloc_scratch_size_matches_header():
    # the binding's constant (used by the tests) is the header's #define
    hdr = open(HEADER).read()
    expr = re.search(r"#define QK_NOALLOC_SCRATCH_BYTES \(([^)]*)\)", hdr).group(1)
    assert re.fullmatch(r"[0-9u*+ ]+", expr), expr
    assert eval(expr.replace("u", "")) == qk.NOALLOC_SCRATCH_BYTES  # integer arithmetic only


def test_status_strings(L):
    for code in range(8):
        assert qk.qk_status_string(code)
    assert qk.qk_status_string(99) == "unknown status"
    hdr = open(HEADER).read()
    for name, val in re.findall(r"(QK_(?:OK|ERR_[A-Z_]+)) = (\d+)", hdr):
        assert getattr(qk, name) == int(val)


NULL = None
P16 = ctypes.c_void_p(0x1000)   # never dereferenced: every call below fails its checks first
P8 = ctypes.c_void_p(0x1008)    # 8-byte aligned only


@pytest.mark.parametrize("args,expect", [
    ((-1, 16, P16, qk.QK_BF16, P16, P16, NULL), qk.QK_ERR_INVALID_ARG),
    ((4, 0, P16, qk.QK_BF16, P16, P16, NULL), qk.QK_ERR_INVALID_ARG),
    ((4, 24, P16, qk.QK_BF16, P16, P16, NULL), qk.QK_ERR_INVALID_ARG),   # k % 16
    ((4, 16, P16, 7, P16, P16, NULL), qk.QK_ERR_INVALID_ARG),            # dtype
    ((4, 16, NULL, qk.QK_BF16, P16, P16, NULL), qk.QK_ERR_INVALID_ARG),
    ((4, 16, P8, qk.QK_BF16, P16, P16, NULL), qk.QK_ERR_MISALIGNED),
    ((4, 16, P16, qk.QK_F32, P8, P16, NULL), qk.QK_ERR_MISALIGNED),
    ((0, 16, NULL, qk.QK_BF16, NULL, NULL, NULL), qk.QK_OK),             # empty: no-op
])
def test_quantize_rejects(L, args, expect):
    assert qk.qk_quantize_per_token(*args) == expect


@pytest.mark.parametrize("args,expect", [
    ((4, 16, P16, P16, 8, qk.QK_BF16, P16, P16, NULL), qk.QK_ERR_INVALID_ARG),   # ld < k
    ((4, 16, P16, NULL, 16, qk.QK_BF16, P16, P16, NULL), qk.QK_ERR_INVALID_ARG),
    ((4, 16, P16, P8, 16, qk.QK_BF16, P16, P16, NULL), qk.QK_ERR_MISALIGNED),
    ((4, 16, P16, P16, 20, qk.QK_BF16, P16, P16, NULL), qk.QK_ERR_MISALIGNED),    # 40-byte rows
    ((0, 16, NULL, NULL, 16, qk.QK_BF16, NULL, NULL, NULL), qk.QK_OK),
])
def test_silu_rejects(L, args, expect):
    assert qk.qk_silu_mul_quant_per_token(*args) == expect


def _gemm(m=4, n=8, k=16, a=P16, b=P16, sa=P16, sw=P16, g=0, c=NULL, out=P16, dt=qk.QK_BF16,
          ws=NULL, wsb=0):
    return qk.qk_w8a8_gemm(m, n, k, a, b, sa, sw, g, 1.0, c, out, dt, ws, wsb, NULL)


@pytest.mark.parametrize("kw,expect", [
    (dict(m=-1), qk.QK_ERR_INVALID_ARG),
    (dict(k=0), qk.QK_ERR_INVALID_ARG),
    (dict(k=40), qk.QK_ERR_INVALID_ARG),
    (dict(n=12), qk.QK_ERR_INVALID_ARG),
    (dict(g=64), qk.QK_ERR_INVALID_ARG),
    (dict(g=128, k=64), qk.QK_ERR_INVALID_ARG),
    (dict(k=133152), qk.QK_ERR_OVERFLOW_BOUND),          # k * 127^2 >= 2^31
    (dict(out=NULL), qk.QK_ERR_INVALID_ARG),              # neither c nor out
    (dict(a=NULL), qk.QK_ERR_INVALID_ARG),
    (dict(sa=NULL), qk.QK_ERR_INVALID_ARG),
    (dict(dt=5), qk.QK_ERR_INVALID_ARG),
    (dict(a=P8), qk.QK_ERR_MISALIGNED),
    (dict(out=P8), qk.QK_ERR_MISALIGNED),
    (dict(sw=P8), qk.QK_ERR_MISALIGNED),
    (dict(m=0), qk.QK_OK),
    (dict(n=0), qk.QK_OK),
])
def test_gemm_rejects(L, kw, expect):
    assert _gemm(**kw) == expect


def test_k_bound_is_exact():
    # 133144 * 127^2 = 2147479576 < 2^31 <= 133145 * 127^2 (133144 is not a multiple
    # of 16; the largest legal k is 133136)
    assert 133144 * 127 ** 2 < 2 ** 31 <= 133145 * 127 ** 2


def test_workspace_query(L):
    assert qk.qk_w8a8_gemm_workspace_size(4096, 4096, 4096, 0) >= 0


def test_kernel_query_host_answers(L):
    # shape checks come before any device query
    assert qk.qk_w8a8_gemm_kernel(16, 64, 20, 0, False) == "unsupported"  # k % 16 != 0
    assert qk.qk_w8a8_gemm_kernel(16, 60, 32, 0, False) == "unsupported"  # n % 8 != 0
    assert qk.qk_w8a8_gemm_kernel(16, 64, 256, 64, False) == "unsupported"  # group_k not 0 / 128
    assert qk.qk_w8a8_gemm_kernel(0, 64, 32, 0, False) == "none (empty output)"
    name = qk.qk_w8a8_gemm_kernel(4096, 4096, 4096, 0, False)
    assert name == "no device" or name.startswith("gemm_i8_pair_kernel")


def test_selftest_arg_check(L):
    assert qk.qk_selftest_bounded_wait(0, NULL) == qk.QK_ERR_INVALID_ARG
    assert qk.qk_selftest_bounded_wait(3000000, NULL) == qk.QK_ERR_INVALID_ARG


def test_no_cpu_fallback(L):
    # every torch helper refuses host tensors before doing any work
    torch = pytest.importorskip("torch")
    x = torch.zeros((4, 16), dtype=torch.bfloat16)
    a = torch.zeros((4, 16), dtype=torch.int8)
    b = torch.zeros((8, 16), dtype=torch.int8)
    s4 = torch.ones((4,), dtype=torch.float32)
    s8 = torch.ones((8,), dtype=torch.float32)
    u8a = torch.zeros((4, 16), dtype=torch.uint8)
    u8b = torch.zeros((8, 16), dtype=torch.uint8)
    zp = torch.zeros((4,), dtype=torch.int32)
    ws = torch.zeros((8,), dtype=torch.int32)
    off = torch.tensor([0, 4], dtype=torch.int32)
    calls = [
        lambda: qk.quantize_per_token(x),
        lambda: qk.silu_mul_quant_per_token(x, x),
        lambda: qk.quantize_per_token_fp8(x),
        lambda: qk.silu_mul_quant_per_token_fp8(x, x),
        lambda: qk.w8a8_gemm(a, b, s4, s8),
        lambda: qk.fp8_gemm(u8a, u8b, s4, s8),
        lambda: qk.quantize_per_token_asym(x),
        lambda: qk.quantize_static(x, torch.ones((1,), dtype=torch.float32)),
        lambda: qk.weight_row_sums(b),
        lambda: qk.w8a8_gemm_asym(a, zp, b, ws, s4, s8),
        lambda: qk.w8a8_moe_gemm(a, off, b, s4, s8, 4),
        lambda: qk.w8a8_linear(x, b, s8),
        lambda: qk.linear(x, b, s8),
        lambda: qk.mlp_down(x, x, b, s8),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA tensors only"):
            call()


def test_product_never_touches_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", text, re.M), f
                assert "qk_oracle" not in text and "libqk_oracle" not in text, f
