"""GPU parity of the asymmetric per-token INT8 mode against the CPU oracle:
q, scales and zero-points bit-exact; the weight row sums exact; the
zero-point GEMM's int32 sums bit-exact and its bf16 / fp32 outputs
bit-identical to the oracle's, on shapes that take every kernel (decode
GEMV, 1-SM with and without the cluster split-K, CTA pair with split-K and
with the tail split)."""
import numpy as np
import pytest

from gpu_util import assert_bits, dev, host, need_gpu, x_dev
from oracle.oracle import Oracle
from w8a8_int8_quantized_qk_b200 import qk, synth

pytestmark = pytest.mark.gpu

import torch  # noqa: E402


@pytest.fixture(scope="module")
def O():
    need_gpu()
    return Oracle()


def _rand(m, k, dtype, seed, shift=0.0):
    r = synth.streams(seed, ["x", "o"])
    x, _ = synth.activation(r["x"], r["o"], m, k, dtype, 0.01, 20.0)
    if shift:
        x32 = synth.bf16_bits_to_f32(x) if x.dtype == np.uint16 else x
        x32 = (x32 + np.float32(shift)).astype(np.float32)
        x = synth.to_bf16_bits(x32) if dtype == "bf16" else x32
    return x


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("m,k,shift", [(1, 64, 0.0), (7, 512, 2.0), (64, 4096, -1.5), (256, 1024, 0.0),
                                       (33, 14336, 3.0), (3, 16, 0.0)])
def test_asym_quant(O, m, k, dtype, shift):
    x = _rand(m, k, dtype, seed=6000 + m + k, shift=shift)
    q, s, z = qk.quantize_per_token_asym(x_dev(x))
    qr, sr, zr = O.quantize_per_token_asym(x)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")
    assert_bits(host(z), zr, "zero point")


def test_asym_quant_special_rows(O):
    x = np.zeros((5, 64), np.float32)
    x[1, :8] = [0.0, 1.0, 127.0, 128.0, 255.0, 2.5, 3.5, 200.4]
    x[2, :4] = [-255.0, -100.0, 0.0, -0.5]
    x[3] = 1e-14
    x[4] = np.linspace(5.0, 9.0, 64, dtype=np.float32)  # all positive: range widened to 0
    q, s, z = qk.quantize_per_token_asym(x_dev(x))
    qr, sr, zr = O.quantize_per_token_asym(x)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")
    assert_bits(host(z), zr, "zero point")


@pytest.mark.parametrize("n,k", [(8, 16), (1032, 4112), (4096, 14336)])
def test_weight_row_sums(O, n, k):
    w = synth.int8_uniform(synth.streams(n + k, ["w"])["w"], (n, k))
    got = host(qk.weight_row_sums(dev(w)))
    assert np.array_equal(got, O.weight_row_sums(w))


ASYM_SHAPES = [(4, 136, 272), (8, 1032, 4112), (9, 256, 128), (100, 1032, 3008), (64, 4096, 4096),
               (257, 520, 1040), (300, 520, 2048), (256, 1024, 14336), (2304, 2304, 2048)]


@pytest.mark.parametrize("m,n,k", ASYM_SHAPES)
def test_asym_gemm(O, m, n, k):
    r = synth.streams(m * 3 + n + k, ["x", "o", "w", "sw"])
    x, _ = synth.activation(r["x"], r["o"], m, k, "bf16", 0.01, 20.0)
    w = synth.int8_uniform(r["w"], (n, k))
    sw = synth.scales_uniform(r["sw"], (n,))
    q, sa, zp = qk.quantize_per_token_asym(x_dev(x))
    wd = dev(w)
    wsum = qk.weight_row_sums(wd)
    alpha = 0.5
    out, c = qk.w8a8_gemm_asym(q, zp, wd, wsum, sa, dev(sw), alpha, want_c=True)
    out32, _ = qk.w8a8_gemm_asym(q, zp, wd, wsum, sa, dev(sw), alpha, out_dtype=torch.float32)
    out_nc, _ = qk.w8a8_gemm_asym(q, zp, wd, wsum, sa, dev(sw), alpha)  # bf16 via TMA stores
    torch.cuda.synchronize()
    assert qk.device_status() == qk.QK_OK
    qh, sah, zh = host(q), host(sa), host(zp)
    qr, sr, zr = O.quantize_per_token_asym(x)
    assert_bits(qh, qr, "q")
    assert_bits(sah, sr, "scale")
    assert_bits(zh, zr, "zero point")
    if m * n * k <= 2 ** 31:
        acc = O.gemm_s32_asym(qh, zh, w)
    else:  # the same sum, from the pinned plain GEMM and row sums (exact in int64)
        acc = (O.gemm_s32(qh, w).astype(np.int64) -
               zh.astype(np.int64)[:, None] * O.weight_row_sums(w).astype(np.int64)[None, :]).astype(np.int32)
    ref = O.epilogue_per_channel(acc, sah, sw, alpha)
    assert_bits(host(c), acc, "acc")
    assert_bits(host(out), O.f32_to_bf16(ref), "bf16 out")
    assert_bits(host(out32), ref, "fp32 out")
    assert_bits(host(out_nc), O.f32_to_bf16(ref), "bf16 out, no c")


def test_asym_errors():
    need_gpu()
    a = torch.zeros((4, 66320), dtype=torch.int8, device="cuda")
    w = torch.zeros((16, 66320), dtype=torch.int8, device="cuda")
    z = torch.zeros((16,), dtype=torch.int32, device="cuda")
    s = torch.ones((16,), dtype=torch.float32, device="cuda")
    out = torch.empty((4, 16), dtype=torch.bfloat16, device="cuda")
    st = qk.qk_w8a8_gemm_asym(4, 16, 66320, qk._ptr(a), qk._ptr(z), qk._ptr(w), qk._ptr(z), qk._ptr(s),
                              qk._ptr(s), 1.0, None, qk._ptr(out), qk.QK_BF16, None, 0, qk._stream())
    assert st == qk.QK_ERR_OVERFLOW_BOUND
    st = qk.qk_w8a8_gemm_asym(4, 16, 64, qk._ptr(a), None, qk._ptr(w), qk._ptr(z), qk._ptr(s),
                              qk._ptr(s), 1.0, None, qk._ptr(out), qk.QK_BF16, None, 0, qk._stream())
    assert st == qk.QK_ERR_INVALID_ARG


# ---------------------------------------------------------------- static per-tensor
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("m,k,scale", [(1, 16, 1.0), (7, 512, 0.02), (300, 4096, 0.05),
                                       (4096, 4096, 0.03), (3, 14336, 0.25)])
def test_static_quant(O, m, k, dtype, scale):
    x = _rand(m, k, dtype, seed=7000 + m + k)
    s = torch.tensor([scale], dtype=torch.float32, device="cuda")
    q = qk.quantize_static(x_dev(x), s)
    torch.cuda.synchronize()
    assert_bits(host(q), O.quantize_static(x, scale), "q")


def test_static_then_gemm(O):
    # a static per-tensor scale feeds the GEMM as an [m] vector of one value
    m, n, k, scale = 200, 264, 384, 0.04
    r = synth.streams(71, ["x", "o", "w", "sw"])
    x, _ = synth.activation(r["x"], r["o"], m, k, "bf16", 0.01, 20.0)
    w = synth.int8_uniform(r["w"], (n, k))
    sw = synth.scales_uniform(r["sw"], (n,))
    q = qk.quantize_static(x_dev(x), torch.tensor([scale], dtype=torch.float32, device="cuda"))
    sa = torch.full((m,), scale, dtype=torch.float32, device="cuda")
    out, c = qk.w8a8_gemm(q, dev(w), sa, dev(sw), 0, 1.0, want_c=True)
    torch.cuda.synchronize()
    qr = O.quantize_static(x, scale)
    ref = O.linear_from_q(qr, np.full((m,), scale, np.float32), w, sw, 0, 1.0)
    assert_bits(host(c), ref["acc"], "acc")
    assert_bits(host(out), ref["out_bf16"], "bf16 out")
