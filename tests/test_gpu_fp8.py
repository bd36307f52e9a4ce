"""GPU parity of the FP8 (e4m3) variant against the CPU oracle: the per-token
FP8 quantisers (plain and fused SiLU; e4m3 codes and scales bit-exact, with
and without the scale upper bound), on the vLLM PR's own test grid (tokens 1,
7, 64, 256 x hidden 64, 512, 4096; its fp16 column is replaced by fp32), on
shapes that take each quantiser kernel, and on the full-size activations."""
import numpy as np
import pytest

from gpu_util import assert_bits, host, need_gpu, x_dev
from oracle.oracle import Oracle
from w8a8_int8_quantized_qk_b200 import qk, synth

pytestmark = pytest.mark.gpu

import torch  # noqa: E402


@pytest.fixture(scope="module")
def O():
    need_gpu()
    return Oracle()


def _rand(m, k, dtype, seed, outliers=0.0):
    r = synth.streams(seed, ["x", "o"])
    x, _ = synth.activation(r["x"], r["o"], m, k, dtype, outliers, 25.0)
    return x


def _ub(v):
    return None if v is None else torch.tensor([v], dtype=torch.float32, device="cuda")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("k", [64, 512, 4096])
@pytest.mark.parametrize("m", [1, 7, 64, 256])
def test_fp8_quant_grid(O, m, k, dtype):
    x = _rand(m, k, dtype, seed=3000 + m + k, outliers=0.01)
    q, s = qk.quantize_per_token_fp8(x_dev(x))
    qr, sr = O.quantize_per_token_fp8(x)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("k", [64, 512, 4096])
@pytest.mark.parametrize("m", [1, 7, 64, 256])
def test_fp8_silu_grid(O, m, k, dtype):
    g, u = synth.make_silu(m, k, seed=4000 + m + k, dtype=dtype)
    q, s = qk.silu_mul_quant_per_token_fp8(x_dev(g), x_dev(u))
    qr, sr = O.silu_mul_quant_per_token_fp8(g, u)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")


@pytest.mark.parametrize("ub", [0.001, 0.01, 1e-9])
def test_fp8_scale_upper_bound(O, ub):
    # rows with absmax / 448 above the bound take the bound as their scale and
    # saturate at +-448; rows below it are unaffected
    x = _rand(40, 1024, "bf16", seed=77, outliers=0.02)
    x32 = synth.bf16_bits_to_f32(x)
    x32[::3] *= 0.01
    x = synth.to_bf16_bits(x32)
    q, s = qk.quantize_per_token_fp8(x_dev(x), scale_ub=_ub(ub))
    qr, sr = O.quantize_per_token_fp8(x, scale_ub=ub)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")
    g, u = synth.make_silu(9, 512, seed=78)
    q2, s2 = qk.silu_mul_quant_per_token_fp8(x_dev(g), x_dev(u), scale_ub=_ub(ub))
    qr2, sr2 = O.silu_mul_quant_per_token_fp8(g, u, scale_ub=ub)
    assert_bits(host(q2), qr2, "q silu")
    assert_bits(host(s2), sr2, "scale silu")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("m,k", [(2, 16), (3, 48), (5, 2064), (2, 16384), (1, 65536), (9, 131072),
                                 (400, 1024), (333, 4112), (600, 8192), (300, 2048)])
def test_fp8_quant_kernel_paths(O, m, k, dtype):
    # few rows (one CTA per row, or a cluster per row), rows too long for the
    # chip (two-pass form), and many rows (persistent form)
    x = _rand(m, k, dtype, seed=5000 + m * 7 + k, outliers=0.005)
    q, s = qk.quantize_per_token_fp8(x_dev(x))
    qr, sr = O.quantize_per_token_fp8(x)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")


def test_fp8_special_rows(O):
    # zero row, a row below the 1e-12 floor, exact e4m3 values and ties
    x = np.zeros((4, 64), np.float32)
    x[1] = 1e-14
    x[2, :7] = [448.0, -1.0, 1.0625, 1.1875, 3.0 * 2.0 ** -10, 17.0, -0.0]
    x[3] = np.linspace(-3.0, 3.0, 64, dtype=np.float32)
    q, s = qk.quantize_per_token_fp8(x_dev(x))
    qr, sr = O.quantize_per_token_fp8(x)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")


@pytest.mark.parametrize("name", ["prefill", "group"])
def test_fp8_workload_activation_quant(O, name):
    w = synth.make(name)
    q, s = qk.quantize_per_token_fp8(x_dev(w.x))
    qr, sr = O.quantize_per_token_fp8(w.x)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")


def test_fp8_workload_mlp_down_prologue(O):
    w = synth.make("mlp_down")
    q, s = qk.silu_mul_quant_per_token_fp8(x_dev(w.gate), x_dev(w.up))
    qr, sr = O.silu_mul_quant_per_token_fp8(w.gate, w.up)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")


# ---------------------------------------------------------------- FP8 GEMM
def _fp8_problem(m, n, k, seed):
    r = synth.streams(seed, ["a", "w", "sa", "sw"])
    return (synth.e4m3_codes(r["a"], (m, k)), synth.e4m3_codes(r["w"], (n, k)),
            synth.scales_uniform(r["sa"], (m,), 0.001, 0.05), synth.scales_uniform(r["sw"], (n,)))


def _fp8_bound(O, a, w, sa, sw, alpha, rows=None):
    """Per-element bound on |gpu - exact| for the fp32 output: fp32 summation
    of k products inside the tensor core (at most k * 2^-24 of the sum of the
    products' magnitudes, the worst case of any summation order) plus the
    three fp32 multiplies of the epilogue (2^-22 of the value)."""
    da = np.abs(O.e4m3_to_f32(a).astype(np.float64))
    dw = np.abs(O.e4m3_to_f32(w).astype(np.float64))
    s_abs = da @ dw.T
    k = a.shape[1]
    scale = np.abs(sa.astype(np.float64))[:, None] * np.abs(sw.astype(np.float64))[None, :] * abs(alpha)
    return (k * 2.0 ** -24 * s_abs) * scale


def _check_fp8(O, got, acc_exact, bound, sa, sw, alpha, bf16):
    ref = acc_exact * sa.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :] * alpha
    g = synth.bf16_bits_to_f32(got).astype(np.float64) if bf16 else got.astype(np.float64)
    extra = np.abs(ref) * (2.0 ** -8 if bf16 else 2.0 ** -22)
    err = np.abs(g - ref)
    assert np.all(err <= bound + extra), float((err - bound - extra).max())
    # the norm criterion of the INT8 path holds as well
    l2 = np.sqrt(np.sum(ref * ref, axis=1, keepdims=True))
    assert float((err / np.where(l2 > 0, l2, 1.0)).max(initial=0.0)) <= 2e-2


FP8_GEMM_SHAPES = [(1, 64, 32), (4, 136, 272), (9, 256, 128), (100, 1032, 3008), (128, 256, 4096),
                   (130, 264, 272), (257, 520, 1040), (300, 1000, 1552), (1024, 2048, 512),
                   # K split over the CTAs of a cluster, fp32 partials added in
                   # slice order: 1-SM kernel, clusters of 4 (few tiles, m <= 128)
                   (64, 512, 8192),
                   # CTA-pair kernel, cluster split-K (few tiles)
                   (256, 1024, 8192),
                   # CTA-pair kernel, more tiles than pairs (whole tiles)
                   (2560, 2048, 2048)]


@pytest.mark.parametrize("m,n,k", FP8_GEMM_SHAPES)
def test_fp8_gemm(O, m, n, k):
    a, w, sa, sw = _fp8_problem(m, n, k, seed=m * 13 + n + 3 * k)
    alpha = 0.75
    acc, _ = O.gemm_fp8(a, w)
    bound = _fp8_bound(O, a, w, sa, sw, alpha)
    for dt in (torch.float32, torch.bfloat16):
        out = qk.fp8_gemm(torch.from_numpy(a).cuda(), torch.from_numpy(w).cuda(),
                          torch.from_numpy(sa).cuda(), torch.from_numpy(sw).cuda(), alpha, dt)
        torch.cuda.synchronize()
        assert qk.device_status() == qk.QK_OK
        _check_fp8(O, host(out), acc, bound, sa, sw, alpha, dt == torch.bfloat16)


def test_fp8_gemm_split_deterministic():
    # the cluster split-K adds the fp32 partials in slice order, whichever CTA
    # finishes first: repeated launches give the same bits
    need_gpu()
    for m, n, k in ((256, 1024, 8192), (64, 512, 8192)):
        a, w, sa, sw = (torch.from_numpy(t).cuda() for t in _fp8_problem(m, n, k, seed=m + n + k))
        ref = qk.fp8_gemm(a, w, sa, sw, 1.0, torch.float32)
        for _ in range(3):
            again = qk.fp8_gemm(a, w, sa, sw, 1.0, torch.float32)
            torch.cuda.synchronize()
            assert torch.equal(again.view(torch.int32), ref.view(torch.int32))
        assert qk.device_status() == qk.QK_OK


def test_fp8_linear_chain(O):
    # quantise per token to e4m3 on the GPU (bit-exact), then the FP8 GEMM of
    # those codes against e4m3 weights at the prefill shape
    w = synth.make("prefill")
    x = x_dev(w.x)
    q, sa = qk.quantize_per_token_fp8(x)
    r = synth.streams(99, ["w", "sw"])
    wq = synth.e4m3_codes(r["w"], (w.n, w.k))
    sw = synth.scales_uniform(r["sw"], (w.n,))
    out = qk.fp8_gemm(q, torch.from_numpy(wq).cuda(), sa, torch.from_numpy(sw).cuda(), 1.0)
    torch.cuda.synchronize()
    assert qk.device_status() == qk.QK_OK
    # every row of the 4096 x 4096 output
    qh, sah = host(q), host(sa)
    qr, sr = O.quantize_per_token_fp8(w.x)
    assert_bits(qh, qr, "q")
    assert_bits(sah, sr, "scale")
    acc, _ = O.gemm_fp8(qh, wq)
    bound = _fp8_bound(O, qh, wq, sah, sw, 1.0)
    _check_fp8(O, host(out), acc, bound, sah, sw, 1.0, True)


def test_fp8_gemm_errors():
    need_gpu()
    a = torch.zeros((4, 40), dtype=torch.uint8, device="cuda")
    w = torch.zeros((16, 40), dtype=torch.uint8, device="cuda")
    s = torch.ones((16,), dtype=torch.float32, device="cuda")
    out = torch.empty((4, 16), dtype=torch.bfloat16, device="cuda")
    st = qk.qk_fp8_gemm(4, 16, 40, qk._ptr(a), qk._ptr(w), qk._ptr(s), qk._ptr(s), 1.0, qk._ptr(out),
                        qk.QK_BF16, qk._stream())
    assert st == qk.QK_ERR_INVALID_ARG  # k % 16 != 0
    st = qk.qk_fp8_gemm(4, 16, 32, qk._ptr(a), qk._ptr(w), qk._ptr(s), qk._ptr(s), 1.0, None,
                        qk.QK_BF16, qk._stream())
    assert st == qk.QK_ERR_INVALID_ARG  # out is required
