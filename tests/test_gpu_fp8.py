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
