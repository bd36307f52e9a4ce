"""GPU parity of the per-token quantisers against the CPU oracle: INT8 values
and scales bit-exact.  Shapes: the vLLM PR's test grid (tokens 1, 7, 64, 256 x
hidden 64, 512, 4096; its fp16 column is replaced by fp32), edge cases, and the
full-size activations of the five workloads."""
import numpy as np
import pytest

from gpu_util import assert_bits, dev, host, need_gpu, x_dev
from oracle.oracle import Oracle
from w8a8_int8_quantized_qk_b200 import qk, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def O():
    need_gpu()
    return Oracle()


def _rand(m, k, dtype, seed, outliers=0.0):
    r = synth.streams(seed, ["x", "o"])
    x, _ = synth.activation(r["x"], r["o"], m, k, dtype, outliers, 25.0)
    return x


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("k", [64, 512, 4096])
@pytest.mark.parametrize("m", [1, 7, 64, 256])
def test_quant_grid(O, m, k, dtype):
    x = _rand(m, k, dtype, seed=1000 + m + k, outliers=0.01)
    q, s = qk.quantize_per_token(x_dev(x))
    qr, sr = O.quantize_per_token(x)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("k", [64, 512, 4096])
@pytest.mark.parametrize("m", [1, 7, 64, 256])
def test_silu_grid(O, m, k, dtype):
    g, u = synth.make_silu(m, k, seed=2000 + m + k, dtype=dtype)
    q, s = qk.silu_mul_quant_per_token(x_dev(g), x_dev(u))
    qr, sr = O.silu_mul_quant_per_token(g, u)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")


def test_silu_packed_layout(O):
    g, u = synth.make_silu(33, 1040, seed=5)
    gu = np.concatenate([g, u], axis=1)
    q, s = qk.silu_mul_quant_packed(x_dev(gu))
    qr, sr = O.silu_mul_quant_packed(gu)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")


def test_silu_wide_range(O):
    # gate values spanning the exp clamp (|g| up to 100) and tiny values
    r = np.random.default_rng(3)
    g = (r.standard_normal((8, 2048)) * np.float32(30)).astype(np.float32)
    g[0, :16] = [0, -0.0, 1e-30, -1e-30, 87, -87, 88, -88, 89, -89, 100, -100, 1e-3, -1e-3, 5, -5]
    u = r.standard_normal((8, 2048)).astype(np.float32)
    q, s = qk.silu_mul_quant_per_token(dev(g), dev(u))
    qr, sr = O.silu_mul_quant_per_token(g, u)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")


def test_quant_half_amax_ties(O):
    # x = amax / 2 makes RN(x * inv) an exact tie at +-63.5 for most amax while
    # the exact product is not a tie; q must come from the rounded product
    # (two roundings, as written), not from a fused multiply-add.
    r = np.random.default_rng(21)
    amax = (r.uniform(1, 100, 512)).astype(np.float32)
    x = np.zeros((512, 64), np.float32)
    x[:, 0] = amax
    x[:, 1:33] = (amax / 2)[:, None] * np.where(r.random((512, 32)) < 0.5, -1, 1)
    x[:, 33:] = (r.standard_normal((512, 31)) * (amax / 8)[:, None])
    import torch
    xb = torch.from_numpy(x).to(torch.bfloat16)
    for xin in (x, xb.view(torch.int16).numpy().view(np.uint16)):
        q, s = qk.quantize_per_token(x_dev(xin))
        qr, sr = O.quantize_per_token(xin)
        assert_bits(host(q), qr, "q")
        assert_bits(host(s), sr, "scale")


def test_quant_special_rows(O):
    k = 256
    x = np.zeros((8, k), np.float32)
    x[1] = 3.0                       # constant row -> all 127
    x[2] = -0.25                     # constant negative row -> all -127
    x[3] = 1e-14                     # below the 1e-12 floor
    x[4, :6] = [127.0, 62.5, 63.5, -0.5, 126.5, -126.5]  # exact ties at scale 1
    x[5] = np.linspace(-1, 1, k, dtype=np.float32)
    x[6, 17] = 1e30                  # a single huge value
    x[7] = np.float32(1e-38)         # subnormal-range values survive (no flush to zero)
    x[7, ::2] = np.float32(1e-40)
    q, s = qk.quantize_per_token(dev(x))
    qr, sr = O.quantize_per_token(x)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")
    assert host(q)[4, :6].tolist() == [127, 62, 64, 0, 126, -126]


@pytest.mark.parametrize("m,k,dtype", [(3, 16, "bf16"), (2, 16, "f32"), (5, 65536, "bf16"),
                                       (3, 131088, "f32"), (2, 131088, "bf16"), (300, 2064, "bf16"),
                                       (1, 8192, "f32")])
def test_quant_shapes(O, m, k, dtype):
    # covers the smallest row, the cluster split, and the two-pass form (rows
    # longer than 8 CTAs x 512 threads x 8 vectors)
    x = _rand(m, k, dtype, seed=m * 7 + k)
    q, s = qk.quantize_per_token(x_dev(x))
    qr, sr = O.quantize_per_token(x)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")
    g, u = synth.make_silu(m, k, seed=k + 1, dtype=dtype)
    q, s = qk.silu_mul_quant_per_token(x_dev(g), x_dev(u))
    qr, sr = O.silu_mul_quant_per_token(g, u)
    assert_bits(host(q), qr, "q silu")
    assert_bits(host(s), sr, "scale silu")


def test_quant_empty(O):
    import torch
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    q, s = qk.quantize_per_token(x)
    assert q.shape == (0, 64) and s.shape == (0,)


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "group"])
def test_workload_activation_quant(O, name):
    w = synth.make(name)
    q, s = qk.quantize_per_token(x_dev(w.x))
    qr, sr = O.quantize_per_token(w.x)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")


def test_workload_mlp_down_prologue(O):
    w = synth.make("mlp_down")
    q, s = qk.silu_mul_quant_per_token(x_dev(w.gate), x_dev(w.up))
    qr, sr = O.silu_mul_quant_per_token(w.gate, w.up)
    assert_bits(host(q), qr, "q")
    assert_bits(host(s), sr, "scale")


def test_silu_arithmetic_every_binary32():
    # The fused SiLU product as the quantisers compute it (partly on packed
    # binary32 pairs) equals the definition's scalar chain on every finite
    # binary32 gate value: the whole domain of that arithmetic, in four
    # launches.
    need_gpu()
    import torch

    bad = torch.zeros((1,), dtype=torch.int64, device="cuda")
    low = torch.full((1,), -1, dtype=torch.int32, device="cuda")  # 0xFFFFFFFF
    for first in range(0, 1 << 32, 1 << 30):
        st = qk.qk_selftest_silu(first, 1 << 30, qk._ptr(bad), qk._ptr(low), qk._stream())
        assert st == qk.QK_OK, qk.qk_status_string(st)
    torch.cuda.synchronize()
    n = int(bad.item())
    assert n == 0, f"{n} mismatches, first at bits 0x{int(low.item()) & 0xFFFFFFFF:08x}"
