"""GPU parity of qk_w8a8_linear, the whole layer in one call (quantiser
into the workspace, then the GEMM), against the CPU oracle and against the
two-call form (qk_quantize_per_token + qk_w8a8_gemm): decode shapes (the
GEMV), larger M and group scales, bf16 and fp32 inputs.  Per-token scales
bit-exact; outputs within the oracle's bf16/fp32 rounding and bit-identical
to the two-call form."""
import numpy as np
import pytest

from gpu_util import assert_bits, check_out, dev, host, need_gpu, x_dev
from oracle.oracle import Oracle
from w8a8_int8_quantized_qk_b200 import qk, synth

pytestmark = pytest.mark.gpu

import torch  # noqa: E402


@pytest.fixture(scope="module")
def O():
    need_gpu()
    return Oracle()


def _two_call(x, w_q, sw, group_k, alpha, out_dtype):
    q, sa = qk.quantize_per_token(x)
    out, _ = qk.w8a8_gemm(q, w_q, sa, sw, group_k, alpha, out_dtype)
    return out, sa


DECODE = [(1, 64, 16), (2, 136, 272), (3, 520, 4096), (4, 1032, 4112), (5, 256, 8192), (8, 264, 4096),
          (4, 128, 12288), (2, 64, 16384), (7, 72, 1040)]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("m,n,k", DECODE)
def test_linear_decode(O, m, n, k, dtype):
    assert qk.qk_w8a8_linear_workspace_size(m, n, k, 0) >= m * k + 4 * m
    w = synth.make_linear(m, n, k, seed=m * 31 + n + k, x_dtype=dtype, outlier_frac=0.01,
                          outlier_scale=20.0)
    x, wq, sw = x_dev(w.x), dev(w.w_q), dev(w.sw)
    alpha = 0.5
    out_dtype = torch.float32 if dtype == "f32" else torch.bfloat16
    out, sa = qk.w8a8_linear(x, wq, sw, 0, alpha, out_dtype, want_scale=True)
    torch.cuda.synchronize()
    assert qk.device_status() == qk.QK_OK
    ref = O.linear(w.x, w.w_q, w.sw, 0, alpha)
    assert_bits(host(sa), ref["sa"], "scale")
    if out_dtype == torch.float32:
        assert_bits(host(out), ref["out_f32"], "fp32 out")
    else:
        assert check_out(host(out), ref["out_f32"], ref["out_bf16"]) == 1.0
    out2, sa2 = _two_call(x, wq, sw, 0, alpha, out_dtype)
    assert_bits(host(out), host(out2), "one call vs two calls")
    # the one-launch form (the quantiser inside the GEMV's grid)
    out3, sa3 = qk.w8a8_linear_fused(x, wq, sw, alpha, out_dtype, want_scale=True)
    torch.cuda.synchronize()
    assert qk.device_status() == qk.QK_OK
    assert_bits(host(sa3), ref["sa"], "scale (one launch)")
    assert_bits(host(out3), host(out2), "one launch vs two calls")


@pytest.mark.parametrize("m,n,k,group_k", [(9, 256, 512, 0), (300, 520, 2048, 0), (200, 264, 384, 128),
                                           (4, 136, 256, 128)])
def test_linear_workspace_form(O, m, n, k, group_k):
    need = qk.qk_w8a8_linear_workspace_size(m, n, k, group_k)
    assert need > 0
    w = synth.make_linear(m, n, k, seed=m + n + k, group_k=group_k)
    x, wq, sw = x_dev(w.x), dev(w.w_q), dev(w.sw)
    ws = torch.zeros((need,), dtype=torch.uint8, device="cuda")
    for _ in range(2):  # the workspace is reused
        out, sa = qk.w8a8_linear(x, wq, sw, group_k, 1.25, want_scale=True, workspace=ws)
        torch.cuda.synchronize()
        assert qk.device_status() == qk.QK_OK
        ref = O.linear(w.x, w.w_q, w.sw, group_k, 1.25)
        assert_bits(host(sa), ref["sa"], "scale")
        assert check_out(host(out), ref["out_f32"], ref["out_bf16"]) == 1.0


def test_linear_decode_workload_and_api(O):
    w = synth.make("decode")
    x, wq, sw = x_dev(w.x), dev(w.w_q), dev(w.sw)
    out = qk.linear(x, wq, sw, 0, w.alpha)  # two calls, torch-allocated q and scales
    out_f, sa = qk.w8a8_linear(x, wq, sw, 0, w.alpha, want_scale=True)
    torch.cuda.synchronize()
    ref = O.linear(w.x, w.w_q, w.sw, 0, w.alpha)
    assert_bits(host(sa), ref["sa"], "scale")
    assert check_out(host(out), ref["out_f32"], ref["out_bf16"]) == 1.0
    assert_bits(host(out), host(out_f), "qk.linear vs qk.w8a8_linear")


@pytest.mark.parametrize("m,k", [(16, 64), (9, 256), (8, 16384), (5, 8208)])
def test_linear_fused_unsupported_shapes(m, k):
    # beyond the decode shapes: m > 8, or m > 4 with k > 8192
    need_gpu()
    n = 16
    x = torch.zeros((m, k), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((n, k), dtype=torch.int8, device="cuda")
    sw = torch.ones((n,), dtype=torch.float32, device="cuda")
    out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros((qk.qk_w8a8_linear_workspace_size(m, n, k, 0),), dtype=torch.uint8, device="cuda")
    st = qk.qk_w8a8_linear_fused(m, n, k, qk._ptr(x), qk.QK_BF16, qk._ptr(w), qk._ptr(sw), 1.0, None,
                                 qk._ptr(out), qk.QK_BF16, qk._ptr(ws), ws.numel(), qk._stream())
    assert st == qk.QK_ERR_UNSUPPORTED


def test_linear_errors():
    need_gpu()
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((16, 64), dtype=torch.int8, device="cuda")
    sw = torch.ones((16,), dtype=torch.float32, device="cuda")
    out = torch.empty((4, 16), dtype=torch.bfloat16, device="cuda")
    st = qk.qk_w8a8_linear(4, 16, 64, qk._ptr(x), qk.QK_BF16, qk._ptr(w), qk._ptr(sw), 0, 1.0, None,
                           None, qk.QK_BF16, None, 0, qk._stream())
    assert st == qk.QK_ERR_INVALID_ARG  # out is required
    st = qk.qk_w8a8_linear(4, 16, 64, qk._ptr(x), qk.QK_BF16, qk._ptr(w), qk._ptr(sw), 0, 1.0, None,
                           qk._ptr(out), qk.QK_BF16, None, 0, qk._stream())
    assert st == qk.QK_ERR_WORKSPACE  # q and the scales live in the workspace


@pytest.mark.parametrize("m,n,k,dtype", [(4, 14336, 4096, "bf16"), (1, 520, 4096, "bf16"), (8, 264, 8192, "f32"),
                                         (4, 264, 16384, "f32"), (3, 1032, 4112, "bf16")])
def test_linear_decode_one_launch_reuses_workspace(O, m, n, k, dtype):
    # qk_w8a8_linear_fused quantises the tokens inside the GEMV's launch and
    # hands them over through flag words in the workspace: three calls with
    # new tokens on one workspace, each bit-identical to the oracle and to the
    # two-call form, and the flags back at zero after every call
    need = qk.qk_w8a8_linear_workspace_size(m, n, k, 0)
    ws = torch.zeros((need,), dtype=torch.uint8, device="cuda")
    g_bytes = 0  # the GEMV takes no GEMM workspace: the flags come first
    assert qk.qk_w8a8_gemm_workspace_size(m, n, k, 0) == 0
    out_dtype = torch.float32 if dtype == "f32" else torch.bfloat16
    for call in range(3):
        w = synth.make_linear(m, n, k, seed=1000 * call + m + n + k, x_dtype=dtype, outlier_frac=0.01,
                              outlier_scale=20.0)
        x, wq, sw = x_dev(w.x), dev(w.w_q), dev(w.sw)
        out, sa = qk.w8a8_linear_fused(x, wq, sw, 0.75, out_dtype, want_scale=True, workspace=ws)
        torch.cuda.synchronize()
        assert qk.device_status() == qk.QK_OK
        assert int(ws[g_bytes:g_bytes + 256].count_nonzero()) == 0, "flags left set"
        ref = O.linear(w.x, w.w_q, w.sw, 0, 0.75)
        assert_bits(host(sa), ref["sa"], "scale")
        if out_dtype == torch.float32:
            assert_bits(host(out), ref["out_f32"], "fp32 out")
        else:
            assert check_out(host(out), ref["out_f32"], ref["out_bf16"]) == 1.0
        out2, _ = _two_call(x, wq, sw, 0, 0.75, out_dtype)
        assert_bits(host(out), host(out2), "one launch vs two calls")
