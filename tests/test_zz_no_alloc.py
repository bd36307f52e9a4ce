"""GPU test of qk_w8a8_gemm_noalloc, the GEMM entry point for callers that
cannot allocate device memory (for example a plugin inside an inference
runtime that owns all device memory, or a path where cudaMalloc's device
synchronisation is not acceptable).  Instead of a caller workspace it uses a
scratch array built into the library.

The test calls it through the C ABI on a problem that needs split-K scratch,
twice in a row, and checks each result against the regular entry point
(qk_w8a8_gemm with its own zero-filled workspace): int32 sums identical,
bf16 outputs within the suite's tolerance.  It also checks that every
split-K problem fits the built-in array.  It works both alone in a fresh
process and after the rest of the suite.
"""
import numpy as np
import pytest

from gpu_util import check_out, dev, host, need_gpu
from w8a8_int8_quantized_qk_b200 import qk, synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

NOALLOC_SCRATCH_BYTES = qk.NOALLOC_SCRATCH_BYTES  # QK_NOALLOC_SCRATCH_BYTES of include/qk.h


def _inputs(m, n, k, seed):
    r = synth.streams(seed, ["a", "w", "sa", "sw"])
    return (synth.int8_uniform(r["a"], (m, k)), synth.int8_uniform(r["w"], (n, k)),
            synth.scales_uniform(r["sa"], (m,), 0.001, 0.05), synth.scales_uniform(r["sw"], (n,)))


def _call_noalloc(m, n, k, a, w, sa, sw, alpha):
    out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    c = torch.empty((m, n), dtype=torch.int32, device="cuda")
    st = qk.qk_w8a8_gemm_noalloc(m, n, k, qk._ptr(a), qk._ptr(w), qk._ptr(sa), qk._ptr(sw), 0,
                                 alpha, qk._ptr(c), qk._ptr(out), qk.QK_BF16, qk._stream())
    assert st == qk.QK_OK, qk.qk_status_string(st)
    torch.cuda.synchronize()
    assert qk.device_status() == qk.QK_OK
    return host(out), host(c)


def _call_regular(m, n, k, a, w, sa, sw, alpha):
    need = qk.qk_w8a8_gemm_workspace_size(m, n, k, 0)
    ws = torch.zeros((max(need, 1),), dtype=torch.uint8, device="cuda")
    out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    c = torch.empty((m, n), dtype=torch.int32, device="cuda")
    st = qk.qk_w8a8_gemm(m, n, k, qk._ptr(a), qk._ptr(w), qk._ptr(sa), qk._ptr(sw), 0, alpha,
                         qk._ptr(c), qk._ptr(out), qk.QK_BF16, qk._ptr(ws), ws.numel(), qk._stream())
    assert st == qk.QK_OK, qk.qk_status_string(st)
    torch.cuda.synchronize()
    return host(out), host(c)


@pytest.mark.parametrize("m,n,k", [(256, 1024, 14336), (256, 8960, 4096), (2304, 2304, 2048),
                                   (4096, 4096, 4096)])
def test_noalloc_matches_regular_entry_point(m, n, k):
    need_gpu()
    need = qk.qk_w8a8_gemm_workspace_size(m, n, k, 0)
    assert 0 < need <= NOALLOC_SCRATCH_BYTES  # split-K or tail split, within the built-in scratch
    a_h, w_h, sa_h, sw_h = _inputs(m, n, k, seed=m + n + k)
    a, w, sa, sw = dev(a_h), dev(w_h), dev(sa_h), dev(sw_h)
    ref_out, ref_c = _call_regular(m, n, k, a, w, sa, sw, 0.5)
    ref_f32 = synth.bf16_bits_to_f32(ref_out)
    for _ in range(2):  # two calls in a row share the built-in scratch
        out, c = _call_noalloc(m, n, k, a, w, sa, sw, 0.5)
        assert np.array_equal(c, ref_c)
        check_out(out, ref_f32, ref_out)


def test_noalloc_without_split_k_and_scratch_bound():
    need_gpu()
    # a shape that needs no scratch behaves like the regular call
    m, n, k = 512, 1024, 512
    a_h, w_h, sa_h, sw_h = _inputs(m, n, k, seed=7)
    a, w, sa, sw = dev(a_h), dev(w_h), dev(sa_h), dev(sw_h)
    assert qk.qk_w8a8_gemm_workspace_size(m, n, k, 0) == 0
    out, c = _call_noalloc(m, n, k, a, w, sa, sw, 1.0)
    ref_out, ref_c = _call_regular(m, n, k, a, w, sa, sw, 1.0)
    assert np.array_equal(c, ref_c) and np.array_equal(out, ref_out)
    # every split-K problem fits the built-in scratch: split-K runs only with
    # fewer than 64 output tiles (4 KB + 256 KB per tile), and the tail split
    # keeps at most 128 partial tiles of 256 KB past 4 KB + 16 MB
    for m, n, k in [(200, 256, 131072), (256, 4096, 14336), (1024, 3072, 8192), (2000, 1800, 4096),
                    (4096, 4096, 4096), (4096, 14336, 4096), (2560, 2048, 4096), (9000, 2304, 8192)]:
        assert qk.qk_w8a8_gemm_workspace_size(m, n, k, 0) <= NOALLOC_SCRATCH_BYTES


def test_noalloc_group_split():
    # group mode, output only: on 148 SMs the 160 tiles of 128 x 256 cut the
    # last wave's 12 tiles at their middle group, whose running sums pass
    # through the scratch (one counter per tile, left zero for the next call)
    need_gpu()
    m, n, k = 1280, 4096, 1024
    need = qk.qk_w8a8_gemm_workspace_size(m, n, k, 128)
    assert need <= NOALLOC_SCRATCH_BYTES
    r = synth.streams(11, ["a", "w", "sa", "sw"])
    a = dev(synth.int8_uniform(r["a"], (m, k)))
    w = dev(synth.int8_uniform(r["w"], (n, k)))
    sa = dev(synth.scales_uniform(r["sa"], (m,), 0.001, 0.05))
    sw = dev(synth.scales_uniform(r["sw"], (n, k // 128)))
    ws = torch.zeros((max(need, 1),), dtype=torch.uint8, device="cuda")
    ref = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    st = qk.qk_w8a8_gemm(m, n, k, qk._ptr(a), qk._ptr(w), qk._ptr(sa), qk._ptr(sw), 128, 1.0, None,
                         qk._ptr(ref), qk.QK_BF16, qk._ptr(ws), ws.numel(), qk._stream())
    assert st == qk.QK_OK, qk.qk_status_string(st)
    for _ in range(2):
        out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        st = qk.qk_w8a8_gemm_noalloc(m, n, k, qk._ptr(a), qk._ptr(w), qk._ptr(sa), qk._ptr(sw), 128,
                                     1.0, None, qk._ptr(out), qk.QK_BF16, qk._stream())
        assert st == qk.QK_OK, qk.qk_status_string(st)
        torch.cuda.synchronize()
        assert qk.device_status() == qk.QK_OK
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    # the regular call left its counters zero: the workspace's first 256 bytes
    assert int(ws[:256].count_nonzero()) == 0
    # every group-mode split fits the built-in scratch (at most 74 cut tiles)
    for m, n, k in [(2048, 8192, 8192), (4096, 14336, 4096), (9472, 4096, 1024), (640, 9472, 2048)]:
        assert qk.qk_w8a8_gemm_workspace_size(m, n, k, 128) <= NOALLOC_SCRATCH_BYTES
