"""GPU tests of the library's runtime behaviour: the bounded-wait path sets
the device status word without faulting, calls honour the caller's stream,
and repeated calls are deterministic."""
import numpy as np
import pytest

from gpu_util import dev, host, need_gpu, x_dev
from w8a8_int8_quantized_qk_b200 import qk, synth

pytestmark = pytest.mark.gpu

import torch  # noqa: E402


def test_bounded_wait_reports_timeout():
    need_gpu()
    assert qk.device_status() == qk.QK_OK
    s = torch.cuda.current_stream()
    assert qk.qk_selftest_bounded_wait(20000, qk._stream(s)) == qk.QK_OK  # 20 ms
    assert qk.device_status() == qk.QK_ERR_TIMEOUT
    assert qk.device_status() == qk.QK_OK  # read clears it
    # the context is still usable afterwards
    x = torch.ones((4, 64), dtype=torch.bfloat16, device="cuda")
    q, sc = qk.quantize_per_token(x)
    torch.cuda.synchronize()
    assert int(q.min()) == 127


def test_side_stream_and_determinism():
    need_gpu()
    w = synth.make_linear(512, 1024, 2048, seed=9)
    x = dev(w.x.view(np.int16)).view(torch.bfloat16)
    wq, sw = dev(w.w_q), dev(w.sw)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out1 = qk.linear(x, wq, sw)
    s.synchronize()
    out2 = qk.linear(x, wq, sw)
    torch.cuda.synchronize()
    assert np.array_equal(host(out1), host(out2))
    assert qk.device_status() == qk.QK_OK


def test_split_k_workspace_left_zero():
    # split-K adds partial sums into the workspace, and the tail split (more
    # tiles than CTA pairs) stores them there; every completed call must
    # leave the counters and the split-K accumulators zero again
    need_gpu()
    for (m, n, k) in [(256, 1024, 14336), (256, 8960, 4096), (2304, 2304, 2048), (2500, 2056, 3008)]:
        need = qk.qk_w8a8_gemm_workspace_size(m, n, k, 0)
        assert need > 0
        r = synth.streams(m + n, ["a", "w", "sa", "sw"])
        a = dev(synth.int8_uniform(r["a"], (m, k)))
        w = dev(synth.int8_uniform(r["w"], (n, k)))
        sa = dev(synth.scales_uniform(r["sa"], (m,), 0.001, 0.05))
        sw = dev(synth.scales_uniform(r["sw"], (n,)))
        ws = torch.zeros((need,), dtype=torch.uint8, device="cuda")
        outs = []
        for _ in range(3):
            out, _ = qk.w8a8_gemm(a, w, sa, sw, workspace=ws)
            torch.cuda.synchronize()
            assert qk.device_status() == qk.QK_OK
            # the counters and split-K accumulators (the first 4 KB + 16 MB);
            # tail-split partials past them are scratch
            assert int(ws[:4096 + (16 << 20)].count_nonzero()) == 0
            outs.append(host(out))
        assert all(np.array_equal(outs[0], o) for o in outs[1:])


def test_group_split_leaves_shared_workspace_usable():
    # group mode's last-wave split passes running sums through the workspace;
    # they must land past the counters and split-K accumulators, so that a
    # per-channel split-K call can reuse the same workspace right after
    need_gpu()
    mg, ng, kg = 1280, 4096, 1024  # 160 group tiles on 148 SMs: 12 cut tiles
    mc, nc, kc = 256, 8960, 4096   # per-channel split-K through the workspace
    need = max(qk.qk_w8a8_gemm_workspace_size(mg, ng, kg, 128),
               qk.qk_w8a8_gemm_workspace_size(mc, nc, kc, 0))
    ws = torch.zeros((need,), dtype=torch.uint8, device="cuda")
    r = synth.streams(21, ["a", "w", "sa", "sw", "a2", "w2", "sa2", "sw2"])
    ag = dev(synth.int8_uniform(r["a"], (mg, kg)))
    wg = dev(synth.int8_uniform(r["w"], (ng, kg)))
    sag = dev(synth.scales_uniform(r["sa"], (mg,), 0.001, 0.05))
    swg = dev(synth.scales_uniform(r["sw"], (ng, kg // 128)))
    ac = dev(synth.int8_uniform(r["a2"], (mc, kc)))
    wc = dev(synth.int8_uniform(r["w2"], (nc, kc)))
    sac = dev(synth.scales_uniform(r["sa2"], (mc,), 0.001, 0.05))
    swc = dev(synth.scales_uniform(r["sw2"], (nc,)))
    ref_c, _ = qk.w8a8_gemm(ac, wc, sac, swc, workspace=torch.zeros_like(ws))
    ref_g, _ = qk.w8a8_gemm(ag, wg, sag, swg, 128, workspace=torch.zeros_like(ws))
    for _ in range(2):
        out_g, _ = qk.w8a8_gemm(ag, wg, sag, swg, 128, workspace=ws)
        torch.cuda.synchronize()
        assert int(ws[:4096 + (16 << 20)].count_nonzero()) == 0
        out_c, _ = qk.w8a8_gemm(ac, wc, sac, swc, workspace=ws)
        torch.cuda.synchronize()
        assert qk.device_status() == qk.QK_OK
        assert torch.equal(out_g.view(torch.int16), ref_g.view(torch.int16))
        assert torch.equal(out_c.view(torch.int16), ref_c.view(torch.int16))


def test_graph_capture_of_the_layer():
    # the same quantise + GEMM calls captured into a CUDA graph and replayed
    # (as the benchmark runs them) give the eager results, including the
    # split-K path and the SiLU prologue
    need_gpu()
    w = synth.make_linear(300, 520, 2048, seed=13)
    x = x_dev(w.x)
    wq, sw = dev(w.w_q), dev(w.sw)
    g_, u_ = synth.make_silu(64, 2048, seed=14)
    gd, ud = x_dev(g_), x_dev(u_)
    ref = host(qk.linear(x, wq, sw))
    q_ref, s_ref = (host(t) for t in qk.silu_mul_quant_per_token(gd, ud))
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        out = qk.linear(x, wq, sw)
        q, s = qk.silu_mul_quant_per_token(gd, ud)
    for _ in range(2):
        out.zero_()
        q.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert qk.device_status() == qk.QK_OK
        assert np.array_equal(host(out), ref)
        assert np.array_equal(host(q), q_ref) and np.array_equal(host(s), s_ref)


def test_kernel_query_names_the_planned_kernel():
    need_gpu()
    q = qk.qk_w8a8_gemm_kernel
    assert q(4, 14336, 4096, 0, False).startswith("gemv_i8_prefetch_kernel")
    assert q(16, 256, 512, 0, False) == "gemm_i8_channel_kernel (1 SM, 128x128 tiles)"
    assert q(128, 4096, 14336, 0, False) == "gemm_i8_channel_kernel (1 SM, 128x128 tiles, cluster split-K in 4 slices)"
    assert q(256, 4096, 14336, 0, False).startswith("gemm_i8_channel_kernel (1 SM, 128x256 tiles, cluster split-K")
    assert q(4096, 4096, 4096, 0, False).startswith("gemm_i8_pair_kernel (CTA pair, 256x256 tiles, last wave cut")
    assert q(2048, 8192, 8192, 128, False) == "gemm_i8_group_pair_kernel (CTA pair, 256x256 tiles)"
    assert q(2048, 8192, 8192, 128, True) == "gemm_i8_group_kernel (1 SM, 128x128 tiles)"
    assert q(64, 8192, 8192, 128, False) == "gemm_i8_group_wide_kernel (1 SM, 128x256 tiles)"


def test_mma_rate_probe_runs():
    # the INT8 peak probe on zero and on random operands: every pair MMA loop
    # completes, and the rate per clock is the same for both
    need_gpu()
    zero = qk.mma_rate(2, 256, 2048, launches=1)
    rnd = qk.mma_rate(2, 256, 2048, launches=1, operand_seed=7)
    assert qk.device_status() == qk.QK_OK
    for r in (zero, rnd):
        assert r["tops"] > 0 and r["cycles"] > 0
    # 8192 multiply-adds per clock per SM at the full rate; allow slack
    assert abs(zero["macs_per_clk_per_sm"] - rnd["macs_per_clk_per_sm"]) < 0.05 * zero["macs_per_clk_per_sm"]


def test_mma_interference_probe_runs():
    # every companion loop stops when the MMAs are done, and the MMA-only
    # form reports about 512 cycles per group of four MMAs
    need_gpu()
    res = qk.mma_interference(groups=512)
    assert qk.device_status() == qk.QK_OK
    assert set(res) == set(qk.MMA_COMPANIONS.values())
    for name, r in res.items():
        assert r["cycles_per_group"] >= 500, (name, r)
    assert res["none"]["cycles_per_group"] < 600


def test_mma_interference_rejects_bad_arguments():
    need_gpu()
    s = qk._stream(torch.cuda.current_stream())
    assert qk.qk_selftest_mma_interference(7, 16, 2, None, s) == qk.QK_ERR_INVALID_ARG
    assert qk.qk_selftest_mma_interference(0, 16, 3, None, s) == qk.QK_ERR_INVALID_ARG
    assert qk.qk_selftest_mma_interference(0, 0, 2, None, s) == qk.QK_ERR_INVALID_ARG
