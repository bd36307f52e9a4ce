"""GPU parity of qk_w8a8_gemm against the CPU oracle.

INT32 accumulators bit-exact; fp32/bf16 outputs within the tolerance of
gpu_util.check_out and, because the kernels keep the oracle's operation
order, bit-identical as well.  Small shapes span several tiles with ragged
M, N and K tails, on each kernel (decode GEMV for m <= 8, the tcgen05 kernel
per channel and per 128-group); the five workloads run at full size, every
output element compared with the oracle."""
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


def _problem(m, n, k, group_k, seed):
    r = synth.streams(seed, ["a", "w", "sa", "sw"])
    a = synth.int8_uniform(r["a"], (m, k))
    w = synth.int8_uniform(r["w"], (n, k))
    sa = synth.scales_uniform(r["sa"], (m,), 0.001, 0.05)
    sw = synth.scales_uniform(r["sw"], (n, k // group_k) if group_k else (n,))
    return a, w, sa, sw


def _run(a, w, sa, sw, group_k, alpha, out_dtype=torch.bfloat16, want_c=True):
    out, c = qk.w8a8_gemm(dev(a), dev(w), dev(sa), dev(sw), group_k, alpha, out_dtype,
                          want_out=out_dtype is not None, want_c=want_c)
    torch.cuda.synchronize()
    assert qk.device_status() == qk.QK_OK
    return (None if out is None else host(out)), (None if c is None else host(c))


SHAPES = [
    # decode GEMV (m <= 8)
    (1, 8, 16), (3, 24, 48), (4, 136, 272), (8, 1032, 4112), (5, 64, 1024),
    # tcgen05 per-channel: one tile, tails in M / N / K, several tiles and waves
    (9, 256, 128), (128, 256, 128), (130, 264, 272), (257, 520, 1040), (300, 1000, 1552),
    (1024, 2048, 512), (640, 256, 4096), (17, 8, 16),
]


@pytest.mark.parametrize("m,n,k", SHAPES)
def test_gemm_per_channel(O, m, n, k):
    a, w, sa, sw = _problem(m, n, k, 0, seed=m * 131 + n * 7 + k)
    alpha = 0.75
    out, c = _run(a, w, sa, sw, 0, alpha)
    ref = O.linear_from_q(a, sa, w, sw, 0, alpha)
    assert_bits(c, ref["acc"], "acc")
    exact = check_out(out, ref["out_f32"], ref["out_bf16"])
    assert exact == 1.0, exact


@pytest.mark.parametrize("m,n,k", [(4, 64, 256), (200, 264, 384)])
def test_gemm_fp32_out_and_c_only(O, m, n, k):
    a, w, sa, sw = _problem(m, n, k, 0, seed=77 + m)
    out, c = _run(a, w, sa, sw, 0, 1.0, out_dtype=torch.float32)
    ref = O.linear_from_q(a, sa, w, sw, 0, 1.0)
    assert_bits(c, ref["acc"], "acc")
    assert_bits(out, ref["out_f32"], "fp32 out")
    out2, c2 = _run(a, w, sa, sw, 0, 1.0, out_dtype=None, want_c=True)
    assert out2 is None
    assert_bits(c2, ref["acc"], "acc (c only)")
    out3, c3 = _run(a, w, sa, sw, 0, 1.0, want_c=False)
    assert c3 is None
    assert_bits(out3, ref["out_bf16"], "bf16 (out only)")


# few output tiles, so K is split across CTA pairs: the partial sums meet
# through distributed shared memory in a cluster of the tile's pairs
# (200x512x4096: 4 splits, 300x520x2048: 2, 256x4096x14336: 3) or in the
# workspace (256x1024x14336 and 256x8960x4096); 129x264x1024 is not split
SPLIT_SHAPES = [(200, 512, 4096), (300, 520, 2048), (256, 4096, 14336), (256, 1024, 14336),
                (256, 8960, 4096), (129, 264, 1024)]


@pytest.mark.parametrize("m,n,k", SPLIT_SHAPES)
def test_gemm_split_k(O, m, n, k):
    # run twice: the workspace form's counters and accumulators must be back
    # at zero
    a, w, sa, sw = _problem(m, n, k, 0, seed=m + 3 * n + k)
    ref = O.linear_from_q(a, sa, w, sw, 0, 1.5)
    for _ in range(2):
        out, c = _run(a, w, sa, sw, 0, 1.5)
        assert_bits(c, ref["acc"], "acc")
        assert_bits(out, ref["out_bf16"], "bf16 out")


# few 128 x 128 or 128 x 256 tiles on the 1-SM kernel (m <= 128, or m <= 256
# when that gives each CTA fewer K blocks than the CTA-pair plan): K is split
# across the CTAs of a cluster and the partials meet in distributed shared
# memory
CHANNEL_SPLIT_SHAPES = [(64, 4096, 4096), (100, 1032, 3008), (17, 520, 2048), (256, 4096, 14336),
                        (100, 10240, 3072)]


@pytest.mark.parametrize("m,n,k", CHANNEL_SPLIT_SHAPES)
def test_gemm_channel_cluster_split(O, m, n, k):
    assert qk.qk_w8a8_gemm_workspace_size(m, n, k, 0) == 0  # no workspace: DSMEM
    a, w, sa, sw = _problem(m, n, k, 0, seed=m * 3 + n + 7 * k)
    ref = O.linear_from_q(a, sa, w, sw, 0, 0.75)
    for _ in range(2):
        out, c = _run(a, w, sa, sw, 0, 0.75)
        assert_bits(c, ref["acc"], "acc")
        assert_bits(out, ref["out_bf16"], "bf16 out")
    out32, _ = _run(a, w, sa, sw, 0, 0.75, out_dtype=torch.float32, want_c=False)
    assert_bits(out32, ref["out_f32"], "fp32 out")
    out16, _ = _run(a, w, sa, sw, 0, 0.75, want_c=False)  # bf16 through TMA stores
    assert_bits(out16, ref["out_bf16"], "bf16 out, no c")


# the two tile widths of the 1-SM kernel: 128 x 128 where it puts more CTAs
# to work (with 4 or 2 cluster K slices, or none), 128 x 256 otherwise
WIDTH_SHAPES = [((128, 4096, 14336), "128x128 tiles, cluster split-K in 4 slices"),
                ((96, 8192, 4096), "128x128 tiles, cluster split-K in 2 slices"),
                ((120, 4104, 2064), "128x128 tiles, cluster split-K in 2 slices"),
                ((100, 1000, 1024), "128x128 tiles)"),
                ((100, 10240, 3072), "128x256 tiles, cluster split-K in "),
                ((256, 4096, 14336), "128x256 tiles, cluster split-K in 4 slices")]


@pytest.mark.parametrize("shape,form", WIDTH_SHAPES)
def test_gemm_channel_tile_widths(O, shape, form):
    m, n, k = shape
    assert qk.qk_w8a8_gemm_kernel(m, n, k, 0, True).startswith("gemm_i8_channel_kernel (1 SM, " + form)
    a, w, sa, sw = _problem(m, n, k, 0, seed=m + 3 * n + k)
    ref = O.linear_from_q(a, sa, w, sw, 0, 1.25)
    out, c = _run(a, w, sa, sw, 0, 1.25)
    assert_bits(c, ref["acc"], "acc")
    assert_bits(out, ref["out_bf16"], "bf16 out")
    out16, _ = _run(a, w, sa, sw, 0, 1.25, want_c=False)  # bf16 through TMA stores
    assert_bits(out16, ref["out_bf16"], "bf16 out, no c")
    out32, _ = _run(a, w, sa, sw, 0, 1.25, out_dtype=torch.float32, want_c=False)
    assert_bits(out32, ref["out_f32"], "fp32 out")


# more output tiles than CTA pairs, not a whole number of waves: the tiles of
# the last partial wave are cut into K slices that run first, and their
# partials meet in the workspace (2, 3 and 4 slices; ragged M, N and K)
TAIL_SHAPES = [(2304, 2304, 2048), (2500, 2056, 3008), (2560, 2048, 4096), (1280, 4096, 8192)]


@pytest.mark.parametrize("m,n,k", TAIL_SHAPES)
def test_gemm_tail_split(O, m, n, k):
    assert qk.qk_w8a8_gemm_workspace_size(m, n, k, 0) > 0  # the tail split is planned
    a, w, sa, sw = _problem(m, n, k, 0, seed=m + 5 * n + k)
    ref = O.linear_from_q(a, sa, w, sw, 0, 0.5)
    for _ in range(2):  # the workspace must be back at zero after each call
        out, c = _run(a, w, sa, sw, 0, 0.5)
        assert_bits(c, ref["acc"], "acc")
        assert_bits(out, ref["out_bf16"], "bf16 out")


def test_gemm_split_k_needs_workspace(O):
    m, n, k = 256, 1024, 14336
    need = qk.qk_w8a8_gemm_workspace_size(m, n, k, 0)
    assert need > 0
    a, w, sa, sw = (dev(t) for t in _problem(m, n, k, 0, seed=1))
    out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    st = qk.qk_w8a8_gemm(m, n, k, qk._ptr(a), qk._ptr(w), qk._ptr(sa), qk._ptr(sw), 0, 1.0, None,
                         qk._ptr(out), qk.QK_BF16, None, 0, qk._stream())
    assert st == qk.QK_ERR_WORKSPACE


GROUP_SHAPES = [(1, 128, 128), (7, 136, 256), (129, 136, 256), (200, 264, 384), (256, 512, 1024),
                (333, 1032, 2048)]


@pytest.mark.parametrize("m,n,k", GROUP_SHAPES)
def test_gemm_group(O, m, n, k):
    a, w, sa, sw = _problem(m, n, k, 128, seed=m * 17 + n + k)
    alpha = 1.25
    out, c = _run(a, w, sa, sw, 128, alpha)
    ref = O.linear_from_q(a, sa, w, sw, 128, alpha)
    assert_bits(c, ref["acc"], "acc")
    exact = check_out(out, ref["out_f32"], ref["out_bf16"])
    assert exact == 1.0, exact
    out_nc, _ = _run(a, w, sa, sw, 128, alpha, want_c=False)
    assert_bits(out_nc, out, "group out without c")


# group mode without the int32 sums runs the CTA-pair kernel for m > 128
# (256 x 256 tiles): more tiles than pairs (several per pair), group counts
# that are not a multiple of the 8-group scale slice (3, 17), ragged M and N
# edges, bf16 (TMA-store) and fp32 outputs.  With 74 pairs, 1100 x 4360 (90
# tiles) and 1280 x 4096 (80 tiles) cut their last wave's tiles at the
# middle group (17 groups: 8 + 9; 2 groups: 1 + 1), one pair continuing
# another's running sums.
# (m <= 128 takes the 1-SM 128 x 256 kernel: 128 x 40448 is 158 tiles on
# 148 SMs, so its last wave is cut too.)
GROUP_WIDE_SHAPES = [(1100, 4360, 2176), (1280, 4096, 256), (300, 2056, 384), (129, 264, 128),
                     (128, 40448, 384)]


@pytest.mark.parametrize("m,n,k", GROUP_WIDE_SHAPES)
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_gemm_group_without_c(O, m, n, k, out_dtype):
    a, w, sa, sw = _problem(m, n, k, 128, seed=m * 5 + n * 3 + k)
    alpha = 0.75
    out, c = _run(a, w, sa, sw, 128, alpha, out_dtype=out_dtype, want_c=False)
    assert c is None
    ref = O.linear_from_q(a, sa, w, sw, 128, alpha)
    if out_dtype == torch.float32:
        assert_bits(out, ref["out_f32"], "fp32 out")
    else:
        exact = check_out(out, ref["out_f32"], ref["out_bf16"])
        assert exact == 1.0, exact


def test_gemm_saturating_closed_form(O):
    # all operands 127: acc = 16129 k at the largest k the bound allows (multiple of 128)
    k = 133120
    a = np.full((3, k), 127, np.int8)
    w = np.full((16, k), 127, np.int8)
    sa = np.ones(3, np.float32)
    sw = np.ones(16, np.float32)
    _, c = _run(a, w, sa, sw, 0, 1.0, out_dtype=None)
    assert np.all(c == 16129 * k)
    a9 = np.full((9, k), 127, np.int8)
    _, c9 = _run(a9, -w, np.ones(9, np.float32), sw, 0, 1.0, out_dtype=None)
    assert np.all(c9 == -16129 * k)


def test_gemm_empty(O):
    a = torch.empty((0, 64), dtype=torch.int8, device="cuda")
    w = torch.zeros((16, 64), dtype=torch.int8, device="cuda")
    sa = torch.empty((0,), dtype=torch.float32, device="cuda")
    sw = torch.ones((16,), dtype=torch.float32, device="cuda")
    out, _ = qk.w8a8_gemm(a, w, sa, sw)
    assert out.shape == (0, 16)


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "mlp_down", "group"])
def test_workload_full_size(O, name):
    w = synth.make(name)
    if name == "tiny":
        # per-output-channel weight quantisation with the same per-row rule
        w_q, sw = qk.quantize_per_token(dev(w.w_f32))
        w_q_ref, sw_ref = O.quantize_per_token(w.w_f32)
        assert_bits(host(w_q), w_q_ref, "weight q")
        assert_bits(host(sw), sw_ref, "weight scale")
        w_q_h, sw_h = w_q_ref, sw_ref
    else:
        w_q, sw = dev(w.w_q), dev(w.sw)
        w_q_h, sw_h = w.w_q, w.sw
    if name == "mlp_down":
        q, sa = qk.silu_mul_quant_per_token(x_dev(w.gate), x_dev(w.up))
        q_ref, sa_ref = O.silu_mul_quant_per_token(w.gate, w.up)
    else:
        q, sa = qk.quantize_per_token(x_dev(w.x))
        q_ref, sa_ref = O.quantize_per_token(w.x)
    assert_bits(host(q), q_ref, "q")
    assert_bits(host(sa), sa_ref, "scale")
    out_dtype = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    out, c = qk.w8a8_gemm(q, w_q, sa, sw, w.group_k, w.alpha, out_dtype, want_c=True)
    torch.cuda.synchronize()
    assert qk.device_status() == qk.QK_OK
    # every row and column of the full-size output against the oracle (the
    # threaded oracle does the 4096^3 layer in seconds)
    ref = O.linear_from_q(q_ref, sa_ref, w_q_h, sw_h, w.group_k, w.alpha)
    out_h, c_h = host(out), host(c)
    assert_bits(c_h, ref["acc"], "acc")
    if out_dtype == torch.float32:
        assert_bits(out_h, ref["out_f32"], "fp32 out")
    else:
        exact = check_out(out_h, ref["out_f32"], ref["out_bf16"])
        assert exact == 1.0, exact
    # the output-only launch (the form the benchmark times; for group mode a
    # different kernel) gives the same bits
    out_only, _ = qk.w8a8_gemm(q, w_q, sa, sw, w.group_k, w.alpha, out_dtype, want_c=False)
    torch.cuda.synchronize()
    assert qk.device_status() == qk.QK_OK
    assert_bits(host(out_only), out_h, "output-only launch")


def _golden(name):
    import json
    import os

    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", name)) as f:
        return json.load(f)


def _hexf(v):
    return np.float32(float.fromhex(v))


# Every output element of these problems is the hand-derived value of the
# golden epilogue_order.json, whose rounding differs under any reordering of
# the epilogue; each shape reaches a different kernel or split form (GEMV,
# 1-SM, 1-SM cluster split-K, CTA pair, pair tail split, pair workspace
# split-K).
ORDER_SHAPES = [(4, 64, 128), (64, 256, 128), (64, 4096, 4096), (512, 512, 128), (2304, 2304, 2048),
                (256, 1024, 14336)]


@pytest.mark.parametrize("m,n,k", ORDER_SHAPES)
def test_epilogue_order_golden(O, m, n, k):
    for case in _golden("epilogue_order.json")["per_channel"]:
        a = np.zeros((m, k), np.int8)
        w = np.zeros((n, k), np.int8)
        a[:, 0] = case["acc"]
        w[:, 0] = 1
        sa = np.full((m,), _hexf(case["sa"]), np.float32)
        sw = np.full((n,), _hexf(case["sw"]), np.float32)
        for want_c in (True, False):
            out, c = _run(a, w, sa, sw, 0, float(_hexf(case["alpha"])), out_dtype=torch.float32,
                          want_c=want_c)
            want = np.full((m, n), _hexf(case["out"]), np.float32)
            assert_bits(out, want, f"per-channel order, case {case['out']}")


# the group chain: the 128 x 128 kernel (with c), the 128 x 256 kernel (m =
# 1), the CTA-pair kernel, and (1280 x 4096, 80 pair tiles on 74 pairs) the
# cut last wave, where one pair continues another's running sums between
# the two groups
@pytest.mark.parametrize("m,n", [(1, 128), (300, 2056), (1280, 4096)])
def test_group_order_golden(O, m, n):
    for case in _golden("epilogue_order.json")["group"]:
        gk = case["group_k"]
        ng = len(case["partials"])
        a = np.zeros((m, gk * ng), np.int8)
        w = np.zeros((n, gk * ng), np.int8)
        for i, (av, wv) in enumerate(case["partials"]):
            a[:, i * gk] = av
            w[:, i * gk] = wv
        sa = np.full((m,), _hexf(case["sa"]), np.float32)
        sw = np.tile(np.float32([_hexf(v) for v in case["sw"]]), (n, 1))
        want = np.full((m, n), _hexf(case["out"]), np.float32)
        for want_c in (True, False):
            out, c = _run(a, w, sa, sw, gk, float(_hexf(case["alpha"])), out_dtype=torch.float32,
                          want_c=want_c)
            assert_bits(out, want, "group order")
            if want_c:
                assert np.all(c == case["acc"])
