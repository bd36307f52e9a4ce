"""GPU parity of the MoE grouped INT8 GEMM (qk_w8a8_moe_gemm) against the
CPU oracle applied expert by expert (the pinned INT8 GEMM and per-channel
epilogue on each expert's rows): int32-exact products, bf16 and fp32 outputs
bit-identical.  Synthetic routing: token counts per expert drawn from a
skewed distribution, including empty experts, experts with a single token,
counts that are not multiples of 128, and one expert with most tokens."""
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
    return Oracle(nthreads=8)


def _moe(counts, n, k, seed):
    r = synth.streams(seed, ["a", "w", "sa", "sw"])
    total = int(sum(counts))
    e = len(counts)
    a = synth.int8_uniform(r["a"], (total, k))
    w = synth.int8_uniform(r["w"], (e, n, k))
    sa = synth.scales_uniform(r["sa"], (total,), 0.001, 0.05)
    sw = synth.scales_uniform(r["sw"], (e, n))
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return a, w, sa, sw, off


# Experts averaging fewer than 128 tokens run on the 1-SM kernel (128-row
# tiles), the others on CTA pairs (256-row tiles): the first, second and
# fourth cases take the 1-SM form, the others (and the synthetic routing
# below) the pair form.  The last has 11 x 9 = 99 pair tiles, more than one
# wave on 74 pairs, and its last N tile holds 8 columns.
@pytest.mark.parametrize("counts,n,k", [
    ([5, 0, 130, 1, 256, 77], 264, 512),
    ([0, 0, 3], 136, 272),
    ([1000, 24, 0, 300, 129, 128, 127, 2], 520, 1040),
    ([64] * 16, 2048, 1024),
    ([256, 257, 511, 0, 128], 776, 2064),
    ([300, 300, 300, 100, 100, 0, 100, 100, 180], 2056, 1040),
])
def test_moe_gemm(O, counts, n, k):
    a, w, sa, sw, off = _moe(counts, n, k, seed=sum(counts) + n + k)
    alpha = 0.75
    for dt in (torch.bfloat16, torch.float32):
        out = qk.w8a8_moe_gemm(dev(a), dev(off), dev(w), dev(sa), dev(sw), max(counts), alpha, dt)
        torch.cuda.synchronize()
        assert qk.device_status() == qk.QK_OK
        got = host(out)
        for e in range(len(counts)):
            r0, r1 = int(off[e]), int(off[e + 1])
            if r1 == r0:
                continue
            ref = O.linear_from_q(a[r0:r1], sa[r0:r1], w[e], sw[e], 0, alpha)
            want = ref["out_bf16"] if dt == torch.bfloat16 else ref["out_f32"]
            assert_bits(got[r0:r1], want, f"expert {e}")


def test_moe_synthetic_routing(O):
    # 8 experts, 2048 tokens routed by a skewed (Zipf-like) draw; the bound on
    # tokens per expert is the largest count
    rng = np.random.default_rng(31)
    probs = 1.0 / np.arange(1, 9)
    probs /= probs.sum()
    counts = np.bincount(rng.choice(8, 2048, p=probs), minlength=8).tolist()
    n, k = 512, 2048
    a, w, sa, sw, off = _moe(counts, n, k, seed=32)
    out = host(qk.w8a8_moe_gemm(dev(a), dev(off), dev(w), dev(sa), dev(sw), max(counts), 1.0))
    torch.cuda.synchronize()
    for e in range(8):
        r0, r1 = int(off[e]), int(off[e + 1])
        ref = O.linear_from_q(a[r0:r1], sa[r0:r1], w[e], sw[e], 0, 1.0)
        assert_bits(out[r0:r1], ref["out_bf16"], f"expert {e}")


def test_moe_errors():
    need_gpu()
    a = torch.zeros((4, 64), dtype=torch.int8, device="cuda")
    b = torch.zeros((2, 16, 64), dtype=torch.int8, device="cuda")
    s = torch.ones((32,), dtype=torch.float32, device="cuda")
    off = torch.tensor([0, 2, 4], dtype=torch.int32, device="cuda")
    out = torch.empty((4, 16), dtype=torch.bfloat16, device="cuda")
    st = qk.qk_w8a8_moe_gemm(2, 4, 16, 40, 4, qk._ptr(off), qk._ptr(a), qk._ptr(b), qk._ptr(s), qk._ptr(s),
                             1.0, qk._ptr(out), qk.QK_BF16, qk._stream())
    assert st == qk.QK_ERR_INVALID_ARG  # k % 16
    st = qk.qk_w8a8_moe_gemm(0, 4, 16, 64, 4, qk._ptr(off), qk._ptr(a), qk._ptr(b), qk._ptr(s), qk._ptr(s),
                             1.0, qk._ptr(out), qk.QK_BF16, qk._stream())
    assert st == qk.QK_ERR_INVALID_ARG  # no experts
