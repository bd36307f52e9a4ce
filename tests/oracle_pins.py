"""Pins of the CPU oracle against facts that do not come from the oracle.

Each ``pin_*`` function takes an :class:`oracle.oracle.Oracle` and raises
``AssertionError`` when the oracle disagrees with the pages or with the
mathematics.  ``test_oracle_pins.py`` runs them on the real oracle;
``test_oracle_mutants.py`` runs them on copies of the oracle with a planted
mistake and requires that some pin fails for every such copy.

What pins what:

* exp / SiLU        -- float64 ``math.exp`` error bound (2 ulp); silu(0) = 0;
                       silu(x) - silu(-x) = x.
* bf16 rounding     -- torch's CPU float32 -> bfloat16 cast.
* quantiser         -- hand-worked fixtures with exact ties (golden
                       ``quant_hand.json``); absmax element -> +-127;
                       scale * 127 ~ absmax; round-trip bound; q monotone
                       in x; bf16 input path == widened fp32 path.
* INT8 GEMM         -- numpy int64 matmul (brute force); closed forms
                       (all-127 operands give 16129 K); identity weights;
                       the int32 bound K * 127^2 < 2^31.
* epilogues         -- float64 value within the rounding bound of the
                       left-to-right fp32 chain; exact power-of-two cases;
                       group mode against a float64 sum of per-group terms;
                       the operation order itself on hand-derived values
                       that round differently under any reordering (golden
                       ``epilogue_order.json``).
* whole chain       -- hand-worked example (golden ``linear_hand.json``).
* FP8 e4m3 codec    -- torch's float8_e4m3fn (decode of all 256 codes; the
                       float32 -> e4m3 cast on random values, every
                       representable value and every tie midpoint);
                       closed forms from the format (448, 2^-6, 2^-9, ties
                       to the even code).
* FP8 quantiser     -- absmax element -> +-448; scale * 448 ~ absmax;
                       round-trip bound of half an e4m3 spacing; the
                       scale_ub clamp; a hand-worked row.
* FP8 GEMM          -- numpy float64 matmul of the decoded operands (exact
                       at these sizes); closed forms (all-448 operands).
* asymmetric INT8   -- hand-worked rows with scale 1 (q = x - 128, ties to
                       even); zero-point and extreme-element invariants;
                       round-trip bound; numpy int64 brute force of the
                       zero-point GEMM and of the weight row sums.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def ulp32(x: float) -> float:
    return float(np.spacing(np.float32(abs(x))))


# --------------------------------------------------------------------------- exp / silu
def pin_exp(O) -> None:
    """qko_exp is within 2 ulp of float64 exp over the clamped range."""
    grid = np.concatenate([np.linspace(-87.0, 88.0, 40001, dtype=np.float32),
                           np.float32([0.0, 1.0, -1.0, 0.5, -0.5, 1e-8, -1e-8, 0.34657359, -0.34657359])])
    got = O.exp_array(grid)
    worst = 0.0
    for t, g in zip(grid.tolist(), got.tolist()):
        ref = math.exp(t)
        err = abs(g - ref) / ulp32(ref)
        worst = max(worst, err)
    assert worst <= 2.0, f"exp error {worst} ulp"
    assert O.exp(0.0) == 1.0


def pin_silu(O) -> None:
    assert O.silu(0.0) == 0.0
    rng = np.random.default_rng(7)
    xs = np.concatenate([rng.standard_normal(2000).astype(np.float32) * 4,
                         np.float32([1e-3, -1e-3, 10.0, -10.0, 30.0, -30.0])])
    for x in xs.tolist():
        s_pos, s_neg = O.silu(x), O.silu(-x)
        # silu(x) - silu(-x) = x * (sigmoid(x) + sigmoid(-x)) = x
        assert abs((s_pos - s_neg) - x) <= 4 * ulp32(x) + 4 * ulp32(max(abs(s_pos), abs(s_neg))), x
        ref = x / (1.0 + math.exp(-x))
        assert abs(s_pos - ref) <= 4 * ulp32(ref) + 1e-37, (x, s_pos, ref)


# --------------------------------------------------------------------------- bf16
def pin_bf16_rounding(O) -> None:
    import torch

    rng = np.random.default_rng(11)
    x = rng.standard_normal(20000).astype(np.float32) * np.float32(100)
    bits = x.view(np.uint32)
    # plant exact ties (low 16 bits == 0x8000) with both parities of the kept lsb
    ties = (bits[:4000] & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    x = np.concatenate([x, ties.view(np.float32), np.float32([0.0, -0.0, 1.0, 3.4e38, -3.4e38, 1e-40])])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.f32_to_bf16(x)
    assert np.array_equal(got, ref), int(np.sum(got != ref))


# --------------------------------------------------------------------------- quantiser
def pin_quant_golden(O) -> None:
    for case in _golden("quant_hand.json")["cases"]:
        x = np.float32([case["x"]])
        q, s = O.quantize_per_token(x)
        assert q[0].tolist() == case["q"], (case["x"], q[0].tolist(), case["q"])
        if "scale" in case:
            assert float(s[0]) == case["scale"]
        else:
            target = case["scale_times_127_approx"]
            assert abs(float(s[0]) * 127.0 - target) <= 1e-6 * target


def _check_quant_invariants(x32: np.ndarray, q: np.ndarray, s: np.ndarray) -> None:
    m, k = x32.shape
    x64 = x32.astype(np.float64)
    amax = np.abs(x64).max(axis=1)
    for r in range(m):
        sc = float(s[r])
        floor = max(float(amax[r]), float(np.float32(1e-12)))
        # scale is the fp32 rounding of max(amax, 1e-12) / 127: within half an ulp (+ the
        # rounding of 1e-12 itself)
        assert abs(sc * 127.0 - floor) <= 127.0 * ulp32(sc), (r, sc, floor)
        # round trip: |x - q * scale| <= scale * (1/2 + 2^-16)
        err = np.abs(x64[r] - q[r].astype(np.float64) * sc)
        assert float(err.max()) <= sc * (0.5 + 2.0 ** -16), (r, float(err.max()), sc)
        # range and the absmax element
        assert int(np.abs(q[r].astype(np.int32)).max()) <= 127
        if amax[r] >= 1e-12:
            i = int(np.argmax(np.abs(x64[r])))
            assert abs(int(q[r, i])) == 127 and np.sign(q[r, i]) == np.sign(x64[r, i])
        # monotone: sorting x sorts q
        order = np.argsort(x64[r], kind="stable")
        assert np.all(np.diff(q[r][order].astype(np.int32)) >= 0)


def pin_quant_invariants(O) -> None:
    rng = np.random.default_rng(3)
    x = rng.standard_normal((9, 333)).astype(np.float32)
    x[1] *= 1e-3
    x[2, 17] = 250.0  # one outlier
    x[3] = 0.0
    x[4] = 1e-14
    x[5] = np.abs(x[5])
    x[6] = -np.abs(x[6]) * 7
    q, s = O.quantize_per_token(x)
    _check_quant_invariants(x, q, s)
    # zero row -> 0; a constant row below the 1e-12 floor -> round(1e-14 * 127 / 1e-12) = 1
    assert np.all(q[3] == 0) and np.all(q[4] == 1)


def pin_quant_bf16_path(O) -> None:
    """bf16 input gives the same result as its exact fp32 widening."""
    import torch

    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, 520)).astype(np.float32) * 3
    xb = torch.from_numpy(x).to(torch.bfloat16)
    bits = xb.view(torch.int16).numpy().view(np.uint16)
    wide = xb.to(torch.float32).numpy()
    q1, s1 = O.quantize_per_token(bits)
    q2, s2 = O.quantize_per_token(wide)
    assert np.array_equal(q1, q2) and np.array_equal(s1.view(np.uint32), s2.view(np.uint32))
    _check_quant_invariants(wide, q1, s1)


def pin_silu_quant(O) -> None:
    """fused path == silu then quantise; packed [T, 2d] == separate tensors."""
    import torch

    rng = np.random.default_rng(9)
    g = rng.standard_normal((5, 264)).astype(np.float32)
    u = rng.standard_normal((5, 264)).astype(np.float32)
    q, s = O.silu_mul_quant_per_token(g, u)
    h = np.empty_like(g)
    for r in range(5):
        for i in range(264):
            h[r, i] = np.float32(O.silu(float(g[r, i]))) * u[r, i]
    _check_quant_invariants(h, q, s)
    qh, sh = O.quantize_per_token(h)
    assert np.array_equal(q, qh) and np.array_equal(s, sh)
    gb = torch.from_numpy(g).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ub = torch.from_numpy(u).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q1, s1 = O.silu_mul_quant_per_token(gb, ub)
    q2, s2 = O.silu_mul_quant_packed(np.concatenate([gb, ub], axis=1))
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


# --------------------------------------------------------------------------- GEMM
def pin_gemm_bruteforce(O) -> None:
    rng = np.random.default_rng(13)
    for (m, n, k) in [(1, 1, 1), (3, 5, 7), (2, 9, 33), (16, 256, 512), (7, 13, 200)]:
        a = rng.integers(-127, 128, (m, k), dtype=np.int8)
        w = rng.integers(-127, 128, (n, k), dtype=np.int8)
        ref = a.astype(np.int64) @ w.astype(np.int64).T
        got = O.gemm_s32(a, w)
        assert np.array_equal(got.astype(np.int64), ref), (m, n, k)


def pin_gemm_closed_forms(O) -> None:
    for k in (4096, 8192, 14336):
        a = np.full((2, k), 127, np.int8)
        w = np.full((3, k), 127, np.int8)
        assert np.all(O.gemm_s32(a, w) == 16129 * k)
        assert np.all(O.gemm_s32(a, -w) == -16129 * k)
    # identity-like weights pick columns of a
    rng = np.random.default_rng(17)
    a = rng.integers(-127, 128, (4, 48), dtype=np.int8)
    w = np.zeros((10, 48), np.int8)
    for n in range(10):
        w[n, n] = 1
    assert np.array_equal(O.gemm_s32(a, w), a[:, :10].astype(np.int32))
    # the int32 bound: K * 127^2 < 2^31 holds up to K = 133144 and fails after it
    ok = O.gemm_s32(np.full((1, 133144), 127, np.int8), np.full((1, 133144), 127, np.int8))
    assert int(ok[0, 0]) == 16129 * 133144 == 2147479576
    try:
        O.gemm_s32(np.full((1, 133145), 127, np.int8), np.full((1, 133145), 127, np.int8))
    except OverflowError:
        pass
    else:
        raise AssertionError("int32 overflow not reported")


# --------------------------------------------------------------------------- epilogues
def pin_epilogue_per_channel(O) -> None:
    rng = np.random.default_rng(19)
    m, n = 12, 40
    acc = rng.integers(-2 ** 31 + 1, 2 ** 31 - 1, (m, n), dtype=np.int64).astype(np.int32)
    acc[0, :] = rng.integers(-1000, 1000, n)
    sa = rng.uniform(1e-4, 1.0, m).astype(np.float32)
    sw = rng.uniform(1e-3, 1e-2, n).astype(np.float32)
    for alpha in (1.0, 0.37):
        got = O.epilogue_per_channel(acc, sa, sw, alpha).astype(np.float64)
        exact = (acc.astype(np.float64) * sa.astype(np.float64)[:, None]
                 * sw.astype(np.float64)[None, :] * np.float64(np.float32(alpha)))
        # four binary32 roundings (int->float and three products): relative <= 4 * 2^-24 (+)
        bound = 4.0001 * 2.0 ** -24 * np.abs(exact)
        assert np.all(np.abs(got - exact) <= bound)
    # exact powers of two
    out = O.epilogue_per_channel(np.int32([[3, -5]]), np.float32([0.5]), np.float32([0.25, 4.0]), 2.0)
    assert out.tolist() == [[0.75, -20.0]]


def pin_group(O) -> None:
    rng = np.random.default_rng(23)
    for (m, n, k, grp) in [(3, 5, 256, 128), (4, 6, 384, 128), (2, 3, 192, 64)]:
        a = rng.integers(-127, 128, (m, k), dtype=np.int8)
        w = rng.integers(-127, 128, (n, k), dtype=np.int8)
        ng = k // grp
        sa = rng.uniform(1e-3, 1.0, m).astype(np.float32)
        sw = rng.uniform(1e-3, 1e-2, (n, ng)).astype(np.float32)
        alpha = 1.5
        out, acc = O.gemm_group(a, w, sa, sw, grp, alpha)
        parts = np.stack([a[:, g * grp:(g + 1) * grp].astype(np.int64)
                          @ w[:, g * grp:(g + 1) * grp].astype(np.int64).T for g in range(ng)])
        assert np.array_equal(acc.astype(np.int64), parts.sum(0))
        terms = parts.astype(np.float64) * sw.astype(np.float64).T[:, None, :]
        exact = terms.sum(0) * sa.astype(np.float64)[:, None] * alpha
        mag = np.abs(terms).sum(0) * sa.astype(np.float64)[:, None] * alpha
        bound = (ng + 2.0001) * 2.0 ** -24 * mag
        assert np.all(np.abs(out.astype(np.float64) - exact) <= bound)
    # one group with power-of-two scales is exact
    a = np.int8([[1, 2, 3, 4]])
    w = np.int8([[5, 6, 7, 8], [-1, -1, -1, -1]])
    out, acc = O.gemm_group(a, w, np.float32([0.5]), np.float32([[0.25], [2.0]]), 4, 1.0)
    assert acc.tolist() == [[70, -10]] and out.tolist() == [[8.75, -10.0]]


def _hexf(v: str) -> np.float32:
    return np.float32(float.fromhex(v))


def pin_epilogue_order_golden(O) -> None:
    """Hand-derived values (golden ``epilogue_order.json``) on which a
    reordered epilogue rounds differently: (acc * sa) * sw before alpha, and
    the fused group chain in ascending group order before sa and alpha."""
    g = _golden("epilogue_order.json")
    for case in g["per_channel"]:
        out = O.epilogue_per_channel(np.int32([[case["acc"]]]), np.float32([_hexf(case["sa"])]),
                                     np.float32([_hexf(case["sw"])]), float(_hexf(case["alpha"])))
        want = _hexf(case["out"])
        assert out.view(np.uint32)[0, 0] == np.float32(want).view(np.uint32), \
            (float(out[0, 0]).hex(), case["out"])
    for case in g["group"]:
        gk = case["group_k"]
        ng = len(case["partials"])
        a = np.zeros((1, gk * ng), np.int8)
        w = np.zeros((1, gk * ng), np.int8)
        for i, (av, wv) in enumerate(case["partials"]):
            a[0, i * gk] = av
            w[0, i * gk] = wv
        sw = np.float32([[_hexf(v) for v in case["sw"]]])
        out, acc = O.gemm_group(a, w, np.float32([_hexf(case["sa"])]), sw, gk, float(_hexf(case["alpha"])))
        assert int(acc[0, 0]) == case["acc"]
        want = _hexf(case["out"])
        assert out.view(np.uint32)[0, 0] == np.float32(want).view(np.uint32), \
            (float(out[0, 0]).hex(), case["out"])


# --------------------------------------------------------------------------- whole chain
def pin_linear_golden(O) -> None:
    g = _golden("linear_hand.json")
    x = np.float32(g["x"])
    w = np.int8(g["w"])
    res = O.linear(x, w, np.float32(g["sw"]), 0, g["alpha"])
    assert res["q"].tolist() == g["q"]
    assert res["sa"].tolist() == g["sa"]
    assert res["acc"].tolist() == g["acc"]
    assert res["out_f32"].tolist() == g["out"]


# --------------------------------------------------------------------------- FP8 e4m3
def _torch_e4m3(x: np.ndarray) -> np.ndarray:
    import torch

    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()


def _e4m3_values() -> np.ndarray:
    """The finite non-negative e4m3 values, from torch's float8_e4m3fn decode."""
    import torch

    codes = torch.arange(0, 0x7F, dtype=torch.uint8)  # 0x00 .. 0x7E, NaN is 0x7F
    return codes.view(torch.float8_e4m3fn).float().numpy()


def pin_e4m3_codec(O) -> None:
    import torch

    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy()
    got = O.e4m3_to_f32(codes)
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin]) and np.all(np.isnan(got[~fin]))
    assert sorted(np.where(~fin)[0].tolist()) == [0x7F, 0xFF]
    vals = _e4m3_values()
    mids = ((vals[:-1].astype(np.float64) + vals[1:]) / 2).astype(np.float32)
    rng = np.random.default_rng(11)
    x = np.concatenate([vals, -vals, mids, -mids, rng.uniform(-448, 448, 20000).astype(np.float32),
                        (rng.standard_normal(20000) * 0.02).astype(np.float32)])
    assert np.array_equal(O.f32_to_e4m3(x), _torch_e4m3(x))
    # closed forms of the format: largest finite, smallest normal and
    # subnormal, 1.0, and ties to the even code
    fixed = {448.0: 0x7E, -448.0: 0xFE, 2.0 ** -6: 0x08, 2.0 ** -9: 0x01, 1.0: 0x38,
             2.0 ** -10: 0x00, 3 * 2.0 ** -10: 0x02, 1.0625: 0x38, 1.1875: 0x3A, 0.0: 0x00,
             240.0: 0x77, 232.0: 0x76, 0.01953125: 0x0A}
    got = O.f32_to_e4m3(np.float32(list(fixed)))
    assert got.tolist() == list(fixed.values()), (got.tolist(), list(fixed.values()))


def _check_fp8_quant(O, x32, q, s, ub=None) -> None:
    x64 = x32.astype(np.float64)
    dec = O.e4m3_to_f32(q).astype(np.float64)
    for r in range(x32.shape[0]):
        amax = float(np.abs(x64[r]).max())
        sc = float(s[r])
        want = max(amax, float(np.float32(1e-12))) / 448.0
        if ub is not None and want > ub:
            assert sc == np.float32(ub), (r, sc, ub)
        else:
            assert abs(sc - want) <= ulp32(sc), (r, sc, want)
        y = x64[r] / sc
        inside = np.abs(y) <= 448.0
        # half an e4m3 spacing at |y| (2^-10 in the subnormal range), plus the
        # fp32 rounding of x * inv
        e = np.floor(np.log2(np.maximum(np.abs(y), 2.0 ** -6)))
        half = np.where(np.abs(y) < 2.0 ** -6, 2.0 ** -10, 2.0 ** (e - 4))
        err = np.abs(dec[r] - y)
        assert np.all(err[inside] <= half[inside] * (1 + 1e-6) + np.abs(y[inside]) * 2.0 ** -22)
        # clamped elements saturate at +-448
        assert np.all(np.abs(dec[r][~inside]) == 448.0)
        assert np.all(np.sign(dec[r][~inside]) == np.sign(y[~inside]))
        if ub is None and amax >= 1e-12:
            i = int(np.argmax(np.abs(x64[r])))
            assert dec[r, i] == 448.0 * np.sign(x64[r, i]), (r, dec[r, i])


def pin_fp8_quant(O) -> None:
    rng = np.random.default_rng(12)
    x = rng.standard_normal((6, 257)).astype(np.float32)
    x[1] *= 1e-4
    x[2, 40] = -300.0
    x[3] = 0.0
    q, s = O.quantize_per_token_fp8(x)
    _check_fp8_quant(O, x, q, s)
    assert np.all(q[3] == 0) and s[3] == np.float32(np.float32(1e-12) / np.float32(448.0))
    # an upper bound on the scale: rows whose absmax / 448 exceeds it clamp
    ub = 0.002
    q2, s2 = O.quantize_per_token_fp8(x, scale_ub=ub)
    _check_fp8_quant(O, x, q2, s2, ub)
    assert np.any(np.abs(O.e4m3_to_f32(q2[0])) == 448.0)
    # hand-worked row: absmax 448 -> scale 1, inv 1; each value is its own
    # nearest e4m3 or a tie
    row = np.float32([[448.0, -1.0, 1.0625, 1.1875, 3.0 * 2.0 ** -10, 17.0, -0.0]])
    q3, s3 = O.quantize_per_token_fp8(row)
    assert s3.tolist() == [1.0]
    assert q3.tolist() == [[0x7E, 0xB8, 0x38, 0x3A, 0x02, 0x58, 0x80]], q3.tolist()  # 17 ties to 16


def pin_fp8_silu_quant(O) -> None:
    rng = np.random.default_rng(13)
    g = rng.standard_normal((3, 100)).astype(np.float32) * 3
    u = rng.standard_normal((3, 100)).astype(np.float32)
    q, s = O.silu_mul_quant_per_token_fp8(g, u)
    h = np.array([[O.silu(float(a)) for a in row] for row in g], np.float32) * u
    q2, s2 = O.quantize_per_token_fp8(h.astype(np.float32))
    assert np.array_equal(q, q2) and np.array_equal(s, s2)


def pin_fp8_gemm(O) -> None:
    rng = np.random.default_rng(14)
    vals = _e4m3_values()
    a = rng.integers(0, 256, (7, 300)).astype(np.uint8)
    w = rng.integers(0, 256, (5, 300)).astype(np.uint8)
    a[(a & 0x7F) == 0x7F] = 0x10  # no NaN codes
    w[(w & 0x7F) == 0x7F] = 0x22
    da = O.e4m3_to_f32(a).astype(np.float64)
    dw = O.e4m3_to_f32(w).astype(np.float64)
    del vals
    acc, _ = O.gemm_fp8(a, w)
    # every e4m3 value is a multiple of 2^-9: the float64 products and their
    # sums at this size are exact, in any order
    assert np.array_equal(acc, da @ dw.T)
    # closed form: all operands 448 -> k * 448^2
    k = 1000
    acc2, out2 = O.gemm_fp8(np.full((2, k), 0x7E, np.uint8), np.full((3, k), 0xFE, np.uint8),
                            np.float32([1.0, 0.5]), np.float32([1.0, 2.0, 0.25]), 1.0)
    assert np.all(acc2 == -k * 448.0 ** 2)
    assert out2.tolist() == [[-k * 448.0 ** 2, -2 * k * 448.0 ** 2, -k * 448.0 ** 2 / 4],
                             [-k * 448.0 ** 2 / 2, -k * 448.0 ** 2, -k * 448.0 ** 2 / 8]]


# --------------------------------------------------------------------------- asymmetric INT8
def pin_asym_quant(O) -> None:
    # range [0, 255]: scale 1, inv 1, zp -128, q = rne(x) - 128
    row = np.float32([[0.0, 1.0, 127.0, 128.0, 255.0, 2.5, 3.5, 200.4]])
    q, s, z = O.quantize_per_token_asym(row)
    assert s.tolist() == [1.0] and z.tolist() == [-128]
    assert q.tolist() == [[-128, -127, -1, 0, 127, -126, -124, 72]], q.tolist()
    # range [-255, 0]: scale 1, zp = 127, q = rne(x) + 127
    q2, s2, z2 = O.quantize_per_token_asym(np.float32([[-255.0, -100.0, 0.0, -0.5]]))
    assert s2.tolist() == [1.0] and z2.tolist() == [127]
    assert q2.tolist() == [[-128, 27, 127, 127]], q2.tolist()
    # random rows: invariants
    rng = np.random.default_rng(21)
    x = rng.standard_normal((6, 301)).astype(np.float32)
    x[1] = np.abs(x[1]) + 0.5  # all positive: lo widened to 0
    x[2] = -np.abs(x[2]) * 9   # all negative
    x[3] = 0.0
    x[4, 10] = 40.0
    q, s, z = O.quantize_per_token_asym(x)
    x64 = x.astype(np.float64)
    for r in range(x.shape[0]):
        lo = min(float(x64[r].min()), 0.0)
        hi = max(float(x64[r].max()), 0.0)
        sc = float(s[r])
        assert abs(sc * 255.0 - max(hi - lo, float(np.float32(1e-12)))) <= 255.0 * ulp32(sc)
        assert -128 <= int(z[r]) <= 127
        deq = (q[r].astype(np.float64) - float(z[r])) * sc
        assert float(np.abs(deq - x64[r]).max()) <= sc * (0.5 + 2.0 ** -12) + 1e-30
        if hi > lo:
            assert abs(int(q[r, int(np.argmin(x64[r]))]) + 128) <= 1 or lo == 0.0
            assert abs(int(q[r, int(np.argmax(x64[r]))]) - 127) <= 1 or hi == 0.0
    assert np.all(q[3] == -128) and z[3] == -128


def pin_asym_gemm(O) -> None:
    rng = np.random.default_rng(22)
    a = rng.integers(-128, 128, (6, 333)).astype(np.int8)
    zp = rng.integers(-128, 128, (6,)).astype(np.int32)
    w = rng.integers(-127, 128, (9, 333)).astype(np.int8)
    ref = (a.astype(np.int64) - zp[:, None].astype(np.int64)) @ w.astype(np.int64).T
    assert np.array_equal(O.gemm_s32_asym(a, zp, w), ref)
    assert np.array_equal(O.weight_row_sums(w), w.astype(np.int64).sum(axis=1))


def pin_static_quant(O) -> None:
    # scale 1: q = clamp(rne(x)); ties to even; saturation at +-127
    x = np.float32([[0.5, 1.5, 2.5, -0.5, -2.5, 126.6, 127.4, 300.0, -1e6, 3.49]])
    assert O.quantize_static(x, 1.0).tolist() == [[0, 2, 2, 0, -2, 127, 127, 127, -127, 3]]
    # scale 0.25: inv 4 exactly
    y = np.float32([[0.125, 0.375, -0.1, 31.75, 40.0]])
    assert O.quantize_static(y, 0.25).tolist() == [[0, 2, 0, 127, 127]]
    # random values: the round trip within half a step inside the range
    rng = np.random.default_rng(23)
    z = rng.standard_normal((4, 200)).astype(np.float32) * 3
    s = 0.02
    q = O.quantize_static(z, s)
    inside = np.abs(z.astype(np.float64) / s) <= 126.5
    err = np.abs(q.astype(np.float64) * s - z.astype(np.float64))
    assert float(err[inside].max()) <= s * (0.5 + 2.0 ** -16)
    assert np.all(np.abs(q[~inside]) == 127)


ALL_PINS = [pin_exp, pin_silu, pin_bf16_rounding, pin_quant_golden, pin_quant_invariants,
            pin_quant_bf16_path, pin_silu_quant, pin_gemm_bruteforce, pin_gemm_closed_forms,
            pin_epilogue_per_channel, pin_group, pin_epilogue_order_golden, pin_linear_golden, pin_e4m3_codec, pin_fp8_quant,
            pin_fp8_silu_quant, pin_fp8_gemm, pin_asym_quant, pin_asym_gemm, pin_static_quant]
