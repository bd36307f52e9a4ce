"""Helpers for the GPU parity tests: host<->device marshalling and the
comparison rules.

Comparison rules:
* int8 values, per-token scales and int32 accumulators: bit-exact.
* bf16 outputs: max relative error <= 1e-2 against the oracle's fp32 value,
  and max |gpu - ref| / ||ref_row||_2 <= 2e-2 (absolute error normalised by
  the L2 norm of the row's fp32 output).  The fraction of bits identical to
  the oracle's bf16 rounding is also returned (1.0 when the operation order
  matches).  A row-RMS normaliser (||ref_row||_2 / sqrt(N)) was tried and
  rejected: the exact bf16 rounding of a large element already exceeds 2e-2
  of the row RMS, so it would fail correct outputs.
"""
from __future__ import annotations

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from w8a8_int8_quantized_qk_b200 import synth  # noqa: E402

REL_TOL = 1e-2
NORM_TOL = 2e-2


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def dev(a: np.ndarray, bf16: bool = False):
    """numpy -> CUDA tensor; uint16 arrays are bf16 bit patterns when bf16."""
    if bf16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().copy()


def x_dev(x: np.ndarray):
    return dev(x, bf16=(x.dtype == np.uint16))


def assert_bits(got: np.ndarray, ref: np.ndarray, what: str):
    if got.dtype == np.float32:
        got, ref = got.view(np.uint32), ref.view(np.uint32)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{what}: {len(bad)} mismatches, first at {bad[:5].tolist()}"


def check_out(got, ref_f32: np.ndarray, ref_bf16: np.ndarray | None = None, what: str = "out"):
    """Tolerance check of a GPU output (bf16 bits or fp32) against the oracle's fp32.
    Returns the fraction of elements bit-identical to the oracle's rounding."""
    if got.dtype == np.uint16:
        g = synth.bf16_bits_to_f32(got).astype(np.float64)
    else:
        g = got.astype(np.float64)
    r = ref_f32.astype(np.float64)
    diff = np.abs(g - r)
    nz = np.abs(r) > 0
    rel = np.where(nz, diff / np.where(nz, np.abs(r), 1.0), diff)
    assert float(rel.max(initial=0.0)) <= REL_TOL, f"{what}: max rel err {rel.max()}"
    l2 = np.sqrt(np.sum(r * r, axis=1, keepdims=True))
    norm = diff / np.where(l2 > 0, l2, 1.0)
    assert float(norm.max(initial=0.0)) <= NORM_TOL, f"{what}: max norm-normalised err {norm.max()}"
    if ref_bf16 is not None and got.dtype == np.uint16:
        return float(np.mean(got == ref_bf16))
    return float(np.mean(got.view(np.uint32) == ref_f32.view(np.uint32)))
