"""Seeded synthetic inputs for the W8A8 linear layer.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no quantisation, no GEMM, no epilogue).  Tests feed the
same arrays to the CPU oracle and to the CUDA library, and the benchmark uses
them as its workload.

Generator: numpy ``Generator(PCG64(SeedSequence(seed)))``; one child stream is
spawned per tensor, in the order the recipe lists the tensors, so adding a
tensor never shifts the draws of another.  bf16 inputs are drawn in float32 and
rounded to bf16 by torch's CPU cast (round to nearest even); they are returned
as their uint16 bit patterns.

Workloads (the pages' shapes; the distributions are stated with each recipe):

* ``tiny``     -- X fp32 [16, 512] ~ N(0, 1); W fp32 [256, 512] ~ N(0, 0.02),
  quantised per output channel before use; fp32 output.
* ``decode``   -- X bf16 [4, 4096] ~ N(0, 1) with 1 % of the K channels scaled
  x20 (outlier channels); W int8 [14336, 4096] uniform on {-127..127};
  per-channel scales U(0.001, 0.01); bf16 output.
* ``prefill``  -- X bf16 [4096, 4096] ~ N(0, 1) with 0.5 % outlier channels
  x30; W int8 [4096, 4096] uniform on {-127..127}; scales U(0.001, 0.01).
* ``mlp_down`` -- gate, up bf16 [256, 14336] ~ N(0, 1); W int8
  [4096, 14336]; per-channel scales U(0.001, 0.01).
* ``group``    -- X bf16 [2048, 8192] ~ N(0, 1); W int8 [8192, 8192];
  scales U(0.001, 0.01) per output channel per 128-wide K group.

Outlier channels are ``round(p * K)`` distinct columns chosen without
replacement; they are multiplied by the factor before the bf16 rounding.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# Names, in order, of the five workloads; workload i draws from seed i.
WORKLOADS = ("tiny", "decode", "prefill", "mlp_down", "group")


@dataclass
class Workload:
    """One synthetic linear-layer problem.

    ``x`` is the activation ([m, k] float32 or bf16 bits), or None for the
    fused SiLU workload, which has ``gate`` and ``up`` instead.  ``w_q`` is the
    int8 weight [n, k] (None when ``w_f32`` must first be quantised per output
    channel), ``sw`` the weight scales ([n] or [n, k // group_k]).
    """

    name: str
    m: int
    n: int
    k: int
    x_dtype: str  # "f32" or "bf16"
    out_dtype: str  # "f32" or "bf16"
    group_k: int = 0
    x: np.ndarray | None = None
    gate: np.ndarray | None = None
    up: np.ndarray | None = None
    w_f32: np.ndarray | None = None
    w_q: np.ndarray | None = None
    sw: np.ndarray | None = None
    alpha: float = 1.0
    meta: dict = field(default_factory=dict)


def streams(seed: int, names: list[str]) -> dict[str, np.random.Generator]:
    """One independent PCG64 stream per name, spawned from ``SeedSequence(seed)``."""
    children = np.random.SeedSequence(seed).spawn(len(names))
    return {n: np.random.Generator(np.random.PCG64(c)) for n, c in zip(names, children)}


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (torch CPU cast, nearest-even); uint16 bits."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def outlier_columns(rng: np.random.Generator, k: int, frac: float) -> np.ndarray:
    cnt = int(round(frac * k))
    return np.sort(rng.choice(k, size=cnt, replace=False)) if cnt else np.zeros(0, np.int64)


def int8_uniform(rng: np.random.Generator, shape) -> np.ndarray:
    """Integers uniform on {-127, ..., 127} (both ends included)."""
    return rng.integers(-127, 128, size=shape, dtype=np.int8)


def e4m3_codes(rng: np.random.Generator, shape) -> np.ndarray:
    """Float8 e4m3 codes drawn uniformly from the 254 finite ones (the two NaN
    codes 0x7F and 0xFF excluded); one byte each."""
    c = rng.integers(0, 254, size=shape, dtype=np.int64)
    c = np.where(c >= 0x7F, c + 1, c)  # skip 0x7F
    return c.astype(np.uint8)


def scales_uniform(rng: np.random.Generator, shape, lo: float = 0.001, hi: float = 0.01):
    return rng.uniform(lo, hi, size=shape).astype(np.float32)


def activation(rng_x, rng_o, m: int, k: int, dtype: str, outlier_frac: float = 0.0,
               outlier_scale: float = 1.0) -> tuple[np.ndarray, np.ndarray]:
    x = normal(rng_x, (m, k))
    cols = outlier_columns(rng_o, k, outlier_frac) if outlier_frac > 0 else np.zeros(0, np.int64)
    if cols.size:
        x[:, cols] *= np.float32(outlier_scale)
    return (to_bf16_bits(x) if dtype == "bf16" else x), cols


def make(name: str, seed: int | None = None) -> Workload:
    """Build workload ``name`` (see the module docstring) with its default seed."""
    idx = WORKLOADS.index(name)
    seed = idx if seed is None else seed
    if name == "tiny":
        r = streams(seed, ["x", "w"])
        return Workload("tiny", 16, 256, 512, "f32", "f32",
                        x=normal(r["x"], (16, 512)), w_f32=normal(r["w"], (256, 512), 0.02))
    if name == "decode":
        r = streams(seed, ["x", "outliers", "w", "sw"])
        x, cols = activation(r["x"], r["outliers"], 4, 4096, "bf16", 0.01, 20.0)
        return Workload("decode", 4, 14336, 4096, "bf16", "bf16", x=x,
                        w_q=int8_uniform(r["w"], (14336, 4096)),
                        sw=scales_uniform(r["sw"], (14336,)), meta={"outlier_cols": cols})
    if name == "prefill":
        r = streams(seed, ["x", "outliers", "w", "sw"])
        x, cols = activation(r["x"], r["outliers"], 4096, 4096, "bf16", 0.005, 30.0)
        return Workload("prefill", 4096, 4096, 4096, "bf16", "bf16", x=x,
                        w_q=int8_uniform(r["w"], (4096, 4096)),
                        sw=scales_uniform(r["sw"], (4096,)), meta={"outlier_cols": cols})
    if name == "mlp_down":
        r = streams(seed, ["gate", "up", "w", "sw"])
        return Workload("mlp_down", 256, 4096, 14336, "bf16", "bf16",
                        gate=to_bf16_bits(normal(r["gate"], (256, 14336))),
                        up=to_bf16_bits(normal(r["up"], (256, 14336))),
                        w_q=int8_uniform(r["w"], (4096, 14336)),
                        sw=scales_uniform(r["sw"], (4096,)))
    if name == "group":
        r = streams(seed, ["x", "w", "sw"])
        return Workload("group", 2048, 8192, 8192, "bf16", "bf16", group_k=128,
                        x=to_bf16_bits(normal(r["x"], (2048, 8192))),
                        w_q=int8_uniform(r["w"], (8192, 8192)),
                        sw=scales_uniform(r["sw"], (8192, 64)))
    raise KeyError(name)


def make_linear(m: int, n: int, k: int, seed: int, x_dtype: str = "bf16", group_k: int = 0,
                outlier_frac: float = 0.0, outlier_scale: float = 1.0) -> Workload:
    """A small problem of the same recipe at an arbitrary shape (parity tests)."""
    r = streams(seed, ["x", "outliers", "w", "sw"])
    x, cols = activation(r["x"], r["outliers"], m, k, x_dtype, outlier_frac, outlier_scale)
    sw_shape = (n, k // group_k) if group_k else (n,)
    return Workload(f"linear_{m}x{n}x{k}", m, n, k, x_dtype, "bf16", group_k=group_k, x=x,
                    w_q=int8_uniform(r["w"], (n, k)), sw=scales_uniform(r["sw"], sw_shape),
                    meta={"outlier_cols": cols})


def make_silu(m: int, k: int, seed: int, dtype: str = "bf16") -> tuple[np.ndarray, np.ndarray]:
    """gate, up [m, k] ~ N(0, 1) (bf16 bits or float32)."""
    r = streams(seed, ["gate", "up"])
    g, u = normal(r["gate"], (m, k)), normal(r["up"], (m, k))
    if dtype == "bf16":
        return to_bf16_bits(g), to_bf16_bits(u)
    return g, u
