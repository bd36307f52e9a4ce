// quant.cuh -- dynamic per-token symmetric INT8 quantisation, plain and fused
// with silu(gate) * up.
//
// Method (vLLM PR "fused silu_and_mul + dynamic per-token FP8 quantization",
// Purpose / Algorithm; "write-int8-quantized-kernel", Inputs): per row,
// amax = max |x|, scale = max(amax, 1e-12) / 127, q = clamp(rne(x / scale)),
// computed through the inverse scale.  The pages' kernel runs one block per
// token in two phases and re-reads the input in phase 2.  Here a row is
// loaded ONCE with 16-byte vector loads into registers (spread over the
// threads of a CTA, or of a 2-8 CTA thread-block cluster when rows are few),
// reduced with a __shfl_xor_sync warp max, a shared-memory block max and, for
// clusters, a distributed-shared-memory exchange, and then quantised from
// registers.  Rows too long to keep on chip fall back to the two-pass form.
#pragma once

#include <atomic>

#include <cooperative_groups.h>

#include "qk_common.cuh"

namespace qk {
namespace quant {

namespace cg = cooperative_groups;

constexpr int kMaxThreads = 512;  // threads per CTA (128 registers each)

struct Args {
  int m, k;
  const void* x;    // plain: [m, k]
  const void* up;   // silu: gate = x, up = up, row stride ld
  int64_t ld;       // row stride of x / up in elements
  int8_t* q;        // [m, k]: int8 codes, or e4m3 codes when fp8
  float* scale;     // [m]
  int fp8;          // 0: int8, qmax 127; 1: float8 e4m3, qmax 448
  const float* ub;  // fp8 only, optional: upper bound of the written scale
};

// 1.5 * 2^23: adding it to |y| < 2^22 rounds y to an integer, ties to even
// (the sum lies in [2^23, 2^24), where the spacing is 1), and the low 22
// mantissa bits of the sum hold that integer offset by 2^22.  The multiply
// that produces y and the add are separate __fmul_rn / __fadd_rn intrinsics,
// which are never contracted into a fused multiply-add.
constexpr float kRoundMagic = 12582912.0f;
constexpr uint32_t kRoundMagicBits = 0x4B400000u;

// ---------------------------------------------------------------------------
// The fixed binary32 exponential used by the fused SiLU: Cody & Waite
// argument reduction (t = n ln2 + r, ln2 as a binary32 head plus tail, both
// subtractions fused), e^r by the degree-7 Taylor polynomial in Horner form,
// scaling by 2^n through the exponent field.  t is clamped to [-87, 88] so
// 2^n stays a normal number; n = rint(RN(t log2 e)) is formed with the
// round-to-integer constant above.  Every step is one IEEE round-to-nearest
// operation in the order written.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float fixed_exp(float t) {
  constexpr float kLog2e = static_cast<float>(1.4426950408889634074);
  constexpr float kLn2Hi = static_cast<float>(0.69314718055994530942);
  constexpr float kLn2Lo =
      static_cast<float>(0.69314718055994530942 - static_cast<double>(kLn2Hi));
  t = fminf(fmaxf(t, -87.0f), 88.0f);
  const float nb = __fadd_rn(__fmul_rn(t, kLog2e), kRoundMagic);
  const float n = __fsub_rn(nb, kRoundMagic);
  float r = __fmaf_rn(-n, kLn2Hi, t);
  r = __fmaf_rn(-n, kLn2Lo, r);
  float p = static_cast<float>(1.0 / 5040.0);
  p = __fmaf_rn(p, r, static_cast<float>(1.0 / 720.0));
  p = __fmaf_rn(p, r, static_cast<float>(1.0 / 120.0));
  p = __fmaf_rn(p, r, static_cast<float>(1.0 / 24.0));
  p = __fmaf_rn(p, r, static_cast<float>(1.0 / 6.0));
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  // 2^n: exponent field n + 127, with n = (bits of nb) - bits of 1.5 * 2^23
  const float two_n = __uint_as_float((__float_as_uint(nb) - kRoundMagicBits + 127u) << 23);
  return __fmul_rn(p, two_n);
}

// h = silu(g) * u = (g / (1 + exp(-g))) * u
__device__ __forceinline__ float silu_mul(float g, float u) {
  const float e = fixed_exp(-g);
  return __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, e)), u);
}

__device__ __forceinline__ uint64_t splat2(float x) {
  return pack2(__float_as_uint(x), __float_as_uint(x));
}


__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// q = RN(g / d) in both lanes, for finite g and d in [1, 2^127] (d = 1 + e,
// e >= 0, as silu forms it), by Markstein's method (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990), applied to (g/2) / (d/2).  The
// caller passes dh = d/2, whose reciprocal is normal for every d the clamp
// allows (d/2 < 2^126).  g/2 is exact except for |g| < 2^-125, where d = 2
// exactly and the rounded g/2 is itself the answer.  The steps: an
// approximate reciprocal of -dh, one Newton step, the quotient, its exact
// remainder by a fused multiply-add, and one fused correction.  Starting
// from the negative reciprocal gives every step the sign it needs, so no
// lane is negated or selected, and a zero g keeps its sign (+0 -> +0,
// -0 -> -0).
__device__ __forceinline__ uint64_t div2_rn(uint64_t g, uint64_t dh) {
  const uint64_t ngh = f32x2_mul(g, splat2(-0.5f));  // -g/2
  uint64_t y = pack2(__float_as_uint(rcp_approx(-lo_of(dh))), __float_as_uint(rcp_approx(-hi_of(dh))));
  const uint64_t e = f32x2_fma(dh, y, splat2(1.0f));  // 1 - dh/dh~
  y = f32x2_fma(y, e, y);                              // ~ -1/dh
  const uint64_t q0 = f32x2_mul(ngh, y);               // ~ (g/2) / dh
  const uint64_t rn = f32x2_fma(dh, q0, ngh);          // dh q0 - g/2, exact
  return f32x2_fma(rn, y, q0);                         // q0 - rn / dh
}

// Two silu_mul at once: the same operations in the same order, with the
// reduction, polynomial and final multiply as packed pairs (per-lane IEEE
// round-to-nearest), so each result is bit-identical to silu_mul's.  No
// packed multiply feeds a packed add (the assembler may fuse such a pair:
// packing the reduction's t * log2e + 1.5 * 2^23 that way gave 7 wrong
// results in 2^32), so the clamp and that step stay scalar; -n * ln2 is
// n * (-ln2).  The two divides are one packed Markstein division (div2_rn),
// checked against the IEEE divide for every binary32 gate value.  Its
// divisor d/2 = 0.5 + p 2^(n-1) is one packed fused multiply-add: p 2^(n-1)
// is exact, so it rounds as 1 + p 2^n does, halved.  (At n = -126 the
// exponent field of 2^(n-1) is zero and the term drops out; there 1 + e
// rounds to 1 anyway.)  mlp_down activations: 8.36 us with the IEEE
// divide, 7.5 us with a scaled division, 6.5 us in this form.
__device__ __forceinline__ void silu_mul2(float g0, float g1, float u0, float u1, float& h0,
                                          float& h1) {
  constexpr float kLog2e = static_cast<float>(1.4426950408889634074);
  constexpr float kLn2Hi = static_cast<float>(0.69314718055994530942);
  constexpr float kLn2Lo =
      static_cast<float>(0.69314718055994530942 - static_cast<double>(kLn2Hi));
  const float t0 = fminf(fmaxf(-g0, -87.0f), 88.0f);
  const float t1 = fminf(fmaxf(-g1, -87.0f), 88.0f);
  const float nb0 = __fadd_rn(__fmul_rn(t0, kLog2e), kRoundMagic);
  const float nb1 = __fadd_rn(__fmul_rn(t1, kLog2e), kRoundMagic);
  const uint64_t t = pack2(__float_as_uint(t0), __float_as_uint(t1));
  const uint64_t n =
      f32x2_add(pack2(__float_as_uint(nb0), __float_as_uint(nb1)), splat2(-kRoundMagic));
  uint64_t r = f32x2_fma(n, splat2(-kLn2Hi), t);
  r = f32x2_fma(n, splat2(-kLn2Lo), r);
  uint64_t p = f32x2_fma(splat2(static_cast<float>(1.0 / 5040.0)), r,
                         splat2(static_cast<float>(1.0 / 720.0)));
  p = f32x2_fma(p, r, splat2(static_cast<float>(1.0 / 120.0)));
  p = f32x2_fma(p, r, splat2(static_cast<float>(1.0 / 24.0)));
  p = f32x2_fma(p, r, splat2(static_cast<float>(1.0 / 6.0)));
  p = f32x2_fma(p, r, splat2(0.5f));
  p = f32x2_fma(p, r, splat2(1.0f));
  p = f32x2_fma(p, r, splat2(1.0f));
  // 2^(n-1): exponent field n + 126
  const float two0 = __uint_as_float((__float_as_uint(nb0) - kRoundMagicBits + 126u) << 23);
  const float two1 = __uint_as_float((__float_as_uint(nb1) - kRoundMagicBits + 126u) << 23);
  const uint64_t dh = f32x2_fma(p, pack2(__float_as_uint(two0), __float_as_uint(two1)), splat2(0.5f));
  const uint64_t sq = div2_rn(pack2(__float_as_uint(g0), __float_as_uint(g1)), dh);
  const uint64_t h = f32x2_mul(sq, pack2(__float_as_uint(u0), __float_as_uint(u1)));
  h0 = lo_of(h);
  h1 = hi_of(h);
}

// Quantise one value: the low byte of (x * inv + 1.5 * 2^23) is
// round_half_even(x * inv) as a two's-complement int8.  The clamp to
// [-127, 127] is never active: |x| <= amax and inv = RN(1 / RN(a / 127)) with
// a = max(amax, 1e-12) give |x * inv| <= 127 (1 + 2^-23), which rounds to at
// most 127.
// Four binary32 values -> four float8 e4m3 codes (bytes in order a..d),
// each rounded to nearest, ties to even, saturating to +-448.
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  // cvt's first source goes to the upper byte of the pair
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

__device__ __forceinline__ uint32_t quant_bits(float x, float inv) {
  return __float_as_uint(__fadd_rn(__fmul_rn(x, inv), kRoundMagic));
}

// Four quantised values (low bytes of a..d) -> one packed int8x4 word.
__device__ __forceinline__ uint32_t pack_q4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// A 16-byte vector widened to binary32 (8 values for bf16, 4 for fp32).
template <bool BF16>
__device__ __forceinline__ void widen(const uint4& v, float (&f)[BF16 ? 8 : 4]) {
  if constexpr (BF16) {
    f[0] = __uint_as_float(v.x << 16); f[1] = __uint_as_float(v.x & 0xFFFF0000u);
    f[2] = __uint_as_float(v.y << 16); f[3] = __uint_as_float(v.y & 0xFFFF0000u);
    f[4] = __uint_as_float(v.z << 16); f[5] = __uint_as_float(v.z & 0xFFFF0000u);
    f[6] = __uint_as_float(v.w << 16); f[7] = __uint_as_float(v.w & 0xFFFF0000u);
  } else {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
}


// Two binary32 values -> round_half_even(x * inv) as int32 each (x * inv
// rounded to binary32 first, on a packed pair; cvt.rni rounds half to even,
// as the 1.5 * 2^23 trick of quant_bits does, and |x * inv| <= 127 (1 +
// 2^-23) keeps both in range).  With the bytes packed by cvt.pack.sat this is
// 16 instructions per 8 values against 22 (7.67 -> 7.49 us for the SiLU
// quantiser of the mlp_down activations).
__device__ __forceinline__ void quant2(float a, float b, uint64_t inv2, int& qa, int& qb) {
  const uint64_t y = f32x2_mul(pack2(__float_as_uint(a), __float_as_uint(b)), inv2);
  asm("cvt.rni.s32.f32 %0, %1;" : "=r"(qa) : "f"(lo_of(y)));
  asm("cvt.rni.s32.f32 %0, %1;" : "=r"(qb) : "f"(hi_of(y)));
}

// Four int32 values in [-127, 127] -> int8x4 (a in the low byte).
__device__ __forceinline__ uint32_t pack_s8x4(int a, int b, int c, int d) {
  uint32_t t, r;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(t) : "r"(d), "r"(c), "r"(0));
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(b), "r"(a), "r"(t));
  return r;
}

// Quantise E values and store E int8 at dst.
template <int E>
__device__ __forceinline__ void store_q(const Args& p, int8_t* dst, const float (&f)[E], float inv) {
  if (p.fp8) {
    // e4m3: y = x * inv (fp32 RN), converted round-to-nearest-even; the
    // satfinite conversion gives +-448 for |y| beyond it, as the clamp to
    // [-448, 448] before an exact conversion does
    if constexpr (E == 8) {
      uint2 o;
      o.x = e4m3x4(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv), __fmul_rn(f[2], inv),
                   __fmul_rn(f[3], inv));
      o.y = e4m3x4(__fmul_rn(f[4], inv), __fmul_rn(f[5], inv), __fmul_rn(f[6], inv),
                   __fmul_rn(f[7], inv));
      *reinterpret_cast<uint2*>(dst) = o;
    } else {
      *reinterpret_cast<uint32_t*>(dst) = e4m3x4(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv),
                                                 __fmul_rn(f[2], inv), __fmul_rn(f[3], inv));
    }
    return;
  }
  const uint64_t inv2 = pack2(__float_as_uint(inv), __float_as_uint(inv));
  int q[E];
#pragma unroll
  for (int i = 0; i < E; i += 2) quant2(f[i], f[i + 1], inv2, q[i], q[i + 1]);
  if constexpr (E == 8) {
    uint2 o;
    o.x = pack_s8x4(q[0], q[1], q[2], q[3]);
    o.y = pack_s8x4(q[4], q[5], q[6], q[7]);
    *reinterpret_cast<uint2*>(dst) = o;
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_s8x4(q[0], q[1], q[2], q[3]);
  }
}

// Cluster barrier without memory ordering: used only to keep a CTA's shared
// memory alive until its peers have finished reading it.
__device__ __forceinline__ void cluster_arrive_wait_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// Max over the CTA (and over the cluster when CLUSTER): every thread gets it.
template <bool CLUSTER>
__device__ __forceinline__ float row_max(float v, float* red /*[33]*/) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  v = warp_max(v);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = lane < nwarps ? red[lane] : 0.0f;
  v = warp_max(v);
  if constexpr (CLUSTER) {
    cg::cluster_group cl = cg::this_cluster();
    if (threadIdx.x == 0) red[32] = v;
    cl.sync();
    float w = 0.0f;
    const unsigned n = cl.num_blocks();
    for (unsigned r = 0; r < n; ++r) w = fmaxf(w, *cl.map_shared_rank(&red[32], r));
    v = w;
  }
  return v;
}

// scale = max(amax, 1e-12) / 127 and inv = 1 / scale, both IEEE RN.
__device__ __forceinline__ void scale_and_inverse(const Args& p, float amax, float& scale,
                                                  float& inv) {
  if (p.fp8) {
    scale = __fdiv_rn(fmaxf(amax, 1e-12f), 448.0f);
    if (p.ub != nullptr) scale = fminf(scale, __ldg(p.ub));
  } else {
    scale = __fdiv_rn(fmaxf(amax, 1e-12f), 127.0f);
  }
  inv = __fdiv_rn(1.0f, scale);
}

// One row per CTA (CLUSTER = false) or per cluster.  The row's 16-byte vectors
// are dealt round-robin to the row's threads; each thread holds up to V of
// them, widened to fp32 in registers.  SILU: x is gate, p.up is up, and the
// registers hold h = silu(g) * u.
template <bool BF16, bool SILU, bool CLUSTER, int V>
__global__ void __launch_bounds__(kMaxThreads) quant_rows_kernel(Args p) {
  constexpr int E = BF16 ? 8 : 4;  // elements per 16-byte vector
  constexpr int ES = BF16 ? 2 : 4;
  __shared__ float red[33];
  int row, rank, nranks;
  if constexpr (CLUSTER) {
    cg::cluster_group cl = cg::this_cluster();
    nranks = static_cast<int>(cl.num_blocks());
    rank = static_cast<int>(cl.block_rank());
    row = blockIdx.x / nranks;
  } else {
    nranks = 1;
    rank = 0;
    row = blockIdx.x;
  }
  const int nvec = p.k / E;
  griddep_wait();  // the previous kernel in the stream is done with our buffers
  griddep_launch_dependents();
  const int stride = nranks * blockDim.x;
  const int t0 = rank * blockDim.x + threadIdx.x;
  const char* xr = static_cast<const char*>(p.x) + static_cast<int64_t>(row) * p.ld * ES;
  int8_t* qr = p.q + static_cast<int64_t>(row) * p.k;
  float vals[V][E];
  float m = 0.0f;
  if constexpr (SILU) {
    const char* ur = static_cast<const char*>(p.up) + static_cast<int64_t>(row) * p.ld * ES;
    uint4 gv[V], uv[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int v = t0 + j * stride;
      if (v < nvec) {
        gv[j] = ld_nc_v4(xr + static_cast<int64_t>(v) * 16);
        uv[j] = ld_nc_v4(ur + static_cast<int64_t>(v) * 16);
      } else {
        gv[j] = make_uint4(0, 0, 0, 0);
        uv[j] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int j = 0; j < V; ++j) {
      float g[E], u[E];
      widen<BF16>(gv[j], g);
      widen<BF16>(uv[j], u);
#pragma unroll
      for (int e = 0; e < E; e += 2) {
        silu_mul2(g[e], g[e + 1], u[e], u[e + 1], vals[j][e], vals[j][e + 1]);
        m = fmaxf(m, fabsf(vals[j][e]));
        m = fmaxf(m, fabsf(vals[j][e + 1]));
      }
    }
  } else {
    uint4 xv[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int v = t0 + j * stride;
      xv[j] = v < nvec ? ld_nc_v4(xr + static_cast<int64_t>(v) * 16) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < V; ++j) {
      widen<BF16>(xv[j], vals[j]);
#pragma unroll
      for (int e = 0; e < E; ++e) m = fmaxf(m, fabsf(vals[j][e]));
    }
  }
  const float amax = row_max<CLUSTER>(m, red);
  float scale, inv;
  scale_and_inverse(p, amax, scale, inv);
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const int v = t0 + j * stride;
    if (v < nvec) store_q<E>(p, qr + static_cast<int64_t>(v) * E, vals[j], inv);
  }
  if (t0 == 0) p.scale[row] = scale;
  if constexpr (CLUSTER) cluster_arrive_wait_relaxed();  // peers may still read red[32]
}

// Many rows: persistent CTAs of 256 threads walk rows blockIdx, blockIdx +
// grid, ...; each row's V 16-byte vectors per thread are loaded one row
// ahead, so the next row's loads are in flight while the current row is
// reduced and quantised.  The per-warp maxima are double-buffered by row
// parity: one CTA barrier per row suffices.
constexpr int kPersistThreads = 256;

template <bool BF16, bool SILU, int V>
__global__ void __launch_bounds__(kPersistThreads) quant_rows_persistent_kernel(Args p) {
  constexpr int E = BF16 ? 8 : 4;
  constexpr int ES = BF16 ? 2 : 4;
  constexpr int NW = kPersistThreads / 32;
  __shared__ float red[2][NW];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nvec = p.k / E;
  griddep_wait();  // the previous kernel in the stream is done with our buffers
  griddep_launch_dependents();
  uint4 xc[V], uc[SILU ? V : 1];
  auto fetch = [&](uint4 (&xv)[V], uint4 (&uv)[SILU ? V : 1], int row) {
    const char* xr = static_cast<const char*>(p.x) + static_cast<int64_t>(row) * p.ld * ES;
    const char* ur = SILU ? static_cast<const char*>(p.up) + static_cast<int64_t>(row) * p.ld * ES
                          : nullptr;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int v = tid + j * kPersistThreads;
      const bool in = row < p.m && v < nvec;
      xv[j] = in ? ld_nc_v4(xr + static_cast<int64_t>(v) * 16) : make_uint4(0, 0, 0, 0);
      if constexpr (SILU) uv[j] = in ? ld_nc_v4(ur + static_cast<int64_t>(v) * 16) : make_uint4(0, 0, 0, 0);
    }
  };
  fetch(xc, uc, blockIdx.x);
  int par = 0;
  for (int row = blockIdx.x; row < p.m; row += gridDim.x) {
    uint4 xn[V], un[SILU ? V : 1];
    fetch(xn, un, row + gridDim.x);
    float vals[V][E];
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      widen<BF16>(xc[j], vals[j]);
      if constexpr (SILU) {
        float u[E];
        widen<BF16>(uc[j], u);
#pragma unroll
        for (int e = 0; e < E; e += 2)
          silu_mul2(vals[j][e], vals[j][e + 1], u[e], u[e + 1], vals[j][e], vals[j][e + 1]);
      }
#pragma unroll
      for (int e = 0; e < E; ++e) m = fmaxf(m, fabsf(vals[j][e]));
    }
    m = warp_max(m);
    if (lane == 0) red[par][warp] = m;
    __syncthreads();
    float amax = lane < NW ? red[par][lane] : 0.0f;
    amax = warp_max(amax);
    float scale, inv;
    scale_and_inverse(p, amax, scale, inv);
    int8_t* qr = p.q + static_cast<int64_t>(row) * p.k;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int v = tid + j * kPersistThreads;
      if (v < nvec) store_q<E>(p, qr + static_cast<int64_t>(v) * E, vals[j], inv);
    }
    if (tid == 0) p.scale[row] = scale;
    par ^= 1;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      xc[j] = xn[j];
      if constexpr (SILU) uc[j] = un[j];
    }
  }
}

// Rows too long to hold on chip: the two-phase form (phase 1 absmax, phase 2
// re-read, recompute and quantise).  One CTA per row.
template <bool BF16, bool SILU>
__global__ void __launch_bounds__(512) quant_rows_twopass_kernel(Args p) {
  constexpr int E = BF16 ? 8 : 4;
  constexpr int ES = BF16 ? 2 : 4;
  __shared__ float red[33];
  const int row = blockIdx.x;
  const int nvec = p.k / E;
  griddep_wait();  // the previous kernel in the stream is done with our buffers
  griddep_launch_dependents();
  const char* xr = static_cast<const char*>(p.x) + static_cast<int64_t>(row) * p.ld * ES;
  const char* ur = SILU ? static_cast<const char*>(p.up) + static_cast<int64_t>(row) * p.ld * ES
                        : nullptr;
  float amax = 0.0f;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float f[E];
    widen<BF16>(ld_nc_v4(xr + static_cast<int64_t>(v) * 16), f);
    if constexpr (SILU) {
      float u[E];
      widen<BF16>(ld_nc_v4(ur + static_cast<int64_t>(v) * 16), u);
#pragma unroll
      for (int e = 0; e < E; e += 2) silu_mul2(f[e], f[e + 1], u[e], u[e + 1], f[e], f[e + 1]);
    }
#pragma unroll
    for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(f[e]));
  }
  amax = row_max<false>(amax, red);
  float scale, inv;
  scale_and_inverse(p, amax, scale, inv);
  int8_t* qr = p.q + static_cast<int64_t>(row) * p.k;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float f[E];
    widen<BF16>(ld_nc_v4(xr + static_cast<int64_t>(v) * 16), f);
    if constexpr (SILU) {
      float u[E];
      widen<BF16>(ld_nc_v4(ur + static_cast<int64_t>(v) * 16), u);
#pragma unroll
      for (int e = 0; e < E; e += 2) silu_mul2(f[e], f[e + 1], u[e], u[e + 1], f[e], f[e + 1]);
    }
    store_q<E>(p, qr + static_cast<int64_t>(v) * E, f, inv);
  }
  if (threadIdx.x == 0) p.scale[row] = scale;
}

// Launch geometry: V = 4 vectors per thread, T = ceil(nvec / V) threads per
// row.  A row is split over a cluster of CL CTAs when T exceeds one CTA (512
// threads), or when there are too few rows to fill the GPU (and each CTA
// keeps >= 64 threads): fewer than four CTAs per SM for the plain quantiser,
// fewer rows than SMs for the SiLU form, whose per-element arithmetic makes
// the cluster's extra synchronisation cost more than the parallelism gains
// once every SM has a row (measured at 256 x 14336: one CTA of 448 threads
// per row, 10.4 us, against 12.2 us for four CTAs of 112).
template <bool SILU>
constexpr int vec_per_thread() { return 4; }

struct Plan {
  int cluster;   // CTAs per row (1 = plain launch), 0 = two-pass kernel
  int threads;   // threads per CTA
};

inline Plan plan(int m, int k, bool bf16, bool silu, int V, int num_sms) {
  const int E = bf16 ? 8 : 4;
  const int nvec = k / E;
  const int T = (nvec + V - 1) / V;
  int cl = 1;
  while (cl < 8 && (T + cl - 1) / cl > kMaxThreads) cl *= 2;
  if ((T + cl - 1) / cl > kMaxThreads) return {0, 512};
  const int64_t fill = (silu ? 1LL : 4LL) * num_sms;
  while (cl < 8 && static_cast<int64_t>(m) * cl < fill && T / (2 * cl) >= 64) cl *= 2;
  int threads = (T + cl - 1) / cl;
  threads = ((threads + 31) / 32) * 32;
  return {cl, threads};
}

template <bool BF16, bool SILU, int V>
inline cudaError_t launch_rows(const Args& a, int num_sms, cudaStream_t stream);

// Persistent grid: as many CTAs per SM as can be resident at once (at most
// eight), never more -- a CTA that waits for a second wave starts its rows
// late and the whole launch waits for it (4 x 148 CTAs of the 4-vector
// kernel, of which only 3 per SM fit, took 14.0 us at 2048 x 8192; all
// resident, 12.4 us).  More resident CTAs keep more rows' loads in flight:
// at 4096 x 4096 bf16 the 2-vector kernel took 10.85 us with four per SM
// and 9.97 us with all that fit.
template <bool BF16, bool SILU, int V>
inline int persistent_ctas_per_sm() {
  static std::atomic<int> cached{0};  // (host threads may race to fill it, with one value)
  int known = cached.load(std::memory_order_relaxed);
  if (known == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, quant_rows_persistent_kernel<BF16, SILU, V>, kPersistThreads, 0) != cudaSuccess ||
        n < 1) {
      cudaGetLastError();
      n = 1;
    }
    known = n < 8 ? n : 8;
    cached.store(known, std::memory_order_relaxed);
  }
  return known;
}

template <bool BF16, bool SILU, int V>
inline cudaError_t launch_persistent(const Args& a, int num_sms, cudaStream_t stream) {
  const int cap = persistent_ctas_per_sm<BF16, SILU, V>() * num_sms;
  const int grid = a.m < cap ? a.m : cap;
  return launch_pdl(quant_rows_persistent_kernel<BF16, SILU, V>, dim3(grid), dim3(kPersistThreads),
                    0, stream, 1, a);
}

template <bool BF16, bool SILU>
inline cudaError_t launch_typed(const Args& a, int num_sms, cudaStream_t stream) {
  // Many rows of a size the persistent kernel holds (<= 4 vectors per thread):
  // persistent row loop with prefetch.
  const int E = BF16 ? 8 : 4;
  const int vp = (a.k / E + kPersistThreads - 1) / kPersistThreads;
  if (a.m >= 2 * num_sms && vp <= 4) {
    switch (vp) {
      case 1: return launch_persistent<BF16, SILU, 1>(a, num_sms, stream);
      case 2: return launch_persistent<BF16, SILU, 2>(a, num_sms, stream);
      default: return launch_persistent<BF16, SILU, 4>(a, num_sms, stream);
    }
  }
  return launch_rows<BF16, SILU, vec_per_thread<SILU>()>(a, num_sms, stream);
}

template <bool BF16, bool SILU, int V>
inline cudaError_t launch_rows(const Args& a, int num_sms, cudaStream_t stream) {
  const Plan pl = plan(a.m, a.k, BF16, SILU, V, num_sms);
  if (pl.cluster == 0) {
    return launch_pdl(quant_rows_twopass_kernel<BF16, SILU>, dim3(a.m), dim3(pl.threads), 0, stream,
                      1, a);
  }
  if (pl.cluster == 1) {
    return launch_pdl(quant_rows_kernel<BF16, SILU, false, V>, dim3(a.m), dim3(pl.threads), 0,
                      stream, 1, a);
  }
  return launch_pdl(quant_rows_kernel<BF16, SILU, true, V>,
                    dim3(static_cast<unsigned>(a.m) * pl.cluster), dim3(pl.threads), 0, stream,
                    static_cast<unsigned>(pl.cluster), a);
}

template <bool SILU>
inline cudaError_t launch(const Args& a, bool bf16, int num_sms, cudaStream_t stream) {
  return bf16 ? launch_typed<true, SILU>(a, num_sms, stream)
              : launch_typed<false, SILU>(a, num_sms, stream);
}

// ---------------------------------------------------------------------------
// Asymmetric per-token INT8 ("write-int8-quantized-kernel", Inputs:
// asymmetric quantisation maps [-128, 127] to an arbitrary range with a
// non-zero zero-point).  Per row: the range [lo, hi] is widened to hold 0;
// scale = max(hi - lo, 1e-12) / 255; inv = 1 / scale;
// zp = clamp(rint(-128 - lo * inv), -128, 127);
// q = clamp(rint(x * inv) + zp, -128, 127).  One CTA of 256 threads per row,
// two passes over the row (the second from L2); every step one IEEE
// round-to-nearest binary32 operation.
// ---------------------------------------------------------------------------
struct AsymArgs {
  int m, k;
  const void* x;  // [m, k]
  int8_t* q;      // [m, k]
  float* scale;   // [m]
  int32_t* zp;    // [m]
};

constexpr int kAsymThreads = 256;

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// low byte of the int8 value r (an integer-valued float in [-128, 127])
__device__ __forceinline__ uint32_t asym_byte(float x, float inv, float z) {
  float r = __fadd_rn(rintf(__fmul_rn(x, inv)), z);
  r = fminf(fmaxf(r, -128.0f), 127.0f);
  return static_cast<uint32_t>(static_cast<int>(r)) & 0xFFu;
}

template <bool BF16>
__global__ void __launch_bounds__(kAsymThreads) quant_asym_kernel(AsymArgs p) {
  constexpr int E = BF16 ? 8 : 4;
  constexpr int ES = BF16 ? 2 : 4;
  __shared__ float rlo[kAsymThreads / 32], rhi[kAsymThreads / 32];
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  griddep_wait();
  griddep_launch_dependents();
  const char* xr = static_cast<const char*>(p.x) + static_cast<int64_t>(row) * p.k * ES;
  const int nvec = p.k / E;
  float lo = 0.0f, hi = 0.0f;
  for (int v = tid; v < nvec; v += kAsymThreads) {
    float f[E];
    widen<BF16>(ld_nc_v4(xr + static_cast<int64_t>(v) * 16), f);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      lo = fminf(lo, f[e]);
      hi = fmaxf(hi, f[e]);
    }
  }
  lo = warp_min(lo);
  hi = warp_max(hi);
  if (lane == 0) {
    rlo[warp] = lo;
    rhi[warp] = hi;
  }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kAsymThreads / 32; ++w) {
    lo = fminf(lo, rlo[w]);
    hi = fmaxf(hi, rhi[w]);
  }
  const float sc = __fdiv_rn(fmaxf(__fsub_rn(hi, lo), 1e-12f), 255.0f);
  const float inv = __fdiv_rn(1.0f, sc);
  const float z = fminf(fmaxf(rintf(__fsub_rn(-128.0f, __fmul_rn(lo, inv))), -128.0f), 127.0f);
  int8_t* qr = p.q + static_cast<int64_t>(row) * p.k;
  for (int v = tid; v < nvec; v += kAsymThreads) {
    float f[E];
    widen<BF16>(ld_nc_v4(xr + static_cast<int64_t>(v) * 16), f);
    uint32_t w[E / 4];
#pragma unroll
    for (int j = 0; j < E / 4; ++j)
      w[j] = asym_byte(f[4 * j], inv, z) | (asym_byte(f[4 * j + 1], inv, z) << 8) |
             (asym_byte(f[4 * j + 2], inv, z) << 16) | (asym_byte(f[4 * j + 3], inv, z) << 24);
    if constexpr (E == 8)
      *reinterpret_cast<uint2*>(qr + static_cast<int64_t>(v) * E) = make_uint2(w[0], w[1]);
    else
      *reinterpret_cast<uint32_t*>(qr + static_cast<int64_t>(v) * E) = w[0];
  }
  if (tid == 0) {
    p.scale[row] = sc;
    p.zp[row] = static_cast<int32_t>(z);
  }
}

inline cudaError_t launch_asym(const AsymArgs& a, bool bf16, cudaStream_t stream) {
  return bf16 ? launch_pdl(quant_asym_kernel<true>, dim3(a.m), dim3(kAsymThreads), 0, stream, 1, a)
              : launch_pdl(quant_asym_kernel<false>, dim3(a.m), dim3(kAsymThreads), 0, stream, 1, a);
}

// ---------------------------------------------------------------------------
// Static per-tensor INT8 ("write-int8-quantized-kernel", Inputs: per-tensor
// granularity, scales computed offline): inv = 1 / scale (scale read from
// device memory), q = clamp(rint(x * inv), -127, 127).  Elementwise:
// persistent grid-stride over the tensor's 16-byte vectors.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t static_byte(float x, float inv) {
  const float r = fminf(fmaxf(rintf(__fmul_rn(x, inv)), -127.0f), 127.0f);
  return static_cast<uint32_t>(static_cast<int>(r)) & 0xFFu;
}

template <bool BF16>
__global__ void __launch_bounds__(256) quant_static_kernel(int64_t nvec, const void* x,
                                                           const float* scale, int8_t* q) {
  constexpr int E = BF16 ? 8 : 4;
  griddep_wait();
  griddep_launch_dependents();
  const float inv = __fdiv_rn(1.0f, __ldg(scale));
  const char* xb = static_cast<const char*>(x);
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < nvec;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float f[E];
    widen<BF16>(ld_nc_v4(xb + v * 16), f);
    uint32_t w[E / 4];
#pragma unroll
    for (int j = 0; j < E / 4; ++j)
      w[j] = static_byte(f[4 * j], inv) | (static_byte(f[4 * j + 1], inv) << 8) |
             (static_byte(f[4 * j + 2], inv) << 16) | (static_byte(f[4 * j + 3], inv) << 24);
    if constexpr (E == 8)
      *reinterpret_cast<uint2*>(q + v * E) = make_uint2(w[0], w[1]);
    else
      *reinterpret_cast<uint32_t*>(q + v * E) = w[0];
  }
}

inline cudaError_t launch_static(int64_t count, const void* x, bool bf16, const float* scale,
                                 int8_t* q, int num_sms, cudaStream_t stream) {
  const int64_t nvec = count / (bf16 ? 8 : 4);
  int64_t blocks = (nvec + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return bf16 ? launch_pdl(quant_static_kernel<true>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                           stream, 1, nvec, x, scale, q)
              : launch_pdl(quant_static_kernel<false>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                           stream, 1, nvec, x, scale, q);
}

// wsum[r] = sum_k w[r][k] for the zero-point correction: one warp per row,
// 16-byte loads, dp4a against bytes of 1 (exact int32 sums).
__global__ void __launch_bounds__(256) weight_row_sums_kernel(int n, int k, const int8_t* w,
                                                              int32_t* wsum) {
  griddep_wait();
  griddep_launch_dependents();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= n) return;
  const char* wr = reinterpret_cast<const char*>(w) + static_cast<int64_t>(row) * k;
  int acc = 0;
  for (int v = lane; v < k / 16; v += 32) {
    const uint4 x = ld_nc_v4(wr + static_cast<int64_t>(v) * 16);
    acc = __dp4a(static_cast<int>(x.x), 0x01010101, acc);
    acc = __dp4a(static_cast<int>(x.y), 0x01010101, acc);
    acc = __dp4a(static_cast<int>(x.z), 0x01010101, acc);
    acc = __dp4a(static_cast<int>(x.w), 0x01010101, acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if (lane == 0) wsum[row] = acc;
}

inline cudaError_t launch_weight_row_sums(int n, int k, const int8_t* w, int32_t* wsum,
                                          cudaStream_t stream) {
  return launch_pdl(weight_row_sums_kernel, dim3((n + 7) / 8), dim3(256), 0, stream, 1, n, k, w,
                    wsum);
}

}  // namespace quant
}  // namespace qk
