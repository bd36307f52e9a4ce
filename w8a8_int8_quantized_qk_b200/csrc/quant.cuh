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

#include <cooperative_groups.h>

#include "qk_common.cuh"

namespace qk {
namespace quant {

namespace cg = cooperative_groups;

constexpr int kVecPerThread = 8;  // 16-byte vectors held per thread
constexpr int kMaxThreads = 512;  // threads per CTA (128 registers each)

struct Args {
  int m, k;
  const void* x;    // plain: [m, k]
  const void* up;   // silu: gate = x, up = up, row stride ld
  int64_t ld;       // row stride of x / up in elements
  int8_t* q;        // [m, k]
  float* scale;     // [m]
};

// ---------------------------------------------------------------------------
// The fixed binary32 exponential used by the fused SiLU: Cody & Waite
// argument reduction (t = n ln2 + r, ln2 as a binary32 head plus tail, both
// subtractions fused), e^r by the degree-7 Taylor polynomial in Horner form,
// scaling by 2^n through the exponent field.  t is clamped to [-87, 88] so
// 2^n stays a normal number.  Every step is an explicit round-to-nearest
// operation so the result does not depend on compiler contraction choices.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float fixed_exp(float t) {
  constexpr float kLog2e = static_cast<float>(1.4426950408889634074);
  constexpr float kLn2Hi = static_cast<float>(0.69314718055994530942);
  constexpr float kLn2Lo =
      static_cast<float>(0.69314718055994530942 - static_cast<double>(kLn2Hi));
  constexpr float kC7 = static_cast<float>(1.0 / 5040.0);
  constexpr float kC6 = static_cast<float>(1.0 / 720.0);
  constexpr float kC5 = static_cast<float>(1.0 / 120.0);
  constexpr float kC4 = static_cast<float>(1.0 / 24.0);
  constexpr float kC3 = static_cast<float>(1.0 / 6.0);
  t = fminf(fmaxf(t, -87.0f), 88.0f);
  const float n = rintf(__fmul_rn(t, kLog2e));
  float r = __fmaf_rn(-n, kLn2Hi, t);
  r = __fmaf_rn(-n, kLn2Lo, r);
  float p = kC7;
  p = __fmaf_rn(p, r, kC6);
  p = __fmaf_rn(p, r, kC5);
  p = __fmaf_rn(p, r, kC4);
  p = __fmaf_rn(p, r, kC3);
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const int e = static_cast<int>(n) + 127;
  return __fmul_rn(p, __int_as_float(e << 23));
}

// h = silu(g) * u = (g / (1 + exp(-g))) * u
__device__ __forceinline__ float silu_mul(float g, float u) {
  const float e = fixed_exp(-g);
  const float d = __fadd_rn(1.0f, e);
  return __fmul_rn(__fdiv_rn(g, d), u);
}

__device__ __forceinline__ int quant1(float x, float inv) {
  const int r = __float2int_rn(__fmul_rn(x, inv));  // round half to even
  return min(max(r, -127), 127);
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return (static_cast<uint32_t>(a) & 0xFFu) | ((static_cast<uint32_t>(b) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(c) & 0xFFu) << 16) | ((static_cast<uint32_t>(d) & 0xFFu) << 24);
}

// Elements of one 16-byte vector, widened to fp32.
template <bool BF16>
__device__ __forceinline__ void widen(const uint4& v, float (&f)[BF16 ? 8 : 4]) {
  if constexpr (BF16) {
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
  } else {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
}

template <bool BF16>
__device__ __forceinline__ void store_q(int8_t* dst, const float (&f)[BF16 ? 8 : 4], float inv) {
  if constexpr (BF16) {
    uint2 o;
    o.x = pack4(quant1(f[0], inv), quant1(f[1], inv), quant1(f[2], inv), quant1(f[3], inv));
    o.y = pack4(quant1(f[4], inv), quant1(f[5], inv), quant1(f[6], inv), quant1(f[7], inv));
    *reinterpret_cast<uint2*>(dst) = o;
  } else {
    *reinterpret_cast<uint32_t*>(dst) =
        pack4(quant1(f[0], inv), quant1(f[1], inv), quant1(f[2], inv), quant1(f[3], inv));
  }
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

__device__ __forceinline__ void scale_and_inverse(float amax, float& scale, float& inv) {
  scale = __fdiv_rn(fmaxf(amax, 1e-12f), 127.0f);
  inv = __fdiv_rn(1.0f, scale);
}

// One row per CTA (CLUSTER = false) or per cluster.  The row's 16-byte vectors
// are dealt round-robin to the row's threads; each thread holds up to
// kVecPerThread of them.  SILU: x is gate, p.up is up, h = silu(g) * u is kept
// in fp32 registers.
template <bool BF16, bool SILU, bool CLUSTER>
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
  const int stride = nranks * blockDim.x;
  const int t0 = rank * blockDim.x + threadIdx.x;
  const char* xr = static_cast<const char*>(p.x) + static_cast<int64_t>(row) * p.ld * ES;
  const char* ur = SILU ? static_cast<const char*>(p.up) + static_cast<int64_t>(row) * p.ld * ES
                        : nullptr;

  float vals[kVecPerThread][E];
  float amax = 0.0f;
  if constexpr (SILU) {
    uint4 gv[kVecPerThread], uv[kVecPerThread];
#pragma unroll
    for (int j = 0; j < kVecPerThread; ++j) {
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
    for (int j = 0; j < kVecPerThread; ++j) {
      float g[E], u[E];
      widen<BF16>(gv[j], g);
      widen<BF16>(uv[j], u);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        vals[j][e] = silu_mul(g[e], u[e]);
        amax = fmaxf(amax, fabsf(vals[j][e]));
      }
    }
  } else {
    uint4 xv[kVecPerThread];
#pragma unroll
    for (int j = 0; j < kVecPerThread; ++j) {
      const int v = t0 + j * stride;
      xv[j] = v < nvec ? ld_nc_v4(xr + static_cast<int64_t>(v) * 16) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < kVecPerThread; ++j) {
      widen<BF16>(xv[j], vals[j]);
#pragma unroll
      for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(vals[j][e]));
    }
  }
  amax = row_max<CLUSTER>(amax, red);
  float scale, inv;
  scale_and_inverse(amax, scale, inv);
  int8_t* qr = p.q + static_cast<int64_t>(row) * p.k;
#pragma unroll
  for (int j = 0; j < kVecPerThread; ++j) {
    const int v = t0 + j * stride;
    if (v < nvec) store_q<BF16>(qr + static_cast<int64_t>(v) * E, vals[j], inv);
  }
  if (t0 == 0) p.scale[row] = scale;
  if constexpr (CLUSTER) cg::this_cluster().sync();  // peers may still read red[32]
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
      for (int e = 0; e < E; ++e) f[e] = silu_mul(f[e], u[e]);
    }
#pragma unroll
    for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(f[e]));
  }
  amax = row_max<false>(amax, red);
  float scale, inv;
  scale_and_inverse(amax, scale, inv);
  int8_t* qr = p.q + static_cast<int64_t>(row) * p.k;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float f[E];
    widen<BF16>(ld_nc_v4(xr + static_cast<int64_t>(v) * 16), f);
    if constexpr (SILU) {
      float u[E];
      widen<BF16>(ld_nc_v4(ur + static_cast<int64_t>(v) * 16), u);
#pragma unroll
      for (int e = 0; e < E; ++e) f[e] = silu_mul(f[e], u[e]);
    }
    store_q<BF16>(qr + static_cast<int64_t>(v) * E, f, inv);
  }
  if (threadIdx.x == 0) p.scale[row] = scale;
}

// Launch geometry: threads per row T = ceil(nvec / 8).  A row is split over a
// cluster of CL CTAs when T exceeds one CTA (512 threads), or when there are too few rows to
// give every SM two CTAs (and each CTA keeps >= 64 threads).
struct Plan {
  int cluster;   // CTAs per row (1 = plain launch), 0 = two-pass kernel
  int threads;   // threads per CTA
};

inline Plan plan(int m, int k, bool bf16, int num_sms) {
  const int E = bf16 ? 8 : 4;
  const int nvec = k / E;
  const int T = (nvec + kVecPerThread - 1) / kVecPerThread;
  int cl = 1;
  while (cl < 8 && (T + cl - 1) / cl > kMaxThreads) cl *= 2;
  if ((T + cl - 1) / cl > kMaxThreads) return {0, 512};
  while (cl < 8 && static_cast<int64_t>(m) * cl < 2LL * num_sms && T / (2 * cl) >= 64) cl *= 2;
  int threads = (T + cl - 1) / cl;
  threads = ((threads + 31) / 32) * 32;
  return {cl, threads};
}

template <bool SILU>
inline cudaError_t launch(const Args& a, bool bf16, int num_sms, cudaStream_t stream) {
  const Plan pl = plan(a.m, a.k, bf16, num_sms);
  if (pl.cluster == 0) {
    if (bf16)
      quant_rows_twopass_kernel<true, SILU><<<a.m, pl.threads, 0, stream>>>(a);
    else
      quant_rows_twopass_kernel<false, SILU><<<a.m, pl.threads, 0, stream>>>(a);
    return cudaGetLastError();
  }
  if (pl.cluster == 1) {
    if (bf16)
      quant_rows_kernel<true, SILU, false><<<a.m, pl.threads, 0, stream>>>(a);
    else
      quant_rows_kernel<false, SILU, false><<<a.m, pl.threads, 0, stream>>>(a);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.m) * pl.cluster, 1, 1);
  cfg.blockDim = dim3(pl.threads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = pl.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (bf16) return cudaLaunchKernelEx(&cfg, quant_rows_kernel<true, SILU, true>, a);
  return cudaLaunchKernelEx(&cfg, quant_rows_kernel<false, SILU, true>, a);
}

}  // namespace quant
}  // namespace qk
