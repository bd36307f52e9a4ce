// gemv.cuh -- small-M (decode) W8A8 GEMM: weight streaming on CUDA cores.
//
// With a handful of tokens the layer is a weight stream: every byte of W is
// used for M multiply-adds only ("dynquant-kernels" page, What is in here:
// the decode GEMV is the memory-bound case; "KV-cache kernels" section 01:
// INT8 moves the memory-bound ceiling).  The design goal is HBM rate:
//  - a CTA owns R consecutive rows of W and sweeps K with all its threads,
//    so every thread has R independent 16-byte streaming loads in flight
//    and the activation chunk it loads is reused R times;
//  - the int8 dot products use dp4a (4 MACs per instruction, int32
//    accumulation, exact);
//  - per-(row, token) sums are reduced with warp redux and shared memory,
//    and the dequant epilogue is applied by one thread per output.
#pragma once

#include "qk_common.cuh"

namespace qk {
namespace gemv {

constexpr int kThreads = 256;
constexpr int kRows = 8;  // rows of W per CTA

struct Args {
  int m, n, k;
  const int8_t* a;  // [m, k]
  const int8_t* w;  // [n, k]
  const float* sa;  // [m]
  const float* sw;  // [n]
  float alpha;
  int32_t* c;       // [m, n] or null
  void* out;        // [m, n] or null
  int out_bf16;
};

__device__ __forceinline__ int dot16(const uint4& w, const uint4& a, int acc) {
  acc = __dp4a(static_cast<int>(w.x), static_cast<int>(a.x), acc);
  acc = __dp4a(static_cast<int>(w.y), static_cast<int>(a.y), acc);
  acc = __dp4a(static_cast<int>(w.z), static_cast<int>(a.z), acc);
  acc = __dp4a(static_cast<int>(w.w), static_cast<int>(a.w), acc);
  return acc;
}

// MT: compile-time token capacity (m <= MT).
template <int MT>
__global__ void __launch_bounds__(kThreads) gemv_i8_kernel(Args p) {
  __shared__ int red[kThreads / 32][kRows * MT];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nchunk = p.k >> 4;  // 16-byte chunks per row
  const int ngroups = (p.n + kRows - 1) / kRows;
  for (int grp = blockIdx.x; grp < ngroups; grp += gridDim.x) {
    const int row0 = grp * kRows;
    int acc[kRows][MT];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
      for (int t = 0; t < MT; ++t) acc[r][t] = 0;

    for (int ch = threadIdx.x; ch < nchunk; ch += kThreads) {
      uint4 wv[kRows];
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const int row = row0 + r;
        wv[r] = row < p.n ? ld_stream_v4(p.w + static_cast<int64_t>(row) * p.k + ch * 16)
                          : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        if (t < p.m) {
          const uint4 av = ld_nc_v4(p.a + static_cast<int64_t>(t) * p.k + ch * 16);
#pragma unroll
          for (int r = 0; r < kRows; ++r) acc[r][t] = dot16(wv[r], av, acc[r][t]);
        }
      }
    }
    // Reduce every (row, token) sum over the CTA.
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int s = __reduce_add_sync(0xFFFFFFFFu, acc[r][t]);
        if (lane == 0) red[warp][r * MT + t] = s;
      }
    __syncthreads();
    if (threadIdx.x < kRows * MT) {
      const int r = threadIdx.x / MT, t = threadIdx.x % MT;
      const int row = row0 + r;
      if (row < p.n && t < p.m) {
        int s = 0;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) s += red[w][threadIdx.x];
        const int64_t o = static_cast<int64_t>(t) * p.n + row;
        if (p.c) p.c[o] = s;
        if (p.out) {
          float v = __int2float_rn(s);
          v = __fmul_rn(v, p.sa[t]);
          v = __fmul_rn(v, p.sw[row]);
          v = __fmul_rn(v, p.alpha);
          if (p.out_bf16)
            static_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(v);
          else
            static_cast<float*>(p.out)[o] = v;
        }
      }
    }
    __syncthreads();
  }
}

inline int max_tokens() { return 8; }

inline cudaError_t launch(const Args& a, int num_sms, cudaStream_t stream) {
  const int ngroups = (a.n + kRows - 1) / kRows;
  const int grid = ngroups < 64 * num_sms ? ngroups : 64 * num_sms;
  if (a.m <= 1)
    gemv_i8_kernel<1><<<grid, kThreads, 0, stream>>>(a);
  else if (a.m <= 2)
    gemv_i8_kernel<2><<<grid, kThreads, 0, stream>>>(a);
  else if (a.m <= 4)
    gemv_i8_kernel<4><<<grid, kThreads, 0, stream>>>(a);
  else
    gemv_i8_kernel<8><<<grid, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace gemv
}  // namespace qk
