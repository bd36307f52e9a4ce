// gemv.cuh -- small-M (decode) W8A8 GEMM: weight streaming on CUDA cores.
//
// With a handful of tokens the layer is a weight stream: every byte of W is
// used for M multiply-adds only ("dynquant-kernels" page, What is in here:
// the decode GEMV is the memory-bound case; "KV-cache kernels" section 01:
// INT8 moves the memory-bound ceiling).  The design goal is HBM rate:
//  - a CTA owns groups of R consecutive rows of W and sweeps K with all its
//    threads, so every thread has R independent 16-byte streaming loads in
//    flight per group (two groups deep) and reuses each activation chunk R
//    times;
//  - the int8 dot products use dp4a (4 MACs per instruction, int32
//    accumulation, exact);
//  - per-(row, token) sums are reduced with warp redux and shared memory,
//    and the dequant epilogue is applied by one thread per output.
#pragma once

#include "qk_common.cuh"
#include "quant.cuh"

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
  // asymmetric activations: zp [m] zero-points and wsum [n] = sum_k w[n][k];
  // the epilogue uses acc - zp[t] * wsum[row] (null: symmetric)
  const int32_t* zp;
  const int32_t* wsum;
};

// acc - zp * wsum in two's-complement arithmetic (exact when the corrected
// sum fits in int32, which the host's bound on k guarantees)
__device__ __forceinline__ int zp_correct(const Args& p, int acc, int t, int row) {
  if (p.zp == nullptr) return acc;
  return static_cast<int>(static_cast<uint32_t>(acc) -
                          static_cast<uint32_t>(p.zp[t]) * static_cast<uint32_t>(p.wsum[row]));
}

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
  griddep_wait();  // the previous kernel in the stream is done with our buffers
  griddep_launch_dependents();

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
        s = zp_correct(p, s, t, row);
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

// ---------------------------------------------------------------------------
// Persistent prefetching form (the default for K <= 16384): a few CTAs per
// SM (PrefCfg), each walking row groups g = blockIdx, blockIdx + grid, ...
// A group is R rows; thread t owns the 16-byte K chunks t, t + 256, ... (J of
// them), so its activation chunks for all tokens are loaded once and stay in
// registers.  D groups of W chunks are held in registers: as soon as a
// group's dot products are done its registers are refilled with the group D
// ahead, so those loads are in flight while the current group is reduced
// (and, for D = 2, while the next one is multiplied).  (Streaming W through
// shared memory with one-dimensional bulk copies was measured and rejected:
// on this part its throughput grows with the copy size and stays far below
// the register path.)
// ---------------------------------------------------------------------------
constexpr int kPrefThreads = 256;
constexpr int kPrefDepth = 2;

// Rows per group for <MT tokens, J chunks per thread>: as many as the
// 128-register budget of two resident CTAs per SM allows (two groups of W
// chunks, R x MT accumulators and MT x J activation chunks per thread).
__host__ __device__ constexpr int pref_rows(int mt, int j) {
  return mt <= 2 ? 8 / j
                 : (mt == 4 ? (j == 1 ? 8 : (j == 2 ? 4 : (j == 3 ? 2 : 1)))
                            : (j == 1 ? 4 : (j == 2 ? 2 : 1)));
}

// Launch shape per <MT, J>: rows per group R, groups of W chunks in flight D,
// resident CTAs per SM (the register budget is 65536 / (256 x minb)).  For
// rows of up to 4096 bytes (J = 1) and up to 4 tokens, more resident CTAs of
// smaller groups keep more warps issuing loads: 5 CTAs of 3-row groups (48
// registers) read a 4 x 14336 x 4096 weight stream in 13.0 us where 2 CTAs of
// 8-row groups, two groups deep, took 16.5 us (same launch method).
template <int MT, int J>
struct PrefCfg {
  static constexpr bool narrow = J == 1 && MT <= 4;
  static constexpr int rows = narrow ? 3 : pref_rows(MT, J);
  static constexpr int depth = narrow ? 1 : kPrefDepth;
  static constexpr int minb = narrow ? 5 : 2;
};

// The activation chunks of all tokens stay in registers: MT x J <= 16.
inline bool pref_supported(int m, int k) {
  const int j = (k / 16 + kPrefThreads - 1) / kPrefThreads;
  const int mt = m <= 1 ? 1 : (m <= 2 ? 2 : (m <= 4 ? 4 : 8));
  return k <= 16384 && mt * j <= 16;
}

template <int MT, int J>
__global__ void __launch_bounds__(kPrefThreads, PrefCfg<MT, J>::minb)
    gemv_i8_prefetch_kernel(Args p) {
  constexpr int R = PrefCfg<MT, J>::rows;
  constexpr int D = PrefCfg<MT, J>::depth;
  __shared__ int red[kPrefThreads / 32][R * MT];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cpr = p.k >> 4;
  const int ngroups = (p.n + R - 1) / R;
  // (Requesting the first weight groups before this wait was measured slower:
  // 13.6 against 13.0 us per decode step.  The weight loads then queue in
  // DRAM ahead of the quantiser's, which is on the critical path.)
  griddep_wait();  // the previous kernel in the stream is done with our buffers
  griddep_launch_dependents();

  // the first groups of the weight stream are requested before the
  // activations are read, so DRAM starts at once
  uint4 buf[D][R][J];
  auto fetch = [&](uint4 (&b)[R][J], int g) {
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int j = 0; j < J; ++j) {
        const int row = g * R + r;
        const int kc = tid + j * kPrefThreads;
        b[r][j] = (g < ngroups && row < p.n && kc < cpr)
                      ? ld_stream_v4(p.w + static_cast<int64_t>(row) * p.k + kc * 16)
                      : make_uint4(0, 0, 0, 0);
      }
  };
#pragma unroll
  for (int d = 0; d < D; ++d) fetch(buf[d], blockIdx.x + d * gridDim.x);
  uint4 av[MT][J];
#pragma unroll
  for (int t = 0; t < MT; ++t)
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int kc = tid + j * kPrefThreads;
      av[t][j] = (t < p.m && kc < cpr) ? ld_nc_v4(p.a + static_cast<int64_t>(t) * p.k + kc * 16)
                                       : make_uint4(0, 0, 0, 0);
    }

  const int my_r = tid / MT, my_t = tid % MT;  // output owned by thread tid < R * MT
  const float my_sa = (tid < R * MT && my_t < p.m && p.out) ? __ldg(p.sa + my_t) : 0.0f;
  int slot = 0;
  for (int g = blockIdx.x; g < ngroups; g += gridDim.x) {
    const int my_row = g * R + my_r;
    const float my_sw = (tid < R * MT && my_row < p.n && p.out) ? __ldg(p.sw + my_row) : 0.0f;
    int acc[R][MT];
#pragma unroll
    for (int d = 0; d < D; ++d) {
      if (d == slot) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            int a = 0;
#pragma unroll
            for (int j = 0; j < J; ++j) a = dot16(buf[d][r][j], av[t][j], a);
            acc[r][t] = a;
          }
        fetch(buf[d], g + D * gridDim.x);
      }
    }
    slot = slot + 1 == D ? 0 : slot + 1;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int v = __reduce_add_sync(0xFFFFFFFFu, acc[r][t]);
        if (lane == 0) red[warp][r * MT + t] = v;
      }
    __syncthreads();
    if (tid < R * MT && my_row < p.n && my_t < p.m) {
      int sum = 0;
#pragma unroll
      for (int w = 0; w < kPrefThreads / 32; ++w) sum += red[w][tid];
      sum = zp_correct(p, sum, my_t, my_row);
      const int64_t o = static_cast<int64_t>(my_t) * p.n + my_row;
      if (p.c) p.c[o] = sum;
      if (p.out) {
        float v = __int2float_rn(sum);
        v = __fmul_rn(v, my_sa);
        v = __fmul_rn(v, my_sw);
        v = __fmul_rn(v, p.alpha);
        if (p.out_bf16)
          static_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(v);
        else
          static_cast<float*>(p.out)[o] = v;
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// The decode linear layer in one launch ("dynquant-kernels" 0.2.0, What is in
// here: the decode GEMV as the memory-bound serving case; "KV-cache kernels"
// section 04: the same fusion instincts carried to this part).  CTAs
// 0 .. m-1 each quantise one token (the per-token rule of the quantisers:
// absmax, scale = max(absmax, 1e-12) / 127, inverse, round half to even)
// into q and sa and counts it in a flag word; the other CTAs run the GEMV
// of gemv_i8_prefetch_kernel: they request their first weight groups at
// once, so DRAM streams weights while the tokens are being quantised, and
// wait (bounded) for the count to reach m only before they read the
// activations.  The grid never exceeds the CTAs the device holds at once,
// so every quantising CTA runs while the GEMV CTAs wait.  The flag words live
// in the caller's workspace: zero before the call, and zeroed again by the
// GEMV CTA that is the last to have read the tokens.
//
// Measured at 4 x 14336 x 4096 on a B200, as CUDA graphs of back-to-back
// calls: 14.9 us against 13.0 us for the quantiser and GEMV as two kernels
// overlapped by programmatic dependent launch.  The weight requests queue in
// DRAM ahead of the tokens' own loads, and the GEMV CTAs hold only a few
// groups in flight while they wait for the tokens.  (Variants measured and
// not kept: prefetching every later weight group into L2 while waiting,
// 16.2 us; holding the weight stream until the quantising CTAs have their
// rows, 16.6 us.)  One launch instead of two still saves the host a launch
// per layer, which matters when decode steps are launched eagerly.
// ---------------------------------------------------------------------------
struct FusedArgs {
  Args g;          // the GEMV; g.a and g.sa point into the workspace (q, sa)
  const void* x;   // [m, k] activations, bf16 or fp32
  int* flags;      // [0]: tokens quantised; [1]: GEMV CTAs done reading them
  int gemv_ctas;   // CTAs of the grid past the m quantising ones
};



// One token row: two passes over x (the second from L1 / L2), 256 threads.
template <bool BF16>
__device__ void fused_quantise_row(const FusedArgs& p, int row) {
  constexpr int E = BF16 ? 8 : 4;
  constexpr int ES = BF16 ? 2 : 4;
  __shared__ float red[kPrefThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nvec = p.g.k / E;
  const char* xr = static_cast<const char*>(p.x) + static_cast<int64_t>(row) * p.g.k * ES;
  float m = 0.0f;
  for (int v = tid; v < nvec; v += kPrefThreads) {
    float f[E];
    quant::widen<BF16>(ld_nc_v4(xr + static_cast<int64_t>(v) * 16), f);
#pragma unroll
    for (int e = 0; e < E; ++e) m = fmaxf(m, fabsf(f[e]));
  }
  m = quant::warp_max(m);
  if (lane == 0) red[warp] = m;
  __syncthreads();
  float amax = lane < kPrefThreads / 32 ? red[lane] : 0.0f;
  amax = quant::warp_max(amax);
  const float scale = __fdiv_rn(fmaxf(amax, 1e-12f), 127.0f);
  const float inv = __fdiv_rn(1.0f, scale);
  int8_t* qr = const_cast<int8_t*>(p.g.a) + static_cast<int64_t>(row) * p.g.k;
  for (int v = tid; v < nvec; v += kPrefThreads) {
    float f[E];
    quant::widen<BF16>(ld_nc_v4(xr + static_cast<int64_t>(v) * 16), f);
    if constexpr (E == 8) {
      uint2 o;
      o.x = quant::pack_q4(quant::quant_bits(f[0], inv), quant::quant_bits(f[1], inv),
                           quant::quant_bits(f[2], inv), quant::quant_bits(f[3], inv));
      o.y = quant::pack_q4(quant::quant_bits(f[4], inv), quant::quant_bits(f[5], inv),
                           quant::quant_bits(f[6], inv), quant::quant_bits(f[7], inv));
      *reinterpret_cast<uint2*>(qr + static_cast<int64_t>(v) * E) = o;
    } else {
      *reinterpret_cast<uint32_t*>(qr + static_cast<int64_t>(v) * E) =
          quant::pack_q4(quant::quant_bits(f[0], inv), quant::quant_bits(f[1], inv),
                         quant::quant_bits(f[2], inv), quant::quant_bits(f[3], inv));
    }
  }
  if (tid == 0) const_cast<float*>(p.g.sa)[row] = scale;
  __syncthreads();  // every store of this row issued
  if (tid == 0) {
    __threadfence();  // ... and visible device-wide before the count
    atomicAdd(p.flags, 1);
  }
}

// Wait (bounded, like every wait of the library) until *count >= target,
// polling with short sleeps.
__device__ __forceinline__ bool count_wait(const int* count, int target) {
  const volatile int* c = count;
  if (*c >= target) return true;
  const uint64_t t0 = cycles_now();
  while (true) {
    __nanosleep(32);
    if (*c >= target) return true;
    if (cycles_now() - t0 > kWaitLimitNs * kCyclesPerNs) {
      record_status(QK_ERR_TIMEOUT);
      return false;
    }
  }
}

template <int MT, int J, bool BF16>
__global__ void __launch_bounds__(kPrefThreads, PrefCfg<MT, J>::minb)
    gemv_i8_fused_kernel(FusedArgs fa) {
  constexpr int R = PrefCfg<MT, J>::rows;
  constexpr int D = PrefCfg<MT, J>::depth;
  __shared__ int red[kPrefThreads / 32][R * MT];
  __shared__ int ready;
  const Args& p = fa.g;
  griddep_wait();  // the previous kernel in the stream is done with our buffers
  griddep_launch_dependents();
  if (static_cast<int>(blockIdx.x) < p.m) {
    fused_quantise_row<BF16>(fa, blockIdx.x);
    return;
  }
  const int cta = static_cast<int>(blockIdx.x) - p.m, nctas = fa.gemv_ctas;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cpr = p.k >> 4;
  const int ngroups = (p.n + R - 1) / R;

  // the weight stream starts before the tokens are ready
  uint4 buf[D][R][J];
  auto fetch = [&](uint4 (&b)[R][J], int g) {
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int j = 0; j < J; ++j) {
        const int row = g * R + r;
        const int kc = tid + j * kPrefThreads;
        b[r][j] = (g < ngroups && row < p.n && kc < cpr)
                      ? ld_stream_v4(p.w + static_cast<int64_t>(row) * p.k + kc * 16)
                      : make_uint4(0, 0, 0, 0);
      }
  };
#pragma unroll
  for (int d = 0; d < D; ++d) fetch(buf[d], cta + d * nctas);

  // wait (bounded) for every token, then read the activations from L2
  if (tid == 0) {
    const int ok = count_wait(fa.flags, p.m) ? 1 : 0;
    __threadfence();
    ready = ok;
  }
  __syncthreads();
  const bool go = ready != 0;
  uint4 av[MT][J];
#pragma unroll
  for (int t = 0; t < MT; ++t)
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int kc = tid + j * kPrefThreads;
      av[t][j] = (go && t < p.m && kc < cpr)
                     ? __ldcg(reinterpret_cast<const uint4*>(p.a + static_cast<int64_t>(t) * p.k + kc * 16))
                     : make_uint4(0, 0, 0, 0);
    }
  const int my_r = tid / MT, my_t = tid % MT;  // output owned by thread tid < R * MT
  const float my_sa = (go && tid < R * MT && my_t < p.m && p.out) ? __ldcg(p.sa + my_t) : 0.0f;
  __syncthreads();  // every thread has read the flags' data
  if (tid == 0 && atomicAdd(fa.flags + 1, 1) == nctas - 1) {
    // the last GEMV CTA to read the tokens leaves the flag words zero
    fa.flags[0] = 0;
    fa.flags[1] = 0;
  }
  if (!go) return;

  int slot = 0;
  for (int g = cta; g < ngroups; g += nctas) {
    const int my_row = g * R + my_r;
    const float my_sw = (tid < R * MT && my_row < p.n && p.out) ? __ldg(p.sw + my_row) : 0.0f;
    int acc[R][MT];
#pragma unroll
    for (int d = 0; d < D; ++d) {
      if (d == slot) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            int a = 0;
#pragma unroll
            for (int j = 0; j < J; ++j) a = dot16(buf[d][r][j], av[t][j], a);
            acc[r][t] = a;
          }
        fetch(buf[d], g + D * nctas);
      }
    }
    slot = slot + 1 == D ? 0 : slot + 1;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int v = __reduce_add_sync(0xFFFFFFFFu, acc[r][t]);
        if (lane == 0) red[warp][r * MT + t] = v;
      }
    __syncthreads();
    if (tid < R * MT && my_row < p.n && my_t < p.m) {
      int sum = 0;
#pragma unroll
      for (int w = 0; w < kPrefThreads / 32; ++w) sum += red[w][tid];
      const int64_t o = static_cast<int64_t>(my_t) * p.n + my_row;
      if (p.c) p.c[o] = sum;
      if (p.out) {
        float v = __int2float_rn(sum);
        v = __fmul_rn(v, my_sa);
        v = __fmul_rn(v, my_sw);
        v = __fmul_rn(v, p.alpha);
        if (p.out_bf16)
          static_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(v);
        else
          static_cast<float*>(p.out)[o] = v;
      }
    }
    __syncthreads();
  }
}

// CTAs of the fused kernel resident at once on the device (queried once per
// device and instance).
template <int MT, int J, bool BF16>
inline int fused_capacity(int dev, int num_sms) {
  static std::atomic<int> cache[64] = {};
  if (dev < 0 || dev >= 64) return 0;
  int known = cache[dev].load(std::memory_order_relaxed);
  if (known == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gemv_i8_fused_kernel<MT, J, BF16>, kPrefThreads, 0) !=
            cudaSuccess ||
        n < 1) {
      cudaGetLastError();
      n = 0;
    }
    known = n > 0 ? n * num_sms : -1;
    cache[dev].store(known, std::memory_order_relaxed);
  }
  return known > 0 ? known : 0;
}

// Launches the fused layer when the shape suits it (the prefetching GEMV's
// shapes, m <= 8).  Returns false without launching otherwise.
template <int MT, bool BF16>
inline bool launch_fused_mt(FusedArgs fa, int dev, int num_sms, cudaStream_t stream, cudaError_t* err) {
  const int J = (fa.g.k / 16 + kPrefThreads - 1) / kPrefThreads;
  auto go = [&](auto kernel, int rows, int minb, int cap) {
    (void)minb;
    const int ngroups = (fa.g.n + rows - 1) / rows;
    int ctas = cap - fa.g.m;
    if (ctas < 1) return false;
    fa.gemv_ctas = ngroups < ctas ? ngroups : ctas;
    *err = launch_pdl(kernel, dim3(fa.g.m + fa.gemv_ctas), dim3(kPrefThreads), 0, stream, 1, fa);
    return true;
  };
  switch (J) {
    case 1:
      return go(gemv_i8_fused_kernel<MT, 1, BF16>, PrefCfg<MT, 1>::rows, PrefCfg<MT, 1>::minb,
                fused_capacity<MT, 1, BF16>(dev, num_sms));
    case 2:
      return go(gemv_i8_fused_kernel<MT, 2, BF16>, PrefCfg<MT, 2>::rows, PrefCfg<MT, 2>::minb,
                fused_capacity<MT, 2, BF16>(dev, num_sms));
    case 3:
      if constexpr (MT <= 4)
        return go(gemv_i8_fused_kernel<MT, 3, BF16>, PrefCfg<MT, 3>::rows, PrefCfg<MT, 3>::minb,
                  fused_capacity<MT, 3, BF16>(dev, num_sms));
      return false;
    default:
      if constexpr (MT <= 4)
        return go(gemv_i8_fused_kernel<MT, 4, BF16>, PrefCfg<MT, 4>::rows, PrefCfg<MT, 4>::minb,
                  fused_capacity<MT, 4, BF16>(dev, num_sms));
      return false;
  }
}

template <bool BF16>
inline bool launch_fused(const FusedArgs& fa, int dev, int num_sms, cudaStream_t stream, cudaError_t* err) {
  if (!pref_supported(fa.g.m, fa.g.k)) return false;
  if (fa.g.m <= 1) return launch_fused_mt<1, BF16>(fa, dev, num_sms, stream, err);
  if (fa.g.m <= 2) return launch_fused_mt<2, BF16>(fa, dev, num_sms, stream, err);
  if (fa.g.m <= 4) return launch_fused_mt<4, BF16>(fa, dev, num_sms, stream, err);
  return launch_fused_mt<8, BF16>(fa, dev, num_sms, stream, err);
}

template <int MT>
inline cudaError_t launch_pref_mt(const Args& a, int num_sms, cudaStream_t stream) {
  const int J = (a.k / 16 + kPrefThreads - 1) / kPrefThreads;
  auto go = [&](auto kernel, int rows, int minb) {
    const int ngroups = (a.n + rows - 1) / rows;
    const int cap = minb * num_sms;
    return launch_pdl(kernel, dim3(ngroups < cap ? ngroups : cap), dim3(kPrefThreads), 0, stream, 1,
                      a);
  };
  switch (J) {
    case 1:
      return go(gemv_i8_prefetch_kernel<MT, 1>, PrefCfg<MT, 1>::rows, PrefCfg<MT, 1>::minb);
    case 2:
      return go(gemv_i8_prefetch_kernel<MT, 2>, PrefCfg<MT, 2>::rows, PrefCfg<MT, 2>::minb);
    case 3:
      if constexpr (MT <= 4)
        return go(gemv_i8_prefetch_kernel<MT, 3>, PrefCfg<MT, 3>::rows,
                  PrefCfg<MT, 3>::minb);
      break;
    default:
      if constexpr (MT <= 4)
        return go(gemv_i8_prefetch_kernel<MT, 4>, PrefCfg<MT, 4>::rows,
                  PrefCfg<MT, 4>::minb);
      break;
  }
  return cudaErrorInvalidValue;  // (pref_supported rules these shapes out)
}

inline cudaError_t launch(const Args& a, int num_sms, cudaStream_t stream) {
  if (pref_supported(a.m, a.k)) {
    if (a.m <= 1) return launch_pref_mt<1>(a, num_sms, stream);
    if (a.m <= 2) return launch_pref_mt<2>(a, num_sms, stream);
    if (a.m <= 4) return launch_pref_mt<4>(a, num_sms, stream);
    return launch_pref_mt<8>(a, num_sms, stream);
  }
  const int ngroups = (a.n + kRows - 1) / kRows;
  const int grid = ngroups < 64 * num_sms ? ngroups : 64 * num_sms;
  const dim3 g(grid), b(kThreads);
  if (a.m <= 1) return launch_pdl(gemv_i8_kernel<1>, g, b, 0, stream, 1, a);
  if (a.m <= 2) return launch_pdl(gemv_i8_kernel<2>, g, b, 0, stream, 1, a);
  if (a.m <= 4) return launch_pdl(gemv_i8_kernel<4>, g, b, 0, stream, 1, a);
  return launch_pdl(gemv_i8_kernel<8>, g, b, 0, stream, 1, a);
}

}  // namespace gemv
}  // namespace qk
