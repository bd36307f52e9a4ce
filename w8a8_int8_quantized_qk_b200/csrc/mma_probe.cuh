// mma_probe.cuh -- the INT8 tensor-core rate of this device, measured: a
// diagnostic kernel that issues tcgen05.mma.kind::i8 back to back on fixed
// shared-memory operands into one TMEM accumulator, with no global-memory
// traffic, so that its duration is the tensor pipe's own time.  The roofline
// of the library's GEMMs ("KV-cache kernels" section 01: the compute
// ceiling against which a kernel's achieved rate is read) divides by the
// rate this kernel reaches.
//
// Forms: cta_group::1 (one CTA per SM, M = 128) and cta_group::2 (a cluster
// of two CTAs on the two SMs of a pair, M = 256, the leader issuing); N is
// 32 .. 256 (a multiple of 16), K = 32 per instruction.  Every CTA's MMA
// thread records the SM clock cycles from its first issue to the completion
// of its last MMA, so the host can also form MACs per clock per SM.
//
// Operands: all zero, or bytes from a counter-based hash of a seed.  The
// rate depends on the values: on a B200 the pair form reaches about 8190
// multiply-adds per clock per SM on zeros and measurably less on uniformly
// random bytes at the same SM clock, so a GEMM on random operands is read
// against the random-operand rate as well.
#pragma once

#include "qk_common.cuh"

namespace qk {
namespace probe {

constexpr int kThreads = 128;
constexpr int kTileBytes = 128 * 128;  // one 128-row x 128-byte swizzled operand tile

struct alignas(1024) ProbeStorage {
  uint8_t a[kTileBytes];
  uint8_t b[2 * kTileBytes];  // up to 256 rows of B
  uint64_t done;
  uint32_t tmem_base;
};

// Word w of a seeded operand tile: a 32-bit finaliser (multiply-xorshift) of
// the word's index and the seed, so every byte is close to uniform.
__device__ __forceinline__ uint32_t operand_word(uint32_t seed, uint32_t w) {
  uint32_t x = w * 0x9E3779B1u ^ seed * 0x85EBCA77u;
  x ^= x >> 16;
  x *= 0x7FEB352Du;
  x ^= x >> 15;
  x *= 0x846CA68Bu;
  x ^= x >> 16;
  return x;
}

// `iters` instructions of shape (M = 128 * PAIR? 256 : 128) x n x 32.
// cycles[cta] (optional): clock64 cycles between the first issue and the
// last completion, on the issuing CTA (0 on a pair's second CTA).
template <bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    mma_rate_kernel(int n, int iters, uint32_t seed, unsigned long long* cycles) {
  extern __shared__ uint8_t smem_raw[];
  ProbeStorage& s = *reinterpret_cast<ProbeStorage*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const uint32_t crank = PAIR ? cluster_rank() : 0u;
  // operands: zeros (seed 0) or hashed bytes, different in every CTA
  const uint32_t cseed = seed == 0 ? 0u : seed + 0x632BE5ABu * blockIdx.x;
  auto fill = [&](uint8_t* dst, int bytes, uint32_t salt) {
    for (int i = threadIdx.x; i < bytes / 16; i += kThreads) {
      int4 v = make_int4(0, 0, 0, 0);
      if (seed != 0) {
        const uint32_t w = (salt + static_cast<uint32_t>(i)) * 4u;
        v = make_int4(static_cast<int>(operand_word(cseed, w)), static_cast<int>(operand_word(cseed, w + 1)),
                      static_cast<int>(operand_word(cseed, w + 2)), static_cast<int>(operand_word(cseed, w + 3)));
      }
      reinterpret_cast<int4*>(dst)[i] = v;
    }
  };
  fill(s.a, kTileBytes, 0u);
  fill(s.b, 2 * kTileBytes, static_cast<uint32_t>(kTileBytes / 16));
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&s.done), 1);
    fence_mbar_init();
  }
  fence_proxy_async_smem();  // the operands are visible to the tensor core
  if (warp == 0) {
    if (PAIR) {
      tmem_alloc_pair(smem_addr(&s.tmem_base), 256);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_addr(&s.tmem_base), 256);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync_all();  // both CTAs' operands, barriers and TMEM exist
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  if (threadIdx.x == 0 && crank == 0) {
    const uint32_t idesc = idesc_i8(PAIR ? 256 : 128, n);
    const uint32_t a0 = smem_addr(s.a), b0 = smem_addr(s.b);
    const long long t0 = clock64();
    for (int i = 0; i < iters; ++i) {
      const uint32_t kk = static_cast<uint32_t>(i & 3) * 32u;  // walk the 128-byte row
      if (PAIR)
        mma_i8_pair(tmem, sdesc_k_sw128(a0 + kk), sdesc_k_sw128(b0 + kk), idesc, i > 0 ? 1u : 0u);
      else
        mma_i8(tmem, sdesc_k_sw128(a0 + kk), sdesc_k_sw128(b0 + kk), idesc, i > 0 ? 1u : 0u);
    }
    if (PAIR)
      mma_commit_pair(smem_addr(&s.done), static_cast<uint16_t>(0x3u));
    else
      mma_commit(smem_addr(&s.done));
    mbar_wait(smem_addr(&s.done), 0u, nullptr);
    const long long t1 = clock64();
    if (cycles) cycles[blockIdx.x] = static_cast<unsigned long long>(t1 - t0);
  } else if (PAIR && threadIdx.x == 0) {
    // the leader's commit also arrives here once the MMAs that wrote this
    // CTA's TMEM are complete
    mbar_wait(smem_addr(&s.done), 0u, nullptr);
    if (cycles) cycles[blockIdx.x] = 0ull;
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync_all();
  tc_fence_after();
  if (warp == 0) {
    if (PAIR)
      tmem_dealloc_pair(tmem, 256);
    else
      tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------- interference
// The pair MMA loop of mma_rate_kernel<true> (256 x 256 x 32, groups of four
// into alternating 256-column buffers, seeded operands) while warps 4..11 of
// both CTAs of the pair run a companion arithmetic loop until the MMAs are
// done (a flag in each CTA's shared memory, bounded by an iteration count):
//   0 none, 1 fp32 fused multiply-add, 2 fp32 multiply, 3 int32 -> fp32
//   conversion and a logic op (the ALU pipe), 4 int32 multiply-add,
//   5 conversion + fused multiply-add (the group-128 epilogue's mix),
//   6 fp32 pair -> bf16x2 conversion (the epilogues' output packing).
// cycles[cta]: the leader's clock64 cycles from the first MMA issue to the
// completion of the last (0 on the second CTA of a pair).
constexpr int kMixThreads = 384;
constexpr int kMixCompanionIters = 200000;  // bound on the companion loop

__device__ float g_mix_sink[kMixThreads];  // keeps the companion loops' results live

struct alignas(1024) MixStorage {
  uint8_t a[kTileBytes];
  uint8_t b[kTileBytes];
  uint64_t done;
  uint32_t tmem_base;
  int stop;
};

template <int MODE>
__device__ __forceinline__ void companion_loop(volatile int* stop) {
  float f[16];
  int v[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    f[j] = 0.0f;
    v[j] = static_cast<int>(operand_word(0x5EEDu, threadIdx.x * 16u + j)) >> 11;
  }
  const float sc = 1.0000001f;
  for (int n = 0; n < kMixCompanionIters && !*stop; ++n) {
#pragma unroll 4
    for (int r = 0; r < 64; ++r) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if constexpr (MODE == 1) f[j] = __fmaf_rn(f[j], sc, 0.5f);
        if constexpr (MODE == 2) f[j] = __fmul_rn(f[j], sc);
        if constexpr (MODE == 3) v[j] = __float_as_int(__int2float_rn(v[j])) ^ 0x1357;
        if constexpr (MODE == 4) v[j] = v[j] * static_cast<int>(threadIdx.x) + 0x1357;
        if constexpr (MODE == 5) {
          f[j] = __fmaf_rn(__int2float_rn(v[j]), sc, f[j]);
          v[j] ^= 0x1357;
        }
        if constexpr (MODE == 6) {
          // the packed pair feeds the next one's operands, so the loop
          // cannot be folded away
          const uint32_t b2 = pack_bf16x2(__int_as_float(v[j]), __int_as_float(v[j] ^ 0x40000000));
          v[j] = static_cast<int>(b2 ^ 0x3F803F80u);
        }
      }
    }
  }
  float acc = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) acc += f[j] + static_cast<float>(v[j]);
  if (acc == 1234.5f) g_mix_sink[threadIdx.x] = acc;
}

template <int MODE>
__global__ void __launch_bounds__(kMixThreads, 1)
    mma_mix_kernel(int groups, unsigned long long* cycles) {
  extern __shared__ uint8_t smem_raw[];
  MixStorage& s = *reinterpret_cast<MixStorage*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_rank();
  for (int i = threadIdx.x; i < kTileBytes / 4; i += kMixThreads) {
    reinterpret_cast<uint32_t*>(s.a)[i] = operand_word(0x9A1u + blockIdx.x, static_cast<uint32_t>(i));
    reinterpret_cast<uint32_t*>(s.b)[i] = operand_word(0x3C7u + blockIdx.x, static_cast<uint32_t>(i));
  }
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&s.done), 1);
    s.stop = 0;
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc_pair(smem_addr(&s.tmem_base), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  if (warp == 0) {
    if (lane == 0) {
      if (crank == 0) {
        const uint32_t idesc = idesc_i8(256, 256);
        const long long t0 = clock64();
        for (int i = 0; i < 4 * groups; ++i) {
          const uint32_t kk = static_cast<uint32_t>(i & 3) * 32u;
          const uint32_t d = tmem + static_cast<uint32_t>((i >> 2) & 1) * 256u;
          mma_i8_pair(d, sdesc_k_sw128(smem_addr(s.a) + kk), sdesc_k_sw128(smem_addr(s.b) + kk), idesc,
                      (i & 3) ? 1u : 0u);
        }
        mma_commit_pair(smem_addr(&s.done), static_cast<uint16_t>(0x3u));
        mbar_wait(smem_addr(&s.done), 0u, nullptr);
        if (cycles) cycles[blockIdx.x] = static_cast<unsigned long long>(clock64() - t0);
      } else {
        mbar_wait(smem_addr(&s.done), 0u, nullptr);
        if (cycles) cycles[blockIdx.x] = 0ull;
      }
      // both CTAs' companions may stop
      *reinterpret_cast<volatile int*>(&s.stop) = 1;
    }
    __syncwarp();
  } else if (warp >= 4 && MODE != 0) {
    companion_loop<MODE>(&s.stop);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

// Both probes request more than half of an SM's shared memory, so that no
// two of their CTAs share an SM: a CTA's TMEM allocation then never waits
// for another CTA's.
constexpr size_t kOneCtaPerSmBytes = 120 * 1024;
inline size_t smem_bytes() {
  return sizeof(ProbeStorage) + 1024 > kOneCtaPerSmBytes ? sizeof(ProbeStorage) + 1024 : kOneCtaPerSmBytes;
}
inline size_t mix_smem_bytes() {
  return sizeof(MixStorage) + 1024 > kOneCtaPerSmBytes ? sizeof(MixStorage) + 1024 : kOneCtaPerSmBytes;
}

// ctas: CTAs of the grid (a multiple of 2 for pairs).
inline cudaError_t launch(bool pair, int n, int iters, int ctas, uint32_t seed, unsigned long long* cycles,
                          cudaStream_t stream) {
  auto k = pair ? mma_rate_kernel<true> : mma_rate_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem_bytes()));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_bytes();
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = pair ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pair ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k, n, iters, seed, cycles);
}

// ctas: CTAs of the grid, a multiple of 2 (pairs).
inline cudaError_t launch_mix(int companion, int groups, int ctas, unsigned long long* cycles,
                              cudaStream_t stream) {
  void (*k)(int, unsigned long long*) = nullptr;
  switch (companion) {
    case 0: k = mma_mix_kernel<0>; break;
    case 1: k = mma_mix_kernel<1>; break;
    case 2: k = mma_mix_kernel<2>; break;
    case 3: k = mma_mix_kernel<3>; break;
    case 4: k = mma_mix_kernel<4>; break;
    case 5: k = mma_mix_kernel<5>; break;
    default: k = mma_mix_kernel<6>; break;
  }
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(mix_smem_bytes()));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(kMixThreads);
  cfg.dynamicSmemBytes = mix_smem_bytes();
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, groups, cycles);
}

}  // namespace probe
}  // namespace qk
