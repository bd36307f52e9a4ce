// gemm_1sm.cuh -- the 1-SM tcgen05 GEMM kernels (cta_group::1, M = 128):
// the per-channel kernel with its cluster split-K and MoE form, and the two
// group-128 kernels (128 x 128 with the int32 sums, 128 x 256 output only).
#pragma once

#include "gemm_core.cuh"

namespace qk {
namespace gemm {

// ---------------------------------------------------------------- kernels
template <class S>
__device__ __forceinline__ S& storage(uint8_t* raw) {
  return *reinterpret_cast<S*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
}

template <class S, int STAGES, int NACC, int EPI_WARPS>
__device__ __forceinline__ void setup(S& s) {
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(smem_addr(&s.full[i]), 1);
      mbar_init(smem_addr(&s.empty[i]), 1);
    }
    for (int i = 0; i < NACC; ++i) {
      mbar_init(smem_addr(&s.acc_full[i]), 1);
      mbar_init(smem_addr(&s.acc_empty[i]), EPI_WARPS);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_addr(&s.aux_full[i]), 32);
      mbar_init(smem_addr(&s.aux_empty[i]), EPI_WARPS);
    }
    mbar_init(smem_addr(&s.drain), 1);
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&s.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

template <class S>
__device__ __forceinline__ void teardown(S& s, uint32_t tmem) {
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if ((threadIdx.x >> 5) == 1) tmem_dealloc(tmem, kTmemCols);
}

// Split-K of the 1-SM kernel through distributed shared memory.  The
// cluster is the `splits` CTAs of one tile (CTA j computed K slice j, and j
// is its cluster rank); each has staged its 128 x BN int32 partial in its
// operand ring as four slots of 32 x BN int32 (32 KB at BN = 256), one per
// TMEM lane quadrant (see epilogue_channel).  After a cluster barrier, CTA j takes the 32-column
// chunks c = j, j + splits, ... of the tile; for each, epilogue warp q sums
// the chunk's 32 rows of quadrant q over the cluster's CTAs (all sources'
// loads in flight together; integer adds, exact), then dequantises and
// stores.  The scales of the whole tile were staged in the warp's slot
// before the accumulator was ready.
template <int BN, bool F8, class S>
__device__ void channel_cluster_reduce(S& s, const Args& p, const CUtensorMap* tmO) {
  const int lane = threadIdx.x & 31;
  const int ew = (threadIdx.x >> 5) - 2;
  const int quad = (threadIdx.x >> 5) & 3;
  const int j = static_cast<int>(cluster_rank());
  const int tile = static_cast<int>(blockIdx.x) / p.sk.splits;
  const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
  const float* sws = s.sw_tile[ew];
  uint8_t* box = s.out_stage[ew];
  const int row0 = tm * BM + quad * 32, row = row0 + lane;
  const bool rv = row < p.m;
  const float sa = (rv && p.out) ? __ldg(p.sa + row) : 0.0f;
  const uint32_t slot = smem_addr(&s.a[0][0]) + static_cast<uint32_t>(quad * (32 * BN * 4));
  for (int c = j; c < BN / 32; c += p.sk.splits) {
    const int col0 = tn * BN + c * 32;
    uint32_t va[32];
    // every source's part of the chunk requested at once (32 loads in
    // flight per lane: one cluster round trip per chunk)
    int4 t4[4][8];
#pragma unroll
    for (int o = 0; o < 4; ++o)
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4)
        t4[o][q4] = o < p.sk.splits
                        ? ld_dsmem_v4(map_to_rank(
                              slot + static_cast<uint32_t>(((c * 8 + q4) * 32 + lane) * 16),
                              static_cast<uint32_t>(o)))
                        : make_int4(0, 0, 0, 0);
#pragma unroll
    for (int o = 0; o < 4; ++o)
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) order_after_loads(t4[o][q4]);
    if constexpr (F8) {
      // slice 0, then the others in ascending order (fp32: order matters)
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        va[q4 * 4] = static_cast<uint32_t>(t4[0][q4].x);
        va[q4 * 4 + 1] = static_cast<uint32_t>(t4[0][q4].y);
        va[q4 * 4 + 2] = static_cast<uint32_t>(t4[0][q4].z);
        va[q4 * 4 + 3] = static_cast<uint32_t>(t4[0][q4].w);
      }
#pragma unroll
      for (int o = 1; o < 4; ++o)
        if (o < p.sk.splits) {
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) acc_add4<true>(va + q4 * 4, t4[o][q4]);
        }
    } else {
      // int32: any order (sources past `splits` were loaded as zero)
#pragma unroll
      for (int i = 0; i < 32; ++i) va[i] = 0;
#pragma unroll
      for (int o = 0; o < 4; ++o)
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) acc_add4<false>(va + q4 * 4, t4[o][q4]);
    }
    if (!F8 && p.asym.zp) apply_zp(p, row, col0, va);
    if (p.tma_out)
      store32_tma<F8>(p, tmO, box, row0, col0, sa, sws + c * 32, va);
    else if (rv && col0 < p.n)
      store32_channel<F8>(p, row, col0, sa, sws + c * 32, va);
  }
  if (p.tma_out && lane == 0) bulk_wait_all();  // the output stores are complete
  __syncwarp();
}

// The per-channel 1-SM kernel comes in two tile widths: 128 x 256 (4
// stages) and 128 x 128 (6 stages, about the same shared memory).  The
// narrow one is taken when it puts more CTAs to work on a small-M problem,
// e.g. 128 x 4096 x 14336: 32 tiles x 4 slices on 128 SMs instead of
// 16 x 4 on 64 (17.6 against 22.3 us), or as many CTAs in fewer, short
// K slices (channel_plan).  At an equal CTA count and long slices the wide
// tile is faster (256 x 4096 x 14336: 22.7 us for 32 tiles x 4 slices,
// 24.2 us for 64 narrow tiles x 2 slices: the narrow tile reads the
// activations twice as often per weight byte).
constexpr int kChannelBN = 256;
constexpr int kChannelThreads = 64 + 4 * 32;
template <int BN>
constexpr int channel_stages() {
  return BN == 256 ? 4 : 6;
}
template <int BN>
struct alignas(1024) ChannelStorageT {
  static constexpr int kStages = channel_stages<BN>();
  uint8_t a[kStages][BM * BK];
  uint8_t b[kStages][BN * BK];
  uint8_t out_stage[4][kOutBoxBytes];  // each epilogue warp's TMA store box
  float sw_tile[4][BN];                // each epilogue warp's channel scales
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t aux_full[2];  // (unused by this kernel; set up with the others)
  uint64_t aux_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
using ChannelStorage = ChannelStorageT<kChannelBN>;

template <bool F8, bool MOE = false, int BN = kChannelBN>
__global__ void __launch_bounds__(kChannelThreads, 1)
    gemm_i8_channel_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmO, const Args p) {
  using S = ChannelStorageT<BN>;
  constexpr int kStages = S::kStages;
  extern __shared__ uint8_t smem_raw[];
  S& s = storage<S>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (p.tma_out) prefetch_tmap(&tmO);
  }
  setup<S, kStages, 2, 4>(s);
  if (warp != 0) {  // (the producer waits inside produce)
    griddep_wait();  // set-up above overlapped the previous kernel
    griddep_launch_dependents();
  }
  const uint32_t tmem = s.tmem_base;
  if (warp == 0) {
    if (lane == 0) produce<BN, kStages, MOE, false, !MOE>(s, &tmA, &tmB, p);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_issue<BN, kStages, 2, false, F8, MOE>(s, tmem, p);
    __syncwarp();
  } else {
    epilogue_channel<BN, 2, F8, MOE>(s, tmem, p, &tmO);
  }
  if (p.sk.csplit) {
    cluster_sync_all();  // every CTA of the cluster has staged its partial
    if (warp >= 2) channel_cluster_reduce<BN, F8>(s, p, &tmO);
    cluster_sync_all();  // the peers are done reading this CTA's slots
  }
  teardown(s, tmem);
}

constexpr int kGroupBN = 128;
constexpr int kGroupStages = 5;
using GroupStorage = Storage<kGroupBN, kGroupStages, 4, 2 * kScaleGroups * kGroupBN>;

template <bool WITH_C>
__global__ void __launch_bounds__(GroupCfg<WITH_C>::threads, 1)
    gemm_i8_group_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB, const Args p) {
  extern __shared__ uint8_t smem_raw[];
  GroupStorage& s = storage<GroupStorage>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  constexpr int kEpiWarps = GroupCfg<WITH_C>::epi_warps;
  setup<GroupStorage, kGroupStages, 4, kEpiWarps>(s);
  if (warp != 0) {  // (the producer waits inside produce)
    griddep_wait();  // set-up above overlapped the previous kernel
    griddep_launch_dependents();
  }
  const uint32_t tmem = s.tmem_base;
  if (warp == 0) {
    if (lane == 0) produce<kGroupBN, kGroupStages>(s, &tmA, &tmB, p);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_issue<kGroupBN, kGroupStages, 4, true>(s, tmem, p);
    __syncwarp();
  } else if (warp < 2 + kEpiWarps) {
    epilogue_group<kGroupBN, 4, WITH_C>(s, tmem, p);
  } else {
    stage_group_scales<kGroupBN, kGroupBN / 32, false>(s, p);
  }
  teardown(s, tmem);
}

// ---------------------------------------------------------------- group-128, 128 x 256 tiles
// Wide form of the group kernel, for outputs without the int32 sums.  The
// 128 x 256 MMA (N = 256) reads fewer operand bytes per multiply-add than
// 128 x 128, so the tensor pipe accepts a group's four MMAs faster; TMEM
// holds two 256-column partial buffers, shared memory four 48 KB stages and
// a 32 KB scale slice.
//
// Warpgroup 0: TMA producer (warp 0), MMA issuer (warp 1), scale stager
// (warp 2), warp 3 idle.  Warpgroups 1-4: 16 epilogue warps; warp w owns
// TMEM lanes 32*(w%4) and columns [64 h, 64 h + 64), h = (w - 4) / 4, so
// each epilogue thread keeps 64 fp32 running sums.  The registers follow the
// work: warpgroup 0 drops to 64 per thread and the epilogue rises to 104
// (128*64 + 512*104 = 61440 = 640*96, the launch allocation).
//
// Work comes as units (group_unit): whole tiles, and, when the last wave
// would be partial, the halves of its tiles cut at the middle group, the
// running sums passing from one CTA to another through the workspace.
//
// Per element and group: one exact int-to-float conversion and one fused
// multiply-add, in ascending group order.  (Packed f32x2 pairs with the
// 1.5 * 2^23 bias trick issue more instructions here, because forming the
// pairs costs moves: 318.6 against 273.8 us at 2048 x 8192 x 8192.)
constexpr int kGroupWideBN = 256;
constexpr int kGroupWideStages = 4;
constexpr int kGroupWideEpiWarps = 16;
constexpr int kGroupWideCols = 64;  // columns per epilogue warp
constexpr int kGroupWideThreads = 128 + kGroupWideEpiWarps * 32;
constexpr int kGroupWideCtrlRegs = 64;
constexpr int kGroupWideEpiRegs = 104;
constexpr int kGroupWideLaunchRegs =  // registers per thread the launch must provide
    (128 * kGroupWideCtrlRegs + kGroupWideEpiWarps * 32 * kGroupWideEpiRegs + kGroupWideThreads - 1) /
    kGroupWideThreads;
using GroupWideStorage =
    Storage<kGroupWideBN, kGroupWideStages, 2, 2 * kScaleGroups * kGroupWideBN>;

// A split tile's running sums in the workspace: [tail tile][region]
// [column][lane], so each column's 32 rows are one 128-byte line.  Each of
// the 16 epilogue warps of the first part adds 1 to the tile's counter
// gflag[tail tile] once its region is written.  In the CTA running the
// second part, the scale stager waits for 16 (bounded) before it publishes
// the part's first scale slice, and leaves the counter zero for the next
// call; the epilogue warps read the sums after that slice's barrier.
__device__ __forceinline__ float* group_state(const Args& p, int tt, int region) {
  return p.gcut.gstate + (static_cast<int64_t>(tt) * 16 + region) * (kGroupWideCols * 32);
}

template <class S>
__device__ void epilogue_group_wide(S& s, uint32_t tmem, const Args& p) {
  constexpr int BN = kGroupWideBN, COLS = kGroupWideCols;
  const int ntiles = p.tiles_m * p.tiles_n;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int quad = warp & 3;
  const int sub = (warp - 4) >> 2;  // column slice of the tile
  const int region = warp - 4;  // 0..15
  uint32_t abuf = 0, aphase = 0, sbuf = 0, sphase = 0;
  bool ok = true;
  GroupUnit u;
  for (int i = 0; ok && group_unit(p, i, u); ++i) {
    const int tm = u.tile % p.tiles_m, tn = u.tile / p.tiles_m;
    const int colbase = tn * BN + sub * COLS;
    float fs[COLS];
#pragma unroll
    for (int j = 0; j < COLS; ++j) fs[j] = 0.0f;
    for (int g = u.g0; g < u.g1; ++g) {
      const int gs = (g - u.g0) % kScaleGroups;
      if (gs == 0 && !warp_wait(smem_addr(&s.aux_full[sbuf]), sphase, &s.abort)) {
        ok = false;
        break;
      }
      if (u.part == 2 && g == u.g0) {
        // continue from the first part's sums (another CTA's; the stager
        // saw them complete before publishing this slice)
        const float* st = group_state(p, u.tile - (ntiles - p.gcut.gsplit), region) + lane;
#pragma unroll
        for (int j = 0; j < COLS; ++j) fs[j] = __ldcg(st + j * 32);
      }
      if (!warp_wait(smem_addr(&s.acc_full[abuf]), aphase, &s.abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem + (static_cast<uint32_t>(quad * 32) << 16) + abuf * BN +
                          sub * COLS;
      const float4* sc4 = reinterpret_cast<const float4*>(s.scales + sbuf * (kScaleGroups * BN) +
                                                          gs * BN + sub * COLS);
#pragma unroll
      for (int c = 0; c < COLS / 16; ++c) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tb + c * 16, v);
        tmem_ld_wait();
        if (c == COLS / 16 - 1) release_acc<2>(s, abuf, aphase, lane);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 s4 = sc4[c * 4 + q];
          const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = c * 16 + q * 4 + e;
            // |P| < 2^24: the conversion is exact
            fs[j] = __fmaf_rn(__int2float_rn(static_cast<int>(v[4 * q + e])), sv[e], fs[j]);
          }
        }
      }
      if (gs == kScaleGroups - 1 || g + 1 == u.g1) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&s.aux_empty[sbuf]));
        if (++sbuf == 2) {
          sbuf = 0;
          sphase ^= 1u;
        }
      }
    }
    if (!ok) break;
    if (u.part == 1) {
      // hand the running sums to the CTA that finishes the tile
      const int tt = u.tile - (ntiles - p.gcut.gsplit);
      float* st = group_state(p, tt, region) + lane;
#pragma unroll
      for (int j = 0; j < COLS; ++j) __stcg(st + j * 32, fs[j]);
      __threadfence();
      __syncwarp();
      if (lane == 0) atomicAdd(p.gcut.gflag + tt, 1);
      continue;
    }
    const int row = tm * BM + quad * 32 + lane;
    if (row < p.m) {
      const float sa = __ldg(p.sa + row);
#pragma unroll
      for (int g8 = 0; g8 < COLS / 8; ++g8) {
        const int col = colbase + g8 * 8;
        if (col >= p.n) break;
        const int64_t o = static_cast<int64_t>(row) * p.n + col;
        float r[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = __fmul_rn(__fmul_rn(fs[g8 * 8 + e], sa), p.alpha);
        if (p.out_bf16) {
          uint4 pk;
          pk.x = pack_bf16x2(r[0], r[1]);
          pk.y = pack_bf16x2(r[2], r[3]);
          pk.z = pack_bf16x2(r[4], r[5]);
          pk.w = pack_bf16x2(r[6], r[7]);
          *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + o) = pk;
        } else {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + o);
          dst[0] = make_float4(r[0], r[1], r[2], r[3]);
          dst[1] = make_float4(r[4], r[5], r[6], r[7]);
        }
      }
    }
  }
}

__global__ void __launch_bounds__(kGroupWideThreads, 1)
    gemm_i8_group_wide_kernel(const __grid_constant__ CUtensorMap tmA,
                              const __grid_constant__ CUtensorMap tmB, const Args p) {
  extern __shared__ uint8_t smem_raw[];
  GroupWideStorage& s = storage<GroupWideStorage>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  setup<GroupWideStorage, kGroupWideStages, 2, kGroupWideEpiWarps>(s);
  if (warp != 0) {  // (the producer waits inside produce)
    griddep_wait();  // set-up above overlapped the previous kernel
    griddep_launch_dependents();
  }
  const uint32_t tmem = s.tmem_base;
  if (warp < 4) {
    regs_dec<kGroupWideCtrlRegs>();
    if (warp == 0) {
      if (lane == 0) produce<kGroupWideBN, kGroupWideStages, false, true>(s, &tmA, &tmB, p);
      __syncwarp();
    } else if (warp == 1) {
      if (lane == 0) mma_issue<kGroupWideBN, kGroupWideStages, 2, true, false, false, true>(s, tmem, p);
      __syncwarp();
    } else if (warp == 2) {
      stage_group_scales<kGroupWideBN, 1, true>(s, p);
    }
  } else {
    regs_inc<kGroupWideEpiRegs>();
    epilogue_group_wide(s, tmem, p);
  }
  teardown(s, tmem);
}

}  // namespace gemm
}  // namespace qk
