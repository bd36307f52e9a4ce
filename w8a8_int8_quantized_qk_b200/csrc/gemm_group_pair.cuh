// gemm_group_pair.cuh -- the group-128 GEMM on CTA pairs (tcgen05.mma
// cta_group::2, 256 x 256 tiles), output only.
//
// Definition ("KV-cache kernels" section 03, per-group scales along K; the
// group-128 workload): P_g = sum over the 128 K of group g of a * b (int32),
// f = fma((float)P_g, sw[n, g], f) in ascending g, out = (f * sa[m]) * alpha.
//
// Why this shape.  Per SM the tensor core turns out 64 (element, group)
// partials per clock at its peak (8192 int8 multiply-adds per clock, 128 per
// partial), and each partial costs the epilogue one int32 -> fp32 conversion,
// which runs on the ALU pipe at 64 lanes per clock: the conversion alone can
// keep pace with the MMA only if nothing else per element touches that pipe.
// So the only other per-element steps are the fused multiply-add (FMA pipe)
// and a quarter of a broadcast shared load for the scales; the running sums
// live in registers (128 per thread), and per-group overhead is amortised
// over 128 columns per warp.
// What bounds the kernel: fp32 arithmetic on the CUDA cores slows the tensor
// core of the same SM (qk_selftest_mma_interference: a group of four pair
// MMAs takes 512 cycles alone, 512 beside conversion or integer loops, and
// 1201-3948 beside fp32 FFMA or FMUL loops).  One FFMA per element per group
// is the minimum this definition allows, so the MMAs run at about a third of
// their rate while the epilogue folds (176 us at 2048 x 8192 x 8192).  Half
// the FFMA instructions as packed fma.rn.f32x2 measured slower (198 us).
// The CTA pair keeps the MMA at N = 256 per SM while each SM loads only its
// own halves of A and B (the streaming rate of this tile is 0.93 of the
// tensor peak, against 0.81 for a 1-SM 128 x 256 tile).
//
// Roles per CTA (384 threads): warp 0 the TMA producer, warp 1 the MMA
// issuer (the pair's leader only), warps 2-3 the scale stagers, warps 4-11
// the epilogue (warp w reads TMEM lanes 32 * (w % 4) and columns [128 h,
// 128 h + 128), h = (w - 4) / 4).  setmaxnreg moves registers from the
// control warpgroup (80 each) to the epilogue (208 each).  A bf16 output
// leaves through TMA bulk tensor stores from each epilogue warp's 2 KB box
// (per-lane global stores of 16 bytes, one row per lane, measured 14.5 us
// slower at 2048 x 8192 x 8192: the tile's stores hold up the next tile's
// first groups).
//
// Work units come from group_plan.h with the pairs as workers: whole tiles,
// and, when the last wave would be partial, its tiles cut at the middle
// group, the first part run early by one pair, the second part run last by
// another that continues the running sums through the workspace.
#pragma once

#include "gemm_pair.cuh"

namespace qk {
namespace gemm {

constexpr int kGpBN = 256;
constexpr int kGpStages = 6;
constexpr int kGpEpiWarps = 8;
constexpr int kGpCols = 128;  // columns per epilogue warp
constexpr int kGpThreads = 128 + kGpEpiWarps * 32;
constexpr int kGpCtrlRegs = 80;
constexpr int kGpEpiRegs = 208;
constexpr int kGpLaunchRegs =  // registers per thread the launch must provide
    (128 * kGpCtrlRegs + kGpEpiWarps * 32 * kGpEpiRegs + kGpThreads - 1) / kGpThreads;
constexpr int kGpSlice = 8;  // groups per staged scale slice

struct alignas(1024) GroupPairStorage {
  uint8_t a[kGpStages][128 * BK];  // this CTA's 128 rows of A
  uint8_t b[kGpStages][128 * BK];  // this CTA's 128 rows of B
  float scales[2][kGpSlice * kGpBN];  // [slice buffer][group][column]
  uint8_t out_stage[kGpEpiWarps][kOutBoxBytes];  // each epilogue warp's bf16 output box
  uint64_t full[kGpStages];
  uint64_t empty[kGpStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t aux_full[2];
  uint64_t aux_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// The i-th unit of pair `pi` of `np` (false past its last).
__device__ __forceinline__ bool gp_unit(const Args& p, int pi, int np, int i, GroupUnit& u) {
  return group_unit_at(pi, np, p.tiles_m * p.tiles_n, p.gcut.gsplit, p.groups, p.gcut.gmid, i, u);
}

// A cut tile's running sums in the workspace: [tail tile][CTA of the pair]
// [epilogue warp][pair of columns][lane], two binary32 per entry, so each
// pair of columns of a warp is one 256-byte line.  The first part's 8 epilogue warps
// of CTA r each add 1 to gflag[2 * tail tile + r] once their region is
// written; in the pair running the second part, CTA r's stager waits for 8
// before it publishes the part's first scale slice and leaves the counter
// zero for the next call.
__device__ __forceinline__ uint64_t* gp_state(const Args& p, int tt, int rank, int ew) {
  return reinterpret_cast<uint64_t*>(p.gcut.gstate) +
         ((static_cast<int64_t>(tt) * 2 + rank) * kGpEpiWarps + ew) * (kGpCols / 2) * 32;
}

__device__ void gp_produce(GroupPairStorage& s, const CUtensorMap* tmA, const CUtensorMap* tmB,
                           const Args& p, uint32_t pr, uint32_t lead) {
  const int np = gridDim.x >> 1, pi = blockIdx.x >> 1;
  uint32_t stage = 0, phase = 0, issued = 0;
  bool ok = true;
  GroupUnit u;
  for (int i = 0; ok && gp_unit(p, pi, np, i, u); ++i) {
    const int tm = u.tile % p.tiles_m, tn = u.tile / p.tiles_m;
    const int ya = tm * 256 + static_cast<int>(pr) * 128;
    const int yb = tn * kGpBN + static_cast<int>(pr) * 128;
    for (int g = u.g0; g < u.g1; ++g) {
      if (!mbar_wait(smem_addr(&s.empty[stage]), phase ^ 1u, &s.abort)) {
        ok = false;
        break;
      }
      const uint32_t fl = smem_addr(&s.full[stage]);
      if (pr == 0) mbar_arrive_expect_tx(fl, 2u * kPairStageBytes);
      const uint32_t fb = map_to_rank(fl, lead);
      tma_load_2d_pair(smem_addr(s.a[stage]), tmA, fb, g * BK, ya);
      tma_load_2d_pair(smem_addr(s.b[stage]), tmB, fb, g * BK, yb);
      ++issued;
      if (++stage == kGpStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  // both CTAs' copies complete on the leader's barriers: the leader waits
  // (bounded) for the last phases it armed before the pair may exit
  if (pr == 0) {
    const uint32_t first = issued > kGpStages ? issued - kGpStages : 0u;
    for (uint32_t i = first; i < issued; ++i)
      mbar_wait(smem_addr(&s.full[i % kGpStages]), (i / kGpStages) & 1u, nullptr);
  }
}

// One group per stage and per accumulator buffer: the four MMAs of a group
// write a fresh int32 partial into buffer abuf, which the epilogue warps of
// both CTAs hand back (acc_empty, on the leader) once they have loaded it.
__device__ void gp_mma(GroupPairStorage& s, uint32_t tmem, const Args& p, uint32_t lead) {
  const uint16_t pair_mask = static_cast<uint16_t>(0x3u << lead);
  const int np = gridDim.x >> 1, pi = blockIdx.x >> 1;
  constexpr uint32_t idesc = idesc_i8(256, kGpBN);
  uint32_t stage = 0, phase = 0, abuf = 0, aphase = 0;
  bool ok = true;
  GroupUnit u;
  for (int i = 0; ok && gp_unit(p, pi, np, i, u); ++i) {
    for (int g = u.g0; g < u.g1; ++g) {
      if (!mbar_wait(smem_addr(&s.acc_empty[abuf]), aphase ^ 1u, &s.abort) ||
          !mbar_wait(smem_addr(&s.full[stage]), phase, &s.abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem + abuf * kGpBN;
      const uint32_t a0 = smem_addr(s.a[stage]), b0 = smem_addr(s.b[stage]);
#pragma unroll
      for (int kk = 0; kk < BK / UMMA_K; ++kk)
        mma_i8_pair(d, sdesc_k_sw128(a0 + kk * UMMA_K), sdesc_k_sw128(b0 + kk * UMMA_K), idesc,
                    kk > 0 ? 1u : 0u);
      mma_commit_pair(smem_addr(&s.empty[stage]), pair_mask);
      mma_commit_pair(smem_addr(&s.acc_full[abuf]), pair_mask);
      if (++stage == kGpStages) {
        stage = 0;
        phase ^= 1u;
      }
      if (++abuf == 2) {
        abuf = 0;
        aphase ^= 1u;
      }
    }
  }
  mma_commit_pair(smem_addr(&s.drain), static_cast<uint16_t>(1u << lead));
  mbar_wait(smem_addr(&s.drain), 0u, nullptr);
}

// Scale stagers (warps 2 and 3): slice i holds sw[n, g] for the tile's 256
// columns and kGpSlice groups, laid out [group][column]; warp 2 + s, lane l
// fetches columns 128 s + 4 l .. + 3 (16-byte loads when the row of groups
// is 16-byte aligned), all of a slice's loads in flight together.
__device__ void gp_stage_scales(GroupPairStorage& s, const Args& p, uint32_t pr) {
  const int np = gridDim.x >> 1, pi = blockIdx.x >> 1;
  const int ntiles = p.tiles_m * p.tiles_n;
  const int lane = threadIdx.x & 31;
  const int sw_warp = (threadIdx.x >> 5) - 2;  // 0 or 1
  const int c_lo = sw_warp * 128 + lane * 4;   // first of this lane's four columns
  const bool vec_rows = (p.groups & 3) == 0;  // rows of scales 16-byte aligned
  uint32_t buf = 0, phase = 0;
  GroupUnit u;
  for (int i = 0; gp_unit(p, pi, np, i, u); ++i) {
    const int col0 = (u.tile / p.tiles_m) * kGpBN + c_lo;
    if (u.part == 2 && sw_warp == 0) {
      // the first part's running sums (another pair's) must be complete
      // before this unit's first slice is published
      bool seen = true;
      if (lane == 0) {
        int* cnt = p.gcut.gflag + 2 * (u.tile - (ntiles - p.gcut.gsplit)) + static_cast<int>(pr);
        seen = flag_wait(cnt, kGpEpiWarps, &s.abort);
        if (seen) {
          __threadfence();
          *cnt = 0;  // ready for the next call
        }
      }
      if (!__shfl_sync(0xFFFFFFFFu, seen ? 1 : 0, 0)) return;
    }
    for (int gb = u.g0; gb < u.g1; gb += kGpSlice) {
      if (!mbar_wait(smem_addr(&s.aux_empty[buf]), phase ^ 1u, &s.abort)) return;
      // the lane's four columns at once (32 values in flight)
      float v[4][kGpSlice];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int col = col0 + c;
        const float* src = p.sw + static_cast<int64_t>(col) * p.groups + gb;
        if (vec_rows && (gb & 3) == 0 && col < p.n && gb + kGpSlice <= u.g1) {
#pragma unroll
          for (int q = 0; q < kGpSlice / 4; ++q) {
            const float4 t = __ldg(reinterpret_cast<const float4*>(src) + q);
            v[c][4 * q] = t.x;
            v[c][4 * q + 1] = t.y;
            v[c][4 * q + 2] = t.z;
            v[c][4 * q + 3] = t.w;
          }
        } else {
#pragma unroll
          for (int gg = 0; gg < kGpSlice; ++gg)
            v[c][gg] = (col < p.n && gb + gg < u.g1) ? __ldg(src + gg) : 0.0f;
        }
      }
      float* dst = s.scales[buf] + c_lo;
#pragma unroll
      for (int gg = 0; gg < kGpSlice; ++gg)
        *reinterpret_cast<float4*>(dst + gg * kGpBN) = make_float4(v[0][gg], v[1][gg], v[2][gg], v[3][gg]);
      mbar_arrive(smem_addr(&s.aux_full[buf]));  // release: this lane's stores
      if (++buf == 2) {
        buf = 0;
        phase ^= 1u;
      }
    }
  }
}

// Register order barrier: values loaded by tcgen05.ld are used only after the
// tcgen05.wait::ld that precedes this point.
__device__ __forceinline__ void after_ld_wait(uint32_t (&v)[16]) {
  asm volatile(""
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                 "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                 "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]));
}

// f[j] = fma((float)P[j], sw[j], f[j]) for the 16 columns of one TMEM chunk:
// the conversions are exact (|P| < 2^24); the scales of four columns come in
// one broadcast 16-byte shared load.  (Running sums kept as packed binary32
// pairs for fma.rn.f32x2 measured slower, 197 against 181 us at 2048 x 8192
// x 8192: forming the pairs from the conversions costs register moves.)
__device__ __forceinline__ void gp_fold16(float* f, const uint32_t (&v)[16], uint32_t sc) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float4 s4;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(s4.x), "=f"(s4.y), "=f"(s4.z), "=f"(s4.w)
                 : "r"(sc + q * 16));
    f[4 * q + 0] = __fmaf_rn(__int2float_rn(static_cast<int>(v[4 * q + 0])), s4.x, f[4 * q + 0]);
    f[4 * q + 1] = __fmaf_rn(__int2float_rn(static_cast<int>(v[4 * q + 1])), s4.y, f[4 * q + 1]);
    f[4 * q + 2] = __fmaf_rn(__int2float_rn(static_cast<int>(v[4 * q + 2])), s4.z, f[4 * q + 2]);
    f[4 * q + 3] = __fmaf_rn(__int2float_rn(static_cast<int>(v[4 * q + 3])), s4.w, f[4 * q + 3]);
  }
}

__device__ void gp_epilogue(GroupPairStorage& s, uint32_t tmem, const Args& p, const CUtensorMap* tmO,
                            uint32_t pr, uint32_t lead) {
  const int np = gridDim.x >> 1, pi = blockIdx.x >> 1;
  const int ntiles = p.tiles_m * p.tiles_n;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int quad = warp & 3;
  const int ew = warp - 4;      // 0 .. 7
  const int half = ew >> 2;     // column half of the tile
  uint32_t abuf = 0, aphase = 0, sbuf = 0, sphase = 0;
  bool ok = true;
  GroupUnit u;
  for (int i = 0; ok && gp_unit(p, pi, np, i, u); ++i) {
    const int tm = u.tile % p.tiles_m, tn = u.tile / p.tiles_m;
    float f[kGpCols];
#pragma unroll
    for (int j = 0; j < kGpCols; ++j) f[j] = 0.0f;
    for (int g = u.g0; g < u.g1; ++g) {
      const int gs = (g - u.g0) % kGpSlice;
      if (gs == 0 && !mbar_wait(smem_addr(&s.aux_full[sbuf]), sphase, &s.abort)) {
        ok = false;
        break;
      }
      if (u.part == 2 && g == u.g0) {
        // continue from the first part's sums (another pair's; the stager saw
        // them complete before publishing this slice)
        const uint64_t* st = gp_state(p, u.tile - (ntiles - p.gcut.gsplit), static_cast<int>(pr), ew) + lane;
#pragma unroll
        for (int j = 0; j < kGpCols / 2; ++j) {
          const unsigned long long w = __ldcg(reinterpret_cast<const unsigned long long*>(st + j * 32));
          f[2 * j] = lo_of(w);
          f[2 * j + 1] = hi_of(w);
        }
      }
      if (!mbar_wait_poll(smem_addr(&s.acc_full[abuf]), aphase, &s.abort, 20)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem + (static_cast<uint32_t>(quad * 32) << 16) + abuf * kGpBN +
                          half * kGpCols;
      const uint32_t sc = smem_addr(s.scales[sbuf] + gs * kGpBN + half * kGpCols);
      uint32_t va[16], vb[16];
      tmem_ld_32x32b_x16(tb, va);
      tmem_ld_wait();
      after_ld_wait(va);
#pragma unroll
      for (int c = 0; c < kGpCols / 16; c += 2) {
        tmem_ld_32x32b_x16(tb + (c + 1) * 16, vb);
        gp_fold16(f + c * 16, va, sc + c * 64);
        tmem_ld_wait();
        after_ld_wait(vb);
        if (c + 2 < kGpCols / 16) {
          tmem_ld_32x32b_x16(tb + (c + 2) * 16, va);
        } else {
          // every chunk of this warp is in registers: hand the buffer back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(map_to_rank(smem_addr(&s.acc_empty[abuf]), lead));
        }
        gp_fold16(f + (c + 1) * 16, vb, sc + (c + 1) * 64);
        if (c + 2 < kGpCols / 16) {
          tmem_ld_wait();
          after_ld_wait(va);
        }
      }
      if (++abuf == 2) {
        abuf = 0;
        aphase ^= 1u;
      }
      if (gs == kGpSlice - 1 || g + 1 == u.g1) {
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
      // hand the running sums to the pair that finishes the tile
      const int tt = u.tile - (ntiles - p.gcut.gsplit);
      uint64_t* st = gp_state(p, tt, static_cast<int>(pr), ew) + lane;
#pragma unroll
      for (int j = 0; j < kGpCols / 2; ++j)
        __stcg(reinterpret_cast<unsigned long long*>(st + j * 32),
               pack2(__float_as_uint(f[2 * j]), __float_as_uint(f[2 * j + 1])));
      __threadfence();
      __syncwarp();
      if (lane == 0) atomicAdd(p.gcut.gflag + 2 * tt + static_cast<int>(pr), 1);
      continue;
    }
    const int row0 = tm * 256 + static_cast<int>(pr) * 128 + quad * 32;
    const int row = row0 + lane;
    const int colbase = tn * kGpBN + half * kGpCols;
    const float sa = row < p.m ? __ldg(p.sa + row) : 0.0f;
    const uint64_t sa2 = pack2(__float_as_uint(sa), __float_as_uint(sa));
    const uint64_t al2 = pack2(__float_as_uint(p.alpha), __float_as_uint(p.alpha));
    if (p.tma_out) {
      // bf16: 32 x 32 boxes through this warp's shared-memory slot and TMA
      // bulk tensor stores (clipped to the output's bounds)
      if (row0 >= p.m) continue;  // warp-uniform
      uint8_t* box = s.out_stage[ew];
      const uint32_t rowaddr = smem_addr(box) + static_cast<uint32_t>(lane) * 64u;
      const uint32_t sx = (static_cast<uint32_t>(lane) >> 1) & 3u;
#pragma unroll
      for (int b = 0; b < kGpCols / 32; ++b) {
        if (colbase + b * 32 >= p.n) break;
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const uint64_t r2 = f32x2_mul(
              f32x2_mul(pack2(__float_as_uint(f[b * 32 + 2 * e]), __float_as_uint(f[b * 32 + 2 * e + 1])), sa2),
              al2);
          w[e] = pack_bf16x2(lo_of(r2), hi_of(r2));
        }
        if (lane == 0) bulk_wait_read_all();  // the previous box has been read
        __syncwarp();
#pragma unroll
        for (uint32_t j = 0; j < 4; ++j)
          st_shared_v4(rowaddr + ((j ^ sx) << 4), w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(tmO, smem_addr(box), colbase + b * 32, row0);
          bulk_commit();
        }
      }
      continue;
    }
    if (row < p.m) {
#pragma unroll
      for (int g8 = 0; g8 < kGpCols / 8; ++g8) {
        const int col = colbase + g8 * 8;
        if (col >= p.n) break;
        const int64_t o = static_cast<int64_t>(row) * p.n + col;
        uint64_t r2[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          r2[e] = f32x2_mul(f32x2_mul(pack2(__float_as_uint(f[g8 * 8 + 2 * e]), __float_as_uint(f[g8 * 8 + 2 * e + 1])), sa2), al2);
        if (p.out_bf16) {
          uint4 pk;
          pk.x = pack_bf16x2(lo_of(r2[0]), hi_of(r2[0]));
          pk.y = pack_bf16x2(lo_of(r2[1]), hi_of(r2[1]));
          pk.z = pack_bf16x2(lo_of(r2[2]), hi_of(r2[2]));
          pk.w = pack_bf16x2(lo_of(r2[3]), hi_of(r2[3]));
          *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + o) = pk;
        } else {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + o);
          dst[0] = make_float4(lo_of(r2[0]), hi_of(r2[0]), lo_of(r2[1]), hi_of(r2[1]));
          dst[1] = make_float4(lo_of(r2[2]), hi_of(r2[2]), lo_of(r2[3]), hi_of(r2[3]));
        }
      }
    }
  }
  if (p.tma_out && lane == 0) bulk_wait_all();  // the output stores are complete
  __syncwarp();
}

__global__ void __launch_bounds__(kGpThreads, 1)
    gemm_i8_group_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                              const __grid_constant__ CUtensorMap tmB,
                              const __grid_constant__ CUtensorMap tmO, const Args p) {
  extern __shared__ uint8_t smem_raw[];
  GroupPairStorage& s = storage<GroupPairStorage>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_rank();
  const uint32_t pr = crank & 1u, lead = crank & ~1u;
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (p.tma_out) prefetch_tmap(&tmO);
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGpStages; ++i) {
      mbar_init(smem_addr(&s.full[i]), 1);
      mbar_init(smem_addr(&s.empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_addr(&s.acc_full[i]), 1);
      mbar_init(smem_addr(&s.acc_empty[i]), 2 * kGpEpiWarps);  // epilogue warps of both CTAs
      mbar_init(smem_addr(&s.aux_full[i]), 64);                // both stager warps' lanes
      mbar_init(smem_addr(&s.aux_empty[i]), kGpEpiWarps);
    }
    mbar_init(smem_addr(&s.drain), 1);
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_addr(&s.tmem_base), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers exist before anyone signals them
  tc_fence_after();
  griddep_wait();  // set-up above overlapped the previous kernel
  griddep_launch_dependents();
  const uint32_t tmem = s.tmem_base;
  if (warp < 4) {
    regs_dec<kGpCtrlRegs>();
    if (warp == 0) {
      if (lane == 0) gp_produce(s, &tmA, &tmB, p, pr, lead);
      __syncwarp();
    } else if (warp == 1) {
      if (lane == 0 && pr == 0) gp_mma(s, tmem, p, lead);
      __syncwarp();
    } else {
      gp_stage_scales(s, p, pr);
    }
  } else {
    regs_inc<kGpEpiRegs>();
    gp_epilogue(s, tmem, p, &tmO, pr, lead);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the leader's MMAs on this CTA's smem / TMEM are done
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
}

}  // namespace gemm
}  // namespace qk
