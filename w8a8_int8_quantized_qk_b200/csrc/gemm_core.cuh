// gemm_core.cuh -- the pieces the tcgen05 GEMM kernels share: the argument
// block, tile maps and work units, shared-memory storage, the TMA producer
// and MMA issuer roles, and the epilogue stores (per channel and per
// group).  The kernels are in gemm_1sm.cuh and gemm_pair.cuh, the host-side
// planning and launches in gemm_host.cuh; gemm_sm100.cuh includes them all.
#pragma once

#include <atomic>
#include <mutex>

#include "group_plan.h"
#include "qk_common.cuh"

namespace qk {
namespace gemm {


constexpr int BM = 128;
constexpr int BK = 128;     // K bytes per stage: one 128-byte swizzle row
constexpr int UMMA_K = 32;  // K of one kind::i8 MMA instruction
constexpr int kTmemCols = 512;

// Args: the problem and its output form, which every GEMM kernel reads,
// then one group of fields per mode.  A mode's group is all zero when the
// mode is off; each kernel reads only the groups of the modes it has.
//
// split-K of a tile's K range (pair and 1-SM per-channel kernels): each
// tile's K blocks are cut into `splits` slices of `kb_per_split`.  The
// partial sums meet in the workspace `ws`, with per-region arrival counters
// in the header (`cnt`: zero before the call, zero again after it), or,
// when `csplit` is 1, in distributed shared memory: the slices are the CTAs
// (pairs) of one cluster, and no workspace is needed.
struct SplitK {
  int splits, kb_per_split;
  int32_t* ws;
  int csplit;
};

// Tail split of a partial last wave (pair kernel; tail_splits > 1 and
// splits == 1).  Tiles [0, dp_tiles) are computed whole.  Each remaining
// tile is cut into `tail_splits` K slices of `tail_kbps` K blocks, and those
// slices are the first unit of pairs 0 .. (tiles - dp_tiles) * tail_splits -
// 1.  Every slice stores its partial in `tail_ws` and counts itself in
// `cnt`.  The slice that arrives last adds the others' partials to its own,
// runs the epilogue and leaves the counter zero (the partials are scratch).
struct TailSplit {
  int dp_tiles, tail_splits, tail_kbps;
  int32_t* tail_ws;
};

// Asymmetric activations (per channel only): zp [m] zero-points and wsum [n]
// = sum_k b[n][k]; the epilogues use acc - zp[m] * wsum[n].
struct ZeroPoints {
  const int32_t* zp;
  const int32_t* wsum;
};

// MoE grouped GEMM (1-SM kernel).  Tokens are grouped by expert: expert e's
// rows are [moe_off[e], moe_off[e + 1]) of a (m rows in all).  b is
// [experts * n, k] and sw [experts, n].  tiles_m = experts * mt_max M tiles,
// and those past an expert's tokens are skipped.
struct MoeTiles {
  int mt_max;
  const int32_t* moe_off;
};

// The group-128 kernels' last wave, cut along K (gsplit > 0).  Tiles
// [0, tiles - gsplit) run whole.  Tail tile (tiles - gsplit + j) is cut at
// group gmid:
// - its first part is worker j's first unit, which leaves its fp32 running
//   sums in gstate and counts itself in gflag;
// - its second part is worker (gsplit + j)'s last unit, which waits for the
//   count, continues the sums in the same group order and leaves the count
//   zero.
struct GroupCut {
  int gsplit, gmid;
  float* gstate;
  int* gflag;
};

struct Args {
  int m, n, k;
  const float* sa;  // [m]
  const float* sw;  // [n] or [n, groups]
  float alpha;
  int32_t* c;       // [m, n] or null
  void* out;        // [m, n] or null
  int out_bf16;
  int tiles_m, tiles_n, num_kb, groups;
  // 1 when bf16 `out` (and no `c`) is written by TMA bulk tensor stores
  // from shared memory (tensor map tmO)
  int tma_out;
  // 1: a and b are float8 e4m3 codes, the MMA is kind::f8f6f4 and the
  // accumulator fp32 (channel and pair kernels, whole tiles or the cluster
  // split-K, no c)
  int f8;
  int* cnt;  // the workspace's arrival counters (split-K and tail split)
  SplitK sk;
  TailSplit tail;
  ZeroPoints asym;
  MoeTiles moe;
  GroupCut gcut;
};

// The i-th unit of this CTA in the wide group kernel's schedule (false past
// its last); every role walks the same list (group_plan.h).
__device__ __forceinline__ bool group_unit(const Args& p, int i, GroupUnit& u) {
  return group_unit_at(static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x),
                       p.tiles_m * p.tiles_n, p.gcut.gsplit, p.groups, p.gcut.gmid, i, u);
}

// One output tile of the 1-SM kernels: A rows from a_row0 (rows from row_end
// on belong to another expert, or to none, and are masked), B rows from
// b_row0, output columns from col0, channel scales from sw.  False for an
// empty MoE tile; every role skips the same tiles.
struct ChanTile {
  int a_row0, b_row0, col0, row_end;
  const float* sw;
};

template <int BN, bool MOE>
__device__ __forceinline__ bool chan_tile(const Args& p, int tile, ChanTile& t) {
  if constexpr (MOE) {
    // compact numbering of the non-empty tiles: expert by expert, M tiles
    // fastest; tile numbers past the last one are empty
    const int experts = p.tiles_m / p.moe.mt_max;
    int u = tile;
    for (int e = 0; e < experts; ++e) {
      const int r0 = __ldg(p.moe.moe_off + e), r1 = __ldg(p.moe.moe_off + e + 1);
      int mt = r1 > r0 ? (r1 - r0 + BM - 1) / BM : 0;
      mt = mt < p.moe.mt_max ? mt : p.moe.mt_max;
      const int cnt = mt * p.tiles_n;
      if (u < cnt) {
        const int tm = u % mt, tn = u / mt;
        t.a_row0 = r0 + tm * BM;
        t.row_end = r1 < p.m ? r1 : p.m;
        t.b_row0 = e * p.n + tn * BN;
        t.col0 = tn * BN;
        t.sw = p.sw + static_cast<int64_t>(e) * p.n;
        return true;
      }
      u -= cnt;
    }
    return false;
  } else {
    const int tmg = tile % p.tiles_m, tn = tile / p.tiles_m;
    t.a_row0 = tmg * BM;
    t.row_end = p.m;
    t.b_row0 = tn * BN;
    t.col0 = tn * BN;
    t.sw = p.sw;
  }
  return true;
}

template <int BN, int STAGES, int NACC, int SCALE_FLOATS>
struct alignas(1024) Storage {
  uint8_t a[STAGES][BM * BK];
  uint8_t b[STAGES][BN * BK];
  float scales[SCALE_FLOATS > 0 ? SCALE_FLOATS : 1];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full[NACC];
  uint64_t acc_empty[NACC];
  uint64_t aux_full[2];   // group kernel: scale slice staged
  uint64_t aux_empty[2];  // group kernel: scale slice consumed
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Warp-uniform bounded wait: lane 0 polls (so a waiting warp does not flood
// the shared-memory pipe the tensor core reads its operands through), then
// every lane confirms the completed phase once for itself; the warp
// proceeds only if all lanes saw it complete.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort);
  ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
  if (ok) ok = mbar_wait(bar, parity, abort);
  const bool all = __all_sync(0xFFFFFFFFu, ok);
  if (!all) *abort = 1;
  return all;
}

// ---------------------------------------------------------------- producer
// GUNITS: the wide group kernel's unit list (group_unit); otherwise units
// blockIdx.x, + gridDim.x, ... of tiles x splits.
//
// Programmatic dependent launch: the producer waits for the previous kernel
// in the stream itself (the other roles wait at kernel entry).  EARLY_B: it
// first requests the weight (B) tiles of its first unit's first STAGES K
// blocks -- the weights are never written by the kernel that precedes a GEMM
// (the quantiser) -- and only after the wait the activation (A) tiles, which
// the quantiser writes.  That overlaps the start of the weight stream with a
// quantiser that leaves DRAM idle (the fused SiLU form before the 1-SM
// per-channel kernel: 30.4 -> 29.1 us per mlp_down step); behind the
// DRAM-bound plain quantiser the early loads only delay it (measured on the
// CTA-pair prefill and the decode GEMV), so the other kernels wait first.
template <int BN, int STAGES, bool MOE = false, bool GUNITS = false, bool EARLY_B = false, class S>
__device__ void produce(S& s, const CUtensorMap* tmA, const CUtensorMap* tmB, const Args& p) {
  const int nunits = p.tiles_m * p.tiles_n * p.sk.splits;
  const uint32_t bytes = static_cast<uint32_t>((BM + BN) * BK);
  uint32_t stage = 0, phase = 0, issued = 0;
  bool ok = true;
  bool waited = !EARLY_B;
  if constexpr (!EARLY_B) {
    griddep_wait();
    griddep_launch_dependents();
  }
  int pre_n = 0, pre_kb0 = 0, pre_row = 0;  // A tiles deferred past griddep_wait
  auto release_deferred = [&]() {
    griddep_wait();
    griddep_launch_dependents();
    for (int j = 0; j < pre_n; ++j)
      tma_load_2d(smem_addr(s.a[j]), tmA, smem_addr(&s.full[j]), (pre_kb0 + j) * BK, pre_row);
    waited = true;
  };
  for (int i = 0; ok; ++i) {
    ChanTile t;
    int kb0, kb1;
    if constexpr (GUNITS) {
      GroupUnit gu;
      if (!group_unit(p, i, gu)) break;
      t.a_row0 = (gu.tile % p.tiles_m) * BM;
      t.b_row0 = (gu.tile / p.tiles_m) * BN;
      kb0 = gu.g0;
      kb1 = gu.g1;
    } else {
      const int unit = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
      if (unit >= nunits) break;
      if (!chan_tile<BN, MOE>(p, unit / p.sk.splits, t)) continue;
      kb0 = (unit % p.sk.splits) * p.sk.kb_per_split;
      kb1 = min(p.num_kb, kb0 + p.sk.kb_per_split);
    }
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!waited && (pre_n == STAGES || (pre_n > 0 && kb != pre_kb0 + pre_n))) release_deferred();
      if (!mbar_wait(smem_addr(&s.empty[stage]), phase ^ 1u, &s.abort)) {
        ok = false;
        break;
      }
      const uint32_t fb = smem_addr(&s.full[stage]);
      mbar_arrive_expect_tx(fb, bytes);
      tma_load_2d(smem_addr(s.b[stage]), tmB, fb, kb * BK, t.b_row0);
      if (waited) {
        tma_load_2d(smem_addr(s.a[stage]), tmA, fb, kb * BK, t.a_row0);
      } else {
        if (pre_n == 0) {
          pre_kb0 = kb;
          pre_row = t.a_row0;
        }
        ++pre_n;
      }
      ++issued;
      if (++stage == STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  if (!waited) release_deferred();
  // No copy may still be landing in shared memory when the CTA exits: wait
  // (bounded, ignoring the abort flag) for the last STAGES copies issued.
  const uint32_t first = issued > STAGES ? issued - STAGES : 0u;
  for (uint32_t i = first; i < issued; ++i)
    mbar_wait(smem_addr(&s.full[i % STAGES]), (i / STAGES) & 1u, nullptr);
}

// ---------------------------------------------------------------- MMA issuer
// GROUP: one accumulator buffer per K block (each K block is one group);
// otherwise one buffer per tile.
template <int BN, int STAGES, int NACC, bool GROUP, bool F8 = false, bool MOE = false,
          bool GUNITS = false, class S>
__device__ void mma_issue(S& s, uint32_t tmem, const Args& p) {
  const int nunits = p.tiles_m * p.tiles_n * p.sk.splits;
  constexpr uint32_t idesc = F8 ? idesc_e4m3(BM, BN) : idesc_i8(BM, BN);
  uint32_t stage = 0, phase = 0, abuf = 0, aphase = 0;
  bool ok = true;
  for (int i = 0; ok; ++i) {
    int kb0, kb1;
    if constexpr (GUNITS) {
      GroupUnit gu;
      if (!group_unit(p, i, gu)) break;
      kb0 = gu.g0;
      kb1 = gu.g1;
    } else {
      const int unit = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
      if (unit >= nunits) break;
      if constexpr (MOE) {
        ChanTile t;
        if (!chan_tile<BN, true>(p, unit, t)) continue;
      }
      kb0 = (unit % p.sk.splits) * p.sk.kb_per_split;
      kb1 = min(p.num_kb, kb0 + p.sk.kb_per_split);
    }
    if (!GROUP) {
      if (!mbar_wait(smem_addr(&s.acc_empty[abuf]), aphase ^ 1u, &s.abort)) break;
      tc_fence_after();
    }
    for (int kb = kb0; kb < kb1; ++kb) {
      if (GROUP) {
        if (!mbar_wait(smem_addr(&s.acc_empty[abuf]), aphase ^ 1u, &s.abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      if (!mbar_wait(smem_addr(&s.full[stage]), phase, &s.abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem + abuf * BN;
      const uint32_t a0 = smem_addr(s.a[stage]);
      const uint32_t b0 = smem_addr(s.b[stage]);
#pragma unroll
      for (int kk = 0; kk < BK / UMMA_K; ++kk) {
        const uint32_t acc = GROUP ? (kk > 0) : (kb > kb0 || kk > 0);
        if constexpr (F8)
          mma_e4m3(d, sdesc_k_sw128(a0 + kk * UMMA_K), sdesc_k_sw128(b0 + kk * UMMA_K), idesc, acc);
        else
          mma_i8(d, sdesc_k_sw128(a0 + kk * UMMA_K), sdesc_k_sw128(b0 + kk * UMMA_K), idesc, acc);
      }
      mma_commit(smem_addr(&s.empty[stage]));
      if (++stage == STAGES) {
        stage = 0;
        phase ^= 1u;
      }
      if (GROUP) {
        mma_commit(smem_addr(&s.acc_full[abuf]));
        if (++abuf == NACC) {
          abuf = 0;
          aphase ^= 1u;
        }
      }
    }
    if (!GROUP && ok) {
      mma_commit(smem_addr(&s.acc_full[abuf]));
      if (++abuf == NACC) {
        abuf = 0;
        aphase ^= 1u;
      }
    }
  }
  // Every MMA issued must be complete before the TMEM can be released.
  mma_commit(smem_addr(&s.drain));
  mbar_wait(smem_addr(&s.drain), 0u, nullptr);
}

// ---------------------------------------------------------------- epilogues
// 8 consecutive outputs (row, col .. col+7) from 8 int32 accumulators.
__device__ __forceinline__ void store8_channel(const Args& p, int row, int col, float sa,
                                               const uint32_t* v) {
  const int64_t o = static_cast<int64_t>(row) * p.n + col;
  if (p.c) {
    int4* dst = reinterpret_cast<int4*>(p.c + o);
    dst[0] = make_int4(v[0], v[1], v[2], v[3]);
    dst[1] = make_int4(v[4], v[5], v[6], v[7]);
  }
  if (p.out) {
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(p.sw + col));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(p.sw + col + 4));
    const float sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    float f[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float t = __int2float_rn(static_cast<int>(v[j]));
      t = __fmul_rn(t, sa);
      t = __fmul_rn(t, sw[j]);
      f[j] = __fmul_rn(t, p.alpha);
    }
    if (p.out_bf16) {
      uint4 pk;
      pk.x = pack_bf16x2(f[0], f[1]);
      pk.y = pack_bf16x2(f[2], f[3]);
      pk.z = pack_bf16x2(f[4], f[5]);
      pk.w = pack_bf16x2(f[6], f[7]);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + o) = pk;
    } else {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + o);
      dst[0] = make_float4(f[0], f[1], f[2], f[3]);
      dst[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
  }
}

// bf16 output staging of one epilogue warp: a 32-row x 32-column box
// (64 bytes a row) for one TMA store
constexpr int kOutBoxBytes = 32 * 32 * 2;

// The accumulator's value as binary32: an int32 sum converted (exact below
// 2^24, round-to-nearest above), or, for the FP8 kind, the fp32 sum itself.
template <bool F8>
__device__ __forceinline__ float acc_value(uint32_t v) {
  if constexpr (F8) return __uint_as_float(v);
  return __int2float_rn(static_cast<int>(v));
}

// Sum of two split-K partials: int32 (exact in any order) for the INT8 kind;
// for the FP8 kind binary32, rounded to nearest.  The reductions add the
// slices in ascending slice order, so that an FP8 result does not depend on
// which CTA finishes first.
template <bool F8>
__device__ __forceinline__ uint32_t acc_add(uint32_t x, uint32_t y) {
  if constexpr (F8) return __float_as_uint(__fadd_rn(__uint_as_float(x), __uint_as_float(y)));
  return x + y;
}
template <bool F8>
__device__ __forceinline__ void acc_add4(uint32_t* v, const int4& t) {
  v[0] = acc_add<F8>(v[0], static_cast<uint32_t>(t.x));
  v[1] = acc_add<F8>(v[1], static_cast<uint32_t>(t.y));
  v[2] = acc_add<F8>(v[2], static_cast<uint32_t>(t.z));
  v[3] = acc_add<F8>(v[3], static_cast<uint32_t>(t.w));
}

// Zero-point correction of 32 int32 accumulators of one row (columns col0 ..
// col0 + 31): v -= zp[row] * wsum[col], in two's-complement arithmetic
// (exact whenever the corrected sum fits in int32, which the host's bound
// on k guarantees).  Rows >= m and columns >= n (n % 8 == 0) take 0.
__device__ __forceinline__ void apply_zp(const Args& p, int row, int col0, uint32_t (&v)[32]) {
  const uint32_t z = row < p.m ? static_cast<uint32_t>(__ldg(p.asym.zp + row)) : 0u;
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    const int col = col0 + g * 4;
    const int4 w4 = col < p.n ? __ldg(reinterpret_cast<const int4*>(p.asym.wsum + col))
                              : make_int4(0, 0, 0, 0);
    v[g * 4 + 0] -= z * static_cast<uint32_t>(w4.x);
    v[g * 4 + 1] -= z * static_cast<uint32_t>(w4.y);
    v[g * 4 + 2] -= z * static_cast<uint32_t>(w4.z);
    v[g * 4 + 3] -= z * static_cast<uint32_t>(w4.w);
  }
}

// 32 outputs of one row (columns col0 .. col0 + 31) from 32 accumulators;
// channel scales come from shared memory.
template <bool F8 = false>
__device__ __forceinline__ void store32_channel(const Args& p, int row, int col0, float sa,
                                                const float* sw, const uint32_t (&v)[32]) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int col = col0 + g * 8;
    if (col >= p.n) break;
    const int64_t o = static_cast<int64_t>(row) * p.n + col;
    if (!F8 && p.c) {
      int4* dst = reinterpret_cast<int4*>(p.c + o);
      dst[0] = make_int4(v[g * 8 + 0], v[g * 8 + 1], v[g * 8 + 2], v[g * 8 + 3]);
      dst[1] = make_int4(v[g * 8 + 4], v[g * 8 + 5], v[g * 8 + 6], v[g * 8 + 7]);
    }
    if (p.out) {
      const float4 s0 = *reinterpret_cast<const float4*>(sw + g * 8);
      const float4 s1 = *reinterpret_cast<const float4*>(sw + g * 8 + 4);
      const float s8[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      float f[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float t = acc_value<F8>(v[g * 8 + j]);
        t = __fmul_rn(t, sa);
        t = __fmul_rn(t, s8[j]);
        f[j] = __fmul_rn(t, p.alpha);
      }
      if (p.out_bf16) {
        uint4 pk;
        pk.x = pack_bf16x2(f[0], f[1]);
        pk.y = pack_bf16x2(f[2], f[3]);
        pk.z = pack_bf16x2(f[4], f[5]);
        pk.w = pack_bf16x2(f[6], f[7]);
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + o) = pk;
      } else {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + o);
        dst[0] = make_float4(f[0], f[1], f[2], f[3]);
        dst[1] = make_float4(f[4], f[5], f[6], f[7]);
      }
    }
  }
}

// 32 bf16 outputs of one row (columns col0 .. col0 + 31), converted exactly
// as store32_channel does, written by the warp into its staging box (row r =
// lane at byte 64 r; 64-byte swizzle: 16-byte chunk j of row r sits at
// 64 r + 16 (j ^ ((r >> 1) & 3))) and stored with one TMA bulk tensor copy
// at (col0, row0), which clips rows >= m and columns >= n.  Lane 0 issues
// the copies; before rewriting the box it waits until the previous copy has
// read it.  Every lane of the warp must call this.
// The three multiplies run on binary32 pairs (mul.rn.f32x2: each lane an
// IEEE round-to-nearest multiply, so the values are those of the scalar
// form): half the FMA-pipe instructions, which compete with the tensor
// core's MMAs on the same SM (0.6 us of a 52 us prefill GEMM).  (Leaving
// out the exact multiply by an output_scale of 1 measured no faster.)
template <bool F8 = false>
__device__ __forceinline__ void store32_tma(const Args& p, const CUtensorMap* tmO, uint8_t* box,
                                            int row0, int col0, float sa, const float* sw,
                                            const uint32_t (&v)[32]) {
  if (col0 >= p.n || row0 >= p.m) return;  // the box lies wholly outside (warp-uniform)
  const int lane = threadIdx.x & 31;
  uint32_t w[16];
  const uint64_t sa2 = pack2(__float_as_uint(sa), __float_as_uint(sa));
  const uint64_t al2 = pack2(__float_as_uint(p.alpha), __float_as_uint(p.alpha));
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint64_t s2 = *reinterpret_cast<const unsigned long long*>(sw + 2 * j);
    uint64_t t;
    if constexpr (F8) {
      t = pack2(v[2 * j], v[2 * j + 1]);
    } else {
      asm("{\n\t.reg .f32 x, y;\n\tcvt.rn.f32.s32 x, %1;\n\tcvt.rn.f32.s32 y, %2;\n\tmov.b64 %0, {x, y};\n\t}"
          : "=l"(t) : "r"(v[2 * j]), "r"(v[2 * j + 1]));
    }
    t = f32x2_mul(f32x2_mul(f32x2_mul(t, sa2), s2), al2);
    w[j] = pack_bf16x2(lo_of(t), hi_of(t));
  }
  if (lane == 0) bulk_wait_read_all();
  __syncwarp();
  const uint32_t rowaddr = smem_addr(box) + static_cast<uint32_t>(lane) * 64u;
  const uint32_t sx = (static_cast<uint32_t>(lane) >> 1) & 3u;
#pragma unroll
  for (uint32_t j = 0; j < 4; ++j)
    st_shared_v4(rowaddr + ((j ^ sx) << 4), w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tmO, smem_addr(box), col0, row0);
    bulk_commit();
  }
}

// Per-channel epilogue, 4 warps; warp w owns TMEM lanes 32*(w%4) (rows)
// and all BN columns of the tile.  Before the accumulator is ready the warp
// stages the tile's channel scales in its shared-memory slot and fetches its
// row's token scale; the 32-column TMEM loads are double-buffered so the
// next load is in flight while the current chunk is converted and stored.
// bf16 output without c leaves through TMA stores (store32_tma).
template <int BN, int NACC, bool F8 = false, bool MOE = false, class S>
__device__ void epilogue_channel(S& s, uint32_t tmem, const Args& p, const CUtensorMap* tmO) {
  const int nunits = p.tiles_m * p.tiles_n * p.sk.splits;
  const int lane = threadIdx.x & 31;
  const int ew = (threadIdx.x >> 5) - 2;  // epilogue warp 0..3
  const int quad = (threadIdx.x >> 5) & 3;
  float* sws = s.sw_tile[ew];
  uint8_t* box = s.out_stage[ew];
  uint32_t abuf = 0, aphase = 0;
  for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x) {
    ChanTile t;
    if (!chan_tile<BN, MOE>(p, unit / p.sk.splits, t)) continue;
    const int row0 = t.a_row0 + quad * 32, row = row0 + lane;
    const bool rv = row >= 0 && row < t.row_end;
    const float sa = (rv && p.out) ? __ldg(p.sa + row) : 0.0f;
    const int colbase = t.col0;
    if (p.out) {
#pragma unroll
      for (int c4 = lane * 4; c4 < BN; c4 += 128) {  // n % 8 == 0: a group of 4 is all in or out
        const int col = colbase + c4;
        *reinterpret_cast<float4*>(sws + c4) =
            col < p.n ? __ldg(reinterpret_cast<const float4*>(t.sw + col))
                      : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      }
    }
    __syncwarp();
    if (!warp_wait(smem_addr(&s.acc_full[abuf]), aphase, &s.abort)) break;
    tc_fence_after();
    const uint32_t tb = tmem + (static_cast<uint32_t>(quad * 32) << 16) + abuf * BN;
    uint32_t va[32], vb[32];
    if (p.sk.csplit) {
      // Split-K inside the cluster (one unit per CTA, so the operand ring is
      // idle once acc_full has fired): stage this warp's 32 x BN partial in
      // its slot of the ring (32 KB at BN = 256), laid out
      // [chunk][column quad][lane][4];
      // channel_cluster_reduce sums the slots over the cluster after a
      // cluster barrier.
      uint8_t* stg = &s.a[0][0] + quad * (32 * BN * 4);
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        tmem_ld_32x32b_x32(tb + ch * 32, va);
        tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          *reinterpret_cast<int4*>(stg + (((ch * 8 + q4) * 32 + lane) * 16)) =
              make_int4(va[q4 * 4], va[q4 * 4 + 1], va[q4 * 4 + 2], va[q4 * 4 + 3]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&s.acc_empty[abuf]));
      break;  // one unit per CTA
    }
    auto emit = [&](int ch, uint32_t(&v)[32]) {
      if constexpr (F8) {
        if (p.tma_out)
          store32_tma<true>(p, tmO, box, row0, colbase + ch * 32, sa, sws + ch * 32, v);
        else if (rv)
          store32_channel<true>(p, row, colbase + ch * 32, sa, sws + ch * 32, v);
      } else {
        if (p.asym.zp) apply_zp(p, row, colbase + ch * 32, v);
        if (p.tma_out)
          store32_tma(p, tmO, box, row0, colbase + ch * 32, sa, sws + ch * 32, v);
        else if (rv)
          store32_channel(p, row, colbase + ch * 32, sa, sws + ch * 32, v);
      }
    };
    tmem_ld_32x32b_x32(tb, va);
    tmem_ld_wait();
#pragma unroll 1
    for (int ch = 0; ch < BN / 32; ch += 2) {
      tmem_ld_32x32b_x32(tb + (ch + 1) * 32, vb);
      emit(ch, va);
      tmem_ld_wait();
      if (ch + 2 < BN / 32) tmem_ld_32x32b_x32(tb + (ch + 2) * 32, va);
      emit(ch + 1, vb);
      tmem_ld_wait();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&s.acc_empty[abuf]));
    if (++abuf == NACC) {
      abuf = 0;
      aphase ^= 1u;
    }
  }
  if (p.tma_out && lane == 0) bulk_wait_all();  // the output stores are complete
  __syncwarp();
}

// Per-group epilogue.  Warp roles of the group kernel: 0 TMA producer, 1 MMA
// issuer, then E epilogue warps, then one scale stager.  Epilogue warp w owns
// TMEM lanes 32*(w%4) and columns [C*h, C*h + C) of the 128-column tile,
// h = (w - 2) / 4, C = 4 * 128 / E.
//
// The stager copies the weight scales of the tile's 128 columns for SG
// groups at a time from [n, groups] (global) into a shared slice laid out
// [group][column], double buffered: slice i is published on aux_full[i]
// (32 lane arrivals) and handed back on aux_empty[i] (one arrival per
// epilogue warp).  So the epilogue warps read their scales of a group as
// broadcast float4 loads and never wait on global memory.
//
// Accumulation per element, in ascending group order as the definition
// states: pf = (float)P_g (exact: |P_g| <= 128 * 127^2 < 2^24),
// f = fma(pf, sw[n, g], f).
constexpr int kScaleGroups = 16;

// Epilogue width of the group kernel: 16 warps of 32 columns (four per TMEM
// lane quadrant, so that more warps hide each one's waits), or 8 warps of 64
// columns when the int32 sums are also kept (64 more registers per thread;
// with 16 warps a thread has at most 96).
template <bool WITH_C>
struct GroupCfg {
  static constexpr int epi_warps = WITH_C ? 8 : 16;
  static constexpr int cols = 4 * 128 / epi_warps;  // columns per warp
  static constexpr int threads = 64 + epi_warps * 32 + 32;
};

// CH column chunks of 32 (CH x kScaleGroups loads) are in flight together;
// CH = BN / 32 makes the slice one memory round trip.
// A unit's groups [g0, g1) are staged in slices of kScaleGroups from g0 on
// (GUNITS: the wide kernel's unit list; otherwise whole tiles).
template <int BN, int CH, bool GUNITS, class S>
__device__ void stage_group_scales(S& s, const Args& p) {
  const int ntiles = p.tiles_m * p.tiles_n;
  const int lane = threadIdx.x & 31;
  uint32_t buf = 0, phase = 0;
  for (int i = 0;; ++i) {
    GroupUnit u;
    if constexpr (GUNITS) {
      if (!group_unit(p, i, u)) break;
    } else {
      u = {static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x), 0, p.groups, 0};
      if (u.tile >= ntiles) break;
    }
    const int col0 = (u.tile / p.tiles_m) * BN;
    const int batches = (u.g1 - u.g0 + kScaleGroups - 1) / kScaleGroups;
    if (GUNITS && u.part == 2) {
      // the first part's running sums (written by another CTA) must be
      // complete before this unit's first slice is published
      bool seen = true;
      if (lane == 0) {
        int* cnt = p.gcut.gflag + (u.tile - (ntiles - p.gcut.gsplit));
        seen = flag_wait(cnt, 16, &s.abort);
        if (seen) {
          __threadfence();
          *cnt = 0;  // ready for the next call
        }
      }
      if (!__shfl_sync(0xFFFFFFFFu, seen ? 1 : 0, 0)) return;
    }
    for (int b = 0; b < batches; ++b) {
      if (!warp_wait(smem_addr(&s.aux_empty[buf]), phase ^ 1u, &s.abort)) return;
      float* dst = s.scales + buf * (kScaleGroups * BN);
      const int gb = u.g0 + b * kScaleGroups;  // first group of the slice
#pragma unroll
      for (int i0 = 0; i0 < BN / 32; i0 += CH) {
        float v[CH][kScaleGroups];
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const int col = col0 + lane + 32 * (i0 + c);
          const float* src = p.sw + static_cast<int64_t>(col) * p.groups + gb;
#pragma unroll
          for (int gg = 0; gg < kScaleGroups; ++gg)
            v[c][gg] = (col < p.n && gb + gg < u.g1) ? __ldg(src + gg) : 0.0f;
        }
#pragma unroll
        for (int c = 0; c < CH; ++c)
#pragma unroll
          for (int gg = 0; gg < kScaleGroups; ++gg)
            dst[gg * BN + lane + 32 * (i0 + c)] = v[c][gg];
      }
      mbar_arrive(smem_addr(&s.aux_full[buf]));  // release: this lane's stores
      if (++buf == 2) {
        buf = 0;
        phase ^= 1u;
      }
    }
  }
}

// f[c] = fma((float)P[c], sw[c], f[c]) for the 32 columns C0 .. C0 + 31 of
// this warp's COLS, plus the int32 sums when NC == COLS.
template <int C0, int COLS, int NC>
__device__ __forceinline__ void group_fma32(float (&f)[COLS], int (&cs)[NC],
                                            const uint32_t (&v)[32], const float* sc) {
  const float4* sc4 = reinterpret_cast<const float4*>(sc + C0);
#pragma unroll
  for (int j4 = 0; j4 < 8; ++j4) {
    const float4 s4 = sc4[j4];
    const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = j4 * 4 + e;
      // |P| < 2^24: the conversion is exact
      const float pf = __int2float_rn(static_cast<int>(v[j]));
      f[C0 + j] = __fmaf_rn(pf, sv[e], f[C0 + j]);
      if constexpr (NC == COLS) cs[C0 + j] += static_cast<int>(v[j]);
    }
  }
}

// The warp is done reading accumulator buffer abuf: hand it back to the MMA.
template <int NACC, class S>
__device__ __forceinline__ void release_acc(S& s, uint32_t& abuf, uint32_t& aphase, int lane) {
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_addr(&s.acc_empty[abuf]));
  if (++abuf == NACC) {
    abuf = 0;
    aphase ^= 1u;
  }
}

template <int BN, int NACC, bool WITH_C, class S>
__device__ void epilogue_group(S& s, uint32_t tmem, const Args& p) {
  constexpr int COLS = GroupCfg<WITH_C>::cols;
  const int ntiles = p.tiles_m * p.tiles_n;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int quad = warp & 3;
  const int sub = (warp - 2) >> 2;  // column slice of the tile
  uint32_t abuf = 0, aphase = 0, sbuf = 0, sphase = 0;
  bool ok = true;
  for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
    const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
    const int colbase = tn * BN + sub * COLS;
    float f[COLS];
    int cs[WITH_C ? COLS : 1];
#pragma unroll
    for (int j = 0; j < COLS; ++j) f[j] = 0.0f;
    if constexpr (WITH_C) {
#pragma unroll
      for (int j = 0; j < COLS; ++j) cs[j] = 0;
    }
    for (int g = 0; g < p.groups; ++g) {
      const int gs = g % kScaleGroups;
      if (gs == 0 && !warp_wait(smem_addr(&s.aux_full[sbuf]), sphase, &s.abort)) {
        ok = false;
        break;
      }
      if (!warp_wait(smem_addr(&s.acc_full[abuf]), aphase, &s.abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem + (static_cast<uint32_t>(quad * 32) << 16) + abuf * BN +
                          sub * COLS;
      const float* sc = s.scales + sbuf * (kScaleGroups * BN) + gs * BN + sub * COLS;
      if constexpr (COLS == 64) {
        // 8 warps of 64 columns (the int32-sum form): two loads of 32 so
        // that the sums and the accumulators stay in registers
        uint32_t v[32];
        tmem_ld_32x32b_x32(tb, v);
        tmem_ld_wait();
        group_fma32<0, COLS>(f, cs, v, sc);
        tmem_ld_32x32b_x32(tb + 32, v);
        tmem_ld_wait();
        release_acc<NACC>(s, abuf, aphase, lane);
        group_fma32<32, COLS>(f, cs, v, sc);
      } else {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tb, v);
        tmem_ld_wait();
        release_acc<NACC>(s, abuf, aphase, lane);
        group_fma32<0, COLS>(f, cs, v, sc);
      }
      if (gs == kScaleGroups - 1 || g + 1 == p.groups) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&s.aux_empty[sbuf]));
        if (++sbuf == 2) {
          sbuf = 0;
          sphase ^= 1u;
        }
      }
    }
    if (!ok) break;
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
        for (int e = 0; e < 8; ++e) r[e] = __fmul_rn(__fmul_rn(f[g8 * 8 + e], sa), p.alpha);
        if (p.out) {
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
        if constexpr (WITH_C) {
          int4* dst = reinterpret_cast<int4*>(p.c + o);
          dst[0] = make_int4(cs[g8 * 8 + 0], cs[g8 * 8 + 1], cs[g8 * 8 + 2], cs[g8 * 8 + 3]);
          dst[1] = make_int4(cs[g8 * 8 + 4], cs[g8 * 8 + 5], cs[g8 * 8 + 6], cs[g8 * 8 + 7]);
        }
      }
    }
  }
}

}  // namespace gemm
}  // namespace qk
