// gemm_sm100.cuh -- large-M W8A8 GEMM on the 5th-generation tensor cores.
//
// acc = A[m, k] * B[n, k]^T in int32 ("write-int8-quantized-kernel", Inputs:
// INT32 accumulation is mandatory; "KV-cache kernels" section 02: int8
// products accumulate in int32 and the scales are applied at the end), then
// the dequant epilogue in registers.  The pages' kernels (dp4a, a Triton
// tl.dot loop, cuBLAS/CUTLASS) are prior art; this is the sm_100a form:
//
//  - one persistent CTA per SM walks output tiles (tile = blockIdx + i*grid);
//  - warp 0 / lane 0 is the TMA producer: 128-byte-swizzled K-major tiles of
//    A (128 x 128 B) and B (BN x 128 B) into a STAGES-deep shared-memory ring,
//    completion counted in bytes on an mbarrier;
//  - warp 1 / lane 0 issues tcgen05.mma.kind::i8 (M = 128, N = BN, K = 32,
//    four per stage) into an int32 accumulator in tensor memory, and frees
//    ring slots / publishes accumulators with tcgen05.commit;
//  - epilogue warps read the accumulator with tcgen05.ld (32 lanes x 32
//    columns per instruction), apply the scales and store the outputs;
//  - per-channel mode keeps two 128 x 256 accumulators in TMEM (all 512
//    columns), so the epilogue of tile i overlaps the MMAs of tile i+1;
//  - per-group mode (group = 128 = one stage of K) keeps int32 partial
//    buffers in TMEM: the MMA writes one group's partial per buffer and moves
//    on while 16 epilogue warps convert each partial exactly to fp32 and fold
//    it in with fmaf(P_g, s[n, g], f), in ascending group order, in
//    registers.  128 x 256 tiles with two buffers when only the output is
//    wanted; 128 x 128 tiles with four buffers when the int32 sums are also
//    written.
//
// Every wait is bounded (about one second): on expiry the kernel records
// QK_ERR_TIMEOUT, every role leaves its loop, the producer waits (bounded)
// for its in-flight copies, the MMA thread waits for its in-flight MMAs, and
// the TMEM is freed before the CTA exits.
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

struct Args {
  int m, n, k;
  const float* sa;  // [m]
  const float* sw;  // [n] or [n, groups]
  float alpha;
  int32_t* c;       // [m, n] or null
  void* out;        // [m, n] or null
  int out_bf16;
  int tiles_m, tiles_n, num_kb, groups;
  // split-K (pair kernel): each tile's K range is cut into `splits` pieces of
  // `kb_per_split` K blocks; partial sums meet in `ws` with per-region
  // arrival counters `cnt` (zero before the call, zero again after it).
  int splits, kb_per_split;
  int32_t* ws;
  int* cnt;
  // pair kernel: 1 when the `splits` K slices of a tile are the CTA pairs of
  // one cluster and are summed through distributed shared memory (no
  // workspace); 0 for the workspace form above
  int csplit;
  // pair kernel, tail split (tail_splits > 1, splits == 1): tiles
  // [0, dp_tiles) are computed whole; each remaining tile is cut into
  // `tail_splits` K slices of `tail_kbps` K blocks, and those slices are the
  // first unit of pairs 0 .. (tiles - dp_tiles) * tail_splits - 1.  Every
  // slice stores its partial in `tail_ws` and then counts itself in `cnt`;
  // the slice that arrives last adds the others' partials to its own, runs
  // the epilogue and leaves the counter zero (the partials are scratch).
  int dp_tiles, tail_splits, tail_kbps;
  int32_t* tail_ws;
  // pair kernel: 1 when bf16 `out` (and no `c`) is written by TMA bulk
  // tensor stores from shared memory (tensor map tmO) on the whole-tile and
  // tail paths
  int tma_out;
  // 1: a and b are float8 e4m3 codes, the MMA is kind::f8f6f4 and the
  // accumulator fp32 (channel and pair kernels, whole tiles or the cluster
  // split-K, no c)
  int f8;
  // asymmetric activations (per channel only): zp [m] zero-points and wsum
  // [n] = sum_k b[n][k]; the epilogues use acc - zp[m] * wsum[n]
  const int32_t* zp;
  const int32_t* wsum;
  // MoE grouped GEMM (1-SM kernel): tokens grouped by expert, expert e's rows
  // [moe_off[e], moe_off[e + 1]) of a (m rows in all); b is [experts * n, k]
  // and sw [experts, n]; tiles_m = experts * mt_max M tiles, those past an
  // expert's tokens are skipped
  int mt_max;
  const int32_t* moe_off;
  // wide group kernel, the last wave split along K (gsplit > 0): tiles
  // [0, tiles - gsplit) run whole; tail tile (tiles - gsplit + j) is cut at
  // group gmid.  Its first part is CTA j's first unit: it leaves its fp32
  // running sums in gstate and sets the tile's 16 region flags in gflag.
  // Its second part is CTA (gsplit + j)'s last unit: it waits for the flags,
  // continues the sums in the same group order and leaves the flags zero.
  int gsplit, gmid;
  float* gstate;
  int* gflag;
};

// The i-th unit of this CTA in the wide group kernel's schedule (false past
// its last); every role walks the same list (group_plan.h).
__device__ __forceinline__ bool group_unit(const Args& p, int i, GroupUnit& u) {
  return group_unit_at(static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x),
                       p.tiles_m * p.tiles_n, p.gsplit, p.groups, p.gmid, i, u);
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
    const int experts = p.tiles_m / p.mt_max;
    int u = tile;
    for (int e = 0; e < experts; ++e) {
      const int r0 = __ldg(p.moe_off + e), r1 = __ldg(p.moe_off + e + 1);
      int mt = r1 > r0 ? (r1 - r0 + BM - 1) / BM : 0;
      mt = mt < p.mt_max ? mt : p.mt_max;
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
template <int BN, int STAGES, bool MOE = false, bool GUNITS = false, class S>
__device__ void produce(S& s, const CUtensorMap* tmA, const CUtensorMap* tmB, const Args& p) {
  const int nunits = p.tiles_m * p.tiles_n * p.splits;
  const uint32_t bytes = static_cast<uint32_t>((BM + BN) * BK);
  uint32_t stage = 0, phase = 0, issued = 0;
  bool ok = true;
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
      if (!chan_tile<BN, MOE>(p, unit / p.splits, t)) continue;
      kb0 = (unit % p.splits) * p.kb_per_split;
      kb1 = min(p.num_kb, kb0 + p.kb_per_split);
    }
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!mbar_wait(smem_addr(&s.empty[stage]), phase ^ 1u, &s.abort)) {
        ok = false;
        break;
      }
      const uint32_t fb = smem_addr(&s.full[stage]);
      mbar_arrive_expect_tx(fb, bytes);
      tma_load_2d(smem_addr(s.a[stage]), tmA, fb, kb * BK, t.a_row0);
      tma_load_2d(smem_addr(s.b[stage]), tmB, fb, kb * BK, t.b_row0);
      ++issued;
      if (++stage == STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
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
  const int nunits = p.tiles_m * p.tiles_n * p.splits;
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
      kb0 = (unit % p.splits) * p.kb_per_split;
      kb1 = min(p.num_kb, kb0 + p.kb_per_split);
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
  const uint32_t z = row < p.m ? static_cast<uint32_t>(__ldg(p.zp + row)) : 0u;
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    const int col = col0 + g * 4;
    const int4 w4 = col < p.n ? __ldg(reinterpret_cast<const int4*>(p.wsum + col))
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
template <bool F8 = false>
__device__ __forceinline__ void store32_tma(const Args& p, const CUtensorMap* tmO, uint8_t* box,
                                            int row0, int col0, float sa, const float* sw,
                                            const uint32_t (&v)[32]) {
  if (col0 >= p.n || row0 >= p.m) return;  // the box lies wholly outside (warp-uniform)
  const int lane = threadIdx.x & 31;
  uint32_t w[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float2 s2 = *reinterpret_cast<const float2*>(sw + 2 * j);
    float t0 = acc_value<F8>(v[2 * j]);
    float t1 = acc_value<F8>(v[2 * j + 1]);
    t0 = __fmul_rn(__fmul_rn(__fmul_rn(t0, sa), s2.x), p.alpha);
    t1 = __fmul_rn(__fmul_rn(__fmul_rn(t1, sa), s2.y), p.alpha);
    w[j] = pack_bf16x2(t0, t1);
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
  const int nunits = p.tiles_m * p.tiles_n * p.splits;
  const int lane = threadIdx.x & 31;
  const int ew = (threadIdx.x >> 5) - 2;  // epilogue warp 0..3
  const int quad = (threadIdx.x >> 5) & 3;
  float* sws = s.sw_tile[ew];
  uint8_t* box = s.out_stage[ew];
  uint32_t abuf = 0, aphase = 0;
  for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x) {
    ChanTile t;
    if (!chan_tile<BN, MOE>(p, unit / p.splits, t)) continue;
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
    if (p.csplit) {
      // Split-K inside the cluster (one unit per CTA, so the operand ring is
      // idle once acc_full has fired): stage this warp's 32 x BN partial in
      // its 32 KB slot of the ring, laid out [chunk][column quad][lane][4];
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
        if (p.zp) apply_zp(p, row, colbase + ch * 32, v);
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
        int* cnt = p.gflag + (u.tile - (ntiles - p.gsplit));
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
// operand ring as four 32 KB slots, one per TMEM lane quadrant (see
// epilogue_channel).  After a cluster barrier, CTA j takes the 32-column
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
  const int tile = static_cast<int>(blockIdx.x) / p.splits;
  const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
  const float* sws = s.sw_tile[ew];
  uint8_t* box = s.out_stage[ew];
  const int row0 = tm * BM + quad * 32, row = row0 + lane;
  const bool rv = row < p.m;
  const float sa = (rv && p.out) ? __ldg(p.sa + row) : 0.0f;
  const uint32_t slot = smem_addr(&s.a[0][0]) + static_cast<uint32_t>(quad * (32 * BN * 4));
  for (int c = j; c < BN / 32; c += p.splits) {
    const int col0 = tn * BN + c * 32;
    uint32_t va[32];
    // every source's part of the chunk requested at once (32 loads in
    // flight per lane: one cluster round trip per chunk)
    int4 t4[4][8];
#pragma unroll
    for (int o = 0; o < 4; ++o)
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4)
        t4[o][q4] = o < p.splits
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
        if (o < p.splits) {
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
    if (!F8 && p.zp) apply_zp(p, row, col0, va);
    if (p.tma_out)
      store32_tma<F8>(p, tmO, box, row0, col0, sa, sws + c * 32, va);
    else if (rv && col0 < p.n)
      store32_channel<F8>(p, row, col0, sa, sws + c * 32, va);
  }
  if (p.tma_out && lane == 0) bulk_wait_all();  // the output stores are complete
  __syncwarp();
}

constexpr int kChannelBN = 256;
constexpr int kChannelStages = 4;
constexpr int kChannelThreads = 64 + 4 * 32;
struct alignas(1024) ChannelStorage {
  uint8_t a[kChannelStages][BM * BK];
  uint8_t b[kChannelStages][kChannelBN * BK];
  uint8_t out_stage[4][kOutBoxBytes];  // each epilogue warp's TMA store box
  float sw_tile[4][kChannelBN];        // each epilogue warp's channel scales
  uint64_t full[kChannelStages];
  uint64_t empty[kChannelStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t aux_full[2];  // (unused by this kernel; set up with the others)
  uint64_t aux_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

template <bool F8, bool MOE = false>
__global__ void __launch_bounds__(kChannelThreads, 1)
    gemm_i8_channel_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmO, const Args p) {
  extern __shared__ uint8_t smem_raw[];
  ChannelStorage& s = storage<ChannelStorage>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (p.tma_out) prefetch_tmap(&tmO);
  }
  setup<ChannelStorage, kChannelStages, 2, 4>(s);
  griddep_wait();  // set-up above overlapped the previous kernel
  griddep_launch_dependents();
  const uint32_t tmem = s.tmem_base;
  if (warp == 0) {
    if (lane == 0) produce<kChannelBN, kChannelStages, MOE>(s, &tmA, &tmB, p);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_issue<kChannelBN, kChannelStages, 2, false, F8, MOE>(s, tmem, p);
    __syncwarp();
  } else {
    epilogue_channel<kChannelBN, 2, F8, MOE>(s, tmem, p, &tmO);
  }
  if (p.csplit) {
    cluster_sync_all();  // every CTA of the cluster has staged its partial
    if (warp >= 2) channel_cluster_reduce<kChannelBN, F8>(s, p, &tmO);
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
  griddep_wait();  // set-up above overlapped the previous kernel
  griddep_launch_dependents();
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
  return p.gstate + (static_cast<int64_t>(tt) * 16 + region) * (kGroupWideCols * 32);
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
        const float* st = group_state(p, u.tile - (ntiles - p.gsplit), region) + lane;
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
      const int tt = u.tile - (ntiles - p.gsplit);
      float* st = group_state(p, tt, region) + lane;
#pragma unroll
      for (int j = 0; j < COLS; ++j) __stcg(st + j * 32, fs[j]);
      __threadfence();
      __syncwarp();
      if (lane == 0) atomicAdd(p.gflag + tt, 1);
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
  griddep_wait();  // set-up above overlapped the previous kernel
  griddep_launch_dependents();
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

// ---------------------------------------------------------------- CTA-pair kernel
// Pair tile 256 x 256: the CTA of pair rank r (cluster rank & 1) owns rows
// [128 r, 128 r + 128) of the tile and loads them (A) plus rows
// [128 r, 128 r + 128) of the tile's 256 B rows (the N half the MMA reads
// from it).  A cluster is one pair, or, for split-K through distributed
// shared memory, the `splits` pairs of one tile; the pair's leader is the
// even cluster rank.  The leader's single MMA thread issues
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 32); each CTA's TMEM
// receives its 128 rows x 256 columns.  Per SM and stage this moves 32 KB for
// 128 x 256 x 128 MACs, two thirds of the single-CTA 128 x 256 tile's 48 KB.
// Both CTAs' copies complete on the leader's full barrier; the leader's
// commits arrive on both CTAs' empty / acc_full barriers; both CTAs'
// epilogue warps arrive on the leader's acc_empty.
constexpr int kPairBM = 256;
constexpr int kPairBN = 256;
constexpr int kPairStages = 6;
constexpr int kPairEpiWarps = 8;  // two per TMEM lane quadrant, 128 columns each
constexpr int kPairThreads = 64 + kPairEpiWarps * 32;
constexpr uint32_t kPairStageBytes = 2u * 128u * BK;  // per CTA: A half + B half

struct alignas(1024) PairStorage {
  uint8_t a[kPairStages][128 * BK];
  uint8_t b[kPairStages][128 * BK];
  uint8_t out_stage[kPairEpiWarps][kOutBoxBytes];
  float sw_tile[kPairEpiWarps][kPairBN / 2];  // each epilogue warp's channel scales
  uint64_t full[kPairStages];
  uint64_t empty[kPairStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// One unit of a pair's work: K blocks [kb0, kb1) of output tile `tile`;
// slice is the K slice index (0 for a whole tile).
struct PairUnit {
  int tile, kb0, kb1, slice;
};

// The i-th unit of pair `pi` (false past its last).  Without the tail split,
// units pi, pi + npairs, ... of the tiles x splits list; with it, the pair's
// tail slice first (if it has one), then data-parallel tiles pi,
// pi + npairs, ... below dp_tiles.
__device__ __forceinline__ bool pair_unit(const Args& p, int pi, int npairs, int i, PairUnit& u) {
  if (p.tail_splits > 1) {
    const int tail_units = (p.tiles_m * p.tiles_n - p.dp_tiles) * p.tail_splits;
    if (pi < tail_units) {
      if (i == 0) {
        u.tile = p.dp_tiles + pi / p.tail_splits;
        u.slice = pi % p.tail_splits;
        u.kb0 = u.slice * p.tail_kbps;
        u.kb1 = min(p.num_kb, u.kb0 + p.tail_kbps);
        return true;
      }
      --i;
    }
    const int t = pi + i * npairs;
    if (t >= p.dp_tiles) return false;
    u.tile = t;
    u.slice = 0;
    u.kb0 = 0;
    u.kb1 = p.num_kb;
    return true;
  }
  const int unit = pi + i * npairs;
  if (unit >= p.tiles_m * p.tiles_n * p.splits) return false;
  u.tile = unit / p.splits;
  u.slice = unit % p.splits;
  u.kb0 = u.slice * p.kb_per_split;
  u.kb1 = min(p.num_kb, u.kb0 + p.kb_per_split);
  return true;
}

// pr: this CTA's rank within its pair; lead: the cluster rank of its pair's
// leader (clusters hold one pair, or the `splits` pairs of one tile).
__device__ void produce_pair(PairStorage& s, const CUtensorMap* tmA, const CUtensorMap* tmB,
                             const Args& p, uint32_t pr, uint32_t lead) {
  const int npairs = gridDim.x >> 1;
  uint32_t stage = 0, phase = 0, issued = 0;
  bool ok = true;
  PairUnit u;
  for (int i = 0; ok && pair_unit(p, blockIdx.x >> 1, npairs, i, u); ++i) {
    const int tm = u.tile % p.tiles_m, tn = u.tile / p.tiles_m;
    const int ya = tm * kPairBM + static_cast<int>(pr) * 128;
    const int yb = tn * kPairBN + static_cast<int>(pr) * 128;
    for (int kb = u.kb0; kb < u.kb1; ++kb) {
      if (!mbar_wait(smem_addr(&s.empty[stage]), phase ^ 1u, &s.abort)) {
        ok = false;
        break;
      }
      const uint32_t fb_local = smem_addr(&s.full[stage]);
      if (pr == 0) mbar_arrive_expect_tx(fb_local, 2u * kPairStageBytes);
      const uint32_t fb = map_to_rank(fb_local, lead);
      tma_load_2d_pair(smem_addr(s.a[stage]), tmA, fb, kb * BK, ya);
      tma_load_2d_pair(smem_addr(s.b[stage]), tmB, fb, kb * BK, yb);
      ++issued;
      if (++stage == kPairStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  // Both CTAs' copies complete on the leader's barriers: the leader waits
  // (bounded) for the last phases it armed before the pair may exit.
  if (pr == 0) {
    const uint32_t first = issued > kPairStages ? issued - kPairStages : 0u;
    for (uint32_t i = first; i < issued; ++i)
      mbar_wait(smem_addr(&s.full[i % kPairStages]), (i / kPairStages) & 1u, nullptr);
  }
}

template <bool F8>
__device__ void mma_issue_pair(PairStorage& s, uint32_t tmem, const Args& p, uint32_t lead) {
  const uint16_t pair_mask = static_cast<uint16_t>(0x3u << lead);
  const int npairs = gridDim.x >> 1;
  constexpr uint32_t idesc = F8 ? idesc_e4m3(kPairBM, kPairBN) : idesc_i8(kPairBM, kPairBN);
  uint32_t stage = 0, phase = 0, abuf = 0, aphase = 0;
  bool ok = true;
  PairUnit u;
  for (int i = 0; ok && pair_unit(p, blockIdx.x >> 1, npairs, i, u); ++i) {
    const int kb0 = u.kb0, kb1 = u.kb1;
    if (!mbar_wait(smem_addr(&s.acc_empty[abuf]), aphase ^ 1u, &s.abort)) break;
    tc_fence_after();
    const uint32_t d = tmem + abuf * kPairBN;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!mbar_wait(smem_addr(&s.full[stage]), phase, &s.abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t a0 = smem_addr(s.a[stage]);
      const uint32_t b0 = smem_addr(s.b[stage]);
#pragma unroll
      for (int kk = 0; kk < BK / UMMA_K; ++kk) {
        if constexpr (F8)
          mma_e4m3_pair(d, sdesc_k_sw128(a0 + kk * UMMA_K), sdesc_k_sw128(b0 + kk * UMMA_K), idesc,
                        (kb > kb0 || kk > 0) ? 1u : 0u);
        else
          mma_i8_pair(d, sdesc_k_sw128(a0 + kk * UMMA_K), sdesc_k_sw128(b0 + kk * UMMA_K), idesc,
                      (kb > kb0 || kk > 0) ? 1u : 0u);
      }
      mma_commit_pair(smem_addr(&s.empty[stage]), pair_mask);
      if (++stage == kPairStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (!ok) break;
    mma_commit_pair(smem_addr(&s.acc_full[abuf]), pair_mask);
    if (++abuf == 2) {
      abuf = 0;
      aphase ^= 1u;
    }
  }
  mma_commit_pair(smem_addr(&s.drain), static_cast<uint16_t>(1u << lead));
  mbar_wait(smem_addr(&s.drain), 0u, nullptr);
}

// Tail split, one epilogue warp's 32 x 128 region (TMEM columns from tb) of
// K slice `u.slice` of tile `u.tile`.  Partial slots in `tail_ws` are
// [tail tile][slice][region][column quad][lane][4] int32, so each group of
// 32 lanes moves 512 contiguous bytes.  Every slice stores its partial,
// hands its TMEM buffer back to the MMA (acc_empty_lead: the lead CTA's
// barrier) and then takes a ticket on the region's counter (release); the
// slice whose ticket is the last one knows every partial is complete
// (acquire), sums them from L2 in ascending slice order (exact for int32,
// fixed order for fp32), runs the per-channel epilogue and resets the
// counter.  No slice waits for another, and none holds its TMEM buffer
// through the reduction.
template <bool F8>
__device__ void tail_slice_epilogue(uint32_t acc_empty_lead, const Args& p,
                                    const PairUnit& u, int region, uint32_t tb, int row, bool rv,
                                    float sa, int colbase, const float* sws,
                                    const CUtensorMap* tmO, uint8_t* box) {
  constexpr int kRegionInts = 32 * (kPairBN / 2);
  const int lane = threadIdx.x & 31;
  const int S = p.tail_splits;
  const int tt = u.tile - p.dp_tiles;
  int* cnt = p.cnt + tt * 16 + region;
  int32_t* slots = p.tail_ws + static_cast<int64_t>(tt) * S * 16 * kRegionInts;
  uint32_t va[32];
  {
    int4* dst = reinterpret_cast<int4*>(slots + (static_cast<int64_t>(u.slice) * 16 + region) * kRegionInts);
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
      tmem_ld_32x32b_x32(tb + ch * 32, va);
      tmem_ld_wait();
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4)
        __stcg(dst + (ch * 8 + q4) * 32 + lane,
               make_int4(va[q4 * 4], va[q4 * 4 + 1], va[q4 * 4 + 2], va[q4 * 4 + 3]));
    }
  }
  // the accumulator is in the workspace: hand the TMEM buffer back to the
  // MMA before the (slower) reduction, so later units are not held up
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive_cluster(acc_empty_lead);
  __threadfence();
  __syncwarp();
  int last = 0;
  if (lane == 0) last = atomicAdd(cnt, 1) == S - 1;
  last = __shfl_sync(0xFFFFFFFFu, last, 0);
  if (!last) return;
  __threadfence();
  // every slice's part of a 32-column chunk requested at once (S <= 4),
  // then added in ascending slice order
#pragma unroll 1
  for (int ch = 0; ch < 4; ++ch) {
    int4 t4[4][8];
#pragma unroll
    for (int o = 0; o < 4; ++o) {
      const int4* src = reinterpret_cast<const int4*>(
          slots + (static_cast<int64_t>(o < S ? o : 0) * 16 + region) * kRegionInts);
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4)
        t4[o][q4] = o < S ? __ldcg(src + (ch * 8 + q4) * 32 + lane) : make_int4(0, 0, 0, 0);
    }
#pragma unroll
    for (int q4 = 0; q4 < 8; ++q4) {
      va[q4 * 4] = static_cast<uint32_t>(t4[0][q4].x);
      va[q4 * 4 + 1] = static_cast<uint32_t>(t4[0][q4].y);
      va[q4 * 4 + 2] = static_cast<uint32_t>(t4[0][q4].z);
      va[q4 * 4 + 3] = static_cast<uint32_t>(t4[0][q4].w);
    }
#pragma unroll
    for (int o = 1; o < 4; ++o)
      if (o < S) {
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) acc_add4<F8>(va + q4 * 4, t4[o][q4]);
      }
    if (!F8 && p.zp) apply_zp(p, row, colbase + ch * 32, va);
    if (p.tma_out)
      store32_tma<F8>(p, tmO, box, row - lane, colbase + ch * 32, sa, sws + ch * 32, va);
    else if (rv)
      store32_channel<F8>(p, row, colbase + ch * 32, sa, sws + ch * 32, va);
  }
  __syncwarp();
  if (lane == 0) *cnt = 0;  // ready for the next call
}

// Epilogue of the pair kernel: 8 warps per CTA; warp w (2..9) reads TMEM
// lanes 32*(w%4) (rows) and columns [128 h, 128 h + 128), h = (w - 2) / 4.
// The tile's channel scales are staged per warp in shared memory, the row's
// token scale is fetched before the accumulator is ready, and the four
// 32-column TMEM loads are double-buffered so the next load is in flight
// while the current chunk is converted and stored.
template <bool F8>
__device__ void epilogue_pair(PairStorage& s, uint32_t tmem, const Args& p, uint32_t pr,
                              uint32_t lead, const CUtensorMap* tmO) {
  const int npairs = gridDim.x >> 1;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int quad = warp & 3;
  const int half = (warp - 2) >> 2;
  const int region = static_cast<int>(pr) * kPairEpiWarps + (warp - 2);  // 0..15
  float* sws = s.sw_tile[warp - 2];
  uint8_t* box = s.out_stage[warp - 2];
  uint32_t abuf = 0, aphase = 0;
  PairUnit u;
  for (int i = 0; pair_unit(p, blockIdx.x >> 1, npairs, i, u); ++i) {
    const int tile = u.tile;
    const bool tail = p.tail_splits > 1 && tile >= p.dp_tiles;
    const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
    const int row = tm * kPairBM + static_cast<int>(pr) * 128 + quad * 32 + lane;
    const bool rv = row < p.m;
    const float sa = (rv && p.out) ? __ldg(p.sa + row) : 0.0f;
    const int colbase = tn * kPairBN + half * (kPairBN / 2);
    if (p.out) {
      const int c4 = colbase + lane * 4;  // n % 8 == 0: a group of 4 is all in or all out
      const float4 v4 = c4 < p.n ? __ldg(reinterpret_cast<const float4*>(p.sw + c4))
                                 : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      *reinterpret_cast<float4*>(sws + lane * 4) = v4;
    }
    __syncwarp();
    if (!warp_wait(smem_addr(&s.acc_full[abuf]), aphase, &s.abort)) break;
    tc_fence_after();
    const uint32_t tb = tmem + (static_cast<uint32_t>(quad * 32) << 16) + abuf * kPairBN +
                        half * (kPairBN / 2);
    uint32_t va[32], vb[32];
    if (tail) {
      // (releases the TMEM buffer itself, before its reduction)
      tail_slice_epilogue<F8>(map_to_rank(smem_addr(&s.acc_empty[abuf]), lead), p, u, region,
                              tb, row, rv, sa, colbase, sws, tmO, box);
    } else if (F8 && !p.csplit) {
      // FP8 kind, whole tile (fp32 accumulator)
      auto emit = [&](int ch, const uint32_t(&v)[32]) {
        if (p.tma_out)
          store32_tma<true>(p, tmO, box, row - lane, colbase + ch * 32, sa, sws + ch * 32, v);
        else if (rv)
          store32_channel<true>(p, row, colbase + ch * 32, sa, sws + ch * 32, v);
      };
      tmem_ld_32x32b_x32(tb, va);
      tmem_ld_wait();
#pragma unroll
      for (int ch = 0; ch < 4; ch += 2) {
        tmem_ld_32x32b_x32(tb + (ch + 1) * 32, vb);
        emit(ch, va);
        tmem_ld_wait();
        if (ch + 2 < 4) tmem_ld_32x32b_x32(tb + (ch + 2) * 32, va);
        emit(ch + 1, vb);
        tmem_ld_wait();
      }
    } else if (p.tma_out) {
      tmem_ld_32x32b_x32(tb, va);
      tmem_ld_wait();
#pragma unroll
      for (int ch = 0; ch < 4; ch += 2) {
        tmem_ld_32x32b_x32(tb + (ch + 1) * 32, vb);
        if (p.zp) apply_zp(p, row, colbase + ch * 32, va);
        store32_tma(p, tmO, box, row - lane, colbase + ch * 32, sa, sws + ch * 32, va);
        tmem_ld_wait();
        if (ch + 2 < 4) tmem_ld_32x32b_x32(tb + (ch + 2) * 32, va);
        if (p.zp) apply_zp(p, row, colbase + (ch + 1) * 32, vb);
        store32_tma(p, tmO, box, row - lane, colbase + (ch + 1) * 32, sa, sws + (ch + 1) * 32, vb);
        tmem_ld_wait();
      }
    } else if (p.splits == 1) {
      tmem_ld_32x32b_x32(tb, va);
      tmem_ld_wait();
#pragma unroll
      for (int ch = 0; ch < 4; ch += 2) {
        tmem_ld_32x32b_x32(tb + (ch + 1) * 32, vb);
        if (p.zp) apply_zp(p, row, colbase + ch * 32, va);
        if (rv) store32_channel(p, row, colbase + ch * 32, sa, sws + ch * 32, va);
        tmem_ld_wait();
        if (ch + 2 < 4) tmem_ld_32x32b_x32(tb + (ch + 2) * 32, va);
        if (p.zp) apply_zp(p, row, colbase + (ch + 1) * 32, vb);
        if (rv) store32_channel(p, row, colbase + (ch + 1) * 32, sa, sws + (ch + 1) * 32, vb);
        tmem_ld_wait();
      }
    } else if (p.csplit) {
      // Split-K inside the cluster: stage this warp's 32 x 128 partial in its
      // 16 KB slot of the (idle) operand ring, [column quad][lane][4]; the
      // sum over the cluster's pairs is taken after the cluster barrier
      // (cluster_reduce_pair).
      uint8_t* stg = &s.a[0][0] + (warp - 2) * (32 * (kPairBN / 2) * 4);
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        tmem_ld_32x32b_x32(tb + ch * 32, va);
        tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          *reinterpret_cast<int4*>(stg + (((ch * 8 + q4) * 32 + lane) * 16)) =
              make_int4(va[q4 * 4], va[q4 * 4 + 1], va[q4 * 4 + 2], va[q4 * 4 + 3]);
      }
    } else {
      // Split-K.  Every pair holds exactly one unit (the host plans at most
      // one unit per pair), so once acc_full has fired the operand ring is
      // idle and serves as staging space: this warp copies its 32 x 128
      // partial region from TMEM into its own 16 KB of the ring, laid out
      // [column quad][lane][4], and one bulk reduction adds it into the
      // tile's int32 accumulator in the workspace (the additions happen at
      // L2).  The warp that brings a region's arrival count to `splits`
      // reads the finished sum, runs the epilogue, and leaves the region and
      // its counter zero for the next call.
      constexpr int kRegionInts = 32 * (kPairBN / 2);
      constexpr uint32_t kRegionBytes = kRegionInts * 4;
      int32_t* acc_region = p.ws + (static_cast<int64_t>(tile) * 16 + region) * kRegionInts;
      uint8_t* stg = &s.a[0][0] + (warp - 2) * kRegionBytes;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        tmem_ld_32x32b_x32(tb + ch * 32, va);
        tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          *reinterpret_cast<int4*>(stg + (((ch * 8 + q4) * 32 + lane) * 16)) =
              make_int4(va[q4 * 4], va[q4 * 4 + 1], va[q4 * 4 + 2], va[q4 * 4 + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        bulk_reduce_add_s32(acc_region, smem_addr(stg), kRegionBytes);
        bulk_commit();
        bulk_wait_all();
        fence_proxy_async_global();
        __threadfence();
        last = atomicAdd(p.cnt + tile * 16 + region, 1) == p.splits - 1;
      }
      last = __shfl_sync(0xFFFFFFFFu, last, 0);
      if (last) {
        __threadfence();
        const int4 zero = make_int4(0, 0, 0, 0);
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          int4 t4[8];
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            t4[q4] = __ldcg(reinterpret_cast<const int4*>(acc_region + ((ch * 8 + q4) * 32 + lane) * 4));
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            va[q4 * 4] = t4[q4].x;
            va[q4 * 4 + 1] = t4[q4].y;
            va[q4 * 4 + 2] = t4[q4].z;
            va[q4 * 4 + 3] = t4[q4].w;
            __stcg(reinterpret_cast<int4*>(acc_region + ((ch * 8 + q4) * 32 + lane) * 4), zero);
          }
          if (p.zp) apply_zp(p, row, colbase + ch * 32, va);
          if (rv) store32_channel(p, row, colbase + ch * 32, sa, sws + ch * 32, va);
        }
        if (lane == 0) p.cnt[tile * 16 + region] = 0;  // ready for the next call
      }
    }
    if (!tail) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(smem_addr(&s.acc_empty[abuf]), lead));
    }
    if (++abuf == 2) {
      abuf = 0;
      aphase ^= 1u;
    }
  }
  if (p.tma_out && lane == 0) bulk_wait_all();  // the output stores are complete
  __syncwarp();
}

// Split-K through distributed shared memory.  The cluster is the `splits`
// CTA pairs of one tile (pair j computed K slice j); every CTA has staged
// its 128 x 256 int32 partial in its operand ring as 8 slots of 32 rows x
// 128 columns (slot = epilogue warp - 2, laid out [column quad][lane][4]).
// After a cluster barrier, CTA (pair j, half h) takes the 32-column chunks
// c = j, j + splits, ... of the tile's 256 columns: for its 128 rows it
// sums chunk c over the `splits` CTAs of half h (plain integer adds, exact),
// then dequantises and stores.  The two epilogue warps of a TMEM lane
// quadrant take alternate chunks.
// Before the cluster barrier: each epilogue warp copies the channel scales of
// the (at most two) chunks it will reduce into its shared-memory slot.
__device__ void cluster_reduce_scales(PairStorage& s, const Args& p, uint32_t crank) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int w2 = (warp - 2) >> 2;
  const int j = static_cast<int>(crank >> 1);
  const int tn = ((blockIdx.x >> 1) / p.splits) / p.tiles_m;
  float* sws = s.sw_tile[warp - 2];
  int t = 0;
  for (int c = j + p.splits * w2; c < kPairBN / 32 && t < 2; c += 2 * p.splits, ++t) {
    const int col = tn * kPairBN + c * 32 + lane;
    sws[t * 32 + lane] = (p.out && col < p.n) ? __ldg(p.sw + col) : 0.0f;
  }
}

template <bool F8>
__device__ void cluster_reduce_pair(PairStorage& s, const Args& p, uint32_t crank) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int quad = warp & 3;
  const int w2 = (warp - 2) >> 2;
  const int j = static_cast<int>(crank >> 1), h = static_cast<int>(crank & 1u);
  const int tile = (blockIdx.x >> 1) / p.splits;
  const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
  const float* sws = s.sw_tile[warp - 2];
  int t = 0;
  const int row = tm * kPairBM + h * 128 + quad * 32 + lane;
  const bool rv = row < p.m;
  const float sa = (rv && p.out) ? __ldg(p.sa + row) : 0.0f;
  const uint32_t base = smem_addr(&s.a[0][0]);
  constexpr uint32_t kSlotBytes = 32 * (kPairBN / 2) * 4;
  for (int c = j + p.splits * w2; c < kPairBN / 32; c += 2 * p.splits, ++t) {
    const int hh = c >> 2, ch = c & 3;
    const uint32_t slot = static_cast<uint32_t>(hh * 4 + ((quad + 2) & 3));  // staging warp of (quad, hh)
    const uint32_t off = base + slot * kSlotBytes + static_cast<uint32_t>((ch * 8 * 32 + lane) * 16);
    uint32_t va[32];
    // all sources' loads of this chunk in flight together (splits <= 4):
    // one round trip through the cluster per chunk
    int4 t4[4][8];
#pragma unroll
    for (int o = 0; o < 4; ++o) {
      const uint32_t peer = static_cast<uint32_t>(2 * o + h);
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4)
        t4[o][q4] = o < p.splits ? ld_dsmem_v4(map_to_rank(off + q4 * 32 * 16, peer))
                                 : make_int4(0, 0, 0, 0);
    }
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
        if (o < p.splits) {
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
    const int col0 = tn * kPairBN + c * 32;
    if (!F8 && p.zp) apply_zp(p, row, col0, va);
    if (rv && col0 < p.n) store32_channel<F8>(p, row, col0, sa, sws + t * 32, va);
  }
}

template <bool F8>
__global__ void __launch_bounds__(kPairThreads, 1)
    gemm_i8_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmO, const Args p) {
  extern __shared__ uint8_t smem_raw[];
  PairStorage& s = storage<PairStorage>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_rank();
  const uint32_t pr = crank & 1u, lead = crank & ~1u;
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (p.tma_out) prefetch_tmap(&tmO);
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kPairStages; ++i) {
      mbar_init(smem_addr(&s.full[i]), 1);
      mbar_init(smem_addr(&s.empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_addr(&s.acc_full[i]), 1);
      mbar_init(smem_addr(&s.acc_empty[i]), 2 * kPairEpiWarps);  // epilogue warps of both CTAs
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
  if (warp == 0) {
    if (lane == 0) produce_pair(s, &tmA, &tmB, p, pr, lead);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && pr == 0) mma_issue_pair<F8>(s, tmem, p, lead);
    __syncwarp();
  } else {
    epilogue_pair<F8>(s, tmem, p, pr, lead, &tmO);
  }
  if (p.csplit) {
    if (warp >= 2) cluster_reduce_scales(s, p, crank);
    cluster_sync_all();  // every CTA of the cluster has staged its partial
    if (warp >= 2) cluster_reduce_pair<F8>(s, p, crank);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the leader's MMAs on this CTA's smem / TMEM are done
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// int8 [rows, k] row-major, box = 128 bytes of K x box_rows rows, 128-byte
// swizzle; out-of-range rows/columns read as zero.
inline bool make_tmap(CUtensorMap* map, const void* base, int rows, int k, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(k)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// bf16 [rows, cols] row-major output, box = 32 columns (64 bytes) x 32 rows,
// 64-byte swizzle (the layout store32_tma writes); stores are clipped to
// the tensor.
inline bool make_out_tmap(CUtensorMap* map, const void* base, int rows, int cols) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor maps depend only on (base, rows, k, box_rows, kind): the recent
// ones are kept so that repeated calls on the same buffers skip the
// driver's encoder (a few microseconds of host time per map).  kind 0: an
// int8 operand (make_tmap); kind 1: a bf16 output (make_out_tmap, k =
// columns).
inline bool cached_tmap(CUtensorMap* map, const void* base, int rows, int k, int box_rows,
                        int kind = 0) {
  struct Entry {
    const void* base;
    int rows, k, box_rows, kind;
    CUtensorMap map;
  };
  constexpr int kEntries = 32;
  static Entry entries[kEntries];
  static int used = 0, next = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i) {
    const Entry& e = entries[i];
    if (e.base == base && e.rows == rows && e.k == k && e.box_rows == box_rows && e.kind == kind) {
      *map = e.map;
      return true;
    }
  }
  if (!(kind == 1 ? make_out_tmap(map, base, rows, k) : make_tmap(map, base, rows, k, box_rows)))
    return false;
  Entry& e = entries[next];
  e.base = base;
  e.rows = rows;
  e.k = k;
  e.box_rows = box_rows;
  e.kind = kind;
  e.map = *map;
  next = (next + 1) % kEntries;
  if (used < kEntries) ++used;
  return true;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (device, kernel).
template <class K>
inline cudaError_t set_smem_once(K kernel, int dev, int slot, size_t bytes) {
  static std::atomic<unsigned long long> done[8] = {};
  const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (done[slot].load(std::memory_order_acquire) & bit)) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess && bit) done[slot].fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

inline size_t channel_smem() { return sizeof(ChannelStorage) + 1024; }
inline size_t pair_smem() { return sizeof(PairStorage) + 1024; }

// Largest number of co-resident clusters of `cluster` CTAs of the pair
// kernel (queried once per device and size; 0 when the size cannot run).
inline int max_pair_clusters(int dev, int cluster) {
  // (relaxed atomics: host threads may race to fill an entry, all with the same value)
  static std::atomic<int> cache[64][5] = {};  // cluster 2, 4, 6, 8 (index cluster / 2)
  const int ci = cluster / 2;
  if (dev < 0 || dev >= 64 || ci < 1 || ci > 4 || cluster % 2) return 0;
  const int known = cache[dev][ci].load(std::memory_order_relaxed);
  if (known != 0) return known > 0 ? known : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cluster) * 16, 1, 1);
  cfg.blockDim = dim3(kPairThreads, 1, 1);
  cfg.dynamicSmemBytes = pair_smem();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaFuncSetAttribute(gemm_i8_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(pair_smem())) != cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, gemm_i8_pair_kernel<false>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cache[dev][ci].store(n > 0 ? n : -1, std::memory_order_relaxed);
  return n > 0 ? n : 0;
}

// Largest number of co-resident CTA pairs (queried once per device).
inline int max_pairs(int dev, int num_sms) {
  static std::atomic<int> cache[64] = {};
  if (dev >= 0 && dev < 64) {
    const int known = cache[dev].load(std::memory_order_relaxed);
    if (known > 0) return known;
  }
  int pairs = num_sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kPairThreads, 1, 1);
  cfg.dynamicSmemBytes = pair_smem();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaFuncSetAttribute(gemm_i8_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(pair_smem())) == cudaSuccess &&
      cudaOccupancyMaxActiveClusters(&n, gemm_i8_pair_kernel<false>, &cfg) == cudaSuccess && n > 0)
    pairs = n < pairs ? n : pairs;
  else
    cudaGetLastError();
  if (dev >= 0 && dev < 64) cache[dev].store(pairs, std::memory_order_relaxed);
  return pairs;
}

// Workspace of the pair kernel's split-K: a fixed header of arrival counters
// (16 per tile; split-K only runs with fewer than 64 tiles), then one int32
// accumulator per output tile that the K slices add into.  The header is at
// a fixed place and every completed call leaves counters and accumulators at
// zero, so one zero-filled workspace can serve problems of any shape.
constexpr size_t kCounterHeaderBytes = 4096;
constexpr int kMaxSplitTiles = static_cast<int>(kCounterHeaderBytes / (16 * 4));
constexpr size_t kTileAccBytes = static_cast<size_t>(256) * 1024;  // one 256 x 256 int32 tile
// Tail-split partials live past the split-K accumulators (so those stay
// zero): at most kMaxTailSlots partial tiles.
constexpr size_t kTailOffset = kCounterHeaderBytes + kMaxSplitTiles * kTileAccBytes;
constexpr int kMaxTailSlots = 128;

// Split-K plan of the pair kernel: when the output has fewer tiles than
// three quarters of the SM pairs, cut K into pieces (>= 8 K blocks each) so
// that about one unit lands on every pair.
//
// Tail split: with more tiles than pairs, the last wave of whole tiles
// would leave pairs idle (4096 x 4096 is 256 tiles on 74 pairs: 3 full
// waves, then 34 tiles).  Those r = tiles mod pairs tiles are instead cut
// into S = min(pairs / r, 4) K slices (>= 8 K blocks each) that run first,
// on r * S pairs, while the data-parallel tiles follow: the work takes
// about (waves + 1 / S) tile times instead of (waves + 1).
struct PairPlan {
  int tiles, splits, kb_per_split;
  int csplit;  // 1: the splits of a tile are the pairs of one cluster (no workspace)
  int dp_tiles, tail_splits, tail_kbps;
};

// f8: the FP8 kind.  Its fp32 partials are summed in a fixed order, which
// the cluster split-K gives; the workspace split-K adds them in arrival
// order and is left to the INT8 kind, and the tail split measured slower
// than whole tiles for FP8 (56.5 against 55.7 us at 4096^3).
inline PairPlan pair_plan(int m, int n, int k, int pairs, int dev, bool f8 = false) {
  PairPlan pl;
  pl.tiles = ((m + kPairBM - 1) / kPairBM) * ((n + kPairBN - 1) / kPairBN);
  pl.csplit = 0;
  pl.dp_tiles = pl.tiles;
  pl.tail_splits = 1;
  pl.tail_kbps = 0;
  const int num_kb = (k + BK - 1) / BK;
  if (pl.tiles > pairs && pairs > 0 && f8) {
    pl.splits = 1;
    pl.kb_per_split = num_kb;
    return pl;
  }
  if (pl.tiles > pairs && pairs > 0) {
    const int r = pl.tiles % pairs;
    int ts = r > 0 ? pairs / r : 1;
    ts = ts < 4 ? ts : 4;
    ts = ts < num_kb / 8 ? ts : num_kb / 8;
    while (ts > 1 && (r > kMaxSplitTiles || ts * r > kMaxTailSlots)) --ts;
    if (ts > 1) {
      const int kbps = (num_kb + ts - 1) / ts;
      pl.tail_splits = (num_kb + kbps - 1) / kbps;
      pl.tail_kbps = kbps;
      pl.dp_tiles = pl.tiles - r;
    }
    pl.splits = 1;
    pl.kb_per_split = num_kb;
    return pl;
  }
  int s = 1;
  if (4 * pl.tiles < 3 * pairs && pl.tiles <= kMaxSplitTiles) {
    s = pairs / pl.tiles;
    const int by_k = num_kb / 8;
    s = s < by_k ? s : by_k;
    s = s > 1 ? s : 1;
  }
  pl.kb_per_split = (num_kb + s - 1) / s;
  pl.splits = (num_kb + pl.kb_per_split - 1) / pl.kb_per_split;
  if (pl.splits > 1) {
    // The split-K tail through the workspace costs about 23 K-block times
    // (measured at 256 x 4096 x 14336); summing the partials through
    // distributed shared memory in a cluster of the tile's pairs costs about
    // 3, but needs the clusters co-resident and allows at most 4 pairs per
    // cluster.  Take whichever is estimated faster (ties: the workspace).
    const double cost_ws = pl.kb_per_split + 23.0;
    for (int cs = 4; cs >= 2; --cs) {
      if (num_kb / cs < 8 || pl.tiles * cs > pairs) continue;
      if (max_pair_clusters(dev, 2 * cs) < pl.tiles) continue;
      const int kbps = (num_kb + cs - 1) / cs;
      if ((num_kb + kbps - 1) / kbps != cs) continue;
      if (kbps + 3.0 < cost_ws || f8) {
        pl.splits = cs;
        pl.kb_per_split = kbps;
        pl.csplit = 1;
      }
      break;
    }
    if (f8 && !pl.csplit) {
      pl.splits = 1;
      pl.kb_per_split = num_kb;
    }
  }
  return pl;
}

// Leading bytes of the workspace that must be zero before a call (and that
// every completed call leaves zero): the counters, and the split-K
// accumulators when the plan adds into them.
inline size_t pair_workspace_zero_bytes(const PairPlan& pl) {
  if (pl.tail_splits > 1) return kCounterHeaderBytes;
  if (pl.splits <= 1 || pl.csplit) return 0;
  return kCounterHeaderBytes + static_cast<size_t>(pl.tiles) * kTileAccBytes;
}

inline size_t pair_workspace_bytes(const PairPlan& pl) {
  if (pl.tail_splits > 1) {
    // counters, the (unused) split-K accumulators, then every slice's
    // partial of every tail tile
    return kTailOffset +
           static_cast<size_t>(pl.tiles - pl.dp_tiles) * pl.tail_splits * kTileAccBytes;
  }
  if (pl.splits <= 1 || pl.csplit) return 0;
  // counters, then one int32 accumulator tile (16 regions of 32 x 128) per tile
  return kCounterHeaderBytes + static_cast<size_t>(pl.tiles) * 16 * 32 * (kPairBN / 2) * 4;
}

// CTA-pair kernel for m > 128.  0 ok, 1 tensor-map failure, 2 CUDA error.
inline int launch_pair(Args a, const int8_t* A, const int8_t* B, int dev, int num_sms,
                       void* workspace, cudaStream_t stream, cudaError_t* err,
                       bool allow_split = true) {
  a.tiles_m = (a.m + kPairBM - 1) / kPairBM;
  a.tiles_n = (a.n + kPairBN - 1) / kPairBN;
  a.num_kb = (a.k + BK - 1) / BK;
  a.groups = 0;
  const int pairs = max_pairs(dev, num_sms);
  PairPlan pl = pair_plan(a.m, a.n, a.k, pairs, dev, a.f8 != 0);
  if (!allow_split || static_cast<int64_t>(pl.tiles) * pl.splits > pairs) {
    // (split-K stages partials in the operand ring: one unit per pair)
    pl.splits = 1;
    pl.kb_per_split = a.num_kb;
  }
  if (!allow_split) {
    pl.tail_splits = 1;
    pl.dp_tiles = pl.tiles;
  }
  if (pl.splits == 1) pl.csplit = 0;
  a.splits = pl.splits;
  a.kb_per_split = pl.kb_per_split;
  a.csplit = pl.csplit;
  a.dp_tiles = pl.dp_tiles;
  a.tail_splits = pl.tail_splits;
  a.tail_kbps = pl.tail_kbps;
  a.ws = nullptr;
  a.cnt = nullptr;
  a.tail_ws = nullptr;
  if ((pl.splits > 1 && !pl.csplit) || pl.tail_splits > 1) {
    a.cnt = static_cast<int*>(workspace);
    a.ws = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + kCounterHeaderBytes);
    a.tail_ws = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + kTailOffset);
  }
  CUtensorMap ta, tb, to;
  if (!cached_tmap(&ta, A, a.m, a.k, 128) || !cached_tmap(&tb, B, a.n, a.k, 128)) return 1;
  // bf16 out without c, outside split-K: TMA stores from shared memory
  a.tma_out = (a.out != nullptr && a.out_bf16 && a.c == nullptr && a.splits == 1) ? 1 : 0;
  if (a.tma_out) {
    if (!cached_tmap(&to, a.out, a.m, a.n, 32, 1)) return 1;
  } else {
    to = ta;  // unused
  }
  const int ntiles = a.tiles_m * a.tiles_n * a.splits;  // > pairs whenever the tail split is on
  const int grid_pairs = ntiles < pairs ? ntiles : pairs;
  cudaError_t e = a.f8 ? set_smem_once(gemm_i8_pair_kernel<true>, dev, 4, pair_smem())
                       : set_smem_once(gemm_i8_pair_kernel<false>, dev, 0, pair_smem());
  if (e == cudaSuccess) {
    // cluster: one pair, or (cluster split-K) the splits pairs of one tile;
    // the grid is then exactly tiles x splits pairs, one unit each
    const unsigned cluster = pl.csplit ? 2u * static_cast<unsigned>(pl.splits) : 2u;
    e = launch_pdl(a.f8 ? gemm_i8_pair_kernel<true> : gemm_i8_pair_kernel<false>, dim3(2 * grid_pairs),
                   dim3(kPairThreads), pair_smem(), stream,
                   cluster, ta, tb, to, a);
  }
  *err = e;
  return e == cudaSuccess ? 0 : 2;
}
inline size_t group_smem() { return sizeof(GroupStorage) + 1024; }
inline size_t group_wide_smem() { return sizeof(GroupWideStorage) + 1024; }

// K split of the wide group kernel's last wave (Args::gsplit): with T tiles
// on P = min(T, num_sms) CTAs and T = q P + r, the r tail tiles are cut in
// two when 0 < 2 r <= P and there are at least two groups, so that CTAs
// 0 .. 2r - 1 each run q tiles and one part (q + 1/2 tiles where whole tiles
// would take q + 1).  Returns r, or 0 when the split is off.
constexpr int kGroupWideMaxSplit = 512;  // (2 r <= SMs per GPU)
inline int group_split_tiles(int m, int n, int k, int num_sms) {
  const int tiles = ((m + BM - 1) / BM) * ((n + kGroupWideBN - 1) / kGroupWideBN);
  if (num_sms > 2 * kGroupWideMaxSplit) return 0;
  return group_split_count(tiles, k / 128, num_sms);
}
// Its workspace follows the layout the pair kernel's splits use, so that one
// workspace serves every call: one arrival counter per tail tile in the
// counter header (zero before a call, zero after it; the first
// group_flag_bytes must be zero), and each tail tile's running sums
// (128 x 256 fp32, scratch) from kTailOffset on, past the split-K
// accumulators that other calls need left zero.
inline size_t group_flag_bytes(int r) {
  return (static_cast<size_t>(r) * sizeof(int) + 255) & ~static_cast<size_t>(255);
}
inline size_t group_workspace_bytes(int r) {
  return r > 0 ? kTailOffset + static_cast<size_t>(r) * BM * kGroupWideBN * sizeof(float) : 0;
}
static_assert(kGroupWideMaxSplit * sizeof(int) <= kCounterHeaderBytes,
              "group split counters fit the counter header");

// The wide group kernel moves registers between warpgroups with setmaxnreg;
// the budgets only add up if the compiled kernel launches with at least
// kGroupWideLaunchRegs registers per thread (otherwise the increase would
// wait for registers that never come back).  Checked once per device.
inline bool group_wide_ok(int dev) {
  static std::atomic<int> cache[64] = {};
  if (dev < 0 || dev >= 64) return false;
  int known = cache[dev].load(std::memory_order_relaxed);
  if (known == 0) {
    cudaFuncAttributes fa;
    const bool ok = cudaFuncGetAttributes(&fa, gemm_i8_group_wide_kernel) == cudaSuccess &&
                    fa.numRegs >= kGroupWideLaunchRegs &&
                    fa.numRegs * kGroupWideThreads <= 65536;
    if (!ok) cudaGetLastError();
    known = ok ? 1 : -1;
    cache[dev].store(known, std::memory_order_relaxed);
  }
  return known > 0;
}

// 0 ok, 1 tensor-map failure, 2 CUDA error
// Largest number of co-resident clusters of `cluster` CTAs of the 1-SM
// channel kernel (queried once per device and size; 0 when it cannot run).
inline int max_channel_clusters(int dev, int cluster) {
  static std::atomic<int> cache[64][5] = {};
  if (dev < 0 || dev >= 64 || cluster < 2 || cluster > 4) return 0;
  const int known = cache[dev][cluster].load(std::memory_order_relaxed);
  if (known != 0) return known > 0 ? known : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cluster) * 16, 1, 1);
  cfg.blockDim = dim3(kChannelThreads, 1, 1);
  cfg.dynamicSmemBytes = channel_smem();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaFuncSetAttribute(gemm_i8_channel_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(channel_smem())) != cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, gemm_i8_channel_kernel<false>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cache[dev][cluster].store(n > 0 ? n : -1, std::memory_order_relaxed);
  return n > 0 ? n : 0;
}

// Split-K plan of the 1-SM channel kernel: with fewer 128 x 256 tiles than
// half the SMs, cut K into S <= 4 slices (>= 8 K blocks each), one CTA per
// slice, the S CTAs of a tile forming one cluster whose partials meet in
// distributed shared memory.  S = 1 when the clusters would not all be
// co-resident.
struct ChannelPlan {
  int tiles, splits, kb_per_split;
};

inline ChannelPlan channel_plan(int m, int n, int k, int num_sms, int dev) {
  ChannelPlan pl;
  pl.tiles = ((m + BM - 1) / BM) * ((n + kChannelBN - 1) / kChannelBN);
  const int num_kb = (k + BK - 1) / BK;
  int s = 1;
  if (2 * pl.tiles <= num_sms) {
    s = num_sms / pl.tiles;
    s = s < 4 ? s : 4;
    s = s < num_kb / 8 ? s : num_kb / 8;
  }
  while (s > 1) {
    const int kbps = (num_kb + s - 1) / s;
    const int ns = (num_kb + kbps - 1) / kbps;
    if (ns > 1 && max_channel_clusters(dev, ns) >= pl.tiles) {
      s = ns;
      break;
    }
    --s;
  }
  if (s < 1) s = 1;
  pl.kb_per_split = (num_kb + s - 1) / s;
  pl.splits = (num_kb + pl.kb_per_split - 1) / pl.kb_per_split;
  return pl;
}

// For 128 < m <= 256 (two 128-row tiles): the 1-SM kernel with cluster
// split-K is preferred over the CTA-pair kernel when it gives each CTA fewer
// K blocks (mlp_down, 256 x 4096 x 14336: 32 tiles x 4 slices of 28 K
// blocks on 128 SMs, against 16 pair tiles x 3 slices of 38 on 96 SMs).
inline bool prefer_channel_split(int m, int n, int k, int num_sms, int dev) {
  if (m <= BM || m > 2 * BM) return false;
  const ChannelPlan cp = channel_plan(m, n, k, num_sms, dev);
  if (cp.splits < 2) return false;
  const PairPlan pp = pair_plan(m, n, k, max_pairs(dev, num_sms), dev);
  const int pair_kb = pp.splits > 1 ? pp.kb_per_split : (k + BK - 1) / BK;
  return cp.kb_per_split < pair_kb;
}

// `workspace`: group_workspace_bytes(group_split_tiles(...)) bytes for the
// wide group kernel's split (null: whole tiles only); unused otherwise.
inline int launch(Args a, const int8_t* A, const int8_t* B, bool group, int dev, int num_sms,
                  cudaStream_t stream, cudaError_t* err, void* workspace = nullptr) {
  // group mode without the int32 sums: the 128 x 256 kernel
  const bool wide = group && a.c == nullptr && group_wide_ok(dev);
  const int bn = group ? (wide ? kGroupWideBN : kGroupBN) : kChannelBN;
  a.tiles_m = (a.m + BM - 1) / BM;
  a.tiles_n = (a.n + bn - 1) / bn;
  a.num_kb = (a.k + BK - 1) / BK;
  a.groups = group ? a.k / 128 : 0;
  a.splits = 1;
  a.kb_per_split = a.num_kb;
  a.csplit = 0;
  a.tail_splits = 1;
  if (!group) {
    const ChannelPlan pl = channel_plan(a.m, a.n, a.k, num_sms, dev);
    if (pl.splits > 1) {
      a.splits = pl.splits;
      a.kb_per_split = pl.kb_per_split;
      a.csplit = 1;
    }
  }
  CUtensorMap ta, tb, to;
  if (!cached_tmap(&ta, A, a.m, a.k, BM) || !cached_tmap(&tb, B, a.n, a.k, bn)) return 1;
  // channel kernel, bf16 out without c: TMA stores from shared memory
  a.tma_out = (!group && a.out != nullptr && a.out_bf16 && a.c == nullptr) ? 1 : 0;
  if (a.tma_out) {
    if (!cached_tmap(&to, a.out, a.m, a.n, 32, 1)) return 1;
  } else {
    to = ta;  // unused
  }
  const int ntiles = a.tiles_m * a.tiles_n;
  // split-K: exactly one CTA per (tile, K slice), in clusters of `splits`
  const int grid = a.csplit ? ntiles * a.splits : (ntiles < num_sms ? ntiles : num_sms);
  cudaError_t e;
  if (!group) {
    const size_t smem = channel_smem();
    e = a.f8 ? set_smem_once(gemm_i8_channel_kernel<true>, dev, 5, smem)
             : set_smem_once(gemm_i8_channel_kernel<false>, dev, 1, smem);
    if (e == cudaSuccess) {
      e = launch_pdl(a.f8 ? gemm_i8_channel_kernel<true> : gemm_i8_channel_kernel<false>, dim3(grid),
                     dim3(kChannelThreads), smem, stream,
                     a.csplit ? static_cast<unsigned>(a.splits) : 1u, ta, tb, to, a);
    }
  } else {
    if (wide) {
      a.gsplit = workspace ? group_split_tiles(a.m, a.n, a.k, num_sms) : 0;
      a.gmid = a.groups / 2;
      a.gflag = static_cast<int*>(workspace);
      a.gstate = a.gsplit ? reinterpret_cast<float*>(static_cast<char*>(workspace) + kTailOffset)
                          : nullptr;
      const size_t smem = group_wide_smem();
      e = set_smem_once(gemm_i8_group_wide_kernel, dev, 7, smem);
      if (e == cudaSuccess) {
        e = launch_pdl(gemm_i8_group_wide_kernel, dim3(grid), dim3(kGroupWideThreads), smem, stream,
                       1, ta, tb, a);
      }
      *err = e;
      return e == cudaSuccess ? 0 : 2;
    }
    const size_t smem = group_smem();
    if (a.c) {
      e = set_smem_once(gemm_i8_group_kernel<true>, dev, 2, smem);
      if (e == cudaSuccess) {
        e = launch_pdl(gemm_i8_group_kernel<true>, dim3(grid), dim3(GroupCfg<true>::threads), smem,
                       stream, 1, ta, tb, a);
      }
    } else {
      e = set_smem_once(gemm_i8_group_kernel<false>, dev, 3, smem);
      if (e == cudaSuccess) {
        e = launch_pdl(gemm_i8_group_kernel<false>, dim3(grid), dim3(GroupCfg<false>::threads), smem,
                       stream, 1, ta, tb, a);
      }
    }
  }
  *err = e;
  return e == cudaSuccess ? 0 : 2;
}

// MoE grouped GEMM on the 1-SM kernel: `experts` groups of tokens (expert e
// owns rows [off[e], off[e + 1]) of A, m rows in all), B stacked [experts *
// n, k], per-channel scales [experts, n]; mt_max bounds every expert's M
// tiles.  Whole tiles, per channel, direct stores (a TMA box could cross
// into the next expert's rows).  0 ok, 1 tensor-map failure, 2 CUDA error.
inline int launch_moe(Args a, const int8_t* A, const int8_t* B, int experts, int mt_max,
                      const int32_t* off, int dev, int num_sms, cudaStream_t stream,
                      cudaError_t* err) {
  a.mt_max = mt_max;
  a.moe_off = off;
  a.tiles_m = experts * mt_max;
  a.tiles_n = (a.n + kChannelBN - 1) / kChannelBN;
  a.num_kb = (a.k + BK - 1) / BK;
  a.groups = 0;
  a.splits = 1;
  a.kb_per_split = a.num_kb;
  a.csplit = 0;
  a.tail_splits = 1;
  a.tma_out = 0;
  a.c = nullptr;
  CUtensorMap ta, tb;
  if (!cached_tmap(&ta, A, a.m, a.k, BM) || !cached_tmap(&tb, B, experts * a.n, a.k, kChannelBN))
    return 1;
  const int64_t ntiles = static_cast<int64_t>(a.tiles_m) * a.tiles_n;
  const int grid = ntiles < num_sms ? static_cast<int>(ntiles) : num_sms;
  const size_t smem = channel_smem();
  cudaError_t e = set_smem_once(gemm_i8_channel_kernel<false, true>, dev, 6, smem);
  if (e == cudaSuccess)
    e = launch_pdl(gemm_i8_channel_kernel<false, true>, dim3(grid), dim3(kChannelThreads), smem,
                   stream, 1u, ta, tb, ta, a);
  *err = e;
  return e == cudaSuccess ? 0 : 2;
}

}  // namespace gemm
}  // namespace qk
