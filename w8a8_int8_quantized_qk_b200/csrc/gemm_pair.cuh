// gemm_pair.cuh -- the CTA-pair tcgen05 GEMM kernel (cta_group::2, 256 x 256
// tiles) with its split-K forms: through the workspace, through distributed
// shared memory in a cluster, and the tail split of a partial last wave;
// and its MoE form (grouped GEMM over per-expert tiles).
#pragma once

#include "gemm_1sm.cuh"

namespace qk {
namespace gemm {

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
// slice is the K slice index (0 for a whole tile).  The MoE form describes
// its tile by the expert, the tile's first A row, the end of the expert's
// rows and the N tile instead.
struct PairUnit {
  int tile, kb0, kb1, slice;
  int expert, row0, row_end, tn;  // the MoE form only (moe_pair_unit)
};

// The i-th unit of pair `pi` (false past its last).  Without the tail split,
// units pi, pi + npairs, ... of the tiles x splits list; with it, the pair's
// tail slice first (if it has one), then data-parallel tiles pi,
// pi + npairs, ... below dp_tiles.
__device__ __forceinline__ bool pair_unit(const Args& p, int pi, int npairs, int i, PairUnit& u) {
  if (p.tail.tail_splits > 1) {
    const int tail_units = (p.tiles_m * p.tiles_n - p.tail.dp_tiles) * p.tail.tail_splits;
    if (pi < tail_units) {
      if (i == 0) {
        u.tile = p.tail.dp_tiles + pi / p.tail.tail_splits;
        u.slice = pi % p.tail.tail_splits;
        u.kb0 = u.slice * p.tail.tail_kbps;
        u.kb1 = min(p.num_kb, u.kb0 + p.tail.tail_kbps);
        return true;
      }
      --i;
    }
    const int t = pi + i * npairs;
    if (t >= p.tail.dp_tiles) return false;
    u.tile = t;
    u.slice = 0;
    u.kb0 = 0;
    u.kb1 = p.num_kb;
    return true;
  }
  const int unit = pi + i * npairs;
  if (unit >= p.tiles_m * p.tiles_n * p.sk.splits) return false;
  u.tile = unit / p.sk.splits;
  u.slice = unit % p.sk.splits;
  u.kb0 = u.slice * p.sk.kb_per_split;
  u.kb1 = min(p.num_kb, u.kb0 + p.sk.kb_per_split);
  return true;
}

// The MoE form (grouped GEMM, whole K, no split): the i-th unit of pair pi
// in the compact list of non-empty 256-row tiles, expert by expert and M
// tiles fastest, so the pairs working at once share their expert's B tile.
// Expert e owns A rows [off[e], off[e + 1]) and B rows [e n, e n + n);
// p.moe.mt_max bounds every expert's M tiles and p.tiles_m = experts x
// mt_max.  A tile's rows past its expert's last are computed (the TMA reads
// the next expert's rows, or zeros past m) and never stored.
__device__ __forceinline__ bool moe_pair_unit(const Args& p, int pi, int npairs, int i, PairUnit& u) {
  int t = pi + i * npairs;
  const int experts = p.tiles_m / p.moe.mt_max;
  for (int e = 0; e < experts; ++e) {
    const int r0 = __ldg(p.moe.moe_off + e), r1 = __ldg(p.moe.moe_off + e + 1);
    int mt = r1 > r0 ? (r1 - r0 + kPairBM - 1) / kPairBM : 0;
    mt = mt < p.moe.mt_max ? mt : p.moe.mt_max;
    const int cnt = mt * p.tiles_n;
    if (t < cnt) {
      const int tm = t % mt;
      u.tn = t / mt;
      u.tile = 0;
      u.slice = 0;
      u.kb0 = 0;
      u.kb1 = p.num_kb;
      u.expert = e;
      u.row0 = r0 + tm * kPairBM;
      u.row_end = r1 < p.m ? r1 : p.m;
      return true;
    }
    t -= cnt;
  }
  return false;
}

template <bool MOE>
__device__ __forceinline__ bool next_unit(const Args& p, int pi, int npairs, int i, PairUnit& u) {
  if constexpr (MOE)
    return moe_pair_unit(p, pi, npairs, i, u);
  else
    return pair_unit(p, pi, npairs, i, u);
}

// pr: this CTA's rank within its pair; lead: the cluster rank of its pair's
// leader (clusters hold one pair, or the `splits` pairs of one tile).
template <bool MOE>
__device__ void produce_pair(PairStorage& s, const CUtensorMap* tmA, const CUtensorMap* tmB,
                             const Args& p, uint32_t pr, uint32_t lead) {
  const int npairs = gridDim.x >> 1;
  uint32_t stage = 0, phase = 0, issued = 0;
  bool ok = true;
  PairUnit u;
  for (int i = 0; ok && next_unit<MOE>(p, blockIdx.x >> 1, npairs, i, u); ++i) {
    int ya, yb;
    if constexpr (MOE) {
      ya = u.row0 + static_cast<int>(pr) * 128;
      yb = u.expert * p.n + u.tn * kPairBN + static_cast<int>(pr) * 128;
    } else {
      const int tm = u.tile % p.tiles_m, tn = u.tile / p.tiles_m;
      ya = tm * kPairBM + static_cast<int>(pr) * 128;
      yb = tn * kPairBN + static_cast<int>(pr) * 128;
    }
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

template <bool F8, bool MOE>
__device__ void mma_issue_pair(PairStorage& s, uint32_t tmem, const Args& p, uint32_t lead) {
  const uint16_t pair_mask = static_cast<uint16_t>(0x3u << lead);
  const int npairs = gridDim.x >> 1;
  constexpr uint32_t idesc = F8 ? idesc_e4m3(kPairBM, kPairBN) : idesc_i8(kPairBM, kPairBN);
  uint32_t stage = 0, phase = 0, abuf = 0, aphase = 0;
  bool ok = true;
  PairUnit u;
  for (int i = 0; ok && next_unit<MOE>(p, blockIdx.x >> 1, npairs, i, u); ++i) {
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
  const int S = p.tail.tail_splits;
  const int tt = u.tile - p.tail.dp_tiles;
  int* cnt = p.cnt + tt * 16 + region;
  int32_t* slots = p.tail.tail_ws + static_cast<int64_t>(tt) * S * 16 * kRegionInts;
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
    if (!F8 && p.asym.zp) apply_zp(p, row, colbase + ch * 32, va);
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
template <bool F8, bool MOE>
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
  for (int i = 0; next_unit<MOE>(p, blockIdx.x >> 1, npairs, i, u); ++i) {
    const int tile = u.tile;
    const bool tail = !MOE && p.tail.tail_splits > 1 && tile >= p.tail.dp_tiles;
    int row, colbase;
    bool rv;
    const float* swe = p.sw;  // this unit's channel scales (MoE: its expert's)
    if constexpr (MOE) {
      row = u.row0 + static_cast<int>(pr) * 128 + quad * 32 + lane;
      rv = row < u.row_end;
      colbase = u.tn * kPairBN + half * (kPairBN / 2);
      swe = p.sw + static_cast<int64_t>(u.expert) * p.n;
    } else {
      const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
      row = tm * kPairBM + static_cast<int>(pr) * 128 + quad * 32 + lane;
      rv = row < p.m;
      colbase = tn * kPairBN + half * (kPairBN / 2);
    }
    const float sa = (rv && p.out) ? __ldg(p.sa + row) : 0.0f;
    if (p.out) {
      const int c4 = colbase + lane * 4;  // n % 8 == 0: a group of 4 is all in or all out
      const float4 v4 = c4 < p.n ? __ldg(reinterpret_cast<const float4*>(swe + c4))
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
    } else if (F8 && !p.sk.csplit) {
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
        if (p.asym.zp) apply_zp(p, row, colbase + ch * 32, va);
        store32_tma(p, tmO, box, row - lane, colbase + ch * 32, sa, sws + ch * 32, va);
        tmem_ld_wait();
        if (ch + 2 < 4) tmem_ld_32x32b_x32(tb + (ch + 2) * 32, va);
        if (p.asym.zp) apply_zp(p, row, colbase + (ch + 1) * 32, vb);
        store32_tma(p, tmO, box, row - lane, colbase + (ch + 1) * 32, sa, sws + (ch + 1) * 32, vb);
        tmem_ld_wait();
      }
    } else if (p.sk.splits == 1) {
      tmem_ld_32x32b_x32(tb, va);
      tmem_ld_wait();
#pragma unroll
      for (int ch = 0; ch < 4; ch += 2) {
        tmem_ld_32x32b_x32(tb + (ch + 1) * 32, vb);
        if (p.asym.zp) apply_zp(p, row, colbase + ch * 32, va);
        if (rv) store32_channel(p, row, colbase + ch * 32, sa, sws + ch * 32, va);
        tmem_ld_wait();
        if (ch + 2 < 4) tmem_ld_32x32b_x32(tb + (ch + 2) * 32, va);
        if (p.asym.zp) apply_zp(p, row, colbase + (ch + 1) * 32, vb);
        if (rv) store32_channel(p, row, colbase + (ch + 1) * 32, sa, sws + (ch + 1) * 32, vb);
        tmem_ld_wait();
      }
    } else if (p.sk.csplit) {
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
      int32_t* acc_region = p.sk.ws + (static_cast<int64_t>(tile) * 16 + region) * kRegionInts;
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
        last = atomicAdd(p.cnt + tile * 16 + region, 1) == p.sk.splits - 1;
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
          if (p.asym.zp) apply_zp(p, row, colbase + ch * 32, va);
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
  const int tn = ((blockIdx.x >> 1) / p.sk.splits) / p.tiles_m;
  float* sws = s.sw_tile[warp - 2];
  int t = 0;
  for (int c = j + p.sk.splits * w2; c < kPairBN / 32 && t < 2; c += 2 * p.sk.splits, ++t) {
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
  const int tile = (blockIdx.x >> 1) / p.sk.splits;
  const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
  const float* sws = s.sw_tile[warp - 2];
  int t = 0;
  const int row = tm * kPairBM + h * 128 + quad * 32 + lane;
  const bool rv = row < p.m;
  const float sa = (rv && p.out) ? __ldg(p.sa + row) : 0.0f;
  const uint32_t base = smem_addr(&s.a[0][0]);
  constexpr uint32_t kSlotBytes = 32 * (kPairBN / 2) * 4;
  for (int c = j + p.sk.splits * w2; c < kPairBN / 32; c += 2 * p.sk.splits, ++t) {
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
        t4[o][q4] = o < p.sk.splits ? ld_dsmem_v4(map_to_rank(off + q4 * 32 * 16, peer))
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
    const int col0 = tn * kPairBN + c * 32;
    if (!F8 && p.asym.zp) apply_zp(p, row, col0, va);
    if (rv && col0 < p.n) store32_channel<F8>(p, row, col0, sa, sws + t * 32, va);
  }
}

template <bool F8, bool MOE = false>
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
    if (lane == 0) produce_pair<MOE>(s, &tmA, &tmB, p, pr, lead);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && pr == 0) mma_issue_pair<F8, MOE>(s, tmem, p, lead);
    __syncwarp();
  } else {
    epilogue_pair<F8, MOE>(s, tmem, p, pr, lead, &tmO);
  }
  if (p.sk.csplit) {
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

}  // namespace gemm
}  // namespace qk
