// gemm_host.cuh -- host side of the tcgen05 GEMMs: tensor maps, occupancy
// queries, the split plans and workspace sizes, and the launches.
#pragma once

#include "gemm_group_pair.cuh"

namespace qk {
namespace gemm {

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
  static std::atomic<unsigned long long> done[16] = {};
  const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (done[slot].load(std::memory_order_acquire) & bit)) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess && bit) done[slot].fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

template <int BN = kChannelBN>
inline size_t channel_smem() {
  return sizeof(ChannelStorageT<BN>) + 1024;
}
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
  a.sk.splits = pl.splits;
  a.sk.kb_per_split = pl.kb_per_split;
  a.sk.csplit = pl.csplit;
  a.tail.dp_tiles = pl.dp_tiles;
  a.tail.tail_splits = pl.tail_splits;
  a.tail.tail_kbps = pl.tail_kbps;
  a.sk.ws = nullptr;
  a.cnt = nullptr;
  a.tail.tail_ws = nullptr;
  if ((pl.splits > 1 && !pl.csplit) || pl.tail_splits > 1) {
    a.cnt = static_cast<int*>(workspace);
    a.sk.ws = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + kCounterHeaderBytes);
    a.tail.tail_ws = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + kTailOffset);
  }
  CUtensorMap ta, tb, to;
  if (!cached_tmap(&ta, A, a.m, a.k, 128) || !cached_tmap(&tb, B, a.n, a.k, 128)) return 1;
  // bf16 out without c, outside split-K: TMA stores from shared memory
  a.tma_out = (a.out != nullptr && a.out_bf16 && a.c == nullptr && a.sk.splits == 1) ? 1 : 0;
  if (a.tma_out) {
    if (!cached_tmap(&to, a.out, a.m, a.n, 32, 1)) return 1;
  } else {
    to = ta;  // unused
  }
  const int ntiles = a.tiles_m * a.tiles_n * a.sk.splits;  // > pairs whenever the tail split is on
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
// counter header (zero before a call, zero after it), and each tail tile's
// running sums (scratch) from kTailOffset on, past the split-K accumulators
// that other calls need left zero (group_plan_workspace_bytes).
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

// ---------------------------------------------------------------- group-128 plans
// The wide 1-SM kernel's K split relies on every CTA of its grid being
// resident at once (a second part waits for a first part run by another
// CTA): checked with the occupancy query, once per device.
inline bool group_wide_resident(int dev, int grid) {
  static std::atomic<int> cache[64] = {};  // CTAs per SM (-1: unknown / failed)
  if (dev < 0 || dev >= 64) return false;
  int per_sm = cache[dev].load(std::memory_order_relaxed);
  if (per_sm == 0) {
    int n = 0;
    if (cudaFuncSetAttribute(gemm_i8_group_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(group_wide_smem())) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gemm_i8_group_wide_kernel, kGroupWideThreads,
                                                      group_wide_smem()) != cudaSuccess) {
      cudaGetLastError();
      n = -1;
    }
    per_sm = n > 0 ? n : -1;
    cache[dev].store(per_sm, std::memory_order_relaxed);
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
  return per_sm > 0 && static_cast<int64_t>(per_sm) * sms >= grid;
}

inline size_t group_pair_smem() { return sizeof(GroupPairStorage) + 1024; }

// The group-128 pair kernel moves registers between warpgroups with
// setmaxnreg; the budgets only add up if the compiled kernel launches with
// at least kGpLaunchRegs registers per thread.  Checked once per device.
inline bool group_pair_ok(int dev) {
  static std::atomic<int> cache[64] = {};
  if (dev < 0 || dev >= 64) return false;
  int known = cache[dev].load(std::memory_order_relaxed);
  if (known == 0) {
    cudaFuncAttributes fa;
    const bool ok = cudaFuncGetAttributes(&fa, gemm_i8_group_pair_kernel) == cudaSuccess &&
                    fa.numRegs >= kGpLaunchRegs && fa.numRegs * kGpThreads <= 65536;
    if (!ok) cudaGetLastError();
    known = ok ? 1 : -1;
    cache[dev].store(known, std::memory_order_relaxed);
  }
  return known > 0;
}

// Pairs of the group-128 pair kernel that are resident at once (queried once
// per device; 0 when it cannot run).  The grid never exceeds it, so every
// pair of a launch is resident together, which the K split's wait needs.
inline int max_group_pairs(int dev, int num_sms) {
  static std::atomic<int> cache[64] = {};
  if (dev < 0 || dev >= 64) return 0;
  const int known = cache[dev].load(std::memory_order_relaxed);
  if (known != 0) return known > 0 ? known : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms - num_sms % 2), 1, 1);
  cfg.blockDim = dim3(kGpThreads, 1, 1);
  cfg.dynamicSmemBytes = group_pair_smem();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaFuncSetAttribute(gemm_i8_group_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(group_pair_smem())) != cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, gemm_i8_group_pair_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  n = n < num_sms / 2 ? n : num_sms / 2;
  cache[dev].store(n > 0 ? n : -1, std::memory_order_relaxed);
  return n > 0 ? n : 0;
}

// Which group-128 kernel runs an output-only problem, and how many tiles of
// its last wave are cut at the middle group.  m > 128: the CTA-pair kernel
// (256 x 256 tiles on the co-resident pairs); otherwise, or when the pair
// kernel's register budget does not hold, the wide 1-SM kernel (128 x 256).
struct GroupPlan {
  bool pair;
  int workers;  // pairs, or CTAs
  int tiles;
  int r;        // cut tail tiles (0: whole tiles only)
};

inline GroupPlan group_plan(int m, int n, int k, int dev, int num_sms) {
  GroupPlan g;
  const int groups = k / 128;
  const int pairs = m > BM && group_pair_ok(dev) ? max_group_pairs(dev, num_sms) : 0;
  if (pairs > 0) {
    g.pair = true;
    g.tiles = ((m + 255) / 256) * ((n + kGpBN - 1) / kGpBN);
    g.workers = g.tiles < pairs ? g.tiles : pairs;
    g.r = g.tiles <= 2 * kGroupWideMaxSplit ? group_split_count(g.tiles, groups, pairs) : 0;
    return g;
  }
  g.pair = false;
  g.tiles = ((m + BM - 1) / BM) * ((n + kGroupWideBN - 1) / kGroupWideBN);
  g.workers = g.tiles < num_sms ? g.tiles : num_sms;
  g.r = group_split_tiles(m, n, k, num_sms);
  if (g.r > 0 && !group_wide_resident(dev, g.workers)) g.r = 0;
  return g;
}

// Bytes of the group kernels' workspace: counters in the 4 KB header (one per
// cut tile and CTA of a pair, or per cut tile), and the running sums past the
// split-K accumulators (256 KB per cut pair tile, 128 KB per cut 1-SM tile).
inline size_t group_plan_flag_bytes(const GroupPlan& g) {
  const size_t n = static_cast<size_t>(g.r) * (g.pair ? 2 : 1) * sizeof(int);
  return (n + 255) & ~static_cast<size_t>(255);
}
inline size_t group_plan_workspace_bytes(const GroupPlan& g) {
  if (g.r <= 0) return 0;
  return kTailOffset + static_cast<size_t>(g.r) * (g.pair ? 2u : 1u) * BM * kGroupWideBN * sizeof(float);
}
static_assert(2 * kGroupWideMaxSplit * sizeof(int) <= kCounterHeaderBytes,
              "group split counters of the pair kernel fit the counter header");

// 0 ok, 1 tensor-map failure, 2 CUDA error
// Largest number of co-resident clusters of `cluster` CTAs of the 1-SM
// channel kernel of tile width BN (queried once per device, width and size;
// 0 when it cannot run).
template <int BN>
inline int max_channel_clusters(int dev, int cluster) {
  static std::atomic<int> cache[64][5] = {};
  if (dev < 0 || dev >= 64 || cluster < 2 || cluster > 4) return 0;
  const int known = cache[dev][cluster].load(std::memory_order_relaxed);
  if (known != 0) return known > 0 ? known : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cluster) * 16, 1, 1);
  cfg.blockDim = dim3(kChannelThreads, 1, 1);
  cfg.dynamicSmemBytes = channel_smem<BN>();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  auto* kernel = gemm_i8_channel_kernel<false, false, BN>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(channel_smem<BN>())) != cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cache[dev][cluster].store(n > 0 ? n : -1, std::memory_order_relaxed);
  return n > 0 ? n : 0;
}

// Split-K plan of the 1-SM channel kernel: with fewer 128 x BN tiles than
// half the SMs, cut K into S <= 4 slices (>= 8 K blocks each), one CTA per
// slice, the S CTAs of a tile forming one cluster whose partials meet in
// distributed shared memory.  S = 1 when the clusters would not all be
// co-resident.  Of the two tile widths, 128 is taken when its plan puts
// more CTAs to work than 256's, or as many with at most 16 K blocks per
// slice, where the fewer slices' shorter reduction outweighs the narrow
// tile's extra activation reads (96 x 8192 x 4096: 12.7 us as 64 narrow
// tiles x 2 slices, 14.5 us as 32 wide tiles x 4; at 256 x 4096 x 14336,
// 56 K blocks per narrow slice, the wide plan wins).
struct ChannelPlan {
  int tiles, splits, kb_per_split, bn;
};

template <int BN>
inline ChannelPlan channel_plan_bn(int m, int n, int k, int num_sms, int dev) {
  ChannelPlan pl;
  pl.bn = BN;
  pl.tiles = ((m + BM - 1) / BM) * ((n + BN - 1) / BN);
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
    if (ns > 1 && max_channel_clusters<BN>(dev, ns) >= pl.tiles) {
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

inline ChannelPlan channel_plan(int m, int n, int k, int num_sms, int dev) {
  const ChannelPlan wide = channel_plan_bn<256>(m, n, k, num_sms, dev);
  const ChannelPlan narrow = channel_plan_bn<128>(m, n, k, num_sms, dev);
  const int ctas_wide = wide.tiles * wide.splits, ctas_narrow = narrow.tiles * narrow.splits;
  if (ctas_narrow > num_sms) return wide;
  if (ctas_narrow > ctas_wide) return narrow;
  if (ctas_narrow == ctas_wide && narrow.splits < wide.splits && narrow.kb_per_split <= 16) return narrow;
  return wide;
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

// `workspace`: group_plan_workspace_bytes(group_plan(...)) bytes for the
// wide group kernel's split (null: whole tiles only); unused otherwise.
inline int launch(Args a, const int8_t* A, const int8_t* B, bool group, int dev, int num_sms,
                  cudaStream_t stream, cudaError_t* err, void* workspace = nullptr) {
  // group mode without the int32 sums: the 128 x 256 kernel
  const bool wide = group && a.c == nullptr && group_wide_ok(dev);
  ChannelPlan cpl = {};
  if (!group) cpl = channel_plan(a.m, a.n, a.k, num_sms, dev);
  const int bn = group ? (wide ? kGroupWideBN : kGroupBN) : cpl.bn;
  a.tiles_m = (a.m + BM - 1) / BM;
  a.tiles_n = (a.n + bn - 1) / bn;
  a.num_kb = (a.k + BK - 1) / BK;
  a.groups = group ? a.k / 128 : 0;
  a.sk.splits = 1;
  a.sk.kb_per_split = a.num_kb;
  a.sk.csplit = 0;
  a.tail.tail_splits = 1;
  if (!group && cpl.splits > 1) {
    a.sk.splits = cpl.splits;
    a.sk.kb_per_split = cpl.kb_per_split;
    a.sk.csplit = 1;
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
  const int grid = a.sk.csplit ? ntiles * a.sk.splits : (ntiles < num_sms ? ntiles : num_sms);
  cudaError_t e;
  if (!group) {
    const unsigned cluster = a.sk.csplit ? static_cast<unsigned>(a.sk.splits) : 1u;
    if (bn == 128) {
      const size_t smem = channel_smem<128>();
      auto* kernel = a.f8 ? gemm_i8_channel_kernel<true, false, 128> : gemm_i8_channel_kernel<false, false, 128>;
      e = set_smem_once(kernel, dev, a.f8 ? 10 : 9, smem);
      if (e == cudaSuccess)
        e = launch_pdl(kernel, dim3(grid), dim3(kChannelThreads), smem, stream, cluster, ta, tb, to, a);
    } else {
      const size_t smem = channel_smem();
      auto* kernel = a.f8 ? gemm_i8_channel_kernel<true> : gemm_i8_channel_kernel<false>;
      e = set_smem_once(kernel, dev, a.f8 ? 5 : 1, smem);
      if (e == cudaSuccess)
        e = launch_pdl(kernel, dim3(grid), dim3(kChannelThreads), smem, stream, cluster, ta, tb, to, a);
    }
  } else {
    if (wide) {
      const GroupPlan gp = group_plan(a.m, a.n, a.k, dev, num_sms);
      if (gp.pair) {
        // 256 x 256 tiles on CTA pairs
        a.tiles_m = (a.m + 255) / 256;
        a.tiles_n = (a.n + kGpBN - 1) / kGpBN;
        CUtensorMap tpa, tpb;
        if (!cached_tmap(&tpa, A, a.m, a.k, 128) || !cached_tmap(&tpb, B, a.n, a.k, 128)) return 1;
        a.gcut.gsplit = workspace ? gp.r : 0;
        a.gcut.gmid = a.groups / 2;
        a.gcut.gflag = static_cast<int*>(workspace);
        a.gcut.gstate = a.gcut.gsplit ? reinterpret_cast<float*>(static_cast<char*>(workspace) + kTailOffset)
                            : nullptr;
        // bf16 out without c: TMA stores from shared memory
        a.tma_out = (a.out != nullptr && a.out_bf16 && a.c == nullptr) ? 1 : 0;
        CUtensorMap tpo = tpa;  // unused unless tma_out
        if (a.tma_out && !cached_tmap(&tpo, a.out, a.m, a.n, 32, 1)) return 1;
        const size_t smem = group_pair_smem();
        e = set_smem_once(gemm_i8_group_pair_kernel, dev, 8, smem);
        if (e == cudaSuccess)
          e = launch_pdl(gemm_i8_group_pair_kernel, dim3(2 * gp.workers), dim3(kGpThreads), smem, stream,
                         2, tpa, tpb, tpo, a);
        *err = e;
        return e == cudaSuccess ? 0 : 2;
      }
      a.gcut.gsplit = workspace ? gp.r : 0;
      a.gcut.gmid = a.groups / 2;
      a.gcut.gflag = static_cast<int*>(workspace);
      a.gcut.gstate = a.gcut.gsplit ? reinterpret_cast<float*>(static_cast<char*>(workspace) + kTailOffset)
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

// MoE grouped GEMM on the CTA-pair kernel (MOE form): 256-row pair tiles over
// the compact list of each expert's tiles (moe_pair_unit), whole K, per
// channel, direct stores (rows past an expert's last are not stored).
// mt_max bounds every expert's 256-row tiles.  0 ok, 1 tensor-map failure,
// 2 CUDA error.
inline int launch_moe_pair(Args a, const int8_t* A, const int8_t* B, int experts, int mt_max,
                           const int32_t* off, int dev, int num_sms, cudaStream_t stream,
                           cudaError_t* err) {
  a.moe.mt_max = mt_max;
  a.moe.moe_off = off;
  a.tiles_m = experts * mt_max;
  a.tiles_n = (a.n + kPairBN - 1) / kPairBN;
  a.num_kb = (a.k + BK - 1) / BK;
  a.groups = 0;
  a.sk.splits = 1;
  a.sk.kb_per_split = a.num_kb;
  a.sk.csplit = 0;
  a.tail.tail_splits = 1;
  a.tma_out = 0;
  a.c = nullptr;
  CUtensorMap ta, tb;
  if (!cached_tmap(&ta, A, a.m, a.k, 128) || !cached_tmap(&tb, B, experts * a.n, a.k, 128)) return 1;
  const int pairs = max_pairs(dev, num_sms);
  const int64_t units = static_cast<int64_t>(a.tiles_m) * a.tiles_n;  // an upper bound
  const int grid_pairs = units < pairs ? static_cast<int>(units) : pairs;
  cudaError_t e = set_smem_once(gemm_i8_pair_kernel<false, true>, dev, 11, pair_smem());
  if (e == cudaSuccess)
    e = launch_pdl(gemm_i8_pair_kernel<false, true>, dim3(2 * grid_pairs), dim3(kPairThreads), pair_smem(),
                   stream, 2u, ta, tb, ta, a);
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
  a.moe.mt_max = mt_max;
  a.moe.moe_off = off;
  a.tiles_m = experts * mt_max;
  a.tiles_n = (a.n + kChannelBN - 1) / kChannelBN;
  a.num_kb = (a.k + BK - 1) / BK;
  a.groups = 0;
  a.sk.splits = 1;
  a.sk.kb_per_split = a.num_kb;
  a.sk.csplit = 0;
  a.tail.tail_splits = 1;
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
