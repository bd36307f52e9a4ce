// group_plan.h -- the work-unit schedule of the wide group-128 GEMM kernel,
// plain integer arithmetic shared by the kernel (device) and by the host
// planner, and compiled on its own by a CPU test of the schedule.
//
// T output tiles run on P CTAs.  Without the split, CTA c takes tiles c,
// c + P, ...  With it (r = T mod P tail tiles, 0 < 2 r <= P, T > P, at least
// two K groups), tail tile (T - r + j) is cut at group gmid: its first part
// is CTA j's first unit, its second part CTA (r + j)'s last unit, so every
// CTA runs (T - r) / P whole tiles and at most one part.
#pragma once

#ifdef __CUDACC__
#define QK_PLAN_FN __host__ __device__ __forceinline__
#else
#define QK_PLAN_FN inline
#endif

namespace qk {
namespace gemm {

// Groups [g0, g1) of output tile `tile`; part 0 whole, 1 the first part of a
// cut tile, 2 its second part.
struct GroupUnit {
  int tile, g0, g1, part;
};

// Number of tail tiles to cut (0: no split).
QK_PLAN_FN int group_split_count(int tiles, int groups, int num_sms) {
  if (num_sms <= 0 || tiles <= num_sms || groups < 2) return 0;
  const int r = tiles % num_sms;
  return (r > 0 && 2 * r <= num_sms) ? r : 0;
}

// The i-th unit of CTA c of P (false past its last).  r tail tiles cut at
// group gmid (r = 0: whole tiles only).
QK_PLAN_FN bool group_unit_at(int c, int P, int tiles, int r, int groups, int gmid, int i,
                              GroupUnit& u) {
  const int dp = tiles - r;
  if (c < r) {
    if (i == 0) {
      u.tile = dp + c;
      u.g0 = 0;
      u.g1 = gmid;
      u.part = 1;
      return true;
    }
    --i;
  }
  const int t = c + i * P;
  if (t < dp) {
    u.tile = t;
    u.g0 = 0;
    u.g1 = groups;
    u.part = 0;
    return true;
  }
  if (c >= r && c < 2 * r && i == (dp - c + P - 1) / P) {
    u.tile = dp + c - r;
    u.g0 = gmid;
    u.g1 = groups;
    u.part = 2;
    return true;
  }
  return false;
}

}  // namespace gemm
}  // namespace qk
