// CPU check of the wide group-128 kernel's work-unit schedule (group_plan.h,
// the same header the kernel includes): for T tiles of G groups on P CTAs,
// every (tile, group) is computed by exactly one unit; a cut tile's first
// part runs on another CTA than its second part and, counting each CTA's
// units in tile-times, ends before the second part starts; no CTA runs more
// than ceil(T / P) tile-times, and with the split the longest CTA runs
// (T - r) / P + 1/2 of them.  Usage: group_plan_check T G P; prints "ok" and
// the longest CTA's tile-times, or the first violation.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "group_plan.h"

using qk::gemm::GroupUnit;

int main(int argc, char** argv) {
  if (argc != 4) return 2;
  const int T = std::atoi(argv[1]), G = std::atoi(argv[2]), P0 = std::atoi(argv[3]);
  const int P = T < P0 ? T : P0;  // the launch's grid
  const int r = qk::gemm::group_split_count(T, G, P0);
  const int gmid = G / 2;
  std::vector<int> seen(static_cast<size_t>(T) * G, 0);
  std::vector<double> end_first(T, -1.0), start_second(T, -1.0);
  std::vector<int> cta_first(T, -1), cta_second(T, -1);
  double longest = 0.0;
  for (int c = 0; c < P; ++c) {
    double t = 0.0;  // this CTA's elapsed tile-times
    GroupUnit u;
    for (int i = 0; qk::gemm::group_unit_at(c, P, T, r, G, gmid, i, u); ++i) {
      if (u.tile < 0 || u.tile >= T || u.g0 < 0 || u.g1 > G || u.g0 >= u.g1) {
        std::printf("bad unit: cta %d unit %d tile %d groups [%d, %d)\n", c, i, u.tile, u.g0, u.g1);
        return 1;
      }
      for (int g = u.g0; g < u.g1; ++g) ++seen[static_cast<size_t>(u.tile) * G + g];
      const double len = static_cast<double>(u.g1 - u.g0) / G;
      if (u.part == 1) {
        end_first[u.tile] = t + len;
        cta_first[u.tile] = c;
      } else if (u.part == 2) {
        start_second[u.tile] = t;
        cta_second[u.tile] = c;
      }
      t += len;
      if (i > T) {
        std::printf("unit list does not end: cta %d\n", c);
        return 1;
      }
    }
    if (t > longest) longest = t;
  }
  for (size_t x = 0; x < seen.size(); ++x)
    if (seen[x] != 1) {
      std::printf("tile %zu group %zu computed %d times\n", x / G, x % G, seen[x]);
      return 1;
    }
  for (int tile = 0; tile < T; ++tile) {
    if ((cta_first[tile] < 0) != (cta_second[tile] < 0)) {
      std::printf("tile %d has one part only\n", tile);
      return 1;
    }
    if (cta_first[tile] >= 0 &&
        (cta_first[tile] == cta_second[tile] || end_first[tile] > start_second[tile])) {
      std::printf("tile %d: second part (cta %d, at %.3f) before the first ends (cta %d, %.3f)\n",
                  tile, cta_second[tile], start_second[tile], cta_first[tile], end_first[tile]);
      return 1;
    }
  }
  const double whole = static_cast<double>((T + P - 1) / P);
  if (longest > whole + 1e-9) {
    std::printf("longest CTA %.3f tile-times, whole tiles take %.0f\n", longest, whole);
    return 1;
  }
  if (r > 0) {
    const double expect = static_cast<double>((T - r) / P) + static_cast<double>(G - gmid) / G;
    if (longest > expect + 1e-9) {
      std::printf("longest CTA %.3f tile-times, expected %.3f with the split\n", longest, expect);
      return 1;
    }
  }
  std::printf("ok %d %.4f\n", r, longest);
  return 0;
}
