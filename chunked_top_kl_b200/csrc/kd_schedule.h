// Tile schedules shared by the host launch code and the GEMM kernel.
// Plain C++ (host and device); a CPU test compiles it with g++ and checks
// that every schedule covers every output tile exactly once.
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define KD_HD __host__ __device__ __forceinline__
#else
#define KD_HD inline
#endif

namespace kd {

constexpr int kMaxSplits = 16;   // column ranges per band in the forward pass

KD_HD int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct Raster {
  int m_tiles;          // 128-row bands
  int n_tiles;          // 256-column tiles
  int splits;           // column ranges per band
  int tiles_per_split;  // tiles in one range (the last may be shorter)
  int group_m;          // bands interleaved within one group of units
  int num_units;        // m_tiles * splits
};

// Unit u -> band m, range index split and column-tile range [n0, n1).
// Consecutive units (which run at the same time on different SMs) walk the
// bands of a group fastest, then the ranges, then the groups; so the SMs of
// one wave share column tiles (L2 reuse of the B operand) across group_m
// bands while each band's A tile is shared across the ranges.
KD_HD void decode_unit(const Raster& r, int u, int& m, int& split, int& n0, int& n1) {
  const int per_group = r.group_m * r.splits;
  const int g = u / per_group;
  const int gm0 = g * r.group_m;
  const int gsz = (r.group_m < r.m_tiles - gm0) ? r.group_m : (r.m_tiles - gm0);
  const int rr = u - g * per_group;
  m = gm0 + rr % gsz;
  split = rr / gsz;
  n0 = split * r.tiles_per_split;
  n1 = (n0 + r.tiles_per_split < r.n_tiles) ? (n0 + r.tiles_per_split) : r.n_tiles;
}

// One tile per unit; bands fastest (group_m = all bands) or column tiles
// fastest (group_m = 1).
KD_HD Raster tile_raster(int64_t m_tiles, int64_t n_tiles, bool bands_fastest) {
  Raster r;
  r.m_tiles = (int)m_tiles;
  r.n_tiles = (int)n_tiles;
  r.splits = (int)n_tiles;
  r.tiles_per_split = 1;
  r.group_m = bands_fastest ? (int)m_tiles : 1;
  r.num_units = (int)(m_tiles * n_tiles);
  return r;
}

// Forward pass: a unit is a band and a range of vocabulary tiles whose
// running log-sum-exp one CTA carries.  Picks the number of ranges
// (<= kMaxSplits) minimising waves x tiles-per-unit on `grid` CTAs; every
// range is non-empty.
inline Raster forward_raster(int64_t m_tiles, int64_t n_tiles, int grid) {
  int best_s = 1;
  int64_t best_cost = INT64_MAX;
  for (int s = 1; s <= kMaxSplits && s <= n_tiles; ++s) {
    const int64_t tps = ceil_div64(n_tiles, s);
    const int64_t se = ceil_div64(n_tiles, tps);
    const int64_t cost = ceil_div64(m_tiles * se, grid) * tps;
    if (cost < best_cost) { best_cost = cost; best_s = (int)se; }
  }
  Raster r;
  r.m_tiles = (int)m_tiles;
  r.n_tiles = (int)n_tiles;
  r.tiles_per_split = (int)ceil_div64(n_tiles, best_s);
  r.splits = (int)ceil_div64(n_tiles, r.tiles_per_split);
  int gm = grid / r.splits;
  r.group_m = gm < 1 ? 1 : (gm > m_tiles ? (int)m_tiles : gm);
  r.num_units = (int)(m_tiles * r.splits);
  return r;
}

// Two problems in one launch: problem 0's U0 units (k0 K blocks each) go
// round-robin over `groups`; problem 1's U1 units (k1 K blocks each) are cut
// into one contiguous range per group, [starts[g], starts[g+1]), sized so
// that every group's total K blocks are as equal as whole units allow
// (largest remainders first).  starts has groups + 1 entries.
inline void balance_ranges(int64_t U0, int64_t k0, int64_t U1, int64_t k1, int groups, int* starts) {
  const double target = (double)(U0 * k0 + U1 * k1) / groups;
  int64_t sum = 0;
  int64_t cnt[256];
  double frac[256];
  for (int g = 0; g < groups; ++g) {
    const int64_t n0 = g < U0 ? (U0 - g + groups - 1) / groups : 0;
    double want = (target - (double)(n0 * k0)) / (double)(k1 > 0 ? k1 : 1);
    if (want < 0) want = 0;
    cnt[g] = (int64_t)want;
    frac[g] = want - (double)cnt[g];
    sum += cnt[g];
  }
  while (sum < U1) {
    int best = 0;
    for (int g = 1; g < groups; ++g)
      if (frac[g] > frac[best]) best = g;
    cnt[best] += 1;
    frac[best] -= 1.0;
    sum += 1;
  }
  while (sum > U1) {
    int best = -1;
    for (int g = 0; g < groups; ++g)
      if (cnt[g] > 0 && (best < 0 || frac[g] < frac[best])) best = g;
    cnt[best] -= 1;
    frac[best] += 1.0;
    sum -= 1;
  }
  starts[0] = 0;
  for (int g = 0; g < groups; ++g) starts[g + 1] = starts[g] + (int)cnt[g];
}

}  // namespace kd
