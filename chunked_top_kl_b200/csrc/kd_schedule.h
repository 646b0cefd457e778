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

constexpr int kMaxSplits = 16;   // column ranges per band in the forward pass (its partials)
constexpr int kMaxDzSplits = 64; // column ranges per band in the dZ recompute (no partials)

KD_HD int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct Raster {
  int m_tiles;          // row bands (one tile high)
  int n_tiles;          // 256-column tiles
  int splits;           // column ranges per band
  int tiles_per_split;  // tiles in the longest range
  int group_m;          // bands interleaved within one group of units
  int num_units;        // m_tiles * splits
};

// Unit u -> band m, range index split and column-tile range [n0, n1).
// Consecutive units (which run at the same time on different SMs) walk the
// bands of a group fastest, then the ranges, then the groups; so the SMs of
// one wave share column tiles (L2 reuse of the B operand) across group_m
// bands while each band's A tile is shared across the ranges.  Range lengths
// differ by at most one tile, so units of one wave stay in step.
KD_HD void decode_unit(const Raster& r, int u, int& m, int& split, int& n0, int& n1) {
  const int per_group = r.group_m * r.splits;
  const int g = u / per_group;
  const int gm0 = g * r.group_m;
  const int gsz = (r.group_m < r.m_tiles - gm0) ? r.group_m : (r.m_tiles - gm0);
  const int rr = u - g * per_group;
  m = gm0 + rr % gsz;
  split = rr / gsz;
  const int base = r.n_tiles / r.splits;
  const int extra = r.n_tiles - base * r.splits;
  n0 = split * base + (split < extra ? split : extra);
  n1 = n0 + base + (split < extra ? 1 : 0);
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

// Wide units (a problem whose every unit computes two neighbouring 256-column
// tiles at once): raster column n stands for column tiles [2n, 2n + count)
// of n_cols, count 2, or 1 for the last of an odd number.
KD_HD int wide_count(int n, int n_cols) { return 2 * n + 1 < n_cols ? 2 : 1; }

// Whether problem 0 of a joint launch (bands x n_cols tiles of k0 K blocks)
// should run wide units beside problem 1's U1 units of k1 K blocks on
// `groups`: a wide unit loads 3/4 of the operand bytes per MMA block, but
// holds twice the work, so it pays only when the busiest group's share, the
// larger of its problem-0 units and the launch's average, does not grow.
KD_HD bool wide_pays(int64_t bands, int64_t n_cols, int64_t k0, int64_t U1, int64_t k1, int groups) {
  const int64_t avg = ceil_div64(bands * n_cols * k0 + U1 * k1, groups);
  auto busiest = [&](int64_t U0, int64_t c0) {
    const int64_t own = ceil_div64(U0, groups) * c0;
    return own > avg ? own : avg;
  };
  return n_cols > 1 && busiest(bands * ceil_div64(n_cols, 2), 2 * k0) <= busiest(bands * n_cols, k0);
}

// Forward pass (and the dZ recompute): a unit is a band and a range of
// vocabulary tiles whose running log-sum-exp (or teacher-column cursor) one
// CTA carries.  Picks the number of ranges (<= max_splits; every range is
// non-empty) that minimises the tiles of the busiest of `grid` CTAs.  Units
// go round-robin and the longer ranges (n_tiles % S of them, one tile
// longer) come first in the unit order, so CTA 0 has both the most units,
// w = ceil(m S / grid), and the most long ones, ceil(m (n_tiles % S) / grid)
// at most: its load is w (n_tiles / S) + min(w, that).  (Exact for one band
// group, and it picks the best S for the grouped forward rasters too.)
//
// The B operand (the vocabulary rows) is the large one, so a wave should
// share each column tile among as many bands as it can: group_m bands walk
// the same ranges side by side, group_m = grid / 2 (two ranges per wave),
// capped so the group's A bands (band_bytes each, kept in L2) take at most
// half of `l2_budget`, and evened out over the groups.
KD_HD Raster forward_raster(int64_t m_tiles, int64_t n_tiles, int grid, int64_t band_bytes = 0,
                            int64_t l2_budget = 0, int max_splits = kMaxSplits) {
  int best_s = 1;
  int64_t best_cost = (int64_t)1 << 62;
  for (int s = 1; s <= max_splits && s <= n_tiles; ++s) {
    const int64_t w = ceil_div64(m_tiles * s, grid);
    const int64_t longs = ceil_div64(m_tiles * (n_tiles % s), grid);
    const int64_t cost = w * (n_tiles / s) + (longs < w ? longs : w);
    if (cost < best_cost) { best_cost = cost; best_s = s; }
  }
  Raster r;
  r.m_tiles = (int)m_tiles;
  r.n_tiles = (int)n_tiles;
  r.splits = best_s;
  r.tiles_per_split = (int)ceil_div64(n_tiles, best_s);
  int64_t gm = grid / 2;
  if (band_bytes > 0 && l2_budget > 0) {
    const int64_t cap = l2_budget / 2 / band_bytes;
    if (gm > cap) gm = cap;
  }
  if (gm < 1) gm = 1;
  if (gm > m_tiles) gm = m_tiles;
  gm = ceil_div64(m_tiles, ceil_div64(m_tiles, gm));
  r.group_m = (int)gm;
  r.num_units = (int)(m_tiles * r.splits);
  return r;
}

// Two problems in one launch.  Problem 0's U0 units (k0 K blocks each) go
// round-robin over `groups`, so groups [0, r), r = U0 % groups, run one more
// of them than the others.  Problem 1's U1 units (k1 K blocks each) are dealt
// so that groups running at the same time hold neighbouring units (which
// share operand tiles in L2) while every group's K blocks add up to about the
// same: first the groups >= r, free one problem-0 unit earlier, take
// wb ~ k0 / k1 units each, round-robin among themselves; then all groups take
// the rest round-robin, the class with less work so far first.
struct JointPlan {
  int r;     // groups [0, r) run one more problem-0 unit
  int wb;    // problem-1 units each group >= r runs before the others join
  int p2;    // first problem-1 unit dealt round-robin to all groups
  int rot;   // group g's place in that round-robin is (g - rot) mod groups
};

KD_HD JointPlan joint_plan(int64_t U0, int64_t k0, int64_t U1, int64_t k1, int groups) {
  JointPlan p;
  p.r = (int)(U0 % groups);
  const int64_t nb = groups - p.r;
  int64_t wb = 0;
  if (p.r > 0 && k1 > 0) {
    wb = (k0 + k1 / 2) / k1;
    if (wb > U1 / nb) wb = U1 / nb;
  }
  p.wb = (int)wb;
  p.p2 = (int)(wb * nb);
  p.rot = (wb * k1 <= k0) ? p.r : 0;
  return p;
}

// Problem-1 units of group g, and the i-th of them.
KD_HD int joint_count(const JointPlan& p, int64_t U1, int groups, int g) {
  const int first = g >= p.r ? p.wb : 0;
  const int64_t gp = (g - p.rot + groups) % groups;
  const int64_t left = U1 - p.p2 - gp;
  return first + (left > 0 ? (int)ceil_div64(left, groups) : 0);
}

KD_HD int joint_unit(const JointPlan& p, int groups, int g, int i) {
  if (g >= p.r) {
    if (i < p.wb) return (g - p.r) + i * (groups - p.r);
    i -= p.wb;
  }
  const int gp = (g - p.rot + groups) % groups;
  return p.p2 + gp + i * groups;
}

// Wave pacing.  In a round-robin over `groups`, the groups that hold their
// j-th unit at the same time share operand tiles; a counter per wave lets
// every group start its j-th unit only once all groups with a j-th unit have
// finished issuing their (j-1)-th.  Counters: problem 0's waves, then those
// of problem 1's early round-robin (joint plan, groups >= r), then those of
// its round-robin over all groups.  A joint launch is paced when its
// problem-1 units have at least kPaceKBlocks K blocks, or kPaceKBlocksWide
// when its problem-0 units are wide (measured: below these the waits cost
// more than the shared reads save; at the 8K Llama head's 32-deep dW tiles,
// wide dH units made the launch 11 % faster paced and 4 % slower unpaced).
constexpr int kPaceKBlocks = 64;
constexpr int kPaceKBlocksWide = 32;

// Counter index that group `group` waits on before its ord-th unit of
// problem `prob` (0 or 1), and the number of groups that arrive there
// (*expected); -1 when that unit starts its round-robin.  U1 = 0 and jp = {}
// for a launch of problem 0 alone.
KD_HD int wave_slot(int prob, int ord, int group, int groups, int U0, int U1, const JointPlan& jp,
                    int* expected) {
  auto clampg = [&](int64_t v) { return (int)(v < 0 ? 0 : (v > groups ? groups : v)); };
  const int w0 = (int)ceil_div64(U0, groups);                         // problem 0's waves
  if (prob == 0) {
    if (ord == 0) return -1;
    *expected = clampg((int64_t)U0 - (int64_t)ord * groups);
    return ord - 1;
  }
  if (group >= jp.r && ord < jp.wb) {
    if (ord == 0) return -1;
    *expected = groups - jp.r;
    return w0 + ord - 1;
  }
  const int j = ord - (group >= jp.r ? jp.wb : 0);
  if (j == 0) return -1;
  *expected = clampg((int64_t)U1 - jp.p2 - (int64_t)j * groups);
  return w0 + jp.wb + j - 1;
}

// Counters a launch needs: an upper bound of every index wave_slot returns, plus one.
KD_HD int64_t wave_slots_bound(int64_t U0, int64_t U1) { return 2 * (U0 + U1) + 4; }

}  // namespace kd
