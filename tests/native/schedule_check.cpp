// Enumerates the GEMM tile schedules of kd_schedule.h for a list of shapes
// and checks that every output tile is visited exactly once, that every
// unit has a non-empty column range, and that the forward schedule keeps
// within its split limit.  Prints "OK <cases>" or the first failure.
#include <cstdio>
#include <vector>

#include "../../chunked_top_kl_b200/csrc/kd_schedule.h"

using namespace kd;

static bool check(const Raster& r, const char* what, long a, long b, long c) {
  if (r.num_units != r.m_tiles * r.splits) { printf("FAIL %s units %ld %ld %ld\n", what, a, b, c); return false; }
  std::vector<int> seen((size_t)r.m_tiles * r.n_tiles, 0);
  for (int u = 0; u < r.num_units; ++u) {
    int m, s, n0, n1;
    decode_unit(r, u, m, s, n0, n1);
    if (m < 0 || m >= r.m_tiles || s < 0 || s >= r.splits || n0 < 0 || n0 >= n1 || n1 > r.n_tiles) {
      printf("FAIL %s unit %d -> m %d s %d [%d,%d) for %ld %ld %ld\n", what, u, m, s, n0, n1, a, b, c);
      return false;
    }
    for (int n = n0; n < n1; ++n) seen[(size_t)m * r.n_tiles + n]++;
  }
  for (size_t i = 0; i < seen.size(); ++i)
    if (seen[i] != 1) { printf("FAIL %s tile %zu seen %d for %ld %ld %ld\n", what, i, seen[i], a, b, c); return false; }
  return true;
}

// A wide problem's raster (two column tiles per raster column): every
// (band, column tile) exactly once.
static bool check_wide(long m_tiles, long n_cols) {
  const Raster r = tile_raster(m_tiles, ceil_div64(n_cols, 2), false);
  std::vector<int> seen((size_t)(m_tiles * n_cols), 0);
  for (int u = 0; u < r.num_units; ++u) {
    int m, s, n0, n1;
    decode_unit(r, u, m, s, n0, n1);
    for (int n = n0; n < n1; ++n)
      for (int h = 0; h < wide_count(n, (int)n_cols); ++h) {
        const long c = 2l * n + h;
        if (m < 0 || m >= m_tiles || c >= n_cols) { printf("FAIL wide unit %d -> m %d col %ld\n", u, m, c); return false; }
        seen[(size_t)(m * n_cols + c)]++;
      }
  }
  for (size_t i = 0; i < seen.size(); ++i)
    if (seen[i] != 1) { printf("FAIL wide tile %zu seen %d (%ld x %ld)\n", i, seen[i], m_tiles, n_cols); return false; }
  return true;
}

int main() {
  const long Ns[] = {1, 127, 128, 129, 512, 1000, 4096, 8192, 32768, 65536, 262144};
  const long Vs[] = {1, 24, 255, 256, 257, 4096, 32000, 128256, 201088};
  const long ds[] = {8, 72, 256, 2048, 2880, 3072};
  const long chunks[] = {1, 64, 128, 1000, 1024, 2048, 4096};
  const int grids[] = {1, 7, 148};
  int cases = 0;
  for (long N : Ns)
    for (long V : Vs)
      for (int g : grids)
        for (long d : ds) {
          Raster r = forward_raster(ceil_div64(N, 128), ceil_div64(V, 256), g, 256 * d * 2, 126l << 20);
          if (r.splits > kMaxSplits) { printf("FAIL splits %d\n", r.splits); return 1; }
          if (r.group_m < 1 || r.group_m > r.m_tiles) { printf("FAIL group_m\n"); return 1; }
          if (!check(r, "fwd", N, V, g)) return 1;
          // the dZ recompute's raster: more ranges allowed, no band groups capped by L2
          Raster rz = forward_raster(ceil_div64(N, 128), ceil_div64(V, 256), g, 0, 0, kMaxDzSplits);
          if (rz.splits > kMaxDzSplits) { printf("FAIL dz splits %d\n", rz.splits); return 1; }
          if (!check(rz, "dzr", N, V, g)) return 1;
          cases += 2;
        }
  for (long C : chunks)
    for (long V : Vs)
      for (long d : ds) {
        if (!check(tile_raster(ceil_div64(C, 128), ceil_div64(V, 256), true), "dz", C, V, d)) return 1;
        if (!check(tile_raster(ceil_div64(C, 128), ceil_div64(d, 256), true), "dh", C, V, d)) return 1;
        if (!check(tile_raster(ceil_div64(V, 128), ceil_div64(d, 256), false), "dw", C, V, d)) return 1;
        if (!check_wide(ceil_div64(C, 256), ceil_div64(d, 256))) return 1;
        cases += 4;
      }
  // joint launches: every problem-1 unit dealt exactly once; when there are
  // enough of them to even out the groups, no group's K blocks differ from
  // another's by more than 1.5 problem-1 units
  const long U0s[] = {0, 1, 16, 32, 96, 192, 400};
  const long k0s[] = {1, 45, 501, 3142, 6284};
  const long U1s[] = {0, 1, 12, 9432, 6012};
  const long k1s[] = {1, 16, 64};
  std::vector<int> seen;
  for (long U0 : U0s)
    for (long k0 : k0s)
      for (long U1 : U1s)
        for (long k1 : k1s)
          for (int g : {1, 7, 74, 148}) {
            const JointPlan p = joint_plan(U0, k0, U1, k1, g);
            seen.assign((size_t)U1, 0);
            long lo = -1, hi = -1;
            for (int i = 0; i < g; ++i) {
              const int n = joint_count(p, U1, g, i);
              for (int j = 0; j < n; ++j) {
                const int u = joint_unit(p, g, i, j);
                if (u < 0 || u >= U1) { printf("FAIL joint unit %d of %ld\n", u, U1); return 1; }
                ++seen[(size_t)u];
              }
              const long n0 = i < U0 ? (U0 - i + g - 1) / g : 0;
              const long tot = n0 * k0 + (long)n * k1;
              lo = lo < 0 || tot < lo ? tot : lo;
              hi = tot > hi ? tot : hi;
            }
            for (long u = 0; u < U1; ++u)
              if (seen[(size_t)u] != 1) { printf("FAIL joint seen %d\n", seen[(size_t)u]); return 1; }
            const long r = U0 % g;
            const bool enough = r == 0 || (long)p.wb == (k0 + k1 / 2) / k1;
            if (enough && U1 >= p.p2 + g && 2 * (hi - lo) > 3 * k1) {
              printf("FAIL joint balance U0 %ld k0 %ld U1 %ld k1 %ld g %d: %ld..%ld\n", U0, k0, U1, k1, g, lo, hi);
              return 1;
            }
            ++cases;
          }
  // wave pacing: every counter a group waits on receives exactly the number
  // of arrivals it waits for (else the barrier would time out), all waits
  // on one counter expect the same number, and indices stay in bounds
  const long ks0[] = {1, 45, 3142, 6284};
  for (long U0 : U0s)
    for (long k0 : ks0)
      for (long U1 : U1s)
        for (long k1 : k1s)
          for (int g : {1, 7, 74, 148}) {
            const JointPlan p = joint_plan(U0, k0, U1, k1, g);
            const long cap = wave_slots_bound(U0, U1);
            std::vector<int> arrivals((size_t)cap, 0), want((size_t)cap, -1);
            for (int grp = 0; grp < g; ++grp) {
              const long n0 = grp < U0 ? (U0 - grp + g - 1) / g : 0;
              const int n1 = joint_count(p, U1, g, grp);
              for (int prob = 0; prob < 2; ++prob)
                for (long ord = 0; ord < (prob == 0 ? n0 : n1); ++ord) {
                  int e = 0;
                  const int slot = wave_slot(prob, (int)ord, grp, g, (int)U0, (int)U1, p, &e);
                  if (slot < 0) continue;
                  if (slot >= cap) { printf("FAIL pace slot %d >= %ld\n", slot, cap); return 1; }
                  if (want[(size_t)slot] >= 0 && want[(size_t)slot] != e) { printf("FAIL pace expected\n"); return 1; }
                  want[(size_t)slot] = e;
                  ++arrivals[(size_t)slot];
                }
            }
            for (long i = 0; i < cap; ++i)
              if (want[(size_t)i] >= 0 && arrivals[(size_t)i] != want[(size_t)i]) {
                printf("FAIL pace U0 %ld k0 %ld U1 %ld k1 %ld g %d: slot %ld %d arrivals for %d\n", U0, k0, U1, k1,
                       g, i, arrivals[(size_t)i], want[(size_t)i]);
                return 1;
              }
            ++cases;
          }
  // wide dH units on 74 CTA pairs: taken at the 32K GPT-OSS head (4096-token
  // chunks, d = 2880, V = 201,088: 96 wide units), the 8K Llama head's
  // 2048-token chunks (d = 3072, V = 128,256: 48) and the long-context sweep's
  // 4096-token chunks (d = 2048: 64); not at the packed 4K head's 1024-token
  // chunks (d = 2048, V = 32,000: 16 wide units of twice the launch's average
  // work), never with one column tile
  if (!wide_pays(16, 12, 3142, 786 * 12, 64, 74)) { printf("FAIL wide gptoss\n"); return 1; }
  if (!wide_pays(8, 12, 2004, 501 * 12, 32, 74)) { printf("FAIL wide llama\n"); return 1; }
  if (!wide_pays(16, 8, 2004, 501 * 8, 64, 74)) { printf("FAIL wide sweep\n"); return 1; }
  if (wide_pays(4, 8, 500, 125 * 8, 16, 74)) { printf("FAIL wide packed\n"); return 1; }
  if (wide_pays(16, 1, 3142, 786, 64, 74)) { printf("FAIL wide one column\n"); return 1; }
  // the GPU parity case for wide units with an odd column count (N = 4096,
  // d = 2640: 11 column tiles, the last 80 columns wide, V = 2048, one
  // 4096-token chunk) takes them
  if (!wide_pays(16, 11, 32, 8 * 11, 64, 74)) { printf("FAIL wide odd case\n"); return 1; }
  cases += 6;
  printf("OK %d\n", cases);
  return 0;
}
