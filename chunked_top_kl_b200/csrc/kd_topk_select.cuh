// Teacher top-K cache writer, selection step: for each row of a block of
// fp32 logits, the K largest values and their column indices, largest first,
// equal values in increasing column order (the order in which an offline
// cache lists a position's top-K teacher logits).
//
// One CTA per row, values mapped to order-preserving 32-bit keys.  The
// threads stream 16-byte loads (kSelVec of them in flight per thread) and a
// value becomes a candidate, appended to a shared-memory list, when its key is
// at least the current threshold tau.  tau is always the K-th largest key
// among a subset of the row's values, so a value below it is beaten by K
// others and can never be in the top K, while every value at or above the
// final tau is on the list.
//
// Which values are streamed.  The logits GEMM also writes, per row and
// 256-column tile, the key of the tile's largest value (EpiZ32).  With at
// least K tiles, tau starts at the K-th largest of these maxima (a radix
// select over shared memory): the K tiles with the largest maxima hold K
// values at or above it, so every value at or above the row's K-th largest
// is at or above tau and lies in a tile whose maximum is too, and only those
// tiles are read: about K of the row's tiles for logits in no particular
// order (at V = 201,088 and K = 100, 1/8 of the row).  Without the maxima, or
// with fewer than K tiles, the whole row is streamed (consecutive threads on
// consecutive addresses), and the first block sets tau to the smallest, over
// the warps, of each warp's ceil(K/warps)-th largest lane maximum (each warp
// then holds that many distinct values at or above it).
//
// Either way tau is then raised to the exact K-th largest key of the list
// after the first block, and whenever the threads meet (every kSelSegment
// blocks) with the list past a quarter of its capacity, and the list is
// compacted.  A thread first compares the maximum of its values with tau in
// floats and only then looks at single values, so after the first blocks a
// value costs a load and a max.  At the end the list is cut to the keys at or
// above its K-th largest and sorted by (key desc, column asc).
//
// For logits in no particular order the list stays small.  Rows where it
// overflows (more candidates in one segment than the list holds: values
// rising along the row, heavy ties, or, streaming the whole row, K above 32
// per warp, where the first block has no threshold and fills the list) are
// selected by the exact fallback below, which reads the whole row again: a
// histogram of the top 12 key bits locates the bin of the K-th largest value;
// when the values in or above it fit the sort buffer they are copied and
// sorted, otherwise a radix select (12 + 8 more bits) finds the K-th largest
// key and a collection pass takes every value above it and, of those equal
// to it, the ones with the lowest column indices (warps own contiguous column
// ranges and read them 32 columns at a time; ballots and the counts of the
// warps before order the ties).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "kd_small_kernels.cuh"

namespace kd {

constexpr int kSelectThreads = 256;
constexpr int kSelWarps = kSelectThreads / 32;
constexpr int kMaxTopK = 512;
constexpr int kSelVec = 8;           // float4 loads per thread per block of the row
constexpr int kSelBlock = kSelectThreads * kSelVec;   // float4s per block (8192 values)
constexpr int kSelSegment = 8;       // blocks between two meetings of the threads
constexpr int kSelTile = 256;        // columns per tile maximum (the logits GEMM's tile width)
constexpr int kSelTilesPerBlock = kSelBlock / (kSelTile / 4);   // tiles per block of the tile route
static_assert(kSelTile / 4 == 64 && kSelectThreads % 64 == 0,
              "the tile route reads a tile as 64 float4s, one per thread of a 64-thread group");
constexpr int kSelCap = 2048;        // candidate list (power of two, >= 2 kMaxTopK)
constexpr int kCandCap = 2048;       // fallback sort buffer (power of two, >= kMaxTopK)

// A (key, column) pair as one sortable word: larger key first, then lower column.
__device__ __forceinline__ unsigned long long pack_pair(uint32_t k, int v) {
  return ((unsigned long long)k << 32) | (unsigned long long)(0xffffffffu - (uint32_t)v);
}

__device__ __forceinline__ uint32_t pair_key(unsigned long long e) { return (uint32_t)(e >> 32); }

// Descending bitonic sort of s[0, P), P a power of two (all threads).
__device__ __forceinline__ void bitonic_sort_desc(unsigned long long* s, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < P; i += kSelectThreads) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long a = s[i], b = s[j];
          if (desc ? (a < b) : (a > b)) {
            s[i] = b;
            s[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Shared state of the selection of one row.  The fallback sorts in the
// candidate list (its first kCandCap entries) and keeps its own histogram;
// until a row falls back, the tile route keeps its selected tiles there.
struct SelShared {
  unsigned long long list[kSelCap];     // candidates (key, column); first, the tile route's tile maxima
  int fhist[4096];                      // the fallback's histogram, or the tile route's selected tiles
  int hist[2][256];                     // radix histograms of the streaming route (alternating passes)
  int scan[kSelWarps];                  // the fallback's per-warp tie counts
  uint32_t wkey[kSelWarps];
  int count, found, need, ncand, over_flag, ntsel;
  uint32_t prefix, mask;
};
static_assert(kCandCap <= kSelCap, "the fallback sorts in the candidate list");
static_assert(kSelCap <= 4096, "the tile route (at most kSelCap tiles) lists its tiles in fhist");

__device__ __forceinline__ unsigned long long* fallback_sort(SelShared& S) { return S.list; }
__device__ __forceinline__ int* fallback_hist(SelShared& S) { return S.fhist; }

// Warp 0: finds, in a 256-bin histogram, the highest bin b whose suffix sum
// (bins b..255) reaches `need`, and writes S.prefix = prefix | b << sh and
// S.need = the count still needed inside bin b.  Lane l owns bins 8l..8l+7.
// With fewer than `need` values in all (not reached by the callers) bin 0.
__device__ __forceinline__ void suffix_bin(SelShared& S, const int* hist, int need, uint32_t prefix, int sh) {
  const int lane = threadIdx.x & 31;
  int c[8], own = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = hist[8 * lane + i];
    own += c[i];
  }
  int suf = own;                          // inclusive suffix sum over lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += x;
  }
  const int above = suf - own;
  const bool mine = above < need && suf >= need;
  if (mine) {
    int acc = above, b = 8 * lane;
#pragma unroll
    for (int i = 7; i >= 0; --i) {
      if (acc + c[i] >= need) { b = 8 * lane + i; break; }
      acc += c[i];
    }
    S.prefix = prefix | ((uint32_t)b << sh);
    S.need = need - acc;
  }
  if (__ballot_sync(0xffffffffu, mine) == 0u && lane == 0) {
    S.prefix = prefix;
    S.need = need;
  }
}

// Adds 1 to hist[bin] for every lane with `pred`, one shared atomic per
// distinct bin of the warp (all 32 lanes call it together).
__device__ __forceinline__ void warp_hist_add(int* hist, bool pred, uint32_t bin) {
  const uint32_t b = pred ? bin : 0xffffffffu;
  const unsigned peers = __match_any_sync(0xffffffffu, b);
  if (pred && (threadIdx.x & 31) == (unsigned)(__ffs(peers) - 1)) atomicAdd(&hist[bin], __popc(peers));
}

// Exact K-th largest key among list[0, n) (n >= K).  Radix select, 4 passes
// of 8 bits; pass p counts into hist[p & 1] while the other histogram is
// cleared for the next pass, so a pass costs two barriers.  All threads call it.
__device__ __forceinline__ uint32_t kth_key(SelShared& S, int n, int K) {
  const int t = threadIdx.x;
  const int lane = t & 31, w = t >> 5;
  uint32_t prefix = 0u, pmask = 0u;
  int need = K;
  for (int i = t; i < 256; i += kSelectThreads) S.hist[0][i] = 0;
  __syncthreads();
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int sh = 24 - 8 * pass;
    int* hist = S.hist[pass & 1];
    for (int i = t; i < 256; i += kSelectThreads) S.hist[(pass + 1) & 1][i] = 0;  // next pass
    for (int base = 32 * w; base < n; base += kSelectThreads) {     // warp-uniform trip count
      const int i = base + lane;
      const uint32_t k = i < n ? pair_key(S.list[i]) : 0u;
      warp_hist_add(hist, i < n && (k & pmask) == prefix, (k >> sh) & 255u);
    }
    __syncthreads();
    if (t < 32) suffix_bin(S, hist, need, prefix, sh);
    __syncthreads();
    prefix = S.prefix;
    need = S.need;
    pmask |= 255u << sh;
  }
  return prefix;
}

// Keeps the entries of list[0, n) whose key is >= tau (order not kept);
// returns the new count.  Each thread reads its kSelCap / kSelectThreads
// entries into registers, then the kept ones are appended again from 0 with
// one shared atomic per warp.  All threads call it.
__device__ __forceinline__ int compact_list(SelShared& S, int n, uint32_t tau) {
  constexpr int kPer = kSelCap / kSelectThreads;
  const int t = threadIdx.x, lane = t & 31;
  unsigned long long e[kPer];
  uint32_t keep = 0u;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int j = t * kPer + i;
    e[i] = j < n ? S.list[j] : 0ull;
    if (j < n && pair_key(e[i]) >= tau) keep |= 1u << i;
  }
  __syncthreads();                        // every entry read before any is overwritten
  if (t == 0) S.count = 0;
  __syncthreads();
  const int cnt = __popc(keep);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  int base = 0;
  if (lane == 31 && incl > 0) base = atomicAdd(&S.count, incl);
  int o = __shfl_sync(0xffffffffu, base, 31) + incl - cnt;
#pragma unroll
  for (int i = 0; i < kPer; ++i)
    if (keep & (1u << i)) S.list[o++] = e[i];
  __syncthreads();
  return S.count;
}

// Calls f(v, value) for every column v < V of a row (16-byte aligned): four
// float4 loads in flight per thread, then the scalar tail.
template <class F>
__device__ __forceinline__ void for_each_value(const float* __restrict__ row, int V, F&& f) {
  const int t = threadIdx.x;
  const int V4 = V >> 2;
  const float4* r4 = reinterpret_cast<const float4*>(row);
  int i = t;
  for (; i + 3 * kSelectThreads < V4; i += 4 * kSelectThreads) {
    float4 q[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) q[u] = r4[i + u * kSelectThreads];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = 4 * (i + u * kSelectThreads);
      f(v, q[u].x);
      f(v + 1, q[u].y);
      f(v + 2, q[u].z);
      f(v + 3, q[u].w);
    }
  }
  for (; i < V4; i += kSelectThreads) {
    const float4 q = r4[i];
    f(4 * i, q.x);
    f(4 * i + 1, q.y);
    f(4 * i + 2, q.z);
    f(4 * i + 3, q.w);
  }
  for (int v = 4 * V4 + t; v < V; v += kSelectThreads) f(v, row[v]);
}

// The exact fallback (see the file comment), reading the row from global
// memory; leaves the K results first in fallback_sort(S).
__device__ __forceinline__ void select_two_pass(SelShared& S, const float* __restrict__ row, int V, int K) {
  const int t = threadIdx.x;
  unsigned long long* s_sort = fallback_sort(S);
  int* fh = fallback_hist(S);
  // pass 1: histogram of the top 12 key bits over the whole row
  for (int b = t; b < 4096; b += kSelectThreads) fh[b] = 0;
  if (t == 0) S.found = 0;
  __syncthreads();
  for_each_value(row, V, [&](int, float x) { atomicAdd(&fh[float_key(x) >> 20], 1); });
  __syncthreads();
  if (t == 0) {
    int need = K, b = 4095;
    for (; b > 0 && fh[b] < need; --b) need -= fh[b];
    S.need = need;                          // values of bin b still to take
    S.prefix = (uint32_t)b << 20;
    S.mask = 0xfff00000u;
    S.ncand = K - need + fh[b];             // values with key >= b << 20
  }
  __syncthreads();
  const int ncand = S.ncand;

  int P = 1;
  if (ncand <= kCandCap) {
    // pass 2: every value in or above the K-th value's bin, sorted exactly
    const uint32_t lo = S.prefix;
    for_each_value(row, V, [&](int v, float x) {
      const uint32_t k = float_key(x);
      if (k >= lo) {
        const int slot = atomicAdd(&S.found, 1);
        if (slot < kCandCap) s_sort[slot] = pack_pair(k, v);
      }
    });
    while (P < ncand) P <<= 1;
    __syncthreads();
    for (int i = ncand + t; i < P; i += kSelectThreads) s_sort[i] = 0ull;   // below every real pair
    __syncthreads();
  } else {
    // radix select: bits 19..8, then 7..0, over the values matching the prefix
    const int shifts[2] = {8, 0};
    const int widths[2] = {12, 8};
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
      const int sh = shifts[pass];
      const int nb = 1 << widths[pass];
      for (int b = t; b < nb; b += kSelectThreads) fh[b] = 0;
      __syncthreads();
      const uint32_t prefix = S.prefix, mask = S.mask;
      for_each_value(row, V, [&](int, float x) {
        const uint32_t k = float_key(x);
        if ((k & mask) == prefix) atomicAdd(&fh[(k >> sh) & (uint32_t)(nb - 1)], 1);
      });
      __syncthreads();
      if (t == 0) {
        int need = S.need, b = nb - 1;
        for (; b > 0 && fh[b] < need; --b) need -= fh[b];
        S.need = need;
        S.prefix = prefix | ((uint32_t)b << sh);
        S.mask = mask | ((uint32_t)(nb - 1) << sh);
      }
      __syncthreads();
    }
    const uint32_t kth = S.prefix;          // key of the K-th largest value
    const int need_eq = S.need;             // how many values equal to it are in the top K

    // collection: values above the K-th, and the first need_eq equal to it
    // in column order.  Warp w owns the contiguous columns [c0, c1) and reads
    // them 32 at a time, lane l at column c0 + 32 i + l (coalesced); a ballot
    // gives each lane its place among the warp's equal values, and a scan of
    // the 8 warps' counts orders the warps.
    const int lane = t & 31, w = t >> 5;
    const int seg = ((V + kSelWarps - 1) / kSelWarps + 31) & ~31;
    const int c0 = w * seg;
    const int c1 = (c0 + seg < V) ? c0 + seg : V;
    int n_eq = 0;                             // this warp's values equal to the K-th
    for (int v0 = c0; v0 < c1; v0 += 32) {
      const int v = v0 + lane;
      n_eq += __popc(__ballot_sync(0xffffffffu, v < c1 && float_key(row[v < c1 ? v : c0]) == kth));
    }
    if (lane == 0) S.scan[w] = n_eq;
    for (int i = t; i < kMaxTopK; i += kSelectThreads) s_sort[i] = 0ull;
    __syncthreads();
    int eq_seen = 0;                          // equal values in the warps before this one
    for (int k = 0; k < w; ++k) eq_seen += S.scan[k];
    for (int v0 = c0; v0 < c1; v0 += 32) {
      const int v = v0 + lane;
      const uint32_t k = v < c1 ? float_key(row[v]) : 0u;
      const bool eq = v < c1 && k == kth;
      const unsigned be = __ballot_sync(0xffffffffu, eq);
      const int rank = eq_seen + __popc(be & ((1u << lane) - 1u));
      const bool take = v < c1 && (k > kth || (eq && rank < need_eq));
      if (take) {
        const int slot = atomicAdd(&S.found, 1);
        if (slot < kMaxTopK) s_sort[slot] = pack_pair(k, v);
      }
      eq_seen += __popc(be);
    }
    while (P < K) P <<= 1;
    __syncthreads();
  }
  bitonic_sort_desc(s_sort, P);
}

// Appends to the list every value of q (a block of the row: value e of
// q[u] is column 4 col4(u) + e, present where bit u of `valid` is set) whose
// key is >= tau: one shared atomic per value.  Returns whether this thread
// appended any; sets *over when the list had no room.
template <class Col4>
__device__ __forceinline__ bool append_block(SelShared& S, const float4 (&q)[kSelVec], uint32_t valid,
                                             const Col4& col4, uint32_t tau, bool* over) {
  float fmx = -INFINITY;
  bool nan = false;
#pragma unroll
  for (int u = 0; u < kSelVec; ++u) {
    fmx = fmaxf(fmx, fmaxf(fmaxf(q[u].x, q[u].y), fmaxf(q[u].z, q[u].w)));
    nan |= (q[u].x != q[u].x) | (q[u].y != q[u].y) | (q[u].z != q[u].z) | (q[u].w != q[u].w);
  }
  // for a number x, key(x) >= tau exactly when x >= the float whose key is
  // tau (a tau at or below the key of -inf bounds nothing); NaNs, whose keys
  // lie beyond the infinities, are checked by key
  if (!(tau <= 0x007fffffu || nan || fmx >= key_float(tau))) return false;
  bool any = false;
#pragma unroll
  for (int u = 0; u < kSelVec; ++u) {
    if (!((valid >> u) & 1u)) continue;
    const float f[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t k = float_key(f[e]);
      if (k >= tau) {
        any = true;
        const int slot = atomicAdd(&S.count, 1);
        if (slot < kSelCap) S.list[slot] = pack_pair(k, 4 * col4(u) + e);
        else *over = true;
      }
    }
  }
  return any;
}

// z: rows of `ldz` fp32 values (ldz a multiple of 4, rows 16-byte aligned),
// the first V of each valid.  tmax (or null): per row, `tmld` order keys, the
// largest of each 256-column tile of the row (EpiZ32).  Writes K int32
// indices and K fp32 logits per row to idx_out / val_out (row r at
// out_row0 + r, K per row).
__global__ void __launch_bounds__(kSelectThreads)
topk_select_kernel(const float* __restrict__ z, int64_t ldz, int V, int K, int out_row0,
                   int32_t* __restrict__ idx_out, float* __restrict__ val_out,
                   const uint32_t* __restrict__ tmax, int tmld) {
  __shared__ SelShared S;
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const float* row = z + (size_t)blockIdx.x * ldz;
  const float4* r4 = reinterpret_cast<const float4*>(row);
  const int V4 = V >> 2;
  const int ntiles = (V + kSelTile - 1) / kSelTile;

  if (t == 0) {
    S.count = 0;
    S.over_flag = 0;
    S.ntsel = 0;
  }
  __syncthreads();

  uint32_t tau = 0u;                      // keys below tau are never in the top K
  // The tile route: tau = the K-th largest tile maximum.  The K tiles with
  // the largest maxima hold K values at or above it, so every value at or
  // above the row's K-th largest is at or above tau, and sits in a tile whose
  // maximum is too: only those tiles are read.
  const bool by_tile = tmax != nullptr && ntiles >= K && ntiles <= kSelCap;
  int* tsel = S.fhist;                    // the selected tiles (the fallback's histogram is free)
  int nsel = 0;
  if (by_tile) {
    const uint32_t* trow = tmax + (size_t)blockIdx.x * tmld;
    for (int i = t; i < ntiles; i += kSelectThreads) S.list[i] = pack_pair(trow[i], i);
    __syncthreads();
    tau = kth_key(S, ntiles, K);
    for (int i = t; i < ntiles; i += kSelectThreads)
      if (pair_key(S.list[i]) >= tau) tsel[atomicAdd(&S.ntsel, 1)] = i;
    __syncthreads();
    nsel = S.ntsel;
  }
  const int nblocks = by_tile ? (nsel + kSelTilesPerBlock - 1) / kSelTilesPerBlock
                              : (V4 > 0 ? (V4 + kSelBlock - 1) / kSelBlock : 1);

  bool fallback = false, mine = false, over = false;
#pragma unroll 1
  for (int b = 0; b < nblocks; ++b) {
    // float4 u of this thread: the row's float4 col4(u), streamed (read once)
    // full row: b kSelBlock + t + u kSelectThreads; by tile: float4 t mod 64
    // of the block's tile u (kSelectThreads / 64) + t / 64
    const int i0 = b * kSelBlock + t;
    const int s0 = b * kSelTilesPerBlock + (t >> 6);
    auto col4 = [&](int u) -> int {
      return by_tile ? tsel[s0 + u * (kSelectThreads / 64)] * (kSelTile / 4) + (t & 63) : i0 + u * kSelectThreads;
    };
    float4 q[kSelVec];
    uint32_t valid = 0u;
#pragma unroll
    for (int u = 0; u < kSelVec; ++u) {
      bool ok;
      int i;
      if (by_tile) {
        ok = s0 + u * (kSelectThreads / 64) < nsel;
        i = ok ? col4(u) : 0;
        ok = ok && i < V4;
      } else {
        i = i0 + u * kSelectThreads;
        ok = i < V4;
      }
      if (ok) {
        q[u] = __ldcs(r4 + i);
        valid |= 1u << u;
      } else {
        q[u] = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      }
    }
    if (!by_tile && b == 0 && K <= kSelWarps * 32) {
      // a first threshold: in every warp, the ceil(K/warps)-th largest of its
      // lanes' maxima; the smallest of these has at least K keys at or above it
      uint32_t m = 0u;
#pragma unroll
      for (int u = 0; u < kSelVec; ++u)
        if ((valid >> u) & 1u)
          m = max(m, max(max(float_key(q[u].x), float_key(q[u].y)), max(float_key(q[u].z), float_key(q[u].w))));
#pragma unroll
      for (int size = 2; size <= 32; size <<= 1) {        // descending bitonic sort of the warp's 32
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          const uint32_t y = __shfl_xor_sync(0xffffffffu, m, stride);
          const bool desc = (lane & size) == 0 || size == 32;
          const bool lower = (lane & stride) == 0;
          m = (lower == desc) ? max(m, y) : min(m, y);
        }
      }
      const uint32_t kj = __shfl_sync(0xffffffffu, m, (K + kSelWarps - 1) / kSelWarps - 1);
      if (lane == 0) S.wkey[w] = kj;
      __syncthreads();
      tau = S.wkey[0];
#pragma unroll
      for (int i = 1; i < kSelWarps; ++i) tau = min(tau, S.wkey[i]);
    }
    mine |= append_block(S, q, valid, col4, tau, &over);
    if (b == nblocks - 1 && t == 0) {
      // the scalar tail 4 V4 .. V-1 (fewer than 4 values; appended whenever at
      // or above tau, whichever route, which keeps every candidate)
      for (int v = 4 * V4; v < V; ++v) {
        const uint32_t k = float_key(row[v]);
        if (k >= tau) {
          mine = true;
          const int slot = atomicAdd(&S.count, 1);
          if (slot < kSelCap) S.list[slot] = pack_pair(k, v);
          else over = true;
        }
      }
    }
    // the threads meet after the first block and then every kSelSegment
    // blocks: one barrier when nothing was appended anywhere
    if (b == 0 || b == nblocks - 1 || (b % kSelSegment) == 0) {
      if (over) S.over_flag = 1;
      if (!__syncthreads_or(mine || over)) continue;
      mine = over = false;
      const int n = S.count;
      const bool any_over = S.over_flag != 0;
      __syncthreads();
      if (any_over) {                     // a candidate was lost: take the exact route
        fallback = true;
        break;
      }
      if (n > K && (b == 0 || n > kSelCap / 4)) {
        // raise tau to the K-th largest key of the list and compact it
        tau = kth_key(S, n, K);
        const int m = compact_list(S, n, tau);
        if (t == 0) S.count = m;
        __syncthreads();
        if (m > kSelCap / 4) {            // most of the list tied at tau
          fallback = true;
          break;
        }
      }
    }
  }

  const unsigned long long* result = S.list;
  if (!fallback && S.count < K) fallback = true;   // (not reached: tau keeps K keys at or above it)
  if (!fallback) {
    // cut the list to the keys at or above its K-th largest, and sort it
    const int n = S.count;
    int m = n;
    if (n > K) {
      const uint32_t kk = kth_key(S, n, K);
      m = compact_list(S, n, kk);
    }
    int P = 1;
    while (P < m) P <<= 1;
    for (int i = m + t; i < P; i += kSelectThreads) S.list[i] = 0ull;   // below every real pair
    __syncthreads();
    bitonic_sort_desc(S.list, P);
  } else {
    __syncthreads();
    select_two_pass(S, row, V, K);
    result = fallback_sort(S);
  }

  const size_t o = (size_t)(out_row0 + blockIdx.x) * K;
  for (int i = t; i < K; i += kSelectThreads) {
    const unsigned long long e = result[i];
    idx_out[o + i] = (int32_t)(0xffffffffu - (uint32_t)(e & 0xffffffffull));
    val_out[o + i] = key_float((uint32_t)(e >> 32));
  }
}

}  // namespace kd
