// Teacher top-K cache writer, selection step: for each row of a block of
// fp32 logits, the K largest values and their column indices, largest first,
// equal values in increasing column order (the order in which an offline
// cache lists a position's top-K teacher logits).
//
// One CTA per row, values mapped to order-preserving 32-bit keys.  A first
// pass over the row (16-byte loads, four in flight per thread) builds a
// histogram of the top 12 key bits, which gives the bin holding the K-th
// largest value and the number of values in or above that bin.  Usually
// that is a few hundred at most: a second pass copies them into shared
// memory as (key, column) pairs and a bitonic sort orders them exactly, so
// the row is read twice.  When the bin is too full (heavily tied rows) the
// select continues as a radix select instead: two more histogram passes
// (12 + 8 bits) over the values matching the key prefix found so far, a
// collection pass that takes every value above the K-th and, of those
// equal to it, the ones with the lowest column indices (threads own
// contiguous column ranges, so a scan of per-thread counts orders them),
// and the same sort of the K pairs.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace kd {

constexpr int kSelectThreads = 256;
constexpr int kMaxTopK = 512;
constexpr int kCandCap = 2048;       // candidates sorted in shared memory (power of two, >= kMaxTopK)

// Order-preserving map of a float onto uint32 (larger float, larger key).
__device__ __forceinline__ uint32_t float_key(float v) {
  if (v == 0.f) v = 0.f;                // -0 and +0 are one value
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Block-wide exclusive scan of one int per thread (kSelectThreads threads).
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_tmp, int* total) {
  const int t = threadIdx.x;
  s_tmp[t] = v;
  __syncthreads();
  for (int off = 1; off < kSelectThreads; off <<= 1) {
    const int x = t >= off ? s_tmp[t - off] : 0;
    __syncthreads();
    s_tmp[t] += x;
    __syncthreads();
  }
  const int incl = s_tmp[t];
  *total = s_tmp[kSelectThreads - 1];
  __syncthreads();
  return incl - v;
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

// A (key, column) pair as one sortable word: larger key first, then lower column.
__device__ __forceinline__ unsigned long long pack_pair(uint32_t k, int v) {
  return ((unsigned long long)k << 32) | (unsigned long long)(0xffffffffu - (uint32_t)v);
}

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

// z: rows of `ldz` fp32 values (ldz a multiple of 4, rows 16-byte aligned),
// the first V of each valid.  Writes K int32 indices and K fp32 logits per
// row to idx_out / val_out (row r at out_row0 + r, K per row).
__global__ void __launch_bounds__(kSelectThreads)
topk_select_kernel(const float* __restrict__ z, int64_t ldz, int V, int K, int out_row0,
                   int32_t* __restrict__ idx_out, float* __restrict__ val_out) {
  __shared__ int s_hist[4096];
  __shared__ int s_scan[kSelectThreads];
  __shared__ unsigned long long s_sort[kCandCap];
  __shared__ int s_found, s_ncand;
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_need;

  const int t = threadIdx.x;
  const float* row = z + (size_t)blockIdx.x * ldz;

  // pass 1: histogram of the top 12 key bits over the whole row
  for (int b = t; b < 4096; b += kSelectThreads) s_hist[b] = 0;
  if (t == 0) s_found = 0;
  __syncthreads();
  for_each_value(row, V, [&](int, float x) { atomicAdd(&s_hist[float_key(x) >> 20], 1); });
  __syncthreads();
  if (t == 0) {
    // walk the bins from the top until K values are covered
    int need = K, b = 4095;
    for (; b > 0 && s_hist[b] < need; --b) need -= s_hist[b];
    s_need = need;                          // values of bin b still to take
    s_prefix = (uint32_t)b << 20;
    s_mask = 0xfff00000u;
    s_ncand = K - need + s_hist[b];         // values with key >= b << 20
  }
  __syncthreads();
  const int ncand = s_ncand;

  int P = 1;
  if (ncand <= kCandCap) {
    // pass 2: every value in or above the K-th value's bin, sorted exactly
    const uint32_t lo = s_prefix;
    for_each_value(row, V, [&](int v, float x) {
      const uint32_t k = float_key(x);
      if (k >= lo) {
        const int slot = atomicAdd(&s_found, 1);
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
      for (int b = t; b < nb; b += kSelectThreads) s_hist[b] = 0;
      __syncthreads();
      const uint32_t prefix = s_prefix, mask = s_mask;
      for_each_value(row, V, [&](int, float x) {
        const uint32_t k = float_key(x);
        if ((k & mask) == prefix) atomicAdd(&s_hist[(k >> sh) & (uint32_t)(nb - 1)], 1);
      });
      __syncthreads();
      if (t == 0) {
        int need = s_need, b = nb - 1;
        for (; b > 0 && s_hist[b] < need; --b) need -= s_hist[b];
        s_need = need;
        s_prefix = prefix | ((uint32_t)b << sh);
        s_mask = mask | ((uint32_t)(nb - 1) << sh);
      }
      __syncthreads();
    }
    const uint32_t kth = s_prefix;          // key of the K-th largest value
    const int need_eq = s_need;             // how many values equal to it are in the top K

    // collection: values above the K-th, and the first need_eq equal to it
    const int per = (V + kSelectThreads - 1) / kSelectThreads;
    const int b0 = t * per;
    const int b1 = (b0 + per < V) ? b0 + per : V;
    int n_eq = 0;
    for (int v = b0; v < b1; ++v) n_eq += float_key(row[v]) == kth ? 1 : 0;
    int tot;
    const int eq_before = block_exclusive_scan(n_eq, s_scan, &tot);
    for (int i = t; i < kMaxTopK; i += kSelectThreads) s_sort[i] = 0ull;
    __syncthreads();
    int eq_seen = eq_before;
    for (int v = b0; v < b1; ++v) {
      const uint32_t k = float_key(row[v]);
      bool take = k > kth;
      if (k == kth) {
        take = eq_seen < need_eq;
        ++eq_seen;
      }
      if (take) {
        const int slot = atomicAdd(&s_found, 1);
        if (slot < kMaxTopK) s_sort[slot] = pack_pair(k, v);
      }
    }
    while (P < K) P <<= 1;
    __syncthreads();
  }
  bitonic_sort_desc(s_sort, P);

  const size_t o = (size_t)(out_row0 + blockIdx.x) * K;
  for (int i = t; i < K; i += kSelectThreads) {
    const unsigned long long e = s_sort[i];
    idx_out[o + i] = (int32_t)(0xffffffffu - (uint32_t)(e & 0xffffffffull));
    val_out[o + i] = key_float((uint32_t)(e >> 32));
  }
}

}  // namespace kd
