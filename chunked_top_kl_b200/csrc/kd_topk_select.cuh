// Teacher top-K cache writer, selection step: for each row of a block of
// fp32 logits, the K largest values and their column indices, largest first,
// equal values in increasing column order (the order in which an offline
// cache lists a position's top-K teacher logits).
//
// One CTA per row.  The K-th largest value is found exactly by a radix select
// on order-preserving 32-bit keys (12 + 12 + 8 bits: three histogram passes
// over the row, each over the values that match the key prefix found so
// far); a fourth pass collects every value above it and, of those equal to
// it, the ones with the lowest column indices (threads own contiguous column
// ranges, so a scan of per-thread counts orders them); the K pairs are then
// sorted in shared memory (bitonic sort on value-major, index-minor keys).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace kd {

constexpr int kSelectThreads = 256;
constexpr int kMaxTopK = 512;

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

// z: rows of `ldz` fp32 values, the first V of each valid.  Writes K int32
// indices and K fp32 logits per row to idx_out / val_out (row r at
// out_row0 + r, K per row).
__global__ void __launch_bounds__(kSelectThreads)
topk_select_kernel(const float* __restrict__ z, int64_t ldz, int V, int K, int out_row0,
                   int32_t* __restrict__ idx_out, float* __restrict__ val_out) {
  __shared__ int s_hist[4096];
  __shared__ int s_scan[kSelectThreads];
  __shared__ unsigned long long s_sort[kMaxTopK];
  __shared__ int s_found;
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_need;

  const int t = threadIdx.x;
  const float* row = z + (size_t)blockIdx.x * ldz;
  if (t == 0) {
    s_prefix = 0u;
    s_mask = 0u;
    s_need = K;
  }

  // three radix passes: bits 31..20, 19..8, 7..0
  const int shifts[3] = {20, 8, 0};
  const int widths[3] = {12, 12, 8};
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int sh = shifts[pass];
    const int nb = 1 << widths[pass];
    for (int b = t; b < nb; b += kSelectThreads) s_hist[b] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int v = t; v < V; v += kSelectThreads) {
      const uint32_t k = float_key(row[v]);
      if ((k & mask) == prefix) atomicAdd(&s_hist[(k >> sh) & (uint32_t)(nb - 1)], 1);
    }
    __syncthreads();
    if (t == 0) {
      // walk the bins from the top until `need` values are covered
      int need = s_need, b = nb - 1;
      for (; b > 0 && s_hist[b] < need; --b) need -= s_hist[b];
      s_need = need;                    // values equal to the final key still to take
      s_prefix = prefix | ((uint32_t)b << sh);
      s_mask = mask | ((uint32_t)(nb - 1) << sh);
    }
    __syncthreads();
  }
  const uint32_t kth = s_prefix;        // key of the K-th largest value
  const int need_eq = s_need;           // how many values equal to it are in the top K

  // collection: values above the K-th, and the first need_eq equal to it
  const int per = (V + kSelectThreads - 1) / kSelectThreads;
  const int b0 = t * per;
  const int b1 = (b0 + per < V) ? b0 + per : V;
  int n_eq = 0;
  for (int v = b0; v < b1; ++v) n_eq += float_key(row[v]) == kth ? 1 : 0;
  int tot;
  const int eq_before = block_exclusive_scan(n_eq, s_scan, &tot);
  if (t == 0) s_found = 0;
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
      if (slot < kMaxTopK)
        s_sort[slot] = ((unsigned long long)k << 32) | (unsigned long long)(0xffffffffu - (uint32_t)v);
    }
  }
  __syncthreads();

  // bitonic sort, descending, over the next power of two >= K
  int P = 1;
  while (P < K) P <<= 1;
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = t; i < P; i += kSelectThreads) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long a = s_sort[i], b = s_sort[j];
          if (desc ? (a < b) : (a > b)) {
            s_sort[i] = b;
            s_sort[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  const size_t o = (size_t)(out_row0 + blockIdx.x) * K;
  for (int i = t; i < K; i += kSelectThreads) {
    const unsigned long long e = s_sort[i];
    idx_out[o + i] = (int32_t)(0xffffffffu - (uint32_t)(e & 0xffffffffull));
    val_out[o + i] = key_float((uint32_t)(e >> 32));
  }
}

}  // namespace kd
