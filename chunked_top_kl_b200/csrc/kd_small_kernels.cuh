// CUDA-core kernels of the path: teacher-cache preparation, the merge of the
// per-split log-sum-exp state into lse and per-token KL terms, and the
// fixed-order scalar reductions.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace kd {

constexpr int kSentinel = 0x7fffffff;       // sorted-index padding; never equals a column
constexpr int kEmptySlot = -1;              // teacher index of an empty cache slot
constexpr int kMaxK = 512;
constexpr int kPrepWarps = 4;               // tokens per block in teacher_prep
constexpr int kMergeThreads = 256;

// Status words at the start of the workspace.
struct Status {
  unsigned int bad_index;      // teacher indices outside [0, V)
  unsigned int timeout;        // a bounded pipeline wait expired
  unsigned int pad[14];
};

// Order-preserving map of a float onto uint32 (larger float, larger key;
// NaNs with the sign bit clear above +inf, with it set below -inf).  The
// teacher top-K selection compares logits by these keys.
__device__ __forceinline__ uint32_t float_key(float v) {
  if (v == 0.f) v = 0.f;                // -0 and +0 are one value
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One warp per token.  For token n it
//  * turns the cached logits of the filled slots into p = softmax(logit / T)
//    and the teacher term sum_k p log p (0 log 0 = 0) -- the renormalised
//    top-K teacher distribution of the offline cache.  A slot with index -1
//    is empty and takes no part; a token without a finite filled logit gets
//    p = 0 throughout (an empty teacher distribution);
//  * drops (and counts) other indices outside [0, V);
//  * sorts the (index, p) pairs by index (rank sort, ties by slot), merges
//    repeated indices by adding their p, and writes the unique pairs padded
//    with kSentinel to a row of Kp >= K + 1 slots, so the GEMM epilogues can
//    walk a row's teacher columns in increasing order with one cursor (and
//    an empty distribution is a row that starts with kSentinel).
// Logits are fp32, or bf16 when logit_bf16 != 0.  Each block also writes the
// sum of its tokens' mask values (fp64).
__global__ void __launch_bounds__(kPrepWarps * 32)
teacher_prep_kernel(const int32_t* __restrict__ idx, const void* __restrict__ logit, int logit_bf16,
                    const float* __restrict__ mask, int N, int K, int Kp, int V, float T,
                    int32_t* __restrict__ tidx, float* __restrict__ tp, float* __restrict__ ent,
                    double* __restrict__ mask_part, Status* status) {
  __shared__ int s_key[kPrepWarps][kMaxK];
  __shared__ float s_p[kPrepWarps][kMaxK];
  __shared__ int s_skey[kPrepWarps][kMaxK];
  __shared__ float s_sp[kPrepWarps][kMaxK];
  __shared__ double s_mask[kPrepWarps];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * kPrepWarps + warp;
  int* key = s_key[warp];
  float* pv = s_p[warp];
  int* sk = s_skey[warp];
  float* sp = s_sp[warp];

  double mval = 0.0;
  if (n < N) {
    const int32_t* irow = idx + (size_t)n * K;
    float tmax = -INFINITY;
    for (int k = lane; k < K; k += 32) {
      const float lg = logit_bf16
          ? __bfloat162float(static_cast<const __nv_bfloat16*>(logit)[(size_t)n * K + k])
          : static_cast<const float*>(logit)[(size_t)n * K + k];
      const float t = irow[k] == kEmptySlot ? -INFINITY : lg / T;
      pv[k] = t;
      tmax = fmaxf(tmax, t);
    }
    tmax = warp_max(tmax);
    float lse_t = INFINITY;                 // empty distribution: every p = 0
    if (tmax != -INFINITY) {
      float s = 0.f;
      for (int k = lane; k < K; k += 32) s += expf(pv[k] - tmax);
      s = warp_sum(s);
      lse_t = tmax + logf(s);
    }
    float e = 0.f;
    unsigned int nbad = 0;
    for (int k = lane; k < K; k += 32) {
      const float logp = pv[k] - lse_t;
      const float p = expf(logp);
      if (p > 0.f) e += p * logp;
      int key_k = irow[k];
      float p_k = p;
      if (key_k < 0 || key_k >= V) {
        nbad += key_k != kEmptySlot;
        key_k = kSentinel;
        p_k = 0.f;
      }
      key[k] = key_k;
      pv[k] = p_k;
    }
    e = warp_sum(e);
    nbad = __reduce_add_sync(0xffffffffu, nbad);
    if (lane == 0) {
      ent[n] = e;
      if (nbad) atomicAdd(&status->bad_index, nbad);
    }
    __syncwarp();
    for (int k = lane; k < K; k += 32) {
      const int kk = key[k];
      int r = 0;
      for (int j = 0; j < K; ++j) {
        const int kj = key[j];
        r += (kj < kk) | ((kj == kk) & (j < k));
      }
      sk[r] = kk;
      sp[r] = pv[k];
    }
    __syncwarp();
    int32_t* orow_i = tidx + (size_t)n * Kp;
    float* orow_p = tp + (size_t)n * Kp;
    int count = 0;
    for (int base = 0; base < K; base += 32) {
      const int pos = base + lane;
      bool head = false;
      if (pos < K) {
        const int kk = sk[pos];
        head = (kk != kSentinel) && (pos == 0 || sk[pos - 1] != kk);
      }
      const unsigned ballot = __ballot_sync(0xffffffffu, head);
      if (head) {
        const int kk = sk[pos];
        float q = sp[pos];
        for (int j = pos + 1; j < K && sk[j] == kk; ++j) q += sp[j];
        const int o = count + __popc(ballot & ((1u << lane) - 1u));
        orow_i[o] = kk;
        orow_p[o] = q;
      }
      count += __popc(ballot);
    }
    for (int j = count + lane; j < Kp; j += 32) {
      orow_i[j] = kSentinel;
      orow_p[j] = 0.f;
    }
    mval = mask ? (double)mask[n] : 1.0;
  }
  if (lane == 0) s_mask[warp] = mval;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < kPrepWarps; ++w) t += s_mask[w];
    mask_part[blockIdx.x] = t;
  }
}

// One thread per token: merges the per-split (max, sum-exp, gathered p.z)
// partials into lse and the token's KL term, and writes each block's sum of
// mask * term (fp64).  The partials hold the maximum of the raw logits z and
// sums of exp((z - max) * zscale), so the merged lse is that of z * zscale
// (zscale = 1, or 1 / T for the student-temperature variant), and
//   term = tfac * (sum p log p - zscale * sum p z + P * lse)
// with P = 1, or 0 for a token without teacher entries (its prepared row
// starts with kSentinel), and tfac = 1 or T^2.
//
// `poison_on` (may be null): status words that earlier kernels of the same
// pass on this stream have set.  When any of them reports a bad teacher
// index or a timed-out wait, every lse is written as NaN, for callers that
// have no way to read the status words themselves.
__device__ __forceinline__ bool status_failed(const Status* s) {
  if (!s) return false;
  const volatile Status* v = s;
  return (v->bad_index | v->timeout) != 0u;
}

__global__ void __launch_bounds__(kMergeThreads)
lse_merge_kernel(const float* __restrict__ part_m, const float* __restrict__ part_s,
                 const float* __restrict__ part_g, int splits, int N,
                 const float* __restrict__ ent, const float* __restrict__ mask,
                 const int32_t* __restrict__ tidx, int Kp, float zscale, float tfac,
                 float* __restrict__ lse_out, double* __restrict__ term_part,
                 const Status* poison_on) {
  __shared__ double s_red[kMergeThreads / 32];
  const int n = blockIdx.x * kMergeThreads + threadIdx.x;
  double contrib = 0.0;
  if (n < N && status_failed(poison_on)) {
    lse_out[n] = __int_as_float(0x7fc00000);
  } else if (n < N) {
    float m = -INFINITY;
    for (int s = 0; s < splits; ++s) m = fmaxf(m, part_m[(size_t)s * N + n]);
    float ssum = 0.f, g = 0.f;
    for (int s = 0; s < splits; ++s) {
      const float ms = part_m[(size_t)s * N + n];
      if (ms != -INFINITY) ssum += part_s[(size_t)s * N + n] * expf((ms - m) * zscale);
      g += part_g[(size_t)s * N + n];
    }
    const float lse = m * zscale + logf(ssum);
    lse_out[n] = lse;
    const float P = tidx[(size_t)n * Kp] == kSentinel ? 0.f : 1.f;
    const float term = tfac * (ent[n] - zscale * g + P * lse);
    const float mv = mask ? mask[n] : 1.f;
    contrib = (mv != 0.f) ? (double)mv * (double)term : 0.0;
  }
  contrib = warp_sum_d(contrib);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = contrib;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < kMergeThreads / 32; ++w) t += s_red[w];
    term_part[blockIdx.x] = t;
  }
}

// Rows that can be skipped in the backward pass: a token whose mask is 0, or
// whose teacher distribution is empty, has a zero dZ row.  One block lists
// the other tokens in increasing order in rowmap[0, *count) (a block-wide
// exclusive scan of per-thread counts over contiguous token segments).
constexpr int kCompactThreads = 1024;

__global__ void __launch_bounds__(kCompactThreads)
compact_rows_kernel(const float* __restrict__ mask, const int32_t* __restrict__ tidx, int Kp, int N,
                    int32_t* __restrict__ rowmap, int* __restrict__ count) {
  __shared__ int s_cnt[kCompactThreads];
  const int t = threadIdx.x;
  const int per = (N + kCompactThreads - 1) / kCompactThreads;
  const int b = t * per;
  const int e = (b + per < N) ? b + per : N;
  auto keep = [&](int n) {
    return (mask == nullptr || mask[n] != 0.f) && tidx[(size_t)n * Kp] != kSentinel;
  };
  int c = 0;
  for (int n = b; n < e; ++n) c += keep(n) ? 1 : 0;
  s_cnt[t] = c;
  __syncthreads();
  for (int off = 1; off < kCompactThreads; off <<= 1) {
    const int v = t >= off ? s_cnt[t - off] : 0;
    __syncthreads();
    s_cnt[t] += v;
    __syncthreads();
  }
  int o = s_cnt[t] - c;
  for (int n = b; n < e; ++n)
    if (keep(n)) rowmap[o++] = n;
  if (t == kCompactThreads - 1) *count = s_cnt[t];
}

// Rows [row0, row0 + C) of the compacted token list: dst[r] = src[rowmap[row0 + r]]
// (16-byte vectors, d8 per row) for the rows below *count, zeros past it.
__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint4* __restrict__ src, int d8, const int32_t* __restrict__ rowmap,
                   const int* __restrict__ count, int row0, int C, uint4* __restrict__ dst) {
  const int live = *count;
  const size_t total = (size_t)C * d8;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / d8);
    const int j = (int)(i - (size_t)r * d8);
    const int q = row0 + r;
    dst[i] = q < live ? src[(size_t)rowmap[q] * d8 + j] : make_uint4(0u, 0u, 0u, 0u);
  }
}

// The inverse for the rows below *count: dst[rowmap[row0 + r]] = src[r].
__global__ void __launch_bounds__(256)
scatter_rows_kernel(const uint4* __restrict__ src, int d8, const int32_t* __restrict__ rowmap,
                    const int* __restrict__ count, int row0, int C, uint4* __restrict__ dst) {
  const int live = *count;
  int rows = live - row0;
  rows = rows < 0 ? 0 : (rows > C ? C : rows);
  const size_t total = (size_t)rows * d8;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / d8);
    const int j = (int)(i - (size_t)r * d8);
    dst[(size_t)rowmap[row0 + r] * d8 + j] = src[i];
  }
}

// Single block.  Sums block partials in a fixed order (deterministic).
//  mode 0: *loss = sum(term_part) / sum(mask_part), or 0 if the mask sums to 0.
//  mode 1: *cscale = g / sum(mask_part) (g = *grad or 1), or 0.
// With `poison_on` set and reporting a failure (see lse_merge_kernel), the
// output is NaN.
__global__ void __launch_bounds__(256)
finalize_kernel(const double* __restrict__ mask_part, int n_mask_part,
                const double* __restrict__ term_part, int n_term_part, int mode,
                const float* __restrict__ grad, float* __restrict__ out,
                const Status* poison_on = nullptr) {
  __shared__ double s_m[256], s_t[256];
  double am = 0.0, at = 0.0;
  for (int i = threadIdx.x; i < n_mask_part; i += 256) am += mask_part[i];
  for (int i = threadIdx.x; i < n_term_part; i += 256) at += term_part[i];
  s_m[threadIdx.x] = am;
  s_t[threadIdx.x] = at;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      s_m[threadIdx.x] += s_m[threadIdx.x + w];
      s_t[threadIdx.x] += s_t[threadIdx.x + w];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double sm = s_m[0];
    if (status_failed(poison_on)) {
      *out = __int_as_float(0x7fc00000);
    } else if (mode == 0) {
      *out = (sm != 0.0) ? (float)(s_t[0] / sm) : 0.f;
    } else {
      const double g = grad ? (double)*grad : 1.0;
      *out = (sm != 0.0) ? (float)(g / sm) : 0.f;
    }
  }
}

}  // namespace kd
