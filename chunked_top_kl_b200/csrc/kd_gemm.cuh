// Persistent, warp-specialised tcgen05 GEMM with pluggable epilogues.
//
// One CTA per SM.  Warp 0 issues TMA loads into a STAGES-deep shared-memory
// ring, warp 1 issues tcgen05.mma (bf16 x bf16 -> fp32 in tensor memory),
// warps 2-5 run the epilogue straight out of tensor memory.  Two 128 x 256
// fp32 accumulators (all 512 TMEM columns) let the epilogue of one tile
// overlap the MMAs of the next.
//
// Work is a list of units; a unit is one 128-row tile band (m) and a
// contiguous range of 256-column tiles [n0, n1).  All three roles walk the
// same unit sequence (u = blockIdx.x, blockIdx.x + gridDim.x, ...), so no
// scheduling state is shared between them.  The epilogue object lives for a
// unit, which is what lets the forward epilogue carry a running
// max / sum-exp across the vocabulary tiles of its range.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kd_ptx.cuh"
#include "kd_schedule.h"
#include "kd_small_kernels.cuh"

namespace kd {

constexpr int BM = 128;          // accumulator rows per CTA (TMEM lanes)
constexpr int BN = 256;          // tile columns (TMEM columns per accumulator)
constexpr int BK = 64;           // bf16 elements per 128-byte swizzle row
constexpr int UMMA_K = 16;       // K of one tcgen05.mma kind::f16
constexpr int GEMM_THREADS = 192;
constexpr int TMEM_COLS = 512;

// Per-variant tile geometry.  PAIR = false: one CTA computes a 128 x 256 tile
// (A 128 rows, B 256 rows per stage).  PAIR = true: a cluster of two CTAs
// computes a 256 x 256 tile with cta_group::2 MMAs; each CTA stages its own
// 128 rows of A and 128 rows of B, holds its 128 accumulator rows in its own
// tensor memory, and the pair leader issues the MMAs.
template <bool PAIR>
struct Geo {
  static constexpr int TILE_M = PAIR ? 2 * BM : BM;
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;          // B rows staged per CTA
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;       // per CTA
  static constexpr int STAGES = PAIR ? 6 : 4;
  static constexpr int STAGING_BYTES = 2 * BM * 128;           // two 128-row x 128-byte store buffers
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + STAGING_BYTES + 1024 /*align*/ + 256 /*barriers*/;
  static constexpr uint32_t TX_BYTES = (PAIR ? 2 : 1) * STAGE_BYTES;  // per stage, whole tile
};

struct GemmArgs {
  Raster raster;
  int num_kb;           // BK-wide K blocks per tile
  int a_row0, b_row0;   // tensor-map offsets added to the row (M / N) coordinate
  int a_k0, b_k0;       // tensor-map offsets added to the K coordinate
  Status* status;
};

// Loads one operand tile (rows x BK) for K block kb into shared memory.
//  K-major: one box {BK, rows} at (k, row).  The smem tile is rows x 128 B,
//           8-row groups 1024 B apart (SBO), 128-byte swizzled.
//  MN-major: rows/64 boxes {64, BK} at (row + 64 i, k).  Each box is BK
//           K-rows of 128 B (64 MN elements); boxes are BK*128 B apart (LBO).
template <bool MN_MAJOR, int ROWS, bool PAIR>
__device__ __forceinline__ void load_operand(uint32_t dst, const CUtensorMap* tm, int row, int k,
                                             uint32_t bar) {
  if constexpr (!MN_MAJOR) {
    if constexpr (PAIR) tma_load_2d_pair(dst, tm, k, row, bar);
    else tma_load_2d(dst, tm, k, row, bar);
  } else {
#pragma unroll
    for (int i = 0; i < ROWS / 64; ++i) {
      if constexpr (PAIR) tma_load_2d_pair(dst + i * (BK * 128), tm, row + 64 * i, k, bar);
      else tma_load_2d(dst + i * (BK * 128), tm, row + 64 * i, k, bar);
    }
  }
}

// Descriptor of the kk-th UMMA_K slice of an operand tile in shared memory.
template <bool MN_MAJOR>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int kk) {
  if constexpr (!MN_MAJOR) {
    // K-major SW128: K advances inside the 128-byte row.
    return smem_desc_sw128(base + kk * UMMA_K * 2, 16, 1024);
  } else {
    // MN-major SW128: K advances by UMMA_K rows of 128 B.
    return smem_desc_sw128(base + kk * UMMA_K * 128, BK * 128, 1024);
  }
}

// What an epilogue thread needs to write its tile through shared memory and
// TMA: two 16 KB staging buffers used alternately, the thread's row in the
// CTA's 128-row slab, the slab's first output row, and whether this thread
// issues the bulk copies (one thread of the 128).
struct EpiCtx {
  uint32_t stage[2];
  int rr;
  int row_base;
  bool issuer;
  uint32_t seq;
};

// Writes one 128-byte segment per thread (its row) into the next staging
// buffer with the 128-byte swizzle, then one thread stores (or adds) the
// 128-row box to global memory at (x, y) with TMA.
__device__ __forceinline__ void stage_store(EpiCtx& cx, const CUtensorMap* tm, int x, int y,
                                            const uint32_t (&w)[32], bool reduce_add) {
  const uint32_t buf = cx.stage[cx.seq & 1u];
  if (cx.issuer && cx.seq >= 2) bulk_wait_read<1>();     // buffer's previous store has read it
  epilogue_bar_sync(128);
  const uint32_t rowa = buf + (uint32_t)cx.rr * 128u;
  const uint32_t sw = (uint32_t)(cx.rr & 7);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    st_shared_v4(rowa + (((uint32_t)k ^ sw) << 4), w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
  fence_proxy_async_shared();
  epilogue_bar_sync(128);
  if (cx.issuer) {
    if (reduce_add) tma_reduce_add_2d(tm, x, y, buf);
    else tma_store_2d(tm, x, y, buf);
    bulk_commit();
  }
  ++cx.seq;
}

template <class Epi, bool A_MN, bool B_MN, bool PAIR>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const GemmArgs args, const __grid_constant__ typename Epi::Params ep) {
  using G = Geo<PAIR>;
  constexpr int STAGES = G::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t staging = sbase + STAGES * G::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * G::STAGE_BYTES + G::STAGING_BYTES);
  const uint32_t bar_base = smem_u32(bars);
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar_base + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar_base + 8u * (2 * STAGES + 2 + a); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Raster& R = args.raster;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;       // CTA within the pair
  const int group = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int ngroups = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  // Barriers that the pair leader owns: stage-full (TMA bytes of both CTAs)
  // and accumulator-empty (epilogue threads of both CTAs).
  auto leader = [&](uint32_t a) { return PAIR ? mapa_shared(a, 0) : a; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), (PAIR ? 2 : 1) * 4 * 32);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync_all(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  bool failed = false;
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (every CTA)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int u = group; u < R.num_units && !failed; u += ngroups) {
        int m, split, n0, n1;
        decode_unit(R, u, m, split, n0, n1);
        for (int n = n0; n < n1 && !failed; ++n) {
          for (int kb = 0; kb < args.num_kb; ++kb) {
            if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag)) { failed = true; break; }
            const uint32_t sa = sbase + stage * G::STAGE_BYTES;
            const uint32_t sb = sa + G::A_BYTES;
            const uint32_t fb = leader(full_bar(stage));
            if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), G::TX_BYTES);
            load_operand<A_MN, BM, PAIR>(sa, &tmA, args.a_row0 + m * G::TILE_M + (int)rank * BM,
                                         args.a_k0 + kb * BK, fb);
            load_operand<B_MN, G::B_ROWS, PAIR>(sb, &tmB, args.b_row0 + n * BN + (int)rank * G::B_ROWS,
                                                args.b_k0 + kb * BK, fb);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (pair leader)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(G::TILE_M, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int u = group; u < R.num_units && !failed; u += ngroups) {
        int m, split, n0, n1;
        decode_unit(R, u, m, split, n0, n1);
        for (int n = n0; n < n1 && !failed; ++n) {
          if (!mbar_wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag)) { failed = true; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * BN;
          for (int kb = 0; kb < args.num_kb; ++kb) {
            if (!mbar_wait_bounded(full_bar(stage), phase, abort_flag)) { failed = true; break; }
            tc_fence_after();
            const uint32_t sa = sbase + stage * G::STAGE_BYTES;
            const uint32_t sb = sa + G::A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / UMMA_K; ++kk) {
              const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
              if constexpr (PAIR)
                tc_mma_bf16_pair(d_tmem, operand_desc<A_MN>(sa, kk), operand_desc<B_MN>(sb, kk), idesc, accum);
              else
                tc_mma_bf16(d_tmem, operand_desc<A_MN>(sa, kk), operand_desc<B_MN>(sb, kk), idesc, accum);
            }
            if constexpr (PAIR) tc_commit_pair_mc(empty_bar(stage), 0x3); else tc_commit(empty_bar(stage));
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
          if (failed) break;
          if constexpr (PAIR) tc_commit_pair_mc(tfull_bar(acc), 0x3); else tc_commit(tfull_bar(acc));
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1u;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (every CTA)
    const int q = warp & 3;                 // TMEM lane quadrant this warp may access
    const int row = (int)rank * BM + q * 32 + lane;   // row of the tile owned by this thread
    const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
    int acc = 0;
    uint32_t acc_phase = 0;
    Epi epi;
    EpiCtx cx;
    cx.stage[0] = staging;
    cx.stage[1] = staging + BM * 128;
    cx.rr = q * 32 + lane;
    cx.issuer = (threadIdx.x == 64);
    cx.seq = 0;
    for (int u = group; u < R.num_units && !failed; u += ngroups) {
      int m, split, n0, n1;
      decode_unit(R, u, m, split, n0, n1);
      const int grow = m * G::TILE_M + row;
      cx.row_base = m * G::TILE_M + (int)rank * BM;
      epi.begin_unit(ep, grow, split, n0);
      for (int n = n0; n < n1; ++n) {
        // One outcome for all 128 epilogue threads: tcgen05.ld needs whole
        // warps and the store path synchronises the four warps.
        const bool ok = epilogue_bar_and(128, mbar_wait_bounded(tfull_bar(acc), acc_phase, abort_flag));
        if (!ok) { failed = true; break; }
        tc_fence_after();
        epi.tile(ep, grow, n, lane_addr + acc * BN, cx);
        tc_fence_before();
        if constexpr (PAIR) mbar_arrive_cluster(leader(tempty_bar(acc)));
        else mbar_arrive(tempty_bar(acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (failed) break;
      epi.end_unit(ep, grow, split);
    }
    if (cx.issuer) bulk_wait<0>();          // every TMA store of this CTA has completed
  }

  if (failed) {
    *abort_flag = 1;
    atomicOr(&args.status->timeout, 1u);
  }
  __syncwarp();
  __syncthreads();
  if (*abort_flag) {
    // Let asynchronous copies and MMAs that were already issued land before
    // the CTA releases its shared and tensor memory.
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) { }
    __syncthreads();
  }
  // Neither CTA of a pair may release its memory while the leader's MMAs can
  // still read the peer's shared memory or write its tensor memory.
  if constexpr (PAIR) cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- epilogues

__device__ __forceinline__ int lower_bound_row(const int32_t* row, int len, int key) {
  int lo = 0, hi = len;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (row[mid] < key) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Forward: running max / sum-exp over the unit's vocabulary columns and the
// gathered sum of p * z at the teacher's columns; one (m, s, g) partial per
// token per split.  Columns >= V are -inf.
struct EpiFwd {
  struct Params {
    int N, V, Kp;
    const int32_t* tidx;
    const float* tp;
    float* part_m;
    float* part_s;
    float* part_g;
  };
  float mrun, srun, grun, np;
  int cur, nidx, grow;
  const int32_t* trow;
  const float* prow;

  __device__ __forceinline__ void begin_unit(const Params& P, int grow_, int, int n0) {
    grow = grow_;
    mrun = -INFINITY;
    srun = 0.f;
    grun = 0.f;
    nidx = kSentinel;
    np = 0.f;
    if (grow < P.N) {
      trow = P.tidx + (size_t)grow * P.Kp;
      prow = P.tp + (size_t)grow * P.Kp;
      cur = lower_bound_row(trow, P.Kp, n0 * BN);
      nidx = trow[cur];
      np = prow[cur];
    }
  }

  __device__ __forceinline__ void tile(const Params& P, int, int n, uint32_t taddr, EpiCtx&) {
#pragma unroll 1
    for (int j = 0; j < BN / 32; ++j) {
      float v[32];
      __syncwarp();
      tmem_ld_32x32b_x32(taddr + j * 32, v);
      const int c0 = n * BN + j * 32;
      if (c0 + 32 > P.V) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c0 + i >= P.V) v[i] = -INFINITY;
      }
      if (nidx < c0 + 32) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (c0 + i == nidx) {
            grun += np * v[i];
            ++cur;
            nidx = trow[cur];
            np = prow[cur];
          }
        }
      }
      float cm = v[0];
#pragma unroll
      for (int i = 1; i < 32; ++i) cm = fmaxf(cm, v[i]);
      const float mn = fmaxf(mrun, cm);
      if (mn == -INFINITY) continue;
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) acc += __expf(v[i] - mn);
      srun = srun * __expf(mrun - mn) + acc;
      mrun = mn;
    }
  }

  __device__ __forceinline__ void end_unit(const Params& P, int, int split) {
    if (grow < P.N) {
      const size_t o = (size_t)split * P.N + grow;
      P.part_m[o] = mrun;
      P.part_s[o] = srun;
      P.part_g[o] = grun;
    }
  }
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Backward, per chunk: dZ = c_n (exp(z - lse_n) - p at the teacher's columns),
// rounded to bf16 and stored for the chunk's tokens (row-major, ldz columns;
// columns in [V, ldz) are written as 0) through shared memory and TMA.
struct EpiDz {
  struct Params {
    CUtensorMap tm;        // dZ chunk [rows_valid][ldz] bf16, box {64, 128}, 128-byte swizzle
    int rows_valid;        // tokens in this chunk
    int row0;              // global token index of chunk row 0
    int V, ldz, Kp;
    const int32_t* tidx;
    const float* tp;
    const float* lse;
    const float* mask;     // may be null
    const float* cscale;   // device scalar g / sum(mask)
  };
  __device__ __forceinline__ void begin_unit(const Params&, int, int, int) {}
  __device__ __forceinline__ void end_unit(const Params&, int, int) {}

  __device__ __forceinline__ void tile(const Params& P, int r, int n, uint32_t taddr, EpiCtx& cx) {
    const bool valid = r < P.rows_valid;
    const int grow = P.row0 + r;
    float L = 0.f, c = 0.f;
    const int32_t* trow = nullptr;
    const float* prow = nullptr;
    int cur = 0, nidx = kSentinel;
    float np = 0.f;
    if (valid) {
      L = P.lse[grow];
      c = (P.mask ? P.mask[grow] : 1.f) * (*P.cscale);
      trow = P.tidx + (size_t)grow * P.Kp;
      prow = P.tp + (size_t)grow * P.Kp;
      cur = lower_bound_row(trow, P.Kp, n * BN);
      nidx = trow[cur];
      np = prow[cur];
    }
#pragma unroll 1
    for (int j = 0; j < BN / 64; ++j) {
      float v[64];
      float (&v0)[32] = *reinterpret_cast<float(*)[32]>(&v[0]);
      float (&v1)[32] = *reinterpret_cast<float(*)[32]>(&v[32]);
      __syncwarp();
      tmem_ld_32x32b_x32(taddr + j * 64, v0);
      tmem_ld_32x32b_x32(taddr + j * 64 + 32, v1);
      const int c0 = n * BN + j * 64;
#pragma unroll
      for (int i = 0; i < 64; ++i) v[i] = __expf(v[i] - L);
      if (nidx < c0 + 64) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          if (c0 + i == nidx) {
            v[i] -= np;
            ++cur;
            nidx = trow[cur];
            np = prow[cur];
          }
        }
      }
      uint32_t w[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float a = (c0 + 2 * i < P.V) ? c * v[2 * i] : 0.f;
        const float b = (c0 + 2 * i + 1 < P.V) ? c * v[2 * i + 1] : 0.f;
        w[i] = pack_bf16x2(a, b);
      }
      stage_store(cx, &P.tm, c0, cx.row_base, w, false);
    }
  }
};

// Backward, per chunk: dH rows of the chunk's tokens, bf16, through shared
// memory and TMA (the map covers the chunk's rows only).
struct EpiDh {
  struct Params {
    CUtensorMap tm;        // dH rows of the chunk [rows][d] bf16, box {64, 128}, 128-byte swizzle
  };
  __device__ __forceinline__ void begin_unit(const Params&, int, int, int) {}
  __device__ __forceinline__ void end_unit(const Params&, int, int) {}

  __device__ __forceinline__ void tile(const Params& P, int, int n, uint32_t taddr, EpiCtx& cx) {
#pragma unroll 1
    for (int j = 0; j < BN / 64; ++j) {
      float v[64];
      float (&v0)[32] = *reinterpret_cast<float(*)[32]>(&v[0]);
      float (&v1)[32] = *reinterpret_cast<float(*)[32]>(&v[32]);
      __syncwarp();
      tmem_ld_32x32b_x32(taddr + j * 64, v0);
      tmem_ld_32x32b_x32(taddr + j * 64 + 32, v1);
      uint32_t w[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
      stage_store(cx, &P.tm, n * BN + j * 64, cx.row_base, w, false);
    }
  }
};

// Backward, per chunk: dW (+)= dZ^T H for 128 vocabulary rows x 256 columns
// per CTA, fp32, stored (first chunk without accumulation) or added in place
// by TMA reductions: the memory system does the read-modify-write.
struct EpiDw {
  struct Params {
    CUtensorMap tm;        // dW [V][d] fp32, box {32, 128}, 128-byte swizzle
    int accumulate;
  };
  __device__ __forceinline__ void begin_unit(const Params&, int, int, int) {}
  __device__ __forceinline__ void end_unit(const Params&, int, int) {}

  __device__ __forceinline__ void tile(const Params& P, int, int n, uint32_t taddr, EpiCtx& cx) {
#pragma unroll 1
    for (int j = 0; j < BN / 32; ++j) {
      float v[32];
      __syncwarp();
      tmem_ld_32x32b_x32(taddr + j * 32, v);
      uint32_t w[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(v[i]);
      stage_store(cx, &P.tm, n * BN + j * 32, cx.row_base, w, P.accumulate != 0);
    }
  }
};

}  // namespace kd
