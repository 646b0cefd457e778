// Persistent, warp-specialised tcgen05 GEMM with pluggable epilogues.
//
// One CTA per SM, CTA pairs (clusters of two) computing 256 x 256 tiles with
// cta_group::2 MMAs.  Warp 0 issues TMA loads into a STAGES-deep shared-memory
// ring, warp 1 of the pair leader issues tcgen05.mma (bf16 x bf16 -> fp32 in
// tensor memory), warps 2-5 run the epilogue straight out of tensor memory.
// Two 128 x 256 fp32 accumulators per CTA (all 512 TMEM columns) let the
// epilogue of one tile overlap the MMAs of the next.
//
// Work is a list of units; a unit is one tile band (m) and a contiguous range
// of 256-column tiles [n0, n1).  All three roles walk the same unit sequence
// (problem 0 round-robin over the pairs, then the pair's share of problem 1;
// see GemmArgs), so no scheduling state is shared between them.  The
// epilogue object lives for a unit, which is what lets the forward epilogue
// carry a running max / sum-exp, and the dZ epilogue its token's scale and
// teacher cursor, across the tiles of a range.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "kd_ptx.cuh"
#include "kd_schedule.h"
#include "kd_small_kernels.cuh"

namespace kd {

constexpr int BM = 128;          // accumulator rows per CTA (TMEM lanes)
constexpr int BN = 256;          // tile columns (TMEM columns per accumulator)
constexpr int BK = 64;           // bf16 elements per 128-byte swizzle row
constexpr int UMMA_K = 16;       // K of one tcgen05.mma kind::f16
constexpr int GEMM_THREADS = 192;   // warps: 0 TMA, 1 MMA, 2-5 epilogue
constexpr float kLog2e = 1.4426950408889634f;   // log2(e)
constexpr int TMEM_COLS = 512;

// Per-variant tile geometry.  PAIR = false: one CTA computes a 128 x 256 tile
// (A 128 rows, B 256 rows per stage).  PAIR = true: a cluster of two CTAs
// computes a 256 x 256 tile with cta_group::2 MMAs; each CTA stages its own
// 128 rows of A and 128 rows of B, holds its 128 accumulator rows in its own
// tensor memory, and the pair leader issues the MMAs.
template <bool PAIR, bool STAGING = true>
struct Geo {
  static constexpr int TILE_M = PAIR ? 2 * BM : BM;
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;          // B rows staged per CTA
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;       // per CTA
  // Epilogues that store through shared memory need two 16 KB staging
  // buffers; without them the pair variant fits a seventh stage.
  static constexpr int STAGES = PAIR ? (STAGING ? 6 : 7) : 4;
  static constexpr int STAGING_BYTES = STAGING ? 2 * BM * 128 : 0;  // two 128-row x 128-byte buffers
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + STAGING_BYTES + 1024 /*align*/ + 256 /*barriers*/;
  static constexpr uint32_t TX_BYTES = (PAIR ? 2 : 1) * STAGE_BYTES;  // per stage, whole tile
  static constexpr uint32_t TX_B_BYTES = (PAIR ? 2 : 1) * B_BYTES;    // per stage holding only B (wide units)
};

// One GEMM as the kernel sees it: its tile schedule, K blocks per tile, and
// offsets added to the tensor-map coordinates of A and B.
struct ProbArgs {
  Raster raster;
  int num_kb;           // BK-wide K blocks per tile
  int a_row0, b_row0;   // added to the row (M / N) coordinate
  int a_k0, b_k0;       // added to the K coordinate
  int dyn_role;         // with GemmArgs::dyn: the live rows are this GEMM's M (1: one tile per
                        // unit, 3: band x column range units) or its K (2)
  int dyn_bands_fastest;
  int dyn_zero_fill;    // role 2 with no live rows: still write the (zero) output tiles
  int wide_cols;        // > 0: wide units (Prob WIDE): its 256-column tiles; the raster counts pairs of them
};

// K blocks of MMA work per unit of a problem, the joint schedule's cost: a
// wide unit's K block runs two MMA blocks (one per column tile).  A problem
// declared WIDE runs wide units when the launch sets wide_cols.
KD_HD int64_t unit_cost(const ProbArgs& pa) {
  return (int64_t)pa.raster.tiles_per_split * pa.num_kb * (pa.wide_cols > 0 ? 2 : 1);
}

// A launch over rows whose number is known only on the device (a chunk of the
// compacted token list): the host plans `chunk` rows; every thread of the
// kernel reads the live total and rebuilds the schedule for
// clamp(*count - row0, 0, chunk) rows.
struct DynRows {
  const int* count;     // null: a static launch
  int row0;
  int chunk;
};

// A launch runs problem 0 and, optionally, problem 1.  Problem 0's units go
// round-robin over the groups (CTAs, or CTA pairs); problem 1's are dealt by
// `joint` (see joint_plan), so that every group gets about the same number
// of K blocks in total.  Every role of a group walks the same sequence.
struct GemmArgs {
  ProbArgs prob[2];
  JointPlan joint;
  DynRows dyn;
  Status* status;
  // Optional wave pacing (zeroed counters, wave_slots_bound of them; see
  // wave_slot): a CTA's producer starts a wave of a round-robin only once
  // every CTA with that wave has issued all loads of the previous one, so the
  // CTAs that share operand tiles keep reading them together.  Pacing only: a
  // wait gives up after kWaveWaitNs and the CTA goes on.
  unsigned int* wave_sync;
};

constexpr uint64_t kWaveWaitNs = 20000000ull;   // 20 ms

__device__ __forceinline__ void wave_barrier(unsigned int* counter, unsigned int expected) {
  atomicAdd(counter, 1u);
  const uint64_t t0 = globaltimer_ns();
  while (*reinterpret_cast<volatile unsigned int*>(counter) < expected) {
    if (globaltimer_ns() - t0 > kWaveWaitNs) break;
    __nanosleep(64);
  }
}

// The schedule of a launch with live row count `rows` (see DynRows).
template <class G, bool HAS_P1>
__device__ __forceinline__ void apply_live_rows(GemmArgs& a, int rows, int ngroups) {
#pragma unroll
  for (int p = 0; p < (HAS_P1 ? 2 : 1); ++p) {
    ProbArgs& pa = a.prob[p];
    if (pa.dyn_role == 1) {
      pa.raster = tile_raster(ceil_div64(rows, G::TILE_M), pa.raster.n_tiles, pa.dyn_bands_fastest != 0);
    } else if (pa.dyn_role == 3) {
      pa.raster = forward_raster(ceil_div64(rows, G::TILE_M), pa.raster.n_tiles, ngroups, 0, 0, kMaxDzSplits);
    } else if (pa.dyn_role == 2) {
      pa.num_kb = (int)ceil_div64(rows, BK);
      if (rows == 0 && !pa.dyn_zero_fill) pa.raster.num_units = 0;
    }
  }
  if constexpr (HAS_P1)
    a.joint = joint_plan(a.prob[0].raster.num_units, unit_cost(a.prob[0]), a.prob[1].raster.num_units,
                         unit_cost(a.prob[1]), ngroups);
}

// Compile-time description of a problem: its epilogue, operand majorness,
// the L2 eviction priority of each operand's loads (L2Hint), and whether its
// units are wide.  A wide unit computes two neighbouring 256-column tiles of
// one band (column tiles 2n and 2n + 1 for raster column n) into the two
// accumulators at once, so each K block's A tile is loaded once for both:
// three quarters of the operand bytes per MMA block of a one-tile unit.  The
// epilogue of a wide unit cannot overlap the next unit's MMAs, so wide units
// suit problems whose tiles run many K blocks.
template <class EpiT, bool AMN, bool BMN, int AH = kL2Normal, int BH = kL2Normal, bool W = false>
struct Prob {
  using Epi = EpiT;
  static constexpr bool A_MN = AMN, B_MN = BMN, present = true, WIDE = W;
  static constexpr int A_HINT = AH, B_HINT = BH;
};

struct EpiNone;
struct NoProb {
  using Epi = EpiNone;
  static constexpr bool A_MN = false, B_MN = false, present = false, WIDE = false;
  static constexpr int A_HINT = kL2Normal, B_HINT = kL2Normal;
};

// Loads one operand tile (rows x BK) for K block kb into shared memory.
//  K-major: one box {BK, rows} at (k, row).  The smem tile is rows x 128 B,
//           8-row groups 1024 B apart (SBO), 128-byte swizzled.
//  MN-major: rows/64 boxes {64, BK} at (row + 64 i, k).  Each box is BK
//           K-rows of 128 B (64 MN elements); boxes are BK*128 B apart (LBO).
template <bool MN_MAJOR, int ROWS, bool PAIR>
__device__ __forceinline__ void load_operand(uint32_t dst, const CUtensorMap* tm, int row, int k,
                                             uint32_t bar, uint64_t policy) {
  if constexpr (!MN_MAJOR) {
    if constexpr (PAIR) tma_load_2d_pair_hint(dst, tm, k, row, bar, policy);
    else tma_load_2d_hint(dst, tm, k, row, bar, policy);
  } else {
#pragma unroll
    for (int i = 0; i < ROWS / 64; ++i) {
      if constexpr (PAIR) tma_load_2d_pair_hint(dst + i * (BK * 128), tm, row + 64 * i, k, bar, policy);
      else tma_load_2d_hint(dst + i * (BK * 128), tm, row + 64 * i, k, bar, policy);
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
  int rows_valid;       // live rows of a DynRows launch, else -1
};

// Writes one 128-byte segment per thread (its row) into the next staging
// buffer with the 128-byte swizzle, then one thread stores (or adds) the
// 128-row box to global memory at (x, y) with TMA.
struct NoFix {
  __device__ __forceinline__ void operator()(uint32_t, uint32_t) const {}
};

// `fix(rowa, sw)` may rewrite elements of the thread's own row after it is
// written (16-byte chunk k of the row sits at rowa + ((k ^ sw) << 4)).
template <class Fix = NoFix>
__device__ __forceinline__ void stage_store(EpiCtx& cx, const CUtensorMap* tm, int x, int y,
                                            const uint32_t (&w)[32], bool reduce_add,
                                            int hint = kL2Normal, const Fix& fix = Fix{}) {
  const uint32_t buf = cx.stage[cx.seq & 1u];
  if (cx.issuer && cx.seq >= 2) bulk_wait_read<1>();     // buffer's previous store has read it
  epilogue_bar_sync(128);
  const uint32_t rowa = buf + (uint32_t)cx.rr * 128u;
  const uint32_t sw = (uint32_t)(cx.rr & 7);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    st_shared_v4(rowa + (((uint32_t)k ^ sw) << 4), w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
  fix(rowa, sw);
  fence_proxy_async_shared();
  epilogue_bar_sync(128);
  if (cx.issuer) {
    const uint64_t pol = make_l2_policy(hint);
    if (reduce_add) tma_reduce_add_2d_hint(tm, x, y, buf, pol);
    else tma_store_2d_hint(tm, x, y, buf, pol);
    bulk_commit();
  }
  ++cx.seq;
}

template <bool FIRST, class A, class B>
__device__ __forceinline__ auto& pick(A& a, B& b) {
  if constexpr (FIRST) return a; else return b;
}

// ---------------------------------------------------------------- pipeline roles
//
// Shared-memory layout of a GEMM CTA (G = Geo<...>): STAGES operand stages,
// the epilogue's staging buffers, then the mbarriers:
//   full[s]   stage s loaded (TMA bytes of both CTAs of a pair, on the leader)
//   empty[s]  stage s consumed by the MMAs (commit, multicast to the pair)
//   tfull[a]  accumulator a written (commit, multicast to the pair)
//   tempty[a] accumulator a drained by every epilogue thread (on the leader)
// followed by the tensor-memory address slot and the CTA's abort flag.
template <class G>
struct Smem {
  uint32_t sbase, staging, bar_base;
  uint32_t* tmem_slot;
  volatile int* abort_flag;
  __device__ __forceinline__ uint32_t full(int s) const { return bar_base + 8u * s; }
  __device__ __forceinline__ uint32_t empty(int s) const { return bar_base + 8u * (G::STAGES + s); }
  __device__ __forceinline__ uint32_t tfull(int a) const { return bar_base + 8u * (2 * G::STAGES + a); }
  __device__ __forceinline__ uint32_t tempty(int a) const { return bar_base + 8u * (2 * G::STAGES + 2 + a); }
};

template <class G>
__device__ __forceinline__ Smem<G> smem_layout(uint8_t* smem_raw) {
  Smem<G> L;
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  L.sbase = smem_u32(smem);
  L.staging = L.sbase + G::STAGES * G::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G::STAGES * G::STAGE_BYTES + G::STAGING_BYTES);
  L.bar_base = smem_u32(bars);
  L.tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * G::STAGES + 4);
  L.abort_flag = reinterpret_cast<volatile int*>(L.tmem_slot + 1);
  return L;
}

// Barrier init and tensor-memory allocation; returns the TMEM base address.
template <class G, bool PAIR>
__device__ __forceinline__ uint32_t pipeline_setup(const Smem<G>& L) {
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < G::STAGES; ++s) {
      mbar_init(L.full(s), 1);
      mbar_init(L.empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(L.tfull(a), 1);
      mbar_init(L.tempty(a), (PAIR ? 2 : 1) * 4 * 32);
    }
    *L.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(L.tmem_slot), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(L.tmem_slot), TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync_all(); else __syncthreads();
  tc_fence_after();
  return *L.tmem_slot;
}

// Records a failure, lets issued asynchronous work land, and releases the
// tensor memory once neither CTA of a pair can still touch the other's.
template <class G, bool PAIR>
__device__ __forceinline__ void pipeline_teardown(const Smem<G>& L, bool failed, Status* status,
                                                  uint32_t tmem_base) {
  if (failed) {
    *L.abort_flag = 1;
    atomicOr(&status->timeout, 1u);
  }
  __syncwarp();
  __syncthreads();
  if (*L.abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) { }
    __syncthreads();
  }
  if constexpr (PAIR) cluster_sync_all();
  if ((threadIdx.x >> 5) == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// Per-role pipeline position, carried across units and problems.
struct RoleState {
  int stage = 0;
  uint32_t phase = 0;
  int acc = 0;
  uint32_t acc_phase = 0;
};

template <class G>
__device__ __forceinline__ void next_stage(RoleState& st) {
  if (++st.stage == G::STAGES) { st.stage = 0; st.phase ^= 1u; }
}

__device__ __forceinline__ void next_acc(RoleState& st) {
  st.acc ^= 1;
  if (st.acc == 0) st.acc_phase ^= 1u;
}

// Column tiles of raster column n: [first, first + count).
template <class P>
__device__ __forceinline__ void unit_cols(const ProbArgs& pa, int n, int& first, int& count) {
  first = n;
  count = 1;
  if constexpr (P::WIDE) {
    if (pa.wide_cols > 0) {
      first = 2 * n;
      count = wide_count(n, pa.wide_cols);
    }
  }
}

// TMA producer: all K blocks of every tile of unit u.
template <class G, bool PAIR, class P>
__device__ __forceinline__ bool produce_unit(const Smem<G>& L, RoleState& st, uint32_t rank,
                                             const ProbArgs& pa, const CUtensorMap* tA,
                                             const CUtensorMap* tB, int u) {
  int m, split, n0, n1;
  decode_unit(pa.raster, u, m, split, n0, n1);
  for (int n = n0; n < n1; ++n) {
    int c0, nc;
    unit_cols<P>(pa, n, c0, nc);
    for (int kb = 0; kb < pa.num_kb; ++kb) {
      // stage 1: A and the first column tile's B; stage 2 (wide units): the second B
      for (int h = 0; h < nc; ++h) {
        if (!mbar_wait_bounded(L.empty(st.stage), st.phase ^ 1u, L.abort_flag)) return false;
        const uint32_t sa = L.sbase + st.stage * G::STAGE_BYTES;
        const uint32_t sb = sa + G::A_BYTES;
        const uint32_t fb = PAIR ? mapa_shared(L.full(st.stage), 0) : L.full(st.stage);
        if (rank == 0) mbar_arrive_expect_tx(L.full(st.stage), h == 0 ? G::TX_BYTES : G::TX_B_BYTES);
        if (h == 0)
          load_operand<P::A_MN, BM, PAIR>(sa, tA, pa.a_row0 + m * G::TILE_M + (int)rank * BM,
                                          pa.a_k0 + kb * BK, fb, make_l2_policy(P::A_HINT));
        load_operand<P::B_MN, G::B_ROWS, PAIR>(sb, tB, pa.b_row0 + (c0 + h) * BN + (int)rank * G::B_ROWS,
                                               pa.b_k0 + kb * BK, fb, make_l2_policy(P::B_HINT));
        next_stage<G>(st);
      }
    }
  }
  return true;
}

// MMA issuer (pair leader, one thread): every tile of unit u into the next
// free accumulator.
template <class G, bool PAIR, class P>
__device__ __forceinline__ bool mma_unit(const Smem<G>& L, RoleState& st, uint32_t tmem_base,
                                         const ProbArgs& pa, int u) {
  constexpr uint32_t idesc = idesc_bf16_f32(G::TILE_M, BN, P::A_MN, P::B_MN);
  int m, split, n0, n1;
  decode_unit(pa.raster, u, m, split, n0, n1);
  for (int n = n0; n < n1; ++n) {
    int c0, nc;
    unit_cols<P>(pa, n, c0, nc);
    // the unit's accumulators: this one and, for a wide unit, the next
    RoleState a2 = st;
    next_acc(a2);
    if (!mbar_wait_bounded(L.tempty(st.acc), st.acc_phase ^ 1u, L.abort_flag)) return false;
    if (nc == 2 && !mbar_wait_bounded(L.tempty(a2.acc), a2.acc_phase ^ 1u, L.abort_flag)) return false;
    tc_fence_after();
    const uint32_t d0 = tmem_base + st.acc * BN, d1 = tmem_base + a2.acc * BN;
    for (int kb = 0; kb < pa.num_kb; ++kb) {
      // stage 1 holds A and the first B, stage 2 (wide units) the second B
      RoleState s2 = st;
      next_stage<G>(s2);
      if (!mbar_wait_bounded(L.full(st.stage), st.phase, L.abort_flag)) return false;
      if (nc == 2 && !mbar_wait_bounded(L.full(s2.stage), s2.phase, L.abort_flag)) return false;
      tc_fence_after();
      const uint32_t sa = L.sbase + st.stage * G::STAGE_BYTES;
      const uint32_t sb0 = sa + G::A_BYTES;
      const uint32_t sb1 = L.sbase + s2.stage * G::STAGE_BYTES + G::A_BYTES;
#pragma unroll
      for (int kk = 0; kk < BK / UMMA_K; ++kk) {
        const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
        const uint64_t da = operand_desc<P::A_MN>(sa, kk);
        if constexpr (PAIR) {
          tc_mma_bf16_pair(d0, da, operand_desc<P::B_MN>(sb0, kk), idesc, accum);
          if (nc == 2) tc_mma_bf16_pair(d1, da, operand_desc<P::B_MN>(sb1, kk), idesc, accum);
        } else {
          tc_mma_bf16(d0, da, operand_desc<P::B_MN>(sb0, kk), idesc, accum);
          if (nc == 2) tc_mma_bf16(d1, da, operand_desc<P::B_MN>(sb1, kk), idesc, accum);
        }
      }
      for (int h = 0; h < nc; ++h) {
        if constexpr (PAIR) tc_commit_pair_mc(L.empty(st.stage), 0x3); else tc_commit(L.empty(st.stage));
        next_stage<G>(st);
      }
    }
    for (int h = 0; h < nc; ++h) {
      if constexpr (PAIR) tc_commit_pair_mc(L.tfull(st.acc), 0x3); else tc_commit(L.tfull(st.acc));
      next_acc(st);
    }
  }
  return true;
}

// Epilogue (all 128 threads of warps 2-5): drain each tile of unit u.
template <class G, bool PAIR, class P, class Epi>
__device__ __forceinline__ bool epi_unit(const Smem<G>& L, RoleState& st, uint32_t rank,
                                         uint32_t lane_addr, int row, Epi& epi,
                                         const typename Epi::Params& ep, const CUtensorMap* out,
                                         const ProbArgs& pa, int u, EpiCtx& cx) {
  int m, split, n0, n1;
  decode_unit(pa.raster, u, m, split, n0, n1);
  const int grow = m * G::TILE_M + row;
  cx.row_base = m * G::TILE_M + (int)rank * BM;
  epi.begin_unit(ep, grow, split, n0, cx);
  for (int n = n0; n < n1; ++n) {
    int c0, nc;
    unit_cols<P>(pa, n, c0, nc);
    for (int h = 0; h < nc; ++h) {      // a wide unit's two tiles, one accumulator each
      // One outcome for all 128 epilogue threads: tcgen05.ld needs whole
      // warps and the store path synchronises the four warps.
      const bool ok = epilogue_bar_and(128, mbar_wait_bounded(L.tfull(st.acc), st.acc_phase, L.abort_flag));
      if (!ok) return false;
      tc_fence_after();
      epi.tile(ep, out, grow, c0 + h, lane_addr + st.acc * BN, cx);
      tc_fence_before();
      if constexpr (PAIR) mbar_arrive_cluster(mapa_shared(L.tempty(st.acc), 0));
      else mbar_arrive(L.tempty(st.acc));
      next_acc(st);
    }
  }
  epi.end_unit(ep, grow, split);
  return true;
}

__device__ __forceinline__ EpiCtx make_epi_ctx(uint32_t staging) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  EpiCtx cx;
  cx.stage[0] = staging;
  cx.stage[1] = staging + BM * 128;
  cx.rr = (warp & 3) * 32 + lane;
  cx.issuer = (threadIdx.x == 64);
  cx.seq = 0;
  cx.row_base = 0;
  cx.rows_valid = -1;
  return cx;
}

// One or two GEMM problems per launch (see GemmArgs).  tmO0 / tmO1 are the
// output maps of epilogues that store through TMA (unused otherwise).
template <class P0, class P1, bool PAIR>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
               const __grid_constant__ CUtensorMap tmO0,
               const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
               const __grid_constant__ CUtensorMap tmO1,
               const __grid_constant__ GemmArgs args,
               const __grid_constant__ typename P0::Epi::Params ep0,
               const __grid_constant__ typename P1::Epi::Params ep1) {
  using G = Geo<PAIR, P0::Epi::kStaging || P1::Epi::kStaging>;
  extern __shared__ uint8_t smem_raw[];
  const Smem<G> L = smem_layout<G>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int group = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int ngroups = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmB0);
    if constexpr (P1::present) {
      tma_prefetch_desc(&tmA1);
      tma_prefetch_desc(&tmB1);
    }
  }
  const uint32_t tmem_base = pipeline_setup<G, PAIR>(L);

  // The schedule; a launch over a device-side row count rebuilds it here.
  GemmArgs A = args;
  int live_rows = -1;
  if (args.dyn.count) {
    int r = *args.dyn.count - args.dyn.row0;
    r = r < 0 ? 0 : (r > args.dyn.chunk ? args.dyn.chunk : r);
    live_rows = r;
    apply_live_rows<G, P1::present>(A, r, ngroups);
  }

  // This group's units: problem 0 round-robin, then its share of problem 1.
  auto for_each_unit = [&](auto&& body) {
    bool ok = true;
    int k = 0;
    for (int u = group; ok && u < A.prob[0].raster.num_units; u += ngroups, ++k)
      ok = body(P0{}, A.prob[0], &tmA0, &tmB0, u, k);
    if constexpr (P1::present) {
      const int n1 = joint_count(A.joint, A.prob[1].raster.num_units, ngroups, group);
      for (int i = 0; ok && i < n1; ++i)
        ok = body(P1{}, A.prob[1], &tmA1, &tmB1, joint_unit(A.joint, ngroups, group, i), i);
    }
    return ok;
  };

  bool failed = false;
  RoleState st;
  if (warp == 0) {
    if (lane == 0)
      failed = !for_each_unit([&](auto pt, const ProbArgs& pa, const CUtensorMap* tA,
                                  const CUtensorMap* tB, int u, int ord) {
        if (A.wave_sync) {
          constexpr int prob = std::is_same<decltype(pt), P0>::value ? 0 : 1;
          int expected = 0;
          const int slot = wave_slot(prob, ord, group, ngroups, A.prob[0].raster.num_units,
                                     P1::present ? A.prob[1].raster.num_units : 0, A.joint, &expected);
          if (slot >= 0) wave_barrier(A.wave_sync + slot, (unsigned int)((PAIR ? 2 : 1) * expected));
        }
        return produce_unit<G, PAIR, decltype(pt)>(L, st, rank, pa, tA, tB, u);
      });
  } else if (warp == 1) {
    if (lane == 0 && rank == 0)
      failed = !for_each_unit([&](auto pt, const ProbArgs& pa, const CUtensorMap*, const CUtensorMap*,
                                  int u, int) { return mma_unit<G, PAIR, decltype(pt)>(L, st, tmem_base, pa, u); });
  } else {
    const int q = warp & 3;
    const int row = (int)rank * BM + q * 32 + lane;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
    typename P0::Epi epi0;
    typename P1::Epi epi1;
    EpiCtx cx = make_epi_ctx(L.staging);
    cx.rows_valid = live_rows;
    failed = !for_each_unit([&](auto pt, const ProbArgs& pa, const CUtensorMap*, const CUtensorMap*,
                                int u, int) {
      using P = decltype(pt);
      constexpr bool first = std::is_same<P, P0>::value;
      return epi_unit<G, PAIR, P>(L, st, rank, lane_addr, row, pick<first>(epi0, epi1), pick<first>(ep0, ep1),
                               first ? &tmO0 : &tmO1, pa, u, cx);
    });
    if (cx.issuer) bulk_wait<0>();          // every TMA store of this CTA has completed
  }
  pipeline_teardown<G, PAIR>(L, failed, A.status, tmem_base);
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

// v[i] for a run-time i in [0, 64), by a tree of selects on i's bits: the
// array stays in registers (an indexed read would put it in local memory).
__device__ __forceinline__ float pick64(const float (&v)[64], int i) {
  float a[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) a[k] = (i & 32) ? v[k + 32] : v[k];
#pragma unroll
  for (int w = 16; w > 0; w >>= 1) {
    const bool hi = (i & w) != 0;
#pragma unroll
    for (int k = 0; k < w; ++k) a[k] = hi ? a[k + w] : a[k];
  }
  return a[0];
}

// A thread's walk over its token's index-sorted teacher entries (row of Kp
// slots ending in kSentinel) as the vocabulary columns stream past in
// increasing order.  (i0, p0) is the next entry; the one after it is loaded
// as soon as i0 is consumed, long before it is compared, so a hit does not
// stall the epilogue on a global load.
struct TeacherCursor {
  const int32_t* trow;
  const float* prow;
  int cur, kp;
  int i0, i1;
  float p0, p1;

  __device__ __forceinline__ void none() {
    trow = nullptr;
    prow = nullptr;
    cur = kp = 0;
    i0 = i1 = kSentinel;
    p0 = p1 = 0.f;
  }
  __device__ __forceinline__ void start(const int32_t* t, const float* p, int kp_, int col) {
    trow = t;
    prow = p;
    kp = kp_;
    cur = lower_bound_row(t, kp_, col);
    i0 = t[cur];
    p0 = p[cur];
    i1 = cur + 1 < kp ? t[cur + 1] : kSentinel;
    p1 = cur + 1 < kp ? p[cur + 1] : 0.f;
  }
  __device__ __forceinline__ void advance() {
    i0 = i1;
    p0 = p1;
    ++cur;
    i1 = cur + 1 < kp ? trow[cur + 1] : kSentinel;
    p1 = cur + 1 < kp ? prow[cur + 1] : 0.f;
  }
};

// Forward: running max / sum-exp over the unit's vocabulary columns and the
// gathered sum of p * z at the teacher's columns; one (m, s, g) partial per
// token per split.  Columns >= V are -inf.  The sum is of exp((z - m) * zs)
// (zs = 1, or 1 / T when the student is taken at temperature T), computed as
// 2^(z * zl2 - m * zl2) with zl2 = zs log2(e).
struct EpiFwd {
  static constexpr bool kStaging = false;
  struct Params {
    int N, V, Kp;
    float zl2;
    const int32_t* tidx;
    const float* tp;
    float* part_m;
    float* part_s;
    float* part_g;
  };
  float mrun, srun, grun;
  int grow;
  TeacherCursor tc;

  __device__ __forceinline__ void begin_unit(const Params& P, int grow_, int, int n0, const EpiCtx&) {
    grow = grow_;
    mrun = -INFINITY;
    srun = 0.f;
    grun = 0.f;
    if (grow < P.N)
      tc.start(P.tidx + (size_t)grow * P.Kp, P.tp + (size_t)grow * P.Kp, P.Kp, n0 * BN);
    else
      tc.none();
  }

  __device__ __forceinline__ void tile(const Params& P, const CUtensorMap*, int, int n, uint32_t taddr,
                                       EpiCtx&) {
#pragma unroll 1
    for (int j = 0; j < BN / 64; ++j) {
      float v[64];
      __syncwarp();
      tmem_ld_32x32b_x64(taddr + j * 64, v);
      const int c0 = n * BN + j * 64;
      if (c0 + 64 > P.V) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (c0 + i >= P.V) v[i] = -INFINITY;
      }
      while (tc.i0 < c0 + 64) {             // a teacher column in this group (rare)
        grun += tc.p0 * pick64(v, tc.i0 - c0);
        tc.advance();
      }
      // group max (pairwise tree), then the rescaled running sum-exp with
      // 2^(z log2(e) - m log2(e)): one FFMA and one ex2 per element
      float t[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) t[i] = fmaxf(v[i], v[i + 32]);
#pragma unroll
      for (int w = 16; w > 0; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) t[i] = fmaxf(t[i], t[i + w]);
      const float mn = fmaxf(mrun, t[0]);
      if (mn == -INFINITY) continue;
      // packed fp32 pairs (FFMA2 / FADD2) halve the epilogue's FMA and add
      // instructions, which compete with the MMA issue for the SM
      const float zl2 = P.zl2;
      const float mb = mn * zl2;
      const float2 zl2v = make_float2(zl2, zl2), nmb = make_float2(-mb, -mb);
      float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 64; i += 4) {
        float2 e01 = __ffma2_rn(make_float2(v[i + 0], v[i + 1]), zl2v, nmb);
        float2 e23 = __ffma2_rn(make_float2(v[i + 2], v[i + 3]), zl2v, nmb);
        e01.x = ex2_approx(e01.x);
        e01.y = ex2_approx(e01.y);
        e23.x = ex2_approx(e23.x);
        e23.y = ex2_approx(e23.y);
        a01 = __fadd2_rn(a01, e01);
        a23 = __fadd2_rn(a23, e23);
      }
      srun = srun * ex2_approx((mrun - mn) * zl2) + ((a01.x + a01.y) + (a23.x + a23.y));
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

// Backward, per chunk: dZ = c_n (exp(z zs - lse_n) - p at the teacher's
// columns), one unit per band and range of column tiles (the row's scale,
// lse and teacher cursor set once per unit), rounded to bf16 and stored for
// the chunk's tokens (row-major,
// ldz columns) through shared memory and TMA (`out`: the chunk buffer, bf16,
// box {64, 128}, 128-byte swizzle).  zs = 1, or 1 / T for the
// student-temperature variant, whose extra factor T on c_n comes in as gfac.
// A token without teacher entries has a zero row.  Columns in [V, ldz) and
// rows at or past the chunk's end (up to the buffer's rows) are written as 0,
// so that a buffer reused for a shorter last chunk holds no stale rows.
struct EpiDz {
  static constexpr bool kStaging = true;
  struct Params {
    int rows_valid;        // tokens in this chunk
    int row0;              // global token index of chunk row 0
    int V, ldz, Kp;
    float zl2;             // zs log2(e)
    float gfac;            // 1, or T
    const int32_t* rowmap; // null, or chunk row r is token rowmap[row0 + r]
    const int32_t* tidx;
    const float* tp;
    const float* lse;
    const float* mask;     // may be null
    const float* cscale;   // device scalar g / sum(mask)
  };
  // The row's state for a unit (a band and a range of column tiles, in
  // increasing order): c exp(z zs - lse) = 2^(z zl2 - bias) with
  // bias = lse log2(e) - log2(c), one FFMA and one ex2 per element.  c = 0
  // (masked token, token without teacher entries) and rows past the chunk
  // give bias = +inf, hence exact zeros.  A negative c (negative upstream
  // gradient or mask weight) is applied as a sign flip of the packed bf16
  // pair.
  float bias, c;
  uint32_t sgn;
  TeacherCursor tc;

  __device__ __forceinline__ void begin_unit(const Params& P, int r, int, int n0, const EpiCtx& cx) {
    bias = INFINITY;
    c = 0.f;
    sgn = 0u;
    tc.none();
    if (r < (cx.rows_valid >= 0 ? cx.rows_valid : P.rows_valid)) {
      const int grow = P.rowmap ? P.rowmap[P.row0 + r] : P.row0 + r;
      const int32_t* trow = P.tidx + (size_t)grow * P.Kp;
      const float* prow = P.tp + (size_t)grow * P.Kp;
      tc.start(trow, prow, P.Kp, n0 * BN);
      const float cs = trow[0] == kSentinel ? 0.f : (P.mask ? P.mask[grow] : 1.f) * (*P.cscale) * P.gfac;
      c = fabsf(cs);
      sgn = cs < 0.f ? 0x80008000u : 0u;
      bias = P.lse[grow] * kLog2e - log2f(c);
    }
  }
  __device__ __forceinline__ void end_unit(const Params&, int, int) {}

  __device__ __forceinline__ void tile(const Params& P, const CUtensorMap* out, int, int n,
                                       uint32_t taddr, EpiCtx& cx) {
    const float zl2 = P.zl2;
#pragma unroll 1
    for (int j = 0; j < BN / 64; ++j) {
      float v[64];
      __syncwarp();
      tmem_ld_32x32b_x64(taddr + j * 64, v);
      const int c0 = n * BN + j * 64;
      const float2 zl2v = make_float2(zl2, zl2), nb = make_float2(-bias, -bias);
#pragma unroll
      for (int i = 0; i < 64; i += 2) {
        const float2 e = __ffma2_rn(make_float2(v[i], v[i + 1]), zl2v, nb);
        v[i] = ex2_approx(e.x);
        v[i + 1] = ex2_approx(e.y);
      }
      if (c0 + 64 > P.V) {                  // last vocabulary tile: zero columns >= V
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (c0 + i >= P.V) v[i] = 0.f;
      }
      uint32_t w[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
      if (sgn) {
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] ^= sgn;
      }
      // the teacher's columns in this group (rare): subtract c p from the
      // staged bf16 value, stored as sign * c exp(..), so minus (signed c) p
      const float cs = sgn ? -c : c;
      TeacherCursor& t = tc;
      stage_store(cx, out, c0, cx.row_base, w, false, kL2Normal, [&](uint32_t rowa, uint32_t sw) {
        while (t.i0 < c0 + 64) {
          const uint32_t off = (uint32_t)(t.i0 - c0);
          const uint32_t a = rowa + (((off >> 3) ^ sw) << 4) + ((off & 7u) << 1);
          const uint16_t h = ld_shared_u16(a);
          const float x = __bfloat162float(__ushort_as_bfloat16(h)) - cs * t.p0;
          st_shared_u16(a, __bfloat16_as_ushort(__float2bfloat16_rn(x)));
          t.advance();
        }
      });
    }
  }
};

// Backward, per chunk: dH rows of the chunk's tokens, bf16, through shared
// memory and TMA (`out`: dH [N][d] bf16, box {64, 128}, 128-byte swizzle;
// chunk row r is dH row row0 + r).
struct EpiDh {
  static constexpr bool kStaging = true;
  struct Params {
    int row0;
  };
  __device__ __forceinline__ void begin_unit(const Params&, int, int, int, const EpiCtx&) {}
  __device__ __forceinline__ void end_unit(const Params&, int, int) {}

  __device__ __forceinline__ void tile(const Params& P, const CUtensorMap* out, int, int n,
                                       uint32_t taddr, EpiCtx& cx) {
#pragma unroll 1
    for (int j = 0; j < BN / 64; ++j) {
      float v[64];
      __syncwarp();
      tmem_ld_32x32b_x64(taddr + j * 64, v);
      uint32_t w[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
      stage_store(cx, out, n * BN + j * 64, P.row0 + cx.row_base, w, false);
    }
  }
};

// Backward, per chunk: dW (+)= dZ^T H for 128 vocabulary rows x 256 columns
// per CTA, fp32, stored (first chunk without accumulation) or added in place
// by TMA reductions: the memory system does the read-modify-write.
struct EpiDw {
  static constexpr bool kStaging = true;
  struct Params {
    int accumulate;        // `out`: dW [V][d] fp32, box {32, 128}, 128-byte swizzle
  };
  __device__ __forceinline__ void begin_unit(const Params&, int, int, int, const EpiCtx&) {}
  __device__ __forceinline__ void end_unit(const Params&, int, int) {}

  __device__ __forceinline__ void tile(const Params& P, const CUtensorMap* out, int, int n,
                                       uint32_t taddr, EpiCtx& cx) {
    // A launch with no live rows (DynRows) ran no MMA: the tile is zero.
    const bool empty = cx.rows_valid == 0;
#pragma unroll 1
    for (int j = 0; j < BN / 32; ++j) {
      float v[32];
      __syncwarp();
      if (empty) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      } else {
        tmem_ld_32x32b_x32(taddr + j * 32, v);
      }
      uint32_t w[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(v[i]);
      stage_store(cx, out, n * BN + j * 32, cx.row_base, w, P.accumulate != 0, kL2EvictFirst);
    }
  }
};

// Teacher logits, per chunk: the fp32 tile stored like EpiDw's first chunk
// (columns past V clipped by the tensor map), and per token row and tile the
// order key (float_key) of the row's largest logit in the tile.  The top-K
// selection takes its first threshold from these maxima and reads only the
// tiles that can hold a top-K logit.
struct EpiZ32 {
  static constexpr bool kStaging = true;
  struct Params {
    uint32_t* tmax;       // [rows][ld] keys
    int ld;               // tiles per row, ceil(V / BN)
    int rows;             // token rows of the chunk
    int V;
  };
  __device__ __forceinline__ void begin_unit(const Params&, int, int, int, const EpiCtx&) {}
  __device__ __forceinline__ void end_unit(const Params&, int, int) {}

  __device__ __forceinline__ void tile(const Params& P, const CUtensorMap* out, int grow, int n,
                                       uint32_t taddr, EpiCtx& cx) {
    float fmx = -INFINITY;                // max of the logits, NaN if any is NaN
#pragma unroll 1
    for (int j = 0; j < BN / 32; ++j) {
      const int c0 = n * BN + j * 32;
      float v[32];
      __syncwarp();
      tmem_ld_32x32b_x32(taddr + j * 32, v);
      uint32_t w[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(v[i]);
      if (c0 + 32 <= P.V) {
#pragma unroll
        for (int i = 0; i < 32; ++i) fmx = fmax_nan(fmx, v[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c0 + i < P.V) fmx = fmax_nan(fmx, v[i]);
      }
      stage_store(cx, out, c0, cx.row_base, w, false);
    }
    uint32_t key = float_key(fmx);
    if (__any_sync(0xffffffffu, fmx != fmx)) {   // NaNs order by key: take the maximum key itself
      uint32_t km = 0u;
#pragma unroll 1
      for (int j = 0; j < BN / 32; ++j) {
        const int c0 = n * BN + j * 32;
        float v[32];
        __syncwarp();
        tmem_ld_32x32b_x32(taddr + j * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c0 + i < P.V) km = max(km, float_key(v[i]));
      }
      key = km;
    }
    if (grow < P.rows) P.tmax[(size_t)grow * P.ld + n] = key;
  }
};

// Placeholder epilogue of an absent second problem.
struct EpiNone {
  static constexpr bool kStaging = false;
  struct Params {
    int unused;
  };
  __device__ __forceinline__ void begin_unit(const Params&, int, int, int, const EpiCtx&) {}
  __device__ __forceinline__ void tile(const Params&, const CUtensorMap*, int, int, uint32_t, EpiCtx&) {}
  __device__ __forceinline__ void end_unit(const Params&, int, int) {}
};

}  // namespace kd
