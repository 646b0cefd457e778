// Host side of libkdtopkl.so: argument checks, workspace layout, TMA tensor
// maps, schedules and kernel launches for the fused chunked top-K KL loss.
//
// Forward (one call):  teacher_prep -> gemm<EpiFwd> (wave-paced) -> lse_merge
//                      -> finalize
// Backward (one call): teacher_prep -> finalize(scale) [-> compact_rows] ->
//                      for each chunk of tokens: [gather_rows ->]
//                      gemm<EpiDz> -> gemm<EpiDh + EpiDw> [-> scatter_rows]
//                      (bracketed steps: skipping masked rows)
// Teacher top-K cache writer: for each chunk, gemm<EpiZ32> (fp32 logits and
//                      their tile maxima) -> topk_select
// The fused chunked loss of "Efficient Knowledge Distillation for LLMs"
// (Japanese summary, method paragraph) projects, normalises and gathers one
// chunk at a time and recomputes each chunk in the backward pass; here the
// forward never stores logits at all (the vocabulary tiles live only in
// tensor memory) and the backward stores one chunk of bf16 dZ.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>

#include "../../include/kd_topk_kl.h"
#include "kd_gemm.cuh"
#include "kd_small_kernels.cuh"
#include "kd_topk_select.cuh"

using namespace kd;

namespace {

constexpr int kMaxDevices = 64;

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

struct Layout {
  int Kp = 0;
  int64_t ldz = 0, C = 0;
  int64_t n_prep_blocks = 0, n_merge_blocks = 0;
  size_t off_status = 0, off_scal = 0, off_mask_part = 0, off_term_part = 0;
  size_t off_tidx = 0, off_tp = 0, off_ent = 0, off_pm = 0, off_ps = 0, off_pg = 0, off_dz = 0;
  size_t off_rowmap = 0, off_nrows = 0, off_hc = 0, off_dhc = 0, off_wave = 0, off_jwave = 0;
  int64_t jwave_per_chunk = 0;
  size_t total = 0;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

Layout make_layout(int64_t N, int64_t d, int64_t V, int64_t K, int64_t chunk) {
  Layout L;
  L.Kp = (int)round_up(K + 1, 4);
  L.ldz = round_up(V, 8);
  L.C = N > 0 ? (chunk < N ? chunk : N) : 1;
  L.n_prep_blocks = ceil_div(N > 0 ? N : 1, kPrepWarps);
  L.n_merge_blocks = ceil_div(N > 0 ? N : 1, kMergeThreads);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o = align256(o + bytes); return r; };
  L.off_status = take(sizeof(Status));
  L.off_scal = take(64);
  L.off_mask_part = take(sizeof(double) * L.n_prep_blocks);
  L.off_term_part = take(sizeof(double) * L.n_merge_blocks);
  L.off_tidx = take(sizeof(int32_t) * (size_t)N * L.Kp);
  L.off_tp = take(sizeof(float) * (size_t)N * L.Kp);
  L.off_ent = take(sizeof(float) * (size_t)N);
  L.off_pm = take(sizeof(float) * (size_t)N * kMaxSplits);
  L.off_ps = take(sizeof(float) * (size_t)N * kMaxSplits);
  L.off_pg = take(sizeof(float) * (size_t)N * kMaxSplits);
  // wave counters: the forward's, and per chunk the joint launch's
  L.off_wave = take(sizeof(unsigned int) * (size_t)wave_slots_bound(ceil_div(N > 0 ? N : 1, 256) * kMaxSplits, 0));
  L.jwave_per_chunk = wave_slots_bound(ceil_div(L.C, 256) * ceil_div(d, 256), ceil_div(V, 256) * ceil_div(d, 256));
  L.off_jwave = take(sizeof(unsigned int) * (size_t)L.jwave_per_chunk * ceil_div(N > 0 ? N : 1, L.C));
  L.off_dz = take(2 * (size_t)L.C * L.ldz);   // one dZ chunk (bf16)
  // skipping rows with zero dZ: the kept tokens in order, their count, and
  // one chunk of their H rows and of their dH rows (bf16)
  L.off_rowmap = take(sizeof(int32_t) * (size_t)N);
  L.off_nrows = take(sizeof(int));
  L.off_hc = take(2 * (size_t)L.C * d);
  L.off_dhc = take(2 * (size_t)L.C * d);
  L.total = o;
  return L;
}

// The regions the forward pass alone uses, laid out as in make_layout: status
// words, scalars, the fp64 block sums, the prepared teacher cache, the
// per-split (m, s, g) partials and the forward's wave counters.  No dZ
// chunk, no joint-launch counters, no row map or row buffers.  About
// 8 Kp + 199 bytes per token, plus under 4 KiB.
Layout make_forward_layout(int64_t N, int64_t K) {
  Layout L;
  L.Kp = (int)round_up(K + 1, 4);
  L.C = 1;
  L.n_prep_blocks = ceil_div(N > 0 ? N : 1, kPrepWarps);
  L.n_merge_blocks = ceil_div(N > 0 ? N : 1, kMergeThreads);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o = align256(o + bytes); return r; };
  L.off_status = take(sizeof(Status));
  L.off_scal = take(64);
  L.off_mask_part = take(sizeof(double) * L.n_prep_blocks);
  L.off_term_part = take(sizeof(double) * L.n_merge_blocks);
  L.off_tidx = take(sizeof(int32_t) * (size_t)N * L.Kp);
  L.off_tp = take(sizeof(float) * (size_t)N * L.Kp);
  L.off_ent = take(sizeof(float) * (size_t)N);
  L.off_pm = take(sizeof(float) * (size_t)N * kMaxSplits);
  L.off_ps = take(sizeof(float) * (size_t)N * kMaxSplits);
  L.off_pg = take(sizeof(float) * (size_t)N * kMaxSplits);
  L.off_wave = take(sizeof(unsigned int) * (size_t)wave_slots_bound(ceil_div(N > 0 ? N : 1, 256) * kMaxSplits, 0));
  L.total = o;
  return L;
}

int check_shapes(int64_t N, int64_t d, int64_t V, int64_t K, float T, int64_t chunk) {
  if (N < 0 || d <= 0 || V <= 0 || K <= 0 || chunk <= 0) return KD_ERR_INVALID_ARG;
  if (!(T > 0.f) || !(T < INFINITY)) return KD_ERR_INVALID_ARG;
  if (d % 8 != 0 || d < 8) return KD_ERR_UNSUPPORTED;
  if (K > kMaxK) return KD_ERR_UNSUPPORTED;
  if (N >= (int64_t(1) << 31) || V >= (int64_t(1) << 31) || d >= (int64_t(1) << 24))
    return KD_ERR_UNSUPPORTED;
  return KD_OK;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ---------------------------------------------------------------- TMA maps

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Row-major matrix [outer][inner] (bf16, or fp32 when `f32`) with row pitch
// `pitch` elements, 128-byte-swizzled boxes of box_inner x box_outer; loads
// out of bounds read zeros, stores out of bounds are dropped.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch,
              uint32_t box_inner, uint32_t box_outer, bool f32 = false) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch * (f32 ? 4 : 2)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- device info

struct DevInfo {
  int sms = 0;
  int pair_groups = 0;          // co-resident CTA pairs of the GEMM kernel
  int64_t l2_bytes = 0;
  bool attr_set[8] = {};
};
DevInfo g_dev[kMaxDevices];

int device_sms(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (!g_dev[dev].sms) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    g_dev[dev].sms = v > 0 ? v : 148;
  }
  return g_dev[dev].sms;
}

int64_t device_l2_bytes(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return 126ll << 20;
  if (!g_dev[dev].l2_bytes) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrL2CacheSize, dev);
    g_dev[dev].l2_bytes = v > 0 ? v : (126ll << 20);
  }
  return g_dev[dev].l2_bytes;
}

// All GEMMs run as CTA pairs (cta_group::2, 256 x 256 tiles).
constexpr bool kPair = true;
using GeoP = Geo<kPair>;

template <class P0, class P1, bool PAIR>
cudaError_t launch_gemm(int slot, int dev, int groups, const CUtensorMap& ta0, const CUtensorMap& tb0,
                        const CUtensorMap& to0, const CUtensorMap& ta1, const CUtensorMap& tb1,
                        const CUtensorMap& to1, const GemmArgs& args,
                        const typename P0::Epi::Params& ep0, const typename P1::Epi::Params& ep1,
                        cudaStream_t s) {
  using G = Geo<PAIR, P0::Epi::kStaging || P1::Epi::kStaging>;
  auto kern = gemm_tc_kernel<P0, P1, PAIR>;
  if (dev >= 0 && dev < kMaxDevices && !g_dev[dev].attr_set[slot]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    g_dev[dev].attr_set[slot] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(groups * (PAIR ? 2 : 1)), 1, 1);
  cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = G::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = PAIR ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta0, tb0, to0, ta1, tb1, to1, args, ep0, ep1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// One problem per launch.
template <class P0>
cudaError_t launch_one(int slot, int dev, int groups, const CUtensorMap& ta, const CUtensorMap& tb,
                       const CUtensorMap& to, const ProbArgs& pa, Status* status,
                       const typename P0::Epi::Params& ep, cudaStream_t s, DynRows dyn = DynRows{},
                       unsigned int* wave_sync = nullptr) {
  GemmArgs a{};
  a.prob[0] = pa;
  a.status = status;
  a.dyn = dyn;
  a.wave_sync = wave_sync;
  EpiNone::Params none{};
  return launch_gemm<P0, NoProb, kPair>(slot, dev, groups, ta, tb, to, ta, tb, to, a, ep, none, s);
}

// Problem 0 round-robin, problem 1 dealt to even out the groups' total K
// blocks (see joint_plan).
void plan_second_problem(GemmArgs& a, int groups) {
  a.joint = joint_plan(a.prob[0].raster.num_units, unit_cost(a.prob[0]), a.prob[1].raster.num_units,
                       unit_cost(a.prob[1]), groups);
}

// Work groups (CTAs, or CTA pairs) that can be resident at once: one per SM,
// or per pair of SMs that the hardware can co-schedule as a cluster.
int resident_groups(int dev) {
  const int sms = device_sms(dev);
  if (!kPair) return sms;
  if (dev < 0 || dev >= kMaxDevices) return sms / 2;
  if (!g_dev[dev].pair_groups) {
    auto kern = gemm_tc_kernel<Prob<EpiDz, false, false>, NoProb, true>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo<true, true>::SMEM_BYTES);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)sms, 1, 1);
    cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = Geo<true, true>::SMEM_BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = sms / 2;
    }
    g_dev[dev].pair_groups = n < sms / 2 ? n : sms / 2;
  }
  return g_dev[dev].pair_groups;
}

inline int grid_for(const Raster& r, int groups) { return r.num_units < groups ? r.num_units : groups; }

// Operands and their L2 priority: a band of H is re-read for every vocabulary
// tile of its unit (keep it); the H chunk is re-read by every dW tile of the
// chunk (keep it); streamed operands use the default priority.
using ProbFwd = Prob<EpiFwd, false, false, kL2EvictLast, kL2Normal>;  // A = H (K-major), B = W (K-major)
using ProbDz = Prob<EpiDz, false, false, kL2EvictLast, kL2Normal>;    // A = H chunk, B = W
using ProbDh = Prob<EpiDh, false, true, kL2Normal, kL2Normal, true>;   // A = dZ (K-major over V), B = W (MN-major
                                                                        // over d); wide units (K = V is long)
using ProbDw = Prob<EpiDw, true, true, kL2Normal, kL2EvictLast>;      // A = dZ^T (MN-major over V), B = H chunk
using ProbZ32 = Prob<EpiZ32, false, false, kL2EvictLast, kL2Normal>;  // teacher logits, fp32 store: A = Ht, B = Wt
static_assert(kSelTile == BN, "the select's tile maxima are those of the logits GEMM's column tiles");

// The loss as one call computes it: the teacher logits and their type, T,
// and the factors of the student-temperature variant (zs on the student
// logits, T^2 on the term, T on dZ).
struct Variant {
  const void* logit;
  int logit_bf16;
  float T;
  float zscale, tfac, gfac;
  bool skip_rows;       // backward over the tokens with a non-zero dZ row only
};

int make_variant(const kd_topk_kl_options* o, const void* logit, float T, Variant* v) {
  kd_topk_kl_options d{};
  if (o) d = *o;
  if ((d.logit_bf16 | d.student_temperature | d.skip_masked_rows) & ~1) return KD_ERR_INVALID_ARG;
  for (int32_t r : d.reserved)
    if (r) return KD_ERR_INVALID_ARG;
  v->logit = logit;
  v->logit_bf16 = d.logit_bf16;
  v->T = T;
  v->zscale = d.student_temperature ? 1.0f / T : 1.0f;
  v->tfac = d.student_temperature ? T * T : 1.0f;
  v->gfac = d.student_temperature ? T : 1.0f;
  v->skip_rows = d.skip_masked_rows != 0;
  return KD_OK;
}

int common_checks(const void* H, const void* W, const int32_t* idx, const Variant& var,
                  int64_t N, int64_t d, int64_t V, int64_t K, int64_t chunk,
                  void* ws, size_t ws_bytes, Layout* L) {
  int st = check_shapes(N, d, V, K, var.T, chunk);
  if (st != KD_OK) return st;
  if (!W || !ws) return KD_ERR_INVALID_ARG;
  if (N > 0 && (!H || !idx || !var.logit)) return KD_ERR_INVALID_ARG;
  if (!aligned(W, 16) || (H && !aligned(H, 16)) || !aligned(ws, 256)) return KD_ERR_INVALID_ARG;
  if ((idx && !aligned(idx, 4)) || (var.logit && !aligned(var.logit, var.logit_bf16 ? 2 : 4)))
    return KD_ERR_INVALID_ARG;
  *L = make_layout(N, d, V, K, chunk);
  if (ws_bytes < L->total) return KD_ERR_WORKSPACE;
  return KD_OK;
}

template <class T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

// Records events[i] (if given) before the i-th kernel launch of a call and
// events[n] after the last one.
struct LaunchEvents {
  cudaEvent_t* ev;
  int64_t n, next;
  cudaStream_t s;
  bool mark() {
    if (!ev) return true;
    if (next >= n) return false;
    return cudaEventRecord(ev[next++], s) == cudaSuccess;
  }
};


int forward_stage(const void* H, const void* W, const int32_t* topk_idx, const Variant& var,
                  const float* mask, int64_t N, int64_t d, int64_t V, int64_t K,
                  const Layout& L, float* loss, float* lse, void* workspace, cudaStream_t s,
                  LaunchEvents& evs, bool poison = false);

}  // namespace

extern "C" {

const char* kd_status_string(int s) {
  switch (s) {
    case KD_OK: return "KD_OK";
    case KD_ERR_INVALID_ARG: return "KD_ERR_INVALID_ARG";
    case KD_ERR_UNSUPPORTED: return "KD_ERR_UNSUPPORTED";
    case KD_ERR_WORKSPACE: return "KD_ERR_WORKSPACE";
    case KD_ERR_CUDA: return "KD_ERR_CUDA";
    case KD_ERR_BAD_INDEX: return "KD_ERR_BAD_INDEX";
    case KD_ERR_TIMEOUT: return "KD_ERR_TIMEOUT";
    default: return "KD_ERR_UNKNOWN";
  }
}

size_t kd_topk_kl_workspace_size(int64_t N, int64_t d, int64_t V, int64_t K, int64_t chunk) {
  if (check_shapes(N, d, V, K, 1.0f, chunk) != KD_OK) return 0;
  return make_layout(N, d, V, K, chunk).total;
}

int kd_topk_kl_forward(const void* H, const void* W, const int32_t* topk_idx,
                       const float* topk_logit, const float* mask, int64_t N, int64_t d,
                       int64_t V, int64_t K, float T, int64_t chunk, float* loss, float* lse,
                       void* workspace, size_t workspace_bytes, void* stream) {
  return kd_topk_kl_forward_ex(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk, loss, lse,
                               workspace, workspace_bytes, stream, nullptr);
}

int kd_topk_kl_forward_ex(const void* H, const void* W, const int32_t* topk_idx,
                          const void* topk_logit, const float* mask, int64_t N, int64_t d,
                          int64_t V, int64_t K, float T, int64_t chunk, float* loss, float* lse,
                          void* workspace, size_t workspace_bytes, void* stream,
                          const kd_topk_kl_options* options) {
  Variant var;
  int st = make_variant(options, topk_logit, T, &var);
  if (st != KD_OK) return st;
  Layout L;
  st = common_checks(H, W, topk_idx, var, N, d, V, K, chunk, workspace, workspace_bytes, &L);
  if (st != KD_OK) return st;
  if (!loss || (N > 0 && !lse)) return KD_ERR_INVALID_ARG;
  if (mask && !aligned(mask, 4)) return KD_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  LaunchEvents evs{nullptr, 0, 0, s};
  return forward_stage(H, W, topk_idx, var, mask, N, d, V, K, L, loss, lse, workspace, s, evs);
}

}  // extern "C"

namespace {

// Forward pass on a checked workspace layout: clears the status words, then
// teacher prep, the logits/lse GEMM, the lse merge and the loss.  With
// `poison`, a bad teacher index or a timed-out wait seen by the pass makes
// the lse and the loss NaN (for callers that cannot read the status words).
int forward_stage(const void* H, const void* W, const int32_t* topk_idx, const Variant& var,
                  const float* mask, int64_t N, int64_t d, int64_t V, int64_t K,
                  const Layout& L, float* loss, float* lse, void* workspace, cudaStream_t s,
                  LaunchEvents& evs, bool poison) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KD_ERR_CUDA;

  if (cudaMemsetAsync(at<Status>(workspace, L.off_status), 0, sizeof(Status), s) != cudaSuccess)
    return KD_ERR_CUDA;
  if (N == 0) {
    return cudaMemsetAsync(loss, 0, sizeof(float), s) == cudaSuccess ? KD_OK : KD_ERR_CUDA;
  }
  Status* status = at<Status>(workspace, L.off_status);
  int32_t* tidx = at<int32_t>(workspace, L.off_tidx);
  float* tp = at<float>(workspace, L.off_tp);
  float* ent = at<float>(workspace, L.off_ent);
  double* mask_part = at<double>(workspace, L.off_mask_part);
  double* term_part = at<double>(workspace, L.off_term_part);

  if (!evs.mark()) return KD_ERR_CUDA;
  teacher_prep_kernel<<<(unsigned)L.n_prep_blocks, kPrepWarps * 32, 0, s>>>(
      topk_idx, var.logit, var.logit_bf16, mask, (int)N, (int)K, L.Kp, (int)V, var.T, tidx, tp, ent,
      mask_part, status);
  if (cudaGetLastError() != cudaSuccess) return KD_ERR_CUDA;

  CUtensorMap tmH, tmW;
  if (!make_map(&tmH, H, d, N, d, BK, BM) || !make_map(&tmW, W, d, V, d, BK, GeoP::B_ROWS))
    return KD_ERR_CUDA;
  const int groups = resident_groups(dev);
  ProbArgs a{};
  a.raster = forward_raster(ceil_div(N, GeoP::TILE_M), ceil_div(V, BN), groups, GeoP::TILE_M * d * 2,
                            device_l2_bytes(dev));
  a.num_kb = (int)ceil_div(d, BK);
  EpiFwd::Params ep{};
  ep.N = (int)N;
  ep.V = (int)V;
  ep.Kp = L.Kp;
  ep.zl2 = var.zscale * kLog2e;
  ep.tidx = tidx;
  ep.tp = tp;
  ep.part_m = at<float>(workspace, L.off_pm);
  ep.part_s = at<float>(workspace, L.off_ps);
  ep.part_g = at<float>(workspace, L.off_pg);
  // wave pacing counters
  unsigned int* wave_sync = at<unsigned int>(workspace, L.off_wave);
  if (cudaMemsetAsync(wave_sync, 0, sizeof(unsigned int) * (size_t)wave_slots_bound(a.raster.num_units, 0), s) !=
      cudaSuccess)
    return KD_ERR_CUDA;
  if (!evs.mark()) return KD_ERR_CUDA;
  if (launch_one<ProbFwd>(0, dev, grid_for(a.raster, groups), tmH, tmW, tmH, a, status, ep, s, DynRows{},
                          wave_sync) != cudaSuccess)
    return KD_ERR_CUDA;

  if (!evs.mark()) return KD_ERR_CUDA;
  lse_merge_kernel<<<(unsigned)L.n_merge_blocks, kMergeThreads, 0, s>>>(
      ep.part_m, ep.part_s, ep.part_g, a.raster.splits, (int)N, ent, mask, tidx, L.Kp, var.zscale,
      var.tfac, lse, term_part, poison ? status : nullptr);
  if (!evs.mark()) return KD_ERR_CUDA;
  finalize_kernel<<<1, 256, 0, s>>>(mask_part, (int)L.n_prep_blocks, term_part,
                                    (int)L.n_merge_blocks, 0, nullptr, loss, poison ? status : nullptr);
  return cudaGetLastError() == cudaSuccess ? KD_OK : KD_ERR_CUDA;
}


int backward_checks(int64_t N, const float* lse, const float* grad_loss, const float* mask,
                    const void* dH, const float* dW) {
  if (!dW || !aligned(dW, 16)) return KD_ERR_INVALID_ARG;
  if (N > 0 && (!lse || !dH || !aligned(dH, 16))) return KD_ERR_INVALID_ARG;
  if ((mask && !aligned(mask, 4)) || (grad_loss && !aligned(grad_loss, 4))) return KD_ERR_INVALID_ARG;
  return KD_OK;
}

// Backward pass on a checked workspace layout.  With run_prep the status
// words are cleared and the teacher cache is prepared here; without it the
// forward pass of the same call has done both.  Then the gradient scale and,
// per chunk, the dZ recompute and the joint dH / dW launch.
//
// With var.skip_rows the chunks run over the compacted list of tokens whose
// dZ row can be non-zero (mask != 0, teacher entries present), built on the
// device: dH is cleared, and per chunk the kept tokens' H rows are gathered,
// the GEMMs read the live row count from the device (chunks past it do no
// work) and the chunk's dH rows are scattered back.
int backward_stage(const void* H, const void* W, const int32_t* topk_idx, const Variant& var,
                   const float* mask, int64_t N, int64_t d, int64_t V, int64_t K,
                   int64_t chunk, const Layout& L, const float* lse, const float* grad_loss,
                   void* dH, float* dW, int accumulate_dW, void* workspace, cudaStream_t s,
                   bool run_prep, LaunchEvents& evs) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KD_ERR_CUDA;
  if (run_prep && cudaMemsetAsync(at<Status>(workspace, L.off_status), 0, sizeof(Status), s) != cudaSuccess)
    return KD_ERR_CUDA;
  if (N == 0) {
    if (!accumulate_dW && cudaMemsetAsync(dW, 0, sizeof(float) * (size_t)V * d, s) != cudaSuccess)
      return KD_ERR_CUDA;
    return KD_OK;
  }
  Status* status = at<Status>(workspace, L.off_status);
  int32_t* tidx = at<int32_t>(workspace, L.off_tidx);
  float* tp = at<float>(workspace, L.off_tp);
  float* ent = at<float>(workspace, L.off_ent);
  double* mask_part = at<double>(workspace, L.off_mask_part);
  float* cscale = at<float>(workspace, L.off_scal);
  __nv_bfloat16* dz = at<__nv_bfloat16>(workspace, L.off_dz);
  const bool compact = var.skip_rows;
  int32_t* rowmap = at<int32_t>(workspace, L.off_rowmap);
  int* nrows = at<int>(workspace, L.off_nrows);
  __nv_bfloat16* hc = at<__nv_bfloat16>(workspace, L.off_hc);
  __nv_bfloat16* dhc = at<__nv_bfloat16>(workspace, L.off_dhc);

  if (run_prep) {
    if (!evs.mark()) return KD_ERR_CUDA;
    teacher_prep_kernel<<<(unsigned)L.n_prep_blocks, kPrepWarps * 32, 0, s>>>(
        topk_idx, var.logit, var.logit_bf16, mask, (int)N, (int)K, L.Kp, (int)V, var.T, tidx, tp, ent,
        mask_part, status);
  }
  if (!evs.mark()) return KD_ERR_CUDA;
  finalize_kernel<<<1, 256, 0, s>>>(mask_part, (int)L.n_prep_blocks, nullptr, 0, 1, grad_loss, cscale);
  if (cudaGetLastError() != cudaSuccess) return KD_ERR_CUDA;
  if (compact) {
    if (cudaMemsetAsync(dH, 0, sizeof(__nv_bfloat16) * (size_t)N * d, s) != cudaSuccess) return KD_ERR_CUDA;
    if (!evs.mark()) return KD_ERR_CUDA;
    compact_rows_kernel<<<1, kCompactThreads, 0, s>>>(mask, tidx, L.Kp, (int)N, rowmap, nrows);
    if (cudaGetLastError() != cudaSuccess) return KD_ERR_CUDA;
  }

  // H as the recompute's A (K-major) and as the dW GEMM's B (MN-major), and
  // the dH target: the caller's arrays, or one chunk of gathered rows
  const void* hsrc = compact ? static_cast<const void*>(hc) : H;
  void* dhdst = compact ? static_cast<void*>(dhc) : dH;
  const int64_t hrows = compact ? L.C : N;
  CUtensorMap tmHk, tmWk, tmWmn, tmHmn, tmDH, tmDW;
  if (!make_map(&tmHk, hsrc, d, hrows, d, BK, BM) || !make_map(&tmWk, W, d, V, d, BK, GeoP::B_ROWS) ||
      !make_map(&tmWmn, W, d, V, d, 64, BK) || !make_map(&tmHmn, hsrc, d, hrows, d, 64, BK) ||
      !make_map(&tmDH, dhdst, d, hrows, d, 64, BM) || !make_map(&tmDW, dW, d, V, d, 32, BM, true))
    return KD_ERR_CUDA;
  const int groups = resident_groups(dev);
  const unsigned copy_blocks = (unsigned)(device_sms(dev) * 8);
  unsigned int* jwave = at<unsigned int>(workspace, L.off_jwave);
  if (cudaMemsetAsync(jwave, 0, sizeof(unsigned int) * (size_t)L.jwave_per_chunk * ceil_div(N, chunk), s) !=
      cudaSuccess)
    return KD_ERR_CUDA;

  for (int64_t c0 = 0; c0 < N; c0 += chunk) {
    const int64_t Cc = (N - c0 < chunk) ? (N - c0) : chunk;
    // the chunk's dZ: [Cc][ldz] bf16, as the recompute's store target and the
    // dH GEMM's A (box {64, 128}), and as the dW GEMM's A (box {64, 64})
    CUtensorMap tmZk, tmZmn;
    if (!make_map(&tmZk, dz, L.ldz, Cc, L.ldz, BK, BM) || !make_map(&tmZmn, dz, L.ldz, Cc, L.ldz, 64, BK))
      return KD_ERR_CUDA;

    const DynRows dyn = compact ? DynRows{nrows, (int)c0, (int)Cc} : DynRows{};
    const int hrow0 = compact ? 0 : (int)c0;
    if (compact) {
      if (!evs.mark()) return KD_ERR_CUDA;
      gather_rows_kernel<<<copy_blocks, 256, 0, s>>>(static_cast<const uint4*>(H), (int)(d / 8), rowmap, nrows,
                                                    (int)c0, (int)Cc, reinterpret_cast<uint4*>(hc));
      if (cudaGetLastError() != cudaSuccess) return KD_ERR_CUDA;
    }

    // dZ for the chunk: recompute z = H W^T tile by tile.
    // Units are a band and a range of column tiles, so each epilogue thread
    // sets up its token (scale, lse, teacher cursor) once per unit.
    ProbArgs a3{};
    a3.raster = forward_raster(ceil_div(Cc, GeoP::TILE_M), ceil_div(V, BN), groups, 0, 0, kMaxDzSplits);
    a3.num_kb = (int)ceil_div(d, BK);
    a3.a_row0 = hrow0;
    a3.dyn_role = 3;
    EpiDz::Params e3{};
    e3.rowmap = compact ? rowmap : nullptr;
    e3.rows_valid = (int)Cc;
    e3.row0 = (int)c0;
    e3.V = (int)V;
    e3.ldz = (int)L.ldz;
    e3.Kp = L.Kp;
    e3.zl2 = var.zscale * kLog2e;
    e3.gfac = var.gfac;
    e3.tidx = tidx;
    e3.tp = tp;
    e3.lse = lse;
    e3.mask = mask;
    e3.cscale = cscale;
    if (!evs.mark()) return KD_ERR_CUDA;
    if (launch_one<ProbDz>(1, dev, grid_for(a3.raster, groups), tmHk, tmWk, tmZk, a3, status, e3, s, dyn) !=
        cudaSuccess)
      return KD_ERR_CUDA;

    // One launch for both gradient products of the chunk:
    //   problem 0: dH[chunk] = dZ W      (few long tiles, K = V; two column tiles
    //              per unit sharing each dZ load where that keeps the pairs
    //              balanced; a band's units side by side, so each dZ band is
    //              fetched once per wave)
    //   problem 1: dW (+)= dZ^T H[chunk] (many short tiles, K = chunk)
    GemmArgs a45{};
    a45.status = status;
    a45.dyn = dyn;
    const int64_t dh_cols = ceil_div(d, BN), dh_bands = ceil_div(Cc, GeoP::TILE_M);
    const bool wide = wide_pays(dh_bands, dh_cols, ceil_div(V, BK), ceil_div(V, GeoP::TILE_M) * dh_cols,
                                ceil_div(Cc, BK), groups);
    a45.prob[0].raster = tile_raster(dh_bands, wide ? ceil_div(dh_cols, 2) : dh_cols, false);
    a45.prob[0].num_kb = (int)ceil_div(V, BK);
    a45.prob[0].dyn_role = 1;
    a45.prob[0].wide_cols = wide ? (int)dh_cols : 0;
    a45.prob[1].raster = tile_raster(ceil_div(V, GeoP::TILE_M), ceil_div(d, BN), false);
    a45.prob[1].num_kb = (int)ceil_div(Cc, BK);
    a45.prob[1].b_k0 = hrow0;
    a45.prob[1].dyn_role = 2;
    plan_second_problem(a45, groups);
    if (a45.prob[1].num_kb >= (wide ? kPaceKBlocksWide : kPaceKBlocks))   // dW tiles long enough to pace
      a45.wave_sync = jwave + (size_t)(c0 / chunk) * L.jwave_per_chunk;        // (see wave_slot)
    EpiDh::Params e4{};
    e4.row0 = hrow0;
    EpiDw::Params e5{};
    e5.accumulate = (accumulate_dW || c0 > 0) ? 1 : 0;
    a45.prob[1].dyn_zero_fill = e5.accumulate ? 0 : 1;    // dW must be written even with no live row
    if (!evs.mark()) return KD_ERR_CUDA;
    if (launch_gemm<ProbDh, ProbDw, kPair>(2, dev, groups, tmZk, tmWmn, tmDH, tmZmn, tmHmn, tmDW, a45, e4, e5, s) != cudaSuccess)
      return KD_ERR_CUDA;
    if (compact) {
      if (!evs.mark()) return KD_ERR_CUDA;
      scatter_rows_kernel<<<copy_blocks, 256, 0, s>>>(reinterpret_cast<const uint4*>(dhc), (int)(d / 8), rowmap,
                                                     nrows, (int)c0, (int)Cc, static_cast<uint4*>(dH));
      if (cudaGetLastError() != cudaSuccess) return KD_ERR_CUDA;
    }
  }
  return KD_OK;
}

}  // namespace

extern "C" {

int kd_topk_kl_backward(const void* H, const void* W, const int32_t* topk_idx,
                        const float* topk_logit, const float* mask, int64_t N, int64_t d,
                        int64_t V, int64_t K, float T, int64_t chunk, const float* lse,
                        const float* grad_loss, void* dH, float* dW, int accumulate_dW,
                        void* workspace, size_t workspace_bytes, void* stream) {
  return kd_topk_kl_backward_ex(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk, lse,
                                grad_loss, dH, dW, accumulate_dW, workspace, workspace_bytes,
                                stream, nullptr, 0, nullptr);
}

int kd_topk_kl_backward_profiled(const void* H, const void* W, const int32_t* topk_idx,
                                 const float* topk_logit, const float* mask, int64_t N, int64_t d,
                                 int64_t V, int64_t K, float T, int64_t chunk, const float* lse,
                                 const float* grad_loss, void* dH, float* dW, int accumulate_dW,
                                 void* workspace, size_t workspace_bytes, void* stream,
                                 void* const* events, int64_t n_events) {
  return kd_topk_kl_backward_ex(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk, lse,
                                grad_loss, dH, dW, accumulate_dW, workspace, workspace_bytes,
                                stream, events, n_events, nullptr);
}

int kd_topk_kl_backward_ex(const void* H, const void* W, const int32_t* topk_idx,
                           const void* topk_logit, const float* mask, int64_t N, int64_t d,
                           int64_t V, int64_t K, float T, int64_t chunk, const float* lse,
                           const float* grad_loss, void* dH, float* dW, int accumulate_dW,
                           void* workspace, size_t workspace_bytes, void* stream,
                           void* const* events, int64_t n_events,
                           const kd_topk_kl_options* options) {
  Variant var;
  int st = make_variant(options, topk_logit, T, &var);
  if (st != KD_OK) return st;
  Layout L;
  st = common_checks(H, W, topk_idx, var, N, d, V, K, chunk, workspace, workspace_bytes, &L);
  if (st != KD_OK) return st;
  if ((st = backward_checks(N, lse, grad_loss, mask, dH, dW)) != KD_OK) return st;
  const int64_t launches = N > 0 ? (var.skip_rows ? 3 + 4 * ceil_div(N, chunk) : 2 + 2 * ceil_div(N, chunk)) : 0;
  if (events && n_events < launches + 1) return KD_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  LaunchEvents evs{reinterpret_cast<cudaEvent_t*>(const_cast<void**>(events)), n_events, 0, s};
  st = backward_stage(H, W, topk_idx, var, mask, N, d, V, K, chunk, L, lse, grad_loss, dH, dW,
                      accumulate_dW, workspace, s, true, evs);
  if (st == KD_OK && N > 0 && !evs.mark()) return KD_ERR_CUDA;
  return st;
}

int kd_topk_kl_forward_backward(const void* H, const void* W, const int32_t* topk_idx,
                                const float* topk_logit, const float* mask, int64_t N, int64_t d,
                                int64_t V, int64_t K, float T, int64_t chunk, float* loss,
                                float* lse, const float* grad_loss, void* dH, float* dW,
                                int accumulate_dW, void* workspace, size_t workspace_bytes,
                                void* stream, void* const* events, int64_t n_events) {
  return kd_topk_kl_forward_backward_ex(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk, loss,
                                        lse, grad_loss, dH, dW, accumulate_dW, workspace,
                                        workspace_bytes, stream, events, n_events, nullptr);
}

int kd_topk_kl_forward_backward_ex(const void* H, const void* W, const int32_t* topk_idx,
                                   const void* topk_logit, const float* mask, int64_t N,
                                   int64_t d, int64_t V, int64_t K, float T, int64_t chunk,
                                   float* loss, float* lse, const float* grad_loss, void* dH,
                                   float* dW, int accumulate_dW, void* workspace,
                                   size_t workspace_bytes, void* stream, void* const* events,
                                   int64_t n_events, const kd_topk_kl_options* options) {
  Variant var;
  int st = make_variant(options, topk_logit, T, &var);
  if (st != KD_OK) return st;
  Layout L;
  st = common_checks(H, W, topk_idx, var, N, d, V, K, chunk, workspace, workspace_bytes, &L);
  if (st != KD_OK) return st;
  if (!loss || (N > 0 && !lse)) return KD_ERR_INVALID_ARG;
  if ((st = backward_checks(N, lse, grad_loss, mask, dH, dW)) != KD_OK) return st;
  const int64_t launches = N > 0 ? (var.skip_rows ? 6 + 4 * ceil_div(N, chunk) : 5 + 2 * ceil_div(N, chunk)) : 0;
  if (events && n_events < launches + 1) return KD_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  LaunchEvents evs{reinterpret_cast<cudaEvent_t*>(const_cast<void**>(events)), n_events, 0, s};
  st = forward_stage(H, W, topk_idx, var, mask, N, d, V, K, L, loss, lse, workspace, s, evs);
  if (st != KD_OK) return st;
  st = backward_stage(H, W, topk_idx, var, mask, N, d, V, K, chunk, L, lse, grad_loss, dH, dW,
                      accumulate_dW, workspace, s, false, evs);
  if (st == KD_OK && N > 0 && !evs.mark()) return KD_ERR_CUDA;
  return st;
}

int kd_topk_kl_check(const void* workspace, void* stream, int64_t* bad_index_count) {
  if (!workspace) return KD_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return KD_ERR_CUDA;
  Status h;
  if (cudaMemcpy(&h, workspace, sizeof(Status), cudaMemcpyDeviceToHost) != cudaSuccess) return KD_ERR_CUDA;
  if (bad_index_count) *bad_index_count = (int64_t)h.bad_index;
  if (h.timeout) return KD_ERR_TIMEOUT;
  if (h.bad_index) return KD_ERR_BAD_INDEX;
  return KD_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- teacher top-K cache writer
//
// The offline cache the loss consumes: for each position, the K largest
// logits of the teacher head and their indices (blog post, "Two systems
// changes", offline distillation paragraph).  Per chunk of tokens, the
// teacher logits z = Ht Wt^T are computed by the same tcgen05 GEMM as the
// loss (fp32 tiles stored through TMA into a chunk buffer, with the largest
// logit of every row's 256-column tile kept beside them) and each row's top
// K are selected exactly (topk_select_kernel), reading only the tiles whose
// maximum can be among them.

namespace {

// Status words first (as in the loss workspace, so kd_topk_kl_check reads
// them), then one chunk of fp32 logits and the keys of their tile maxima.
struct TopkLayout {
  int64_t C = 0, ldz = 0, tmld = 0;
  size_t off_status = 0, off_z = 0, off_tmax = 0, total = 0;
};

TopkLayout make_topk_layout(int64_t N, int64_t V, int64_t chunk) {
  TopkLayout L;
  L.C = N > 0 ? (chunk < N ? chunk : N) : 1;
  L.ldz = round_up(V, 4);
  L.tmld = ceil_div(V, BN);
  L.off_status = 0;
  L.off_z = align256(sizeof(Status));
  L.off_tmax = L.off_z + align256(sizeof(float) * (size_t)L.C * L.ldz);
  L.total = L.off_tmax + align256(sizeof(uint32_t) * (size_t)L.C * L.tmld);
  return L;
}

int topk_checks(int64_t N, int64_t d, int64_t V, int64_t K, int64_t chunk) {
  if (N < 0 || d <= 0 || V <= 0 || K <= 0 || chunk <= 0) return KD_ERR_INVALID_ARG;
  if (d % 8 != 0 || K > kMaxTopK || K > V) return KD_ERR_UNSUPPORTED;
  if (N >= (int64_t(1) << 31) || V >= (int64_t(1) << 31) || d >= (int64_t(1) << 24)) return KD_ERR_UNSUPPORTED;
  return KD_OK;
}

}  // namespace

extern "C" {

size_t kd_teacher_topk_workspace_size(int64_t N, int64_t d, int64_t V, int64_t K, int64_t chunk) {
  if (topk_checks(N, d, V, K, chunk) != KD_OK) return 0;
  return make_topk_layout(N, V, chunk).total;
}

int kd_teacher_topk(const void* Ht, const void* Wt, int64_t N, int64_t d, int64_t V, int64_t K,
                    int64_t chunk, int32_t* topk_idx, float* topk_logit, void* workspace,
                    size_t workspace_bytes, void* stream) {
  int st = topk_checks(N, d, V, K, chunk);
  if (st != KD_OK) return st;
  if (!Wt || !workspace || (N > 0 && (!Ht || !topk_idx || !topk_logit))) return KD_ERR_INVALID_ARG;
  if (!aligned(Wt, 16) || (Ht && !aligned(Ht, 16)) || !aligned(workspace, 256) ||
      (topk_idx && !aligned(topk_idx, 4)) || (topk_logit && !aligned(topk_logit, 4)))
    return KD_ERR_INVALID_ARG;
  const TopkLayout L = make_topk_layout(N, V, chunk);
  if (workspace_bytes < L.total) return KD_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Status* status = at<Status>(workspace, L.off_status);
  if (cudaMemsetAsync(status, 0, sizeof(Status), s) != cudaSuccess) return KD_ERR_CUDA;
  if (N == 0) return KD_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KD_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KD_ERR_UNSUPPORTED;
  float* zbuf = at<float>(workspace, L.off_z);
  uint32_t* tmax = at<uint32_t>(workspace, L.off_tmax);

  CUtensorMap tmH, tmW;
  if (!make_map(&tmH, Ht, d, N, d, BK, BM) || !make_map(&tmW, Wt, d, V, d, BK, GeoP::B_ROWS)) return KD_ERR_CUDA;
  const int groups = resident_groups(dev);
  for (int64_t c0 = 0; c0 < N; c0 += chunk) {
    const int64_t Cc = (N - c0 < chunk) ? (N - c0) : chunk;
    // fp32 logits of the chunk: [Cc][ldz], columns >= V never written (TMA clips them)
    CUtensorMap tmZ;
    if (!make_map(&tmZ, zbuf, V, Cc, L.ldz, 32, BM, true)) return KD_ERR_CUDA;
    ProbArgs a{};
    a.raster = tile_raster(ceil_div(Cc, GeoP::TILE_M), ceil_div(V, BN), true);
    a.num_kb = (int)ceil_div(d, BK);
    a.a_row0 = (int)c0;
    EpiZ32::Params e{};
    e.tmax = tmax;
    e.ld = (int)L.tmld;
    e.rows = (int)Cc;
    e.V = (int)V;
    if (launch_one<ProbZ32>(3, dev, grid_for(a.raster, groups), tmH, tmW, tmZ, a, status, e, s) != cudaSuccess)
      return KD_ERR_CUDA;
    topk_select_kernel<<<(unsigned)Cc, kSelectThreads, 0, s>>>(zbuf, L.ldz, (int)V, (int)K, (int)c0, topk_idx,
                                                               topk_logit, tmax, (int)L.tmld);
    if (cudaGetLastError() != cudaSuccess) return KD_ERR_CUDA;
  }
  return KD_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- failure-detection self-test
//
// Every pipeline wait in the kernels is bounded: when a barrier phase does not
// complete in time, the waiting thread gives up, the kernel records a timeout
// in the workspace's status words, lets issued copies land and exits, and
// kd_topk_kl_check reports KD_ERR_TIMEOUT.  This kernel exercises that path
// on purpose: it waits on an mbarrier that nothing ever arrives on.

namespace {

__global__ void wait_selftest_kernel(Status* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    const uint32_t b = smem_u32(&bar);
    mbar_init(b, 1);
    fence_barrier_init();
    abort_flag = 0;
    if (!mbar_wait_bounded(b, 0, &abort_flag, limit_ns)) atomicOr(&status->timeout, 1u);
  }
}

}  // namespace

extern "C" int kd_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int64_t limit_us, void* stream) {
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < sizeof(Status)) return KD_ERR_INVALID_ARG;
  if (limit_us < 1 || limit_us > 2000000) return KD_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Status* status = at<Status>(workspace, 0);
  if (cudaMemsetAsync(status, 0, sizeof(Status), s) != cudaSuccess) return KD_ERR_CUDA;
  wait_selftest_kernel<<<1, 32, 0, s>>>(status, (uint64_t)limit_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? KD_OK : KD_ERR_CUDA;
}

// ---------------------------------------------------------------- forward without a workspace
//
// Some callers cannot allocate device memory at the point where they need
// the loss: code running under a runtime that owns every byte of device
// memory (a serving process that reserves HBM up front and hands out only
// fixed buffers), plug-ins called while their host framework holds its
// allocator lock, and latency-critical loops for which cudaMalloc's implicit
// synchronisation is not acceptable.  For them the forward pass can run on a
// fixed scratch array that lives in this library's own device image.
//
// The array is kNoAllocScratchBytes (16 MiB) on every device that loads the
// library and stays allocated until the process exits.  It holds the
// forward pass's own regions only (make_forward_layout: about
// 8 round_up(K + 1, 4) + 199 bytes per token).  In host code the symbol is
// only a host-side stand-in, so its device address is looked up with
// cudaGetSymbolAddress once per device, on that device's first call, and
// kept (an atomic per device, so concurrent first calls from several host
// threads are benign).  Such a kept address belongs to the device's context
// of that time: it does not survive cudaDeviceReset.

namespace {
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
std::atomic<void*> g_noalloc_scratch_ptr[kMaxDevices];
}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

extern "C" int kd_topk_kl_forward_noalloc(const void* H, const void* W, const int32_t* topk_idx,
                                          const float* topk_logit, const float* mask, int64_t N,
                                          int64_t d, int64_t V, int64_t K, float T, float* loss,
                                          float* lse, void* stream) {
  int st = check_shapes(N, d, V, K, T, 1);
  if (st != KD_OK) return st;
  if (!W || !loss || (N > 0 && (!H || !topk_idx || !topk_logit || !lse))) return KD_ERR_INVALID_ARG;
  if (!aligned(W, 16) || (H && !aligned(H, 16)) || (topk_idx && !aligned(topk_idx, 4)) ||
      (topk_logit && !aligned(topk_logit, 4)) || (mask && !aligned(mask, 4)))
    return KD_ERR_INVALID_ARG;
  const Layout L = make_forward_layout(N, K);
  if (L.total > kNoAllocScratchBytes) return KD_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KD_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KD_ERR_UNSUPPORTED;
  void* scratch = g_noalloc_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!scratch) {
    if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || scratch == nullptr)
      return KD_ERR_CUDA;
    g_noalloc_scratch_ptr[dev].store(scratch, std::memory_order_release);
  }
  // Every word the pass reads from the scratch is written earlier in the
  // same call (the status words are cleared at its start), so nothing left
  // over from a previous call is used.  The status words cannot be read by
  // the caller here, so a bad teacher index or a timed-out wait turns the
  // loss and every lse into NaN instead.
  Variant var;
  if ((st = make_variant(nullptr, topk_logit, T, &var)) != KD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  LaunchEvents evs{nullptr, 0, 0, s};
  return forward_stage(H, W, topk_idx, var, mask, N, d, V, K, L, loss, lse, scratch, s, evs, true);
}
