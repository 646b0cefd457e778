/*
 * kd_topk_kl.h - C ABI of the fused chunked top-K KL distillation loss
 * (libkdtopkl.so, CUDA sm_100a).
 *
 * The operation is the one of "Efficient Knowledge Distillation for LLMs:
 * Offline Top-K Logits and a Fused Chunked KL Loss": the student is trained
 * against an offline cache of the teacher's top-K logits per position
 * (blog post, "Two systems changes", offline distillation paragraph) with a
 * KL loss whose output projection is fused into the loss and recomputed per
 * chunk in the backward pass, so that the N x V logit grid is never stored
 * and peak memory is linear in the number of tokens (Japanese summary,
 * method paragraph: the fused chunked variant; abstract).
 *
 * For student hidden states H[N,d], LM-head weight W[V,d], teacher cache
 * (idx[N,K], logit[N,K]), mask m[N], temperature T:
 *   z[n,v]  = sum_j H[n,j] W[v,j]
 *   lse[n]  = log sum_v exp(z[n,v])
 *   p[n,k]  = softmax_k(logit[n,k] / T)
 *   term[n] = sum_k p[n,k] (log p[n,k] - (z[n,idx[n,k]] - lse[n]))
 *   loss    = sum_n m[n] term[n] / sum_n m[n]        (0 when sum m = 0)
 * and, for an upstream scalar g,
 *   dZ[n,v] = g m[n] / sum m * (exp(z[n,v] - lse[n]) - sum_{k: idx[n,k]=v} p[n,k])
 *   dH      = dZ W            dW (+)= dZ^T H
 * T divides the teacher logits only.  Duplicate teacher indices add their
 * probabilities at that column (the loss keeps the per-slot sum).
 *
 * A teacher index of -1 marks an empty cache slot (a cache that holds fewer
 * than K entries for some tokens): the slot takes no part in the teacher
 * softmax, so p is renormalised over the filled slots.  A token without a
 * filled slot (or whose filled logits are all -inf) has an empty teacher
 * distribution: term = 0 and a zero dZ row (d term / dz = P softmax(z) -
 * scatter(p) with P = sum_k p = 0); its mask still counts in sum m.
 *
 * Variants selected through kd_topk_kl_options (the *_ex entry points; the
 * pages describe none of them; skip_masked_rows changes only the work done):
 *  - logit_bf16: topk_logit holds bf16 values instead of fp32.
 *  - student_temperature: the usual distillation temperature on both sides:
 *      lse[n]  = log sum_v exp(z[n,v] / T)
 *      term[n] = T^2 sum_k p (log p - (z[n,idx]/T - lse[n]))
 *      dZ[n,v] = g m[n] / sum m * T (exp(z[n,v]/T - lse[n]) - scatter(p))
 *    lse is then that of z / T, and the backward pass must be given it.
 *
 * Conventions shared by every entry point:
 *  - All array pointers are DEVICE pointers owned by the caller.  No call
 *    allocates device or host memory.  The library keeps no state between
 *    calls except a per-device, per-kernel attribute cache and, for
 *    kd_topk_kl_forward_noalloc only, a fixed scratch array in its own
 *    device image.
 *  - Layouts are dense row-major: H bf16 [N][d], W bf16 [V][d],
 *    topk_idx int32 [N][K], topk_logit fp32 [N][K], mask fp32 [N],
 *    lse fp32 [N], dH bf16 [N][d], dW fp32 [V][d].  bf16 is IEEE bfloat16
 *    stored as uint16.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls
 *    enqueue work and return without synchronising.  Argument errors are
 *    reported synchronously by the return value and nothing is enqueued.
 *  - Supported shapes: N >= 0, 1 <= V < 2^31, d >= 8 with d % 8 == 0,
 *    1 <= K <= 512, T > 0 and finite, chunk >= 1.  H, W, dH and dW must be
 *    16-byte aligned, the workspace 256-byte aligned.
 *  - Teacher indices outside [0, V) other than -1 are not an argument
 *    error: they are dropped (contribute nothing), counted in the workspace
 *    and reported by kd_topk_kl_check as KD_ERR_BAD_INDEX; the results are
 *    then undefined in value but every memory access stays in bounds.
 *  - Results are deterministic: the same inputs give bitwise the same
 *    outputs on every run (fixed-order reductions, no float atomics).
 *  - A workspace may be used by one call at a time (calls on one stream
 *    are serialised; calls on different streams need different workspaces).
 */
#ifndef KD_TOPK_KL_H
#define KD_TOPK_KL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kd_status {
  KD_OK = 0,
  KD_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad alignment, T <= 0 */
  KD_ERR_UNSUPPORTED = 2,  /* shape outside the supported set (d % 8, K > 512, ...) */
  KD_ERR_WORKSPACE = 3,    /* workspace_bytes smaller than kd_topk_kl_workspace_size */
  KD_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
  KD_ERR_BAD_INDEX = 5,    /* (from kd_topk_kl_check) a teacher index was outside [0, V) */
  KD_ERR_TIMEOUT = 6       /* (from kd_topk_kl_check) a pipeline wait gave up; results invalid */
} kd_status;

/* Every entry point returns one of the kd_status values above as a plain
 * int, not as the enum type: an enum's size is up to the compiler (C allows
 * a smaller type; -fshort-enums picks one), whereas int is 32 bits for every
 * caller that binds this library, C or a foreign-function interface. */

/* Human-readable name of a status code.  Never returns NULL. */
const char* kd_status_string(int status);

/* Bytes of device workspace that kd_topk_kl_forward / kd_topk_kl_backward
 * need for these sizes (the same workspace size serves both).  Returns 0
 * for sizes that the entry points would reject.  It holds the prepared
 * teacher cache (sorted indices and probabilities, N x (K+1..K+4) x 8 B),
 * per-token partial log-sum-exp state, one chunk of dZ
 * (chunk x round_up(V, 8) bf16), and for skip_masked_rows a token list
 * (4 B per token) and two chunk x d bf16 row buffers: linear in N, and in
 * chunk x V. */
size_t kd_topk_kl_workspace_size(int64_t N, int64_t d, int64_t V, int64_t K, int64_t chunk);

/* Forward pass.  Writes *loss (device fp32 scalar) and lse[N] (device fp32;
 * every token's student log-sum-exp, masked tokens included), which the
 * backward pass consumes.  mask may be NULL (all ones).  The logit grid is
 * never stored: each vocabulary tile of z = H W^T lives only in tensor
 * memory while its running max / sum-exp and the teacher gather are updated
 * (Japanese summary, method paragraph: fused chunked KL). */
int kd_topk_kl_forward(const void* H, const void* W,
                       const int32_t* topk_idx, const float* topk_logit,
                       const float* mask,
                       int64_t N, int64_t d, int64_t V, int64_t K, float T, int64_t chunk,
                       float* loss, float* lse,
                       void* workspace, size_t workspace_bytes, void* stream);

/* Backward pass.  Recomputes z chunk by chunk (chunk tokens at a time; the
 * pages' "recompute each chunk during the backward pass", Japanese
 * summary, method paragraph), forms dZ for that chunk only, and writes
 * dH (bf16 [N][d], overwritten) and dW (fp32 [V][d]; overwritten when
 * accumulate_dW == 0, added to when accumulate_dW != 0).  lse must be the
 * forward pass's output for the same inputs.  grad_loss is a device fp32
 * scalar (the upstream gradient of the loss) or NULL for 1.0.  dZ is
 * rounded to bf16 before the two gradient products. */
int kd_topk_kl_backward(const void* H, const void* W,
                        const int32_t* topk_idx, const float* topk_logit,
                        const float* mask,
                        int64_t N, int64_t d, int64_t V, int64_t K, float T, int64_t chunk,
                        const float* lse, const float* grad_loss,
                        void* dH, float* dW, int accumulate_dW,
                        void* workspace, size_t workspace_bytes, void* stream);

/* Same as kd_topk_kl_backward, and also records CUDA events on `stream`
 * around every kernel launch, for timing the pass's kernels live without a
 * profiler.  events[i] (a cudaEvent_t created by the caller) is recorded
 * just before the i-th launch and events[n] after the last, n being the
 * number of launches: 2 + 2 * ceil(N / chunk) for N > 0 (teacher prep,
 * gradient scale, then per chunk the logit recompute into dZ and the joint
 * dH / dW launch), 0 for N = 0.  n_events must be at least n + 1, else
 * KD_ERR_INVALID_ARG and nothing is enqueued. */
int kd_topk_kl_backward_profiled(const void* H, const void* W,
                                 const int32_t* topk_idx, const float* topk_logit,
                                 const float* mask,
                                 int64_t N, int64_t d, int64_t V, int64_t K, float T, int64_t chunk,
                                 const float* lse, const float* grad_loss,
                                 void* dH, float* dW, int accumulate_dW,
                                 void* workspace, size_t workspace_bytes, void* stream,
                                 void* const* events, int64_t n_events);

/* Forward and backward pass in one call, for a training step whose loss is
 * this one: writes *loss and lse[N] as kd_topk_kl_forward, then dH and dW as
 * kd_topk_kl_backward (grad_loss as there; NULL for 1.0).  The teacher cache
 * is prepared once for both passes.  events may be NULL; otherwise it holds
 * cudaEvent_t handles recorded on `stream` before each kernel launch and
 * after the last: n = 5 + 2 * ceil(N / chunk) launches for N > 0 (teacher
 * prep, logits/lse GEMM, lse merge, loss, gradient scale, then per chunk the
 * dZ recompute and the joint dH / dW launch), n_events >= n + 1. */
int kd_topk_kl_forward_backward(const void* H, const void* W,
                                const int32_t* topk_idx, const float* topk_logit,
                                const float* mask,
                                int64_t N, int64_t d, int64_t V, int64_t K, float T, int64_t chunk,
                                float* loss, float* lse, const float* grad_loss,
                                void* dH, float* dW, int accumulate_dW,
                                void* workspace, size_t workspace_bytes, void* stream,
                                void* const* events, int64_t n_events);

/* Forward pass for callers that cannot allocate device memory.  The paper
 * has no counterpart to this entry point; it exists for callers such as a
 * runtime that owns all device memory and hands out only fixed buffers, a
 * plug-in called while its host framework holds its allocator lock, or a
 * latency-critical loop that cannot afford cudaMalloc's implicit
 * synchronisation.
 *
 * Same inputs and outputs as kd_topk_kl_forward (fp32 logits, no options,
 * no chunk, no workspace).  Instead of a caller workspace it uses a 16 MiB
 * scratch array compiled into the library: every device that loads the
 * library holds those 16 MiB until the process exits.  It allocates nothing
 * itself (no cudaMalloc, no cudaFree, no allocating library call).
 *  - Size limit: the scratch holds the forward pass's own state only, about
 *    8 * round_up(K + 1, 4) + 199 bytes per token plus under 4 KiB.  Sizes
 *    with (8 * round_up(K + 1, 4) + 199) * N + 4096 <= 16 MiB are accepted
 *    (N <= 16,268 at K = 100, 46,721 at K = 16), any d and V; sizes with
 *    (8 * round_up(K + 1, 4) + 198) * N > 16 MiB return KD_ERR_WORKSPACE
 *    and enqueue nothing.
 *  - The first call on each device looks up the scratch array's device
 *    address (cudaGetSymbolAddress) with that device current and keeps it
 *    for later calls; make that first call before any stream capture
 *    begins.  The kept address belongs to the device's context at that
 *    time and does not survive cudaDeviceReset.
 *  - All calls share the one array and it keeps the last call's contents;
 *    the pass clears its status words and overwrites everything else it
 *    reads before reading it.  Calls that overlap on the GPU (different
 *    streams, or different host threads) race on the array and must not be
 *    issued.
 *  - The device-side status words cannot be read by the caller of this
 *    entry point (kd_topk_kl_check takes a workspace).  Instead, when the
 *    pass meets a teacher index outside [0, V) or a pipeline wait times
 *    out, it writes NaN to *loss and to every lse[n]. */
int kd_topk_kl_forward_noalloc(const void* H, const void* W,
                               const int32_t* topk_idx, const float* topk_logit,
                               const float* mask,
                               int64_t N, int64_t d, int64_t V, int64_t K, float T,
                               float* loss, float* lse, void* stream);

/* Options of the *_ex entry points.  A NULL pointer, or a zero-filled
 * struct, selects the definition above (fp32 logits, T on the teacher
 * only).  Every field is 0 or 1; reserved fields must be 0, else
 * KD_ERR_INVALID_ARG. */
typedef struct kd_topk_kl_options {
  int32_t logit_bf16;           /* 1: topk_logit is bf16 [N][K] (2-byte aligned) */
  int32_t student_temperature;  /* 1: student logits divided by T too, term times T^2 */
  int32_t skip_masked_rows;     /* 1: the backward pass works on the tokens whose dZ row can be
                                   non-zero only (mask != 0 and teacher entries present): they are
                                   listed on the device and processed chunk by chunk, rows of the
                                   others are skipped (their dH rows are written as 0).  Same
                                   results except for the fp32 summation order of dW.  Launches
                                   (for events): backward 3 + 4 * ceil(N / chunk), fused
                                   6 + 4 * ceil(N / chunk) (a compaction kernel, and per chunk a
                                   row gather and a dH row scatter around the two GEMMs). */
  int32_t reserved[5];
} kd_topk_kl_options;

/* kd_topk_kl_forward with options; topk_logit is fp32 or bf16 as
 * options->logit_bf16 says. */
int kd_topk_kl_forward_ex(const void* H, const void* W,
                          const int32_t* topk_idx, const void* topk_logit,
                          const float* mask,
                          int64_t N, int64_t d, int64_t V, int64_t K, float T, int64_t chunk,
                          float* loss, float* lse,
                          void* workspace, size_t workspace_bytes, void* stream,
                          const kd_topk_kl_options* options);

/* kd_topk_kl_backward_profiled with options (events may be NULL).  With
 * student_temperature, lse must come from a forward pass with the same
 * options. */
int kd_topk_kl_backward_ex(const void* H, const void* W,
                           const int32_t* topk_idx, const void* topk_logit,
                           const float* mask,
                           int64_t N, int64_t d, int64_t V, int64_t K, float T, int64_t chunk,
                           const float* lse, const float* grad_loss,
                           void* dH, float* dW, int accumulate_dW,
                           void* workspace, size_t workspace_bytes, void* stream,
                           void* const* events, int64_t n_events,
                           const kd_topk_kl_options* options);

/* kd_topk_kl_forward_backward with options. */
int kd_topk_kl_forward_backward_ex(const void* H, const void* W,
                                   const int32_t* topk_idx, const void* topk_logit,
                                   const float* mask,
                                   int64_t N, int64_t d, int64_t V, int64_t K, float T,
                                   int64_t chunk, float* loss, float* lse, const float* grad_loss,
                                   void* dH, float* dW, int accumulate_dW,
                                   void* workspace, size_t workspace_bytes, void* stream,
                                   void* const* events, int64_t n_events,
                                   const kd_topk_kl_options* options);

/* Teacher top-K cache writer: the offline cache that the loss consumes (blog
 * post, "Two systems changes", offline distillation paragraph: the teacher's
 * top-K logits stored per position).  For teacher hidden states Ht bf16
 * [N][d] and teacher head Wt bf16 [V][d] it writes, per token, the K largest
 * logits z = Ht Wt^T (fp32 accumulation of the bf16 products) and their
 * column indices, largest first, equal logits in increasing column order:
 * topk_idx int32 [N][K], topk_logit fp32 [N][K] (device, caller-owned).
 * Tokens are processed `chunk` at a time: the logits of one chunk are stored
 * in the workspace (chunk x round_up(V, 4) fp32, and per row the largest
 * logit of each 256-column tile) and each row's top K is selected exactly,
 * reading only the tiles whose maximum reaches the K-th largest tile
 * maximum when the row has at least K tiles.  Supported: 1 <= K <= min(V, 512), d % 8 == 0; Ht and Wt
 * 16-byte aligned, the workspace 256-byte aligned.  kd_topk_kl_check on this
 * workspace reports a pipeline timeout. */
size_t kd_teacher_topk_workspace_size(int64_t N, int64_t d, int64_t V, int64_t K, int64_t chunk);
int kd_teacher_topk(const void* Ht, const void* Wt, int64_t N, int64_t d, int64_t V, int64_t K,
                    int64_t chunk, int32_t* topk_idx, float* topk_logit,
                    void* workspace, size_t workspace_bytes, void* stream);

/* Failure-detection self-test.  Every pipeline wait in the kernels is
 * bounded: a barrier phase that does not complete within its limit makes the
 * waiting kernel record a timeout in the workspace's status words and exit,
 * and kd_topk_kl_check then returns KD_ERR_TIMEOUT; the device stays usable.
 * This call exercises that path: it clears the status words and launches a
 * kernel that waits on a barrier nothing ever arrives on, with a limit of
 * limit_us microseconds (1 .. 2,000,000).  Any workspace of this library
 * (>= 256 bytes, 256-byte aligned) will do; the next call on it clears the
 * status again. */
int kd_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int64_t limit_us, void* stream);

/* Synchronises `stream`, then reads the device-side status words that the
 * last forward or backward call on this workspace wrote.  Returns KD_OK,
 * KD_ERR_BAD_INDEX (teacher index outside [0, V) seen), KD_ERR_TIMEOUT (a
 * bounded pipeline wait expired), or KD_ERR_CUDA.  If bad_index_count is
 * not NULL it receives the number of out-of-range teacher indices. */
int kd_topk_kl_check(const void* workspace, void* stream, int64_t* bad_index_count);

#ifdef __cplusplus
}
#endif

#endif /* KD_TOPK_KL_H */
