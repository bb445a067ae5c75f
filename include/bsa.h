/*
 * bsa.h -- C ABI of libbsa.so: block-sparse video self-attention forward on
 * NVIDIA B200 (sm_100a).
 *
 * The method (sources are web pages, cited by title and section):
 *   "h3-sparse-attn 0.1.0" (PyPI project page), opening description: each
 *   query block of 128 tokens attends to its top-k key blocks; the skipped
 *   key blocks are folded back in as one summary row each.  Section "Use":
 *   top_k counts 128-token key blocks.
 *   "Spark-H3: Block Sparse Attention Speeds Up MiniMax-H3 in ComfyUI",
 *   section "What Spark-Attn changes": exact branch + compressed branch; the
 *   Spark-Reweight bullet: weighted summaries plus a log-mass bias, with the
 *   mean of the video queries as one anchor per head.
 *   "H3 Sparse Attention" (comfy.icu WAS node and video_budget node): prompt /
 *   text rows are read exactly and stay dense (the optional dense prefix).
 *
 * Conventions shared by every entry point
 *   - Q, K, V, O are bf16 [B, H, N, D] contiguous (row-major, D fastest),
 *     D == 128.  Their base addresses must be 16-byte aligned (the kernels
 *     stage them with TMA), otherwise BSA_ERR_ALIGN.
 *   - Block size 128; nb = ceil(N / 128); the last block may be ragged.
 *     pb = prefix / 128 dense-prefix blocks, nbv = nb - pb video blocks,
 *     k_eff = min(top_k, nbv).
 *   - Every pointer argument is a DEVICE pointer owned by the caller, except
 *     in bsa_forward_host, whose h* arguments are HOST pointers.  The library
 *     allocates no memory and keeps no per-call state.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous on that stream: a return of BSA_OK
 *     means the arguments were valid and the kernels were enqueued without a
 *     launch error; device-side completion is observed by synchronising.
 *   - On any error nothing is enqueued (argument checks run before the first
 *     launch) except BSA_ERR_CUDA, which reports cudaGetLastError() after a
 *     launch.
 *   - The library is thread-safe for concurrent calls on different streams;
 *     calls on one stream are ordered by that stream.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID = 1,     /* bad size, range, variant or null pointer   */
  BSA_ERR_ALIGN = 2,       /* a pointer is not 16-byte aligned           */
  BSA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed       */
  BSA_ERR_TIMEOUT = 4,     /* written to *dev_status by a kernel whose
                              bounded wait expired (never returned)      */
  BSA_ERR_UNSUPPORTED = 5, /* device is not sm_100 / driver lacks TMA    */
  BSA_ERR_SCRATCH = 6      /* bsa_forward_noalloc: the problem needs more
                              workspace than its static scratch holds    */
} bsa_status;

typedef enum {
  BSA_SUMMARY_ANCHOR = 0,  /* Spark-Reweight: softmax-at-the-anchor weighted
                              k~, v~; bias = ln n + (LSE - ln n - qbar.k~/sqrt d) */
  BSA_SUMMARY_MEAN = 1     /* mean-pooled k~, v~; bias = ln n            */
} bsa_variant;

typedef struct {
  int32_t B, H, N, D;   /* D must be 128; B, H >= 1; 1 <= N <= 2^21          */
  int32_t top_k;        /* >= 1; clamped to nbv                              */
  int32_t prefix;       /* dense-prefix tokens: multiple of 128, 0 <= prefix < N */
  int32_t variant;      /* bsa_variant                                       */
  int32_t* dev_status;  /* optional device int (may be NULL).  Kernels with
                           bounded waits write BSA_ERR_TIMEOUT there if a wait
                           expires (~2 s); the caller zeroes it beforehand.  */
} bsa_params;

/* ---- sizes ------------------------------------------------------------ */

/* nb = ceil(N / 128), or -1 if p is invalid. */
int32_t bsa_num_blocks(const bsa_params* p);

/* kcap: row length of the idx array written by bsa_select,
 * = nb if prefix > 0 (prefix query rows list every block), else pb + k_eff.
 * Returns -1 if p is invalid. */
int32_t bsa_select_capacity(const bsa_params* p);

/* Bytes of the workspace bsa_forward / bsa_forward_host need (256-byte
 * aligned sub-buffers: qpool, anchor, kpool, ksum, vsum, bias, idx, cnt).
 * Returns 0 if p is invalid. */
size_t bsa_workspace_bytes(const bsa_params* p);

/* ---- the four stages -------------------------------------------------- */

/* Step 1-2 (pool + anchor).  Per (b, h): qpool[i] = mean of the real query
 * rows of block i (fp32 [B,H,nb,D]); anchor = mean of the video query rows
 * t >= prefix (fp32 [B,H,D]) -- "the mean of the video queries as one anchor
 * per head" (Spark-H3 page, Spark-Reweight bullet).  Reads Q once.
 * Deterministic (fixed reduction order). */
int bsa_pool(const bsa_params* p, const void* Q, float* qpool, float* anchor,
             void* stream);

/* Step 1 + 3 (key pooling and one summary row per key block), fused so K and
 * V are each read once.  Outputs, all [B,H,nb,...]:
 *   kpool fp32 [.., D]  mean of the real keys of block j;
 *   ksum  bf16 [.., D]  k~_j;   vsum bf16 [.., D]  v~_j;   bias fp32 [..]  bias_j.
 * ANCHOR variant: x_t = anchor . k_t / sqrt(D), w = softmax_t(x) over the
 * block, k~ = sum w k, v~ = sum w v, bias = LSE(x) - anchor . bf16(k~) / sqrt(D)
 * (the ln n_j terms of ln n + (LSE - ln n - ..) cancel; bf16(k~) is the value
 * the attention MMA later uses).  MEAN variant: k~ = mean k, v~ = mean v,
 * bias = ln n_j; `anchor` may then be NULL.  Summaries of prefix blocks are
 * computed but never used. */
int bsa_summarize(const bsa_params* p, const void* K, const void* V,
                  const float* anchor, float* kpool, void* ksum, void* vsum,
                  float* bias, void* stream);

/* Step 4-5 (block score + top-k).  S_ij = qpool_i . kpool_j / sqrt(D) in fp32
 * for video key blocks j >= pb.  Video query block i >= pb keeps the k_eff
 * largest S_ij, ties to the lower j, and writes
 *   idx[b,h,i,:] = 0..pb-1 followed by the chosen j ascending, then -1 padding
 *   (int32 [B,H,nb,kcap]),  cnt[b,h,i] = pb + k_eff  (int32 [B,H,nb]).
 * Prefix query block i < pb lists every block: idx = 0..nb-1, cnt = nb.
 * Deterministic. */
int bsa_select(const bsa_params* p, const float* qpool, const float* kpool,
               int32_t* idx, int32_t* cnt, void* stream);

/* Step 6 (exact branch + compressed branch + epilogue).  For query row t of
 * block i: logits q_t.k_u/sqrt(D) for the tokens u of the blocks idx[b,h,i,
 * 0..cnt) (ragged tail masked) and, for a video query block, q_t.k~_j/sqrt(D)
 * + bias_j for every video block j not listed; O_t = softmax(logits) @ [V ; v~]
 * written as bf16.  lse (fp32 [B,H,N], natural log) is written when non-NULL.
 * tcgen05 MMA (bf16 in, fp32 accumulate in TMEM), online softmax in fp32.
 * idx/cnt must be what bsa_select wrote for the same parameters. */
int bsa_attend(const bsa_params* p, const void* Q, const void* K, const void* V,
               const int32_t* idx, const int32_t* cnt, const void* ksum,
               const void* vsum, const float* bias, void* O, float* lse,
               void* stream);

/* ---- whole path ------------------------------------------------------- */

/* bsa_pool, bsa_summarize, bsa_select, bsa_attend in order on `stream`.
 * `workspace` is a caller-owned device buffer of at least
 * bsa_workspace_bytes(p) bytes, 256-byte aligned. */
int bsa_forward(const bsa_params* p, const void* Q, const void* K, const void* V,
                void* O, float* lse, void* workspace, size_t workspace_bytes,
                void* stream);

/* bsa_forward from HOST buffers.  hQ, hK, hV (bf16 [B,H,N,D]) are copied to
 * the caller's device buffers dQ, dK, dV, the forward runs, and dO is copied
 * back to hO (and dlse to hlse when both are non-NULL).  The work is
 * pipelined over up to 16 chunks of (b, h) slices: the host->device copies
 * (one cudaMemcpyAsync per tensor and chunk) run on a helper stream, the
 * forward of each chunk on `stream`, the copies back on a second helper
 * stream, ordered by events, so copies overlap compute and each other.
 * Host buffers must be pinned for the copies to be asynchronous.  The helper
 * streams / events are created per call and released once their work is
 * done; `stream` waits for the last copy, so synchronising `stream` covers
 * the whole call.  Returns after enqueueing.  On BSA_ERR_CUDA part of the
 * work may already be enqueued. */
int bsa_forward_host(const bsa_params* p, const void* hQ, const void* hK,
                     const void* hV, void* hO, float* hlse, void* dQ, void* dK,
                     void* dV, void* dO, float* dlse, void* workspace,
                     size_t workspace_bytes, void* stream);

/* The same host-buffer pipeline for the options: the FP8 forward
 * (bsa_forward_fp8, workspace bsa_forward_fp8_workspace_bytes), threshold
 * selection (bsa_forward_threshold, workspace
 * bsa_forward_threshold_workspace_bytes), extra tokens (bsa_forward_extra,
 * workspace bsa_forward_extra_workspace_bytes) and adaptive reblocking
 * (bsa_forward_reblock, workspace bsa_forward_reblock_workspace_bytes), each
 * chunk's forward being the option's own forward on a sub-call of its
 * slices (up to 8 chunks for extra tokens, whose token selection needs many
 * heads per launch to fill the GPU).  Arguments, streams and error behaviour
 * as bsa_forward_host. */
int bsa_forward_fp8_host(const bsa_params* p, const void* hQ, const void* hK, const void* hV,
                         void* hO, float* hlse, void* dQ, void* dK, void* dV, void* dO,
                         float* dlse, void* workspace, size_t workspace_bytes, void* stream);
int bsa_forward_threshold_host(const bsa_params* p, float tau, const void* hQ, const void* hK,
                               const void* hV, void* hO, float* hlse, void* dQ, void* dK,
                               void* dV, void* dO, float* dlse, void* workspace,
                               size_t workspace_bytes, void* stream);
int bsa_forward_extra_host(const bsa_params* p, int32_t n_extra, const void* hQ, const void* hK,
                           const void* hV, void* hO, float* hlse, void* dQ, void* dK, void* dV,
                           void* dO, float* dlse, void* workspace, size_t workspace_bytes,
                           void* stream);
int bsa_forward_reblock_host(const bsa_params* p, const void* hQ, const void* hK,
                             const void* hV, void* hO, float* hlse, void* dQ, void* dK, void* dV,
                             void* dO, float* dlse, void* workspace, size_t workspace_bytes,
                             void* stream);

/* ---- forward without any allocation ---------------------------------- */

/* Size of the static device scratch behind bsa_forward_noalloc: 64 MiB. */
#define BSA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/* bsa_forward for callers that cannot allocate device memory.  The pages
 * describe nothing like it (it has no counterpart there); it exists for hosts
 * where cudaMalloc is not an option: a plugin inside a framework whose memory
 * pool owns the device, a server that reserves all memory at start-up and
 * treats later allocations as faults, or latency-critical code that cannot
 * take cudaMalloc's implicit device synchronisation.
 *
 * Same arguments and results as bsa_forward, minus the workspace: the
 * intermediates live in a file-scope static device array of
 * BSA_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library holds
 * until the process exits.  The call allocates nothing (no cudaMalloc,
 * cudaFree or allocating library routine); the caller still passes Q, K, V,
 * O and the optional lse.
 *   - Problems whose bsa_workspace_bytes(p) exceeds the scratch size are
 *     rejected with BSA_ERR_SCRATCH before anything is enqueued (64 MiB covers
 *     e.g. B=1, H=56, N=73,416, top_k=64).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is kept for the life of the
 *     process: calling on a device after cudaDeviceReset, or from a driver
 *     context other than the device's primary context, is not supported
 *     (the array may then live at another address).
 *   - All calls share the one array per device and it keeps the last call's
 *     contents.  No part of it needs to start at zero (every stage fully
 *     writes what the next stage reads), but calls that overlap on the GPU
 *     (e.g. on two streams without ordering) race on it: order them. */
int bsa_forward_noalloc(const bsa_params* p, const void* Q, const void* K, const void* V,
                        void* O, float* lse, void* stream);

/* ---- adaptive reblocking (Spark-Reblock) ------------------------------ */

/* Spark-H3 page, section "What Spark-Attn changes", Spark-Reblock bullet:
 * the fixed token blocks are replaced by an adaptive partition in which two
 * queries are similar when their score patterns over the keys are similar (a
 * Mahalanobis cosine induced by the keys' second moment); a hierarchical
 * partitioner splits groups down to one block, in O(N log N).  Section
 * "Workflows": keys reuse the query layout (q_reuse_k).  This library's
 * reading:
 *   M = sum_{t >= prefix} k_t k_t^T, L L^T = M + 1e-6 * trace(M) / 128 * I,
 *   u_t = L^T q_t / |L^T q_t| (u . u' = cosine of the two score vectors);
 *   a group of n tokens with b = ceil(n/128) >= 2 blocks is bisected along
 *   its principal axis (8 power iterations of the centred scatter of u from
 *   the all-ones direction): the floor(b/2) * 128 tokens of smallest
 *   projection go left (ties to the lower original index);
 *   leaves left to right, ascending inside a leaf; prefix rows stay put.
 * The GPU stores u in bf16, so tokens within ~2^-9 of a split's threshold may
 * land on either side of it. */

/* Scratch of bsa_reblock (device, caller-owned, 256-byte aligned). */
size_t bsa_reblock_workspace_bytes(const bsa_params* p);

/* perm (int32 [B,H,N], caller-owned): perm[b,h,i] = the original index of the
 * token at position i of the reblocked layout. */
int bsa_reblock(const bsa_params* p, const void* Q, const void* K, int32_t* perm,
                void* workspace, size_t workspace_bytes, void* stream);

/* Qp[b,h,i] = Q[b,h,perm[b,h,i]] (and K, V): the reblocked layout. */
int bsa_permute(const bsa_params* p, const void* Q, const void* K, const void* V,
                const int32_t* perm, void* Qp, void* Kp, void* Vp, void* stream);

/* bsa_permute of Q followed by bsa_pool on Qp, in one pass: Qp[b,h,i] =
 * Q[b,h,perm[b,h,i]] is written and the pooled means (qpool, anchor) are
 * those of the reblocked layout, bit for bit what the two calls give.  perm
 * is bsa_reblock's permutation of [0, N) per (b, h) (an entry outside [0, N)
 * is clamped into it).  Q, Qp 16-byte aligned; Qp must not overlap Q. */
int bsa_pool_permuted(const bsa_params* p, const void* Q, const int32_t* perm, void* Qp,
                      float* qpool, float* anchor, void* stream);

/* bsa_permute of K and V followed by bsa_summarize on Kp, Vp, in one pass:
 * writes Kp, Vp and the summaries of the reblocked layout, bit for bit what
 * the two calls give.  Same perm contract as bsa_pool_permuted. */
int bsa_summarize_permuted(const bsa_params* p, const void* K, const void* V,
                           const int32_t* perm, void* Kp, void* Vp, const float* anchor,
                           float* kpool, void* ksum, void* vsum, float* bias, void* stream);

/* O[b,h,perm[b,h,i]] = Op[b,h,i] (and lse from lsep when lse is non-NULL):
 * back to the original token order. */
int bsa_unpermute(const bsa_params* p, const void* Op, const float* lsep, const int32_t* perm,
                  void* O, float* lse, void* stream);

/* Workspace of bsa_forward_reblock: perm, the reblocked Q/K/V/O and lse, the
 * reblocking scratch and the forward's workspace. */
size_t bsa_forward_reblock_workspace_bytes(const bsa_params* p);

/* bsa_reblock, then bsa_pool_permuted and bsa_summarize_permuted (the
 * reblocked layout without a separate gather), bsa_select and bsa_attend on
 * it, bsa_unpermute: O (and lse) in the original order. */
int bsa_forward_reblock(const bsa_params* p, const void* Q, const void* K, const void* V,
                        void* O, float* lse, void* workspace, size_t workspace_bytes,
                        void* stream);

/* ---- FP8 (e4m3) exact and compressed branch --------------------------- */

/* The pages name a quantised sparse kernel ("H3 Sparse Attention", comfy.icu
 * WAS node, section "What it actually does": the sparse layers compute in
 * INT8 inside the kernel, at some cost in fidelity).  This is that option
 * with FP8: the attention operands are e4m3 codes, the path before it (pool,
 * summarize, select) is the bf16 path unchanged.  Format and scaling are this
 * library's reading:
 *   - e4m3 (OCP FP8, max 448), round to nearest even, saturating;
 *   - one scale per 128-row group: each 128-token block of Q, K and V (real
 *     rows only) and each 128-row tile of the summary tables k~ and v~;
 *   - codes = e4m3(x * fp32(448 / amax)), scale = fp32(amax / 448) (both 1
 *     for an all-zero group);
 *   - in the kernel, logits use the scales of the query block and of the key
 *     block / summary tile; softmax numerators p enter the PV product as
 *     e4m3(p * s_v / v_ref), v_ref the head's largest value scale, and the
 *     row sum stays in fp32.
 * All pointers are device pointers owned by the caller (16-byte aligned for
 * the code arrays, 4-byte for the scales).  ntile = ceil(nb / 128). */
typedef struct {
  void* q8;         /* e4m3 [B,H,N,128], row-major like Q                     */
  float* q_scale;   /* [B,H,nb]                                               */
  void* k8;         /* e4m3 [B,H,N,128]                                       */
  float* k_scale;   /* [B,H,nb]                                               */
  void* vt8;        /* e4m3 [B,H,nb,128,128]: block j of V as [dim][key],
                       keys past N zero                                       */
  float* v_scale;   /* [B,H,nb]                                               */
  void* ks8;        /* e4m3 [B,H,nb,128], the bf16 k~ rows quantised per tile */
  float* ks_scale;  /* [B,H,ntile]                                            */
  void* vst8;       /* e4m3 [B,H,ntile,128,128]: tile u of v~ as [dim][row],
                       rows past nb zero                                      */
  float* vs_scale;  /* [B,H,ntile]                                            */
  float* v_ref;     /* [B,H]: max of v_scale and vs_scale of the head         */
} bsa_fp8_operands;

/* Bytes of one operand set carved from a single buffer (each piece 256-byte
 * aligned, in field order); 0 for invalid parameters. */
size_t bsa_fp8_operands_bytes(const bsa_params* p);

/* Fills *out with pointers into the caller's buffer `base` (256-byte
 * aligned, at least bsa_fp8_operands_bytes(p) bytes).  Allocates nothing. */
int bsa_fp8_operands_carve(const bsa_params* p, void* base, size_t bytes,
                           bsa_fp8_operands* out);

/* Quantises Q, K, V (bf16 [B,H,N,128]) and the summary tables ksum, vsum
 * (bf16 [B,H,nb,128] as bsa_summarize wrote them) into *ops, and writes
 * ops->v_ref.  Six launches on `stream`; every byte of *ops is written. */
int bsa_quantize_fp8(const bsa_params* p, const void* Q, const void* K, const void* V,
                     const void* ksum, const void* vsum, const bsa_fp8_operands* ops,
                     void* stream);

/* bsa_attend on the e4m3 operands of bsa_quantize_fp8 (tcgen05
 * kind::f8f6f4, fp32 accumulate in TMEM), with the same idx/cnt/bias and the
 * same outputs (O bf16, optional lse). */
int bsa_attend_fp8(const bsa_params* p, const bsa_fp8_operands* ops, const int32_t* idx,
                   const int32_t* cnt, const float* bias, void* O, float* lse,
                   void* stream);

/* Workspace of bsa_forward_fp8: bsa_workspace_bytes(p) followed by one
 * operand set. */
size_t bsa_forward_fp8_workspace_bytes(const bsa_params* p);

/* bsa_pool, bsa_summarize, bsa_select, bsa_quantize_fp8, bsa_attend_fp8 in
 * order on `stream`, intermediates in the caller's workspace (256-byte
 * aligned, at least bsa_forward_fp8_workspace_bytes(p) bytes). */
int bsa_forward_fp8(const bsa_params* p, const void* Q, const void* K, const void* V,
                    void* O, float* lse, void* workspace, size_t workspace_bytes,
                    void* stream);

/* ---- option: threshold selection (content-adaptive count) ---------------
 * "H3 Sparse Attention" (comfy.icu, WAS node page), "The inputs that
 * matter": the content-adaptive method takes a threshold tau instead of a
 * block count, and keeps about 16 %, 7 % and 3 % of the key blocks at
 * tau = 1.0, 1.5 and 2.0 -- the standard normal's upper tail at tau, so the
 * threshold is read as a z-score of the pooled block scores.  Lists then
 * vary in length from row to row; p->top_k is not used by these calls
 * (any value >= 1). */

/* Row length of the idx array written by bsa_select_threshold: nb. */
int32_t bsa_threshold_capacity(const bsa_params* p);

/* Steps 4-5 with threshold selection.  For video query block i >= pb, with
 * S_ij as in bsa_select over the video key blocks j in [pb, nb), mu_i their
 * mean and sigma_i their population standard deviation (fp32): keep every j
 * with S_ij - mu_i >= tau * sigma_i; every j when the row's scores are all
 * equal; the top-scoring j (lowest index on ties) when none qualifies.
 *   idx[b,h,i,:] = 0..pb-1, then the kept j ascending, then -1 padding
 *   (int32 [B,H,nb,nb]),  cnt[b,h,i] = pb + number kept  (int32 [B,H,nb]).
 * Prefix query blocks list every block, as in bsa_select.  tau must be
 * finite (else BSA_ERR_INVALID).  Deterministic. */
int bsa_select_threshold(const bsa_params* p, float tau, const float* qpool,
                         const float* kpool, int32_t* idx, int32_t* cnt, void* stream);

/* Scratch of bsa_attend_lists (the work schedule): bytes, or 0 if p is
 * invalid. */
size_t bsa_attend_lists_workspace_bytes(const bsa_params* p);

/* Step 6 over variable-length lists: as bsa_attend, but row i of idx has
 * stride kcap and holds cnt[b,h,i] listed blocks (ascending, the pb prefix
 * blocks first; prefix query blocks list all nb).  Counts are clamped to
 * [1, kcap].  Requires kcap <= nb, and kcap == nb when prefix > 0
 * (BSA_ERR_INVALID otherwise).  `workspace` (device, 256-byte aligned, at
 * least bsa_attend_lists_workspace_bytes(p) bytes) holds the schedule that
 * pairs rows of similar length; its contents need not be initialised.
 * Deterministic: no row's result depends on the rows it is scheduled with. */
int bsa_attend_lists(const bsa_params* p, const void* Q, const void* K, const void* V,
                     const int32_t* idx, int32_t kcap, const int32_t* cnt,
                     const void* ksum, const void* vsum, const float* bias, void* O,
                     float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace of bsa_forward_threshold. */
size_t bsa_forward_threshold_workspace_bytes(const bsa_params* p);

/* bsa_pool, bsa_summarize, bsa_select_threshold, bsa_attend_lists in order on
 * `stream`, intermediates in the caller's workspace (256-byte aligned, at
 * least bsa_forward_threshold_workspace_bytes(p) bytes). */
int bsa_forward_threshold(const bsa_params* p, float tau, const void* Q, const void* K,
                          const void* V, void* O, float* lse, void* workspace,
                          size_t workspace_bytes, void* stream);

/* ---- option: extra top-scoring tokens per query block -------------------
 * "H3 Sparse Attention" (comfy.icu, WAS node page), "The inputs that
 * matter": besides its chosen blocks, each query block reads a number of
 * individually chosen top-scoring tokens (`extra_tokens`, 256 by default, 0
 * the fastest setting).  This library's readings (the page gives no
 * formula):
 *   - token u scores s_iu = qhat_i . k_u / sqrt(D) for query block i (the
 *     token analogue of the pooled block score);
 *   - the candidates are the video tokens of the video blocks NOT listed for
 *     i; dense-prefix query blocks take none;
 *   - the min(n_extra, #candidates) highest scores are taken, ties to the
 *     lower token index;
 *   - every key token enters the softmax once: an extra token is read
 *     exactly, so the summary row of its block stands for the block's
 *     remaining tokens (the block-summary definition of bsa_summarize over
 *     those tokens only; no row once all of the block's tokens are extra).
 * The selection computes the scores on the tensor cores with qhat split into
 * bf16 hi + lo parts (about 16 significant bits, K is exact bf16) and fp32
 * accumulation, so two tokens whose scores differ by less than about
 * 2^-16 * sum_d |qhat_d k_ud| / sqrt(D) may be ordered either way.
 * 0 <= n_extra <= BSA_MAX_EXTRA_TOKENS, and B*H*N < 2^31, else
 * BSA_ERR_INVALID.  These calls use the fixed top-k lists of bsa_select. */
#define BSA_MAX_EXTRA_TOKENS 512

/* Row capacity scap of the side summary table: min(n_extra, nbv) rounded up
 * to a multiple of 128 (0 for n_extra = 0); -1 for invalid arguments. */
int32_t bsa_extra_side_capacity(const bsa_params* p, int32_t n_extra);

/* bsa_summarize plus the fp32 statistics the side summaries start from:
 * kstat, vstat fp32 [B,H,nb,D] = k~ and v~ before bf16 rounding (anchor
 * variant) or the mean key and mean value (mean variant); lse_blk fp32
 * [B,H,nb] = the block's log-sum-exp at the anchor, LSE_j (ln n_j for the
 * mean variant).  Same reads as bsa_summarize (K and V once). */
int bsa_summarize_stats(const bsa_params* p, const void* K, const void* V, const float* anchor,
                        float* kpool, void* ksum, void* vsum, float* bias, float* kstat,
                        float* vstat, float* lse_blk, void* stream);

/* Scratch of bsa_select_extra: two candidate buffers per video query block,
 * one per half of each key block's tokens (0 for n_extra = 0); 0 also for
 * invalid arguments. */
size_t bsa_select_extra_workspace_bytes(const bsa_params* p, int32_t n_extra);

/* Extra tokens of every query block.  qpool as bsa_pool wrote it, K bf16
 * [B,H,N,D], idx/cnt as bsa_select wrote them.  Writes extra int32
 * [B,H,nb,n_extra] (token indices within the head, ascending, -1 padded) and
 * ecnt int32 [B,H,nb] (0 for dense-prefix query blocks).  `workspace`
 * (device, 256-byte aligned, bsa_select_extra_workspace_bytes bytes; may be
 * NULL for n_extra = 0) holds the candidate buffers; its contents need not be
 * initialised.  Deterministic. */
int bsa_select_extra(const bsa_params* p, int32_t n_extra, const float* qpool, const void* K,
                     const int32_t* idx, const int32_t* cnt, int32_t* extra, int32_t* ecnt,
                     void* workspace, size_t workspace_bytes, void* stream);

/* Summary rows of the blocks that lose some (not all) of their tokens to a
 * query block's extra tokens.  For video query block i, its affected blocks
 * j in ascending order get row a of
 *   side_k, side_v bf16 [B,H,nb,scap,D]  (k~', v~' over the remaining tokens),
 *   side_bias fp32 [B,H,nb,scap]         (bias', natural log; anchor variant:
 *                                          LSE'_j - anchor . bf16(k~')/sqrt(D),
 *                                          mean variant: ln(remaining count)),
 *   side_blk int32 [B,H,nb,scap]         (j),
 * side_cnt int32 [B,H,nb] = number of rows (0 for prefix query blocks).  Rows
 * from side_cnt up to the next multiple of 128 are zero with bias -inf and
 * block -1.  Anchor variant: the rows are downdates of kstat/vstat/lse_blk by
 * the extra tokens' softmax weights at the anchor, recomputed from the
 * remaining rows when less than 2^-6 of the block's anchor mass remains;
 * mean variant: downdates of the mean key (kpool) and mean value (vstat). */
int bsa_extra_summaries(const bsa_params* p, int32_t n_extra, const void* K, const void* V,
                        const float* anchor, const float* kpool, const float* kstat,
                        const float* vstat, const float* lse_blk, const int32_t* extra,
                        const int32_t* ecnt, void* side_k, void* side_v, float* side_bias,
                        int32_t* side_blk, int32_t* side_cnt, void* stream);

/* Step 6 with extra tokens: as bsa_attend, plus for every video query row
 * the extra tokens of its block as exact logits (rows gathered from K and V
 * by index), and in the compressed branch the global summary rows of blocks
 * that hold any of the row's extra tokens replaced by the row's side summary
 * rows.  With n_extra = 0 (ecnt and side_cnt all zero) it computes exactly
 * what bsa_attend computes. */
int bsa_attend_extra(const bsa_params* p, int32_t n_extra, const void* Q, const void* K,
                     const void* V, const int32_t* idx, const int32_t* cnt, const int32_t* extra,
                     const int32_t* ecnt, const void* ksum, const void* vsum, const float* bias,
                     const void* side_k, const void* side_v, const float* side_bias,
                     const int32_t* side_cnt, void* O, float* lse, void* stream);

/* Workspace of bsa_forward_extra: bsa_workspace_bytes(p) followed by the
 * statistics, lists, side table and candidate buffers (0 if invalid). */
size_t bsa_forward_extra_workspace_bytes(const bsa_params* p, int32_t n_extra);

/* bsa_pool, bsa_summarize_stats, bsa_select, bsa_select_extra,
 * bsa_extra_summaries, bsa_attend_extra in order on `stream`, intermediates in
 * the caller's workspace (256-byte aligned). */
int bsa_forward_extra(const bsa_params* p, int32_t n_extra, const void* Q, const void* K,
                      const void* V, void* O, float* lse, void* workspace, size_t workspace_bytes,
                      void* stream);

/* Human-readable name of a bsa_status value (static string). */
const char* bsa_status_string(int status);

/* Launches a single-CTA kernel that waits on a barrier nothing will ever
 * release, bounded by timeout_ns, then writes BSA_ERR_TIMEOUT to *dev_status
 * and returns.  Exists so tests can check on a GPU that an expired wait ends
 * with a status the host can read and leaves the context usable. */
int bsa_debug_expired_wait(int32_t* dev_status, uint64_t timeout_ns, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* BSA_H_ */
