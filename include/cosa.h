/*
 * cosa.h -- C ABI of the CoSA block-sparse prefill attention library for
 * B200 (sm_100a): the Kernel-Aware Proxy (KAP, cosa_plan) and the
 * Ordered-Skipping Kernel (OSK, cosa_attend).
 *
 * Method: "CoSA: Accelerating Long-Context Inference via Proxy-Kernel
 * Co-Designed Sparse Attention" (gist.science/paper/2607.25291), technical
 * summary Sec. 2.1 (order invariance, computation-order mask), Sec. 2.2
 * (KAP), Sec. 2.3 (OSK).  The KV-head-major layout [B, Hkv, L, d] and the
 * paged-cache form follow "CompactAttention: Accelerating Chunked Prefill
 * with Block-Union KV Selection" (gist.science/de/paper/2605.16839),
 * execution stage.
 *
 * Conventions for every entry point:
 *  - All tensor arguments are DEVICE pointers owned by the caller; the
 *    library allocates no device memory and keeps no pointer after a call
 *    returns.  Work is enqueued asynchronously on `stream` (0 = legacy
 *    default stream); outputs are valid once the stream reaches that point.
 *  - Tensors are dense, row-major, bf16 (uint16 bit patterns) unless stated.
 *    Q is [B, Hq, Nq, d]; K and V are [B, Hkv, Nkv, d] or, when
 *    shape->paged, a page pool [num_pages, Hkv, bk, d] addressed through
 *    page_table [B, ceil(Nkv/bk)] (int32 physical page of each logical KV
 *    block).  q, k, v and out must be 16-byte aligned.
 *  - Causality: query i sits at absolute position Nkv - Nq + i and sees keys
 *    0 .. Nkv - Nq + i.  GQA: query head h reads kv-head h / (Hq / Hkv).
 *  - Arguments are validated on the host before anything is launched; on
 *    error nothing is enqueued and a cosa_status other than COSA_OK is
 *    returned.  Device code never traps: every wait in a kernel is bounded,
 *    and a timed-out wait writes a nonzero code to *dev_status (optional,
 *    caller-zeroed uint32 in device memory) before the kernel returns.
 */
#ifndef COSA_H
#define COSA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define COSA_API __attribute__((visibility("default")))
#else
#define COSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  COSA_OK = 0,
  COSA_EINVAL = 1,        /* null required pointer or parameter out of range */
  COSA_EALIGN = 2,        /* a tensor pointer is not 16-byte aligned */
  COSA_ESHAPE = 3,        /* inconsistent shape (divisibility, Nkv < Nq, ...) */
  COSA_EWORKSPACE = 4,    /* workspace missing or smaller than cosa_plan_workspace_bytes */
  COSA_ECUDA = 5,         /* a CUDA runtime/driver call or a launch failed */
  COSA_EUNSUPPORTED = 6   /* valid but outside what the kernels implement (e.g. d != 128) */
} cosa_status;

typedef struct {
  int B, Hq, Hkv;   /* batch, query heads, kv heads (Hq % Hkv == 0) */
  int Nq, Nkv;      /* query tokens, key tokens (Nkv >= Nq; both multiples of stride) */
  int d;            /* head dimension; the kernels implement d == 128 */
  int bq, bk;       /* Q-block rows and KV-block (page) size, each 64 or 128 */
  int stride;       /* KAP pooling stride s (power of two, s | bq, s | bk, bk/s <= 32, bq/s <= 32) */
  int paged;        /* 0: K,V are [B,Hkv,Nkv,d]; 1: page pool [num_pages,Hkv,bk,d] + page_table */
  int num_pages;    /* pages in the pool when paged */
} cosa_shape;

/* Number of Q-blocks ceil(Nq/bq) and KV blocks ceil(Nkv/bk). */
COSA_API int cosa_num_qblocks(const cosa_shape* shape);
COSA_API int cosa_num_kblocks(const cosa_shape* shape);

/* Budget rule (Sec. 2.2 "moderate budget"; the formula is this library's
 * reading): Q-block I has n_I causally visible KV blocks; KAP keeps
 * k_I = max(1, ceil(n_I * bp / 10000)) of them, bp = round(budget * 10000).
 * Returns max over I of k_I: the minimum last dimension of `order` for
 * cosa_plan.  Returns -1 for an invalid shape or budget outside (0, 1]. */
COSA_API int cosa_kmax(const cosa_shape* shape, double budget);

/* Bytes of device workspace cosa_plan needs (pooled Q, pooled K, the
 * max-pooled block scores of every pooled query row and partial row maxima).
 * 0 for an invalid shape. */
COSA_API size_t cosa_plan_workspace_bytes(const cosa_shape* shape);

/* KAP, stage 1 (Sec. 2.2): downsample Q and K (mean of `stride` consecutive
 * tokens), score pooled queries against pooled keys, MaxPool the scores over
 * the keys of each KV block, MaxNorm each pooled row (subtract its max),
 * flag HRM blocks (the first block holding a pooled row's max), aggregate
 * over the pooled rows of each Q-block (max), and sort each Q-block's
 * causally visible blocks by (HRM desc, score desc, block index asc),
 * keeping k_I of them.
 *  order      [B, Hq, nQB, kmax] int32 out: KV block indices in visit
 *             order, entries >= count padded with -1.
 *  count      [B, Hq, nQB] int32 out: k_I.
 *  hrm_count  [B, Hq, nQB] int32 out (nullable): number of HRM blocks.
 *  block_score [B, Hq, nQB, nKB] fp32 out (nullable): aggregated MaxNorm
 *             score of every block (-inf where not causally visible).
 *  hrm_flags  [B, Hq, nQB, nKB] uint8 out (nullable): 1 for HRM blocks.
 *  workspace  device scratch of ws_bytes >= cosa_plan_workspace_bytes.
 * Returns COSA_EINVAL if kmax < cosa_kmax(shape, budget). */
COSA_API cosa_status cosa_plan(const cosa_shape* shape, const void* q, const void* k, const int32_t* page_table,
                      double budget, int kmax, int32_t* order, int32_t* count, int32_t* hrm_count,
                      float* block_score, uint8_t* hrm_flags, void* workspace, size_t ws_bytes,
                      uint32_t* dev_status, cudaStream_t stream);

/* cosa_plan for one chunk of a chunked prefill, with the pooled keys kept
 * from one chunk to the next.  In chunked prefill ("CompactAttention:
 * Accelerating Chunked Prefill with Block-Union KV Selection", selection
 * stage and evaluation setup) each chunk of Nq new queries attends to a
 * cache of Nkv keys that holds every earlier chunk plus its own; re-pooling
 * the whole cache per chunk reads all of K again.  Here the pooled keys live
 * in a caller-owned cache and only the keys not yet pooled are read.
 *  kp_cache    [B, Hkv, kp_capacity, d] bf16, device, 16-byte aligned,
 *              owned by the caller and kept across chunks.  Row c of a head
 *              holds the mean of keys stride*c .. stride*c + stride - 1.
 *  kp_capacity pooled-key rows per head in the cache (>= Nkv / stride).
 *  kp_valid    rows 0 .. kp_valid-1 of every head were written by an
 *              earlier call for the same keys and are used as they are;
 *              rows kp_valid .. Nkv/stride - 1 are pooled from k (contiguous
 *              or paged, as for cosa_plan) and written to the cache before
 *              scoring.  0 <= kp_valid <= Nkv / stride; kp_valid = 0 pools
 *              every key.  Chunk after chunk, pass the previous call's
 *              Nkv / stride.
 * Every other argument and result is cosa_plan's, and the results are
 * bit-identical to cosa_plan's on the same q and k (pooling is
 * deterministic per row).  The workspace is sized by
 * cosa_plan_workspace_bytes (its pooled-key region goes unused).  Returns
 * COSA_EINVAL for a null cache or kp_capacity / kp_valid out of range,
 * COSA_EALIGN for a misaligned cache. */
COSA_API cosa_status cosa_plan_chunk(const cosa_shape* shape, const void* q, const void* k,
                                     const int32_t* page_table, void* kp_cache, int kp_capacity, int kp_valid,
                                     double budget, int kmax, int32_t* order, int32_t* count,
                                     int32_t* hrm_count, float* block_score, uint8_t* hrm_flags,
                                     void* workspace, size_t ws_bytes, uint32_t* dev_status,
                                     cudaStream_t stream);

/* The Kernel-Aware Proxy for one decode step.  The CoSA pages treat only
 * prefill and name decoding as future work (technical summary Sec. 4); this
 * is the plainest single-row reading of Sec. 2.2: shape->Nq == 1, the query
 * of each head sits at position Nkv - 1 and is not pooled, the keys are
 * pooled as in prefill (mean of `stride` keys, kept in the caller's pooled-key
 * cache exactly as for cosa_plan_chunk), and per head
 *   S[c] = q . Kp[c] over every pooled key, MaxPool over each KV block's
 *   pooled keys, MaxNorm (minus the maximum), HRM = the first block holding
 *   the maximum, order = (HRM, score desc, block asc), the first
 *   k = max(1, ceil(nKB * budget)) kept.
 *  q          [B, Hq, 1, d] bf16 (16-byte aligned).
 *  k          keys as for cosa_plan (contiguous or paged); rows kp_valid ..
 *             Nkv/stride - 1 of kp_cache are pooled from it first.
 *  kp_cache, kp_capacity, kp_valid: as for cosa_plan_chunk (Nkv must be a
 *             multiple of stride).
 *  order      [B, Hq, 1, kmax] int32 out (kmax >= k), padded -1; count,
 *             hrm_count [B, Hq] out; block_score [B, Hq, nKB] fp32 and
 *             hrm_flags [B, Hq, nKB] uint8 out (nullable).
 * The decode step's attention is cosa_decode_attend (or cosa_attend) on the
 * same shape (Nq = 1): with one valid row the tile-wide skip vote is that
 * row's own test.
 * Returns COSA_ESHAPE if Nq != 1, COSA_EINVAL for null pointers, a budget
 * outside (0, 1], kp arguments out of range or kmax < k. */
COSA_API cosa_status cosa_decode_plan(const cosa_shape* shape, const void* q, const void* k,
                                      const int32_t* page_table, void* kp_cache, int kp_capacity, int kp_valid,
                                      double budget, int kmax, int32_t* order, int32_t* count,
                                      int32_t* hrm_count, float* block_score, uint8_t* hrm_flags,
                                      cudaStream_t stream);

/* The attention of one decode step (shape->Nq == 1): OSK (technical summary
 * Sec. 2.3) on the single query row of each head, at position Nkv - 1:
 * visit order[b,h,0,0..count-1]; skip a visit when fp32(m_loc - m_run) < T,
 * T = fp32(ln(skip_eps) * sqrt(d)) (with one row the tile-wide vote is the
 * row's own test); fold the others into the softmax (scale 1/sqrt(d)).  The
 * pages leave decoding to future work (Sec. 4): the decisions, skip bits and
 * results are those of cosa_attend on the same one-row shape, computed by
 * kernels shaped for a memory-bound step: the logits of every visited block
 * in parallel, the decisions as a prefix-max scan (a skipped visit never
 * raises the running max, since T <= 0), the P.V of the computed visits in
 * parallel against their common maximum.  Logits are fp32 sums on the CUDA
 * cores and P stays fp32, so on real-valued inputs a decision can differ
 * from cosa_attend's where m_loc - m_run - T is within fp32 rounding of 0.
 *  q          [B, Hq, 1, d] bf16.
 *  order      [B, Hq, 1, kmax] int32 (cosa_decode_plan's); count [B, Hq, 1].
 *  out        [B, Hq, 1, d] bf16 out; lse [B, Hq] fp32 out (nullable);
 *             skip_bits [B, Hq, ceil(kmax/32)] uint32 out (nullable).
 *  workspace  >= cosa_decode_attend_workspace_bytes(shape, kmax) bytes of
 *             device memory, 256-byte aligned (logits of every visit, the
 *             visits' row maxima, per-CTA partial sums).
 * Entries of order outside [0, nKB) count as skipped visits.  Returns
 * COSA_ESHAPE if Nq != 1, COSA_EWORKSPACE for a missing or small workspace,
 * COSA_EUNSUPPORTED when kmax is too large for the scan's shared memory. */
COSA_API size_t cosa_decode_attend_workspace_bytes(const cosa_shape* shape, int kmax);
COSA_API cosa_status cosa_decode_attend(const cosa_shape* shape, const void* q, const void* k, const void* v,
                                        const int32_t* page_table, const int32_t* order, const int32_t* count,
                                        int kmax, double skip_eps, void* out, float* lse, uint32_t* skip_bits,
                                        void* workspace, size_t ws_bytes, cudaStream_t stream);

/* Block union ("CompactAttention: Accelerating Chunked Prefill with
 * Block-Union KV Selection", method, selection stage): turn a per-head
 * selection into one KV block table per (batch, kv-head group), the union
 * over every Q-block of the call (the chunk) and every query head sharing
 * the kv-head.  Every block any of them selected is in the table, no other
 * block is, and the table ascends.
 *  order, count  [B, Hq, nQB, kmax], [B, Hq, nQB] int32 in: the selection
 *                (typically cosa_plan's M_KAP); entries at or beyond count
 *                and indices outside [0, nKB) are ignored; count is clamped
 *                to [0, kmax].
 *  table         [B, Hkv, nKB] int32 out: the union, ascending, padded -1.
 *  table_len     [B, Hkv] int32 out: its length.
 *  union_order   [B, Hq, nQB, union_kmax] int32 out (nullable, together with
 *                union_count): per Q-block, the table entries it can see
 *                causally, ascending, padded -1 -- an order cosa_attend
 *                executes (skip_eps = 0 gives the dense attention over the
 *                union the paper runs).  union_kmax must be >= the number of
 *                causally visible blocks of the last Q-block.
 *  union_count   [B, Hq, nQB] int32 out: length of each union_order row.
 * Returns COSA_EINVAL for null outputs, a missing order/count, or a
 * union_kmax that is too small. */
COSA_API cosa_status cosa_block_union(const cosa_shape* shape, const int32_t* order, const int32_t* count,
                                      int kmax, int32_t* table, int32_t* table_len, int32_t* union_order,
                                      int32_t* union_count, int union_kmax, cudaStream_t stream);

/* Fill `order`/`count` with every causally visible block of each Q-block in
 * natural order (0, 1, ..., n_I - 1): the dense path, which cosa_attend runs
 * with skip_eps = 0 (Sec. 4 reports speedup against dense attention).
 * kmax must be >= cosa_num_kblocks(shape). */
COSA_API cosa_status cosa_dense_order(const cosa_shape* shape, int kmax, int32_t* order, int32_t* count,
                             cudaStream_t stream);

/* Host-side check of a visit order before cosa_attend, for a caller that
 * edits or builds `order` itself (the computation-order mask of Sec. 2.1:
 * a block visited twice would be folded into the softmax twice, which no
 * kernel can detect).  order_host [B, Hq, nQB, kmax] and count_host
 * [B, Hq, nQB] are int32 in HOST memory (copy them back first); nothing is
 * launched.  Every count must lie in [0, kmax]; every entry t < count of a
 * row must be a KV block its Q-block can see causally (0 <= j < n_I, as in
 * cosa_kmax), and no block may appear twice in a row.  cosa_plan's and
 * cosa_dense_order's results always pass.
 *  first_bad  (nullable) out: the flat index row * kmax + t of the first bad
 *             entry, or -1 - row for a bad count; 0 when all is well.
 * Returns COSA_OK, COSA_EINVAL at the first bad count or entry (or a null
 * array), COSA_ESHAPE for an invalid shape or kmax < 1. */
COSA_API cosa_status cosa_check_order(const cosa_shape* shape, const int32_t* order_host,
                                      const int32_t* count_host, int kmax, int64_t* first_bad);

/* OSK, stage 2 (Sec. 2.3): for each (b, h, Q-block I) visit only the KV
 * blocks order[b,h,I,0..count-1], in that order (mask-skipped blocks are
 * never touched); per visited block compute S = Q K^T exactly, and skip the
 * block when every row of the Q-block satisfies m_loc - m_run < T with
 * T = fp32(ln(skip_eps) * sqrt(d)) in raw-logit units (a row with no visible
 * key in the block always agrees; the bucket effect of Sec. 1 makes the
 * decision tile-wide); otherwise update the online softmax (scale
 * 1/sqrt(d)) and accumulate P V.
 *  skip_eps   in [0, 1); 0 never skips.
 *  out        [B, Hq, Nq, d] bf16 out; a row that saw no key is 0.
 *  lse        [B, Hq, Nq] fp32 out (nullable): log-sum-exp of the scaled
 *             logits (natural log), -inf for a row that saw no key.
 *  skip_bits  [B, Hq, nQB, ceil(kmax/32)] uint32 out (nullable): bit t of
 *             word t/32 set iff visit t was skipped in-kernel.
 * order entries outside [0, nKB) are treated as skipped blocks; count is
 * clamped to [0, kmax]. */
COSA_API cosa_status cosa_attend(const cosa_shape* shape, const void* q, const void* k, const void* v,
                        const int32_t* page_table, const int32_t* order, const int32_t* count, int kmax,
                        double skip_eps, void* out, float* lse, uint32_t* skip_bits, uint32_t* dev_status,
                        cudaStream_t stream);

/* OSK over one visit order per GQA group: the execution form of
 * "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
 * Selection" (method, execution stage: one block table per (batch, kv-head
 * group), read in place), run with CoSA's ordered skipping (technical
 * summary Sec. 2.3).  Every query head of kv-head g visits the blocks
 * order[b,g,I,0..count-1] in that order; per head the arithmetic, the skip
 * vote (on that head's own 128-row tile) and the results are exactly those
 * of cosa_attend given the same order for each head of the group, but each
 * K/V tile is loaded once for two heads.
 *  order      [B, Hkv, nQB, kmax] int32 in (cosa_block_union's union_order
 *             rows are the same for every head of a group: any one of them
 *             serves; cosa_dense_order on a shape with Hq = Hkv gives the
 *             dense path's).
 *  count      [B, Hkv, nQB] int32 in.
 *  out, lse, skip_bits, dev_status: as for cosa_attend (per query head).
 * Returns COSA_EUNSUPPORTED when Hq / Hkv is odd and above 1 (G = 1 runs
 * cosa_attend's kernel, whose order layout is then the same), and otherwise
 * what cosa_attend returns for the same arguments. */
COSA_API cosa_status cosa_attend_group(const cosa_shape* shape, const void* q, const void* k, const void* v,
                                       const int32_t* page_table, const int32_t* order, const int32_t* count,
                                       int kmax, double skip_eps, void* out, float* lse, uint32_t* skip_bits,
                                       uint32_t* dev_status, cudaStream_t stream);

/* Failure-detection test hook (no counterpart in the papers): runs
 * cosa_attend's kernel with skip_eps = 0 on the given arguments, except that
 * in every CTA the issuing thread, before the first QK^T, waits on a barrier
 * that nothing ever arrives at.  That wait, like every other wait of the
 * kernel, gives up after wait_limit_ns nanoseconds of %globaltimer; the
 * kernel then records a timeout code in *dev_status (COSA_DEV_TIMEOUT_PIPE
 * from that wait, or COSA_DEV_TIMEOUT_MMA from the softmax threads' wait for
 * the QK^T that never comes, whichever gives up first), every thread
 * runs through the rest of its barriers without waiting, the issuing thread
 * waits (again bounded) for the copies it started, TMEM is released and the
 * CTA exits; CTAs that start after the status is set exit at once.  The
 * call returns COSA_OK; the CTAs that ran write zeros to their rows of
 * `out`, the others leave them as they were; the context stays usable.  A
 * test calls it to check that a wait that runs out ends in an error status
 * rather than a hang or a fault.  Not for use in production.
 *  dev_status     required; should be 0 before the call.
 *  wait_limit_ns  in [1e3, 1e9].
 * Returns COSA_EINVAL for a null dev_status or a limit out of range, and
 * otherwise what cosa_attend returns for the same arguments. */
#define COSA_DEV_TIMEOUT_TMA 0x100u    /* device status: a TMA transaction never completed */
#define COSA_DEV_TIMEOUT_MMA 0x200u    /* device status: a tensor-core commit never arrived */
#define COSA_DEV_TIMEOUT_PIPE 0x300u   /* device status: a producer/consumer hand-off never arrived */
COSA_API cosa_status cosa_test_attend_wait_timeout(const cosa_shape* shape, const void* q, const void* k,
                                                   const void* v, const int32_t* page_table, const int32_t* order,
                                                   const int32_t* count, int kmax, void* out, uint32_t* dev_status,
                                                   uint64_t wait_limit_ns, cudaStream_t stream);

/* cosa_plan without a workspace argument, for callers that cannot obtain
 * device memory of their own (for example a serving engine that reserves the
 * whole GPU at start-up and only hands kernels the tensors it owns, or a
 * plug-in whose host framework keeps the allocator to itself).  The paper has
 * no counterpart to this call; it exists only for such callers.
 * Same arguments and results as cosa_plan, minus workspace/ws_bytes.  The
 * scratch is one fixed array of COSA_STATIC_SCRATCH_BYTES inside the
 * library's device image: every GPU that loads it holds that memory until the
 * process exits; shapes with cosa_plan_workspace_bytes(shape) larger than it
 * get COSA_EWORKSPACE and nothing is launched; calls that can overlap on the
 * GPU (different streams without ordering) race on the shared array, calls on
 * one stream do not.  The first call on each device looks up the array's
 * device address with that device current: make it before any stream
 * capture.  Nothing is allocated, ever. */
#define COSA_STATIC_SCRATCH_BYTES (64u << 20)
COSA_API cosa_status cosa_plan_static(const cosa_shape* shape, const void* q, const void* k,
                                      const int32_t* page_table, double budget, int kmax, int32_t* order,
                                      int32_t* count, int32_t* hrm_count, float* block_score,
                                      uint8_t* hrm_flags, uint32_t* dev_status, cudaStream_t stream);

/* The skip threshold T = fp32(ln(eps) * sqrt(d)) cosa_attend uses (-inf for eps == 0). */
COSA_API float cosa_skip_threshold(double eps, int d);

/* Human-readable name of a status code (static storage). */
COSA_API const char* cosa_status_string(cosa_status status);

/* Library ABI version (major * 100 + minor). */
COSA_API int cosa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* COSA_H */
