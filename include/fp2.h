/*
 * fp2.h -- C ABI of libfp2: FlashPrefill V2 block-sparse prefill attention
 * for NVIDIA B200 (sm_100a).
 *
 * The operation is the one described in "FlashPrefill V2: Block-Sparse
 * Prefill Attention for Long-Context LLM Serving" (metallab.ai summary of
 * arXiv 2608.19758):
 *   - Figure 3: stage 1 ("pattern discovery") pools block-mean statistics
 *     under PackGQA and emits a CSR index of the selected key blocks;
 *     stage 2 runs sparse attention over the selected blocks while the
 *     unselected ones go through the mean-correction path, and both merge
 *     inside one online softmax.
 *   - Figure 4: a pruned block J contributes the surrogate
 *     |B_J| e^{s_J} (v_J, 1) to the softmax numerator and denominator.
 *   - Abstract: "max-based dynamic thresholding" (Table 9: alpha, here tau).
 *   - Table 7: CSR of selected blocks, per KV head, int32.
 *   - Figure 1 / Table 7: paged KV cache and continuous batching (varlen).
 *   - Table 1 footnote: FP8 by direct online quantisation.
 *
 * Formulas.  Hq query heads, Hkv kv-heads, G = Hq / Hkv (query head h reads
 * kv-head h / G), head dim d, block size B.  Sequence s of length L_s has
 * nb_s = ceil(L_s / B) blocks; NB = sum_s nb_s.  For the row (s, g, i):
 *   sc_j = max_{h in group g} mean(Q_block i, h) . mean(K_block j, g) / sqrt(d)
 *   tau == 0 keeps every block j <= i; otherwise block j is kept when
 *   sc_j >= tau * max_{j' <= i} sc_j', and blocks 0 and i are always kept.
 *   Attention covers the kept blocks exactly (causal inside block i) and
 *   adds, for every skipped block j (always a full block, n_j = B), one
 *   pseudo-token with logit q . Kbar_j / sqrt(d) + ln n_j and value Vbar_j.
 *   O = numerator / denominator; LSE = ln(denominator) in the 1/sqrt(d)-
 *   scaled logit units, pseudo-tokens included.
 *
 * Conventions for every entry point:
 *   - Device pointers are CUDA global-memory addresses on the current
 *     device; host pointers are ordinary process memory.  Every buffer is
 *     owned by the caller.  The library allocates no memory, never frees,
 *     and never synchronises except inside fp2_status_check.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously in stream order; inputs must
 *     stay unchanged until the enqueued work has completed.
 *   - Return value: FP2_OK (0) or a negative FP2_ERR_* code.  Argument
 *     errors are detected on the host before anything is enqueued.
 *     Inconsistencies that can only be seen on the device (cu_seqlens that
 *     disagree with seqlens, page ids out of range, a wait that timed out)
 *     are recorded in the plan's status word and reported by
 *     fp2_status_check; kernels that see a bad plan do no work.
 *   - Calls that use distinct plan and workspace buffers may run
 *     concurrently from several host threads.
 */
#ifndef FP2_H_
#define FP2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FP2_VERSION 3

/* ---- error codes -------------------------------------------------------- */
#define FP2_OK 0
#define FP2_ERR_INVALID_ARG -1   /* a host-visible argument is wrong                 */
#define FP2_ERR_UNSUPPORTED -2   /* a valid configuration this build does not handle */
#define FP2_ERR_CAPACITY -3      /* a caller buffer is smaller than fp2_plan_sizes asks */
#define FP2_ERR_CUDA -4          /* a CUDA call or kernel launch failed              */
#define FP2_ERR_TIMEOUT -5       /* a device-side wait gave up (status word)         */
#define FP2_ERR_DEVICE_CHECK -6  /* a device-side consistency check failed (status)  */

/* ---- status word bits (fp2_status_check *device_status) ------------------ */
#define FP2_STATUS_BAD_SEQLENS 0x1u   /* cu_seqlens not consistent with the problem sizes */
#define FP2_STATUS_BAD_PAGE 0x2u      /* a page id outside [0, num_pages)                 */
#define FP2_STATUS_TIMEOUT 0x4u       /* a bounded wait inside a kernel ran out           */
#define FP2_STATUS_BOUNDS 0x8u        /* an index check of the debug build (libfp2_debug.so,
                                         built with FP2_DEBUG) failed; the access was
                                         clamped or skipped                                */

/* ---- element types -------------------------------------------------------- */
#define FP2_DTYPE_BF16 0   /* bfloat16 Q, K, V                                     */
#define FP2_DTYPE_E4M3 1   /* float8 e4m3 Q, K, V with per-(block, head) fp32 scales */

/* ---- fp2_prefill flags ---------------------------------------------------- */
#define FP2_NO_CORRECTION 0x1u     /* skipped blocks are dropped (no pseudo-tokens)   */
#define FP2_DEBUG_DROP_Q_LOAD 0x100u /* fault injection: never load Q, so the first
                                        wait on it runs out; the kernel records
                                        FP2_STATUS_TIMEOUT and returns */

/*
 * One prefill problem: a varlen batch of num_seqs causal sequences packed
 * along the token axis (T = sum of seqlens tokens).
 *
 *   seqlens      HOST int32 [num_seqs], each >= 1.  Used for validation and
 *                sizing on the host.
 *   cu_seqlens   DEVICE int32 [num_seqs + 1]; cu_seqlens[0] = 0 and
 *                cu_seqlens[s+1] - cu_seqlens[s] = seqlens[s].  Checked on the
 *                device (FP2_STATUS_BAD_SEQLENS).
 *   num_q_heads, num_kv_heads   Hq, Hkv with Hq % Hkv == 0 and
 *                (Hq / Hkv) * block_size a multiple of 128 (PackGQA tiles of
 *                128 query rows).
 *   head_dim     d in {64, 128}.   block_size   B in {64, 128}.
 *   tau          threshold >= 0 (0 = dense: every causal block kept).
 *   page_size    0: K and V are contiguous [T, Hkv, d].  64: K and V are page
 *                pools [num_pages, 64, Hkv, d]; token t of sequence s is in
 *                page page_table[s * page_table_stride + t / 64], slot t % 64.
 *   num_pages, page_table (DEVICE int32), page_table_stride
 *                describe the pool when page_size == 64; the stride must be
 *                >= ceil(max L_s / 64).  Page ids are checked on the device
 *                (FP2_STATUS_BAD_PAGE; such a page reads as zeros).
 *   q_seqlens, cu_q_seqlens   chunked prefill (Table 6's serving mode); both
 *                NULL for a full prefill.  q_seqlens HOST int32 [num_seqs]:
 *                Q_s new queries of sequence s, 1 <= Q_s <= seqlens[s], at
 *                positions seqlens[s] - Q_s .. seqlens[s] - 1; K and V hold all
 *                seqlens[s] tokens (the earlier ones and the chunk's).
 *                cu_q_seqlens DEVICE int32 [num_seqs + 1], their prefix sums
 *                (checked on the device).  q, o and lse then have Tq = sum Q_s
 *                tokens.  Blocks stay on the absolute position grid: query
 *                block i holds the chunk's queries in [iB, (i+1)B) and its mean
 *                covers only them; rows of query blocks below the chunk keep no
 *                block.  The e4m3 path takes a chunk too: fp2_quantize_fp8
 *                of q gives a query block the scale of its chunk positions.
 *                fp2_plan_kv8 returns FP2_ERR_UNSUPPORTED for a chunked
 *                problem.
 *   kv_head_begin, num_kv_heads_total   a slice of a layer's heads, run in
 *                place (the kv-head split of one layer across GPUs: each
 *                kv-head and its G query heads are planned and attended on
 *                their own).  num_kv_heads_total = 0 (or num_kv_heads, with
 *                kv_head_begin = 0): the tensors hold exactly the problem's
 *                heads.  Otherwise q, o are [T(q), G * num_kv_heads_total, d],
 *                k, v are [T, num_kv_heads_total, d] (or the paged pool
 *                [num_pages, 64, num_kv_heads_total, d]) and lse is
 *                [G * num_kv_heads_total, T(q)]; the call reads and writes only
 *                kv-heads kv_head_begin .. kv_head_begin + num_kv_heads - 1 and
 *                their query heads G * kv_head_begin .. (every other head of o,
 *                lse and of fp2_quantize_fp8's output is left untouched), with
 *                0 <= kv_head_begin and kv_head_begin + num_kv_heads <=
 *                num_kv_heads_total.  The plan and every per-(block, head)
 *                scale array (fp2_quantize_fp8, fp2_prefill, fp2_plan_kv8)
 *                cover the slice's heads only, numbered from 0.
 *   prev_kbar, prev_vbar   chunked prefill only (NULL otherwise, and both or
 *                neither): DEVICE float [num_blocks, num_kv_heads, d], 16-byte
 *                aligned, the K and V block means the caller already holds for
 *                the blocks that lie wholly before each sequence's chunk
 *                (blocks j with (j + 1) * block_size <= seqlens[s] - q_seqlens[s]),
 *                numbered like the plan's kbar / vbar of this problem (e.g. an
 *                earlier chunk's plan of a single sequence).  fp2_plan copies
 *                those blocks' means instead of reading their K and V again,
 *                so planning a chunk reads only the chunk's tokens; other
 *                entries are not read.  The float64 re-scoring of such blocks
 *                then uses these fp32 means.
 */
typedef struct fp2_problem {
    int32_t num_seqs;
    const int32_t* seqlens;
    const int32_t* cu_seqlens;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t block_size;
    double tau;
    int32_t page_size;
    int32_t num_pages;
    const int32_t* page_table;
    int32_t page_table_stride;
    const int32_t* q_seqlens;
    const int32_t* cu_q_seqlens;
    int32_t kv_head_begin;
    int32_t num_kv_heads_total;
    const float* prev_kbar;
    const float* prev_vbar;
} fp2_problem;

/*
 * Sizes and the layout of the plan buffer, all in bytes from its start
 * (every offset is 256-byte aligned).  Filled by fp2_plan_sizes.
 *
 *   row_ptr     int32 [num_rows + 1]      CSR row pointers.  Row r is the
 *               (sequence s, kv-head g, query block i) with
 *               r = g * num_blocks + (blocks of sequences before s) + i.
 *   col_idx     int32 [nnz_cap]           kept key-block ids, local to the
 *               sequence, ascending within a row (0 first, i last).
 *   kept_mask   uint32 [num_rows, mask_words]  bit j of row r set iff block j
 *               is kept (same information as the CSR row).
 *   kbar, vbar  float [num_blocks, Hkv, d] block means of K and V.
 *   kbar_bf16, vbar_bf16  the same means rounded to bfloat16 (operands of the
 *               correction's tensor-core products).
 *   kbar_e4m3, vbar_e4m3  uint8 [num_blocks, Hkv, d] e4m3 codes of the fp32
 *               means, with one scale per chunk of B consecutive blocks of a
 *               sequence (blocks B*c .. B*c+B-1, the pseudo-key tile of the
 *               FP8 correction) and kv-head: scale = absmax / 448 over the
 *               chunk (1 when all zero), code = e4m3_rne_sat(mean / scale).
 *   kbar_scale, vbar_scale float [num_blocks, Hkv]: the chunk scale, stored
 *               at the chunk's first block (other entries unused).
 *   kbar_e4m3_lo  uint8 [num_blocks, Hkv, d] e4m3 codes of the residual
 *               mean / scale - kbar_e4m3 (same chunk scale), so that
 *               kbar ~ scale * (kbar_e4m3 + kbar_e4m3_lo) to about 2^-8
 *               relative: the FP8 correction's pseudo-key logits use both
 *               terms (one e4m3 term alone, 2^-4, moves the LSE by ~2e-3).
 *   status      int32 [1] status word (FP2_STATUS_* bits), cleared by fp2_plan.
 *   (the rest is private to the library)
 */
typedef struct fp2_plan_layout {
    int64_t num_tokens;
    int64_t num_blocks;
    int64_t num_rows;
    int64_t nnz_cap;
    int32_t mask_words;
    int32_t max_blocks_per_seq;
    size_t off_row_ptr;
    size_t off_col_idx;
    size_t off_kept_mask;
    size_t off_kbar;
    size_t off_vbar;
    size_t off_kbar_bf16;
    size_t off_vbar_bf16;
    size_t off_kbar_e4m3;
    size_t off_vbar_e4m3;
    size_t off_kbar_scale;
    size_t off_vbar_scale;
    size_t off_status;
    size_t off_meta;
    size_t plan_bytes;        /* bytes the plan buffer must have      */
    size_t workspace_bytes;   /* bytes fp2_plan's scratch must have    */
    int64_t num_work_items;   /* fp2_prefill's work items (rows x splits x query-tile pairs) */
    int64_t num_split_slots;  /* row splits of the rows fp2_prefill splits (0: none)          */
    size_t off_kbar_e4m3_lo;
} fp2_plan_layout;

/* Library version (FP2_VERSION of the build). */
int fp2_version(void);

/* Static description of an error code; never NULL. */
const char* fp2_strerror(int code);

/*
 * Host-only: validates *problem (device pointers are not dereferenced) and
 * fills *layout.  The work schedule's split rule (fp2_prefill) depends on the
 * current device's SM count, read here (148 when no device is visible), so
 * call it with the device current that will run the plan.  nnz_cap is the dense count
 * Hkv * sum_s nb_s (nb_s + 1) / 2, so the CSR can never overflow.
 */
int fp2_plan_sizes(const fp2_problem* problem, fp2_plan_layout* layout);

/*
 * Stage 1, pattern discovery (Figure 3).  Reads bf16 q [T, Hq, d] and bf16
 * k, v (contiguous or paged, per problem->page_size) once, and writes into
 * `plan` (plan_bytes >= layout.plan_bytes) the CSR index, the kept-block
 * masks, the K/V block means (fp32, bf16 and e4m3 + scales) and a cleared
 * status word.  `workspace` (workspace_bytes >= layout.workspace_bytes,
 * device memory, 256-byte aligned) is scratch, free again once the enqueued
 * work completes.  Block lists are decided as if every score were computed in
 * float64: scores are computed on the tensor cores (tf32 MMAs of the means
 * rounded to tf32) and any block within that computation's error bound of the
 * threshold (or of the row maximum) is re-scored in float64.
 */
int fp2_plan(const fp2_problem* problem, const void* q, const void* k, const void* v,
             void* plan, size_t plan_bytes, void* workspace, size_t workspace_bytes,
             void* stream);

/*
 * Stage 1 from an FP8 KV cache: as fp2_plan, with K and V given as e4m3 codes
 * (same layout as the bf16 tensors, one byte per element, contiguous or paged)
 * and one fp32 scale per (block, kv-head) each, k_scale / v_scale [NB, Hkv]
 * indexed by the global block (the layout fp2_quantize_fp8 writes); Q stays
 * bf16.  The block means of K and V are the means of the dequantised values
 * code * scale (computed as scale * mean of the codes, in float64), so the plan
 * is the plan of the dequantised cache.  All pointers are device memory: q, k,
 * v 16-byte aligned, scales 4-byte aligned; ownership, workspace and errors as
 * for fp2_plan.
 */
int fp2_plan_kv8(const fp2_problem* problem, const void* q, const void* k_e4m3,
                 const void* v_e4m3, const float* k_scale, const float* v_scale, void* plan,
                 size_t plan_bytes, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Direct online FP8 quantisation (Table 1 footnote): for every (block, head)
 * of x, scale = absmax / 448 (1 for an all-zero block) and
 * x_e4m3 = round-to-nearest-even-saturating(x / scale), both in fp32.
 *   which = 0: x is q [T, Hq, d];  scales [num_blocks, Hq].
 *   which = 1 or 2: x is k or v in the problem's K/V layout (contiguous or
 *                   paged); x_e4m3 has the same layout; scales [num_blocks, Hkv].
 *                   In a paged pool only the slots of real tokens are written.
 * `plan` must come from fp2_plan on the same problem (it holds the block map).
 */
int fp2_quantize_fp8(const fp2_problem* problem, const void* plan, size_t plan_bytes,
                     const void* x, int32_t which, void* x_e4m3, float* scales, void* stream);

/*
 * fp2_quantize_fp8 of q, k and v in one launch (which = 0, 1, 2 in turn):
 * the same codes and scales as three fp2_quantize_fp8 calls, with one launch
 * instead of three (the launches dominate on short layers).  Arguments as for
 * fp2_quantize_fp8, one tensor, code tensor and scale array per input.
 */
int fp2_quantize_fp8_qkv(const fp2_problem* problem, const void* plan, size_t plan_bytes,
                         const void* q, const void* k, const void* v, void* q_e4m3,
                         void* k_e4m3, void* v_e4m3, float* q_scales, float* k_scales,
                         float* v_scales, void* stream);

/*
 * Stage 2, sparse attention with mean correction (Figure 3 / Figure 4).
 *   dtype FP2_DTYPE_BF16: q, k, v are the bf16 tensors given to fp2_plan and
 *     q_scale, k_scale, v_scale must be NULL.
 *   dtype FP2_DTYPE_E4M3: q, k, v are e4m3 tensors from fp2_quantize_fp8 and
 *     the three scale arrays are the ones it produced.
 *   o    DEVICE bf16 [T, Hq, d]   attention output.
 *   lse  DEVICE float [Hq, T]     natural-log softmax denominator.
 *   flags  FP2_NO_CORRECTION and FP2_DEBUG_* bits.
 * Work is spread over one persistent CTA per SM.  A work item is two 128-row
 * PackGQA query tiles of one row (kv-head g, query block i); fp2_plan lists
 * the items longest row first within chunks of kv-heads whose K and V fit
 * together in L2, and CTA c takes the c-th item of each pass over the grid
 * (from the other end on odd passes, when there are at most 16 passes).  KV
 * splitting (Table 7, "count-balanced CSR splits"): when the longest row's
 * tile bound i + 1 + ceil(i / B) exceeds both 32 and the layer's mean tiles
 * per CTA (one CTA per SM of the current device; 148 when no device is visible), every row whose bound exceeds half that mean (and
 * at least 8) is cut into
 * splits of equal numbers of its tiles (kept blocks in CSR order, then pseudo
 * tiles); each split writes its normalised fp32 O and log-sum-exp into the
 * plan's private scratch, and a merge kernel combines them by log-sum-exp into
 * o and lse.  Because fp2_prefill writes that scratch, two fp2_prefill calls
 * on one plan must not overlap on the GPU (order them on one stream).
 */
int fp2_prefill(const fp2_problem* problem, const void* plan, size_t plan_bytes,
                const void* q, const void* k, const void* v,
                const float* q_scale, const float* k_scale, const float* v_scale,
                int32_t dtype, void* o, float* lse, uint32_t flags, void* stream);

/*
 * fp2_plan_static -- the same stage 1 as fp2_plan, for callers that cannot
 * allocate device memory for a workspace (for example a serving process
 * whose KV-cache pool or caching allocator already holds the device
 * memory, or a host that only receives device pointers from another
 * runtime and has no allocator of its own).  The paper has no counterpart:
 * this is an interface convenience of this library.
 *
 * The scratch lives in one fixed array of FP2_STATIC_WORKSPACE_BYTES (32 MiB)
 * inside the library's device image, which every device that loads the
 * library holds until the process exits.  Problems whose
 * layout.workspace_bytes exceed it are rejected with FP2_ERR_CAPACITY; it
 * covers, e.g., one 32K-token layer with 32 query / 8 kv heads of dim 128 and
 * block 128 (about 16.8 MB of scratch), not a 64K-token one of that shape.
 * The call allocates and frees nothing.  Every call looks up the array's
 * device address in the current device's context (cudaGetSymbolAddress, with
 * the device the caller made current), so a reset or re-created context is
 * followed; the first lookup on a device loads the library's device code
 * there, so make the first call on each device before any stream capture.
 * Every call shares the one array and leaves the last call's scratch in it
 * (no entry needs to start at zero), so calls whose work overlaps on the GPU
 * -- on two streams, or from two threads -- race; order them on one stream.
 * Arguments, outputs and errors are otherwise those of fp2_plan.
 */
#define FP2_STATIC_WORKSPACE_BYTES ((size_t)32 << 20)
int fp2_plan_static(const fp2_problem* problem, const void* q, const void* k, const void* v,
                    void* plan, size_t plan_bytes, void* stream);

/*
 * Synchronises `stream`, then reads the plan's status word into
 * *device_status (may be NULL).  Returns FP2_OK when it is zero,
 * FP2_ERR_TIMEOUT when FP2_STATUS_TIMEOUT is set, otherwise
 * FP2_ERR_DEVICE_CHECK; FP2_ERR_CUDA when the synchronisation itself fails.
 */
int fp2_status_check(const void* plan, size_t plan_bytes, void* stream, int32_t* device_status);

#ifdef __cplusplus
}
#endif

#endif /* FP2_H_ */
