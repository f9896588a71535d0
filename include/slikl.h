/*
 * slikl.h — C ABI of the B200 (sm_100a) sparse Lightning Indexer KL-loss backward.
 *
 * The operation is the one defined by aclnnSparseLightningIndexerKLLossGrad (Ascend
 * CANN operator documentation, section "计算公式"). For each query token t:
 *
 *   S_t   = q_t . K_topk(t)^T          K_topk(t) = key rows named by sparse_indices[t]
 *   I_t   = W_t . ReLU(S_t)            W = w
 *   y_t   = Softmax(I_t)               over the valid slots; written to softmax_out
 *   dI_t  = y_t - p_t                  p = attn_softmax_l1norm
 *   dW_t  = dI_t . ReLU(S_t)^T         -> dw
 *   dS_t  = dI_t * W_t * 1[S_t > 0]    (chain rule on I_t = W_t . ReLU(S_t))
 *   dq_t  = dS_t . K_topk(t)           -> dq
 *   dK_topk(t) = dS_t^T . q_t          scatter-added into the key rows -> dk
 *
 * Invalid top-k slots hold -1 and take no part in any of these sums (same section):
 * softmax_out is exactly 0 there and nothing is added for them. A token with no valid
 * slot gets softmax_out = 0 and zero dq/dw. Key rows that no valid slot names get dk = +0.
 *
 * The call sequence follows the page's two-phase interface (section "函数原型": first
 * "...GetWorkspaceSize", which validates the parameters and returns the workspace size,
 * then the asynchronous launch on a stream): slikl_grad_workspace_size(), then slikl_grad().
 *
 * Conventions for every entry point
 *   - Ownership: the caller allocates every tensor and the workspace. The library
 *     allocates no memory and keeps no state between calls (slikl_grad_noalloc, for
 *     callers that cannot allocate, uses a fixed device array of the library instead).
 *   - Pointers named "device" are CUDA device pointers on the current device; tensors are
 *     dense and contiguous in the layouts stated below.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Launch-phase calls are
 *     asynchronous: they return after queueing work on `stream`.
 *   - Return codes mirror the aclnn convention (161001 parameter null pointer, 161002
 *     parameter invalid, 561103 inner null pointer), plus two codes of this library.
 */
#ifndef SLIKL_H
#define SLIKL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Entry points are the only symbols the shared library exports. */
#if defined(__GNUC__)
#define SLIKL_API __attribute__((visibility("default")))
#else
#define SLIKL_API
#endif

typedef int32_t slikl_status;

#define SLIKL_OK                      0
#define SLIKL_ERR_PARAM_NULLPTR       161001  /* a required pointer argument is NULL          */
#define SLIKL_ERR_PARAM_INVALID       161002  /* dtype, layout, shape or attribute not supported */
#define SLIKL_ERR_WORKSPACE_TOO_SMALL 161003  /* workspace_bytes below slikl_grad_workspace_size */
#define SLIKL_ERR_INNER_NULLPTR       561103  /* the size/flags output pointer is NULL         */
#define SLIKL_ERR_CUDA                561001  /* a CUDA runtime call or kernel launch failed   */

/* dtype of q, k, dq, dk ("公共约束": the four share one dtype, FLOAT16 or BFLOAT16). */
#define SLIKL_FP16 0
#define SLIKL_BF16 1

/* layoutQ / layoutK ("公共约束": BSND or TND; TND needs cuSeqLens of that side). */
#define SLIKL_BSND 0
#define SLIKL_TND  1

/*
 * Problem description (host memory).
 *
 *   layout_q = BSND: q [B,S1,N1,D], w/dw [B,S1,N1], sparse_indices, attn_softmax_l1norm and
 *                    softmax_out [B,S1,1,topk]; requires B > 0 and S1 > 0; T1 is ignored
 *                    (taken as B*S1).
 *   layout_q = TND:  q [T1,N1,D], w/dw [T1,N1], the three top-k tensors [T1,1,topk];
 *                    cu_seqlens_q [B+1] on the device with cu_seqlens_q[0] = 0 and
 *                    cu_seqlens_q[B] = T1; S1 is ignored.
 *   layout_k = BSND: k/dk [B,S2,1,D], requires S2 > 0; T2 is ignored (taken as B*S2).
 *   layout_k = TND:  k/dk [T2,1,D], cu_seqlens_k [B+1] on the device, cu_seqlens_k[B] = T2;
 *                    S2 > 0 promises that no batch has more than S2 key rows (it lets the
 *                    key-major dK path size its records; 0 = no promise, that path is off).
 *
 * The key tensor has one head (N2 = 1): the page's formulas carry no key-head index.
 * Valid indices of a batch-b token are local to batch b's key range: key row =
 * (BSND) b*S2 + index, (TND) cu_seqlens_k[b] + index, and must lie in [0, len_k(b)).
 *
 * Supported set: N1 in [1, 128]; D in {64, 128}; topk in [1, 8192]; B >= 1;
 * T1*topk < 2^31; T2 < 2^31. deterministic: 0 = dk by fp32 atomic adds (the page's default,
 * section "确定性计算"), 1 = bitwise reproducible dk by a fixed-order reduction.
 */
typedef struct {
    int32_t dtype;           /* SLIKL_FP16 or SLIKL_BF16 */
    int32_t layout_q;        /* SLIKL_BSND or SLIKL_TND */
    int32_t layout_k;        /* SLIKL_BSND or SLIKL_TND */
    int32_t deterministic;   /* 0 or 1 */
    int64_t B;               /* batches (TND: number of sequences = len(cu_seqlens) - 1) */
    int64_t S1, S2;          /* BSND query / key lengths; TND keys: S2 = longest key range or 0 */
    int64_t T1, T2;          /* TND total query / key rows */
    int64_t N1, D, topk;     /* query heads, head dim, top-k slots per token */
} slikl_problem;

/* Tensors of one call. All DEVICE pointers, caller-owned, contiguous; q, k, dq, dk 16-byte
 * aligned, the others 4-byte aligned (SLIKL_ERR_PARAM_INVALID otherwise). A tensor with no
 * elements may be NULL: with TND queries and T1 = 0, q, w, attn_softmax_l1norm,
 * sparse_indices, dq, dw and softmax_out; with TND keys and T2 = 0, k and dk. */
typedef struct {
    const void *q;                      /* dtype  [B,S1,N1,D] / [T1,N1,D]            */
    const void *k;                      /* dtype  [B,S2,1,D]  / [T2,1,D]             */
    const float *w;                     /* fp32   [B,S1,N1]   / [T1,N1]              */
    const float *attn_softmax_l1norm;   /* fp32   [.., 1, topk] target distribution p  */
    const int32_t *sparse_indices;      /* int32  [.., 1, topk], -1 = invalid slot     */
    const int32_t *cu_seqlens_q;        /* int32  [B+1], TND query side only, else NULL */
    const int32_t *cu_seqlens_k;        /* int32  [B+1], TND key side only, else NULL   */
    void *dq;                           /* out dtype  same shape as q                  */
    void *dk;                           /* out dtype  same shape as k                  */
    float *dw;                          /* out fp32   same shape as w                  */
    float *softmax_out;                 /* out fp32   same shape as sparse_indices     */
} slikl_tensors;

/*
 * Phase 1 (host only, no CUDA call). Validates `problem` and writes the workspace size in
 * bytes that slikl_grad needs.
 * Errors: SLIKL_ERR_INNER_NULLPTR if workspace_bytes is NULL; SLIKL_ERR_PARAM_NULLPTR if
 * problem is NULL; SLIKL_ERR_PARAM_INVALID for any value outside the supported set.
 */
SLIKL_API slikl_status slikl_grad_workspace_size(const slikl_problem *problem, size_t *workspace_bytes);

/*
 * Phase 2. Re-validates, then queues on `stream`: zeroing of the status word and of the
 * fp32 dk accumulator, the work-split kernel, the fused per-token kernel, the dK stage of the
 * chosen path (below) and the dk cast.
 * Writes dq, dk, dw and softmax_out in full.
 * `workspace` (device, >= the phase-1 size, 256-byte aligned) is scratch owned by the
 * caller for the duration of the call; its first 256 bytes hold the device status word
 * read by slikl_read_device_status().
 * Errors: SLIKL_ERR_PARAM_NULLPTR (problem, tensors, a required tensor pointer or
 * workspace is NULL; cu_seqlens of a TND side is NULL), SLIKL_ERR_PARAM_INVALID,
 * SLIKL_ERR_WORKSPACE_TOO_SMALL, SLIKL_ERR_CUDA (launch failure or no usable sm_100 device).
 * Problems that only the device can see (an index outside its batch's key range, malformed
 * cu_seqlens) never fault: the slot is treated as invalid and a bit is set in the status word.
 */
SLIKL_API slikl_status slikl_grad(const slikl_problem *problem, const slikl_tensors *tensors,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * dK paths (slikl_options.dk_path). Both give dK to within the input type's rounding: the
 * scatter path multiplies q by dS = dI w [S > 0] rounded to the input type, the key-major path
 * multiplies w q rounded to the input type by dI [S > 0] rounded to it; the fp32 additions run
 * in different orders.
 *   SLIKL_DK_SCATTER   every named slot adds its dK row into an fp32 accumulator with
 *                      atomic adds (the page's default), or, deterministic = 1, stores it for
 *                      a sort by key and a fixed-order reduction;
 *   SLIKL_DK_KEYMAJOR  the fused kernel stores, per named (query row, key), dI and the heads
 *                      with S > 0; a second tensor-core kernel then forms dK one 256-key block
 *                      at a time from every query row that names a key of the block.
 *                      Needs a key-range bound (BSND: S2; TND: problem->S2 > 0) of at most
 *                      16384 keys; its workspace holds T1 x roundup(S2, 256) records of 8
 *                      (N1 <= 32), 16 (N1 <= 64; also N1 <= 32 with deterministic = 1) or 32
 *                      bytes, and the w-scaled copy of q (T1 x N1 x D of the input type). With deterministic = 1 repeated slots of a key sum their dI as
 *                      64-bit fixed-point integers and every key row is summed in a fixed
 *                      order, so the result is bitwise repeatable.
 *   SLIKL_DK_AUTO      the key-major path when it is possible, the key range is at most 16x
 *                      topk and its records take at most 8 GiB; else the scatter path.
 * The workspace size depends on the path: size and launch with the same options.
 */
#define SLIKL_DK_AUTO     0
#define SLIKL_DK_SCATTER  1
#define SLIKL_DK_KEYMAJOR 2

typedef struct {
    int32_t dk_path;     /* SLIKL_DK_AUTO, SLIKL_DK_SCATTER or SLIKL_DK_KEYMAJOR */
    void *fused_begin;   /* optional cudaEvent_t recorded just before the fused kernel, or NULL */
    void *fused_end;     /* optional cudaEvent_t recorded just after it, or NULL */
    void *dk_begin;      /* optional cudaEvent_t recorded before the dK stage that follows the
                            fused kernel (w-scaled q, key-major kernel and cast, the cast alone,
                            or the deterministic reduction), or NULL */
    void *dk_end;        /* optional cudaEvent_t recorded after that stage, or NULL */
    float *loss;         /* optional DEVICE output, fp32 [T1] (4-byte aligned), or NULL: the KL
                            loss per query row, L_t = sum over valid slots with p > 0 of
                            p log(p / y) (section "计算公式"), from the softmax_out of this
                            call; 0 for a row without a valid slot */
    const int32_t *seq_used_q;  /* optional DEVICE input, int32 [B] (4-byte aligned), or NULL:
                            the query rows of batch b in use (seqUsedQOptional of
                            aclnnSparseLightningIndexerKLLossGrad; the page fixes only its
                            type). Rows of batch b at local position >= seq_used_q[b] are
                            padding: their indices are not read, softmax_out / dq / dw are 0
                            there and they add nothing to dk. NULL = every row in use. */
    const int32_t *seq_used_k;  /* optional DEVICE input, int32 [B] (4-byte aligned), or NULL:
                            the key rows of batch b in use (seqUsedKOptional). A slot naming a
                            key at local position >= seq_used_k[b] (and < the batch's key
                            count) is invalid, like -1, without a status flag; dk rows of
                            unused keys stay 0. NULL = every key in use.
                            A value outside [0, the batch's row count] sets
                            SLIKL_DEV_BAD_SEQ_USED and is clamped into that range. */
} slikl_options;

/*
 * slikl_grad_workspace_size / slikl_grad with options (NULL options = SLIKL_DK_AUTO, no
 * events; slikl_grad_workspace_size and slikl_grad are these calls with NULL options).
 * Errors: as the plain calls; SLIKL_ERR_PARAM_INVALID also for an unknown dk_path or
 * SLIKL_DK_KEYMAJOR on a problem that path cannot run.
 */
SLIKL_API slikl_status slikl_grad_workspace_size_ex(const slikl_problem *problem,
                                                    const slikl_options *options,
                                                    size_t *workspace_bytes);
SLIKL_API slikl_status slikl_grad_ex(const slikl_problem *problem, const slikl_tensors *tensors,
                                     void *workspace, size_t workspace_bytes, void *stream,
                                     const slikl_options *options);

/*
 * The dK path slikl_grad_ex would take for `problem` with `options` (NULL = SLIKL_DK_AUTO):
 * writes SLIKL_DK_SCATTER or SLIKL_DK_KEYMAJOR to *path. Host only, no CUDA call.
 * Errors: SLIKL_ERR_INNER_NULLPTR (path NULL) and those of slikl_grad_workspace_size_ex.
 */
SLIKL_API slikl_status slikl_grad_dk_path(const slikl_problem *problem,
                                          const slikl_options *options, int32_t *path);

/*
 * slikl_grad with a measurement aid: when fused_begin / fused_end are not NULL they are
 * cudaEvent_t handles (created by the caller) recorded on `stream` immediately before and
 * after the fused per-token kernel, so its duration can be read with cudaEventElapsedTime.
 * Everything else, including errors, is as slikl_grad (which is this call with NULL events);
 * the same as slikl_grad_ex with SLIKL_DK_AUTO and these events.
 */
SLIKL_API slikl_status slikl_grad_with_events(const slikl_problem *problem,
                                              const slikl_tensors *tensors, void *workspace,
                                              size_t workspace_bytes, void *stream,
                                              void *fused_begin, void *fused_end);

/* Device status bits (see slikl_read_device_status). */
#define SLIKL_DEV_INDEX_OUT_OF_RANGE  0x1u  /* an index of a row in use was >= len_k(b) or < -1
                                               (len_k(b): the batch's key count, used or not) */
#define SLIKL_DEV_BAD_CU_SEQLENS_Q    0x2u  /* cu_seqlens_q not 0..T1 non-decreasing           */
#define SLIKL_DEV_BAD_CU_SEQLENS_K    0x4u  /* cu_seqlens_k not 0..T2 non-decreasing; the key
                                               ranges of the batches were emptied            */
#define SLIKL_DEV_WAIT_TIMEOUT        0x8u  /* an internal bounded wait gave up; outputs invalid */
#define SLIKL_DEV_KEY_RANGE_ABOVE_S2  0x10u /* key-major dK path: a batch holds more key rows
                                               than problem->S2 promised (TND); the rows of
                                               that batch are left out, outputs invalid    */
#define SLIKL_DEV_BAD_SEQ_USED        0x20u /* a seq_used_q / seq_used_k entry was outside
                                               [0, the batch's row count]; it was clamped  */

/*
 * Copies the status word of the last slikl_grad call that used `workspace` (device) into
 * *flags (host) after synchronising `stream`. Bits are the SLIKL_DEV_* values above.
 * Errors: SLIKL_ERR_PARAM_NULLPTR (workspace NULL), SLIKL_ERR_INNER_NULLPTR (flags NULL),
 * SLIKL_ERR_CUDA.
 */
SLIKL_API slikl_status slikl_read_device_status(const void *workspace, void *stream, uint32_t *flags);

/*
 * Work split ("metadata"), the analogue of DenseLightningIndexerKLLossGradMetadata (article
 * on that AICPU operator, sections "功能定位" and "Metadata 输出布局"): the merged B*S1 query
 * rows are split into contiguous ranges, one per worker (CTA) of the fused kernel.
 * slikl_grad runs the same kernel into its workspace; this entry point exposes it.
 *
 * metadata (device, int32, slikl_grad_metadata_size(num_workers) entries) receives:
 *   [0] totalSize      merged query rows T1
 *   [1] formerCoreSize ceil(T1 / num_workers)
 *   [2] remainCoreSize formerCoreSize - 1 (0 if T1 == 0)
 *   [3] remainCoreNum  workers that take remainCoreSize rows in the row-count split
 *   [4] usedCoreNum    min(num_workers, T1)
 *   [5] maxSeqK        longest key range of a batch
 *   [6] mode           0 = row-count split (the page's), 1 = cost-weighted split
 *   [7] num_workers
 *   [8 + 2c], [9 + 2c] first and one-past-last query row of worker c.
 * Fields 0..5 follow the page's layout; the page's fixed 64-entry size is not kept, since
 * the ranges of every worker are stored. In mode 1 the ranges balance
 * cost(t) = 1 + (number of 128-slot tiles of row t holding an index >= 0).
 * `tensors` needs sparse_indices and, for TND sides, cu_seqlens_q/k; other fields ignored.
 * `workspace` (device, >= slikl_grad_metadata_workspace_size bytes) is scratch.
 * Errors: as slikl_grad; SLIKL_ERR_PARAM_INVALID if num_workers is not in [1, 4096] or
 * mode is not 0/1.
 */
SLIKL_API int64_t slikl_grad_metadata_size(int32_t num_workers);
SLIKL_API slikl_status slikl_grad_metadata_workspace_size(const slikl_problem *problem,
                                                size_t *workspace_bytes);
SLIKL_API slikl_status slikl_grad_metadata(const slikl_problem *problem, const slikl_tensors *tensors,
                                 int32_t num_workers, int32_t mode, int32_t *metadata,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * slikl_grad for callers that cannot allocate device memory when they call (code that runs
 * under an allocator which forbids cudaMalloc, or that has no way to reach its framework's
 * allocator). Nothing is allocated per call: the scratch that slikl_grad takes as
 * `workspace` is a fixed array of SLIKL_NOALLOC_SCRATCH_BYTES in the library's device code,
 * which every GPU that loads the library keeps until the process exits. The operator pages
 * have no counterpart of this call; it is an addition of this library.
 *
 * `problem`, `tensors` and `stream` are as for slikl_grad; the caller still owns every input
 * and output tensor. The first call on each device looks up the array's device address
 * (make that first call outside any stream capture). All calls share the array: calls whose
 * GPU work overlaps (unordered streams) race and give wrong results.
 * Errors: as slikl_grad; SLIKL_ERR_WORKSPACE_TOO_SMALL if the problem needs more scratch than
 * SLIKL_NOALLOC_SCRATCH_BYTES; slikl_grad_workspace_size_ex with options.dk_path =
 * SLIKL_DK_SCATTER (the path this call takes) tells how much it needs;
 * SLIKL_ERR_PARAM_INVALID for deterministic = 1, whose per-slot scratch does not fit.
 */
#define SLIKL_NOALLOC_SCRATCH_BYTES (32u << 20)
SLIKL_API slikl_status slikl_grad_noalloc(const slikl_problem *problem,
                                          const slikl_tensors *tensors, void *stream);

/*
 * Dense variant (DenseLightningIndexerKLLossGrad). The article on that operator's metadata
 * generator (sections 功能定位, 第一段接口参数说明 and 特殊约束) names the operator and its
 * interface: one key head, layouts BSND / TND, maskMode 0 (no mask) or 3 (rightDownCausal, the
 * lower triangle anchored at the bottom-right vertex), cmpRatio 1 for uncompressed keys. The
 * pages print no formula of its own. This library reads it as the formulas at the top of this
 * header, with the top-k slots of a query replaced by every key of its batch that the mask
 * leaves visible; slot j of a row is key j, local to the batch:
 *   mask_mode 0: all klen keys of the batch;
 *   mask_mode 3: query s (0-based, of qlen queries) sees keys 0 .. s + (klen - qlen), none when
 *                that bound is negative.
 * With options->seq_used_q / seq_used_k the used lengths stand for qlen / klen; rows past a
 * batch's used queries are padding (outputs 0).
 *
 * attn_softmax_l1norm and softmax_out are [B,S1,1,Ld] (BSND) / [T1,1,Ld] (TND) with
 * Ld = row_len slots per row; slots past a row's visible keys are invalid (p there is ignored,
 * softmax_out is exactly 0). q, k, w, dq, dk, dw and cu_seqlens are as in slikl_tensors.
 * The call runs the sparse operator's kernels on index rows 0, 1, .., L_t - 1 (then -1) that a
 * device kernel writes into the workspace, so every dK path and option of slikl_grad_ex
 * applies (options->loss included).
 */
typedef struct {
    int32_t dtype;           /* SLIKL_FP16 or SLIKL_BF16 */
    int32_t layout_q;        /* SLIKL_BSND or SLIKL_TND */
    int32_t layout_k;        /* SLIKL_BSND or SLIKL_TND */
    int32_t deterministic;   /* 0 or 1 */
    int64_t B, S1, S2;       /* as in slikl_problem (TND keys: S2 = 0 or a key-range bound) */
    int64_t T1, T2;          /* TND total query / key rows */
    int64_t N1, D;           /* query heads, head dim */
    int64_t row_len;         /* Ld, slots per row, in [1, 8192]; 0 = S2 (BSND keys only). Must
                                cover the longest key range in use; keys of a batch past it are
                                left out and SLIKL_DEV_ROW_LEN_BELOW_KEYS is set */
    int32_t mask_mode;       /* 0 or 3 */
    int32_t reserved;        /* must be 0 */
} slikl_dense_problem;

typedef struct {
    const void *q;                      /* dtype  [B,S1,N1,D] / [T1,N1,D]             */
    const void *k;                      /* dtype  [B,S2,1,D]  / [T2,1,D]              */
    const float *w;                     /* fp32   [B,S1,N1]   / [T1,N1]               */
    const float *attn_softmax_l1norm;   /* fp32   [.., 1, Ld] target distribution p    */
    const int32_t *cu_seqlens_q;        /* int32  [B+1], TND query side only, else NULL */
    const int32_t *cu_seqlens_k;        /* int32  [B+1], TND key side only, else NULL   */
    void *dq;                           /* out dtype  same shape as q                   */
    void *dk;                           /* out dtype  same shape as k                   */
    float *dw;                          /* out fp32   same shape as w                   */
    float *softmax_out;                 /* out fp32   [.., 1, Ld]                       */
} slikl_dense_tensors;

#define SLIKL_DEV_ROW_LEN_BELOW_KEYS  0x40u /* dense variant: a batch holds more keys than
                                               row_len; the keys past it were left out  */

/*
 * Two-phase dense call, the same contract as slikl_grad_workspace_size_ex / slikl_grad_ex
 * (options may be NULL). Errors: as those calls; SLIKL_ERR_PARAM_INVALID also for mask_mode
 * not 0 or 3, reserved != 0, row_len outside [1, 8192] (after 0 -> S2), or row_len < S2 with
 * BSND keys.
 */
SLIKL_API slikl_status slikl_dense_grad_workspace_size(const slikl_dense_problem *problem,
                                                       const slikl_options *options,
                                                       size_t *workspace_bytes);
SLIKL_API slikl_status slikl_dense_grad(const slikl_dense_problem *problem,
                                        const slikl_dense_tensors *tensors, void *workspace,
                                        size_t workspace_bytes, void *stream,
                                        const slikl_options *options);

/*
 * The dK path slikl_dense_grad would take for `problem` with `options` (NULL = SLIKL_DK_AUTO):
 * writes SLIKL_DK_SCATTER or SLIKL_DK_KEYMAJOR to *path. Host only, no CUDA call.
 * Errors: SLIKL_ERR_INNER_NULLPTR (path NULL) and those of slikl_dense_grad_workspace_size.
 */
SLIKL_API slikl_status slikl_dense_grad_dk_path(const slikl_dense_problem *problem,
                                                const slikl_options *options, int32_t *path);

/*
 * ---------------------------------------------------------------------------------------
 * The older fused variant: p formed from the main attention
 * (aclnnSparseLightningIndexerKLLossGrad, sections 功能说明 and 计算公式: the older operator,
 * SparseLightningIndexerGradKLLoss, computed attn_softmax_l1norm inside its kernel from the
 * main attention's scores, summed over the heads and L1-normalised, and output the loss).
 * The pages give none of that operator's inputs; the reading taken here:
 *   - a main-attention query q_main with Nm heads of Dm, laid out like q
 *     (BSND [B][S1][Nm][Dm] or TND [T1][Nm][Dm]), and one main-attention key head k_main on
 *     the same key rows as k (BSND [B][S2][1][Dm] or TND [T2][1][Dm]), both of problem->dtype;
 *   - for query row t and head h, A_h(t, j) = softmax over the row's valid slots j of
 *     scale * q_main[t, h] . k_main[key(t, j)] (the keys a sparse main attention attends to;
 *     valid slots as for the sparse operator, used lengths included);
 *   - p(t, j) = sum_h A_h(t, j) / sum_j sum_h A_h(t, j) = sum_h A_h(t, j) / Nm, 0 at invalid
 *     slots and on rows without a valid slot.
 * The backward then runs on that p exactly as slikl_grad_ex; options->loss returns the
 * per-row KL loss the older operator output.
 * ---------------------------------------------------------------------------------------
 */
typedef struct slikl_main_attention {
    int32_t Nm;                 /* main-attention query heads, 1..128 */
    int32_t Dm;                 /* their head dimension: 64 or 128 */
    float scale;                /* softmax scale of the main attention (e.g. 1 / sqrt(Dm)) */
    int32_t reserved;           /* 0 */
} slikl_main_attention;

/*
 * Phase 1 (host only, no CUDA call): the workspace size of slikl_grad_recompute_p, equal to
 * slikl_grad_workspace_size_ex for the same problem and options.
 * Errors: SLIKL_ERR_PARAM_NULLPTR (main NULL), SLIKL_ERR_PARAM_INVALID (Nm outside 1..128,
 * Dm not 64 or 128, scale not finite, reserved != 0), and those of
 * slikl_grad_workspace_size_ex.
 */
SLIKL_API slikl_status slikl_grad_recompute_p_workspace_size(const slikl_problem *problem,
                                                             const slikl_main_attention *main,
                                                             const slikl_options *options,
                                                             size_t *workspace_bytes);
/*
 * Phase 2: forms p from q_main and k_main (device, 16-byte aligned, layouts above) into
 * p_out (device fp32 [T1][topk], 4-byte aligned, written in full), then runs the backward
 * of slikl_grad_ex with it; tensors->attn_softmax_l1norm is not read. Same streams,
 * workspace and status-word rules as slikl_grad_ex.
 * Errors: as phase 1; SLIKL_ERR_PARAM_NULLPTR for NULL tensors, q_main or p_out (when there
 * are query rows) or k_main (when there are key rows); SLIKL_ERR_PARAM_INVALID for a
 * misaligned q_main, k_main or p_out; and those of slikl_grad_ex.
 */
SLIKL_API slikl_status slikl_grad_recompute_p(const slikl_problem *problem,
                                              const slikl_main_attention *main,
                                              const slikl_tensors *tensors, const void *q_main,
                                              const void *k_main, float *p_out, void *workspace,
                                              size_t workspace_bytes, void *stream,
                                              const slikl_options *options);

/* Human-readable name of a status code (static string, never NULL). */
SLIKL_API const char *slikl_status_string(slikl_status status);

#ifdef __cplusplus
}
#endif

#endif /* SLIKL_H */
