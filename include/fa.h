/*
 * fa.h -- C ABI of the B200 (sm_100a) fused scaled-dot-product attention
 * forward.
 *
 * The operation (page 1, "CANN ops-transformer FlashAttentionScore", section
 * 平方级显存的精确来源, and page 2, "FlashAttention on Ascend via
 * ops-transformer", section 标准 vs IO-Aware 实现):
 *
 *     S = scale * Q K^T        (masked entries -> -inf when causal)
 *     P = softmax(S)           (row-wise)
 *     O = P V
 *     LSE[i] = log(sum_j exp(S[i, j]))   (natural log of the scaled scores)
 *
 * computed tile by tile with the online softmax (page 1, sections 分块 Tiling
 * 的计算骨架 and 在线 Softmax 的数学原理拆解; page 3, "ops-nn efficient
 * attention for AIGC", section 2.2), so that the Nq x Nkv score matrix never
 * reaches device memory.  The argument list follows page 2's
 * flash_attention_score (scale_value, input_layout in {BSND, ...},
 * pre_tokens/next_tokens for causal) and page 3's Config (softmax_scale = -1
 * meaning 1/sqrt(d), causal flag).
 *
 * All entry points are plain C: pointers, sizes, ints.  No function throws,
 * traps or aborts; every failure is a return code.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Memory layouts of q, k, v and o (page 2: input_layout; page 3: [B, H, N, D]).
 *   FA_LAYOUT_BHND: element (b, h, n, c) at ((b*H + h)*N + n)*d + c
 *   FA_LAYOUT_BSND: element (b, n, h, c) at ((b*N + n)*H + h)*d + c
 * with N = Nq for q and o, N = Nkv for k and v.  Tensors are dense. */
typedef enum { FA_LAYOUT_BHND = 0, FA_LAYOUT_BSND = 1 } fa_layout_t;

/* Storage type of q, k, v and o.  BF16 and FP16 run on the tcgen05 tensor-core
 * kernel (fp32 accumulation, P rounded to the input type before P V).  FP32
 * runs on an exact-fp32 CUDA-core kernel.  LSE is always fp32. */
typedef enum { FA_DTYPE_BF16 = 0, FA_DTYPE_FP16 = 1, FA_DTYPE_FP32 = 2 } fa_dtype_t;

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad enum, Nkv == 0 with Nq > 0 */
  FA_ERR_UNSUPPORTED = 2,  /* head dim not supported by the entry point, or a size beyond the index range */
  FA_ERR_MISALIGNED = 3,   /* q, k, v, o not 16-byte aligned, or lse not 4-byte aligned */
  FA_ERR_LAUNCH = 4,       /* the CUDA launch or tensor-map creation failed */
  FA_ERR_TIMEOUT = 5,      /* a bounded device-side wait expired (see fa_get_device_status) */
  FA_ERR_NO_DEVICE = 6,    /* no usable sm_100 device for the current context */
  FA_ERR_TOO_LARGE = 7,    /* fa_fwd_noalloc only: the call needs more than its fixed scratch */
  FA_ERR_CHECK = 8         /* debug builds (FA_CHECKS) only: a kernel found a computed index out of
                              bounds and skipped that access (see fa_get_device_status) */
} fa_status_t;

/*
 * fa_fwd -- O = softmax(scale * Q K^T [+ causal mask]) V and LSE.
 *
 *   q      [B,H,Nq,d] or [B,Nq,H,d] (layout), device memory, read only
 *   k, v   [B,H,Nkv,d] or [B,Nkv,H,d], device memory, read only
 *   o      same shape, layout and dtype as q, device memory, written
 *   lse    [B,H,Nq] fp32 device memory (head-major whatever the layout),
 *          written; may be NULL, in which case no LSE is written
 *   d      head dimension, 64, 128 or 256 (256: bf16/fp16 only; page 1,
 *          section 分块 Tiling 的计算骨架, gives head dims of 64-256)
 *   scale  softmax scale; scale <= 0 or NaN selects 1/sqrt(d)
 *   causal 0 or 1.  Causal masking is top-left aligned: query row i sees key j
 *          iff j <= i (page 3, section 6.1: triu(ones(Nq, Nkv), diagonal=1)
 *          is masked).  Every row therefore sees key 0.
 *   layout fa_layout_t, shared by q, k, v and o
 *   dtype  fa_dtype_t, shared by q, k, v and o
 *   stream a cudaStream_t (NULL = the legacy default stream)
 *
 * Ownership: every buffer belongs to the caller and must stay alive until the
 * stream has finished the call.  The library keeps no pointer after return.
 * On its first call on a device it allocates 8 KB of device memory for the
 * tile scheduler's per-launch work counters (kept until the process exits;
 * make that first call outside any stream capture); later calls allocate
 * nothing.  The call is asynchronous: it validates, encodes TMA descriptors
 * on the host and launches one kernel on `stream`.  (Head dim 64 with
 * Nkv <= 128 runs a dependent launch: the kernel may start while the
 * previous work on the stream drains, and waits for it before touching any
 * memory.)
 *
 * Returns FA_OK (also for B*H*Nq == 0, a no-op), or FA_ERR_INVALID_ARG /
 * FA_ERR_UNSUPPORTED / FA_ERR_MISALIGNED before anything is launched, or
 * FA_ERR_LAUNCH / FA_ERR_NO_DEVICE.  Device-side failures (a bounded wait that
 * expired) are reported later by fa_get_device_status().
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int64_t B, int64_t H, int64_t Nq, int64_t Nkv, int64_t d,
           float scale, int causal, int layout, int dtype, void* stream);

/*
 * fa_fwd_gqa -- fa_fwd for grouped-query (and multi-query) attention: k and v
 * hold Hkv heads, fewer than q's H (page 1, "CANN ops-transformer
 * FlashAttentionScore", section GatherPAKVCache 的显存管理逻辑: under GQA/MQA
 * the K/V head count is below the query head count and the needed K/V head
 * is selected; page 3, section 7.3 names GQA and MQA).  The pages do not fix
 * which query heads share a K/V head; here they are contiguous groups: query
 * head h reads K/V head h / (H / Hkv).
 *
 *   k, v   [B,Hkv,Nkv,d] (BHND) or [B,Nkv,Hkv,d] (BSND), device memory
 *   Hkv    K/V heads, 1 <= Hkv, H % Hkv == 0 (Hkv == H is fa_fwd, Hkv == 1 is
 *          multi-query attention); otherwise FA_ERR_INVALID_ARG
 *
 * q, o and lse keep H heads.  Other arguments, ownership, the first-call
 * allocation and errors are as for fa_fwd.
 */
int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
               int64_t B, int64_t H, int64_t Hkv, int64_t Nq, int64_t Nkv, int64_t d,
               float scale, int causal, int layout, int dtype, void* stream);

/*
 * fa_bwd_workspace_size -- bytes of device workspace fa_bwd needs for B, H,
 * Nq and d (0 when B * H * Nq == 0): an fp32 dQ accumulator of B*H*Nq*d
 * values and two fp32 row arrays of B*H*ceil(Nq/128)*128 values, each part
 * rounded up to 256 bytes.  Returns FA_OK, FA_ERR_INVALID_ARG (negative size,
 * d not 64 or 128, NULL out pointer) or FA_ERR_UNSUPPORTED (sizes beyond the
 * index range).  Needs no GPU.
 */
int fa_bwd_workspace_size(int64_t B, int64_t H, int64_t Nq, int64_t d, int64_t* workspace_bytes);

/*
 * fa_bwd -- the gradients dQ, dK, dV of fa_fwd_gqa's O with respect to q, k
 * and v, given dO (page 1, "CANN ops-transformer FlashAttentionScore",
 * section 反向传播的重算策略及其合理性: the backward keeps no N x N matrix; it
 * recomputes each tile of P from Q, K and the forward's row statistics).  With
 * S = scale Q K^T [+ causal mask] and P = exp(S - LSE):
 *     dV = P^T dO,  dP = dO V^T,  dS = P o (dP - D),  D_i = sum_c dO_ic O_ic,
 *     dQ = scale dS K,  dK = scale dS^T Q.
 * Under grouped K/V heads a K/V head's gradient is the sum over the query
 * heads that read it.
 *
 *   q, k, v, o, lse   the forward's inputs, output and LSE (fa_fwd_gqa with
 *                     the same scale, causal flag, layout and dtype); lse
 *                     must not be NULL
 *   dout              dO, q's shape, layout and dtype
 *   dq                written, q's shape, layout and dtype
 *   dk, dv            written, k's shape, layout and dtype
 *   workspace         caller-owned device memory of at least
 *                     fa_bwd_workspace_size() bytes, 256-byte aligned; its
 *                     contents on entry do not matter, and it is in use until
 *                     the stream has finished the call
 *   d                 64 or 128; dtype bf16 or fp16 (fp32 returns
 *                     FA_ERR_UNSUPPORTED)
 *
 * Errors: as for fa_fwd_gqa, plus FA_ERR_INVALID_ARG for a missing or too
 * small workspace and FA_ERR_MISALIGNED for a misaligned one, both before
 * any launch.  The call launches three kernels on `stream` (the first
 * also clears the accumulator); Nq == 0 only clears dk and dv.  The
 * first-call allocation is fa_fwd's.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
           void* dq, void* dk, void* dv, void* workspace, int64_t workspace_bytes,
           int64_t B, int64_t H, int64_t Hkv, int64_t Nq, int64_t Nkv, int64_t d,
           float scale, int causal, int layout, int dtype, void* stream);

/*
 * fa_fwd_block_sparse -- fa_fwd_gqa with a block-sparse mask: query tile qt
 * (rows [128 qt, 128 qt + 128)) of batch entry b and head h sees key tile kt
 * (keys [128 kt, 128 kt + 128)) iff
 *     block_mask[b * mask_batch_stride + h * mask_head_stride + qt * KT + kt] != 0,
 * KT = ceil(Nkv / 128); with causal = 1 the causal mask applies as well.  Key
 * tiles a query tile does not see are skipped (page 1, "CANN ops-transformer
 * FlashAttentionScore", section 总结: SparseFlashAttention skips the key
 * blocks a sparse mask marks as not needed).
 *
 *   block_mask         uint8 device memory, [.., .., ceil(Nq/128), KT] with the
 *                      last two dimensions dense; read only
 *   mask_batch_stride, mask_head_stride
 *                      element strides of the batch and head dimensions of
 *                      block_mask (>= 0; 0 shares one mask across that
 *                      dimension)
 *   d                  64, 128 or 256
 *   dtype              bf16 or fp16 (fp32 returns FA_ERR_UNSUPPORTED)
 *
 * A query row with no visible key (all of its tile's mask entries zero, or
 * zero within its causal range) gets O = 0 and LSE = -inf: softmax over an
 * empty set is not defined, and these are the limits of an empty sum.  KT may
 * be at most 4096 (Nkv <= 524288), else FA_ERR_UNSUPPORTED.  The mask must be
 * readable for every (b, h, qt, kt) the strides address.  Other arguments,
 * ownership, the first-call allocation and errors are as for fa_fwd_gqa.
 */
int fa_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                        const uint8_t* block_mask, int64_t mask_batch_stride, int64_t mask_head_stride,
                        int64_t B, int64_t H, int64_t Hkv, int64_t Nq, int64_t Nkv, int64_t d,
                        float scale, int causal, int layout, int dtype, void* stream);

/*
 * fa_fwd_band -- fa_fwd_gqa with a band mask in place of the causal flag:
 * key j is visible to query row i iff i - pre_tokens <= j <= i + next_tokens
 * (and j < Nkv).  Page 2's flash_attention_score takes pre_tokens and
 * next_tokens and calls them with pre_tokens = seq_len, next_tokens = 0 for
 * causal attention; other values are read the same way (a sliding window:
 * pre_tokens = W - 1, next_tokens = 0).  KV tiles outside a query tile's band
 * are skipped.
 *
 *   pre_tokens, next_tokens  >= 0, and pre_tokens >= Nq - Nkv so that every
 *                            query row sees at least one key; otherwise
 *                            FA_ERR_INVALID_ARG
 *   dtype                    bf16 or fp16 (fp32 returns FA_ERR_UNSUPPORTED)
 *
 * Other arguments, ownership and errors are as for fa_fwd_gqa.
 */
int fa_fwd_band(const void* q, const void* k, const void* v, void* o, float* lse,
                int64_t B, int64_t H, int64_t Hkv, int64_t Nq, int64_t Nkv, int64_t d,
                float scale, int64_t pre_tokens, int64_t next_tokens, int layout, int dtype, void* stream);

/*
 * fa_fwd_paged -- fa_fwd_gqa with K and V read through a paged cache (page
 * 1, section GatherPAKVCache 的显存管理逻辑: the cache is kept in fixed-size
 * physical blocks, and a block table translates each sequence's logical
 * blocks to the physical blocks that hold them).
 *
 *   k_cache, v_cache  [num_blocks, block_size, Hkv, d] device memory: block,
 *                     then key within the block, head, feature
 *   block_table       int32 [B, max_blocks] device memory: keys
 *                     [i*block_size, (i+1)*block_size) of batch entry b are
 *                     physical block block_table[b*max_blocks + i]; entries for
 *                     i >= ceil(Nkv / block_size) are not read
 *   Nkv               keys per sequence (the same for every batch entry)
 *   block_size        a power of two >= 16
 *   num_blocks        physical blocks in each cache (>= 1)
 *   max_blocks        entries per table row, >= ceil(Nkv / block_size)
 *   dtype             bf16 or fp16 (fp32 returns FA_ERR_UNSUPPORTED)
 *
 * q, o, lse (H heads, `layout`), Hkv, scale and causal are as for fa_fwd_gqa.
 * Cache rows past Nkv in a sequence's last block are never used and may hold
 * anything; a table entry outside [0, num_blocks) reads as zeros.  Ownership,
 * the first-call allocation and errors are as for fa_fwd; block_table must be
 * 4-byte aligned.
 */
int fa_fwd_paged(const void* q, const void* k_cache, const void* v_cache, const int* block_table, void* o,
                 float* lse, int64_t B, int64_t H, int64_t Hkv, int64_t Nq, int64_t Nkv, int64_t d,
                 int64_t block_size, int64_t num_blocks, int64_t max_blocks, float scale, int causal, int layout,
                 int dtype, void* stream);

/*
 * Split-KV (flash-decoding) forms, for calls with few query rows per head
 * (decoding: one new token per step against a long key cache, page 1,
 * sections GatherPAKVCache 的显存管理逻辑 and the inference path's decode
 * stage), where one unit per (batch, head, pair of 128-row query tiles)
 * would leave most SMs idle while each unit walks every key tile.
 *
 * The key tiles (128 keys each) are cut into n_splits slices of equal length
 * (the last may be shorter, none is empty).  A unit per (batch, head, tile
 * pair, slice) computes its rows' attention over its slice alone: O_s,
 * normalised, and LSE_s, written in fp32 to the caller's workspace.  A merge
 * kernel then combines the slices with the online softmax's rule applied to
 * whole slices (page 1, section 在线 Softmax 的数学原理拆解):
 *     LSE = m + ln sum_s exp(LSE_s - m),  m = max_s LSE_s
 *     O   = sum_s exp(LSE_s - LSE) O_s
 * The result is attention over all Nkv keys, as from fa_fwd_gqa with
 * causal = 0 (these forms take no mask: every query row sees every key, as
 * a decoding step's new tokens see the whole cache).  O and LSE differ from
 * the unsplit call only by rounding.
 *
 * Calls with at most 8 query rows per K/V head (Nq * H / Hkv <= 8),
 * contiguous or paged, run a CUDA-core streaming kernel instead of the
 * tensor-core units: one CTA per (slice, batch, K/V head) takes all of the
 * K/V head's query rows; same plan, workspace and merge.  That kernel and
 * the merge are launched as dependent launches (programmatic stream
 * serialisation): each may start while the previous work on the stream
 * drains, and waits for it before touching any memory, so stream order is
 * kept.
 *
 * fa_splitkv_plan -- the slice count and workspace size of a split-KV call.
 *
 *   num_splits       > 0: that many slices, at most one per key tile;
 *                    <= 0: chosen by the library for num_sms SMs (a wave
 *                    model of its grid: enough units to fill the SMs in
 *                    whole waves, slices no shorter than needed; for
 *                    Nq <= 8 two CTAs per SM, the decoding kernel's)
 *   num_sms          SMs to plan for; <= 0: the current device's (which then
 *                    needs a usable sm_100 device, else FA_ERR_NO_DEVICE)
 *   *splits          out: the slice count the call will use (1 means the call
 *                    runs the unsplit kernel and needs no workspace)
 *   *workspace_bytes out: bytes of device workspace the call needs,
 *                    splits * B*H*Nq * (d + 1) * 4, or 0 for one slice
 *
 * Errors: FA_ERR_INVALID_ARG (negative size, d not in {64, 128}, null out
 * pointer), FA_ERR_UNSUPPORTED (sizes beyond the index range).
 */
int fa_splitkv_plan(int64_t B, int64_t H, int64_t Nq, int64_t Nkv, int64_t d, int num_splits, int num_sms,
                    int* splits, int64_t* workspace_bytes);

/*
 * fa_fwd_splitkv -- fa_fwd_gqa (causal = 0) computed as above.
 *
 *   num_splits       as for fa_splitkv_plan, planned for the current device
 *   workspace        device memory of at least the planned workspace_bytes,
 *                    16-byte aligned, owned by the caller and not read after
 *                    the call's work on `stream` has finished; it holds the
 *                    slices' fp32 O [splits, B, H, Nq, d] and then their LSE
 *                    [splits, B, H, Nq].  May be NULL when the plan has one
 *                    slice.
 *   workspace_bytes  its size in bytes
 *   dtype            bf16 or fp16 (fp32 returns FA_ERR_UNSUPPORTED)
 *
 * The other arguments are as for fa_fwd_gqa.  Two kernels are launched on
 * `stream` (the split kernel, then the merge), or one when the plan has one
 * slice.  Errors as for fa_fwd_gqa, and FA_ERR_INVALID_ARG for a missing or
 * too small workspace, FA_ERR_MISALIGNED for a misaligned one.
 */
int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                   int64_t Hkv, int64_t Nq, int64_t Nkv, int64_t d, float scale, int num_splits, void* workspace,
                   int64_t workspace_bytes, int layout, int dtype, void* stream);

/*
 * fa_fwd_paged_splitkv -- fa_fwd_paged (causal = 0) computed as above: K and
 * V through the paged cache and block table, described as for fa_fwd_paged;
 * num_splits and the workspace as for fa_fwd_splitkv.
 */
int fa_fwd_paged_splitkv(const void* q, const void* k_cache, const void* v_cache, const int* block_table, void* o,
                         float* lse, int64_t B, int64_t H, int64_t Hkv, int64_t Nq, int64_t Nkv, int64_t d,
                         int64_t block_size, int64_t num_blocks, int64_t max_blocks, float scale, int num_splits,
                         void* workspace, int64_t workspace_bytes, int layout, int dtype, void* stream);

/*
 * fa_fwd_noalloc -- the same computation, arguments and results as fa_fwd,
 * for callers that must never allocate device memory: code that runs inside
 * a memory pool or arena it does not own, real-time or embedded services that
 * reserve all device memory when they start, or hosts that forbid cudaMalloc
 * after start-up.  (The surveyed pages have no counterpart: this is a property
 * of the library, not of the method.)
 *
 * fa_fwd's tile scheduler keeps its per-launch work counters in 8 KB that it
 * allocates on its first call on a device.  This entry point keeps them in a
 * fixed 256-byte static device array instead, which every GPU that loads the
 * library holds until the process exits; no call allocates or frees
 * anything.  Slot 0 of the array (8 bytes: the work-ticket counter and the
 * finished-CTA counter) is cleared with cudaMemsetAsync on `stream` before
 * each launch; the rest of the array is unused padding.
 *
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) and sets kernel attributes; make that first call
 *     before any stream capture.
 *   - Every call on a device shares the array and it keeps the last call's
 *     contents: calls that overlap on the GPU (other streams, other threads)
 *     race on the counter and may compute wrong results.  Serialise them.
 *   - Limit: the work-ticket counter is 32-bit, so a bf16/fp16
 *     call may have at most 2^31 - 1025 work units (a unit is a pair of
 *     128-row query tiles of one batch and head, or one such tile at
 *     d = 256); larger calls return FA_ERR_TOO_LARGE before anything is
 *     launched.  fp32 inputs, and calls with at most 128 keys, use no
 *     scratch.
 *
 * Other arguments, ownership and errors are as for fa_fwd.
 */
int fa_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                   int64_t B, int64_t H, int64_t Nq, int64_t Nkv, int64_t d,
                   float scale, int causal, int layout, int dtype, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* fa_status_string(int status);

/*
 * fa_get_device_status -- synchronise `stream`, then read and clear the
 * current device's status word.  Returns FA_OK, FA_ERR_CHECK if a kernel of
 * a debug build (FA_CHECKS) found a computed index out of bounds since the
 * last read (it skipped that access), FA_ERR_TIMEOUT if any kernel gave up on
 * a bounded wait (its outputs are then undefined; the CUDA context stays
 * usable), or FA_ERR_LAUNCH if the stream itself reported an error.
 */
int fa_get_device_status(void* stream);

/*
 * fa_set_wait_timeout_us -- upper bound, in microseconds, on any single
 * device-side wait (mbarrier phase) inside the kernels launched afterwards
 * from this process.  0 restores the default (2,000,000 us).  Returns the
 * previous value.  Host-side setting; affects later launches only.
 */
uint32_t fa_set_wait_timeout_us(uint32_t us);

/*
 * fa_debug_set_fault -- test hook for failure detection, off by default.
 *   0: none
 *   1: the softmax warps of the tensor-core kernel never signal that P is
 *      ready, so the MMA warp's bounded wait expires; every role then leaves
 *      its loop, the CTA waits (bounded) for its own TMA copies and MMAs,
 *      frees its tensor memory and exits, and the status word reads
 *      FA_ERR_TIMEOUT.  No trap, no fault, no unbounded wait.
 * Applies to launches made after the call.  Returns the previous mode.
 */
int fa_debug_set_fault(int mode);

/* ABI version of this header, (major << 16) | minor (1.1: fa_fwd_gqa, 1.2: fa_fwd_paged, 1.3: fa_fwd_band,
 * 1.4: fa_splitkv_plan, fa_fwd_splitkv, fa_fwd_paged_splitkv, 1.5: FA_ERR_CHECK, 1.6: d = 256 in fa_fwd,
 * fa_fwd_gqa and fa_fwd_noalloc; fa_fwd_block_sparse, 1.7: fa_bwd_workspace_size, fa_bwd). */
int fa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
