/*
 * mxfa.h -- C ABI of the fused attention forward library (libmxfa.so).
 *
 * Every entry point computes, per query row i of sequence b and query head h,
 *
 *     O[i,h,:] = sum_j P_ij * v[j, h/G, :],   P_ij = exp(s_ij - m_i) / l_i
 *     s_ij     = softmax_scale * <q[i,h,:], k[j, h/G, :]>   for j visible,
 *     LSE[i,h] = m_i + ln(l_i)                 (natural log, fp32)
 *
 * without materialising the score matrix: KV is consumed tile by tile with a
 * running max, running sum and rescaled accumulator (the online softmax of
 * mxflashattn 1.4.0 prefill.py, prefill_chunked_reference, and of
 * oxillama-runtime 0.1.0 flash_attention.rs, flash_attention).
 *
 *   - G = Hq / Hkv: q head h reads kv head h / G (grouped-query attention,
 *     oxillama-runtime flash_attention.rs, flash_attention_gqa).
 *   - causal: key j is visible to query i of a sequence with Sq queries and
 *     Sk keys iff j <= i + Sk - Sq (bottom-right alignment, mxflashattn
 *     prefill.py); keys j >= Sk are never visible.
 *   - A row with no visible key gets O = 0 and LSE = -inf.
 *   - softmax_scale: pass NaN for the default Dqk^-0.5 (mxflashattn api.py,
 *     _resolved_scale); 0.0 is a legal scale (uniform attention).
 *
 * Conventions shared by all entry points
 *   Pointers: q, k, v, o, lse, cu_seqlens / indptr arrays and workspace are
 *     DEVICE pointers owned by the caller; the library never allocates,
 *     frees or synchronises.  q, k, v, o must be 16-byte aligned and every
 *     row/head stride must be a multiple of 16 bytes.  lse may be NULL (not
 *     written).
 *   Dtypes: q, k, v and o share one dtype (mxfa_dtype_t); lse is fp32.
 *   Stream: the work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Nothing is launched when a check fails.
 *   Errors: the return value is MXFA_OK or an error code; mxfa_last_error()
 *     returns a message for the calling thread's last failure.  Faults that
 *     can only be seen on the device (a bounded wait that ran out) are
 *     recorded in the workspace status word, read by
 *     mxfa_read_device_status().
 *   Workspace: each call needs `workspace` of at least the size returned by
 *     the matching *_workspace_size function (256-byte aligned device
 *     memory).  It holds the status word, the tile schedule and, for decode,
 *     the split partials.  Calls that share one workspace must be ordered on
 *     the device (same stream, or synchronised).
 *   Strict mode: with the environment variable MXFA_STRICT_VALIDATION=1 the
 *     varlen and decode entry points copy cu_seqlens / indptr to the host
 *     and check them (start at 0, non-decreasing, end at the totals, lengths
 *     within the stated maxima), as mxflashattn api.py does under
 *     MXFLASHATTN_STRICT_VALIDATION.  This synchronises the stream.
 */
#ifndef MXFA_H
#define MXFA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MXFA_OK = 0,
  MXFA_ERR_INVALID_ARG = 1,  /* bad pointer, size, stride or alignment */
  MXFA_ERR_UNSUPPORTED = 2,  /* legal but not implemented (head dim, dtype) */
  MXFA_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or too small */
  MXFA_ERR_CUDA = 4,         /* a CUDA runtime call failed */
  MXFA_ERR_TIMEOUT = 5       /* a device-side bounded wait ran out */
} mxfa_status_t;

typedef enum { MXFA_F32 = 0, MXFA_F16 = 1, MXFA_BF16 = 2 } mxfa_dtype_t;

/*
 * Batched attention forward, layout [B, S, H, D]
 * (mxflashattn 1.4.0 api.py, flash_attn_func).
 *   q: [B, Sq, Hq, D]   element (b,i,h,d) at b*Sq*q_row_stride + i*q_row_stride + h*q_head_stride + d
 *   k: [B, Sk, Hkv, D]  likewise with k_row_stride / k_head_stride (v the same with v_*)
 *   o: [B, Sq, Hq, D]   written; o_row_stride / o_head_stride
 *   lse: [B, Sq, Hq] fp32, contiguous (or NULL)
 * Strides are in elements; the batch stride is S * row stride (batches are
 * contiguous); the last dimension is contiguous.
 * Supported: D in {64, 128}; dtypes bf16 and f16 run on the tensor-core
 * kernel, f32 on the exact CUDA-core kernel; Hq a positive multiple of Hkv.
 * Sq = 0 or B = 0 is a no-op; Sk = 0 gives O = 0, LSE = -inf.
 */
size_t mxfa_attn_fwd_workspace_size(int B, int Sq, int Sk, int Hq, int Hkv, int D, mxfa_dtype_t dtype);
mxfa_status_t mxfa_attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                            int B, int Sq, int Sk, int Hq, int Hkv, int D, mxfa_dtype_t dtype,
                            int64_t q_row_stride, int64_t q_head_stride,
                            int64_t k_row_stride, int64_t k_head_stride,
                            int64_t v_row_stride, int64_t v_head_stride,
                            int64_t o_row_stride, int64_t o_head_stride,
                            float softmax_scale, int causal,
                            void *workspace, size_t workspace_bytes, void *stream);

/*
 * Variable-length attention forward, packed layout [total_tokens, H, D]
 * (mxflashattn 1.4.0 api.py, flash_attn_varlen_func; lattice-inference
 * 0.7.1 standard.rs, multi_head_attention_batched: cu_seqlens has batch+1
 * entries, starts at 0 and ends at the total).
 *   q: [total_q, Hq, D], k/v: [total_k, Hkv, D], o: [total_q, Hq, D] -- contiguous
 *   lse: [total_q, Hq] fp32 (or NULL)
 *   cu_seqlens_q / cu_seqlens_k: DEVICE int32 arrays of batch+1 entries;
 *   sequence b holds tokens [cu[b], cu[b+1]).  max_seqlen_q / max_seqlen_k
 *   must bound every sequence length (they size the schedule; values beyond
 *   them are an error caught in strict mode and otherwise undefined).
 * Supported as mxfa_attn_fwd.  Empty query sequences are skipped; a
 * sequence with no keys gives O = 0 and LSE = -inf.
 */
size_t mxfa_attn_varlen_fwd_workspace_size(int batch, int max_seqlen_q, int max_seqlen_k, int Hq, int D,
                                           mxfa_dtype_t dtype);
mxfa_status_t mxfa_attn_varlen_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                                   const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                   int batch, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                                   int Hq, int Hkv, int D, mxfa_dtype_t dtype,
                                   float softmax_scale, int causal,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * mxfa_attn_varlen_fwd without a workspace argument.  The pages have no
 * counterpart: this exists for callers that cannot allocate device memory
 * when they run attention (plugins and services that plan all device memory
 * up front, or code without access to the allocator that owns the device).
 * Same arguments, layouts and results as mxfa_attn_varlen_fwd.
 *   - Scratch: the schedule lives in a 1 MiB array owned by the library,
 *     which every GPU that loads the library holds until the process exits.
 *     A problem whose schedule needs more (mxfa_attn_varlen_fwd_workspace_size
 *     above 1 MiB, e.g. very large batch x max_seqlen_q) is rejected with
 *     MXFA_ERR_WORKSPACE and nothing is launched.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current.
 *   - Calls share the one array: calls that overlap on the GPU (different
 *     streams without ordering, or several host threads) race and must not
 *     be issued; order them on one stream.
 *   - No device memory is allocated or freed.
 *   - A rejected call (any check of mxfa_attn_varlen_fwd, or the size
 *     limit) writes nothing; an accepted one first clears the status word
 *     at the head of the array, so read it (mxfa_read_noalloc_status) after
 *     a call and before the next one.
 */
mxfa_status_t mxfa_attn_varlen_fwd_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                                           const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                           int batch, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                                           int Hq, int Hkv, int D, mxfa_dtype_t dtype,
                                           float softmax_scale, int causal, void *stream);

/*
 * Device-side status of the last mxfa_attn_varlen_fwd_noalloc call on the
 * current device: what mxfa_read_device_status returns for a caller
 * workspace (MXFA_OK; MXFA_ERR_TIMEOUT when a bounded wait gave up;
 * MXFA_ERR_INVALID_ARG when a sequence was longer than max_seqlen_q, so
 * part of O was not written), read from the library's scratch array.
 * Synchronises `stream`, clears the word when it is set, and sets
 * mxfa_device_status_detail() to the site code.  No pages have a
 * counterpart.
 */
mxfa_status_t mxfa_read_noalloc_status(void *stream);

/*
 * Split-KV decode (few queries per sequence, long KV), with the partial
 * (accumulator, max, sum) combine of kernelbot-amd-mixed-mla submission
 * 588924 (_flash_splitk / _reduce_splitk).
 *   q: [total_q, Hq, Dqk] contiguous; sequence b owns queries
 *      [qo_indptr[b], qo_indptr[b+1]) and keys [kv_indptr[b], kv_indptr[b+1])
 *   k: key row t, head g at k + t*k_row_stride + g*Dqk  (Dqk contiguous)
 *   v: value row t, head g at v + t*v_row_stride + g*Dv (Dv contiguous)
 *   o: [total_q, Hq, Dv] contiguous; lse: [total_q, Hq] fp32 (or NULL)
 *   qo_indptr / kv_indptr: DEVICE int32, batch+1 entries each.
 * MLA (DeepSeek-style latent cache): k = v = the kv base pointer, Hkv = 1,
 * Dqk = 576, Dv = 512, k_row_stride = v_row_stride = 576: value = first 512
 * columns of each cached row; the tensor-core kernel reads each KV tile once
 * and uses it as both operands.  That path needs bf16/f16 and
 * max_q_len <= 64.
 * Grouped-query decode (mxflashattn flash_attn_with_kvcache shape): Dqk = Dv
 * = 64 or 128, bf16/f16, max_q_len <= 64 and row strides that are multiples
 * of 8 elements run on the tensor-core kernel, which streams each KV head
 * once for the Hq / Hkv query heads that share it.  Other shapes (or f32)
 * run on the exact CUDA-core kernel.
 * Both tensor-core kernels compute 64 query rows (token, head) per pass over
 * a KV head: when max_q_len * Hq / Hkv exceeds 64, the query heads of each KV
 * head are split into the fewest equal groups of at most 64 rows (e.g. MLA
 * q_len 8 x 16 heads: two groups of 8 heads), and each group streams the KV
 * head again (the groups of one sequence run at about the same time, so the
 * repeated reads mostly come from L2).
 * The workspace size takes Hkv because the grouped-query kernel schedules
 * batch * Hkv * groups decode sequences.
 * num_splits: 0 = automatic: one run of KV tiles per SM, either whole
 *   sequences dealt out in order or the KV of all sequences cut into
 *   near-equal pieces, whichever balances better once the cost of merging a
 *   split sequence's partials is counted; k >= 1 = every sequence's KV is cut
 *   into k pieces.  The result does not depend on it beyond fp32 rounding.
 * Small problems (the MLA-shaped kernel, num_splits = 0, batch no larger
 *   than the SM count and batch * ceil(max_kv_len / 64) at most four tiles per
 *   SM) run as one cooperative kernel launch, preceded by a small memset of
 *   per-sequence counters in the workspace.  Each sequence is cut into
 *   near-equal pieces, one CTA each, and the pieces of a sequence merge their
 *   partials in the same kernel, so no schedule or combine kernel runs.  This
 *   is the launch-bound regime for which the MLA decode page switches to a
 *   different kernel (q_len * kv_len <= 4096).
 */
size_t mxfa_attn_decode_splitkv_workspace_size(int batch, int max_q_len, int Hq, int Hkv, int Dv, int max_kv_len,
                                               int num_splits, mxfa_dtype_t dtype);
mxfa_status_t mxfa_attn_decode_splitkv(const void *q, const void *k, const void *v, void *o, float *lse,
                                       const int32_t *qo_indptr, const int32_t *kv_indptr,
                                       int batch, int total_q, int total_kv, int max_q_len, int max_kv_len,
                                       int Hq, int Hkv, int Dqk, int Dv,
                                       int64_t k_row_stride, int64_t v_row_stride,
                                       mxfa_dtype_t dtype, float softmax_scale, int causal, int num_splits,
                                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * MLA split-KV decode over an fp8 latent cache (kernelbot-amd-mixed-mla
 * submission 588924 names an fp8 KV cache in its docstring; its code reads
 * the bf16 cache).  The page gives no fp8 format or scaling; this entry
 * point reads it as
 *   kv: [total_kv, 576] bytes, OCP 8-bit floating point E4M3 codes (sign,
 *       4 exponent bits with bias 7, 3 mantissa bits, subnormals, no
 *       infinities; the format torch calls float8_e4m3fn), row t at
 *       kv + t*kv_row_stride (bytes, a multiple of 16, >= 576);
 *   kv_scale: one per-tensor dequantisation factor, finite:
 *       key / value element = kv_scale * E4M3 value of its code.
 * The value of row t is its first 512 dequantised columns, as in
 * mxfa_attn_decode_splitkv's MLA shape.  The codes 0x7f and 0xff (NaN) are
 * not valid cache entries: they are read as +-480.
 *   q: [total_q, Hq, 576] bf16 contiguous; o: [total_q, Hq, 512] bf16;
 *   lse: [total_q, Hq] fp32 (or NULL); qo_indptr / kv_indptr, max lengths,
 *   causal, num_splits and the workspace as for mxfa_attn_decode_splitkv.
 *   Requires max_q_len <= 64 (else MXFA_ERR_UNSUPPORTED); more than 64
 *   query rows per sequence are split into head groups as for
 *   mxfa_attn_decode_splitkv.  kv must be a valid 16-byte aligned pointer
 *   even when total_kv = 0.
 * The kernel widens each staged tile of codes to bf16 exactly in shared
 * memory and applies kv_scale to the scores and to the outputs, so the
 * result equals attention over the dequantised cache up to the bf16 path's
 * rounding.
 */
size_t mxfa_attn_decode_mla_fp8kv_workspace_size(int batch, int max_q_len, int Hq, int max_kv_len, int num_splits);
mxfa_status_t mxfa_attn_decode_mla_fp8kv(const void *q, const void *kv, float kv_scale, void *o, float *lse,
                                         const int32_t *qo_indptr, const int32_t *kv_indptr, int batch, int total_q,
                                         int total_kv, int max_q_len, int max_kv_len, int Hq, int64_t kv_row_stride,
                                         float softmax_scale, int causal, int num_splits, void *workspace,
                                         size_t workspace_bytes, void *stream);

/*
 * Decode over a KV cache, with an optional append (mxflashattn 1.4.0 api.py,
 * flash_attn_with_kvcache: q, k_cache, v_cache, k, v, cache_seqlens,
 * block_table, causal).
 *   q: [batch, Sq, Hq, D] contiguous, bf16 or f16, D = 64 or 128,
 *      Sq <= 64 (otherwise MXFA_ERR_UNSUPPORTED; Sq * Hq / Hkv above 64 is
 *      split into head groups as for mxfa_attn_decode_splitkv).
 *   k_cache, v_cache: [num_pages, page_size, Hkv, D] contiguous.  Dense cache
 *      (block_table == NULL): num_pages = batch, page_size = the cache length,
 *      key position pos of batch entry b is row b*page_size + pos.  Paged
 *      cache: block_table [batch, max_blocks_per_seq] int32 (device) gives the
 *      page of key positions [i*page_size, (i+1)*page_size) of entry b;
 *      page_size is a power of two in [16, 128] or a multiple of 128.
 *   cache_seqlens: [batch] int32 (device), keys already cached per entry.
 *   k_new, v_new: [batch, Snew, Hkv, D] contiguous or both NULL (Snew = 0).
 *      Row i of entry b is written to key position cache_seqlens[b] + i
 *      before the attention, and cache_seqlens[b] is then advanced by Snew
 *      in place (a position beyond the cache's capacity is not written and
 *      the workspace status reports MXFA_ERR_INVALID_ARG).
 *   Attention: query i of entry b (of Sq) sees key positions [0, L_b),
 *      L_b = cache_seqlens[b] + Snew (as passed in); causal: j <= i + L_b - Sq.
 *   o: [batch, Sq, Hq, D] contiguous; lse: [batch, Sq, Hq] fp32 (or NULL).
 *   max_len: an upper bound of every L_b (sizes the workspace schedule).
 *   num_splits: as for mxfa_attn_decode_splitkv.
 * The caller owns every buffer; the library writes k_cache / v_cache only at
 * the appended positions and cache_seqlens only by the advance.
 */
size_t mxfa_attn_decode_kvcache_workspace_size(int batch, int Sq, int Hq, int Hkv, int D, int max_len,
                                               int num_splits, mxfa_dtype_t dtype);
mxfa_status_t mxfa_attn_decode_kvcache(const void *q, void *k_cache, void *v_cache, const void *k_new,
                                       const void *v_new, int32_t *cache_seqlens, const int32_t *block_table,
                                       int batch, int Sq, int Snew, int Hq, int Hkv, int D, int num_pages,
                                       int page_size, int max_blocks_per_seq, int max_len, mxfa_dtype_t dtype,
                                       float softmax_scale, int causal, int num_splits, void *o, float *lse,
                                       void *workspace, size_t workspace_bytes, void *stream);

/* Message for the calling thread's most recent failure ("" if none). */
const char *mxfa_last_error(void);

/*
 * Synchronises `stream`, reads the status word the last call wrote into
 * `workspace` and returns it (MXFA_OK, or MXFA_ERR_TIMEOUT when a bounded
 * device wait gave up; the kernel then skipped its remaining work and left
 * the outputs incomplete), and clears it when it is set.
 * mxfa_device_status_detail() returns the site code from the same read:
 * for a timeout the wait that ran out; for MXFA_ERR_INVALID_ARG 0x201 (a
 * varlen sequence longer than max_seqlen_q: its blocks beyond the schedule
 * were not computed), 0x401 (decode pieces beyond the workspace schedule)
 * or 0x402 (a KV-cache length beyond the cache's capacity: attention ran
 * over the first page_size keys of a dense entry, or max_blocks_per_seq
 * pages of a paged one).
 */
mxfa_status_t mxfa_read_device_status(const void *workspace, void *stream);
uint32_t mxfa_device_status_detail(void);

/* Library version, (major << 16) | (minor << 8) | patch. */
uint32_t mxfa_version(void);

/*
 * Testing hooks (for the library's own tests; the pages have no
 * counterpart).  Process-wide settings read by every later call:
 *   wait_budget_ns: budget of every bounded device-side wait of later
 *     launches, in nanoseconds (0 restores the default of 2 s).  A wait that
 *     runs out records MXFA_ERR_TIMEOUT and its site code in the workspace
 *     status word and the kernel returns without finishing its work.
 *   keep_merge_counters: non-zero makes the one-launch decode schedule (see
 *     mxfa_attn_decode_splitkv) skip its memset of the per-sequence merge
 *     counters and use the values the caller left in the workspace; a
 *     counter that cannot reach its sequence's piece count makes the merge
 *     wait run out (its site code is 0x309).
 * Production code does not call this.
 */
void mxfa_test_hooks(uint64_t wait_budget_ns, int keep_merge_counters);

#ifdef __cplusplus
}
#endif

#endif /* MXFA_H */
