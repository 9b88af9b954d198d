/*
 * gqa.h -- C ABI of the B200 (sm_100a) grouped-query attention library
 * (libgqa_b200.so).
 *
 * Both calls compute exact attention, O_i = softmax(Q_i K_{g(i)}^T * scale) V_{g(i)},
 * over the whole MHA (n_kv = h) / GQA (1 < n_kv < h) / MQA (n_kv = 1) range:
 *   - "Evolution of AI Attention Mechanisms" (toolsku), "MHA Mathematical
 *     Formulation": per-head softmax(Q_i K_i^T / sqrt(d_h)) V_i, heads being
 *     contiguous d_h slices of the hidden dimension;
 *   - same page, "GQA Implementation": with n_rep = h / n_kv, query head i
 *     uses KV head g(i) = i / n_rep (K/V repeated per contiguous group);
 *   - "Multi-Query Attention" (inferensys glossary), "Decoding Step": one
 *     decode step is softmax(Q_all K_shared^T) V_shared;
 *   - "Attention variants" (saadho), "What this topic covers": the result is
 *     exact; the score matrix is built tile by tile on chip and never written
 *     to device memory (online softmax with a running max and running sum).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers, row-major, 16-byte aligned,
 *     owned by the caller; q/k/v/out are bf16 (IEEE bfloat16) unless an entry
 *     point says otherwise (8-bit caches, int32 lengths and page tables,
 *     float32 scales).  The library keeps no
 *     pointer after the call returns, allocates no device memory and creates
 *     no stream.
 *   - Work is enqueued asynchronously on `stream` (0 = legacy default stream).
 *     Inputs must stay unmodified, and `out` unread, until the stream reaches
 *     the call.
 *   - The return value is a gqa_status_t.  Argument errors are reported
 *     synchronously with nothing launched and `out` untouched.  A fault that
 *     happens while the kernel runs surfaces at the caller's next
 *     synchronisation, as with any CUDA kernel; a kernel that gives up on an
 *     internal wait records GQA_ERR_TIMEOUT, which gqa_get_device_status()
 *     returns.
 *   - `scale` must be finite and >= 0 (softmax temperature; the pages use
 *     1/sqrt(d_h)).  d_h must be 64 or 128.
 */
#ifndef GQA_B200_H
#define GQA_B200_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GQA_OK = 0,
    GQA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, h % n_kv != 0, bad scale */
    GQA_ERR_UNSUPPORTED = 2,   /* a valid request the library does not implement (e.g. d_h not 64/128) */
    GQA_ERR_CUDA = 3,          /* the launch failed (see cudaGetLastError) */
    GQA_ERR_TIMEOUT = 4        /* a kernel gave up on an internal wait (device status only) */
} gqa_status_t;

/*
 * Prefill (and chunked prefill): every query row of every head at once.
 *   q   [B, S_q,  h,    d_h]   bf16   queries (the "BSHD" layout of the
 *                                     flash_attn_func call shown on the toolsku
 *                                     page, "Flash Attention Usage")
 *   k   [B, S_kv, n_kv, d_h]   bf16   keys
 *   v   [B, S_kv, n_kv, d_h]   bf16   values
 *   out [B, S_q,  h,    d_h]   bf16   result, rounded to nearest even
 * causal != 0: query row r sees keys j <= r + (S_kv - S_q).  The new queries
 * are the LAST S_q positions of the S_kv keys, as when past K/V are
 * concatenated in front of the new ones ("MHA Implementation", past_kv);
 * S_q > S_kv is then rejected (a row would see no key).  causal == 0: every
 * row sees all S_kv keys.
 * Errors: GQA_ERR_INVALID_ARG for a null or non-16-byte-aligned pointer,
 * B, S_q, S_kv, h, n_kv <= 0, h % n_kv != 0, causal with S_q > S_kv, a
 * non-finite or negative scale, or sizes whose element counts overflow
 * int32 indexing of a dimension; GQA_ERR_UNSUPPORTED for d_h not in {64, 128};
 * GQA_ERR_CUDA if the launch fails.
 */
int gqa_prefill(const void *q, const void *k, const void *v, void *out,
                int B, int S_q, int S_kv, int h, int n_kv, int d_h,
                int causal, float scale, cudaStream_t stream);

/*
 * Decode: one new query token per sequence against its KV cache.
 *   q        [B, h, d_h]               bf16   the new tokens' queries
 *   k_cache  [sum_b seqlens[b], n_kv, d_h] bf16  packed keys: sequence b's
 *   v_cache  [sum_b seqlens[b], n_kv, d_h] bf16  tokens start at row
 *                                               sum_{b' < b} seqlens[b'];
 *                                               with equal lengths S this is
 *                                               exactly [B, S, n_kv, d_h]
 *   seqlens  [B]                       int32  DEVICE array; seqlens[b] counts
 *                                             every cached token of sequence b,
 *                                             the new token's own K/V included
 *                                             (K/V are concatenated before the
 *                                             attention, toolsku "MHA
 *                                             Implementation")
 *   out      [B, h, d_h]               bf16   result
 * Query head i of sequence b attends to all seqlens[b] tokens of KV head
 * i / (h / n_kv).  A length <= 0 produces a zero row (counted as zero rows
 * of the packed caches).  The caches must hold at least sum(max(seqlens, 0))
 * rows: this entry point has no row count to check against (the lengths live
 * on the device), so it only cuts and reports a sequence that would end past
 * row 2^30; gqa_decode_rows checks the actual row count.
 * Errors: as gqa_prefill (B, h, n_kv <= 0, h % n_kv != 0, pointers, scale,
 * d_h), plus GQA_ERR_INVALID_ARG for B > 65535.
 */
int gqa_decode(const void *q, const void *k_cache, const void *v_cache,
               const int32_t *seqlens, void *out,
               int B, int h, int n_kv, int d_h, float scale, cudaStream_t stream);

/*
 * gqa_decode with the caches' row count: the same computation, over packed
 * caches that hold `cache_rows` rows ([cache_rows, n_kv, d_h] each).  The
 * lengths live on the device, so the host cannot compare them with the
 * caches; here the kernel does.  A sequence whose rows would end past
 * cache_rows (its first row is the sum of the earlier non-negative lengths,
 * summed in 64 bits) is cut to the rows that exist, and GQA_ERR_INVALID_ARG
 * is recorded in the device status word (gqa_get_device_status); no row past
 * cache_rows is ever read.  The Python binding calls this form.
 * Errors: as gqa_decode, plus GQA_ERR_INVALID_ARG for cache_rows < 0 or
 * cache_rows > INT32_MAX (tile coordinates are 32-bit).
 */
int gqa_decode_rows(const void *q, const void *k_cache, const void *v_cache, int64_t cache_rows,
                    const int32_t *seqlens, void *out,
                    int B, int h, int n_kv, int d_h, float scale, cudaStream_t stream);

/*
 * Decode with the batch's cached tokens divided evenly among the SMs: the same
 * result as gqa_decode_rows (same arguments, same row check, same device
 * status), built for groups of many query heads per KV head (MQA, wide GQA)
 * and for ragged lengths.  Per byte of K/V a group of h / n_kv heads does
 * h / n_kv multiply-adds for each product ("Multi-query attention"
 * (pranaymahendrakar), "Why this is a bandwidth argument, not a FLOP
 * argument"), and a fixed number of splits per sequence leaves SMs idle
 * while the longest sequences finish; here the tokens of the whole batch are
 * laid end to end and each SM's CTAs take an equal share, whatever the
 * sequence boundaries.  By group size (as measured): 17 to 64 heads at
 * d_h = 128 run warp-level MMAs, two CTAs per SM; smaller groups at
 * d_h = 128 run tcgen05 products with the tokens as the rows; d_h = 64 and
 * groups above 64 heads run tcgen05 products with the heads as the rows (a
 * group of at most 64 (32) heads as 2 (4) copies, each over its own share of
 * every stage's tokens).  The pieces of a sequence that fell to several CTAs
 * are merged (log-sum-exp rule) from the workspace by a second kernel.
 *   workspace        DEVICE memory of at least
 *                    gqa_decode_split_workspace_bytes(B, h, n_kv, d_h) bytes
 *                    (which depends on the current device's SM count),
 *                    256-byte aligned, owned by the caller.  It is scratch:
 *                    every call writes what it reads, so it needs no
 *                    initialisation.  Calls that share a workspace must not
 *                    overlap on the GPU (one stream, or ordered).
 * The call enqueues two kernels on `stream`: the split decode, then the merge
 * of the sequences whose tokens fell to several SMs.
 * Errors: as gqa_decode_rows, plus GQA_ERR_INVALID_ARG for a null,
 * misaligned or too small workspace, GQA_ERR_UNSUPPORTED when
 * n_kv * ceil(h / n_kv / 128) * B exceeds 2^24.
 */
int gqa_decode_split(const void *q, const void *k_cache, const void *v_cache, int64_t cache_rows,
                     const int32_t *seqlens, void *out,
                     int B, int h, int n_kv, int d_h, float scale,
                     void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Workspace bytes gqa_decode_split needs for these sizes on the current
 * device; 0 for sizes gqa_decode_split rejects. */
size_t gqa_decode_split_workspace_bytes(int B, int h, int n_kv, int d_h);

/*
 * gqa_decode_split for callers that may not allocate device memory -- for
 * instance a plug-in running inside another framework that must not touch
 * that framework's memory pool, or a serving loop that forbids allocations
 * once it has started (cudaMalloc synchronises the device and fails when the
 * memory is fully reserved).  The pages describe no such call: this is an
 * interface convenience, not part of the method.
 *   Same arguments and result as gqa_decode_split, without the workspace:
 *   the workspace is a fixed 16 MiB array inside the library, which every
 *   device that loads the library holds until the process exits.  The call
 *   allocates nothing (no cudaMalloc, no allocating library routine) and
 *   needs no clearing (every call writes what it reads).
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 *   Every call uses the same array: calls that overlap on the GPU (on
 *   different streams, or from different threads without ordering) race and
 *   their results are undefined.
 * Errors: as gqa_decode_split (without the workspace checks), plus
 * GQA_ERR_UNSUPPORTED when the sizes need more than the 16 MiB array, that is
 * when gqa_decode_split_workspace_bytes(B, h, n_kv, d_h) exceeds 16 MiB (on a
 * 148-SM B200: n_kv * B above 208 for 17 to 64 query heads per KV head at
 * d_h = 128; otherwise n_kv * ceil(h / n_kv / 128) * B above 104 at
 * d_h = 128, above 348 at d_h = 64), and GQA_ERR_CUDA if the address lookup
 * or a launch fails.
 * Nothing is launched on an argument or size error.
 */
int gqa_decode_split_noalloc(const void *q, const void *k_cache, const void *v_cache, int64_t cache_rows,
                             const int32_t *seqlens, void *out,
                             int B, int h, int n_kv, int d_h, float scale, cudaStream_t stream);

/*
 * Decode over an 8-bit cache ("Multi-Query Attention (MQA)" (inferensys
 * glossary), "KV cache quantization": the cache is kept in FP8 with scaling
 * factors; "Multi-query attention" (pranaymahendrakar), "Interaction with
 * other techniques": fp8 halves the bytes per cached element).
 *   k_cache, v_cache  [sum_b seqlens[b], n_kv, d_h]  uint8   OCP E4M3 codes
 *                     (the variant without infinities; 0x7f / 0xff are NaN),
 *                     packed exactly as in gqa_decode
 *   k_scale, v_scale  [n_kv]  float32  DEVICE arrays: the cached value of a
 *                     code of KV head g is code * k_scale[g] (keys) or
 *                     code * v_scale[g] (values)
 *   q, seqlens, out   as in gqa_decode (bf16 q and out)
 * The products run with f16 operands: Q is rounded to f16 (exact for
 * magnitudes in [2^-14, 65504]; larger ones overflow) and the softmax weights
 * are rounded to f16; the codes are exact in f16.  Accumulation is fp32.
 * Scales must be finite and >= 0; any other value is recorded as
 * GQA_ERR_INVALID_ARG in the device status word (gqa_get_device_status) and
 * the affected rows are unspecified.
 * Errors: as gqa_decode, plus GQA_ERR_INVALID_ARG for a null or
 * non-4-byte-aligned scale pointer.
 */
int gqa_decode_fp8(const void *q, const void *k_cache, const void *v_cache,
                   const float *k_scale, const float *v_scale,
                   const int32_t *seqlens, void *out,
                   int B, int h, int n_kv, int d_h, float scale, cudaStream_t stream);

/* gqa_decode_fp8 over packed E4M3 caches of `cache_rows` rows, with the row
 * check of gqa_decode_rows (lengths past the caches cut and reported). */
int gqa_decode_fp8_rows(const void *q, const void *k_cache, const void *v_cache, int64_t cache_rows,
                        const float *k_scale, const float *v_scale,
                        const int32_t *seqlens, void *out,
                        int B, int h, int n_kv, int d_h, float scale, cudaStream_t stream);

/*
 * Decode over a paged bf16 cache ("Multi-Query Attention (MQA)" (inferensys
 * glossary), "PagedAttention": each sequence's cache is cut into fixed-size
 * pages that may lie anywhere in device memory).
 *   k_pages, v_pages  [num_pages, page_size, n_kv, d_h]  bf16
 *   block_table       [B, max_blocks]  int32  DEVICE array: token t of
 *                     sequence b is slot t % page_size of page
 *                     block_table[b * max_blocks + t / page_size]; entries
 *                     past a sequence's last page are never read
 *   seqlens           [B]  int32  DEVICE array, tokens per sequence (<= 0:
 *                     zero row)
 *   q, out            [B, h, d_h]  bf16
 * page_size is a power of two in [16, 65536].  Slots of a page past the
 * sequence's end may hold anything (NaN included): they are never used.
 * A page id outside [0, num_pages), or a length above max_blocks * page_size,
 * is recorded as GQA_ERR_INVALID_ARG in the device status word; such pages
 * read as zeros and such lengths are cut to max_blocks * page_size.
 * Errors: as gqa_decode, plus GQA_ERR_INVALID_ARG for a null or misaligned
 * block_table, max_blocks or num_pages <= 0, a page_size that is not a power
 * of two in [16, 65536], or max_blocks * page_size above INT32_MAX.
 */
int gqa_decode_paged(const void *q, const void *k_pages, const void *v_pages,
                     const int32_t *block_table, int max_blocks, int page_size, int num_pages,
                     const int32_t *seqlens, void *out,
                     int B, int h, int n_kv, int d_h, float scale, cudaStream_t stream);

/* Paged E4M3 pages [num_pages, page_size, n_kv, d_h] (uint8 codes) with the
 * per-KV-head scales of gqa_decode_fp8; everything else as gqa_decode_paged. */
int gqa_decode_paged_fp8(const void *q, const void *k_pages, const void *v_pages,
                         const float *k_scale, const float *v_scale,
                         const int32_t *block_table, int max_blocks, int page_size, int num_pages,
                         const int32_t *seqlens, void *out,
                         int B, int h, int n_kv, int d_h, float scale, cudaStream_t stream);

/*
 * Chunked prefill over a paged bf16 cache, with the append
 * ("Evolution of AI Attention Mechanisms" (toolsku), "MHA Implementation":
 * the new K/V are concatenated after the past ones; "Multi-Query Attention
 * (MQA)" (inferensys glossary), "PagedAttention").
 *   q               [B, S_q, h, d_h]        bf16  the chunk's queries
 *   k_new, v_new    [B, S_q, n_kv, d_h]     bf16  the chunk's keys and values
 *   k_pages, v_pages [num_pages, page_size, n_kv, d_h]  bf16  the cache, as in
 *                   gqa_decode_paged; WRITTEN: row t of k_new[b] / v_new[b]
 *                   goes to position past_lens[b] + t of sequence b (every KV
 *                   head).  Slots at other positions are not touched.
 *   block_table     [B, max_blocks]  int32  DEVICE array; must cover positions
 *                   0 .. past_lens[b] + S_q - 1 of every sequence
 *   past_lens       [B]  int32  DEVICE array: tokens already cached per
 *                   sequence (<= 0: none)
 *   out             [B, S_q, h, d_h]        bf16
 * Query row r of sequence b sits at position past_lens[b] + r and attends to
 * the keys at positions <= past_lens[b] + r (bottom-right causal), the past
 * ones read from the pages and the chunk's from k_new / v_new.  The caller
 * must not read or write the pages of these sequences until the stream
 * reaches the call.  A page id outside [0, num_pages) or past_lens[b] + S_q
 * above max_blocks * page_size is recorded as GQA_ERR_INVALID_ARG in the
 * device status word (such pages read as zeros and are not written; such a
 * past length is cut).
 * Errors: as gqa_prefill (pointers, sizes, scale, d_h) and gqa_decode_paged
 * (block_table, max_blocks, page_size, num_pages), plus GQA_ERR_INVALID_ARG
 * for S_q > max_blocks * page_size.
 */
int gqa_prefill_paged(const void *q, const void *k_new, const void *v_new,
                      void *k_pages, void *v_pages,
                      const int32_t *block_table, int max_blocks, int page_size, int num_pages,
                      const int32_t *past_lens, void *out,
                      int B, int S_q, int h, int n_kv, int d_h, float scale, cudaStream_t stream);

/*
 * Absorbed multi-head latent attention (MLA) decode ("Evolution of AI
 * Attention Mechanisms" (toolsku), "Generation 3: MLA Multi-Head Latent
 * Attention": one latent vector c_kv per token is cached for all heads; with
 * the key up-projection absorbed into the query, Q K^T = (Q W_k_up) c_kv^T,
 * and the softmax weights multiply c_kv itself).
 *   q_absorbed  [B, h, d_c]            bf16  q' = q W_k_up per head (the
 *                                            caller's projection)
 *   c_kv        [sum_b seqlens[b], d_c] bf16  packed latent cache, sequence b
 *                                            starting at row sum_{b'<b} seqlens[b']
 *   seqlens     [B]  int32  DEVICE array (<= 0: zero row)
 *   out         [B, h, d_c]            bf16  softmax(q' c_kv^T * scale) c_kv
 * d_c must be 512 (the pages' latent width); the pages' code uses
 * scale = d_c^-0.5.  Errors: GQA_ERR_INVALID_ARG for null or misaligned
 * pointers, B <= 0 or > 65535, h <= 0, a bad scale; GQA_ERR_UNSUPPORTED for
 * d_c != 512.
 */
int gqa_mla_decode(const void *q_absorbed, const void *c_kv, const int32_t *seqlens, void *out,
                   int B, int h, int d_c, float scale, cudaStream_t stream);

/* gqa_mla_decode over a latent cache of `cache_rows` rows, with the row check
 * of gqa_decode_rows (lengths past the cache cut and reported).  With the row
 * count known, long sequences in small batches run on a second kernel (see
 * gqa_mla_decode_path); the results agree within the same bound. */
int gqa_mla_decode_rows(const void *q_absorbed, const void *c_kv, int64_t cache_rows,
                        const int32_t *seqlens, void *out,
                        int B, int h, int d_c, float scale, cudaStream_t stream);

/*
 * gqa_mla_decode_rows with a workspace: the tensor-core kernel can then split a
 * sequence over any number of SMs (one CTA per SM) and merge the splits' partial
 * results from the workspace in a second launch (log-sum-exp rule), instead of
 * within a thread-block cluster of at most 16.  Used where gqa_mla_decode_path
 * (..., 1) answers 2; otherwise the call runs as gqa_mla_decode_rows and the
 * workspace is not touched.
 *   workspace        DEVICE memory of at least
 *                    gqa_mla_decode_split_workspace_bytes(B, h, d_c) bytes,
 *                    256-byte aligned, owned by the caller, needing no
 *                    initialisation.  Calls that share a workspace must not
 *                    overlap on the GPU.
 * Errors: as gqa_mla_decode_rows, plus GQA_ERR_INVALID_ARG for a null,
 * misaligned or too small workspace.
 */
int gqa_mla_decode_split(const void *q_absorbed, const void *c_kv, int64_t cache_rows,
                         const int32_t *seqlens, void *out,
                         int B, int h, int d_c, float scale,
                         void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Bytes of workspace gqa_mla_decode_split needs on the current device: the
 * tensor-core kernel's partials, ceil(h / 32) * B * splits * (32 * 512 + 64)
 * floats with splits = max(1, min(256, SMs / (ceil(h / 32) * B))), for shapes
 * where that kernel can be picked (h > 16 and the warp-level kernel's CTAs
 * fewer than the SMs); 0 for the other shapes (any non-null, aligned
 * workspace pointer then does) and for sizes the call refuses (B <= 0 or
 * > 65535, h <= 0 or > 65535 * 16, d_c != 512).  Host-only. */
size_t gqa_mla_decode_split_workspace_bytes(int B, int h, int d_c);

/* Which kernel runs for a shape on the current device: gqa_mla_decode_rows
 * (with_workspace = 0) or gqa_mla_decode_split (with_workspace != 0).
 *   0  warp-level MMA: 16-head groups, the splits of one sequence merged in a
 *      thread-block cluster (gqa_mla_decode always runs it);
 *   1  5th-generation tensor cores with q' resident in tensor memory, 32-head
 *      groups, one CTA per SM, splits merged in a cluster: taken when h > 16,
 *      the warp-level kernel's CTAs (B * ceil(h / 16) times up to 8 splits) are
 *      fewer than the SMs, and cache_rows >= 8192 * B;
 *   2  the same tensor-core kernel with its splits merged through the workspace
 *      (with_workspace only; any number of splits, every SM busy): taken when
 *      h > 16, the warp-level kernel's CTAs are fewer than the SMs, and
 *      cache_rows >= 2048 * B.
 * Host-only (reads the SM count; 148 when no device answers).  Returns -1 for
 * B <= 0, h <= 0, d_c != 512 or cache_rows outside [0, 2^31). */
int gqa_mla_decode_path(int B, int h, int d_c, int64_t cache_rows, int with_workspace);

/* A static, human-readable name for a gqa_status_t value. */
const char *gqa_status_string(int status);

/*
 * Returns and clears the library's device status word for the current
 * device: GQA_OK, GQA_ERR_TIMEOUT if a kernel gave up on an internal wait
 * since the last read, or GQA_ERR_INVALID_ARG if a kernel met a bad value
 * that lives on the device (a page id, a length beyond the block table or
 * the caches, a negative or non-finite cache scale).  The first error
 * recorded since the last read wins.
 * The word is per DEVICE, not per stream: it collects what every kernel of
 * this library on the device recorded, whatever its stream.  The read is
 * enqueued on `stream` as one atomic exchange (the word is swapped for 0),
 * then `stream` is synchronised; an error that a kernel on another stream
 * records meanwhile is never lost -- it is returned by this read or by the
 * next.  To attribute an error to one call, synchronise the device (or every
 * stream that runs this library's kernels) before the call and read the word
 * after it.  Returns GQA_ERR_CUDA if the read or the synchronisation fails.
 */
int gqa_get_device_status(cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GQA_B200_H */
