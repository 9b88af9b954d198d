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
 *   - All tensor pointers are DEVICE pointers to bf16 (IEEE bfloat16) data,
 *     row-major, 16-byte aligned, owned by the caller.  The library keeps no
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

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GQA_OK = 0,
    GQA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, h % n_kv != 0, bad scale */
    GQA_ERR_UNSUPPORTED = 2,   /* a valid request this build does not implement (d_h not 64/128) */
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
 * rows; the library cannot check this (the lengths live on the device).
 * Errors: as gqa_prefill (B, h, n_kv <= 0, h % n_kv != 0, pointers, scale,
 * d_h), plus GQA_ERR_INVALID_ARG for B > 65535.
 */
int gqa_decode(const void *q, const void *k_cache, const void *v_cache,
               const int32_t *seqlens, void *out,
               int B, int h, int n_kv, int d_h, float scale, cudaStream_t stream);

/* A static, human-readable name for a gqa_status_t value. */
const char *gqa_status_string(int status);

/*
 * Synchronises `stream`, then returns and clears the library's device status
 * word for the current device: GQA_OK, or GQA_ERR_TIMEOUT if a kernel gave up
 * on an internal wait since the last call.  Returns GQA_ERR_CUDA if the
 * synchronisation itself fails.
 */
int gqa_get_device_status(cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GQA_B200_H */
