// The C ABI (include/gqa.h): argument validation, dispatch, device status.
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "gqa.h"
#include "common.cuh"

namespace gqa {
__device__ int g_status = 0;         // see gqa_get_device_status()
__device__ int g_status_taken = 0;   // the value the last status read exchanged out of g_status
#ifdef GQA_WAIT_TEST
__device__ int g_test_stall = 0;     // wait-test build: producers leave their first stage unloaded
#endif

// Exchange the status word for 0 in one atomic step, so that an error a kernel
// records concurrently is either returned now or kept for the next read.
__global__ void take_status_kernel() { g_status_taken = atomicExch(&g_status, 0); }

int launch_prefill(const void *q, const void *k, const void *v, void *out, int B, int S_q, int S_kv, int h, int n_kv,
                   int d, int causal, float scale, cudaStream_t stream);
int launch_decode(const void *q, const void *k, const void *v, const int32_t *seqlens, void *out, int B, int h,
                  int n_kv, int d, float scale, long long cache_rows, cudaStream_t stream);
int launch_prefill_paged(const void *q, const void *k_new, const void *v_new, void *k_pages, void *v_pages,
                         const int32_t *block_table, int max_blocks, int page_size, int num_pages,
                         const int32_t *past_lens, void *out, int B, int S_q, int h, int n_kv, int d, float scale,
                         cudaStream_t stream);
int launch_mla_decode(const void *q, const void *c_kv, const int32_t *seqlens, void *out, int B, int h, float scale,
                      long long cache_rows, bool rows_known, cudaStream_t stream);
bool mla_prefers_tc(int B, int h, long long cache_rows, bool rows_known, int sms);
bool mla_ws_prefers_tc(int B, int h, long long cache_rows, int sms);
size_t mla_ws_bytes(int B, int h, int sms);
int launch_mla_decode_ws(const void *q, const void *c_kv, const int32_t *seqlens, void *out, int B, int h,
                         float scale, long long cache_rows, void *ws, size_t ws_bytes, cudaStream_t stream);
int launch_decode_ex(const void *q, const void *k, const void *v, const float *k_scale, const float *v_scale,
                     const int32_t *seqlens, const int32_t *block_table, int max_blocks, int page_size,
                     int num_pages, void *out, int B, int h, int n_kv, int d, float scale, long long cache_rows,
                     cudaStream_t stream);
int launch_decode_split(const void *q, const void *k, const void *v, long long cache_rows, const int32_t *seqlens,
                        void *out, int B, int h, int n_kv, int d, float scale, void *workspace, size_t ws_bytes,
                        cudaStream_t stream);
size_t split_workspace_bytes(int B, int h, int n_kv, int d);
int launch_decode_split_noalloc(const void *q, const void *k, const void *v, long long cache_rows,
                                const int32_t *seqlens, void *out, int B, int h, int n_kv, int d, float scale,
                                cudaStream_t stream);
}  // namespace gqa

namespace gqa_host {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

bool encode_tensor_map(CUtensorMap *map, const void *base, int rank, const uint64_t *dims,
                       const uint64_t *strides_bytes, const uint32_t *box) {
    return encode_tensor_map_ex(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_128B, base, rank, dims,
                                strides_bytes, box);
}

bool encode_tensor_map_ex(CUtensorMap *map, CUtensorMapDataType dtype, CUtensorMapSwizzle swizzle,
                          const void *base, int rank, const uint64_t *dims, const uint64_t *strides_bytes,
                          const uint32_t *box) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[5];
    cuuint64_t gstride[4];
    cuuint32_t bdim[5], estride[5];
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        bdim[i] = box[i];
        estride[i] = 1;
        if (i + 1 < rank) gstride[i] = strides_bytes[i];
    }
    CUresult r = fn(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void *>(base),
                    gdim, gstride, bdim, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int *device_status() {
    static int *ptrs[64] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, gqa::g_status) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<int *>(p);
    }
    return ptrs[dev];
}

#ifdef GQA_WAIT_TEST
int *device_test_stall() {
    static int *ptrs[64] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, gqa::g_test_stall) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<int *>(p);
    }
    return ptrs[dev];
}
#endif

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

}  // namespace gqa_host

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool scale_ok(float s) { return std::isfinite(s) && s >= 0.f; }

// The token extent the packed-cache entry points without a row count give
// their tensor maps: the caller's contract covers the rows, and offsets past
// it are cut and reported by the kernels.
constexpr long long kOpenRows = 1LL << 30;

static bool rows_ok(int64_t rows) { return rows >= 0 && rows <= 0x7FFFFFFFLL; }

extern "C" {

int gqa_prefill(const void *q, const void *k, const void *v, void *out, int B, int S_q, int S_kv, int h, int n_kv,
                int d_h, int causal, float scale, cudaStream_t stream) {
    if (!q || !k || !v || !out) return GQA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return GQA_ERR_INVALID_ARG;
    if (B <= 0 || S_q <= 0 || S_kv <= 0 || h <= 0 || n_kv <= 0 || h % n_kv != 0) return GQA_ERR_INVALID_ARG;
    if (causal && S_q > S_kv) return GQA_ERR_INVALID_ARG;
    if (!scale_ok(scale)) return GQA_ERR_INVALID_ARG;
    if (d_h != 64 && d_h != 128) return GQA_ERR_UNSUPPORTED;
    // tensor-map coordinates are int32 per dimension; the extents themselves are int already
    return gqa::launch_prefill(q, k, v, out, B, S_q, S_kv, h, n_kv, d_h, causal, scale, stream);
}

static int decode_bf16(const void *q, const void *k_cache, const void *v_cache, long long cache_rows,
                       const int32_t *seqlens, void *out, int B, int h, int n_kv, int d_h, float scale,
                       cudaStream_t stream) {
    if (!q || !k_cache || !v_cache || !seqlens || !out) return GQA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(seqlens) & 3u))
        return GQA_ERR_INVALID_ARG;
    if (B <= 0 || B > 65535 || h <= 0 || n_kv <= 0 || h % n_kv != 0) return GQA_ERR_INVALID_ARG;
    if (!scale_ok(scale)) return GQA_ERR_INVALID_ARG;
    if (d_h != 64 && d_h != 128) return GQA_ERR_UNSUPPORTED;
    if (static_cast<long>(n_kv) * ((h / n_kv + 63) / 64) > 65535) return GQA_ERR_UNSUPPORTED;
    return gqa::launch_decode(q, k_cache, v_cache, seqlens, out, B, h, n_kv, d_h, scale, cache_rows, stream);
}

int gqa_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens, void *out, int B,
               int h, int n_kv, int d_h, float scale, cudaStream_t stream) {
    return decode_bf16(q, k_cache, v_cache, kOpenRows, seqlens, out, B, h, n_kv, d_h, scale, stream);
}

int gqa_decode_rows(const void *q, const void *k_cache, const void *v_cache, int64_t cache_rows,
                    const int32_t *seqlens, void *out, int B, int h, int n_kv, int d_h, float scale,
                    cudaStream_t stream) {
    if (!rows_ok(cache_rows)) return GQA_ERR_INVALID_ARG;
    return decode_bf16(q, k_cache, v_cache, cache_rows, seqlens, out, B, h, n_kv, d_h, scale, stream);
}

size_t gqa_decode_split_workspace_bytes(int B, int h, int n_kv, int d_h) {
    if (B <= 0 || B > 65535 || h <= 0 || n_kv <= 0 || h % n_kv != 0 || (d_h != 64 && d_h != 128)) return 0;
    if (static_cast<long long>(n_kv) * ((h / n_kv + 127) / 128) * B > (1LL << 24)) return 0;   // as gqa_decode_split
    return gqa::split_workspace_bytes(B, h, n_kv, d_h);
}

int gqa_decode_split(const void *q, const void *k_cache, const void *v_cache, int64_t cache_rows,
                     const int32_t *seqlens, void *out, int B, int h, int n_kv, int d_h, float scale,
                     void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (!rows_ok(cache_rows)) return GQA_ERR_INVALID_ARG;
    if (!q || !k_cache || !v_cache || !seqlens || !out || !workspace) return GQA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(seqlens) & 3u) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return GQA_ERR_INVALID_ARG;
    if (B <= 0 || B > 65535 || h <= 0 || n_kv <= 0 || h % n_kv != 0) return GQA_ERR_INVALID_ARG;
    if (!scale_ok(scale)) return GQA_ERR_INVALID_ARG;
    if (d_h != 64 && d_h != 128) return GQA_ERR_UNSUPPORTED;
    if (static_cast<long long>(n_kv) * ((h / n_kv + 127) / 128) * B > (1LL << 24)) return GQA_ERR_UNSUPPORTED;
    if (workspace_bytes < gqa::split_workspace_bytes(B, h, n_kv, d_h)) return GQA_ERR_INVALID_ARG;
    return gqa::launch_decode_split(q, k_cache, v_cache, cache_rows, seqlens, out, B, h, n_kv, d_h, scale, workspace,
                                    workspace_bytes, stream);
}

int gqa_decode_split_noalloc(const void *q, const void *k_cache, const void *v_cache, int64_t cache_rows,
                             const int32_t *seqlens, void *out, int B, int h, int n_kv, int d_h, float scale,
                             cudaStream_t stream) {
    if (!rows_ok(cache_rows)) return GQA_ERR_INVALID_ARG;
    if (!q || !k_cache || !v_cache || !seqlens || !out) return GQA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(seqlens) & 3u))
        return GQA_ERR_INVALID_ARG;
    if (B <= 0 || B > 65535 || h <= 0 || n_kv <= 0 || h % n_kv != 0) return GQA_ERR_INVALID_ARG;
    if (!scale_ok(scale)) return GQA_ERR_INVALID_ARG;
    if (d_h != 64 && d_h != 128) return GQA_ERR_UNSUPPORTED;
    if (static_cast<long long>(n_kv) * ((h / n_kv + 127) / 128) * B > (1LL << 24)) return GQA_ERR_UNSUPPORTED;
    const int st = gqa::launch_decode_split_noalloc(q, k_cache, v_cache, cache_rows, seqlens, out, B, h, n_kv, d_h,
                                                    scale, stream);
    return st == 0 ? GQA_OK : (st == 1 || st == 2) ? GQA_ERR_UNSUPPORTED : GQA_ERR_CUDA;
}

// Checks shared by every decode entry point (cache pointers are checked by the caller).
static int decode_args_ok(const void *q, const int32_t *seqlens, const void *out, int B, int h, int n_kv, int d_h,
                          float scale) {
    if (!q || !seqlens || !out) return GQA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out) || (reinterpret_cast<uintptr_t>(seqlens) & 3u)) return GQA_ERR_INVALID_ARG;
    if (B <= 0 || B > 65535 || h <= 0 || n_kv <= 0 || h % n_kv != 0) return GQA_ERR_INVALID_ARG;
    if (!scale_ok(scale)) return GQA_ERR_INVALID_ARG;
    if (d_h != 64 && d_h != 128) return GQA_ERR_UNSUPPORTED;
    if (static_cast<long>(n_kv) * ((h / n_kv + 63) / 64) > 65535) return GQA_ERR_UNSUPPORTED;
    return GQA_OK;
}

static int caches_ok(const void *k, const void *v) {
    return (k && v && aligned16(k) && aligned16(v)) ? GQA_OK : GQA_ERR_INVALID_ARG;
}

static int scales_ok(const float *k_scale, const float *v_scale) {
    if (!k_scale || !v_scale) return GQA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(k_scale) & 3u) || (reinterpret_cast<uintptr_t>(v_scale) & 3u))
        return GQA_ERR_INVALID_ARG;
    return GQA_OK;
}

static int pages_ok(const int32_t *block_table, int max_blocks, int page_size, int num_pages) {
    if (!block_table || (reinterpret_cast<uintptr_t>(block_table) & 3u)) return GQA_ERR_INVALID_ARG;
    if (max_blocks <= 0 || num_pages <= 0) return GQA_ERR_INVALID_ARG;
    if (page_size < 16 || page_size > 65536 || (page_size & (page_size - 1))) return GQA_ERR_INVALID_ARG;
    if (static_cast<long long>(max_blocks) * page_size > 0x7FFFFFFFLL) return GQA_ERR_INVALID_ARG;
    return GQA_OK;
}

int gqa_decode_fp8(const void *q, const void *k_cache, const void *v_cache, const float *k_scale,
                   const float *v_scale, const int32_t *seqlens, void *out, int B, int h, int n_kv, int d_h,
                   float scale, cudaStream_t stream) {
    int st = caches_ok(k_cache, v_cache);
    if (st == GQA_OK) st = scales_ok(k_scale, v_scale);
    if (st == GQA_OK) st = decode_args_ok(q, seqlens, out, B, h, n_kv, d_h, scale);
    if (st != GQA_OK) return st;
    return gqa::launch_decode_ex(q, k_cache, v_cache, k_scale, v_scale, seqlens, nullptr, 0, 0, 0, out, B, h, n_kv,
                                 d_h, scale, kOpenRows, stream);
}

int gqa_decode_fp8_rows(const void *q, const void *k_cache, const void *v_cache, int64_t cache_rows,
                        const float *k_scale, const float *v_scale, const int32_t *seqlens, void *out, int B, int h,
                        int n_kv, int d_h, float scale, cudaStream_t stream) {
    if (!rows_ok(cache_rows)) return GQA_ERR_INVALID_ARG;
    int st = caches_ok(k_cache, v_cache);
    if (st == GQA_OK) st = scales_ok(k_scale, v_scale);
    if (st == GQA_OK) st = decode_args_ok(q, seqlens, out, B, h, n_kv, d_h, scale);
    if (st != GQA_OK) return st;
    return gqa::launch_decode_ex(q, k_cache, v_cache, k_scale, v_scale, seqlens, nullptr, 0, 0, 0, out, B, h, n_kv,
                                 d_h, scale, cache_rows, stream);
}

int gqa_decode_paged(const void *q, const void *k_pages, const void *v_pages, const int32_t *block_table,
                     int max_blocks, int page_size, int num_pages, const int32_t *seqlens, void *out, int B, int h,
                     int n_kv, int d_h, float scale, cudaStream_t stream) {
    int st = caches_ok(k_pages, v_pages);
    if (st == GQA_OK) st = pages_ok(block_table, max_blocks, page_size, num_pages);
    if (st == GQA_OK) st = decode_args_ok(q, seqlens, out, B, h, n_kv, d_h, scale);
    if (st != GQA_OK) return st;
    return gqa::launch_decode_ex(q, k_pages, v_pages, nullptr, nullptr, seqlens, block_table, max_blocks, page_size,
                                 num_pages, out, B, h, n_kv, d_h, scale, kOpenRows, stream);
}

int gqa_decode_paged_fp8(const void *q, const void *k_pages, const void *v_pages, const float *k_scale,
                         const float *v_scale, const int32_t *block_table, int max_blocks, int page_size,
                         int num_pages, const int32_t *seqlens, void *out, int B, int h, int n_kv, int d_h,
                         float scale, cudaStream_t stream) {
    int st = caches_ok(k_pages, v_pages);
    if (st == GQA_OK) st = scales_ok(k_scale, v_scale);
    if (st == GQA_OK) st = pages_ok(block_table, max_blocks, page_size, num_pages);
    if (st == GQA_OK) st = decode_args_ok(q, seqlens, out, B, h, n_kv, d_h, scale);
    if (st != GQA_OK) return st;
    return gqa::launch_decode_ex(q, k_pages, v_pages, k_scale, v_scale, seqlens, block_table, max_blocks, page_size,
                                 num_pages, out, B, h, n_kv, d_h, scale, kOpenRows, stream);
}

int gqa_prefill_paged(const void *q, const void *k_new, const void *v_new, void *k_pages, void *v_pages,
                      const int32_t *block_table, int max_blocks, int page_size, int num_pages,
                      const int32_t *past_lens, void *out, int B, int S_q, int h, int n_kv, int d_h, float scale,
                      cudaStream_t stream) {
    if (!q || !k_new || !v_new || !out || !past_lens) return GQA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(past_lens) & 3u))
        return GQA_ERR_INVALID_ARG;
    int st = caches_ok(k_pages, v_pages);
    if (st == GQA_OK) st = pages_ok(block_table, max_blocks, page_size, num_pages);
    if (st != GQA_OK) return st;
    if (B <= 0 || S_q <= 0 || h <= 0 || n_kv <= 0 || h % n_kv != 0) return GQA_ERR_INVALID_ARG;
    if (static_cast<long long>(S_q) > static_cast<long long>(max_blocks) * page_size) return GQA_ERR_INVALID_ARG;
    if (!scale_ok(scale)) return GQA_ERR_INVALID_ARG;
    if (d_h != 64 && d_h != 128) return GQA_ERR_UNSUPPORTED;
    return gqa::launch_prefill_paged(q, k_new, v_new, k_pages, v_pages, block_table, max_blocks, page_size,
                                     num_pages, past_lens, out, B, S_q, h, n_kv, d_h, scale, stream);
}

static int mla_decode(const void *q_absorbed, const void *c_kv, long long cache_rows, bool rows_known,
                      const int32_t *seqlens, void *out, int B, int h, int d_c, float scale, cudaStream_t stream) {
    if (!q_absorbed || !c_kv || !seqlens || !out) return GQA_ERR_INVALID_ARG;
    if (!aligned16(q_absorbed) || !aligned16(c_kv) || !aligned16(out) || (reinterpret_cast<uintptr_t>(seqlens) & 3u))
        return GQA_ERR_INVALID_ARG;
    if (B <= 0 || B > 65535 || h <= 0 || h > 65535 * 16) return GQA_ERR_INVALID_ARG;
    if (!scale_ok(scale)) return GQA_ERR_INVALID_ARG;
    if (d_c != 512) return GQA_ERR_UNSUPPORTED;
    return gqa::launch_mla_decode(q_absorbed, c_kv, seqlens, out, B, h, scale, cache_rows, rows_known, stream);
}

int gqa_mla_decode(const void *q_absorbed, const void *c_kv, const int32_t *seqlens, void *out, int B, int h,
                   int d_c, float scale, cudaStream_t stream) {
    return mla_decode(q_absorbed, c_kv, kOpenRows, false, seqlens, out, B, h, d_c, scale, stream);
}

int gqa_mla_decode_rows(const void *q_absorbed, const void *c_kv, int64_t cache_rows, const int32_t *seqlens,
                        void *out, int B, int h, int d_c, float scale, cudaStream_t stream) {
    if (!rows_ok(cache_rows)) return GQA_ERR_INVALID_ARG;
    return mla_decode(q_absorbed, c_kv, cache_rows, true, seqlens, out, B, h, d_c, scale, stream);
}

int gqa_mla_decode_path(int B, int h, int d_c, int64_t cache_rows, int with_workspace) {
    if (B <= 0 || h <= 0 || d_c != 512 || !rows_ok(cache_rows)) return -1;
    const int sms = gqa_host::sm_count();
    if (with_workspace && gqa::mla_ws_prefers_tc(B, h, cache_rows, sms)) return 2;
    return gqa::mla_prefers_tc(B, h, cache_rows, true, sms) ? 1 : 0;
}

static bool mla_sizes_ok(int B, int h) { return B > 0 && B <= 65535 && h > 0 && h <= 65535 * 16; }

size_t gqa_mla_decode_split_workspace_bytes(int B, int h, int d_c) {
    if (!mla_sizes_ok(B, h) || d_c != 512) return 0;
    return gqa::mla_ws_bytes(B, h, gqa_host::sm_count());
}

int gqa_mla_decode_split(const void *q_absorbed, const void *c_kv, int64_t cache_rows, const int32_t *seqlens,
                         void *out, int B, int h, int d_c, float scale, void *workspace, size_t workspace_bytes,
                         cudaStream_t stream) {
    if (!rows_ok(cache_rows)) return GQA_ERR_INVALID_ARG;
    if (!q_absorbed || !c_kv || !seqlens || !out || !workspace) return GQA_ERR_INVALID_ARG;
    if (!aligned16(q_absorbed) || !aligned16(c_kv) || !aligned16(out) || (reinterpret_cast<uintptr_t>(seqlens) & 3u) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return GQA_ERR_INVALID_ARG;
    if (!mla_sizes_ok(B, h)) return GQA_ERR_INVALID_ARG;
    if (!scale_ok(scale)) return GQA_ERR_INVALID_ARG;
    if (d_c != 512) return GQA_ERR_UNSUPPORTED;
    const int st = gqa::launch_mla_decode_ws(q_absorbed, c_kv, seqlens, out, B, h, scale, cache_rows, workspace,
                                             workspace_bytes, stream);
    return st == 0 ? GQA_OK : st == 1 ? GQA_ERR_INVALID_ARG : GQA_ERR_CUDA;
}

const char *gqa_status_string(int status) {
    switch (status) {
        case GQA_OK: return "GQA_OK";
        case GQA_ERR_INVALID_ARG: return "GQA_ERR_INVALID_ARG: invalid argument";
        case GQA_ERR_UNSUPPORTED: return "GQA_ERR_UNSUPPORTED: unsupported configuration";
        case GQA_ERR_CUDA: return "GQA_ERR_CUDA: CUDA launch failure";
        case GQA_ERR_TIMEOUT: return "GQA_ERR_TIMEOUT: a kernel gave up on an internal wait";
        default: return "unknown gqa status";
    }
}

int gqa_get_device_status(cudaStream_t stream) {
    // one reader at a time per process: the exchanged value passes through g_status_taken
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    gqa::take_status_kernel<<<1, 1, 0, stream>>>();
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, gqa::g_status_taken, sizeof(int), 0, cudaMemcpyDeviceToHost, stream) !=
        cudaSuccess)
        return GQA_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GQA_ERR_CUDA;
    return v;
}

#ifdef GQA_WAIT_TEST
int gqa_test_set_stall(int on) {
    const int v = on ? 1 : 0;
    return cudaMemcpyToSymbol(gqa::g_test_stall, &v, sizeof(int)) == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}
#endif

}  // extern "C"
