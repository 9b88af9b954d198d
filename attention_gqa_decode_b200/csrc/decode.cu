// Decode: one query token per sequence against a packed bf16 KV cache.
//
// Semantics: "Multi-Query Attention" (inferensys glossary), "Decoding Step":
// softmax(Q_all K_shared^T) V_shared, generalised to G = h / n_kv query heads
// per shared K/V head ("Evolution of AI Attention Mechanisms" (toolsku),
// "GQA Implementation": query head i reads KV head i / (h / n_kv)).
//
// Design (B200): the step is bound by HBM bandwidth ("Multi-query
// attention" (pranaymahendrakar), "Why this is a bandwidth argument": the
// bytes read scale with n_kv, the FLOPs do not).  So each CTA owns one
// (sequence b, KV head g, split s) and streams its token range of K/V head g
// from HBM exactly once for all G query heads of the group:
//   - a producer warp issues 128-byte-swizzled TMA tile loads (64 tokens x
//     64 dims per box) into a ring of shared-memory stages, completion on
//     mbarriers;
//   - four consumer warps compute S = Q K^T and O += P V on the tensor cores
//     (m16n8k16, the G query heads of the group as the M rows, padded to 16),
//     with the online softmax (running max and running sum, rescaling O when
//     the max grows) in registers between the two products.  Every consumer
//     warp takes every stage, in order (warp = m-tile x token sub-range of the
//     stage), so a warp never waits on a ring slot more than one phase ahead;
//   - the P splits of one (b, g) form a thread-block cluster; their partial
//     (max, sum, O) triples are merged through distributed shared memory
//     with the log-sum-exp rule and rank-parallel bf16 stores.  No global
//     scratch memory is used.
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"

#ifndef GQA_DECODE_CTAS_PER_SM
#define GQA_DECODE_CTAS_PER_SM 2   // resident CTAs per SM (shared memory allows two)
#endif
#ifndef GQA_DECODE_MAX_SPLIT
#define GQA_DECODE_MAX_SPLIT 8     // splits per (sequence, KV head) = thread-block cluster size
#endif

namespace cg = cooperative_groups;

namespace gqa {

constexpr int kDecTok = 64;        // tokens per pipeline stage
constexpr int kDecWarps = 4;       // consumer warps
constexpr int kDecThreads = (kDecWarps + 1) * 32;
constexpr int kDecMaxHeads = 64;   // query heads one CTA serves (4 m-tiles of 16)

struct DecodeParams {
    const __nv_bfloat16 *q;
    const int32_t *seqlens;
    __nv_bfloat16 *out;
    int B, h, n_kv, G, slices;     // slices = ceil(G / kDecMaxHeads)
    float scale_log2;              // scale * log2(e), >= 0
    int *status;                   // the library's device status word
};

template <int D, int STAGES>
struct DecodeSmem {
    static constexpr uint32_t kTileBytes = kDecTok * D * 2;          // K or V of one stage
    static constexpr uint32_t kStageBytes = 2 * kTileBytes;
    static constexpr uint32_t kRingBytes = STAGES * kStageBytes;
    static constexpr uint32_t kCtrlBytes = 256;                       // barriers, flags
    static constexpr uint32_t kTotal = kRingBytes + kCtrlBytes + 1024;  // + alignment slack
    // After the ring has drained it is reused for the partial results:
    //   per-warp partials  part[WT][HS][D], pm[WT][HS], pl[WT][HS]
    //   per-CTA partial    co[HS][D], cm[HS], cl[HS]
    static constexpr uint32_t kPartBytes = 4 * 16 * D * 4;            // WT * HS <= 64 rows
    static_assert(kPartBytes * 2 + 4 * 64 * 4 <= kRingBytes, "partials must fit in the drained ring");
};

// WT = token sub-ranges per stage (4, 2 or 1): consumer warp w serves m-tile
// w / WT (16 query heads) on tokens [(w % WT) * 64 / WT, ...) of every stage.
template <int D, int STAGES, int WT>
__global__ void __launch_bounds__(kDecThreads, 2)
    gqa_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const DecodeParams p) {
    using SM = DecodeSmem<D, STAGES>;
    constexpr int KSTEPS = D / 16;     // k-steps of Q K^T
    constexpr int NT_O = D / 8;        // n-tiles of O (dims)
    constexpr int TPW = kDecTok / WT;  // tokens of a stage one warp handles
    constexpr int NTS = TPW / 8;       // n-tiles of its scores
    constexpr int KKS = TPW / 16;      // k-steps of its P V
    constexpr int HALF_BYTES = kDecTok * 128;   // one 64-dim half of a tile

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + SM::kRingBytes);
    uint64_t *empty = full + STAGES;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + STAGES);
    int *red = reinterpret_cast<int *>(empty + STAGES) + 1;   // [kDecWarps + 1] partial sums

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = gridDim.x, split = blockIdx.x;
    const int b = blockIdx.z;
    const int g = blockIdx.y / p.slices, slice = blockIdx.y % p.slices;
    const int head0 = g * p.G + slice * kDecMaxHeads;
    const int HS = min(p.G - slice * kDecMaxHeads, kDecMaxHeads);
    const int WM = (HS + 15) >> 4;                  // m-tiles (WM * WT <= 4, chosen by the host)

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], WM * WT);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kDecWarps && lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }

    // first cache row of sequence b: sum of the earlier (non-negative) lengths
    int acc = 0;
    for (int i = threadIdx.x; i < b; i += kDecThreads) acc += max(p.seqlens[i], 0);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) red[warp] = acc;
    __syncthreads();
    int off = 0;
#pragma unroll
    for (int w = 0; w <= kDecWarps; ++w) off += red[w];
    const int L = max(p.seqlens[b], 0);

    // this split's stages: stage i covers tokens [t0, min(t0 + 64, L)), t0 = 64 * (first + i)
    const int n_total = (L + kDecTok - 1) / kDecTok;
    const int per_split = (n_total + P - 1) / P;
    const int first = split * per_split;
    const int n_stages = max(0, min(n_total, first + per_split) - first);

    if (warp == kDecWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < n_stages; ++i) {
                const int slot = i % STAGES, use = i / STAGES;
                if (use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1, abort_flag, p.status)) break;
                const int t0 = (first + i) * kDecTok;
                // The last stage of a sequence is shifted back so it ends at the
                // sequence end: the box never reads past the packed cache.
                const int z = off + min(t0, L - kDecTok);
                uint8_t *kdst = smem + slot * SM::kStageBytes;
                uint8_t *vdst = kdst + SM::kTileBytes;
                mbar_arrive_expect_tx(&full[slot], SM::kStageBytes);
#pragma unroll
                for (int hf = 0; hf < D / 64; ++hf) {
                    tma_load_3d(kdst + hf * HALF_BYTES, &tm_k, &full[slot], hf * 64, g, z);
                    tma_load_3d(vdst + hf * HALF_BYTES, &tm_v, &full[slot], hf * 64, g, z);
                }
                ++issued;
            }
            if (*abort_flag) {   // let the copies in flight land before the CTA moves on
                for (int i = max(0, issued - STAGES); i < issued; ++i)
                    mbar_wait_drain(&full[i % STAGES], (i / STAGES) & 1, p.status);
            }
        }
        __syncwarp();
    }

    // consumer state (kept outside the branch so every thread reaches the
    // shared-memory reuse below)
    const int mi = warp / WT, ti = warp % WT;
    const bool consumer = warp < kDecWarps && mi < WM;
    float o[NT_O][4];
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < NT_O; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;

    if (consumer) {
        // ------------------------------------------------------------ consumers
        // Q fragments of m-tile mi (rows = query heads of the group), kept in registers
        const int r0 = mi * 16 + (lane >> 2), r1 = r0 + 8;
        const int cq = 2 * (lane & 3);
        const __nv_bfloat16 *qb = p.q + (static_cast<size_t>(b) * p.h + head0) * D;
        uint32_t qa[KSTEPS][4];
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
            const int c = ks * 16 + cq;
            qa[ks][0] = r0 < HS ? *reinterpret_cast<const uint32_t *>(qb + r0 * D + c) : 0u;
            qa[ks][1] = r1 < HS ? *reinterpret_cast<const uint32_t *>(qb + r1 * D + c) : 0u;
            qa[ks][2] = r0 < HS ? *reinterpret_cast<const uint32_t *>(qb + r0 * D + c + 8) : 0u;
            qa[ks][3] = r1 < HS ? *reinterpret_cast<const uint32_t *>(qb + r1 * D + c + 8) : 0u;
        }
        const float cl2 = p.scale_log2;
        const int tw0 = ti * TPW;                                   // first row of this warp's tokens
        // ldmatrix lane roles
        const uint32_t lrow = ((lane >> 4) & 1) * 8 + (lane & 7);   // QK: token within a 16-token pair
        const uint32_t lchk = (lane >> 3) & 1;                      // QK: low/high 8 dims of a k-step
        const uint32_t vrow = ((lane >> 3) & 1) * 8 + (lane & 7);   // PV: token within a 16-token k-step
        const uint32_t vchk = lane >> 4;                            // PV: which 8-dim n-tile of a pair

        for (int i = 0; i < n_stages; ++i) {
            const int slot = i % STAGES, use = i / STAGES;
            const bool landed = mbar_wait(&full[slot], use & 1, abort_flag, p.status);
            if (!__all_sync(0xffffffffu, landed)) break;   // warp-uniform: the mma/ldmatrix below are .aligned
            const int t0 = (first + i) * kDecTok;
            const int row_lo = max(0, t0 - (L - kDecTok));   // rows of the box before this stage's tokens
            if (row_lo >= tw0 + TPW) {                      // none of this warp's rows are new tokens
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[slot]);
                continue;
            }
            const uint32_t kbase = smem_u32(smem + slot * SM::kStageBytes) + tw0 * 128;
            const uint32_t vbase = kbase + SM::kTileBytes;

            // S = Q K^T  (16 heads x TPW tokens)
            float s[NTS][4];
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
                const uint32_t chunk = 2 * ks + lchk;
                const uint32_t hbase = kbase + (chunk >> 3) * HALF_BYTES + ((((chunk & 7) ^ (lane & 7))) << 4);
#pragma unroll
                for (int np = 0; np < NTS / 2; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(b0, b1, b2, b3, hbase + (np * 16 + lrow) * 128);
                    mma_bf16_16816(s[2 * np], qa[ks], b0, b1);
                    mma_bf16_16816(s[2 * np + 1], qa[ks], b2, b3);
                }
            }
            // online softmax over these tokens (rows r0 and r1 of the m-tile)
            const bool partial = row_lo > tw0;
            if (partial) {
#pragma unroll
                for (int nt = 0; nt < NTS; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (tw0 + nt * 8 + cq + (e & 1) < row_lo) s[nt][e] = -INFINITY;
            }
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt) {
                mx[0] = fmax3(mx[0], s[nt][0], s[nt][1]);
                mx[1] = fmax3(mx[1], s[nt][2], s[nt][3]);
            }
            float alpha[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
                const float m_new = fmaxf(m_run[r], mx[r] * cl2);   // mx is finite: >= 1 new token
                alpha[r] = exp2f(m_run[r] - m_new);
                m_run[r] = m_new;
                l_run[r] *= alpha[r];
            }
#pragma unroll
            for (int nt = 0; nt < NT_O; ++nt) {
                o[nt][0] *= alpha[0];
                o[nt][1] *= alpha[0];
                o[nt][2] *= alpha[1];
                o[nt][3] *= alpha[1];
            }
            // P as bf16 A fragments; the running sums add the rounded weights
            uint32_t pa[KKS][4];
            float2 ls0 = make_float2(0.f, 0.f), ls1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt) {
                const float2 x0 = ffma2_bcast(s[nt][0], s[nt][1], cl2, -m_run[0]);
                const float2 x1 = ffma2_bcast(s[nt][2], s[nt][3], cl2, -m_run[1]);
                float e0 = exp2f(x0.x), e1 = exp2f(x0.y), e2 = exp2f(x1.x), e3 = exp2f(x1.y);
                if (partial) {   // masked tokens add nothing (also when scale == 0)
                    const int tok = tw0 + nt * 8 + cq;
                    if (tok < row_lo) {
                        e0 = 0.f;
                        e2 = 0.f;
                    }
                    if (tok + 1 < row_lo) {
                        e1 = 0.f;
                        e3 = 0.f;
                    }
                }
                const uint32_t lo = pack_bf16x2(e0, e1), hi = pack_bf16x2(e2, e3);
                pa[nt >> 1][(nt & 1) * 2 + 0] = lo;
                pa[nt >> 1][(nt & 1) * 2 + 1] = hi;
                ls0 = fadd2(ls0, unpack_bf16x2(lo));
                ls1 = fadd2(ls1, unpack_bf16x2(hi));
            }
            l_run[0] += ls0.x + ls0.y;
            l_run[1] += ls1.x + ls1.y;
            // O += P V
#pragma unroll
            for (int kk = 0; kk < KKS; ++kk) {
                const uint32_t rowaddr = vbase + (kk * 16 + vrow) * 128;
#pragma unroll
                for (int dp = 0; dp < NT_O / 2; ++dp) {
                    const uint32_t chunk = 2 * dp + vchk;
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4_trans(b0, b1, b2, b3,
                                      rowaddr + (chunk >> 3) * HALF_BYTES + (((chunk & 7) ^ (lane & 7)) << 4));
                    mma_bf16_16816(o[2 * dp], pa[kk], b0, b1);
                    mma_bf16_16816(o[2 * dp + 1], pa[kk], b2, b3);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
            l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
        }
    }

    // ---------------------------------------------------------------- combine
    __syncthreads();   // the ring has drained: reuse it for the partials
    float *part = reinterpret_cast<float *>(smem);               // [WT][HS][D]
    float *pm = part + 4 * 16 * D;                               // [WT][HS]
    float *pl = pm + 64;                                         // [WT][HS]
    float *co = reinterpret_cast<float *>(smem + SM::kPartBytes + 4 * 64 * 2);   // [HS][D]
    float *cm = co + 64 * D;                                     // [HS]
    float *cl = cm + 64;                                         // [HS]
    if (consumer) {
        const int r0 = mi * 16 + (lane >> 2), r1 = r0 + 8;
        const int cq = 2 * (lane & 3);
#pragma unroll
        for (int nt = 0; nt < NT_O; ++nt) {
            if (r0 < HS) *reinterpret_cast<float2 *>(&part[(ti * HS + r0) * D + nt * 8 + cq]) = make_float2(o[nt][0], o[nt][1]);
            if (r1 < HS) *reinterpret_cast<float2 *>(&part[(ti * HS + r1) * D + nt * 8 + cq]) = make_float2(o[nt][2], o[nt][3]);
        }
        if ((lane & 3) == 0) {
            if (r0 < HS) { pm[ti * HS + r0] = m_run[0]; pl[ti * HS + r0] = l_run[0]; }
            if (r1 < HS) { pm[ti * HS + r1] = m_run[1]; pl[ti * HS + r1] = l_run[1]; }
        }
    }
    __syncthreads();
    // merge the WT token groups of this CTA: item = (head row, pair of dims)
    for (int it = threadIdx.x; it < HS * (D / 2); it += kDecThreads) {
        const int r = it / (D / 2), c = 2 * (it % (D / 2));
        float M = -INFINITY;
        for (int t = 0; t < WT; ++t) M = fmaxf(M, pm[t * HS + r]);
        float sl = 0.f, s0 = 0.f, s1 = 0.f;
        if (M != -INFINITY) {
            for (int t = 0; t < WT; ++t) {
                const float w = exp2f(pm[t * HS + r] - M);
                sl += w * pl[t * HS + r];
                const float2 v = *reinterpret_cast<const float2 *>(&part[(t * HS + r) * D + c]);
                s0 += w * v.x;
                s1 += w * v.y;
            }
        }
        *reinterpret_cast<float2 *>(&co[r * D + c]) = make_float2(s0, s1);
        if (c == 0) { cm[r] = M; cl[r] = sl; }
    }

    __nv_bfloat16 *ob = p.out + (static_cast<size_t>(b) * p.h + head0) * D;
    const bool ok = (*abort_flag == 0);
    if (P == 1) {
        __syncthreads();
        for (int it = threadIdx.x; it < HS * (D / 2); it += kDecThreads) {
            const int r = it / (D / 2), c = 2 * (it % (D / 2));
            const float inv = cl[r] > 0.f ? 1.f / cl[r] : 0.f;
            const float2 v = *reinterpret_cast<const float2 *>(&co[r * D + c]);
            if (ok) *reinterpret_cast<__nv_bfloat162 *>(ob + r * D + c) = __floats2bfloat162_rn(v.x * inv, v.y * inv);
        }
        return;
    }
    // merge across the P splits of the cluster; rank s finalises rows r = s, s + P, ...
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int nrows = (HS - split + P - 1) / P;
    for (int it = threadIdx.x; it < nrows * (D / 2); it += kDecThreads) {
        const int r = split + P * (it / (D / 2)), c = 2 * (it % (D / 2));
        float M = -INFINITY;
        for (int q = 0; q < P; ++q) M = fmaxf(M, *cluster.map_shared_rank(&cm[r], q));
        float sl = 0.f, s0 = 0.f, s1 = 0.f;
        if (M != -INFINITY) {
            for (int q = 0; q < P; ++q) {
                const float w = exp2f(*cluster.map_shared_rank(&cm[r], q) - M);
                sl += w * *cluster.map_shared_rank(&cl[r], q);
                const float2 v = *reinterpret_cast<const float2 *>(cluster.map_shared_rank(&co[r * D + c], q));
                s0 += w * v.x;
                s1 += w * v.y;
            }
        }
        const float inv = sl > 0.f ? 1.f / sl : 0.f;
        if (ok) *reinterpret_cast<__nv_bfloat162 *>(ob + r * D + c) = __floats2bfloat162_rn(s0 * inv, s1 * inv);
    }
    cluster.sync();   // no CTA leaves while a peer may still read its shared memory
}

// ---------------------------------------------------------------------------
// host launcher

template <int D, int STAGES, int WT>
static int launch_decode_t(const void *q, const void *k, const void *v, const int32_t *seqlens, void *out, int B,
                           int h, int n_kv, float scale, cudaStream_t stream) {
    using SM = DecodeSmem<D, STAGES>;
    auto kern = gqa_decode_kernel<D, STAGES, WT>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 3;
    static unsigned long long attr_done = 0;   // one bit per device
    if (dev < 64 && !(attr_done >> dev & 1ull)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kTotal) != cudaSuccess)
            return 3;
        if (GQA_DECODE_MAX_SPLIT > 8 &&
            cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
            return 3;
        attr_done |= 1ull << dev;
    }
    CUtensorMap tk, tv;
    const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(n_kv), 1ull << 30};
    const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(n_kv) * D * 2};
    const uint32_t box[3] = {64, 1, kDecTok};
    if (!gqa_host::encode_tensor_map(&tk, k, 3, dims, strides, box)) return 3;
    if (!gqa_host::encode_tensor_map(&tv, v, 3, dims, strides, box)) return 3;

    const int G = h / n_kv;
    const int slices = (G + kDecMaxHeads - 1) / kDecMaxHeads;
    const long units = static_cast<long>(B) * n_kv * slices;
    const int sms = gqa_host::sm_count();
    // Splits per (sequence, KV head): as many as fit in one wave of resident
    // CTAs (two per SM), at most the cluster limit.  Longer CTAs amortise their
    // start and merge; a second, partial wave would leave SMs idle at the end.
    const long slots = static_cast<long>(GQA_DECODE_CTAS_PER_SM) * sms;
    const int P = static_cast<int>(std::max(1L, std::min(static_cast<long>(GQA_DECODE_MAX_SPLIT), slots / units)));

    DecodeParams prm;
    prm.q = static_cast<const __nv_bfloat16 *>(q);
    prm.seqlens = seqlens;
    prm.out = static_cast<__nv_bfloat16 *>(out);
    prm.B = B;
    prm.h = h;
    prm.n_kv = n_kv;
    prm.G = G;
    prm.slices = slices;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.status = gqa_host::device_status();
    if (!prm.status) return 3;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P, n_kv * slices, B);
    cfg.blockDim = dim3(kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = SM::kTotal;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = P;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tk, tv, prm) != cudaSuccess) return 3;
    return 0;
}

template <int D, int STAGES>
static int launch_decode_d(const void *q, const void *k, const void *v, const int32_t *seqlens, void *out, int B,
                           int h, int n_kv, float scale, cudaStream_t stream) {
    const int HS = min(h / n_kv, kDecMaxHeads);   // query heads per CTA
    if (HS <= 16) return launch_decode_t<D, STAGES, 4>(q, k, v, seqlens, out, B, h, n_kv, scale, stream);
    if (HS <= 32) return launch_decode_t<D, STAGES, 2>(q, k, v, seqlens, out, B, h, n_kv, scale, stream);
    return launch_decode_t<D, STAGES, 1>(q, k, v, seqlens, out, B, h, n_kv, scale, stream);
}

int launch_decode(const void *q, const void *k, const void *v, const int32_t *seqlens, void *out, int B, int h,
                  int n_kv, int d, float scale, cudaStream_t stream) {
    if (d == 128) return launch_decode_d<128, 3>(q, k, v, seqlens, out, B, h, n_kv, scale, stream);
    return launch_decode_d<64, 6>(q, k, v, seqlens, out, B, h, n_kv, scale, stream);
}

}  // namespace gqa
