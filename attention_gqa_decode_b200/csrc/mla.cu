// Absorbed multi-head latent attention (MLA) decode.
//
// Semantics: "Evolution of AI Attention Mechanisms" (toolsku), "Generation 3:
// MLA Multi-Head Latent Attention": the cache holds one latent vector c_kv of
// width d_c per token, shared by every head; with the key up-projection
// absorbed into the query (q' = q W_k_up, computed by the caller), the scores
// are q' c_kv^T * scale and the softmax weights multiply c_kv itself (the
// page's "attn_to_c").  This is decode of one KV head whose keys and values
// are the same d_c = 512 wide rows.
//
// Design (B200): HBM-bound like the other decodes, but 512 wide: a 16-head
// score tile against 32 tokens needs the whole 512-long contraction, and
// O (16 heads x 512) does not fit one warp's registers.  So each CTA owns
// (split, group of 16 heads, sequence) and its four consumer warps split the
// latent width: warp w holds q' and O for dims [128 w, 128 w + 128) and
// computes the partial scores over its dims (m16n8k16, heads as M rows).  The
// four partial score tiles are summed through shared memory (mbarrier
// handshakes with bounded waits), every warp then runs the same online
// softmax on the same sums, and P V touches only its own dims.  Each latent
// byte comes from HBM once per 16-head group (groups of one sequence are
// adjacent CTAs, so larger head counts read it again from L2).  A producer
// warp streams 32-token stages of the packed cache (eight 64-dim panels of
// 128-byte rows, 128B-swizzled TMA boxes) into a 3-stage ring.  The splits of
// one (group, sequence) form a cluster and merge through distributed shared
// memory, as in the GQA decode.  No global scratch.
#include <cooperative_groups.h>

#include <algorithm>

#include <type_traits>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace gqa {

constexpr int kMlaDc = 512;                       // latent width
constexpr int kMlaTok = 32;                       // tokens per stage
constexpr int kMlaStages = 3;
constexpr int kMlaWarps = 4;                      // consumer warps: warp w owns dims [128 w, 128 w + 128)
constexpr int kMlaThreads = (kMlaWarps + 1) * 32;
constexpr int kMlaHeads = 16;                     // query heads per CTA (one m-tile)
constexpr int kMlaPanels = kMlaDc / 64;           // 64-dim panels of 128-byte rows
constexpr int kMlaPanelBytes = kMlaTok * 128;
constexpr int kMlaStageBytes = kMlaPanels * kMlaPanelBytes;   // 32 KB
constexpr int kMlaMaxSplit = 8;
constexpr float kMlaRescale = 8.0f;               // lazy rescale threshold (log2 units)
// The softmax weights reach the tensor cores as bf16.  For a sequence of at
// most this many tokens, where a few keys can carry most of a row's weight,
// they also go as the bf16 remainder p - bf16(p) in a second product.
constexpr int kMlaSplitAllBelow = 256;

struct MlaParams {
    const __nv_bfloat16 *q;
    const int32_t *seqlens;
    __nv_bfloat16 *out;
    int B, h, groups;              // groups = ceil(h / 16)
    long long cache_rows;          // rows the latent cache holds (the tensor map's extent)
    float scale_log2;              // scale * log2(e), >= 0
    int *status;
    GQA_TEST_STALL_FIELD
};

struct MlaSmem {
    static constexpr uint32_t kRing = kMlaStages * kMlaStageBytes;
    static constexpr uint32_t kRed = kMlaWarps * 4 * 32 * 16;    // partial scores: [warp][n-tile][lane] float4
    static constexpr uint32_t kCtrl = 256;
    static constexpr uint32_t kTotal = kRing + kRed + kCtrl + 1024;
    // after the ring drains: co[16][512] fp32, cm[16], cl[16]
    static_assert(kMlaHeads * kMlaDc * 4 + 2 * 64 * 4 <= kRing, "partials must fit in the drained ring");
};

__global__ void __launch_bounds__(kMlaThreads, 2)
    gqa_mla_decode_kernel(const __grid_constant__ CUtensorMap tm_c, const MlaParams p) {
    constexpr int KSTEPS = 128 / 16;               // k-steps of a warp's partial scores
    constexpr int NTS = kMlaTok / 8;               // n-tiles of the scores
    constexpr int KKS = kMlaTok / 16;              // k-steps of P V
    constexpr int NT_O = 128 / 8;                  // n-tiles of a warp's O
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float4 *sred = reinterpret_cast<float4 *>(smem + MlaSmem::kRing);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + MlaSmem::kRing + MlaSmem::kRed);
    uint64_t *empty = full + kMlaStages;
    uint64_t *sfull = empty + kMlaStages;          // all partial scores of a stage written
    uint64_t *sfree = sfull + 1;                   // all partial scores of a stage read
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sfree + 1);
    long long *red = reinterpret_cast<long long *>(sfree + 2);   // [kMlaWarps + 1]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = gridDim.x, split = blockIdx.x;
    const int grp = blockIdx.y, b = blockIdx.z;
    const int head0 = grp * kMlaHeads;
    const int HS = min(p.h - head0, kMlaHeads);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kMlaStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kMlaWarps);
        }
        mbar_init(sfull, kMlaWarps);
        mbar_init(sfree, kMlaWarps);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kMlaWarps && lane == 0) tma_prefetch_desc(&tm_c);

    // first cache row of sequence b (64-bit sum of the earlier non-negative lengths)
    long long acc = 0;
    for (int i = threadIdx.x; i < b; i += kMlaThreads) acc += max(p.seqlens[i], 0);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) red[warp] = acc;
    __syncthreads();
    long long off64 = 0;
#pragma unroll
    for (int w = 0; w <= kMlaWarps; ++w) off64 += red[w];
    int L = max(p.seqlens[b], 0);
    if (off64 + L > p.cache_rows) {   // the lengths ask for rows the cache does not hold
        if (threadIdx.x == 0) record_status(p.status, kStatusInvalid);
        L = static_cast<int>(max(0LL, p.cache_rows - off64));
    }
    // off + L <= cache_rows <= INT32_MAX whenever a row is read (the host bounds cache_rows)
    const int off = static_cast<int>(min(off64, p.cache_rows));
    const int n_total = (L + kMlaTok - 1) / kMlaTok;
    const int per_split = (n_total + P - 1) / P;
    const int first = split * per_split;
    const int n_stages = max(0, min(n_total, first + per_split) - first);

    if (warp == kMlaWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0;
            const int first_loaded = GQA_STALLED(p) ? 1 : 0;   // wait-test build: stage 0 never arrives
            for (int i = 0; i < n_stages; ++i) {
                const int slot = i % kMlaStages, use = i / kMlaStages;
                if (use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1, abort_flag, p.status)) break;
                if (i < first_loaded) {
                    ++issued;
                    continue;
                }
                const int t0 = (first + i) * kMlaTok;
                // the last stage is shifted back to end at the sequence end (never past the cache)
                const int z = off + min(t0, L - kMlaTok);
                uint8_t *dst = smem + slot * kMlaStageBytes;
                mbar_arrive_expect_tx(&full[slot], kMlaStageBytes);
#pragma unroll
                for (int pp = 0; pp < kMlaPanels; ++pp)
                    tma_load_2d(dst + pp * kMlaPanelBytes, &tm_c, &full[slot], pp * 64, z);
                ++issued;
            }
            if (*abort_flag) {
                for (int i = max(first_loaded, issued - kMlaStages); i < issued; ++i)
                    mbar_wait_drain(&full[i % kMlaStages], (i / kMlaStages) & 1, p.status);
            }
        }
        __syncwarp();
    }

    const bool consumer = warp < kMlaWarps;
    const int dq = warp;                            // this warp's quarter of the latent width
    float o[NT_O][4];
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < NT_O; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;

    if (consumer) {
        // ------------------------------------------------------------ consumers
        const int r0 = lane >> 2, r1 = r0 + 8;     // head rows of the m-tile
        const int cq = 2 * (lane & 3);
        const __nv_bfloat16 *qb = p.q + (static_cast<size_t>(b) * p.h + head0) * kMlaDc + dq * 128;
        uint32_t qa[KSTEPS][4];
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
            const int c = ks * 16 + cq;
            qa[ks][0] = r0 < HS ? *reinterpret_cast<const uint32_t *>(qb + r0 * kMlaDc + c) : 0u;
            qa[ks][1] = r1 < HS ? *reinterpret_cast<const uint32_t *>(qb + r1 * kMlaDc + c) : 0u;
            qa[ks][2] = r0 < HS ? *reinterpret_cast<const uint32_t *>(qb + r0 * kMlaDc + c + 8) : 0u;
            qa[ks][3] = r1 < HS ? *reinterpret_cast<const uint32_t *>(qb + r1 * kMlaDc + c + 8) : 0u;
        }
        const float cl2 = p.scale_log2;
        const uint32_t lrow = ((lane >> 4) & 1) * 8 + (lane & 7);   // scores: token within a 16-token pair
        const uint32_t lchk = (lane >> 3) & 1;                      //   low/high 8 dims of a k-step
        const uint32_t vrow = ((lane >> 3) & 1) * 8 + (lane & 7);   // P V: token within a 16-token k-step
        const uint32_t vchk = lane >> 4;                            //   which 8-dim n-tile of a pair

        // partial scores over this warp's 128 dims (16 heads x 32 tokens) of the stage at `stage`
        auto partial_scores = [&](uint32_t stage, float (&s)[NTS][4]) {
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
                const uint32_t chunk = 2 * ks + lchk;                     // 16-byte chunk within the quarter
                const uint32_t hbase = stage + (dq * 2 + (chunk >> 3)) * kMlaPanelBytes +
                                       ((((chunk & 7) ^ (lane & 7))) << 4);
#pragma unroll
                for (int np = 0; np < NTS / 2; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(b0, b1, b2, b3, hbase + (np * 16 + lrow) * 128);
                    mma_bf16_16816(s[2 * np], qa[ks], b0, b1);
                    mma_bf16_16816(s[2 * np + 1], qa[ks], b2, b3);
                }
            }
        };
        auto stage_addr = [&](int i) { return smem_u32(smem + (i % kMlaStages) * kMlaStageBytes); };
        auto landed = [&](int i) {
            return __all_sync(0xffffffffu, mbar_wait(&full[i % kMlaStages], (i / kMlaStages) & 1, abort_flag, p.status));
        };

        // Software-pipelined: the partial scores of stage i + 1 are computed between
        // publishing this warp's partial of stage i and waiting for the other warps'.
        float s[NTS][4];
        bool ok = n_stages == 0 || landed(0);
        if (ok && n_stages > 0) partial_scores(stage_addr(0), s);
        // the stage loop, compiled twice: with the weights' bf16 remainders (sequences of at
        // most kMlaSplitAllBelow tokens) and without, so the long-sequence path carries no
        // extra registers
        auto stage_loop = [&](auto split_tag) {
            constexpr bool kSplit = decltype(split_tag)::value;
        for (int i = 0; i < n_stages && ok; ++i) {
            const int slot = i % kMlaStages;
            const int t0 = (first + i) * kMlaTok;
            const int row_lo = max(0, t0 - (L - kMlaTok));   // rows of the box before this stage's tokens
            const uint32_t stage = stage_addr(i);

            // publish this warp's partial once every warp has read the previous stage's
            if (i > 0 && !__all_sync(0xffffffffu, mbar_wait(sfree, (i - 1) & 1, abort_flag, p.status))) break;
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt)
                sred[(warp * NTS + nt) * 32 + lane] = make_float4(s[nt][0], s[nt][1], s[nt][2], s[nt][3]);
            __syncwarp();
            if (lane == 0) mbar_arrive(sfull);
            float sn[NTS][4];
            if (i + 1 < n_stages) {
                if (!landed(i + 1)) break;
                partial_scores(stage_addr(i + 1), sn);
            }
            // the sum of the four partials (the same order in every warp)
            if (!__all_sync(0xffffffffu, mbar_wait(sfull, i & 1, abort_flag, p.status))) break;
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt) {
                float4 t = sred[nt * 32 + lane];
#pragma unroll
                for (int w = 1; w < kMlaWarps; ++w) {
                    const float4 u = sred[(w * NTS + nt) * 32 + lane];
                    t.x += u.x;
                    t.y += u.y;
                    t.z += u.z;
                    t.w += u.w;
                }
                s[nt][0] = t.x;
                s[nt][1] = t.y;
                s[nt][2] = t.z;
                s[nt][3] = t.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(sfree);

            // online softmax (the same sums in every warp, so the same state)
            const bool partial = row_lo > 0;
            if (partial) {
#pragma unroll
                for (int nt = 0; nt < NTS; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (nt * 8 + cq + (e & 1) < row_lo) s[nt][e] = -INFINITY;
            }
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt) {
                mx[0] = fmax3(mx[0], s[nt][0], s[nt][1]);
                mx[1] = fmax3(mx[1], s[nt][2], s[nt][3]);
            }
            // lazy rescale: the running max moves only when a row's stage max exceeds it
            // by 2^8 (every warp sees the same sums, so all take the same decisions)
            float m_tile[2];
            bool need = false;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
                m_tile[r] = mx[r] * cl2;                             // >= 1 valid token per stage
                need |= m_tile[r] > m_run[r] + kMlaRescale;
            }
            if (i == 0) {
                m_run[0] = m_tile[0];
                m_run[1] = m_tile[1];
            } else if (__any_sync(0xffffffffu, need)) {
                float alpha[2];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const float m_new = fmaxf(m_run[r], m_tile[r]);
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
            }
            constexpr bool split = kSplit;
            uint32_t pa[KKS][4], par[KKS][4];   // the weights and, on split stages, their bf16 remainders
            float2 ls0 = make_float2(0.f, 0.f), ls1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt) {
                const float2 y0 = ffma2_bcast(s[nt][0], s[nt][1], cl2, -m_run[0]);
                const float2 y1 = ffma2_bcast(s[nt][2], s[nt][3], cl2, -m_run[1]);
                float e0 = exp2f(y0.x), e1 = exp2f(y0.y), e2 = exp2f(y1.x), e3 = exp2f(y1.y);
                if (partial) {
                    const int tok = nt * 8 + cq;
                    if (tok < row_lo) e0 = e2 = 0.f;
                    if (tok + 1 < row_lo) e1 = e3 = 0.f;
                }
                const uint32_t lo = pack_bf16x2(e0, e1), hi = pack_bf16x2(e2, e3);
                pa[nt >> 1][(nt & 1) * 2 + 0] = lo;
                pa[nt >> 1][(nt & 1) * 2 + 1] = hi;
                const float2 ul = unpack_bf16x2(lo), uh = unpack_bf16x2(hi);
                ls0 = fadd2(ls0, ul);
                ls1 = fadd2(ls1, uh);
                if constexpr (split) {   // remainders (exact in fp32), rounded to bf16 for the second product
                    const uint32_t rl = pack_bf16x2(e0 - ul.x, e1 - ul.y), rh = pack_bf16x2(e2 - uh.x, e3 - uh.y);
                    par[nt >> 1][(nt & 1) * 2 + 0] = rl;
                    par[nt >> 1][(nt & 1) * 2 + 1] = rh;
                    ls0 = fadd2(ls0, unpack_bf16x2(rl));
                    ls1 = fadd2(ls1, unpack_bf16x2(rh));
                }
            }
            l_run[0] += ls0.x + ls0.y;
            l_run[1] += ls1.x + ls1.y;
            // O (this warp's dims) += P C; rows before row_lo are zeroed in registers
#pragma unroll
            for (int kk = 0; kk < KKS; ++kk) {
                uint32_t mlo = 0xFFFFFFFFu, mhi = 0xFFFFFFFFu;
                if (partial) {
                    const int row = kk * 16 + cq;
                    mlo = (row >= row_lo ? 0x0000FFFFu : 0u) | (row + 1 >= row_lo ? 0xFFFF0000u : 0u);
                    mhi = (row + 8 >= row_lo ? 0x0000FFFFu : 0u) | (row + 9 >= row_lo ? 0xFFFF0000u : 0u);
                }
                const uint32_t rowaddr = stage + (kk * 16 + vrow) * 128;
#pragma unroll
                for (int dp = 0; dp < NT_O / 2; ++dp) {
                    const uint32_t chunk = 2 * dp + vchk;
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4_trans(b0, b1, b2, b3, rowaddr + (dq * 2 + (chunk >> 3)) * kMlaPanelBytes +
                                                          (((chunk & 7) ^ (lane & 7)) << 4));
                    mma_bf16_16816(o[2 * dp], pa[kk], b0 & mlo, b1 & mhi);
                    mma_bf16_16816(o[2 * dp + 1], pa[kk], b2 & mlo, b3 & mhi);
                    if constexpr (split) {
                        mma_bf16_16816(o[2 * dp], par[kk], b0 & mlo, b1 & mhi);
                        mma_bf16_16816(o[2 * dp + 1], par[kk], b2 & mlo, b3 & mhi);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt) {
                s[nt][0] = sn[nt][0];
                s[nt][1] = sn[nt][1];
                s[nt][2] = sn[nt][2];
                s[nt][3] = sn[nt][3];
            }
        }
        };
        if (L <= kMlaSplitAllBelow)
            stage_loop(std::true_type{});
        else
            stage_loop(std::false_type{});
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
            l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
        }
    }

    // ---------------------------------------------------------------- combine
    __syncthreads();   // the ring has drained: reuse it
    float *co = reinterpret_cast<float *>(smem);          // [16][512]
    float *cm = co + kMlaHeads * kMlaDc;                   // [16]
    float *cl = cm + 64;                                   // [16]
    if (consumer) {
        const int r0 = lane >> 2, r1 = r0 + 8;
        const int cq = 2 * (lane & 3);
#pragma unroll
        for (int nt = 0; nt < NT_O; ++nt) {
            const int c = dq * 128 + nt * 8 + cq;
            *reinterpret_cast<float2 *>(&co[r0 * kMlaDc + c]) = make_float2(o[nt][0], o[nt][1]);
            *reinterpret_cast<float2 *>(&co[r1 * kMlaDc + c]) = make_float2(o[nt][2], o[nt][3]);
        }
        if (warp == 0 && (lane & 3) == 0) {
            cm[r0] = m_run[0];
            cl[r0] = l_run[0];
            cm[r1] = m_run[1];
            cl[r1] = l_run[1];
        }
    }
    __nv_bfloat16 *ob = p.out + (static_cast<size_t>(b) * p.h + head0) * kMlaDc;
    const bool ok = (*abort_flag == 0);
    if (P == 1) {
        __syncthreads();
        for (int it = threadIdx.x; it < HS * (kMlaDc / 2); it += kMlaThreads) {
            const int r = it / (kMlaDc / 2), c = 2 * (it % (kMlaDc / 2));
            const float inv = (cm[r] != -INFINITY && cl[r] > 0.f) ? 1.f / cl[r] : 0.f;
            const float2 v = *reinterpret_cast<const float2 *>(&co[r * kMlaDc + c]);
            if (ok) *reinterpret_cast<__nv_bfloat162 *>(ob + r * kMlaDc + c) = __floats2bfloat162_rn(v.x * inv, v.y * inv);
        }
        return;
    }
    // this CTA combines rows split, split + P, ...: first each row's weights over the splits
    // (into the partial-score area, which no peer reads), then the rows, with every split's
    // float4 loaded at once
    float *wn = reinterpret_cast<float *>(sred);   // [row][kMlaMaxSplit]
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int nrows = (HS - split + P - 1) / P;
    for (int k = threadIdx.x; k < nrows; k += kMlaThreads) {
        const int r = split + P * k;
        float mq[kMlaMaxSplit], lq[kMlaMaxSplit];
        float M = -INFINITY;
#pragma unroll
        for (int q = 0; q < kMlaMaxSplit; ++q) {
            mq[q] = q < P ? *cluster.map_shared_rank(&cm[r], q) : -INFINITY;
            lq[q] = q < P ? *cluster.map_shared_rank(&cl[r], q) : 0.f;
        }
#pragma unroll
        for (int q = 0; q < kMlaMaxSplit; ++q) M = fmaxf(M, mq[q]);
        float sl = 0.f;
#pragma unroll
        for (int q = 0; q < kMlaMaxSplit; ++q) {
            mq[q] = (M == -INFINITY || mq[q] == -INFINITY) ? 0.f : exp2f(mq[q] - M);   // a split with no tokens adds nothing
            sl += mq[q] * lq[q];
        }
        const float inv = sl > 0.f ? 1.f / sl : 0.f;
#pragma unroll
        for (int q = 0; q < kMlaMaxSplit; ++q) wn[k * kMlaMaxSplit + q] = mq[q] * inv;
    }
    __syncthreads();
    for (int it = threadIdx.x; it < nrows * (kMlaDc / 4); it += kMlaThreads) {
        const int k = it / (kMlaDc / 4), c = 4 * (it % (kMlaDc / 4));
        const int r = split + P * k;
        float4 v[kMlaMaxSplit];
#pragma unroll
        for (int q = 0; q < kMlaMaxSplit; ++q)
            if (q < P) v[q] = *reinterpret_cast<const float4 *>(cluster.map_shared_rank(&co[r * kMlaDc + c], q));
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < kMlaMaxSplit; ++q)
            if (q < P) {
                const float w = wn[k * kMlaMaxSplit + q];
                a.x += w * v[q].x;
                a.y += w * v[q].y;
                a.z += w * v[q].z;
                a.w += w * v[q].w;
            }
        if (ok) {
            const __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
            uint2 pk;
            pk.x = *reinterpret_cast<const uint32_t *>(&lo);
            pk.y = *reinterpret_cast<const uint32_t *>(&hi);
            *reinterpret_cast<uint2 *>(ob + static_cast<size_t>(r) * kMlaDc + c) = pk;
        }
    }
    cluster.sync();
}

// ---------------------------------------------------------------------------
// host launcher

int launch_mla_decode_tc(const void *q, const void *c_kv, const int32_t *seqlens, void *out, int B, int h,
                         float scale, long long cache_rows, void *ws, size_t ws_bytes, cudaStream_t stream);
size_t mla_tc_workspace_bytes(int B, int h, int sms);

// The tensor-core kernel (mla_tc.cu) for long sequences in batches too small to
// fill the GPU with this kernel: more than 16 heads (its products are 32 heads
// wide), this kernel's CTAs (16-head groups x up to 8 splits) fewer than the
// SMs, and, by the caller's row count, at least kMlaTcMinAvgRows tokens per
// sequence on average.  Measured on B200 (us, this kernel / tensor cores):
// B8 h32 L32768 208 / 168, B1 h32 L20000 109 / 73; it loses where this kernel
// fills the SMs (B16 h32 L4096 34 / 46) or on short or 16-head work.
constexpr long long kMlaTcMinAvgRows = 8192;

// This kernel's CTAs for a shape: 16-head groups x sequences, each in up to 8 splits (two
// CTAs per SM).
static long mla_warp_level_ctas(int B, int h, int sms) {
    const long units = static_cast<long>(B) * ((h + kMlaHeads - 1) / kMlaHeads);
    return units * std::max(1L, std::min(static_cast<long>(kMlaMaxSplit), 2L * sms / units));
}

bool mla_prefers_tc(int B, int h, long long cache_rows, bool rows_known, int sms) {
    if (!rows_known || h <= kMlaHeads) return false;
    return mla_warp_level_ctas(B, h, sms) < sms && cache_rows >= kMlaTcMinAvgRows * B;
}

// With a workspace the tensor-core kernel's splits merge there instead of in a cluster, so
// it keeps every SM busy (one CTA per SM, any number of splits): taken in the same regime
// (h > 16, this kernel's CTAs fewer than the SMs) down to kMlaWsMinAvgRows tokens per
// sequence.  Measured on B200 (us, this kernel / tensor cores with the workspace):
// B8 h32 L8192 57.9 / 37.7, B2 h32 L8192 47.7 / 21.8, B4 h32 L65536 340.5 / 108.3,
// B1 h32 L20000 108.7 / 28.9; where this kernel fills the SMs it stays ahead
// (B16 h32 L4096 34.3 / 37.7, B16 h64 L4096 58.7 / 61.5, B32 h32 L2048 34.1 / 37.8).
constexpr long long kMlaWsMinAvgRows = 2048;

bool mla_ws_prefers_tc(int B, int h, long long cache_rows, int sms) {
    if (h <= kMlaHeads) return false;
    return mla_warp_level_ctas(B, h, sms) < sms && cache_rows >= kMlaWsMinAvgRows * B;
}

// The workspace a shape needs: none where the tensor-core kernel can never be picked
// (16 heads or fewer, or this kernel already filling the SMs), whatever the lengths.
size_t mla_ws_bytes(int B, int h, int sms) {
    if (h <= kMlaHeads || mla_warp_level_ctas(B, h, sms) >= sms) return 0;
    return mla_tc_workspace_bytes(B, h, sms);
}

int launch_mla_decode(const void *q, const void *c_kv, const int32_t *seqlens, void *out, int B, int h, float scale,
                      long long cache_rows, bool rows_known, cudaStream_t stream) {
    if (mla_prefers_tc(B, h, cache_rows, rows_known, gqa_host::sm_count()))
        return launch_mla_decode_tc(q, c_kv, seqlens, out, B, h, scale, cache_rows, nullptr, 0, stream);
    auto kern = gqa_mla_decode_kernel;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 3;
    static std::atomic<unsigned long long> attr_done{0};
    if (!gqa_host::once_per_device(attr_done, dev, [&] {
            return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, MlaSmem::kTotal) ==
                   cudaSuccess;
        }))
        return 3;
    CUtensorMap tc;
    // token extent = the cache's rows (the kernel cuts lengths that ask for more and reports them)
    const uint64_t dims[2] = {static_cast<uint64_t>(kMlaDc), static_cast<uint64_t>(std::max(cache_rows, 1LL))};
    const uint64_t strides[1] = {static_cast<uint64_t>(kMlaDc) * 2};
    const uint32_t box[2] = {64, kMlaTok};
    if (!gqa_host::encode_tensor_map(&tc, c_kv, 2, dims, strides, box)) return 3;

    const int groups = (h + kMlaHeads - 1) / kMlaHeads;
    const long units = static_cast<long>(B) * groups;
    const long slots = 2L * gqa_host::sm_count();
    const int P = static_cast<int>(std::max(1L, std::min(static_cast<long>(kMlaMaxSplit), slots / units)));
    MlaParams prm;
    prm.q = static_cast<const __nv_bfloat16 *>(q);
    prm.seqlens = seqlens;
    prm.out = static_cast<__nv_bfloat16 *>(out);
    prm.B = B;
    prm.h = h;
    prm.groups = groups;
    prm.cache_rows = cache_rows;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.status = gqa_host::device_status();
    if (!prm.status) return 3;
    GQA_SET_TEST_STALL(prm);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P, groups, B);
    cfg.blockDim = dim3(kMlaThreads, 1, 1);
    cfg.dynamicSmemBytes = MlaSmem::kTotal;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = P;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tc, prm) != cudaSuccess) return 3;
    return 0;
}

// 0 = launched, 1 = workspace too small, 3 = a CUDA call failed.
int launch_mla_decode_ws(const void *q, const void *c_kv, const int32_t *seqlens, void *out, int B, int h,
                         float scale, long long cache_rows, void *ws, size_t ws_bytes, cudaStream_t stream) {
    const int sms = gqa_host::sm_count();
    if (ws_bytes < mla_ws_bytes(B, h, sms)) return 1;
    if (mla_ws_prefers_tc(B, h, cache_rows, sms))
        return launch_mla_decode_tc(q, c_kv, seqlens, out, B, h, scale, cache_rows, ws, ws_bytes, stream);
    return launch_mla_decode(q, c_kv, seqlens, out, B, h, scale, cache_rows, true, stream);
}

}  // namespace gqa
