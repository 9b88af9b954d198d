// Absorbed multi-head latent attention (MLA) decode on the 5th-generation
// tensor cores: the kernel for long sequences in batches too small to fill the
// GPU with the warp-level kernel (mla.cu picks between the two by shape).
//
// Semantics: "Evolution of AI Attention Mechanisms" (toolsku), "Generation 3:
// MLA Multi-Head Latent Attention": one latent row c_kv (d_c = 512) per token,
// shared by every head; with the key up-projection absorbed into the query
// (q' = q W_k_up, supplied by the caller) the scores are q' c_kv^T * scale and
// the softmax weights multiply c_kv itself.
//
// Design (B200).  At 32 heads the path does 64 flops per latent byte, so both
// products run on tcgen05, with operands chosen so that shared memory feeds
// only the latent:
//   S   = q' C^T     M = 128 rows (the CTA's 32 heads; rows 32..127 are never
//                    read), N = 64 tokens, K = 512.  A = q' resident in TMEM
//                    (written once per CTA), B = the latent stage (K-major).
//   O^T += C^T P^T   four MMAs M = 128 latent dims, N = 32 heads, K = 16
//                    tokens per step.  A = the same latent stage read
//                    MN-major, B = P^T written by the softmax warp.
// TMEM (512 columns): two S buffers of 64, O^T 4 x 32, q' 32 k-steps x 8.
// The softmax warp owns TMEM lanes 0..31, so each thread holds one head's 64
// scores of a stage: row maxima and sums need no shuffles.  The running max
// moves only when a head's stage max exceeds it by 2^8 (lazy rescale); then
// warps 0-3 (all four TMEM lane quarters) rescale O^T once the previous
// stage's products are done.  Sequences of at most kSplitAllBelow tokens also
// send the weights' bf16 remainders through a second product.
//
// Two warps issue the MMAs, one the score products and one the O^T products,
// each committing only its own, so that O^T(i) issues as soon as its weights
// are written.
//
// Ring: twelve 16 KB slots, each 64 tokens x 128 latent dims (two 64-dim
// panels of 128-byte swizzled rows, one M block of O^T): three stages.  One
// CTA per SM (shared memory and all of TMEM).  The splits of one (sequence,
// 32-head group) either form a cluster (at most 16) and merge through
// distributed shared memory, or, given a workspace, write their partial
// results there for a second launch to merge (any number of splits).  Every
// wait is bounded.
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace gqa {

namespace mla_tc {

constexpr int kDc = 512;                                // latent width
constexpr int kTok = 64;                                // tokens per stage (N of the score MMA)
constexpr int kHeads = 32;                              // heads per CTA (N of the P V MMA)
constexpr int kPanelBytes = kTok * 128;                 // 64 tokens x 64 dims
constexpr int kPairBytes = 2 * kPanelBytes;             // 128 dims: one M block of O^T
constexpr int kPairs = kDc / 128;                       // pairs per stage
constexpr int kSlots = 12;                              // ring of pair slots (three stages)
constexpr int kThreads = 7 * 32;                        // 0 softmax, 0-3 O^T lanes, 4 TMA, 5 S MMAs, 6 O^T MMAs
constexpr int kMaxSplit = 16;                          // splits of one cluster (its largest size)
constexpr int kMaxSplitWs = 256;                        // splits merged through a workspace
constexpr int kPartFloats = kHeads * kDc + 2 * kHeads;  // a workspace partial: O [32][512], m [32], l [32]
constexpr float kRescale = 8.0f;                        // lazy rescale threshold (log2 units)
constexpr int kSplitAllBelow = 256;                     // remainder product for sequences this short
// TMEM columns
constexpr uint32_t kColS = 0;                           // S buffers [0, 64), [64, 128)
constexpr uint32_t kColO = 128;                         // O^T block j at kColO + 32 j
constexpr uint32_t kColQ = 256;                         // q': k-step ks at kColQ + 8 ks

struct Params {
    const __nv_bfloat16 *q;
    const int32_t *seqlens;
    __nv_bfloat16 *out;
    int B, h;
    long long cache_rows;          // rows the latent cache holds (the tensor map's extent)
    float scale_log2;              // scale * log2(e), >= 0
    int *status;
    float *part;                   // null: the splits merge in their cluster; else [CTA][kPartFloats]
    GQA_TEST_STALL_FIELD
};

struct Smem {
    static constexpr uint32_t kRing = kSlots * kPairBytes;          // 192 KB
    static constexpr uint32_t kPT = kHeads * 128;                    // P^T: 32 head rows x 64 tokens
    static constexpr uint32_t kOffP = kRing;                         // [2 buffers][weights, remainders]
    // q' staged once (eight 64-dim panels of 32 swizzled head rows) before any P^T is written
    static constexpr uint32_t kQPanel = kHeads * 128;
    static constexpr uint32_t kOffCtrl = kOffP + 8 * kQPanel;
    static constexpr uint32_t kCtrl = 1024;
    static constexpr uint32_t kTotal = kOffCtrl + kCtrl + 1024;
    // after the ring drains: co[32][512] fp32, cm[32], cl[32]
    static constexpr uint32_t kOffCm = kHeads * kDc * 4;
    static_assert(kOffCm + 2 * 32 * 4 <= kRing, "partials fit in the drained ring");
    static_assert(8 * kQPanel >= 4 * kPT, "the q' staging covers the P^T buffers");
    static_assert(kTotal <= 232448, "dynamic shared memory per CTA");
    // one CTA per SM: two would not both get their 512 TMEM columns
    static_assert(2 * kTotal > 233472, "shared memory keeps one CTA per SM");
};

__global__ void __launch_bounds__(kThreads, 1)
    mla_decode_tc_kernel(const __grid_constant__ CUtensorMap tm_c, const Params p) {
    using SM = Smem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sRing = smem;
    uint8_t *sP = smem + SM::kOffP;
    uint8_t *ctrl = smem + SM::kOffCtrl;
    uint64_t *full = reinterpret_cast<uint64_t *>(ctrl);   // [slots] a pair slot landed
    uint64_t *empty = full + kSlots;                       // [slots] the P V products that read it completed
    uint64_t *qready = empty + kSlots;                     // q' is in TMEM
    uint64_t *sfull = qready + 1;                          // [2] S of a stage in TMEM buffer b
    uint64_t *sfree = sfull + 2;                           // [2] ... read by the softmax warp
    uint64_t *mfull = sfree + 2;                           // [2] the stage's rescale decision published
    uint64_t *pfull = mfull + 2;                           // [2] P^T written and O^T rescaled
    uint64_t *pvdone = pfull + 2;                          // [2] the stage's P V products completed
    uint64_t *ack = pvdone + 2;                            // [2] warps 1-3 read the decision (and rescaled)
    uint64_t *odone = ack + 2;
    uint64_t *drain = odone + 1;                           // the S issuer's products completed
    uint64_t *drain_o = drain + 1;                         // the O^T issuer's, when it gave up
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ctrl + 320);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(ctrl + 324);
    long long *red = reinterpret_cast<long long *>(ctrl + 328);          // [7]
    float *av = reinterpret_cast<float *>(ctrl + 384);                   // [2][32] rescale factor per head
    volatile int *rflag = reinterpret_cast<volatile int *>(ctrl + 640);  // [2] the stage rescales O^T

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = gridDim.x, split = blockIdx.x;
    const int grp = blockIdx.y, b = blockIdx.z;
    const int head0 = grp * kHeads;
    const int HS = min(p.h - head0, kHeads);
    // with a workspace, the merge launch that follows may start now (it waits for this grid)
    if (p.part) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (threadIdx.x == 0) {
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(qready, 1);
        for (int t = 0; t < 2; ++t) {
            mbar_init(&sfull[t], 1);
            mbar_init(&sfree[t], 1);
            mbar_init(&mfull[t], 1);
            mbar_init(&pfull[t], 1);
            mbar_init(&pvdone[t], 1);
            mbar_init(&ack[t], 3);
        }
        mbar_init(odone, 1);
        mbar_init(drain, 1);
        mbar_init(drain_o, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    // first cache row of sequence b (64-bit sum of the earlier non-negative lengths)
    long long acc = 0;
    for (int i = threadIdx.x; i < b; i += kThreads) acc += max(p.seqlens[i], 0);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) red[warp] = acc;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    long long off64 = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) off64 += red[w];
    int L = max(p.seqlens[b], 0);
    if (off64 + L > p.cache_rows) {   // the lengths ask for rows the cache does not hold
        if (threadIdx.x == 0) record_status(p.status, kStatusInvalid);
        L = static_cast<int>(max(0LL, p.cache_rows - off64));
    }
    // off + L <= cache_rows <= INT32_MAX whenever a row is read (the host bounds cache_rows)
    const int off = static_cast<int>(min(off64, p.cache_rows));
    const int n_total = (L + kTok - 1) / kTok;
    const int per_split = (n_total + P - 1) / P;
    const int first = split * per_split;
    const int n_stages = max(0, min(n_total, first + per_split) - first);
    const bool rem = L <= kSplitAllBelow;   // the weights' bf16 remainders go through a second product
    const float cl2 = p.scale_log2;

    float m_run = -INFINITY, l_run = 0.f;   // softmax warp: head `lane`
    bool ok = true;

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_c);
            const int first_loaded = GQA_STALLED(p) ? 1 : 0;   // wait-test build: stage 0 never arrives
            int issued = 0;
            for (int i = 0; i < n_stages && ok; ++i) {
                const int t0 = (first + i) * kTok;
                // the last stage is shifted back to end at the sequence end (never past the cache)
                const int z = off + min(t0, L - kTok);
                for (int j = 0; j < kPairs; ++j) {
                    const int n = i * kPairs + j, slot = n % kSlots, use = n / kSlots;
                    if (use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    ++issued;
                    if (i < first_loaded) continue;
                    uint8_t *dst = sRing + slot * kPairBytes;
                    mbar_arrive_expect_tx(&full[slot], kPairBytes);
                    tma_load_2d(dst, &tm_c, &full[slot], 2 * j * 64, z);
                    tma_load_2d(dst + kPanelBytes, &tm_c, &full[slot], (2 * j + 1) * 64, z);
                }
            }
            if (*abort_flag) {
                for (int n = max(first_loaded * kPairs, issued - kSlots); n < issued; ++n)
                    mbar_wait_drain(&full[n % kSlots], (n / kSlots) & 1, p.status);
            }
        }
        __syncwarp();
    } else if (warp == 5 || warp == 6) {
        // ------------------------------------------------------------ MMA issuers: S (warp 5), O^T (warp 6)
        // Two issuing threads, each committing only its own products, so that neither waits on
        // the other's condition: O^T(i) issues as soon as its weights are written, whether or
        // not the stage after it has landed.
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, kTok, false, false);
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, kHeads, true, false);
            const uint32_t ring_base = smem_u32(sRing);
            const uint32_t p_base = smem_u32(sP);
            auto slot_addr = [&](int i, int j) { return ring_base + ((i * kPairs + j) % kSlots) * kPairBytes; };
            if (warp == 5) {
                ok = mbar_wait(qready, 0, abort_flag, p.status);
                for (int i = 0; i < n_stages && ok; ++i) {
                    // S(i) reuses the buffer of S(i - 2): after the softmax read it
                    if (i >= 2 && !mbar_wait(&sfree[i & 1], ((i - 2) >> 1) & 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    for (int j = 0; j < kPairs && ok; ++j) {
                        const int n = i * kPairs + j;
                        ok = mbar_wait(&full[n % kSlots], (n / kSlots) & 1, abort_flag, p.status);
                    }
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t tS = tmem + kColS + (i & 1) * kTok;
#pragma unroll
                    for (int ks = 0; ks < kDc / 16; ++ks) {
                        // k-step ks: pair ks / 8, panel (ks / 4) % 2, 32-byte column (ks % 4) of the 128-byte rows
                        const uint32_t bad = slot_addr(i, ks >> 3) + ((ks >> 2) & 1) * kPanelBytes + (ks & 3) * 32;
                        umma_ts(tS, tmem + kColQ + ks * 8, sdesc_sw128(bad, 16, 1024), idesc_s, ks ? 1u : 0u);
                    }
                    umma_commit(&sfull[i & 1]);
                }
                umma_commit(drain);   // every S product complete before TMEM is freed
                mbar_wait_drain(drain, 0, p.status);
            } else {
                for (int i = 0; i < n_stages && ok; ++i) {
                    if (!mbar_wait(&pfull[i & 1], (i >> 1) & 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t pb = p_base + (i & 1) * 2 * Smem::kPT;
                    // block by block, each slot released as soon as its products complete
#pragma unroll
                    for (int j = 0; j < kPairs; ++j) {
#pragma unroll
                        for (int kk = 0; kk < kTok / 16; ++kk)
                            umma_ss(tmem + kColO + 32 * j,
                                    sdesc_sw128(slot_addr(i, j) + kk * 16 * 128, kPanelBytes, 1024),
                                    sdesc_sw128(pb + kk * 32, 16, 1024), idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
                        if (rem) {
#pragma unroll
                            for (int kk = 0; kk < kTok / 16; ++kk)
                                umma_ss(tmem + kColO + 32 * j,
                                        sdesc_sw128(slot_addr(i, j) + kk * 16 * 128, kPanelBytes, 1024),
                                        sdesc_sw128(pb + Smem::kPT + kk * 32, 16, 1024), idesc_o, 1u);
                        }
                        umma_commit(&empty[(i * kPairs + j) % kSlots]);
                    }
                    umma_commit(&pvdone[i & 1]);
                }
                umma_commit(ok ? odone : drain_o);
                if (!ok) mbar_wait_drain(drain_o, 0, p.status);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax (warp 0), O^T lanes (warps 0-3)
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        {
            // q' of the group (zeros past it), coalesced, into eight swizzled 64-dim panels of 32 head rows
            const uint4 *qg = reinterpret_cast<const uint4 *>(p.q + (static_cast<size_t>(b) * p.h + head0) * kDc);
            constexpr int kPer = kHeads * (kDc / 8) / 128;   // 16-byte pieces per thread
            uint4 t[kPer];
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int u = threadIdx.x + 128 * k, row = u / (kDc / 8);
                t[k] = row < HS ? qg[u] : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int u = threadIdx.x + 128 * k, row = u / (kDc / 8), c64 = u % (kDc / 8);
                *reinterpret_cast<uint4 *>(sP + (c64 >> 3) * Smem::kQPanel + sw128_offset(row, c64 & 7)) = t[k];
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");   // warps 0-3 only, all of which get here
        }
        if (warp == 0) {
            // q' row `lane` into TMEM columns [kColQ, kColQ + 256): column c holds the bf16 pair
            // (2c, 2c + 1), the A-operand layout of the score MMA
#pragma unroll 1
            for (int pn = 0; pn < 8; ++pn) {
                uint32_t w[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(sP + pn * Smem::kQPanel + sw128_offset(lane, c));
                    w[4 * c] = v.x;
                    w[4 * c + 1] = v.y;
                    w[4 * c + 2] = v.z;
                    w[4 * c + 3] = v.w;
                }
                tmem_st32(tmem + kColQ + 32 * pn, w);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(qready);
        }
        // O^T *= alpha per head column (this warp's 32 TMEM lanes), once the previous stage's products are done
        auto rescale_o = [&](int i) -> bool {
            const bool done = mbar_wait(&pvdone[(i - 1) & 1], ((i - 1) >> 1) & 1, abort_flag, p.status);
            if (!__all_sync(0xffffffffu, done)) return false;
            tc_fence_after();
            const float *a = av + (i & 1) * 32;
#pragma unroll 1
            for (int j = 0; j < kPairs; ++j) {
                uint32_t o[32];
                tmem_ld32(tmem + kColO + 32 * j + lane_off, o);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * a[e]);
                tmem_st32(tmem + kColO + 32 * j + lane_off, o);
            }
            tmem_wait_st();
            return true;
        };
        for (int i = 0; i < n_stages; ++i) {
            const int buf = i & 1;
            bool resc = false;
            if (warp == 0) {
                const int t0 = (first + i) * kTok;
                const int row_lo = max(0, t0 - (L - kTok));   // rows of the box before this stage's tokens
                const bool got = mbar_wait(&sfull[buf], (i >> 1) & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t s[kTok];
                {
                    uint32_t s0[32], s1[32];
                    tmem_ld32(tmem + kColS + buf * kTok, s0);
                    tmem_ld32(tmem + kColS + buf * kTok + 32, s1);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        s[e] = s0[e];
                        s[32 + e] = s1[e];
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfree[buf]);
                // stage max of head `lane` over the valid tokens (>= 1 per stage)
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // four chains, not one
#pragma unroll
                for (int t = 0; t < kTok; ++t) m4[t & 3] = fmaxf(m4[t & 3], t >= row_lo ? __uint_as_float(s[t]) : -INFINITY);
                const float tile = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * cl2;
                float alpha = 1.f;
                if (i == 0) {
                    m_run = tile;
                } else {
                    resc = __any_sync(0xffffffffu, lane < HS && tile > m_run + kRescale);
                    if (resc) {
                        const float m_new = fmaxf(m_run, tile);
                        alpha = exp2f(m_run - m_new);
                        m_run = m_new;
                        l_run *= alpha;
                    }
                }
                if (i >= 2) {   // warps 1-3 have read the decision of stage i - 2 (normally long since)
                    const bool rd = mbar_wait(&ack[buf], ((i - 2) >> 1) & 1, abort_flag, p.status);
                    if (!__all_sync(0xffffffffu, rd)) {
                        ok = false;
                        break;
                    }
                }
                av[buf * 32 + lane] = alpha;
                if (lane == 0) rflag[buf] = resc ? 1 : 0;
                __syncwarp();
                if (lane == 0) mbar_arrive(&mfull[buf]);
                if (resc) {   // O^T's four lane quarters: this warp's, then wait for warps 1-3
                    if (!rescale_o(i)) {
                        ok = false;
                        break;
                    }
                    const bool rd = mbar_wait(&ack[buf], (i >> 1) & 1, abort_flag, p.status);
                    if (!__all_sync(0xffffffffu, rd)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                // the weights (and on short sequences their remainders), packed bf16 pairs of tokens
                uint32_t pw[kTok / 2], pr[kTok / 2];
                float2 ls[4] = {};   // four chains of packed sums
#pragma unroll
                for (int e = 0; e < kTok / 2; ++e) {
                    const int t = 2 * e;
                    const float2 y = ffma2_bcast(__uint_as_float(s[t]), __uint_as_float(s[t + 1]), cl2, -m_run);
                    const float x0 = t >= row_lo ? exp2f(y.x) : 0.f;
                    const float x1 = t + 1 >= row_lo ? exp2f(y.y) : 0.f;
                    pw[e] = pack_bf16x2(x0, x1);
                    const float2 u = unpack_bf16x2(pw[e]);
                    ls[e & 3] = fadd2(ls[e & 3], u);
                    if (rem) {
                        pr[e] = pack_bf16x2(x0 - u.x, x1 - u.y);
                        ls[e & 3] = fadd2(ls[e & 3], unpack_bf16x2(pr[e]));
                    }
                }
                l_run += ((ls[0].x + ls[0].y) + (ls[1].x + ls[1].y)) + ((ls[2].x + ls[2].y) + (ls[3].x + ls[3].y));
                if (i >= 2) {   // P^T buffer `buf` was read by the products of stage i - 2
                    const bool free_p = mbar_wait(&pvdone[buf], ((i - 2) >> 1) & 1, abort_flag, p.status);
                    if (!__all_sync(0xffffffffu, free_p)) {
                        ok = false;
                        break;
                    }
                }
                // P^T row `lane` = head lane: 64 tokens of 2 bytes, 128-byte swizzled (a K-major B operand)
                uint8_t *pb = sP + buf * 2 * Smem::kPT;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(pb + sw128_offset(lane, c)) =
                        make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
                if (rem) {
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4 *>(pb + Smem::kPT + sw128_offset(lane, c)) =
                            make_uint4(pr[4 * c], pr[4 * c + 1], pr[4 * c + 2], pr[4 * c + 3]);
                }
                if (row_lo > 0) {
                    // rows before row_lo hold other tokens: zero them so that no value there
                    // (even a NaN) reaches O^T through a zero weight
                    for (int it = lane; it < row_lo * 64; it += 32) {
                        const int q8 = it & 7, chk = (it >> 3) & 7, row = it >> 6;
                        const int slot = (i * kPairs + (q8 >> 1)) % kSlots;
                        *reinterpret_cast<uint4 *>(sRing + slot * kPairBytes + (q8 & 1) * kPanelBytes + row * 128 +
                                                   chk * 16) = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&pfull[buf]);
            } else {
                // warps 1-3 take part only in the (rare) rescales, off the softmax warp's path
                const bool got = mbar_wait(&mfull[buf], (i >> 1) & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                resc = rflag[buf] != 0;
                if (resc && !rescale_o(i)) {
                    ok = false;
                    break;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ack[buf]);
            }
        }
        if (ok && n_stages > 0) {
            const bool fin = mbar_wait(odone, 0, abort_flag, p.status);
            ok = __all_sync(0xffffffffu, fin);
        }
    }

    // ---------------------------------------------------------------- this CTA's partial
    tc_fence_before();
    __syncthreads();   // every role has finished; the producer has drained its copies
    tc_fence_after();
    const bool good = (*abort_flag == 0);
    if (p.part) {
        // this split's partial into the workspace (unnormalised O, running max, sum), read by
        // the merge launch; rows past the group are left unwritten
        float *pp = p.part + static_cast<size_t>((b * gridDim.y + grp) * P + split) * kPartFloats;
        if (warp < 4 && good) {
            const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll 1
            for (int j = 0; j < kPairs; ++j) {
                uint32_t o[32];
                if (n_stages > 0) {
                    tmem_ld32(tmem + kColO + 32 * j + lane_off, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = 0u;
                }
                const int d = 128 * j + 32 * warp + lane;
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    if (e < HS) pp[e * kDc + d] = __uint_as_float(o[e]);
            }
            if (warp == 0 && lane < HS) {
                pp[kHeads * kDc + lane] = n_stages > 0 ? m_run : -INFINITY;
                pp[kHeads * kDc + kHeads + lane] = l_run;
            }
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 5) {
            tc_fence_after();
            tmem_dealloc(tmem, 512);
        }
        return;
    }
    float *co = reinterpret_cast<float *>(sRing);              // [32 heads][512] fp32
    float *cm = reinterpret_cast<float *>(sRing + SM::kOffCm);  // [32]
    float *cl = cm + 32;                                        // [32]
    if (warp < 4 && good) {
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll 1
        for (int j = 0; j < kPairs; ++j) {
            uint32_t o[32];
            if (n_stages > 0) {
                tmem_ld32(tmem + kColO + 32 * j + lane_off, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = 0u;
            }
            const int d = 128 * j + 32 * warp + lane;
#pragma unroll
            for (int e = 0; e < 32; ++e) co[e * kDc + d] = __uint_as_float(o[e]);
        }
        if (warp == 0) {
            cm[lane] = n_stages > 0 ? m_run : -INFINITY;
            cl[lane] = l_run;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }

    // ---------------------------------------------------------------- merge the splits
    __nv_bfloat16 *ob = p.out + (static_cast<size_t>(b) * p.h + head0) * kDc;
    auto store4 = [&](int r, int c, float4 a) {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
        uint2 pk;
        pk.x = *reinterpret_cast<const uint32_t *>(&lo);
        pk.y = *reinterpret_cast<const uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(ob + static_cast<size_t>(r) * kDc + c) = pk;
    };
    if (P == 1) {
        for (int it = threadIdx.x; it < HS * (kDc / 4); it += kThreads) {
            const int r = it / (kDc / 4), c = 4 * (it % (kDc / 4));
            const float inv = (cm[r] != -INFINITY && cl[r] > 0.f) ? 1.f / cl[r] : 0.f;
            const float4 v = *reinterpret_cast<const float4 *>(&co[r * kDc + c]);
            if (good) store4(r, c, make_float4(v.x * inv, v.y * inv, v.z * inv, v.w * inv));
        }
        return;
    }
    // this CTA combines rows split, split + P, ...: first each row's weights over the splits
    // (into the P^T area, which no peer reads), then the rows, with every split's float4 loaded at once
    float *wn = reinterpret_cast<float *>(sP);   // [row][kMaxSplit]
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int nrows = (HS - split + P - 1) / P;
    for (int k = threadIdx.x; k < nrows; k += kThreads) {
        const int r = split + P * k;
        float mq[kMaxSplit], lq[kMaxSplit];
        float M = -INFINITY;
#pragma unroll
        for (int q = 0; q < kMaxSplit; ++q) {
            const int qq = min(q, P - 1);   // every load issued at once, the ones past P discarded
            const float m0 = *cluster.map_shared_rank(&cm[r], qq), l0 = *cluster.map_shared_rank(&cl[r], qq);
            mq[q] = q < P ? m0 : -INFINITY;
            lq[q] = q < P ? l0 : 0.f;
        }
#pragma unroll
        for (int q = 0; q < kMaxSplit; ++q) M = fmaxf(M, mq[q]);
        float sl = 0.f;
#pragma unroll
        for (int q = 0; q < kMaxSplit; ++q) {
            mq[q] = (M == -INFINITY || mq[q] == -INFINITY) ? 0.f : exp2f(mq[q] - M);   // a split with no tokens adds nothing
            sl += mq[q] * lq[q];
        }
        const float inv = sl > 0.f ? 1.f / sl : 0.f;
#pragma unroll
        for (int q = 0; q < kMaxSplit; ++q) wn[k * kMaxSplit + q] = mq[q] * inv;
    }
    __syncthreads();
    for (int it = threadIdx.x; it < nrows * (kDc / 4); it += kThreads) {
        const int k = it / (kDc / 4), c = 4 * (it % (kDc / 4));
        const int r = split + P * k;
        float4 v[kMaxSplit];
#pragma unroll
        for (int q = 0; q < kMaxSplit; ++q)
            if (q < P) v[q] = *reinterpret_cast<const float4 *>(cluster.map_shared_rank(&co[r * kDc + c], q));
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < kMaxSplit; ++q)
            if (q < P) {
                const float w = wn[k * kMaxSplit + q];
                a.x += w * v[q].x;
                a.y += w * v[q].y;
                a.z += w * v[q].z;
                a.w += w * v[q].w;
            }
        if (good) store4(r, c, a);
    }
    cluster.sync();
}

// The merge of the workspace partials: one block per (sequence x group, head), eight warps
// each folding every eighth split with the log-sum-exp rule (running max, sum, unnormalised
// O; a lane holds 16 of the 512 dims), then the eight folds combined through shared memory.
constexpr int kMergeWarps = 8;

__global__ void __launch_bounds__(kMergeWarps * 32)
    mla_merge_kernel(const float *part, __nv_bfloat16 *out, int h, int groups, int P) {
    asm volatile("griddepcontrol.wait;" ::: "memory");   // the partials' launch has completed
    __shared__ float sM[kMergeWarps], sL[kMergeWarps];
    __shared__ float4 sO[kMergeWarps][kDc / 4];
    const int u = blockIdx.x, r = blockIdx.y;
    const int grp = u % groups, b = u / groups;
    const int head = grp * kHeads + r;
    if (head >= h) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float M = -INFINITY, L = 0.f;
    float4 acc[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
    for (int q = warp; q < P; q += kMergeWarps) {
        const float *pp = part + static_cast<size_t>(u * P + q) * kPartFloats;
        const float m = __ldcg(pp + kHeads * kDc + r);
        const float l = __ldcg(pp + kHeads * kDc + kHeads + r);
        float4 o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) o[k] = __ldcg(reinterpret_cast<const float4 *>(pp + r * kDc) + lane + 32 * k);
        if (m == -INFINITY) continue;   // a split with no tokens
        const float M2 = fmaxf(M, m);
        const float a = exp2f(M - M2), w = exp2f(m - M2);   // M2 is finite: a = 0 while M is -inf
        L = L * a + l * w;
#pragma unroll
        for (int k = 0; k < 4; ++k)
            acc[k] = make_float4(acc[k].x * a + o[k].x * w, acc[k].y * a + o[k].y * w, acc[k].z * a + o[k].z * w,
                                 acc[k].w * a + o[k].w * w);
        M = M2;
    }
    if (lane == 0) {
        sM[warp] = M;
        sL[warp] = L;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) sO[warp][lane + 32 * k] = acc[k];
    __syncthreads();
    float Mf = -INFINITY;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) Mf = fmaxf(Mf, sM[w]);
    float wt[kMergeWarps], Lf = 0.f;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) {
        wt[w] = sM[w] == -INFINITY ? 0.f : exp2f(sM[w] - Mf);
        Lf += wt[w] * sL[w];
    }
    const float inv = Lf > 0.f ? 1.f / Lf : 0.f;
    // thread t writes dims 2t, 2t + 1
    const float *so = reinterpret_cast<const float *>(sO);
    float x0 = 0.f, x1 = 0.f;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) {
        x0 += wt[w] * so[w * kDc + 2 * threadIdx.x];
        x1 += wt[w] * so[w * kDc + 2 * threadIdx.x + 1];
    }
    *reinterpret_cast<__nv_bfloat162 *>(out + (static_cast<size_t>(b) * h + head) * kDc + 2 * threadIdx.x) =
        __floats2bfloat162_rn(x0 * inv, x1 * inv);
}

}  // namespace mla_tc

// ---------------------------------------------------------------------------
// host launcher

namespace {

// How many clusters of P CTAs (one per SM) fit on the device at once, cached per device.
int max_active_clusters_tc(int P) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || P < 1 || P > mla_tc::kMaxSplit) return 0;
    static std::atomic<int> cache[64][mla_tc::kMaxSplit + 1];
    int n = cache[dev][P].load(std::memory_order_relaxed);
    if (n == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(P, 1, 1);
        cfg.blockDim = dim3(mla_tc::kThreads, 1, 1);
        cfg.dynamicSmemBytes = mla_tc::Smem::kTotal;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = P;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int got = 0;
        if (cudaOccupancyMaxActiveClusters(&got, mla_tc::mla_decode_tc_kernel, &cfg) != cudaSuccess) {
            cudaGetLastError();
            got = 0;
        }
        n = got > 0 ? got : -1;
        cache[dev][P].store(n, std::memory_order_relaxed);
    }
    return n > 0 ? n : 0;
}

}  // namespace

// Splits per (sequence, 32-head group) when they merge through a workspace: one CTA per SM.
static int mla_tc_ws_splits(long units, int sms) {
    return static_cast<int>(std::max(1L, std::min(static_cast<long>(mla_tc::kMaxSplitWs), sms / units)));
}

size_t mla_tc_workspace_bytes(int B, int h, int sms) {
    const long units = static_cast<long>(B) * ((h + mla_tc::kHeads - 1) / mla_tc::kHeads);
    return static_cast<size_t>(units) * mla_tc_ws_splits(units, sms) * mla_tc::kPartFloats * sizeof(float);
}

// ws == null: the splits of a sequence form a cluster (at most 16, as many as fit at once) and
// merge in it.  Otherwise one CTA per SM (any number of splits) writes its partial to ws, and
// a second launch merges them (programmatic dependent launch: it is scheduled while the
// first runs and waits for it).  0 = launched, 1 = ws too small, 3 = a CUDA call failed.
int launch_mla_decode_tc(const void *q, const void *c_kv, const int32_t *seqlens, void *out, int B, int h,
                         float scale, long long cache_rows, void *ws, size_t ws_bytes, cudaStream_t stream) {
    using namespace mla_tc;
    auto kern = mla_decode_tc_kernel;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 3;
    static std::atomic<unsigned long long> attr_done{0};
    if (!gqa_host::once_per_device(attr_done, dev, [&] {
            return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Smem::kTotal) ==
                       cudaSuccess &&
                   cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
        }))
        return 3;
    const int sms = gqa_host::sm_count();
    if (ws && ws_bytes < mla_tc_workspace_bytes(B, h, sms)) return 1;
    CUtensorMap tc;
    // token extent = the cache's rows (the kernel cuts lengths that ask for more and reports them)
    const uint64_t dims[2] = {static_cast<uint64_t>(kDc), static_cast<uint64_t>(std::max(cache_rows, 1LL))};
    const uint64_t strides[1] = {static_cast<uint64_t>(kDc) * 2};
    const uint32_t box[2] = {64, kTok};
    if (!gqa_host::encode_tensor_map(&tc, c_kv, 2, dims, strides, box)) return 3;

    const int groups = (h + kHeads - 1) / kHeads;
    const long units = static_cast<long>(B) * groups;
    int P;
    if (ws) {
        P = mla_tc_ws_splits(units, sms);
    } else {   // one CTA per SM: the most splits whose clusters all fit at once
        P = static_cast<int>(std::max(1L, std::min(static_cast<long>(kMaxSplit), sms / units)));
        while (P > 1 && max_active_clusters_tc(P) < units) --P;
    }
    Params prm;
    prm.q = static_cast<const __nv_bfloat16 *>(q);
    prm.seqlens = seqlens;
    prm.out = static_cast<__nv_bfloat16 *>(out);
    prm.B = B;
    prm.h = h;
    prm.cache_rows = cache_rows;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.status = gqa_host::device_status();
    if (!prm.status) return 3;
    prm.part = static_cast<float *>(ws);
    GQA_SET_TEST_STALL(prm);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P, groups, B);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = Smem::kTotal;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ws ? 1 : P;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tc, prm) != cudaSuccess) return 3;
    if (!ws) return 0;
    // the merge: one block per (sequence x group, head)
    cudaLaunchConfig_t mc = {};
    mc.gridDim = dim3(static_cast<unsigned>(units), kHeads, 1);
    mc.blockDim = dim3(kMergeWarps * 32, 1, 1);
    mc.stream = stream;
    cudaLaunchAttribute ma[1];
    ma[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    ma[0].val.programmaticStreamSerializationAllowed = 1;
    mc.attrs = ma;
    mc.numAttrs = 1;
    const float *cpart = static_cast<const float *>(ws);
    __nv_bfloat16 *cout = static_cast<__nv_bfloat16 *>(out);
    if (cudaLaunchKernelEx(&mc, mla_merge_kernel, cpart, cout, h, groups, P) != cudaSuccess) {
        cudaGetLastError();   // without programmatic launch (stream order still holds)
        mla_merge_kernel<<<mc.gridDim, mc.blockDim, 0, stream>>>(cpart, cout, h, groups, P);
        if (cudaGetLastError() != cudaSuccess) return 3;
    }
    return 0;
}

}  // namespace gqa
