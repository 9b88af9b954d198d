// Split-KV decode for wide query groups, on the 5th-generation tensor cores,
// with the cached tokens of the whole batch divided evenly among the SMs.
//
// Semantics: as gqa_decode ("Multi-Query Attention" (inferensys glossary),
// "Decoding Step": softmax(Q_all K_shared^T) V_shared, with G = h / n_kv query
// heads per shared K/V head, "Evolution of AI Attention Mechanisms" (toolsku),
// "GQA Implementation").
//
// Why a second decode kernel.  Per byte of K/V a decode step does G
// multiply-adds for Q K^T and G for P V ("Multi-query attention"
// (pranaymahendrakar), "Why this is a bandwidth argument, not a FLOP
// argument": the bytes scale with n_kv, the FLOPs with h).  For groups of 32
// and more heads the warp-level mma.sync path of the cluster decode kernel
// cannot keep up with HBM; and with ragged lengths a fixed number of splits
// per sequence leaves most SMs idle while the longest sequences finish.  Here:
//   - the G heads of a group are the M = 128 rows of tcgen05 MMAs (padded),
//     the stage's 64 tokens the N columns: S = Q K^T lands in TMEM, one
//     softmax thread per head row turns it into P (bf16, written back over
//     S), and O += P V accumulates in TMEM (A = P from TMEM, B = V from shared
//     memory), exactly the structure of the prefill kernel with the heads of
//     one token in place of the query rows of one head;
//   - work = (KV head, head slice, sequence, token); the batch's tokens of
//     every (KV head, slice) are laid end to end and CTA c of the persistent
//     grid (one per SM) takes the range [c W / NC, (c + 1) W / NC), whatever
//     the sequence boundaries.  A CTA's range is a run of segments (pieces of
//     sequences); a segment wholly inside one CTA is finished there, the
//     pieces of a segment cut between CTAs leave partial results (running
//     max, running sum, unnormalised O) in the caller's workspace, and the
//     last CTA to finish a piece of that segment (an arrival counter per
//     segment) merges them with the log-sum-exp rule and writes the output;
//   - roles: warp 4 streams Q (once per segment) and K/V stages with TMA into
//     a ring, warp 5 allocates TMEM and issues the MMAs, warps 0-3 run the
//     softmax (lazy rescale: the running max moves only when a row's stage
//     max exceeds it by 2^8) and the epilogue.  S is double-buffered in TMEM,
//     so Q K^T of stage i + 1 runs while the softmax of stage i does.
// Workspace: one arrival counter per segment first (padded to 256 bytes),
// then the partial slots (CTA c's piece of segment s goes to slot c + s --
// each CTA's segments and each segment's CTAs are runs, so the (CTA,
// segment) pairs form a staircase and c + s is unique).  The counters must be
// zero when a call starts; every call leaves them zero (the last arriver
// resets its segment's counter), also when a wait times out.
#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace gqa {

constexpr int kSpRows = 128;                 // MMA M: query heads of one KV group (padded)
constexpr int kSpTok = 64;                   // tokens per stage (N of S = Q K^T, K of O += P V)
constexpr int kSpThreads = 192;              // warps 0-3 softmax + epilogue, 4 producer, 5 MMA
constexpr int kSpRingBytes = 192 * 1024;     // K/V ring
constexpr float kSpRescale = 8.0f;           // lazy rescale threshold (log2 units)
constexpr int kSpSplitAllBelow = 256;        // sequences this short also send the weights' bf16 remainders
constexpr uint32_t kSpTmemCols = 256;        // S0 [0, 64), S1 [64, 128), O [128, 128 + D)

template <int D>
struct SplitGeom {
    static constexpr uint32_t kQ = kSpRows * D * 2;     // Q tile: D / 64 panels of 128 rows x 128 bytes
    static constexpr uint32_t kQPanel = kSpRows * 128;
    static constexpr uint32_t kKV = kSpTok * D * 2;     // K (or V) of a stage: D / 64 panels of 64 rows x 128 B
    static constexpr uint32_t kKVPanel = kSpTok * 128;
    static constexpr uint32_t kSlot = 2 * kKV;
    static constexpr int kRing = kSpRingBytes / kSlot;  // 6 (D = 128) or 12 (D = 64)
    static constexpr uint32_t kCtrl = 512;
    static constexpr uint32_t kTotal = kQ + kRing * kSlot + kCtrl + 1024;
    static constexpr uint32_t kPartFloats = kSpRows * D + 2 * kSpRows;   // one partial slot: O, m, l
    static_assert(kRing >= 3, "the ring must hold the stage being multiplied and two ahead");
};

struct SplitParams {
    const __nv_bfloat16 *q;      // [B, h, D]
    const int32_t *seqlens;      // [B]
    __nv_bfloat16 *out;          // [B, h, D]
    float *part;                 // workspace: partial slots
    int *count;                  // workspace: one arrival counter per segment
    int B, h, n_kv, G, slices, nctas;
    uint32_t q_bytes;            // bytes of one Q box (min(128, h) heads)
    long long cache_rows;
    float scale_log2;
    int *status;
    GQA_TEST_STALL_FIELD
};

// One sequence piece of a CTA's range: tokens [t0, t1) of sequence b, for the
// (KV head, head slice) pair gs; w = the segment's first work index.
struct SplitSeg {
    int gs, b, t0, t1, L;        // L = the sequence's (cut) length
    long long off, w;            // first cache row of sequence b; work index of the segment's token 0
};

// Cursor over the segments of a CTA's work range [w_lo, w_hi).  Every role
// runs its own copy; they all see the same sequence of segments.
struct SplitCursor {
    const SplitParams *p;
    long long T, w_cur, w_hi;    // tokens per (KV head, slice); current and end work index
    int gs, b;
    long long off, wb;           // cache row of b (uncut lengths); cut-prefix of b

    // the (cut) length of sequence b given its first row
    __device__ int cut_len(int bb, long long o) const {
        const int l = max(p->seqlens[bb], 0);
        return static_cast<int>(max(0LL, min(static_cast<long long>(l), p->cache_rows - o)));
    }
    // advance to the next sequence (wrapping to the next (KV head, slice) pair)
    __device__ void next_seq() {
        off += max(p->seqlens[b], 0);
        if (++b == p->B) {
            b = 0;
            off = 0;
            wb = 0;
            ++gs;
        }
    }
    __device__ bool next(SplitSeg &s) {
        while (w_cur < w_hi) {
            const int L = cut_len(b, off);
            const long long w0 = gs * T + wb;     // work index of token 0 of this segment
            if (L > 0 && w_cur < w0 + L) {
                s.gs = gs;
                s.b = b;
                s.L = L;
                s.off = off;
                s.w = w0;
                s.t0 = static_cast<int>(w_cur - w0);
                s.t1 = static_cast<int>(min(w_hi, w0 + L) - w0);
                w_cur = w0 + s.t1;
                wb += L;
                next_seq();
                return true;
            }
            wb += L;
            next_seq();
        }
        return false;
    }
};

// owner(w): the CTA whose range [floor(c W / NC), floor((c + 1) W / NC)) holds w
__device__ __forceinline__ int split_owner(long long w, long long W, int nc) {
    return static_cast<int>(((w + 1) * nc - 1) / W);
}

template <int D>
__global__ void __launch_bounds__(kSpThreads, 1)
    gqa_decode_split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const SplitParams p) {
    using SG = SplitGeom<D>;
    constexpr int R = SG::kRing;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sRing = smem + SG::kQ;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sRing + R * SG::kSlot);
    uint64_t *qfull = bars;               // Q of the segment landed
    uint64_t *qfree = qfull + 1;          // the segment's last Q K^T is done (Q may be replaced)
    uint64_t *full = qfree + 1;           // [R] stage landed
    uint64_t *empty = full + R;           // [R] stage's P V done
    uint64_t *sfull = empty + R;          // [2] S buffer written
    uint64_t *pfull = sfull + 2;          // [2] P written over the S buffer (one arrival per softmax warp)
    // [2] P V of stage gi completes phase gi / 2 of pvdone[gi % 2].  Two barriers, because a
    // parity wait only tells the latest phase from the one before it: the softmax waits for
    // P V(x) when P V(x - 2) is known done (S(x + 1) or S(x) ready implies it) and P V(x + 2)
    // cannot have started, so pvdone[x % 2] is then at most one phase from the awaited one
    uint64_t *pvdone = pfull + 2;
    uint64_t *ofree = pvdone + 2;         // the segment's O has been read out of TMEM (one arrival per warp)
    uint64_t *drain = ofree + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    long long *scan = reinterpret_cast<long long *>(drain + 2);   // [8]: block-scan scratch (after tmem/abort)
    int *flag = reinterpret_cast<int *>(scan + 8);                // [1]: last-arriver broadcast

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, NC = p.nctas;

    if (threadIdx.x == 0) {
        mbar_init(qfull, 1);
        mbar_init(qfree, 1);
        for (int i = 0; i < R; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sfull[i], 1);
            mbar_init(&pfull[i], 4);
        }
        mbar_init(&pvdone[0], 1);
        mbar_init(&pvdone[1], 1);
        mbar_init(ofree, 4);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, kSpTmemCols);
        tmem_relinquish();
    }

    // ---- the batch's tokens per (KV head, slice): T = sum of the cut lengths
    // (a sequence is cut where its rows would pass the caches' rows; offsets use
    // the uncut lengths, as the packed layout does)
    long long T = 0;
    {
        long long base_off = 0;
        for (int b0 = 0; b0 < p.B; b0 += kSpThreads) {
            const int bb = b0 + threadIdx.x;
            const long long l = bb < p.B ? max(p.seqlens[bb], 0) : 0;
            // block-wide exclusive scan of l (uncut offsets within this chunk)
            long long x = l;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (lane == 31) scan[warp] = x;
            __syncthreads();
            long long before = 0, chunk = 0;
            for (int w = 0; w < kSpThreads / 32; ++w) {
                if (w < warp) before += scan[w];
                chunk += scan[w];
            }
            const long long off_b = base_off + before + x - l;
            const long long cut = bb < p.B ? max(0LL, min(l, p.cache_rows - off_b)) : 0;
            if (cut < l) record_status(p.status, kStatusInvalid);
            if (bb < p.B && cut == 0 && bb % NC == c) {   // no tokens: a zero output row for every head
                uint4 *o4 = reinterpret_cast<uint4 *>(p.out + static_cast<size_t>(bb) * p.h * D);
                for (int i = 0; i < p.h * D / 8; ++i) o4[i] = make_uint4(0u, 0u, 0u, 0u);
            }
            // block-wide sum of the cut lengths
            long long s = cut;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            __syncthreads();
            if (lane == 0) scan[warp] = s;
            __syncthreads();
            for (int w = 0; w < kSpThreads / 32; ++w) T += scan[w];
            base_off += chunk;
            __syncthreads();
        }
    }
    const long long W = static_cast<long long>(p.n_kv) * p.slices * T;
    // with fewer tokens than CTAs, only the first W CTAs take work (one token each), so
    // that every CTA between a segment's first and last owner holds a piece of it
    const int NCe = W < NC ? static_cast<int>(W) : NC;
    const long long w_lo = c < NCe ? W * c / NCe : W, w_hi = c < NCe ? W * (c + 1) / NCe : W;
    const float cl2 = p.scale_log2;

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto cursor = [&]() {
        SplitCursor cu;
        cu.p = &p;
        cu.T = T;
        cu.w_cur = w_lo;
        cu.w_hi = w_hi;
        cu.gs = 0;
        cu.b = 0;
        cu.off = 0;
        cu.wb = 0;
        // skip whole (KV head, slice) blocks, then whole sequences, before w_lo
        if (T > 0) {
            cu.gs = static_cast<int>(w_lo / T);
            long long r = w_lo - cu.gs * T;
            while (cu.b < p.B) {
                const int L = cu.cut_len(cu.b, cu.off);
                if (r < L) break;
                r -= L;
                cu.wb += L;
                cu.off += max(p.seqlens[cu.b], 0);
                ++cu.b;
            }
        }
        return cu;
    };
    auto n_stages = [](const SplitSeg &s) { return (s.t1 - s.t0 + kSpTok - 1) / kSpTok; };

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            SplitCursor cu = cursor();
            SplitSeg sg;
            int gi = 0, seg = 0;
            const int first_loaded = GQA_STALLED(p) ? 1 : 0;   // wait-test build: stage 0 never arrives
            bool ok = true;
            while (ok && cu.next(sg)) {
                const int g = sg.gs / p.slices, sl = sg.gs % p.slices;
                const int head0 = g * p.G + sl * kSpRows;
                if (seg > 0 && !mbar_wait(qfree, (seg - 1) & 1, abort_flag, p.status)) break;
                mbar_arrive_expect_tx(qfull, p.q_bytes);
                for (int hf = 0; hf < D / 64; ++hf)
                    tma_load_3d(sQ + hf * SG::kQPanel, &tm_q, qfull, hf * 64, head0, sg.b);
                ++seg;   // Q loads issued
                const int n = n_stages(sg);
                for (int i = 0; i < n; ++i, ++gi) {
                    const int slot = gi % R, use = gi / R;
                    if (use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    if (gi < first_loaded) continue;
                    const int z = static_cast<int>(sg.off) + sg.t0 + i * kSpTok;   // first cache row of the stage
                    uint8_t *kd = sRing + slot * SG::kSlot;
                    mbar_arrive_expect_tx(&full[slot], SG::kSlot);
                    for (int hf = 0; hf < D / 64; ++hf) {
                        tma_load_3d(kd + hf * SG::kKVPanel, &tm_k, &full[slot], hf * 64, g, z);
                        tma_load_3d(kd + SG::kKV + hf * SG::kKVPanel, &tm_v, &full[slot], hf * 64, g, z);
                    }
                }
            }
            if (*abort_flag) {   // let the copies in flight land before the CTA moves on
                if (seg > 0) mbar_wait_drain(qfull, (seg - 1) & 1, p.status);
                for (int i = max(first_loaded, gi - R); i < gi; ++i)
                    mbar_wait_drain(&full[i % R], (i / R) & 1, p.status);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer (warp-wide loop, lane 0 issues)
        constexpr uint32_t idesc_qk = idesc_bf16_f32(kSpRows, kSpTok, false, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(kSpRows, D, false, true);
        const uint32_t q_base = smem_u32(sQ);
        const uint32_t ring_base = smem_u32(sRing);
        auto wait1 = [&](uint64_t *bar, uint32_t parity) -> bool {   // lane 0 waits, the warp learns the outcome
            int r = 1;
            if (lane == 0) r = mbar_wait(bar, parity, abort_flag, p.status);
            return __shfl_sync(0xffffffffu, r, 0) != 0;
        };
        auto issue_qk = [&](int gi) {   // S[gi % 2] = Q K(stage gi)^T
            const uint32_t d_tmem = tmem + (gi & 1) * kSpTok;
            const uint32_t b0 = ring_base + (gi % R) * SG::kSlot;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
                umma_ss(d_tmem, sdesc_sw128(q_base + (ks >> 2) * SG::kQPanel + (ks & 3) * 32, 16, 1024),
                        sdesc_sw128(b0 + (ks >> 2) * SG::kKVPanel + (ks & 3) * 32, 16, 1024), idesc_qk, ks > 0);
        };
        auto issue_pv = [&](int gi, bool acc, bool rem) {   // O (+)= P[gi % 2] V(stage gi); rem: the remainders
            const uint32_t a_tmem = tmem + (gi & 1) * kSpTok + (rem ? kSpTok / 2 : 0);
            const uint32_t b0 = ring_base + (gi % R) * SG::kSlot + SG::kKV;
#pragma unroll
            for (int kk = 0; kk < kSpTok / 16; ++kk)
                umma_ts(tmem + 2 * kSpTok, a_tmem + kk * 8, sdesc_sw128(b0 + kk * 16 * 128, SG::kKVPanel, 1024),
                        idesc_pv, (acc || rem || kk > 0) ? 1u : 0u);
        };
        SplitCursor cu = cursor();
        SplitSeg sg;
        int gi0 = 0, seg = 0;
        bool ok = true;
        while (ok && cu.next(sg)) {
            const int n = n_stages(sg);
            const bool split = sg.L <= kSpSplitAllBelow;
            ok = wait1(qfull, seg & 1);
            // Q K^T of the first two stages
            for (int i = 0; i < min(n, 2) && ok; ++i) {
                ok = wait1(&full[(gi0 + i) % R], ((gi0 + i) / R) & 1);
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    issue_qk(gi0 + i);
                    umma_commit(&sfull[(gi0 + i) & 1]);
                    if (i == n - 1) umma_commit(qfree);
                }
                __syncwarp();
            }
            for (int i = 0; i < n && ok; ++i) {
                const int gi = gi0 + i;
                ok = wait1(&pfull[gi & 1], (gi >> 1) & 1);
                if (ok && i == 0 && seg > 0) ok = wait1(ofree, (seg - 1) & 1);   // the last segment's O is read out
                if (!ok) break;
                tc_fence_after();
                const int valid = min(kSpTok, sg.t1 - (sg.t0 + i * kSpTok));
                if (valid < kSpTok) {
                    // the stage runs past the segment: its V rows there belong to other CTAs or
                    // other sequences (or read as zeros); clear them so that 0 * (whatever they
                    // hold) adds nothing
                    uint8_t *vt = sRing + (gi % R) * SG::kSlot + SG::kKV;
                    for (int hf = 0; hf < D / 64; ++hf)
                        for (int it = lane; it < (kSpTok - valid) * 8; it += 32) {
                            const int r = valid + it / 8, ch = it % 8;
                            *reinterpret_cast<uint4 *>(vt + hf * SG::kKVPanel + r * 128 + ch * 16) =
                                make_uint4(0u, 0u, 0u, 0u);
                        }
                    fence_proxy_async_smem();   // generic-proxy stores before the tensor core reads
                    __syncwarp();
                }
                if (lane == 0) {
                    issue_pv(gi, i > 0, false);
                    if (split) issue_pv(gi, true, true);
                    umma_commit(&empty[gi % R]);
                    umma_commit(&pvdone[gi & 1]);
                }
                __syncwarp();
                if (i + 2 < n) {
                    ok = wait1(&full[(gi + 2) % R], ((gi + 2) / R) & 1);
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) {
                        issue_qk(gi + 2);
                        umma_commit(&sfull[gi & 1]);
                        if (i + 2 == n - 1) umma_commit(qfree);
                    }
                    __syncwarp();
                }
            }
            gi0 += n;
            ++seg;
        }
        if (!ok && lane == 0) {   // nothing may still write TMEM when it is freed
            umma_commit(drain);
            mbar_wait_drain(drain, 0, p.status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue (warps 0-3, row = head)
        const int r = warp * 32 + lane;                                  // TMEM lane = head row of the tile
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tO = tmem + 2 * kSpTok + lane_off;
        SplitCursor cu = cursor();
        SplitSeg sg;
        int gi0 = 0, seg = 0;
        bool ok = true;
        while (cu.next(sg)) {
            const int g = sg.gs / p.slices, sl = sg.gs % p.slices;
            const int head0 = g * p.G + sl * kSpRows;
            const int HS = min(p.G - sl * kSpRows, kSpRows);
            const bool live = warp * 32 < HS;                            // this warp holds real heads
            const int n = n_stages(sg);
            const bool split = sg.L <= kSpSplitAllBelow;
            float m_used = -INFINITY, l = 0.f;
            for (int i = 0; i < n && ok; ++i) {
                const int gi = gi0 + i;
                const uint32_t tS = tmem + (gi & 1) * kSpTok + lane_off;
                const bool landed = mbar_wait(&sfull[gi & 1], (gi >> 1) & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, landed)) {   // tcgen05.ld/st are warp-aligned
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (live) {
                    const int valid = min(kSpTok, sg.t1 - (sg.t0 + i * kSpTok));   // columns < valid are tokens
                    uint32_t s0[32], s1[32];
                    tmem_ld32(tS, s0);
                    tmem_ld32(tS + 32, s1);
                    tmem_wait_ld();
#define GQA_SP(cc) ((cc) < 32 ? s0[(cc)] : s1[(cc) - 32])
                    float mx = -INFINITY;
#pragma unroll
                    for (int cc = 0; cc < kSpTok; cc += 2)
                        mx = fmax3(mx, cc < valid ? __uint_as_float(GQA_SP(cc)) : -INFINITY,
                                   cc + 1 < valid ? __uint_as_float(GQA_SP(cc + 1)) : -INFINITY);
                    const float m_tile = mx * cl2;   // >= 1 valid token per stage
                    if (i == 0) {
                        m_used = m_tile;
                    } else {
                        const bool need = m_tile > m_used + kSpRescale;
                        if (__any_sync(0xffffffffu, need)) {
                            // O holds the P V of the earlier stages: wait for the last one, then rescale
                            const bool pv_ok = mbar_wait(&pvdone[(gi - 1) & 1], ((gi - 1) >> 1) & 1, abort_flag,
                                                         p.status);
                            if (!__all_sync(0xffffffffu, pv_ok)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            const float m_new = need ? m_tile : m_used;
                            const float alpha = exp2f(m_used - m_new);
#pragma unroll
                            for (int cc = 0; cc < D / 32; ++cc) {
                                uint32_t ro[32];
                                tmem_ld32(tO + cc * 32, ro);
                                tmem_wait_ld();
#pragma unroll
                                for (int e = 0; e < 32; ++e) ro[e] = __float_as_uint(__uint_as_float(ro[e]) * alpha);
                                tmem_st32(tO + cc * 32, ro);
                            }
                            tmem_wait_st();
                            l *= alpha;
                            m_used = m_new;
                        }
                    }
                    float2 rs = make_float2(0.f, 0.f);
                    auto weights = [&](int cc) -> float2 {
                        const float2 x = ffma2_bcast(__uint_as_float(GQA_SP(cc)), __uint_as_float(GQA_SP(cc + 1)),
                                                     cl2, -m_used);
                        float2 w = make_float2(exp2f(x.x), exp2f(x.y));
                        if (cc >= valid) w.x = 0.f;   // columns past the segment's tokens add nothing
                        if (cc + 1 >= valid) w.y = 0.f;
                        return w;
                    };
                    if (split) {   // the bf16 remainders w - bf16(w) over the upper half of S
                        uint32_t rk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const float2 w = weights(2 * e);
                            const float2 u = unpack_bf16x2(pack_bf16x2(w.x, w.y));
                            rk[e] = pack_bf16x2(w.x - u.x, w.y - u.y);
                            rs = fadd2(rs, unpack_bf16x2(rk[e]));
                        }
                        tmem_st16(tS + kSpTok / 2, rk);
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const float2 w = weights(32 + 2 * e);
                            const float2 u = unpack_bf16x2(pack_bf16x2(w.x, w.y));
                            rk[e] = pack_bf16x2(w.x - u.x, w.y - u.y);
                            rs = fadd2(rs, unpack_bf16x2(rk[e]));
                        }
                        tmem_st16(tS + kSpTok / 2 + 16, rk);
                    }
#pragma unroll
                    for (int ch = 0; ch < kSpTok / 32; ++ch) {
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const float2 w = weights(ch * 32 + 2 * e);
                            pk[e] = pack_bf16x2(w.x, w.y);
                            rs = fadd2(rs, unpack_bf16x2(pk[e]));
                        }
                        tmem_st16(tS + ch * 16, pk);
                    }
#undef GQA_SP
                    l += rs.x + rs.y;
                    tmem_wait_st();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&pfull[gi & 1]);
            }
            gi0 += n;

            // ---- epilogue of the segment: O / l directly, or a partial result and the merge
            const int first_c = split_owner(sg.w, W, NCe), last_c = split_owner(sg.w + sg.L - 1, W, NCe);
            const bool whole = first_c == last_c;
            const int sidx = sg.gs * p.B + sg.b;
            float *slot = p.part + static_cast<size_t>(c + sidx) * SG::kPartFloats;
            bool have_o = false;
            if (ok) {
                const bool fin = mbar_wait(&pvdone[(gi0 - 1) & 1], ((gi0 - 1) >> 1) & 1, abort_flag, p.status);
                have_o = __all_sync(0xffffffffu, fin);
                if (!have_o) ok = false;
            }
            if (have_o && live) {
                tc_fence_after();
                const bool row_ok = r < HS;
                const float inv = 1.f / l;
                __nv_bfloat16 *orow = p.out + (static_cast<size_t>(sg.b) * p.h + head0 + (row_ok ? r : 0)) * D;
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t raw[32];
                    tmem_ld32(tO + cc * 32, raw);
                    tmem_wait_ld();
                    if (!row_ok) continue;
                    if (whole) {
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            pk[e] = pack_bf16x2(__uint_as_float(raw[2 * e]) * inv, __uint_as_float(raw[2 * e + 1]) * inv);
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + cc * 32);
#pragma unroll
                        for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                    } else {
                        uint4 *dst = reinterpret_cast<uint4 *>(slot + static_cast<size_t>(r) * D + cc * 32);
#pragma unroll
                        for (int e = 0; e < 8; ++e) dst[e] = make_uint4(raw[4 * e], raw[4 * e + 1], raw[4 * e + 2], raw[4 * e + 3]);
                    }
                }
                if (!whole && row_ok) {
                    slot[kSpRows * D + r] = m_used;
                    slot[kSpRows * D + kSpRows + r] = l;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ofree);
            ++seg;
            if (!whole) {
                // arrival: the last of the segment's pieces merges them (also after a timeout,
                // so that every counter returns to zero; the outputs are then unspecified)
                __threadfence();
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (threadIdx.x == 0) {
                    const int prev = atomicAdd(&p.count[sidx], 1);
                    const int last = prev == last_c - first_c;
                    if (last) p.count[sidx] = 0;
                    *flag = last;
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (*reinterpret_cast<volatile int *>(flag)) {
                    __threadfence();
                    if (r < HS) {
                        float M = -INFINITY;
                        for (int cc = first_c; cc <= last_c; ++cc)
                            M = fmaxf(M, __ldcg(p.part + static_cast<size_t>(cc + sidx) * SG::kPartFloats + kSpRows * D + r));
                        float Lsum = 0.f;
                        for (int cc = first_c; cc <= last_c; ++cc) {
                            const float *sp = p.part + static_cast<size_t>(cc + sidx) * SG::kPartFloats;
                            Lsum += exp2f(__ldcg(sp + kSpRows * D + r) - M) * __ldcg(sp + kSpRows * D + kSpRows + r);
                        }
                        const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
                        __nv_bfloat16 *orow = p.out + (static_cast<size_t>(sg.b) * p.h + head0 + r) * D;
                        for (int ch = 0; ch < D / 8; ++ch) {
                            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                            for (int cc = first_c; cc <= last_c; ++cc) {
                                const float *sp = p.part + static_cast<size_t>(cc + sidx) * SG::kPartFloats;
                                const float wgt = exp2f(__ldcg(sp + kSpRows * D + r) - M);
                                const float4 a = __ldcg(reinterpret_cast<const float4 *>(sp + static_cast<size_t>(r) * D + ch * 8));
                                const float4 b = __ldcg(reinterpret_cast<const float4 *>(sp + static_cast<size_t>(r) * D + ch * 8 + 4));
                                acc[0] += wgt * a.x; acc[1] += wgt * a.y; acc[2] += wgt * a.z; acc[3] += wgt * a.w;
                                acc[4] += wgt * b.x; acc[5] += wgt * b.y; acc[6] += wgt * b.z; acc[7] += wgt * b.w;
                            }
                            *reinterpret_cast<uint4 *>(orow + ch * 8) =
                                make_uint4(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv),
                                           pack_bf16x2(acc[4] * inv, acc[5] * inv), pack_bf16x2(acc[6] * inv, acc[7] * inv));
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, kSpTmemCols);
    }
}

// ---------------------------------------------------------------------------
// host side

static size_t counter_bytes_for(int B, int n_kv, int slices) {
    const size_t ns = static_cast<size_t>(n_kv) * slices * B;
    return (ns * sizeof(int) + 255) & ~static_cast<size_t>(255);
}

template <int D>
static size_t split_workspace_bytes_t(int B, int n_kv, int slices, int nctas) {
    const size_t ns = static_cast<size_t>(n_kv) * slices * B;
    return counter_bytes_for(B, n_kv, slices) +
           (static_cast<size_t>(nctas) + ns) * SplitGeom<D>::kPartFloats * sizeof(float);
}

size_t split_counter_bytes(int B, int h, int n_kv) {
    const int G = h / n_kv;
    return counter_bytes_for(B, n_kv, (G + kSpRows - 1) / kSpRows);
}

size_t split_workspace_bytes(int B, int h, int n_kv, int d) {
    const int G = h / n_kv;
    const int slices = (G + kSpRows - 1) / kSpRows;
    const int nctas = gqa_host::sm_count();
    return d == 128 ? split_workspace_bytes_t<128>(B, n_kv, slices, nctas)
                    : split_workspace_bytes_t<64>(B, n_kv, slices, nctas);
}

template <int D>
static int launch_split_t(const void *q, const void *k, const void *v, long long cache_rows, const int32_t *seqlens,
                          void *out, int B, int h, int n_kv, float scale, void *workspace, size_t ws_bytes,
                          cudaStream_t stream) {
    using SG = SplitGeom<D>;
    auto kern = gqa_decode_split_kernel<D>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 3;
    static std::atomic<unsigned long long> attr_done{0};
    if (!gqa_host::once_per_device(attr_done, dev, [&] {
            return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SG::kTotal) == cudaSuccess;
        }))
        return 3;
    const int G = h / n_kv;
    const int slices = (G + kSpRows - 1) / kSpRows;
    const int nctas = gqa_host::sm_count();
    if (static_cast<long long>(n_kv) * slices * B > (1LL << 24)) return 2;   // segment indices stay int
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        ws_bytes < split_workspace_bytes_t<D>(B, n_kv, slices, nctas))
        return 1;
    CUtensorMap tq, tk, tv;
    {
        // q [B, h, D]: boxes of 64 dims x min(128, h) heads; rows past h read as zeros, rows of
        // other groups are never stored
        const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(h), static_cast<uint64_t>(B)};
        const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(h) * D * 2};
        const uint32_t box[3] = {64, static_cast<uint32_t>(std::min(kSpRows, h)), 1};
        if (!gqa_host::encode_tensor_map(&tq, q, 3, dims, strides, box)) return 3;
    }
    {
        const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(n_kv),
                                  static_cast<uint64_t>(std::max(cache_rows, 1LL))};
        const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(n_kv) * D * 2};
        const uint32_t box[3] = {64, 1, static_cast<uint32_t>(kSpTok)};
        if (!gqa_host::encode_tensor_map(&tk, k, 3, dims, strides, box)) return 3;
        if (!gqa_host::encode_tensor_map(&tv, v, 3, dims, strides, box)) return 3;
    }
    SplitParams prm = {};
    prm.q = static_cast<const __nv_bfloat16 *>(q);
    prm.seqlens = seqlens;
    prm.out = static_cast<__nv_bfloat16 *>(out);
    prm.count = static_cast<int *>(workspace);
    prm.part = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + counter_bytes_for(B, n_kv, slices));
    prm.B = B;
    prm.h = h;
    prm.n_kv = n_kv;
    prm.G = G;
    prm.slices = slices;
    prm.nctas = nctas;
    prm.q_bytes = static_cast<uint32_t>(D * 2 * std::min(kSpRows, h));
    prm.cache_rows = cache_rows;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.status = gqa_host::device_status();
    if (!prm.status) return 3;
    GQA_SET_TEST_STALL(prm);
    kern<<<nctas, kSpThreads, SG::kTotal, stream>>>(tq, tk, tv, prm);
    return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

int launch_decode_split(const void *q, const void *k, const void *v, long long cache_rows, const int32_t *seqlens,
                        void *out, int B, int h, int n_kv, int d, float scale, void *workspace, size_t ws_bytes,
                        cudaStream_t stream) {
    if (d == 128)
        return launch_split_t<128>(q, k, v, cache_rows, seqlens, out, B, h, n_kv, scale, workspace, ws_bytes, stream);
    return launch_split_t<64>(q, k, v, cache_rows, seqlens, out, B, h, n_kv, scale, workspace, ws_bytes, stream);
}

// ---------------------------------------------------------------------------
// The allocation-free variant: the same kernel, with its workspace in a fixed
// array of the library's own.  Every device that loads the library holds the
// array (kNoAllocScratchBytes) until the process exits.

constexpr size_t kNoAllocScratchBytes = 16u << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_split_scratch[kNoAllocScratchBytes];

// Device address of g_split_scratch on the current device, looked up once per
// device (thread-safe) and kept; null if the lookup fails.
static void *noalloc_scratch() {
    static void *ptrs[64] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_split_scratch) != cudaSuccess) return nullptr;
        ptrs[dev] = ptr;
    }
    return ptrs[dev];
}

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// 0 = launched; 1 = the sizes need more than the fixed array; 3 = a CUDA call failed.
int launch_decode_split_noalloc(const void *q, const void *k, const void *v, long long cache_rows,
                                const int32_t *seqlens, void *out, int B, int h, int n_kv, int d, float scale,
                                cudaStream_t stream) {
    const size_t need = split_workspace_bytes(B, h, n_kv, d);
    if (need > kNoAllocScratchBytes) return 1;
    void *scratch = noalloc_scratch();
    if (!scratch) return 3;
    // the arrival counters must start at zero: clear them on the stream (the rest is scratch)
    if (cudaMemsetAsync(scratch, 0, split_counter_bytes(B, h, n_kv), stream) != cudaSuccess) return 3;
    return launch_decode_split(q, k, v, cache_rows, seqlens, out, B, h, n_kv, d, scale, scratch, need, stream);
}

}  // namespace gqa
