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
//   - the G heads of a group are the M = 128 rows of tcgen05 MMAs, the
//     stage's 64 tokens the N columns: S = Q K^T lands in TMEM (A = Q, held
//     in TMEM; B = K from shared memory), one softmax thread per row turns it
//     into P (bf16, written back over S), and O += P V accumulates in TMEM
//     (A = P from TMEM, B = V from shared memory): the structure of the
//     prefill kernel with the heads of one token in place of the query rows
//     of one head.  A group of at most 64 (32) heads fills the 128 rows with
//     2 (4) copies of its queries; copy k takes its own quarter (half) of
//     every stage's tokens, with its own running max and sum, and the
//     segment's epilogue merges the copies (log-sum-exp, through shared
//     memory), so all four softmax warps work whatever the group size;
//   - work = (KV head, head slice, sequence, token); the batch's tokens of
//     every (KV head, slice) are laid end to end and CTA c of the persistent
//     grid (one per SM) takes the range [c W / NC, (c + 1) W / NC), whatever
//     the sequence boundaries.  A CTA's range is a run of segments (pieces of
//     sequences); a segment wholly inside one CTA is finished there, the
//     pieces of a segment cut between CTAs leave partial results (running
//     max, running sum, unnormalised O) in the caller's workspace, and a
//     second, small kernel merges them with the log-sum-exp rule, one block
//     per (segment, head) on every SM at once;
//   - roles: warp 4 streams the K/V stages with TMA into a ring, warp 5
//     allocates TMEM and issues the MMAs, warps 0-3 write each segment's Q
//     into TMEM (the next segment's as soon as the last S of the current one
//     is read), run the softmax (lazy rescale: the running max moves only
//     when a row's stage max exceeds it by 2^8) and the epilogue.  S is
//     double-buffered in TMEM, so Q K^T of stage i + 1 runs while the
//     softmax of stage i does.
// Workspace: one record per segment first (the CTAs of its first and last
// piece, written by the CTA of the first piece; (-1, -1) for an empty
// sequence), padded to 256 bytes, then the partial slots (CTA c's piece of
// segment s goes to slot c + s -- each CTA's segments and each segment's CTAs
// are runs, so the (CTA, segment) pairs form a staircase and c + s is
// unique).  Every call writes what it reads: the workspace needs no
// initialisation.
#include <algorithm>
#include <mutex>
#include <type_traits>

#include "common.cuh"

namespace gqa {

constexpr int kSpRows = 128;                 // MMA M: query heads of one KV group (padded, or replicated)
constexpr int kSpTok = 64;                   // tokens per stage (N of S = Q K^T, K of O += P V)
constexpr int kSpThreads = 192;              // warps 0-3 softmax + epilogue, 4 producer, 5 MMA
constexpr int kSpRingBytes = 192 * 1024;     // K/V ring
constexpr float kSpRescale = 8.0f;           // lazy rescale threshold (log2 units)
constexpr int kSpSplitAllBelow = 256;        // sequences this short also send the weights' bf16 remainders
constexpr uint32_t kSpTmemCols = 512;        // S0 [0, 64), S1 [64, 128), O [128, 128 + D), Q [256, 256 + D / 2)
constexpr uint32_t kSpQCol = 256;
constexpr int kSpMrgStride = 36;             // floats per row of the replica-merge buffer (32 + 4: no bank conflicts)

template <int D>
struct SplitGeom {
    static constexpr uint32_t kKV = kSpTok * D * 2;     // K (or V) of a stage: D / 64 panels of 64 rows x 128 B
    static constexpr uint32_t kKVPanel = kSpTok * 128;
    static constexpr uint32_t kSlot = 2 * kKV;
    static constexpr int kRing = kSpRingBytes / kSlot;  // 6 (D = 128) or 12 (D = 64)
    static constexpr uint32_t kCtrl = 512;
    static constexpr uint32_t kMerge = (kSpRows * kSpMrgStride + 2 * kSpRows) * 4;   // replica merge: O chunk, m, l
    static constexpr uint32_t kTotal = kRing * kSlot + kCtrl + kMerge + 1024;
    static constexpr uint32_t kPartFloats = kSpRows * D + 2 * kSpRows;   // one partial slot: O, m, l
    static_assert(kRing >= 3, "the ring must hold the stage being multiplied and two ahead");
};

struct SplitParams {
    const __nv_bfloat16 *q;      // [B, h, D]
    const int32_t *seqlens;      // [B]
    __nv_bfloat16 *out;          // [B, h, D]
    float *part;                 // workspace: partial slots
    int2 *seg;                   // workspace: per segment, the CTAs of its first and last piece
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

// T = the batch's tokens per (KV head, slice): the sum of the cut lengths (a
// sequence is cut where its rows would pass the caches' rows, and reported;
// offsets use the uncut lengths, as the packed layout does).  A sequence with
// no tokens gets a zero output row for every head and a (-1, -1) segment
// record, from CTA b % NC.  Called by all NT threads of the block; scan = 8
// long longs of shared memory.
template <int D, int NT>
__device__ long long split_batch_tokens(const SplitParams &p, long long *scan, int c, int NC) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long long T = 0, base_off = 0;
    for (int b0 = 0; b0 < p.B; b0 += NT) {
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
        for (int w = 0; w < NT / 32; ++w) {
            if (w < warp) before += scan[w];
            chunk += scan[w];
        }
        const long long off_b = base_off + before + x - l;
        const long long cut = bb < p.B ? max(0LL, min(l, p.cache_rows - off_b)) : 0;
        if (cut < l) record_status(p.status, kStatusInvalid);
        if (bb < p.B && cut == 0 && bb % NC == c) {   // no tokens: a zero output row for every head
            uint4 *o4 = reinterpret_cast<uint4 *>(p.out + static_cast<size_t>(bb) * p.h * D);
            for (int i = 0; i < p.h * D / 8; ++i) o4[i] = make_uint4(0u, 0u, 0u, 0u);
            for (int gs = 0; gs < p.n_kv * p.slices; ++gs) p.seg[gs * p.B + bb] = make_int2(-1, -1);
        }
        // block-wide sum of the cut lengths
        long long s = cut;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        __syncthreads();
        if (lane == 0) scan[warp] = s;
        __syncthreads();
        for (int w = 0; w < NT / 32; ++w) T += scan[w];
        base_off += chunk;
        __syncthreads();
    }
    return T;
}

// A cursor over the work range [w_lo, w_hi): whole (KV head, slice) blocks,
// then whole sequences, before w_lo are skipped
__device__ SplitCursor split_cursor_at(const SplitParams &p, long long T, long long w_lo, long long w_hi) {
    SplitCursor cu;
    cu.p = &p;
    cu.T = T;
    cu.w_cur = w_lo;
    cu.w_hi = w_hi;
    cu.gs = 0;
    cu.b = 0;
    cu.off = 0;
    cu.wb = 0;
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
}

// bar.red.and over the first n threads of the block on named barrier id: true iff
// pred holds in every one of them
__device__ __forceinline__ bool bar_red_and(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// GP = rows of one copy of the group's heads: 128 (groups of more than 64 heads, in
// slices of 128), 64 or 32.  With GP < 128 the 128 MMA rows hold 128 / GP copies of
// the group's queries, and copy k takes columns [k TPR, (k + 1) TPR) of every stage
// (TPR = 64 GP / 128 tokens): each copy keeps its own running max, sum and O rows,
// over its share of the tokens (its weights for the other copies' tokens are zero),
// and the epilogue merges the copies with the log-sum-exp rule.  So all four softmax
// warps share every stage whatever the group size, and each thread exponentiates
// TPR scores instead of 64.
template <int D, int GP>
__global__ void __launch_bounds__(kSpThreads, 1)
    gqa_decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                            const SplitParams p) {
    using SG = SplitGeom<D>;
    constexpr int NR = SG::kRing;
    constexpr int REP = kSpRows / GP;       // copies of the group's queries down the MMA rows
    constexpr int TPR = kSpTok / REP;       // stage columns of one copy
    static_assert(GP == 32 || GP == 64 || GP == 128, "one copy spans whole warps");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sRing = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sRing + NR * SG::kSlot);
    uint64_t *qfull = bars;               // the segment's Q is in TMEM (one arrival per softmax warp)
    uint64_t *full = qfull + 1;           // [NR] stage landed
    uint64_t *empty = full + NR;          // [NR] stage's P V done
    uint64_t *sfull = empty + NR;         // [2] S buffer written
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
    float *mrg = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(bars) + SG::kCtrl);   // [128][36]
    float *mrg_m = mrg + kSpRows * kSpMrgStride;                  // [128]
    float *mrg_l = mrg_m + kSpRows;                               // [128]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, NC = p.nctas;

    if (threadIdx.x == 0) {
        mbar_init(qfull, 4);
        for (int i = 0; i < NR; ++i) {
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

    const long long T = split_batch_tokens<D, kSpThreads>(p, scan, c, NC);
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

    auto cursor = [&]() { return split_cursor_at(p, T, w_lo, w_hi); };
    auto n_stages = [](const SplitSeg &s) { return (s.t1 - s.t0 + kSpTok - 1) / kSpTok; };

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            SplitCursor cu = cursor();
            SplitSeg sg;
            int gi = 0;
            const int first_loaded = GQA_STALLED(p) ? 1 : 0;   // wait-test build: stage 0 never arrives
            bool ok = true;
            while (ok && cu.next(sg)) {
                const int g = sg.gs / p.slices;
                const int n = n_stages(sg);
                for (int i = 0; i < n; ++i, ++gi) {
                    const int slot = gi % NR, use = gi / NR;
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
                for (int i = max(first_loaded, gi - NR); i < gi; ++i)
                    mbar_wait_drain(&full[i % NR], (i / NR) & 1, p.status);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer (warp-wide loop, lane 0 issues)
        constexpr uint32_t idesc_qk = idesc_bf16_f32(kSpRows, kSpTok, false, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(kSpRows, D, false, true);
        const uint32_t ring_base = smem_u32(sRing);
        auto wait1 = [&](uint64_t *bar, uint32_t parity) -> bool {   // lane 0 waits, the warp learns the outcome
            int r = 1;
            if (lane == 0) r = mbar_wait(bar, parity, abort_flag, p.status);
            return __shfl_sync(0xffffffffu, r, 0) != 0;
        };
        auto issue_qk = [&](int gi) {   // S[gi % 2] = Q K(stage gi)^T, A = Q from TMEM
            const uint32_t d_tmem = tmem + (gi & 1) * kSpTok;
            const uint32_t b0 = ring_base + (gi % NR) * SG::kSlot;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
                umma_ts(d_tmem, tmem + kSpQCol + ks * 8,
                        sdesc_sw128(b0 + (ks >> 2) * SG::kKVPanel + (ks & 3) * 32, 16, 1024), idesc_qk,
                        ks > 0 ? 1u : 0u);
        };
        auto issue_pv = [&](int gi, bool acc, bool rem) {   // O (+)= P[gi % 2] V(stage gi); rem: the remainders
            const uint32_t a_tmem = tmem + (gi & 1) * kSpTok + (rem ? kSpTok / 2 : 0);
            const uint32_t b0 = ring_base + (gi % NR) * SG::kSlot + SG::kKV;
#pragma unroll
            for (int kk = 0; kk < kSpTok / 16; ++kk)
                umma_ts(tmem + 2 * kSpTok, a_tmem + kk * 8, sdesc_sw128(b0 + kk * 16 * 128, SG::kKVPanel, 1024),
                        idesc_pv, (acc || rem || kk > 0) ? 1u : 0u);
        };
        // lane 0 tests a barrier without blocking, the warp learns the outcome
        auto test1 = [&](uint64_t *bar, uint32_t parity) -> bool {
            int r = 0;
            if (lane == 0) r = mbar_try_wait(bar, parity);
            return __shfl_sync(0xffffffffu, r, 0) != 0;
        };
        SplitCursor cu = cursor();
        SplitSeg sg;
        int gi0 = 0, seg = 0;
        bool ok = true;
        while (ok && cu.next(sg)) {
            const int n = n_stages(sg);
            const bool split = sg.L <= kSpSplitAllBelow;
            ok = wait1(qfull, seg & 1);
            // Issue Q K^T(nq) once its stage has landed and P V(nq - 2) is issued (S buffer
            // nq % 2 is free), and P V(np) once its P is written -- whichever is ready first,
            // so that a stage still in flight does not hold back the P V (and the ring slot
            // it frees) of one that is done.  Gives up like mbar_wait when nothing moves.
            int nq = 0, np = 0;
            bool ofree_ok = seg == 0;
            uint32_t idle = 0;
            unsigned long long t_idle = 0;
            while (ok && np < n) {
                bool moved = false;
                if (np < nq) {
                    const int gi = gi0 + np;
                    if (!ofree_ok) ofree_ok = test1(ofree, (seg - 1) & 1);   // the last segment's O is read out
                    if (ofree_ok && test1(&pfull[gi & 1], (gi >> 1) & 1)) {
                        tc_fence_after();
                        const int valid = min(kSpTok, sg.t1 - (sg.t0 + np * kSpTok));
                        if (valid < kSpTok) {
                            // the stage runs past the segment: its V rows there belong to other CTAs or
                            // other sequences (or read as zeros); clear them so that 0 * (whatever they
                            // hold) adds nothing
                            uint8_t *vt = sRing + (gi % NR) * SG::kSlot + SG::kKV;
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
                            issue_pv(gi, np > 0, false);
                            if (split) issue_pv(gi, true, true);
                            umma_commit(&empty[gi % NR]);
                            umma_commit(&pvdone[gi & 1]);
                        }
                        __syncwarp();
                        ++np;
                        moved = true;
                    }
                }
                if (nq < n && nq <= np + 1) {
                    const int gi = gi0 + nq;
                    if (test1(&full[gi % NR], (gi / NR) & 1)) {
                        tc_fence_after();
                        if (lane == 0) {
                            issue_qk(gi);
                            umma_commit(&sfull[gi & 1]);
                        }
                        __syncwarp();
                        ++nq;
                        moved = true;
                    }
                }
                if (moved) {
                    idle = 0;
                } else if (++idle == 1) {
                    t_idle = global_ns();
                } else if ((idle & 63u) == 0) {
                    int give_up = 0;
                    if (lane == 0) {
                        if (*abort_flag) {
                            give_up = 1;
                        } else if (global_ns() - t_idle > kWaitLimitNs) {
                            record_timeout(p.status);
                            *abort_flag = 1;
                            give_up = 1;
                        }
                    }
                    if (__shfl_sync(0xffffffffu, give_up, 0)) ok = false;
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
        // ------------------------------------------------------------ softmax + epilogue (warps 0-3)
        // thread r = TMEM lane r = row r: head hr of copy kr, which owns stage columns [c0, c0 + TPR)
        const int r = warp * 32 + lane;
        const int kr = r / GP, hr = r % GP;            // kr is warp-uniform
        const int c0 = kr * TPR;
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tO = tmem + 2 * kSpTok + lane_off;
        // Q of a segment into TMEM (row r = head hr of the slice; rows past the group's heads are zero)
        auto write_q = [&](const SplitSeg &s) {
            const int g = s.gs / p.slices, sl = s.gs % p.slices;
            const int HS = min(p.G - sl * kSpRows, GP);
            const uint4 *src = reinterpret_cast<const uint4 *>(
                p.q + (static_cast<size_t>(s.b) * p.h + g * p.G + sl * kSpRows + (hr < HS ? hr : 0)) * D);
#pragma unroll
            for (int half = 0; half < D / 64; ++half) {
                uint32_t x[32];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint4 v = hr < HS ? src[half * 8 + e] : make_uint4(0u, 0u, 0u, 0u);
                    x[4 * e] = v.x;
                    x[4 * e + 1] = v.y;
                    x[4 * e + 2] = v.z;
                    x[4 * e + 3] = v.w;
                }
                tmem_st32(tmem + kSpQCol + half * 32 + lane_off, x);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(qfull);
        };
        // this thread's packed weights (TPR / 2 columns from c0 / 2) and zeros in the other
        // copies' columns, over columns [base, base + 32) of its S row
        auto put_p = [&](uint32_t tS, uint32_t base, const uint32_t (&pk)[TPR / 2]) {
            if constexpr (REP == 1) {
                uint32_t a[16], b2[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    a[e] = pk[e];
                    b2[e] = pk[16 + e];
                }
                tmem_st16(tS + base, a);
                tmem_st16(tS + base + 16, b2);
            } else if constexpr (REP == 2) {
                uint32_t z[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) z[e] = 0u;
                tmem_st16(tS + base + c0 / 2, pk);
                tmem_st16(tS + base + (16 - c0 / 2), z);
            } else {
                uint32_t z[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) z[e] = 0u;
                tmem_st8(tS + base + c0 / 2, pk);
#pragma unroll
                for (int k = 1; k < REP; ++k) tmem_st8(tS + base + ((kr + k) % REP) * 8, z);
            }
        };
        SplitCursor cu = cursor();
        SplitSeg sg;
        int gi0 = 0, seg = 0;
        bool ok = true;
        bool have = cu.next(sg);
        if (have) write_q(sg);
        while (have) {
            const int g = sg.gs / p.slices, sl = sg.gs % p.slices;
            const int head0 = g * p.G + sl * kSpRows;
            const int HS = min(p.G - sl * kSpRows, GP);
            const bool live = REP > 1 || warp * 32 < HS;                 // this warp holds real heads
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
                    // columns c0 + j, j < vm, are tokens of the segment (vm may be <= 0 for a copy
                    // whose share of the segment's last stage is empty)
                    const int vm = min(kSpTok, sg.t1 - (sg.t0 + i * kSpTok)) - c0;
                    uint32_t s[TPR];
                    if constexpr (TPR == 16) {
                        tmem_ld16(tS + c0, s);
                    } else if constexpr (TPR == 32) {
                        tmem_ld32(tS + c0, s);
                    } else {
                        uint32_t s0[32], s1[32];
                        tmem_ld32(tS, s0);
                        tmem_ld32(tS + 32, s1);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            s[j] = s0[j];
                            s[32 + j] = s1[j];
                        }
                    }
                    tmem_wait_ld();
                    float mx = -INFINITY;
#pragma unroll
                    for (int j = 0; j < TPR; j += 2)
                        mx = fmax3(mx, j < vm ? __uint_as_float(s[j]) : -INFINITY,
                                   j + 1 < vm ? __uint_as_float(s[j + 1]) : -INFINITY);
                    const float m_tile = mx == -INFINITY ? -INFINITY : mx * cl2;
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
                            const float alpha = exp2f(m_used - m_new);   // 0 while m_used is -inf
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
                    auto weights = [&](int j) -> float2 {
                        const float2 x = ffma2_bcast(__uint_as_float(s[j]), __uint_as_float(s[j + 1]), cl2, -m_used);
                        float2 w = make_float2(exp2f(x.x), exp2f(x.y));
                        if (j >= vm) w.x = 0.f;   // columns past the segment's tokens add nothing
                        if (j + 1 >= vm) w.y = 0.f;
                        return w;
                    };
                    uint32_t pk[TPR / 2];
                    if (split) {   // the bf16 remainders w - bf16(w), over the upper half of S
#pragma unroll
                        for (int e = 0; e < TPR / 2; ++e) {
                            const float2 w = weights(2 * e);
                            const float2 u = unpack_bf16x2(pack_bf16x2(w.x, w.y));
                            pk[e] = pack_bf16x2(w.x - u.x, w.y - u.y);
                            rs = fadd2(rs, unpack_bf16x2(pk[e]));
                        }
                        put_p(tS, kSpTok / 2, pk);
                    }
#pragma unroll
                    for (int e = 0; e < TPR / 2; ++e) {
                        const float2 w = weights(2 * e);
                        pk[e] = pack_bf16x2(w.x, w.y);
                        rs = fadd2(rs, unpack_bf16x2(pk[e]));
                    }
                    put_p(tS, 0, pk);
                    l += rs.x + rs.y;
                    tmem_wait_st();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&pfull[gi & 1]);
            }
            gi0 += n;
            const SplitSeg cur = sg;
            have = cu.next(sg);
            // the next segment's Q: every Q K^T of this one is done (its S were all read above)
            if (have && ok) write_q(sg);

            // ---- epilogue of the segment: O / l directly, or a partial result and the merge
            const int first_c = split_owner(cur.w, W, NCe), last_c = split_owner(cur.w + cur.L - 1, W, NCe);
            const bool whole = first_c == last_c;
            const int sidx = cur.gs * p.B + cur.b;
            float *slot = p.part + static_cast<size_t>(c + sidx) * SG::kPartFloats;
            bool have_o = false;
            if (ok) {
                const bool fin = mbar_wait(&pvdone[(gi0 - 1) & 1], ((gi0 - 1) >> 1) & 1, abort_flag, p.status);
                have_o = __all_sync(0xffffffffu, fin);
                if (!have_o) ok = false;
            }
            if constexpr (REP == 1) {
                if (have_o && live) {
                    tc_fence_after();
                    const bool row_ok = r < HS;
                    const float inv = 1.f / l;
                    __nv_bfloat16 *orow = p.out + (static_cast<size_t>(cur.b) * p.h + head0 + (row_ok ? r : 0)) * D;
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
                                pk[e] = pack_bf16x2(__uint_as_float(raw[2 * e]) * inv,
                                                    __uint_as_float(raw[2 * e + 1]) * inv);
                            uint4 *dst = reinterpret_cast<uint4 *>(orow + cc * 32);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                        } else {
                            uint4 *dst = reinterpret_cast<uint4 *>(slot + static_cast<size_t>(r) * D + cc * 32);
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                dst[e] = make_uint4(raw[4 * e], raw[4 * e + 1], raw[4 * e + 2], raw[4 * e + 3]);
                        }
                    }
                    if (!whole && row_ok) {
                        slot[kSpRows * D + r] = m_used;
                        slot[kSpRows * D + kSpRows + r] = l;
                    }
                }
            } else {
                // merge the copies of head hr through shared memory, 32 columns of O at a time;
                // thread (kr, hr) then produces columns [kr CW, (kr + 1) CW) of each chunk.
                // Every softmax thread takes the same barriers whatever happened above.
                constexpr int CW = 32 / REP;
                const bool go = bar_red_and(1, 128, have_o);
                mrg_m[r] = m_used;
                asm volatile("bar.sync 1, 128;" ::: "memory");
                float M = -INFINITY;
#pragma unroll
                for (int k = 0; k < REP; ++k) M = fmaxf(M, mrg_m[k * GP + hr]);
                const float sc = m_used == -INFINITY ? 0.f : exp2f(m_used - M);
                mrg_l[r] = l * sc;
                const bool row_ok = go && hr < HS;
                __nv_bfloat16 *orow = p.out + (static_cast<size_t>(cur.b) * p.h + head0 + (hr < HS ? hr : 0)) * D;
                float inv = 0.f, lsum = 0.f;
                if (go) tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t raw[32];
                    if (go) {
                        tmem_ld32(tO + cc * 32, raw);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) raw[e] = 0u;
                    }
                    float4 *mine = reinterpret_cast<float4 *>(mrg + r * kSpMrgStride);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        mine[e] = make_float4(__uint_as_float(raw[4 * e]) * sc, __uint_as_float(raw[4 * e + 1]) * sc,
                                              __uint_as_float(raw[4 * e + 2]) * sc,
                                              __uint_as_float(raw[4 * e + 3]) * sc);
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                    if (cc == 0) {
#pragma unroll
                        for (int k = 0; k < REP; ++k) lsum += mrg_l[k * GP + hr];
                        inv = 1.f / lsum;
                    }
                    float acc[CW];
#pragma unroll
                    for (int e = 0; e < CW; ++e) acc[e] = 0.f;
#pragma unroll
                    for (int k = 0; k < REP; ++k) {
                        const float4 *src = reinterpret_cast<const float4 *>(mrg + (k * GP + hr) * kSpMrgStride + kr * CW);
#pragma unroll
                        for (int e = 0; e < CW / 4; ++e) {
                            const float4 v = src[e];
                            acc[4 * e] += v.x;
                            acc[4 * e + 1] += v.y;
                            acc[4 * e + 2] += v.z;
                            acc[4 * e + 3] += v.w;
                        }
                    }
                    if (row_ok) {
                        const int col = cc * 32 + kr * CW;
                        if (whole) {
                            uint4 *dst = reinterpret_cast<uint4 *>(orow + col);
#pragma unroll
                            for (int e = 0; e < CW / 8; ++e)
                                dst[e] = make_uint4(pack_bf16x2(acc[8 * e] * inv, acc[8 * e + 1] * inv),
                                                    pack_bf16x2(acc[8 * e + 2] * inv, acc[8 * e + 3] * inv),
                                                    pack_bf16x2(acc[8 * e + 4] * inv, acc[8 * e + 5] * inv),
                                                    pack_bf16x2(acc[8 * e + 6] * inv, acc[8 * e + 7] * inv));
                        } else {
                            float4 *dst = reinterpret_cast<float4 *>(slot + static_cast<size_t>(hr) * D + col);
#pragma unroll
                            for (int e = 0; e < CW / 4; ++e)
                                dst[e] = make_float4(acc[4 * e], acc[4 * e + 1], acc[4 * e + 2], acc[4 * e + 3]);
                        }
                    }
                    asm volatile("bar.sync 1, 128;" ::: "memory");   // the buffer is free for the next chunk
                }
                if (row_ok && !whole && kr == 0) {
                    slot[kSpRows * D + hr] = M;
                    slot[kSpRows * D + kSpRows + hr] = lsum;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ofree);
            ++seg;
            // the segment's record for the merge kernel, from the CTA of its first piece
            if (c == first_c && threadIdx.x == 0) p.seg[sidx] = make_int2(first_c, last_c);
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
// Tokens as rows, for groups of at most 64 heads (d = 128).  With the heads
// as the rows, a group of 32 heads leaves its softmax to one warp of the
// four that can reach its TMEM lanes; here a stage's 128 tokens are the M
// rows instead, so all four softmax warps share the work:
//   S^T = K Q^T        M = 128 tokens, N = 64 heads (padded), K = d      (TMEM)
//   P^T = exp2(S^T c - m)  per column (head), thread = token row, written as
//                      bf16 to shared memory (token rows of 64 heads)
//   O^T += V^T P^T     M = 128 (d), N = 64 heads, K = 128 tokens; A = V read
//                      MN-major from the stage's tile, B = P^T        (TMEM)
// The running max per head is lazy: taken over the segment's first stage
// (a column max across the 128 token threads), it moves only when a score
// passes it by more than 2^8 (a vote among the softmax warps; then the O^T
// columns and the sums are rescaled).  Each thread keeps its own partial
// column sums; they are reduced across the threads when the segment ends.
// K and V stream through one ring of 32 KB items (K(i) = item 2i, V(i) =
// item 2i + 1), so a K tile is released as soon as its Q K^T is done.

constexpr int kTkTok = 128;              // tokens per stage: MMA M of S^T = K Q^T
constexpr int kTkN = 64;                 // MMA N: the slice's heads, padded
constexpr int kTkItems = 6;              // ring of K / V items
constexpr uint32_t kTkTmemCols = 256;    // S^T [0, 64) and [64, 128); O^T [128, 192)
constexpr float kTkRescale = 8.0f;       // lazy rescale threshold (log2 units)

struct TokGeom {                         // D = 128
    static constexpr int D = 128;
    static constexpr uint32_t kQPanel = kTkN * 128;        // Q: 2 panels of 64 heads x 128 B
    static constexpr uint32_t kQ = 2 * kQPanel;
    static constexpr uint32_t kItemPanel = kTkTok * 128;   // K or V of a stage: 2 panels of 128 tokens x 128 B
    static constexpr uint32_t kItem = 2 * kItemPanel;
    static constexpr uint32_t kP = kTkTok * 128;           // P^T: 128 token rows of 64 bf16 heads, 128B swizzled
    static constexpr uint32_t kRed = 4 * kTkN * 4;         // [4 warps][64 heads] float exchange buffer
    static constexpr uint32_t kMsh = kTkN * 4;             // running max per head
    static constexpr uint32_t kCres = kTkN * 4;            // a column reduction's 64 results
    static constexpr uint32_t kCtrl = 512;
    static constexpr uint32_t kTotal = kQ + kP + kTkItems * kItem + kRed + kMsh + kCres + kCtrl + 1024;
    static constexpr uint32_t kPartFloats = SplitGeom<128>::kPartFloats;   // the workspace slot of the other kernel
};
static_assert(TokGeom::kTotal <= 232448, "shared memory of the tokens-as-rows kernel");

template <int NH>   // the slice's heads as the N of S^T = K Q^T: 16, 32 or 64 (the group, rounded up)
__global__ void __launch_bounds__(kSpThreads, 1)
    gqa_decode_split_tok_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                                const __grid_constant__ CUtensorMap tm_v, const SplitParams p) {
    using TG = TokGeom;
    constexpr int D = TG::D;
    constexpr int R = kTkItems;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sP = sQ + TG::kQ;
    uint8_t *sRing = sP + TG::kP;
    float *red = reinterpret_cast<float *>(sRing + R * TG::kItem);   // [4][64]
    float *msh = red + 4 * kTkN;                                  // [64] running max (log2 units)
    float *cres = msh + kTkN;                                     // [64] a column reduction's results
    uint64_t *bars = reinterpret_cast<uint64_t *>(cres + kTkN);
    uint64_t *qfull = bars;
    uint64_t *qfree = qfull + 1;
    uint64_t *full = qfree + 1;            // [R]
    uint64_t *empty = full + R;            // [R]
    uint64_t *sfull = empty + R;           // [2] S^T buffer written
    uint64_t *sfree = sfull + 2;           // [2] S^T buffer read by every softmax warp
    uint64_t *pfull = sfree + 2;           // P^T published (one arrival per softmax warp per publication)
    uint64_t *pvdone = pfull + 1;          // every P V, in order (phase k = publication k)
    uint64_t *ofree = pvdone + 1;          // the segment's O^T read out (one arrival per warp)
    uint64_t *drain = ofree + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    long long *scan = reinterpret_cast<long long *>(drain + 2);   // [8]
    int *vote = reinterpret_cast<int *>(scan + 8);                // [3] rescale votes, by stage % 3

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
            mbar_init(&sfree[i], 4);
        }
        mbar_init(pfull, 4);
        mbar_init(pvdone, 1);
        mbar_init(ofree, 4);
        mbar_init(drain, 1);
        *abort_flag = 0;
        vote[0] = vote[1] = vote[2] = 0;
        fence_barrier_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, kTkTmemCols);
        tmem_relinquish();
    }
    // P^T columns NH..63 are read by P V (N = 64) and never written: zero them once
    for (int i = threadIdx.x; i < static_cast<int>(TG::kP / 16); i += kSpThreads)
        reinterpret_cast<uint4 *>(sP)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();

    const long long T = split_batch_tokens<D, kSpThreads>(p, scan, c, NC);
    const long long W = static_cast<long long>(p.n_kv) * p.slices * T;
    const int NCe = W < NC ? static_cast<int>(W) : NC;
    const long long w_lo = c < NCe ? W * c / NCe : W, w_hi = c < NCe ? W * (c + 1) / NCe : W;
    const float cl2 = p.scale_log2;

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto cursor = [&]() { return split_cursor_at(p, T, w_lo, w_hi); };
    auto n_stages = [](const SplitSeg &sg) { return (sg.t1 - sg.t0 + kTkTok - 1) / kTkTok; };

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            SplitCursor cu = cursor();
            SplitSeg sg;
            int it = 0, seg = 0;
            const int first_loaded = GQA_STALLED(p) ? 1 : 0;   // wait-test build: item 0 never arrives
            bool ok = true;
            while (ok && cu.next(sg)) {
                const int g = sg.gs / p.slices;
                const int head0 = g * p.G;
                if (seg > 0 && !mbar_wait(qfree, (seg - 1) & 1, abort_flag, p.status)) break;
                mbar_arrive_expect_tx(qfull, p.q_bytes);
                for (int hf = 0; hf < D / 64; ++hf)
                    tma_load_3d(sQ + hf * TG::kQPanel, &tm_q, qfull, hf * 64, head0, sg.b);
                ++seg;
                const int n = n_stages(sg);
                for (int i = 0; i < n && ok; ++i) {
                    const int z = static_cast<int>(sg.off) + sg.t0 + i * kTkTok;   // first cache row of the stage
                    for (int kv = 0; kv < 2; ++kv, ++it) {
                        const int slot = it % R, use = it / R;
                        if (use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1, abort_flag, p.status)) {
                            ok = false;
                            break;
                        }
                        if (it < first_loaded) continue;
                        uint8_t *dst = sRing + slot * TG::kItem;
                        mbar_arrive_expect_tx(&full[slot], TG::kItem);
                        for (int hf = 0; hf < D / 64; ++hf)
                            tma_load_3d(dst + hf * TG::kItemPanel, kv ? &tm_v : &tm_k, &full[slot], hf * 64, g, z);
                    }
                }
            }
            if (*abort_flag) {   // let the copies in flight land before the CTA moves on
                if (seg > 0) mbar_wait_drain(qfull, (seg - 1) & 1, p.status);
                for (int i = max(first_loaded, it - R); i < it; ++i)
                    mbar_wait_drain(&full[i % R], (i / R) & 1, p.status);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer (warp-wide, lane 0 issues)
        constexpr uint32_t idesc_qk = idesc_bf16_f32(kTkTok, NH, false, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(kTkTok, kTkN, true, true);
        const uint32_t q_base = smem_u32(sQ);
        const uint32_t p_base = smem_u32(sP);
        const uint32_t ring_base = smem_u32(sRing);
        auto wait1 = [&](uint64_t *bar, uint32_t parity) -> bool {
            int r = 1;
            if (lane == 0) r = mbar_wait(bar, parity, abort_flag, p.status);
            return __shfl_sync(0xffffffffu, r, 0) != 0;
        };
        auto issue_qk = [&](int gi) {   // S^T[gi % 2] = K(gi) Q^T
            const uint32_t a0 = ring_base + ((2 * gi) % R) * TG::kItem;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
                umma_ss(tmem + (gi & 1) * kTkN,
                        sdesc_sw128(a0 + (ks >> 2) * TG::kItemPanel + (ks & 3) * 32, 16, 1024),
                        sdesc_sw128(q_base + (ks >> 2) * TG::kQPanel + (ks & 3) * 32, 16, 1024), idesc_qk, ks > 0);
        };
        auto issue_pv = [&](int gi, bool acc) {   // O^T (+)= V(gi)^T P^T
            const uint32_t a0 = ring_base + ((2 * gi + 1) % R) * TG::kItem;
#pragma unroll
            for (int kk = 0; kk < kTkTok / 16; ++kk)
                umma_ss(tmem + 2 * kTkN, sdesc_sw128(a0 + kk * 16 * 128, TG::kItemPanel, 1024),
                        sdesc_sw128(p_base + kk * 16 * 128, TG::kItemPanel, 1024), idesc_pv, (acc || kk > 0) ? 1u : 0u);
        };
        SplitCursor cu = cursor();
        SplitSeg sg;
        int gi0 = 0, seg = 0, pub = 0;
        bool ok = true;
        while (ok && cu.next(sg)) {
            const int n = n_stages(sg);
            const int pubs = sg.L <= kSpSplitAllBelow ? 2 : 1;   // P^T published once, or twice (bf16 + remainders)
            ok = wait1(qfull, seg & 1);
            for (int i = 0; i < min(n, 2) && ok; ++i) {
                ok = wait1(&full[(2 * (gi0 + i)) % R], ((2 * (gi0 + i)) / R) & 1);
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    issue_qk(gi0 + i);
                    umma_commit(&sfull[(gi0 + i) & 1]);
                    umma_commit(&empty[(2 * (gi0 + i)) % R]);
                    if (i == n - 1) umma_commit(qfree);
                }
                __syncwarp();
            }
            for (int i = 0; i < n && ok; ++i) {
                const int gi = gi0 + i;
                if (i + 2 < n) {   // Q K^T two stages ahead, as soon as S^T(gi) has been read
                    ok = wait1(&sfree[gi & 1], (gi >> 1) & 1) && wait1(&full[(2 * (gi + 2)) % R], ((2 * (gi + 2)) / R) & 1);
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) {
                        issue_qk(gi + 2);
                        umma_commit(&sfull[gi & 1]);
                        umma_commit(&empty[(2 * (gi + 2)) % R]);
                        if (i + 2 == n - 1) umma_commit(qfree);
                    }
                    __syncwarp();
                }
                ok = wait1(&full[(2 * gi + 1) % R], ((2 * gi + 1) / R) & 1);
                if (ok && i == 0 && seg > 0) ok = wait1(ofree, (seg - 1) & 1);   // the last segment's O^T is read out
                if (!ok) break;
                const int valid = min(kTkTok, sg.t1 - (sg.t0 + i * kTkTok));
                if (valid < kTkTok) {   // V rows past the segment's tokens: cleared (0 * whatever adds nothing)
                    uint8_t *vt = sRing + ((2 * gi + 1) % R) * TG::kItem;
                    for (int hf = 0; hf < D / 64; ++hf)
                        for (int e = lane; e < (kTkTok - valid) * 8; e += 32) {
                            const int r = valid + e / 8, ch = e % 8;
                            *reinterpret_cast<uint4 *>(vt + hf * TG::kItemPanel + r * 128 + ch * 16) =
                                make_uint4(0u, 0u, 0u, 0u);
                        }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                for (int ps = 0; ps < pubs && ok; ++ps, ++pub) {
                    ok = wait1(pfull, pub & 1);
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) {
                        issue_pv(gi, i > 0 || ps > 0);
                        if (ps == pubs - 1) umma_commit(&empty[(2 * gi + 1) % R]);
                        umma_commit(pvdone);
                    }
                    __syncwarp();
                }
            }
            gi0 += n;
            ++seg;
        }
        if (!ok && lane == 0) {
            umma_commit(drain);
            mbar_wait_drain(drain, 0, p.status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue (warps 0-3)
        const int r = warp * 32 + lane;                                  // TMEM lane: token row of S^T, d of O^T
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tO = tmem + 2 * kTkN + lane_off;
        const int tid = threadIdx.x;                                      // 0..127
        SplitCursor cu = cursor();
        SplitSeg sg;
        int gi0 = 0, pub = 0;
        bool ok = true;
        // NH consecutive 32-bit TMEM columns of this thread's lane
        auto tmem_row = [&](uint32_t taddr, float (&x)[NH]) {
            if constexpr (NH == 16) {
                uint32_t raw[16];
                tmem_ld16(taddr, raw);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < 16; ++h) x[h] = __uint_as_float(raw[h]);
            } else {
#pragma unroll
                for (int q32 = 0; q32 < NH / 32; ++q32) {
                    uint32_t raw[32];
                    tmem_ld32(taddr + q32 * 32, raw);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < 32; ++h) x[q32 * 32 + h] = __uint_as_float(raw[h]);
                }
            }
        };
        // column reduction over the 128 token threads of NH per-thread values (max or sum)
        // into dst[NH] in shared memory (each use separated from the next by a barrier)
        auto colreduce = [&](const float (&x)[NH], bool is_max, float *dst) {
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                float v = x[h];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float u = __shfl_xor_sync(0xffffffffu, v, o);
                    v = is_max ? fmaxf(v, u) : v + u;
                }
                if (lane == 0) red[warp * kTkN + h] = v;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (tid < NH) {
                const float a = red[tid], b2 = red[kTkN + tid], c2 = red[2 * kTkN + tid], d2 = red[3 * kTkN + tid];
                dst[tid] = is_max ? fmaxf(fmaxf(a, b2), fmaxf(c2, d2)) : (a + b2) + (c2 + d2);
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
        };
        auto load_m = [&](float (&m)[NH]) {
#pragma unroll
            for (int h = 0; h < NH; h += 4) {
                const float4 v4 = *reinterpret_cast<const float4 *>(msh + h);
                m[h] = v4.x;
                m[h + 1] = v4.y;
                m[h + 2] = v4.z;
                m[h + 3] = v4.w;
            }
        };
        while (cu.next(sg)) {
            const int g = sg.gs / p.slices;
            const int head0 = g * p.G;
            const int HS = min(p.G, NH);
            const int n = n_stages(sg);
            const bool split = sg.L <= kSpSplitAllBelow;
            float2 ls[NH / 2];   // this thread's share of the column sums
#pragma unroll
            for (int j = 0; j < NH / 2; ++j) ls[j] = make_float2(0.f, 0.f);
            // the running max per head (log2 units): msh, copied into registers when they allow
            constexpr bool kMReg = NH <= 32;
            float m[kMReg ? NH : 1];
#pragma unroll
            for (int h = 0; h < (kMReg ? NH : 1); ++h) m[h] = -INFINITY;   // set from msh before first use
            auto mv = [&](int h) -> float {
                if constexpr (kMReg) return m[h];
                else return msh[h];
            };
            for (int i = 0; i < n && ok; ++i) {
                const int gi = gi0 + i;
                const bool landed = mbar_wait(&sfull[gi & 1], (gi >> 1) & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, landed)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float x[NH];
                tmem_row(tmem + (gi & 1) * kTkN + lane_off, x);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfree[gi & 1]);   // S^T(gi) may be overwritten
                const int valid = min(kTkTok, sg.t1 - (sg.t0 + i * kTkTok));
                const bool tok_ok = r < valid;
                if (i == 0) {   // the segment's running max starts at its first stage's column max
                    float xs[NH];
#pragma unroll
                    for (int h = 0; h < NH; ++h) xs[h] = tok_ok ? x[h] * cl2 : -INFINITY;
                    colreduce(xs, true, msh);
                    if constexpr (kMReg) load_m(m);
                }
                // exponent arguments e = S c - m, in place, and this thread's largest (real heads)
                float emax = -INFINITY;
#pragma unroll
                for (int h = 0; h < NH; h += 2) {
                    const float2 e = ffma2(x[h], x[h + 1], cl2, -mv(h), -mv(h + 1));
                    x[h] = e.x;
                    x[h + 1] = e.y;
                    emax = fmax3(emax, h < HS ? e.x : -INFINITY, h + 1 < HS ? e.y : -INFINITY);
                }
                // vote[gi % 3] collects this stage's votes; after the barrier everyone reads it,
                // and vote[(gi + 2) % 3] -- read at the stage before this one, written next at
                // the stage after the next barrier -- is cleared
                bool rescale = false;
                if (i > 0) {
                    if (__any_sync(0xffffffffu, tok_ok && emax > kTkRescale) && lane == 0) atomicOr(&vote[gi % 3], 1);
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                    rescale = *reinterpret_cast<volatile int *>(&vote[gi % 3]) != 0;
                }
                if (tid == 0) vote[(gi + 2) % 3] = 0;
                if (rescale) {
                    // the new column max (into cres); O^T (after the last P V), the sums and the
                    // exponent arguments move to it
                    {
                        float xs[NH];
#pragma unroll
                        for (int h = 0; h < NH; ++h) xs[h] = tok_ok ? x[h] + mv(h) : -INFINITY;
                        colreduce(xs, true, cres);
                    }
                    const bool pv_ok = mbar_wait(pvdone, (pub - 1) & 1, abort_flag, p.status);
                    if (!__all_sync(0xffffffffu, pv_ok)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        const float mo = mv(h), mn = fmaxf(mo, cres[h]);
                        const float a = exp2f(mo - mn);
                        x[h] += mo - mn;
                        if (h & 1) ls[h / 2].y *= a; else ls[h / 2].x *= a;
                        if constexpr (kMReg) m[h] = mn;   // (msh keeps the old max until below)
                    }
#pragma unroll 1
                    for (int q8 = 0; q8 < NH / 8; ++q8) {   // O^T columns in groups of 8
                        uint32_t raw[8];
                        tmem_ld8(tO + q8 * 8, raw);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int h = q8 * 8 + e;
                            const float mo = msh[h], mn = fmaxf(mo, cres[h]);
                            raw[e] = __float_as_uint(__uint_as_float(raw[e]) * exp2f(mo - mn));
                        }
                        tmem_st8(tO + q8 * 8, raw);
                    }
                    tmem_wait_st();
                    asm volatile("bar.sync 1, 128;" ::: "memory");   // every thread has read msh and cres
                    if (tid < NH) msh[tid] = fmaxf(msh[tid], cres[tid]);
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                }
                // P^T row of this token: the weights exp2(e) of the HS heads (0 past them and for
                // rows past the segment's tokens); twice for a split segment (bf16, then the bf16
                // remainders), each after the previous P V has read the buffer
                for (int ps = 0; ps < (split ? 2 : 1); ++ps, ++pub) {
                    if (pub > 0) {   // the previous P V has read the buffer
                        const bool pv_ok = mbar_wait(pvdone, (pub - 1) & 1, abort_flag, p.status);
                        if (!__all_sync(0xffffffffu, pv_ok)) {
                            ok = false;
                            break;
                        }
                    }
                    uint8_t *prow = sP + r * 128;
#pragma unroll
                    for (int ch = 0; ch < NH / 8; ++ch) {   // 8 heads per 16-byte chunk of the row
                        uint32_t pk[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const int h = ch * 8 + 2 * e2;
                            float w0 = tok_ok && h < HS ? exp2f(x[h]) : 0.f;
                            float w1 = tok_ok && h + 1 < HS ? exp2f(x[h + 1]) : 0.f;
                            uint32_t q2 = pack_bf16x2(w0, w1);
                            if (ps == 1) {   // the remainders w - bf16(w), exact in fp32
                                const float2 u = unpack_bf16x2(q2);
                                q2 = pack_bf16x2(w0 - u.x, w1 - u.y);
                            }
                            ls[h / 2] = fadd2(ls[h / 2], unpack_bf16x2(q2));
                            pk[e2] = q2;
                        }
                        *reinterpret_cast<uint4 *>(prow + (((ch ^ r) & 7) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(pfull);
                }
            }
            gi0 += n;

            // ---- epilogue: column sums, O^T, then the output or a partial result
            const int first_c = split_owner(sg.w, W, NCe), last_c = split_owner(sg.w + sg.L - 1, W, NCe);
            const bool whole = first_c == last_c;
            const int sidx = sg.gs * p.B + sg.b;
            float *slot = p.part + static_cast<size_t>(c + sidx) * TG::kPartFloats;
            {
                float lf[NH];
#pragma unroll
                for (int j = 0; j < NH / 2; ++j) {
                    lf[2 * j] = ls[j].x;
                    lf[2 * j + 1] = ls[j].y;
                }
                colreduce(lf, false, cres);   // cres[h] = the segment's column sum of head h
            }
            bool have_o = false;
            if (ok) {
                const bool fin = mbar_wait(pvdone, (pub - 1) & 1, abort_flag, p.status);
                have_o = __all_sync(0xffffffffu, fin);
                if (!have_o) ok = false;
            }
            __nv_bfloat16 *orow0 = p.out + (static_cast<size_t>(sg.b) * p.h + head0) * D;
            if (have_o) {
                tc_fence_after();
                float o[NH];
                tmem_row(tO, o);
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    if (h >= HS) break;
                    if (whole)
                        orow0[static_cast<size_t>(h) * D + r] = __float2bfloat16_rn(cres[h] > 0.f ? o[h] / cres[h] : 0.f);
                    else
                        slot[static_cast<size_t>(h) * D + r] = o[h];
                }
                if (!whole && tid < HS) {
                    slot[kSpRows * D + tid] = msh[tid];
                    slot[kSpRows * D + kSpRows + tid] = cres[tid];
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ofree);
            asm volatile("bar.sync 1, 128;" ::: "memory");   // msh, red and cres are free for the next segment
            if (c == first_c && tid == 0) p.seg[sidx] = make_int2(first_c, last_c);   // for the merge kernel
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, kTkTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Warp-level MMAs over the balanced partition, for groups of 17 to 64 heads
// (d = 128).  At these group sizes the rows of a 128-row tcgen05 MMA are
// mostly padding (or copies), while mma.sync m16n8k16 fits the group: the
// consumer warps are those of the cluster decode kernel -- warp (mi, ti) takes
// query heads [16 mi, 16 mi + 16) as the M rows and tokens [ti TOK / WT,
// (ti + 1) TOK / WT) of every stage, S = Q K^T and O += P V with K and V read
// from the TMA-filled ring by ldmatrix, the online softmax on the fragments --
// but the work is the batch's tokens divided evenly among two CTAs per SM, as
// in the kernels above, instead of a fixed number of splits per sequence.  A
// segment's two token groups (WT = 2) merge through a small shared buffer; a
// segment cut between CTAs leaves a partial result (a slot of 64 rows) for
// the merge kernel.
constexpr int kBlTok = 64;             // tokens per stage
constexpr int kBlStages = 3;           // ring depth (two CTAs per SM)
constexpr int kBlWarps = 4;            // consumer warps
constexpr int kBlThreads = (kBlWarps + 1) * 32;
constexpr int kBlRows = 64;            // heads of a partial slot
constexpr int kBlCtasPerSm = 2;

struct BalGeom {   // d = 128, bf16
    static constexpr int D = 128;
    static constexpr uint32_t kPanelBytes = kBlTok * 128;          // 64 tokens x 64 dims
    static constexpr uint32_t kTileBytes = (D / 64) * kPanelBytes;  // K or V of a stage
    static constexpr uint32_t kStageBytes = 2 * kTileBytes;
    static constexpr uint32_t kRing = kBlStages * kStageBytes;
    static constexpr uint32_t kMrg = (2 * 16 * 64 + 2 * 2 * 16) * 4;   // 2 m-tiles: half of O (16 x 64), m, l
    static constexpr uint32_t kCtrl = 256;
    static constexpr uint32_t kTotal = kRing + kMrg + kCtrl + 1024;
    static constexpr uint32_t kPartFloats = kBlRows * D + 2 * kBlRows;
};

template <int WT>
__global__ void __launch_bounds__(kBlThreads, kBlCtasPerSm)
    gqa_decode_bal_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const SplitParams p) {
    using BG = BalGeom;
    constexpr int D = BG::D;
    constexpr int TOK = kBlTok;
    constexpr int RB = 128;                  // bytes of a token row in a panel
    constexpr int KSTEPS = D / 16;
    constexpr int NT_O = D / 8;
    constexpr int TWARP = TOK / WT;          // tokens of a stage one warp handles
    constexpr int TPW = TWARP < 32 ? TWARP : 32;   // tokens per pass (O takes 64 registers)
    constexpr int NPASS = TWARP / TPW;
    constexpr int NTS = TPW / 8;             // n-tiles of the scores of a pass
    constexpr int KKS = TPW / 16;            // k-steps of its P V
    static_assert(WT == 1 || WT == 2, "one or two token groups");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *mrg = reinterpret_cast<float *>(smem + BG::kRing);    // [2][16][64]: token group 1's O, one half
    float *mrg_ml = mrg + 2 * 16 * 64;                          // [2][2][16]: its m and l
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + BG::kRing + BG::kMrg);
    uint64_t *empty = full + kBlStages;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + kBlStages);
    long long *scan = reinterpret_cast<long long *>(empty + kBlStages + 1);   // [8]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, NC = p.nctas;
    const int HS = p.G;                      // <= 64: one slice
    const int WM = (HS + 15) >> 4;           // m-tiles (WM * WT <= 4, chosen by the host)

    if (threadIdx.x == 0) {
        for (int i = 0; i < kBlStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], WM * WT);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kBlWarps && lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    const long long T = split_batch_tokens<D, kBlThreads>(p, scan, c, NC);
    __syncthreads();   // (the barriers' initialisation is visible to every thread)
    const long long W = static_cast<long long>(p.n_kv) * T;
    const int NCe = W < NC ? static_cast<int>(W) : NC;
    const long long w_lo = c < NCe ? W * c / NCe : W, w_hi = c < NCe ? W * (c + 1) / NCe : W;
    auto n_stages = [](const SplitSeg &s) { return (s.t1 - s.t0 + TOK - 1) / TOK; };

    if (warp == kBlWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            SplitCursor cu = split_cursor_at(p, T, w_lo, w_hi);
            SplitSeg sg;
            int gi = 0;
            const int first_loaded = GQA_STALLED(p) ? 1 : 0;   // wait-test build: stage 0 never arrives
            bool ok = true;
            while (ok && cu.next(sg)) {
                const int g = sg.gs;
                const int n = n_stages(sg);
                for (int i = 0; i < n; ++i, ++gi) {
                    const int slot = gi % kBlStages, use = gi / kBlStages;
                    if (use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    if (gi < first_loaded) continue;
                    // the stage's box may run past the segment (into rows the consumers mask)
                    const int z = static_cast<int>(sg.off) + sg.t0 + i * TOK;
                    uint8_t *kd = smem + slot * BG::kStageBytes;
                    mbar_arrive_expect_tx(&full[slot], BG::kStageBytes);
#pragma unroll
                    for (int pp = 0; pp < D / 64; ++pp) {
                        tma_load_3d(kd + pp * BG::kPanelBytes, &tm_k, &full[slot], pp * 64, g, z);
                        tma_load_3d(kd + BG::kTileBytes + pp * BG::kPanelBytes, &tm_v, &full[slot], pp * 64, g, z);
                    }
                }
            }
            if (*abort_flag) {   // let the copies in flight land before the CTA exits
                for (int i = max(first_loaded, gi - kBlStages); i < gi; ++i)
                    mbar_wait_drain(&full[i % kBlStages], (i / kBlStages) & 1, p.status);
            }
        }
        __syncwarp();
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int mi = warp / WT, ti = warp % WT;
    const bool consumer = mi < WM;
    if (WT == 1 && !consumer) return;        // (WT = 2 runs with WM = 2: every warp consumes)
    const float cl2 = p.scale_log2;
    const int r0 = mi * 16 + (lane >> 2), r1 = r0 + 8;   // this lane's heads (rows of the m-tile)
    const int cq = 2 * (lane & 3);
    // ldmatrix lane roles
    const uint32_t lrow = ((lane >> 4) & 1) * 8 + (lane & 7);   // QK: token within a 16-token pair
    const uint32_t lchk = (lane >> 3) & 1;                      // QK: low/high 8 dims of a k-step
    const uint32_t frow = ((lane >> 3) & 1) * 8 + (lane & 7);   // PV: token within 16 tokens
    const uint32_t fchk = lane >> 4;                            // PV: chunk within a pair of chunks

    SplitCursor cu = split_cursor_at(p, T, w_lo, w_hi);
    SplitSeg sg;
    int gi0 = 0;
    bool ok = true;
    while (cu.next(sg)) {
        const int g = sg.gs;
        const int head0 = g * p.G;
        const int n = n_stages(sg);
        const bool split = sg.L <= kSpSplitAllBelow;   // short sequence: the weights' bf16 remainders too
        float o[NT_O][4];
        float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < NT_O; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
        if (consumer && ok) {
            // Q fragments of m-tile mi (rows = the group's heads)
            const __nv_bfloat16 *qb = p.q + (static_cast<size_t>(sg.b) * p.h + head0) * D;
            uint32_t qa[KSTEPS][4];
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
                const int cc = ks * 16 + cq;
                qa[ks][0] = r0 < HS ? *reinterpret_cast<const uint32_t *>(qb + r0 * D + cc) : 0u;
                qa[ks][1] = r1 < HS ? *reinterpret_cast<const uint32_t *>(qb + r1 * D + cc) : 0u;
                qa[ks][2] = r0 < HS ? *reinterpret_cast<const uint32_t *>(qb + r0 * D + cc + 8) : 0u;
                qa[ks][3] = r1 < HS ? *reinterpret_cast<const uint32_t *>(qb + r1 * D + cc + 8) : 0u;
            }
            // the stage loop, compiled with and without the remainder products (registers)
            auto stages = [&](auto split_tag) {
                constexpr bool SPLIT = decltype(split_tag)::value;
                for (int i = 0; i < n; ++i) {
                    const int gi = gi0 + i;
                    const int slot = gi % kBlStages, use = gi / kBlStages;
                    const bool landed = mbar_wait(&full[slot], use & 1, abort_flag, p.status);
                    if (!__all_sync(0xffffffffu, landed)) {   // warp-uniform: the mma/ldmatrix below are .aligned
                        ok = false;
                        break;
                    }
                    // valid rows of the stage: [0, row_hi); the rest belong to other CTAs or sequences
                    const int row_hi = min(TOK, sg.t1 - (sg.t0 + i * TOK));
                    const uint32_t stage = smem_u32(smem + slot * BG::kStageBytes);
    #pragma unroll
                    for (int pass = 0; pass < NPASS; ++pass) {
                        const int tw0 = ti * TWARP + pass * TPW;   // first row of this pass
                        if (row_hi <= tw0) continue;                // no valid row here
                        const bool partial = row_hi < tw0 + TPW;
                        const uint32_t kbase = stage + tw0 * RB;
                        const uint32_t vbase = kbase + BG::kTileBytes;

                        // S = Q K^T  (16 heads x TPW tokens)
                        float s[NTS][4];
    #pragma unroll
                        for (int nt = 0; nt < NTS; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    #pragma unroll
                        for (int ks = 0; ks < KSTEPS; ++ks) {
                            const uint32_t chunk = 2 * ks + lchk;
                            const uint32_t hbase = kbase + (chunk >> 3) * BG::kPanelBytes + (((chunk & 7) ^ (lane & 7)) << 4);
    #pragma unroll
                            for (int np = 0; np < NTS / 2; ++np) {
                                uint32_t b0, b1, b2, b3;
                                ldmatrix_x4(b0, b1, b2, b3, hbase + (np * 16 + lrow) * RB);
                                mma_bf16_16816(s[2 * np], qa[ks], b0, b1);
                                mma_bf16_16816(s[2 * np + 1], qa[ks], b2, b3);
                            }
                        }
                        if (partial) {
    #pragma unroll
                            for (int nt = 0; nt < NTS; ++nt)
    #pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    if (tw0 + nt * 8 + cq + (e & 1) >= row_hi) s[nt][e] = -INFINITY;
                        }
                        // online softmax over these tokens (rows r0 and r1 of the m-tile)
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
                            const float m_new = fmaxf(m_run[r], mx[r] * cl2);   // mx is finite: >= 1 valid token
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
                        uint32_t pa[KKS][4], par[KKS][4];   // the weights and, for short sequences, their remainders
                        float2 ls0 = make_float2(0.f, 0.f), ls1 = make_float2(0.f, 0.f);
    #pragma unroll
                        for (int nt = 0; nt < NTS; ++nt) {
                            const float2 y0 = ffma2_bcast(s[nt][0], s[nt][1], cl2, -m_run[0]);
                            const float2 y1 = ffma2_bcast(s[nt][2], s[nt][3], cl2, -m_run[1]);
                            float e0 = exp2f(y0.x), e1 = exp2f(y0.y), e2 = exp2f(y1.x), e3 = exp2f(y1.y);
                            if (partial) {   // masked tokens add nothing (also when the scale is 0)
                                const int row = tw0 + nt * 8 + cq;
                                if (row >= row_hi) e0 = e2 = 0.f;
                                if (row + 1 >= row_hi) e1 = e3 = 0.f;
                            }
                            const uint32_t lo = pack_bf16x2(e0, e1), hi = pack_bf16x2(e2, e3);
                            const float2 ul = unpack_bf16x2(lo), uh = unpack_bf16x2(hi);
                            ls0 = fadd2(ls0, ul);
                            ls1 = fadd2(ls1, uh);
                            if constexpr (SPLIT) {   // remainders (exact in fp32), rounded to bf16 for a second product
                                const uint32_t rl = pack_bf16x2(e0 - ul.x, e1 - ul.y);
                                const uint32_t rh = pack_bf16x2(e2 - uh.x, e3 - uh.y);
                                ls0 = fadd2(ls0, unpack_bf16x2(rl));
                                ls1 = fadd2(ls1, unpack_bf16x2(rh));
                                par[nt >> 1][(nt & 1) * 2 + 0] = rl;
                                par[nt >> 1][(nt & 1) * 2 + 1] = rh;
                            }
                            pa[nt >> 1][(nt & 1) * 2 + 0] = lo;
                            pa[nt >> 1][(nt & 1) * 2 + 1] = hi;
                        }
                        l_run[0] += ls0.x + ls0.y;
                        l_run[1] += ls1.x + ls1.y;
                        // O += P V.  On a partial pass the V values of invalid rows are zeroed in
                        // registers (each half of a transposed fragment register is one token), so
                        // that 0 * (whatever those rows hold) adds nothing.
                        auto pv = [&](auto masked) {
                            constexpr bool MASKED = decltype(masked)::value;
    #pragma unroll
                            for (int kk = 0; kk < KKS; ++kk) {
                                uint32_t mlo = 0xFFFFFFFFu, mhi = 0xFFFFFFFFu;
                                if constexpr (MASKED) {
                                    const int row = tw0 + kk * 16 + cq;   // this lane's tokens: row, row + 1 (and + 8)
                                    mlo = (row < row_hi ? 0x0000FFFFu : 0u) | (row + 1 < row_hi ? 0xFFFF0000u : 0u);
                                    mhi = (row + 8 < row_hi ? 0x0000FFFFu : 0u) | (row + 9 < row_hi ? 0xFFFF0000u : 0u);
                                }
                                const uint32_t rowaddr = vbase + (kk * 16 + frow) * RB;
    #pragma unroll
                                for (int dp = 0; dp < NT_O / 2; ++dp) {
                                    const uint32_t chunk = 2 * dp + fchk;
                                    uint32_t b0, b1, b2, b3;
                                    ldmatrix_x4_trans(b0, b1, b2, b3,
                                                      rowaddr + (chunk >> 3) * BG::kPanelBytes +
                                                          (((chunk & 7) ^ (lane & 7)) << 4));
                                    if constexpr (MASKED) {
                                        b0 &= mlo;
                                        b1 &= mhi;
                                        b2 &= mlo;
                                        b3 &= mhi;
                                    }
                                    mma_bf16_16816(o[2 * dp], pa[kk], b0, b1);
                                    mma_bf16_16816(o[2 * dp + 1], pa[kk], b2, b3);
                                    if constexpr (SPLIT) {
                                        mma_bf16_16816(o[2 * dp], par[kk], b0, b1);
                                        mma_bf16_16816(o[2 * dp + 1], par[kk], b2, b3);
                                    }
                                }
                            }
                        };
                        if (partial)
                            pv(std::true_type{});
                        else
                            pv(std::false_type{});
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[slot]);
                }
            };
            if (split)
                stages(std::true_type{});
            else
                stages(std::false_type{});
        }
        gi0 += n;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
            l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
        }

        // ---- the segment's result: token group 1 hands its partial to group 0 through
        // shared memory (half of O at a time), which merges and writes
        if constexpr (WT == 2) {
            const int lr0 = lane >> 2, lr1 = lr0 + 8;   // rows within the m-tile
            float a_me[2] = {1.f, 1.f}, a_ot[2] = {0.f, 0.f};
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                if (ti == 1) {
#pragma unroll
                    for (int nt = 0; nt < NT_O / 2; ++nt) {
                        const int col = nt * 8 + cq;
                        float *m0 = mrg + (mi * 16 + lr0) * 64 + col, *m1 = mrg + (mi * 16 + lr1) * 64 + col;
                        *reinterpret_cast<float2 *>(m0) = make_float2(o[half * 8 + nt][0], o[half * 8 + nt][1]);
                        *reinterpret_cast<float2 *>(m1) = make_float2(o[half * 8 + nt][2], o[half * 8 + nt][3]);
                    }
                    if (half == 0 && (lane & 3) == 0) {
                        mrg_ml[(mi * 2 + 0) * 16 + lr0] = m_run[0];
                        mrg_ml[(mi * 2 + 0) * 16 + lr1] = m_run[1];
                        mrg_ml[(mi * 2 + 1) * 16 + lr0] = l_run[0];
                        mrg_ml[(mi * 2 + 1) * 16 + lr1] = l_run[1];
                    }
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (ti == 0) {
                    if (half == 0) {
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            const int lr = r ? lr1 : lr0;
                            const float mo = mrg_ml[(mi * 2 + 0) * 16 + lr], lo = mrg_ml[(mi * 2 + 1) * 16 + lr];
                            const float M = fmaxf(m_run[r], mo);
                            a_me[r] = M == -INFINITY ? 0.f : exp2f(m_run[r] - M);
                            a_ot[r] = M == -INFINITY ? 0.f : exp2f(mo - M);
                            l_run[r] = l_run[r] * a_me[r] + lo * a_ot[r];
                            m_run[r] = M;
                        }
                    }
#pragma unroll
                    for (int nt = 0; nt < NT_O / 2; ++nt) {
                        const int col = nt * 8 + cq;
                        const float2 x0 = *reinterpret_cast<const float2 *>(mrg + (mi * 16 + lr0) * 64 + col);
                        const float2 x1 = *reinterpret_cast<const float2 *>(mrg + (mi * 16 + lr1) * 64 + col);
                        float *oo = o[half * 8 + nt];
                        oo[0] = oo[0] * a_me[0] + x0.x * a_ot[0];
                        oo[1] = oo[1] * a_me[0] + x0.y * a_ot[0];
                        oo[2] = oo[2] * a_me[1] + x1.x * a_ot[1];
                        oo[3] = oo[3] * a_me[1] + x1.y * a_ot[1];
                    }
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");   // the buffer is free again
            }
        }
        const int first_c = split_owner(sg.w, W, NCe), last_c = split_owner(sg.w + sg.L - 1, W, NCe);
        const int sidx = g * p.B + sg.b;
        if (ti == 0 && consumer && ok) {
            if (first_c == last_c) {   // the whole sequence: O / l
                __nv_bfloat16 *ob = p.out + (static_cast<size_t>(sg.b) * p.h + head0) * D;
                const float inv0 = 1.f / l_run[0], inv1 = 1.f / l_run[1];
#pragma unroll
                for (int nt = 0; nt < NT_O; ++nt) {
                    if (r0 < HS)
                        *reinterpret_cast<uint32_t *>(ob + r0 * D + nt * 8 + cq) =
                            pack_bf16x2(o[nt][0] * inv0, o[nt][1] * inv0);
                    if (r1 < HS)
                        *reinterpret_cast<uint32_t *>(ob + r1 * D + nt * 8 + cq) =
                            pack_bf16x2(o[nt][2] * inv1, o[nt][3] * inv1);
                }
            } else {                   // a piece: unnormalised O, m, l into slot c + sidx
                float *slot = p.part + static_cast<size_t>(c + sidx) * BG::kPartFloats;
#pragma unroll
                for (int nt = 0; nt < NT_O; ++nt) {
                    if (r0 < HS) *reinterpret_cast<float2 *>(slot + r0 * D + nt * 8 + cq) = make_float2(o[nt][0], o[nt][1]);
                    if (r1 < HS) *reinterpret_cast<float2 *>(slot + r1 * D + nt * 8 + cq) = make_float2(o[nt][2], o[nt][3]);
                }
                if ((lane & 3) == 0) {
                    if (r0 < HS) {
                        slot[kBlRows * D + r0] = m_run[0];
                        slot[kBlRows * D + kBlRows + r0] = l_run[0];
                    }
                    if (r1 < HS) {
                        slot[kBlRows * D + r1] = m_run[1];
                        slot[kBlRows * D + kBlRows + r1] = l_run[1];
                    }
                }
            }
        }
        // the segment's record for the merge kernel, from the CTA of its first piece
        if (c == first_c && threadIdx.x == 0) p.seg[sidx] = make_int2(first_c, last_c);
    }
}

// ---------------------------------------------------------------------------
// The merge of the pieces of the segments that were cut between CTAs, in a
// second launch so that it runs on every SM at once: one block per (segment,
// head), four warps each folding a quarter of the pieces with the log-sum-exp
// rule (running max M, sum L, unnormalised O), then warp 0 folds the four.

template <int D, int ROWS>   // ROWS: heads of a partial slot (O [ROWS][D], then m [ROWS], l [ROWS])
__global__ void __launch_bounds__(128)
    gqa_decode_split_merge_kernel(const float *part, const int2 *seg, __nv_bfloat16 *out, int B, int h, int G,
                                  int slices, int rows) {
    constexpr uint32_t SLOT = ROWS * D + 2 * ROWS;
    __shared__ float sM[4], sL[4];
    __shared__ float4 sO[4][D / 4];
    const int sidx = blockIdx.x, hh = blockIdx.y;
    const int gs = sidx / B, b = sidx % B;
    const int g = gs / slices, sl = gs % slices;
    const int HS = min(G - sl * rows, rows);
    if (hh >= HS) return;
    const int2 info = seg[sidx];
    if (info.x < 0 || info.x == info.y) return;   // an empty sequence, or finished by one CTA
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool act = lane < D / 4;
    float M = -INFINITY, L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int cc = info.x + warp; cc <= info.y; cc += 4) {
        const float *sp = part + static_cast<size_t>(cc + sidx) * SLOT;
        const float m = __ldcg(sp + ROWS * D + hh);
        const float l = __ldcg(sp + ROWS * D + ROWS + hh);
        const float4 o = act ? __ldcg(reinterpret_cast<const float4 *>(sp + static_cast<size_t>(hh) * D) + lane)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        const float M2 = fmaxf(M, m);
        const float a = M2 == -INFINITY ? 0.f : exp2f(M - M2), w = M2 == -INFINITY ? 0.f : exp2f(m - M2);
        L = L * a + l * w;
        acc = make_float4(acc.x * a + o.x * w, acc.y * a + o.y * w, acc.z * a + o.z * w, acc.w * a + o.w * w);
        M = M2;
    }
    if (lane == 0) {
        sM[warp] = M;
        sL[warp] = L;
    }
    if (act) sO[warp][lane] = acc;
    __syncthreads();
    if (warp != 0 || !act) return;
    float Mf = fmaxf(fmaxf(sM[0], sM[1]), fmaxf(sM[2], sM[3]));
    float Lf = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int w = 0; w < 4; ++w) {
        const float wt = sM[w] == -INFINITY ? 0.f : exp2f(sM[w] - Mf);
        Lf += wt * sL[w];
        const float4 x = sO[w][lane];
        o = make_float4(o.x + wt * x.x, o.y + wt * x.y, o.z + wt * x.z, o.w + wt * x.w);
    }
    const float inv = Lf > 0.f ? 1.f / Lf : 0.f;
    __nv_bfloat16 *orow = out + (static_cast<size_t>(b) * h + g * G + sl * rows + hh) * D;
    *reinterpret_cast<uint2 *>(orow + 4 * lane) =
        make_uint2(pack_bf16x2(o.x * inv, o.y * inv), pack_bf16x2(o.z * inv, o.w * inv));
}

// ---------------------------------------------------------------------------
// host side

// The merge launch: one block per (segment, head)
template <int D, int ROWS>
static int launch_merge(const SplitParams &prm, int n_segments, int heads, cudaStream_t stream) {
    gqa_decode_split_merge_kernel<D, ROWS><<<dim3(static_cast<unsigned>(n_segments), static_cast<unsigned>(heads)), 128,
                                             0, stream>>>(prm.part, prm.seg, prm.out, prm.B, prm.h, prm.G, prm.slices,
                                                          ROWS);
    return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

// bytes of the per-segment records at the start of the workspace (a multiple of 256)
static size_t seg_bytes_for(int B, int n_kv, int slices) {
    const size_t ns = static_cast<size_t>(n_kv) * slices * B;
    return (ns * sizeof(int2) + 255) & ~static_cast<size_t>(255);
}

template <int D>
static size_t split_workspace_bytes_t(int B, int n_kv, int slices, int nctas) {
    const size_t ns = static_cast<size_t>(n_kv) * slices * B;
    return seg_bytes_for(B, n_kv, slices) +
           (static_cast<size_t>(nctas) + ns) * SplitGeom<D>::kPartFloats * sizeof(float);
}


// The kernel gqa_decode_split runs for a shape (by group size, as measured): warp-level
// MMAs over the balanced partition for 17 to 64 heads at d = 128, tokens as rows up to
// 16, heads as rows otherwise.
enum class SplitPath { kTok, kHeads, kBal };
static SplitPath split_path(int h, int n_kv, int d) {
    const int G = h / n_kv;
    if (d == 128 && G > 16 && G <= kBlRows) return SplitPath::kBal;
    if (d == 128 && G <= 16) return SplitPath::kTok;
    return SplitPath::kHeads;
}

static size_t bal_workspace_bytes(int B, int n_kv, int nctas) {
    return seg_bytes_for(B, n_kv, 1) +
           (static_cast<size_t>(nctas) + static_cast<size_t>(n_kv) * B) * BalGeom::kPartFloats * sizeof(float);
}

size_t split_workspace_bytes(int B, int h, int n_kv, int d) {
    const int G = h / n_kv;
    const int slices = (G + kSpRows - 1) / kSpRows;
    const int sms = gqa_host::sm_count();
    if (split_path(h, n_kv, d) == SplitPath::kBal) return bal_workspace_bytes(B, n_kv, kBlCtasPerSm * sms);
    return d == 128 ? split_workspace_bytes_t<128>(B, n_kv, slices, sms)
                    : split_workspace_bytes_t<64>(B, n_kv, slices, sms);
}

template <int D, int GP>
static int launch_split_t(const void *q, const void *k, const void *v, long long cache_rows, const int32_t *seqlens,
                          void *out, int B, int h, int n_kv, float scale, void *workspace, size_t ws_bytes,
                          cudaStream_t stream) {
    using SG = SplitGeom<D>;
    auto kern = gqa_decode_split_kernel<D, GP>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 3;
    static std::atomic<unsigned long long> attr_done{0};
    if (!gqa_host::once_per_device(attr_done, dev, [&] {
            return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SG::kTotal) == cudaSuccess;
        }))
        return 3;
    const int G = h / n_kv;
    const int slices = (G + kSpRows - 1) / kSpRows;
    if (GP < kSpRows && G > GP) return 2;   // (the dispatcher never asks for this)
    const int nctas = gqa_host::sm_count();
    if (static_cast<long long>(n_kv) * slices * B > (1LL << 24)) return 2;   // segment indices stay int
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        ws_bytes < split_workspace_bytes_t<D>(B, n_kv, slices, nctas))
        return 1;
    CUtensorMap tk, tv;
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
    prm.seg = static_cast<int2 *>(workspace);
    prm.part = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + seg_bytes_for(B, n_kv, slices));
    prm.B = B;
    prm.h = h;
    prm.n_kv = n_kv;
    prm.G = G;
    prm.slices = slices;
    prm.nctas = nctas;
    prm.q_bytes = 0;   // (Q goes to TMEM through registers)
    prm.cache_rows = cache_rows;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.status = gqa_host::device_status();
    if (!prm.status) return 3;
    GQA_SET_TEST_STALL(prm);
    kern<<<nctas, kSpThreads, SG::kTotal, stream>>>(tk, tv, prm);
    if (cudaGetLastError() != cudaSuccess) return 3;
    return launch_merge<D, kSpRows>(prm, n_kv * slices * B, std::min(G, kSpRows), stream);
}

// The tokens-as-rows kernel (d = 128, groups of at most 64 heads); the workspace
// layout and size are those of the heads-as-rows kernel at d = 128.
template <int NH>
static int launch_split_tok(const void *q, const void *k, const void *v, long long cache_rows,
                            const int32_t *seqlens, void *out, int B, int h, int n_kv, float scale, void *workspace,
                            size_t ws_bytes, cudaStream_t stream) {
    using TG = TokGeom;
    auto kern = gqa_decode_split_tok_kernel<NH>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 3;
    static std::atomic<unsigned long long> attr_done{0};
    if (!gqa_host::once_per_device(attr_done, dev, [&] {
            return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TG::kTotal) == cudaSuccess;
        }))
        return 3;
    const int G = h / n_kv;
    const int nctas = gqa_host::sm_count();
    if (static_cast<long long>(n_kv) * B > (1LL << 24)) return 2;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        ws_bytes < split_workspace_bytes_t<128>(B, n_kv, 1, nctas))
        return 1;
    CUtensorMap tq, tk, tv;
    {
        const uint64_t dims[3] = {128, static_cast<uint64_t>(h), static_cast<uint64_t>(B)};
        const uint64_t strides[2] = {128 * 2, static_cast<uint64_t>(h) * 128 * 2};
        const uint32_t box[3] = {64, static_cast<uint32_t>(std::min(NH, h)), 1};
        if (!gqa_host::encode_tensor_map(&tq, q, 3, dims, strides, box)) return 3;
    }
    {
        const uint64_t dims[3] = {128, static_cast<uint64_t>(n_kv), static_cast<uint64_t>(std::max(cache_rows, 1LL))};
        const uint64_t strides[2] = {128 * 2, static_cast<uint64_t>(n_kv) * 128 * 2};
        const uint32_t box[3] = {64, 1, static_cast<uint32_t>(kTkTok)};
        if (!gqa_host::encode_tensor_map(&tk, k, 3, dims, strides, box)) return 3;
        if (!gqa_host::encode_tensor_map(&tv, v, 3, dims, strides, box)) return 3;
    }
    SplitParams prm = {};
    prm.q = static_cast<const __nv_bfloat16 *>(q);
    prm.seqlens = seqlens;
    prm.out = static_cast<__nv_bfloat16 *>(out);
    prm.seg = static_cast<int2 *>(workspace);
    prm.part = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + seg_bytes_for(B, n_kv, 1));
    prm.B = B;
    prm.h = h;
    prm.n_kv = n_kv;
    prm.G = G;
    prm.slices = 1;
    prm.nctas = nctas;
    prm.q_bytes = static_cast<uint32_t>(128 * 2 * std::min(NH, h));
    prm.cache_rows = cache_rows;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.status = gqa_host::device_status();
    if (!prm.status) return 3;
    GQA_SET_TEST_STALL(prm);
    kern<<<nctas, kSpThreads, TG::kTotal, stream>>>(tq, tk, tv, prm);
    if (cudaGetLastError() != cudaSuccess) return 3;
    return launch_merge<128, kSpRows>(prm, n_kv * B, G, stream);
}

template <int WT>
static int launch_split_bal(const void *q, const void *k, const void *v, long long cache_rows, const int32_t *seqlens,
                            void *out, int B, int h, int n_kv, float scale, void *workspace, size_t ws_bytes,
                            cudaStream_t stream) {
    using BG = BalGeom;
    auto kern = gqa_decode_bal_kernel<WT>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 3;
    static std::atomic<unsigned long long> attr_done{0};
    if (!gqa_host::once_per_device(attr_done, dev, [&] {
            return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, BG::kTotal) == cudaSuccess;
        }))
        return 3;
    const int G = h / n_kv;
    const int WM = (G + 15) / 16;
    if (G > kBlRows || WM * WT > kBlWarps || (WT == 2 && WM != 2)) return 2;   // (the dispatcher never asks)
    const int nctas = kBlCtasPerSm * gqa_host::sm_count();
    if (static_cast<long long>(n_kv) * B > (1LL << 24)) return 2;   // segment indices stay int
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < bal_workspace_bytes(B, n_kv, nctas))
        return 1;
    CUtensorMap tk, tv;
    {
        const uint64_t dims[3] = {static_cast<uint64_t>(BG::D), static_cast<uint64_t>(n_kv),
                                  static_cast<uint64_t>(std::max(cache_rows, 1LL))};
        const uint64_t strides[2] = {static_cast<uint64_t>(BG::D) * 2, static_cast<uint64_t>(n_kv) * BG::D * 2};
        const uint32_t box[3] = {64, 1, static_cast<uint32_t>(kBlTok)};
        if (!gqa_host::encode_tensor_map(&tk, k, 3, dims, strides, box)) return 3;
        if (!gqa_host::encode_tensor_map(&tv, v, 3, dims, strides, box)) return 3;
    }
    SplitParams prm = {};
    prm.q = static_cast<const __nv_bfloat16 *>(q);
    prm.seqlens = seqlens;
    prm.out = static_cast<__nv_bfloat16 *>(out);
    prm.seg = static_cast<int2 *>(workspace);
    prm.part = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + seg_bytes_for(B, n_kv, 1));
    prm.B = B;
    prm.h = h;
    prm.n_kv = n_kv;
    prm.G = G;
    prm.slices = 1;
    prm.nctas = nctas;
    prm.q_bytes = 0;
    prm.cache_rows = cache_rows;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.status = gqa_host::device_status();
    if (!prm.status) return 3;
    GQA_SET_TEST_STALL(prm);
    kern<<<nctas, kBlThreads, BG::kTotal, stream>>>(tk, tv, prm);
    if (cudaGetLastError() != cudaSuccess) return 3;
    return launch_merge<BG::D, kBlRows>(prm, n_kv * B, G, stream);
}

int launch_decode_split(const void *q, const void *k, const void *v, long long cache_rows, const int32_t *seqlens,
                        void *out, int B, int h, int n_kv, int d, float scale, void *workspace, size_t ws_bytes,
                        cudaStream_t stream) {
    const int G = h / n_kv;
    const SplitPath path = split_path(h, n_kv, d);
    if (path == SplitPath::kBal) {
        if (G <= 32)
            return launch_split_bal<2>(q, k, v, cache_rows, seqlens, out, B, h, n_kv, scale, workspace, ws_bytes,
                                       stream);
        return launch_split_bal<1>(q, k, v, cache_rows, seqlens, out, B, h, n_kv, scale, workspace, ws_bytes, stream);
    }
    if (path == SplitPath::kTok)
        return launch_split_tok<16>(q, k, v, cache_rows, seqlens, out, B, h, n_kv, scale, workspace, ws_bytes, stream);
    if (d == 128)
        return launch_split_t<128, 128>(q, k, v, cache_rows, seqlens, out, B, h, n_kv, scale, workspace, ws_bytes,
                                        stream);
    if (G <= 32)
        return launch_split_t<64, 32>(q, k, v, cache_rows, seqlens, out, B, h, n_kv, scale, workspace, ws_bytes, stream);
    if (G <= 64)
        return launch_split_t<64, 64>(q, k, v, cache_rows, seqlens, out, B, h, n_kv, scale, workspace, ws_bytes, stream);
    return launch_split_t<64, 128>(q, k, v, cache_rows, seqlens, out, B, h, n_kv, scale, workspace, ws_bytes, stream);
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
    return launch_decode_split(q, k, v, cache_rows, seqlens, out, B, h, n_kv, d, scale, scratch, need, stream);
}

}  // namespace gqa
