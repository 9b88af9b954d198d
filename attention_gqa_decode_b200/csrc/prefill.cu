// Prefill: exact (optionally causal) grouped-query attention over all query
// rows, on the 5th-generation tensor cores.
//
// Semantics: "Evolution of AI Attention Mechanisms" (toolsku), "MHA
// Implementation" / "GQA Implementation" (scores Q K^T * scale, -inf where
// masked, row softmax, times V; query head i reads KV head i / (h / n_kv));
// "Flash Attention Principle" box (split Q, K, V into blocks, softmax on chip,
// write only O); "Attention variants" (saadho), "What this topic covers"
// (exact result, the n x n score matrix never reaches device memory; online
// softmax with a running max and running sum).
//
// Design (B200): one CTA owns one (batch, query head) and a pair of 128-row
// query tiles; it walks the 128-key tiles of the head's KV group.
//   warp 8      TMA producer: both Q tiles once, then K(j), V(j) alternately
//               into a 5-slot ring of 128-byte-swizzled shared-memory tiles;
//   warp 9      allocates 512 TMEM columns and, from one thread, issues
//               tcgen05.mma: S_t = Q_t K^T (M=128, N=128, both K-major) into
//               TMEM, and O_t += P_t V (A = P_t read from TMEM, B = V
//               MN-major from shared memory), committing to mbarriers;
//   warps 0-7   two softmax warpgroups, one per query tile (thread = query
//               row = TMEM lane), holding 208 registers each (setmaxnreg;
//               warps 8-11 give theirs up): load the whole S row from TMEM
//               once, mask (causal diagonal and ragged tail), running max
//               with lazy rescaling of O in TMEM (only when the max grows by
//               more than 2^8), exp2 with the scale folded in, P as packed
//               bf16 written back over S, then the epilogue O / l -> bf16.
// The two query tiles ping-pong: while one warpgroup computes its softmax,
// the tensor cores run the other tile's P V and next Q K^T.  Causal CTAs are
// ordered heaviest first; tiles wholly above the diagonal are never loaded.
//
// Chunked prefill over a paged cache (PAGED): sequence b holds past_lens[b]
// tokens in cache pages ("Multi-Query Attention (MQA)" (inferensys glossary),
// "PagedAttention") and the call adds a chunk of S_q tokens whose K/V are
// concatenated after them ("MHA Implementation", past_kv), so query row r
// sees keys at positions <= past + r.  The key tiles are the past tiles,
// loaded from the pages with one TMA box per page piece (page ids read one
// tile ahead by the producer warp), then the chunk's tiles, loaded from the
// new K/V directly.  The last past tile ends at position `past`: its columns
// beyond are masked in the softmax, and its V rows beyond are zeroed in
// shared memory by the MMA warp before the P V that reads them (whatever the
// cache holds there, 0 * NaN must not reach O).  The append itself is done by
// the two idle warps: the CTA of the first query head of a KV group copies
// the new K/V rows of its own two query tiles into the pages, while the other
// warps attend.  The attention never reads a slot that is being written:
// past tiles only cover positions < past.
//
// Rows that see few keys (a query tile whose first row sees at most
// kPfSplitKeys keys) do not average out the bf16 rounding of their softmax
// weights; for them the weights' bf16 remainders p - bf16(p) are written over
// the upper half of S as well and multiplied by V in a second product, so the
// weights are carried to about 16 bits.  That path is a separate
// instantiation (SPLIT), launched only for the query-tile pairs that need it,
// so the common path is compiled without it.
#include <algorithm>
#include <type_traits>

#include "common.cuh"

namespace gqa {

constexpr int kPfRows = 128;     // query rows per tile (MMA M)
constexpr int kPfKeys = 128;     // keys per KV tile
constexpr int kPfRing = 5;       // K/V tiles in flight
constexpr int kPfThreads = 384;  // softmax warpgroups 0 and 1; warpgroup 2 = producer, MMA, 2 idle warps
// Register split (setmaxnreg): the launch gives 168 per thread (384 x 168 =
// 64512); warpgroup 2 drops to 80 and the softmax warpgroups rise to 208:
// 256 x 208 + 128 x 80 = 63488 <= 64512.  (Both regions then compile without
// spills: 216/64 spilled in the MMA issuer, 200/96 in the softmax.)
constexpr uint32_t kRegsSoftmax = 208, kRegsOther = 80;
static_assert(256 * kRegsSoftmax + 128 * kRegsOther <= kPfThreads * 168, "register split exceeds the launch");
constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr int kPfSplitKeys = 256;            // first-row keys up to which a query tile splits its weights

struct PrefillParams {
    __nv_bfloat16 *out;
    int B, S_q, S_kv, h, n_kv, G, causal;
    int pair_lo, pair_hi;          // the query-tile pairs of this launch: [pair_lo, pair_hi)
    float scale_log2;
    int *status;                   // the library's device status word
    // chunked prefill over a paged cache
    const int32_t *block_table, *past_lens;
    const __nv_bfloat16 *k_new, *v_new;
    __nv_bfloat16 *k_pages, *v_pages;
    int max_blocks, page_size, num_pages;
    GQA_TEST_STALL_FIELD
};

template <int D>
struct PrefillSmem {
    static constexpr uint32_t kTile = kPfRows * D * 2;   // one Q, K or V tile
    static constexpr uint32_t kHalf = kPfRows * 128;     // one 64-dim half of a tile
    static constexpr uint32_t kQ = 2 * kTile;
    static constexpr uint32_t kRing = kPfRing * kTile;
    static constexpr uint32_t kCtrl = 256;
    static constexpr uint32_t kTotal = kQ + kRing + kCtrl + 1024;
};

__device__ __forceinline__ int kv_tiles_for(int rows_begin, int S_q, int S_kv, int causal) {
    if (rows_begin >= S_q) return 0;
    const int r_last = min(rows_begin + kPfRows - 1, S_q - 1);
    const int limit = causal ? min(S_kv - 1, r_last + (S_kv - S_q)) : S_kv - 1;
    return limit / kPfKeys + 1;
}

// Key tiles a paged-chunk query tile starting at row rows_begin walks: all
// past tiles, then the chunk's tiles up to its last row (causal).
__device__ __forceinline__ int chunk_tiles_for(int rows_begin, int S_q, int n_past) {
    if (rows_begin >= S_q) return 0;
    return n_past + min(rows_begin + kPfRows - 1, S_q - 1) / kPfKeys + 1;
}

// The keys the first row of the query tile at row0 sees (the fewest of the tile's rows).
__host__ __device__ __forceinline__ int first_row_keys(bool paged, int causal, int S_q, int S_kv, int row0,
                                                       int past) {
    return paged ? past + row0 + 1 : causal ? min(S_kv, row0 + (S_kv - S_q) + 1) : S_kv;
}

// The second P V product of a split tile (A = the weights' bf16 remainders in
// TMEM, B = V): out of line, so the 80-register MMA issuer keeps its registers.
__device__ __noinline__ void pf_issue_pv_rem(uint32_t d_tmem, uint32_t a_tmem, uint32_t b0, uint32_t lbo,
                                             uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < kPfKeys / 16; ++kk)
        umma_ts(d_tmem, a_tmem + kk * 8, sdesc_sw128(b0 + kk * 16 * 128, lbo, 1024), idesc, 1u);
}

template <int D, bool PAGED, bool SPLIT>
__global__ void __launch_bounds__(kPfThreads, 1)
    gqa_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kp,
                       const __grid_constant__ CUtensorMap tm_vp, const PrefillParams p) {
    using SM = PrefillSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sRing = smem + SM::kQ;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kQ + SM::kRing);
    uint64_t *qfull = bars;
    uint64_t *full = bars + 1;                 // [kPfRing]
    uint64_t *empty = full + kPfRing;          // [kPfRing]
    uint64_t *sfull = empty + kPfRing;         // [2] S_t ready
    uint64_t *pfull = sfull + 2;               // [2] P_t written
    uint64_t *odone = pfull + 2;               // [2] last P V of tile t done
    uint64_t *drain = odone + 2;               // MMA drain on the give-up path
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    // the short-row pairs' launch (SPLIT, queued behind this one) may start on SMs this
    // launch's last wave leaves idle: the two write disjoint rows
    if constexpr (!SPLIT && !PAGED) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // work unit: heaviest causal query-tile pairs first; consecutive CTAs share a KV group
    const int BH = p.B * p.h;
    const int bh = blockIdx.x % BH;
    const int pr = blockIdx.x / BH;
    const int pair = p.causal ? (p.pair_hi - 1 - pr) : (p.pair_lo + pr);
    const int b = bh / p.h, head = bh % p.h, kvh = head / p.G;
    const int q0 = pair * 2 * kPfRows;
    // paged chunk: past tokens of this sequence (cut to what the block table can hold)
    int past = 0;
    if constexpr (PAGED) {
        past = max(p.past_lens[b], 0);
        const int cap = p.max_blocks * p.page_size - p.S_q;
        if (past > cap) {
            if (threadIdx.x == 0) record_status(p.status, kStatusInvalid);
            past = max(cap, 0);
        }
    }
    const int n_past = (past + kPfKeys - 1) / kPfKeys;
    const int n_t0 = PAGED ? chunk_tiles_for(q0, p.S_q, n_past) : kv_tiles_for(q0, p.S_q, p.S_kv, p.causal);
    const int n_t1 = PAGED ? chunk_tiles_for(q0 + kPfRows, p.S_q, n_past)
                           : kv_tiles_for(q0 + kPfRows, p.S_q, p.S_kv, p.causal);
    const int nmax = max(n_t0, n_t1);

    if (threadIdx.x == 0) {
        mbar_init(qfull, 1);
        for (int i = 0; i < kPfRing; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&sfull[t], 1);
            mbar_init(&pfull[t], kPfRows);
            mbar_init(&odone[t], 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 8) {
        regs_dec<kRegsOther>();   // warpgroup 2: producer, MMA issuer, two idle warps
        if (warp == 8) {
            // ------------------------------------------------------------ producer
            // (the whole warp runs the loop; lane 0 waits and issues, lanes hold page ids)
            if (lane == 0) {
                tma_prefetch_desc(&tm_q);
                tma_prefetch_desc(&tm_k);
                tma_prefetch_desc(&tm_v);
                if (PAGED) {
                    tma_prefetch_desc(&tm_kp);
                    tma_prefetch_desc(&tm_vp);
                }
                mbar_arrive_expect_tx(qfull, SM::kQ);
                for (int t = 0; t < 2; ++t)
                    for (int hf = 0; hf < D / 64; ++hf)
                        tma_load_4d(sQ + t * SM::kTile + hf * SM::kHalf, &tm_q, qfull, hf * 64, head, q0 + t * kPfRows, b);
            }
            const int pb = PAGED ? min(p.page_size, kPfKeys) : kPfKeys;   // rows per page box
            const int pieces = kPfKeys / pb;                               // boxes per past tile
            // piece n = j * pieces + k covers past rows [n pb, n pb + pb); lane l holds the
            // page id of piece 32 * batch + l, the next batch loaded a batch ahead
            auto batch_of = [&](int batch) -> int {
                int page = 0;
                const int pos = (batch * 32 + lane) * pb;
                if (PAGED && pos < past) {
                    page = p.block_table[static_cast<size_t>(b) * p.max_blocks + pos / p.page_size];
                    if (page < 0 || page >= p.num_pages) {   // read as zeros, reported
                        record_status(p.status, kStatusInvalid);
                        page = p.num_pages;
                    }
                }
                return page;
            };
            int cur_batch = 0;
            int ids = PAGED ? batch_of(0) : 0;
            int ids_next = (PAGED && n_past * pieces > 32) ? batch_of(1) : 0;
            int item = 0;
            bool stop = false;
            const int first_loaded = GQA_STALLED(p) ? 1 : 0;   // wait-test build: K tile 0 never arrives
            for (int j = 0; j < nmax && !stop; ++j) {
                for (int kv = 0; kv < 2; ++kv, ++item) {
                    const int slot = item % kPfRing, use = item / kPfRing;
                    int ok = 1;
                    if (lane == 0 && use > 0) ok = mbar_wait(&empty[slot], (use - 1) & 1, abort_flag, p.status);
                    if (!__shfl_sync(0xffffffffu, ok, 0)) {
                        stop = true;
                        break;
                    }
                    if (item < first_loaded) continue;
                    uint8_t *dst = sRing + slot * SM::kTile;
                    if (PAGED && j < n_past) {
                        // rows [0, valid) of this tile are cached tokens: one box per page piece
                        const int valid = min(kPfKeys, past - j * kPfKeys);
                        const int nb = (valid + pb - 1) / pb;
                        const CUtensorMap *map = kv ? &tm_vp : &tm_kp;
                        if (lane == 0) mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(nb * pb * 128 * (D / 64)));
                        for (int k = 0; k < nb; ++k) {
                            const int n = j * pieces + k;
                            if (n / 32 != cur_batch) {   // warp-uniform
                                cur_batch = n / 32;
                                ids = ids_next;
                                if ((cur_batch + 1) * 32 < n_past * pieces) ids_next = batch_of(cur_batch + 1);
                            }
                            const int page = __shfl_sync(0xffffffffu, ids, n % 32);
                            if (lane == 0) {
                                const int slot_in_page = (j * kPfKeys + k * pb) % p.page_size;
                                for (int hf = 0; hf < D / 64; ++hf)
                                    tma_load_4d(dst + hf * SM::kHalf + k * pb * 128, map, &full[slot], hf * 64, kvh,
                                                slot_in_page, page);
                            }
                        }
                    } else if (lane == 0) {
                        // the chunk's own K/V (PAGED), or the K/V tensors
                        mbar_arrive_expect_tx(&full[slot], SM::kTile);
                        const CUtensorMap *map = kv ? &tm_v : &tm_k;
                        for (int hf = 0; hf < D / 64; ++hf)
                            tma_load_4d(dst + hf * SM::kHalf, map, &full[slot], hf * 64, kvh, (j - n_past) * kPfKeys, b);
                    }
                }
            }
            if (lane == 0 && *abort_flag) {   // let the copies in flight land before TMEM and smem go away
                mbar_wait_drain(qfull, 0, p.status);
                for (int i = max(first_loaded, item - kPfRing); i < item; ++i)
                    mbar_wait_drain(&full[i % kPfRing], (i / kPfRing) & 1, p.status);
            }
            __syncwarp();
        } else if (warp == 9) {
            // ------------------------------------------------------------ MMA issuer
            if (lane == 0) {
                constexpr uint32_t idesc_qk = idesc_bf16_f32(kPfRows, kPfKeys, false, false);
                constexpr uint32_t idesc_pv = idesc_bf16_f32(kPfRows, D, false, true);
                const uint32_t q_base = smem_u32(sQ);
                const uint32_t ring_base = smem_u32(sRing);
                auto ready = [&](int item) -> bool {
                    if (!mbar_wait(&full[item % kPfRing], (item / kPfRing) & 1, abort_flag, p.status)) return false;
                    tc_fence_after();
                    return true;
                };
                auto issue_qk = [&](int t, int item) {
                    const uint32_t d_tmem = tmem + t * 128;
                    const uint32_t a0 = q_base + t * SM::kTile;
                    const uint32_t b0 = ring_base + (item % kPfRing) * SM::kTile;
    #pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t o = (ks >> 2) * SM::kHalf + (ks & 3) * 32;
                        umma_ss(d_tmem, sdesc_sw128(a0 + o, 16, 1024), sdesc_sw128(b0 + o, 16, 1024), idesc_qk, ks > 0);
                    }
                };
                auto issue_pv = [&](int t, int item, bool acc) {
                    const uint32_t d_tmem = tmem + 256 + t * D;
                    const uint32_t a_tmem = tmem + t * 128;
                    const uint32_t b0 = ring_base + (item % kPfRing) * SM::kTile;
    #pragma unroll
                    for (int kk = 0; kk < kPfKeys / 16; ++kk)
                        umma_ts(d_tmem, a_tmem + kk * 8, sdesc_sw128(b0 + kk * 16 * 128, SM::kHalf, 1024), idesc_pv,
                                (acc || kk > 0) ? 1u : 0u);
                };
                // SPLIT: the query tiles whose weights' remainders also multiply V
                // (tile 0 splits whenever tile 1 does: its rows see fewer keys)
                int n_split = 0;
                if constexpr (SPLIT)
                    n_split = first_row_keys(PAGED, p.causal, p.S_q, p.S_kv, q0 + kPfRows, past) <= kPfSplitKeys ? 2
                              : first_row_keys(PAGED, p.causal, p.S_q, p.S_kv, q0, past) <= kPfSplitKeys   ? 1
                                                                                                            : 0;
                bool ok = mbar_wait(qfull, 0, abort_flag, p.status) && ready(0);
                if (ok) {
                    if (n_t0 > 0) { issue_qk(0, 0); umma_commit(&sfull[0]); }
                    if (n_t1 > 0) { issue_qk(1, 0); umma_commit(&sfull[1]); }
                    umma_commit(&empty[0]);
                }
                for (int j = 0; j < nmax && ok; ++j) {
                    bool v_ready = false, k_next = false;
    #pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const int n_t = t ? n_t1 : n_t0;
                        if (!ok || j >= n_t) continue;
                        if (!mbar_wait(&pfull[t], j & 1, abort_flag, p.status)) { ok = false; continue; }
                        tc_fence_after();
                        if (!v_ready) {
                            if (!ready(2 * j + 1)) { ok = false; continue; }
                            v_ready = true;
                            if (PAGED && j == n_past - 1 && (past % kPfKeys) != 0) {
                                // V rows past the cached tokens hold whatever the pages hold: zero them
                                uint8_t *vt = sRing + ((2 * j + 1) % kPfRing) * SM::kTile;
                                for (int hf = 0; hf < D / 64; ++hf)
                                    for (int r = past % kPfKeys; r < kPfKeys; ++r) {
                                        uint4 *row = reinterpret_cast<uint4 *>(vt + hf * SM::kHalf + r * 128);
#pragma unroll
                                        for (int c = 0; c < 8; ++c) row[c] = make_uint4(0u, 0u, 0u, 0u);
                                    }
                                fence_proxy_async_smem();   // generic-proxy stores before the tensor core reads
                            }
                        }
                        issue_pv(t, 2 * j + 1, j > 0);
                        if constexpr (SPLIT) {
                            if (t < n_split)
                                pf_issue_pv_rem(tmem + 256 + t * D, tmem + t * 128 + kPfKeys / 2,
                                                ring_base + ((2 * j + 1) % kPfRing) * SM::kTile, SM::kHalf, idesc_pv);
                        }
                        if (j + 1 < n_t) {
                            if (!k_next) {
                                if (!ready(2 * j + 2)) { ok = false; continue; }
                                k_next = true;
                            }
                            issue_qk(t, 2 * j + 2);
                            umma_commit(&sfull[t]);
                        } else {
                            umma_commit(&odone[t]);
                        }
                    }
                    if (v_ready) umma_commit(&empty[(2 * j + 1) % kPfRing]);
                    if (k_next) umma_commit(&empty[(2 * j + 2) % kPfRing]);
                }
                if (!ok) {   // nothing may still write TMEM when it is freed
                    umma_commit(drain);
                    mbar_wait_drain(drain, 0, p.status);
                }
            }
            __syncwarp();
        } else if (PAGED && head % p.G == 0) {
            // ------------------------------------------------------------ the append (warps 10, 11)
            // rows of this CTA's two query tiles -> cache positions past + row, K and V
            constexpr int CH = D * 2 / 16;   // 16-byte chunks per row
            const int w = threadIdx.x - 10 * 32;
            const int r0 = q0, r1 = min(q0 + 2 * kPfRows, p.S_q);
            const size_t row_elems = static_cast<size_t>(p.n_kv) * D;
            for (int it = w; it < (r1 - r0) * CH; it += 64) {
                const int t = r0 + it / CH, c = it % CH;
                const int pos = past + t;
                const int page = p.block_table[static_cast<size_t>(b) * p.max_blocks + pos / p.page_size];
                if (page < 0 || page >= p.num_pages) {
                    record_status(p.status, kStatusInvalid);
                    continue;
                }
                const size_t src = (static_cast<size_t>(b) * p.S_q + t) * row_elems + static_cast<size_t>(kvh) * D + c * 8;
                const size_t dst = (static_cast<size_t>(page) * p.page_size + pos % p.page_size) * row_elems +
                                   static_cast<size_t>(kvh) * D + c * 8;
                *reinterpret_cast<uint4 *>(p.k_pages + dst) = *reinterpret_cast<const uint4 *>(p.k_new + src);
                *reinterpret_cast<uint4 *>(p.v_pages + dst) = *reinterpret_cast<const uint4 *>(p.v_new + src);
            }
        }
    } else {
        regs_inc<kRegsSoftmax>();
        // ------------------------------------------------------------ softmax + epilogue
        const int t = warp >> 2;                    // query tile of this warpgroup
        const int quad = warp & 3;                  // TMEM lane quadrant
        const int n_t = t ? n_t1 : n_t0;
        const int r = quad * 32 + lane;             // row within the tile == TMEM lane
        const int row = q0 + t * kPfRows + r;       // absolute query row
        const int limit = p.causal ? min(p.S_kv - 1, row + (p.S_kv - p.S_q)) : p.S_kv - 1;   // (not PAGED)
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t tS = tmem + t * 128 + lane_off;
        const uint32_t tO = tmem + 256 + t * D + lane_off;
        const float cl2 = p.scale_log2;
        bool split = false;   // (SPLIT only) this tile's weights also go as bf16 remainders; warpgroup-uniform
        if constexpr (SPLIT)
            split = first_row_keys(PAGED, p.causal, p.S_q, p.S_kv, q0 + t * kPfRows, past) <= kPfSplitKeys;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        // the key-tile loop; the SPLIT instantiation compiles it twice (with the remainder pass
        // and without) and picks one per query tile, so the loop that runs stays compact
        auto tile_loop = [&](auto rem_tag) {
            constexpr bool kRem = decltype(rem_tag)::value;
            for (int j = 0; j < n_t; ++j) {
                const bool landed = mbar_wait(&sfull[t], j & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, landed)) { ok = false; break; }   // tcgen05.ld/st are warp-aligned
                tc_fence_after();
                // the whole S row of this thread, read once.  Columns c <= lim_c are visible:
                // PAGED past tile: cached tokens below `past`; chunk tile: causal within the chunk
                const int lim_c = !PAGED ? limit - j * kPfKeys
                                  : j < n_past ? past - 1 - j * kPfKeys
                                               : row - (j - n_past) * kPfKeys;
                const bool masked = lim_c < kPfKeys - 1;
                static_assert(kPfKeys == 128, "four 32-column TMEM loads per row");
                uint32_t r0[32], r1[32], r2[32], r3[32];
                tmem_ld32(tS, r0);
                tmem_ld32(tS + 32, r1);
                tmem_ld32(tS + 64, r2);
                tmem_ld32(tS + 96, r3);
                tmem_wait_ld();
                // column c of the row (c is a compile-time constant after unrolling)
    #define GQA_S(c) ((c) < 32 ? r0[(c)] : (c) < 64 ? r1[(c) - 32] : (c) < 96 ? r2[(c) - 64] : r3[(c) - 96])
                float mx;
                if (!masked) {
                    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    #pragma unroll
                    for (int c = 0; c < kPfKeys; c += 8) {
                        m4[0] = fmax3(m4[0], __uint_as_float(GQA_S(c)), __uint_as_float(GQA_S(c + 1)));
                        m4[1] = fmax3(m4[1], __uint_as_float(GQA_S(c + 2)), __uint_as_float(GQA_S(c + 3)));
                        m4[2] = fmax3(m4[2], __uint_as_float(GQA_S(c + 4)), __uint_as_float(GQA_S(c + 5)));
                        m4[3] = fmax3(m4[3], __uint_as_float(GQA_S(c + 6)), __uint_as_float(GQA_S(c + 7)));
                    }
                    mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                } else {
                    mx = -INFINITY;
    #pragma unroll
                    for (int c = 0; c < kPfKeys; ++c)
                        if (c <= lim_c) mx = fmaxf(mx, __uint_as_float(GQA_S(c)));
                }
                const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * cl2;
                if (j == 0) {
                    m_used = m_tile;
                } else {
                    const bool need = m_tile > m_used + kRescaleThreshold;
                    if (__any_sync(0xffffffffu, need)) {
                        const float m_new = need ? m_tile : m_used;
                        const float alpha = exp2f(m_used - m_new);
    #pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t ro[32];
                            tmem_ld32(tO + c * 32, ro);
                            tmem_wait_ld();
    #pragma unroll
                            for (int e = 0; e < 32; ++e) ro[e] = __float_as_uint(__uint_as_float(ro[e]) * alpha);
                            tmem_st32(tO + c * 32, ro);
                        }
                        tmem_wait_st();
                        l *= alpha;
                        m_used = m_new;
                    }
                }
                // P = exp2(S * scale * log2(e) - m) as packed bf16, written back over S;
                // the running sum adds exactly the rounded weights P V uses
                float2 rs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                if constexpr (kRem) {   // first the remainders w - bf16(w) (exact in fp32), as bf16, over
                                        // the upper half of S (its scores are in registers already)
    #pragma unroll
                    for (int ch = 0; ch < kPfKeys / 16; ++ch) {
                        uint32_t rk[8];
    #pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int c = ch * 16 + 2 * e;
                            const float2 x =
                                ffma2_bcast(__uint_as_float(GQA_S(c)), __uint_as_float(GQA_S(c + 1)), cl2, -m_used);
                            float w0 = exp2f(x.x), w1 = exp2f(x.y);
                            if (masked) {
                                if (c > lim_c) w0 = 0.f;
                                if (c + 1 > lim_c) w1 = 0.f;
                            }
                            const float2 u = unpack_bf16x2(pack_bf16x2(w0, w1));
                            rk[e] = pack_bf16x2(w0 - u.x, w1 - u.y);
                            rs2[e & 1] = fadd2(rs2[e & 1], unpack_bf16x2(rk[e]));
                        }
                        tmem_st8(tS + kPfKeys / 2 + ch * 8, rk);
                    }
                }
    #pragma unroll
                for (int ch = 0; ch < kPfKeys / 32; ++ch) {
                    uint32_t pk[16];
    #pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int c = ch * 32 + 2 * e;
                        const float2 x = ffma2_bcast(__uint_as_float(GQA_S(c)), __uint_as_float(GQA_S(c + 1)), cl2, -m_used);
                        uint32_t pp = pack_bf16x2(exp2f(x.x), exp2f(x.y));
                        if (masked) {   // masked keys add nothing (also when scale == 0)
                            if (c > lim_c) pp &= 0xFFFF0000u;
                            if (c + 1 > lim_c) pp &= 0x0000FFFFu;
                        }
                        pk[e] = pp;
                        rs2[e & 1] = fadd2(rs2[e & 1], unpack_bf16x2(pp));
                    }
                    tmem_st16(tS + ch * 16, pk);
                }
    #undef GQA_S
                const float rs = (rs2[0].x + rs2[1].x) + (rs2[0].y + rs2[1].y);
                l += rs;
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&pfull[t]);
            }
        };
        if constexpr (SPLIT) {
            if (split)
                tile_loop(std::true_type{});
            else
                tile_loop(std::false_type{});
        } else {
            tile_loop(std::false_type{});
        }
        // epilogue: O / l -> bf16 -> out[b, row, head, :]
        const bool fin = n_t > 0 && ok && mbar_wait(&odone[t], 0, abort_flag, p.status);
        if (__all_sync(0xffffffffu, fin)) {
            tc_fence_after();
            const float inv = 1.f / l;
            const bool store = row < p.S_q;
            __nv_bfloat16 *orow = p.out + ((static_cast<size_t>(b) * p.S_q + (store ? row : 0)) * p.h + head) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t raw[32];
                tmem_ld32(tO + c * 32, raw);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = pack_bf16x2(__uint_as_float(raw[2 * e]) * inv, __uint_as_float(raw[2 * e + 1]) * inv);
                if (store) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
            }
        }
    }

    // a short-row launch that started beside the common one finishes only after it, so that
    // work queued behind this launch still sees every output row
    if constexpr (SPLIT && !PAGED) asm volatile("griddepcontrol.wait;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// host launcher

struct PrefillCall {
    const void *q, *k, *v;          // PAGED: k, v = the chunk's new K/V [B, S_q, n_kv, D]
    void *out;
    int B, S_q, S_kv, h, n_kv, causal;
    float scale;
    cudaStream_t stream;
    // PAGED only
    void *k_pages, *v_pages;
    const int32_t *block_table, *past_lens;
    int max_blocks, page_size, num_pages;
};

template <int D, bool PAGED, bool SPLIT>
static int launch_prefill_range(const PrefillCall &c, int pair_lo, int pair_hi) {
    using SM = PrefillSmem<D>;
    auto kern = gqa_prefill_kernel<D, PAGED, SPLIT>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 3;
    static std::atomic<unsigned long long> attr_done{0};
    if (!gqa_host::once_per_device(attr_done, dev, [&] {
            return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kTotal) == cudaSuccess;
        }))
        return 3;
    CUtensorMap tq, tk, tv, tkp, tvp;
    const uint32_t box[4] = {64, 1, kPfRows, 1};
    {
        const uint64_t dims[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(c.h), static_cast<uint64_t>(c.S_q),
                                  static_cast<uint64_t>(c.B)};
        const uint64_t strides[3] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(c.h) * D * 2,
                                     static_cast<uint64_t>(c.S_q) * c.h * D * 2};
        if (!gqa_host::encode_tensor_map(&tq, c.q, 4, dims, strides, box)) return 3;
    }
    {
        const int S = PAGED ? c.S_q : c.S_kv;
        const uint64_t dims[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(c.n_kv), static_cast<uint64_t>(S),
                                  static_cast<uint64_t>(c.B)};
        const uint64_t strides[3] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(c.n_kv) * D * 2,
                                     static_cast<uint64_t>(S) * c.n_kv * D * 2};
        if (!gqa_host::encode_tensor_map(&tk, c.k, 4, dims, strides, box)) return 3;
        if (!gqa_host::encode_tensor_map(&tv, c.v, 4, dims, strides, box)) return 3;
    }
    if (PAGED) {
        // [num_pages, page_size, n_kv, D]; page ids past num_pages read as zeros
        const uint64_t dims[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(c.n_kv),
                                  static_cast<uint64_t>(c.page_size), static_cast<uint64_t>(c.num_pages)};
        const uint64_t strides[3] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(c.n_kv) * D * 2,
                                     static_cast<uint64_t>(c.page_size) * c.n_kv * D * 2};
        const uint32_t pbox[4] = {64, 1, static_cast<uint32_t>(std::min(c.page_size, kPfKeys)), 1};
        if (!gqa_host::encode_tensor_map(&tkp, c.k_pages, 4, dims, strides, pbox)) return 3;
        if (!gqa_host::encode_tensor_map(&tvp, c.v_pages, 4, dims, strides, pbox)) return 3;
    } else {
        tkp = tk;   // not read
        tvp = tv;
    }
    PrefillParams prm = {};
    prm.out = static_cast<__nv_bfloat16 *>(c.out);
    prm.B = c.B;
    prm.S_q = c.S_q;
    prm.S_kv = c.S_kv;
    prm.h = c.h;
    prm.n_kv = c.n_kv;
    prm.G = c.h / c.n_kv;
    prm.pair_lo = pair_lo;
    prm.pair_hi = pair_hi;
    prm.causal = c.causal ? 1 : 0;
    prm.scale_log2 = c.scale * 1.4426950408889634f;
    prm.status = gqa_host::device_status();
    if (!prm.status) return 3;
    GQA_SET_TEST_STALL(prm);
    prm.block_table = c.block_table;
    prm.past_lens = c.past_lens;
    prm.k_new = static_cast<const __nv_bfloat16 *>(c.k);
    prm.v_new = static_cast<const __nv_bfloat16 *>(c.v);
    prm.k_pages = static_cast<__nv_bfloat16 *>(c.k_pages);
    prm.v_pages = static_cast<__nv_bfloat16 *>(c.v_pages);
    prm.max_blocks = c.max_blocks;
    prm.page_size = c.page_size;
    prm.num_pages = c.num_pages;
    const long ctas = static_cast<long>(pair_hi - pair_lo) * c.B * c.h;
    if (ctas <= 0) return 0;
    if (ctas > 0x7fffffffL) return 1;
    if constexpr (SPLIT && !PAGED) {
        // a programmatic dependent of the common launch just queued (a plain launch where the
        // attribute is refused: the kernel's final wait is then a no-op)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
        cfg.blockDim = dim3(kPfThreads, 1, 1);
        cfg.dynamicSmemBytes = SM::kTotal;
        cfg.stream = c.stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, tkp, tvp, prm) == cudaSuccess) return 0;
        (void)cudaGetLastError();
    }
    kern<<<static_cast<unsigned>(ctas), kPfThreads, SM::kTotal, c.stream>>>(tq, tk, tv, tkp, tvp, prm);
    return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

// The pairs whose first query tile splits its weights go to the SPLIT instantiation
// (pairs [0, n_sp): the keys a tile's first row sees grow with the pair), the rest to
// the common one.  The chunked prefill (PAGED) cannot tell on the host (the past
// lengths live on the device): it runs the SPLIT instantiation, which decides per tile.
template <int D, bool PAGED>
static int launch_prefill_t(const PrefillCall &c) {
    const int n_pairs = (c.S_q + 2 * kPfRows - 1) / (2 * kPfRows);
    if constexpr (PAGED) {
        return launch_prefill_range<D, true, true>(c, 0, n_pairs);
    } else {
        int n_sp = 0;
        while (n_sp < n_pairs &&
               first_row_keys(false, c.causal, c.S_q, c.S_kv, n_sp * 2 * kPfRows, 0) <= kPfSplitKeys)
            ++n_sp;
        int st = launch_prefill_range<D, false, false>(c, n_sp, n_pairs);
        if (st == 0) st = launch_prefill_range<D, false, true>(c, 0, n_sp);
        return st;
    }
}

int launch_prefill(const void *q, const void *k, const void *v, void *out, int B, int S_q, int S_kv, int h, int n_kv,
                   int d, int causal, float scale, cudaStream_t stream) {
    PrefillCall c = {};
    c.q = q;
    c.k = k;
    c.v = v;
    c.out = out;
    c.B = B;
    c.S_q = S_q;
    c.S_kv = S_kv;
    c.h = h;
    c.n_kv = n_kv;
    c.causal = causal;
    c.scale = scale;
    c.stream = stream;
    if (d == 128) return launch_prefill_t<128, false>(c);
    return launch_prefill_t<64, false>(c);
}

int launch_prefill_paged(const void *q, const void *k_new, const void *v_new, void *k_pages, void *v_pages,
                         const int32_t *block_table, int max_blocks, int page_size, int num_pages,
                         const int32_t *past_lens, void *out, int B, int S_q, int h, int n_kv, int d, float scale,
                         cudaStream_t stream) {
    PrefillCall c = {};
    c.q = q;
    c.k = k_new;
    c.v = v_new;
    c.out = out;
    c.B = B;
    c.S_q = S_q;
    c.S_kv = S_q;
    c.h = h;
    c.n_kv = n_kv;
    c.causal = 1;
    c.scale = scale;
    c.stream = stream;
    c.k_pages = k_pages;
    c.v_pages = v_pages;
    c.block_table = block_table;
    c.past_lens = past_lens;
    c.max_blocks = max_blocks;
    c.page_size = page_size;
    c.num_pages = num_pages;
    if (d == 128) return launch_prefill_t<128, true>(c);
    return launch_prefill_t<64, true>(c);
}

}  // namespace gqa
