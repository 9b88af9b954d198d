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

struct PrefillParams {
    __nv_bfloat16 *out;
    int B, S_q, S_kv, h, n_kv, G, n_pairs, causal;
    float scale_log2;
    int *status;                   // the library's device status word
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

template <int D>
__global__ void __launch_bounds__(kPfThreads, 1)
    gqa_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
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

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // work unit: heaviest causal query-tile pairs first; consecutive CTAs share a KV group
    const int BH = p.B * p.h;
    const int bh = blockIdx.x % BH;
    const int pr = blockIdx.x / BH;
    const int pair = p.causal ? (p.n_pairs - 1 - pr) : pr;
    const int b = bh / p.h, head = bh % p.h, kvh = head / p.G;
    const int q0 = pair * 2 * kPfRows;
    const int n_t0 = kv_tiles_for(q0, p.S_q, p.S_kv, p.causal);
    const int n_t1 = kv_tiles_for(q0 + kPfRows, p.S_q, p.S_kv, p.causal);
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
            if (lane == 0) {
                tma_prefetch_desc(&tm_q);
                tma_prefetch_desc(&tm_k);
                tma_prefetch_desc(&tm_v);
                mbar_arrive_expect_tx(qfull, SM::kQ);
                for (int t = 0; t < 2; ++t)
                    for (int hf = 0; hf < D / 64; ++hf)
                        tma_load_4d(sQ + t * SM::kTile + hf * SM::kHalf, &tm_q, qfull, hf * 64, head, q0 + t * kPfRows, b);
                int item = 0;
                bool stop = false;
                for (int j = 0; j < nmax && !stop; ++j) {
                    for (int kv = 0; kv < 2; ++kv, ++item) {
                        const int slot = item % kPfRing, use = item / kPfRing;
                        if (use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1, abort_flag, p.status)) { stop = true; break; }
                        mbar_arrive_expect_tx(&full[slot], SM::kTile);
                        const CUtensorMap *map = kv ? &tm_v : &tm_k;
                        for (int hf = 0; hf < D / 64; ++hf)
                            tma_load_4d(sRing + slot * SM::kTile + hf * SM::kHalf, map, &full[slot], hf * 64, kvh,
                                        j * kPfKeys, b);
                    }
                }
                if (*abort_flag) {   // let the copies in flight land before TMEM and smem go away
                    mbar_wait_drain(qfull, 0, p.status);
                    for (int i = max(0, item - kPfRing); i < item; ++i)
                        mbar_wait_drain(&full[i % kPfRing], (i / kPfRing) & 1, p.status);
                }
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
                        }
                        issue_pv(t, 2 * j + 1, j > 0);
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
        }
    } else {
        regs_inc<kRegsSoftmax>();
        // ------------------------------------------------------------ softmax + epilogue
        const int t = warp >> 2;                    // query tile of this warpgroup
        const int quad = warp & 3;                  // TMEM lane quadrant
        const int n_t = t ? n_t1 : n_t0;
        const int r = quad * 32 + lane;             // row within the tile == TMEM lane
        const int row = q0 + t * kPfRows + r;       // absolute query row
        const int limit = p.causal ? min(p.S_kv - 1, row + (p.S_kv - p.S_q)) : p.S_kv - 1;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t tS = tmem + t * 128 + lane_off;
        const uint32_t tO = tmem + 256 + t * D + lane_off;
        const float cl2 = p.scale_log2;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_t; ++j) {
            const bool landed = mbar_wait(&sfull[t], j & 1, abort_flag, p.status);
            if (!__all_sync(0xffffffffu, landed)) { ok = false; break; }   // tcgen05.ld/st are warp-aligned
            tc_fence_after();
            // the whole S row of this thread, read once
            const int key0 = j * kPfKeys;
            const bool masked = key0 + kPfKeys - 1 > limit;
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
                    if (key0 + c <= limit) mx = fmaxf(mx, __uint_as_float(GQA_S(c)));
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
#pragma unroll
            for (int ch = 0; ch < kPfKeys / 32; ++ch) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int c = ch * 32 + 2 * e;
                    const float2 x = ffma2_bcast(__uint_as_float(GQA_S(c)), __uint_as_float(GQA_S(c + 1)), cl2, -m_used);
                    uint32_t pp = pack_bf16x2(exp2f(x.x), exp2f(x.y));
                    if (masked) {   // masked keys add nothing (also when scale == 0)
                        if (key0 + c > limit) pp &= 0xFFFF0000u;
                        if (key0 + c + 1 > limit) pp &= 0x0000FFFFu;
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

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// host launcher

template <int D>
static int launch_prefill_t(const void *q, const void *k, const void *v, void *out, int B, int S_q, int S_kv, int h,
                            int n_kv, int causal, float scale, cudaStream_t stream) {
    using SM = PrefillSmem<D>;
    auto kern = gqa_prefill_kernel<D>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 3;
    static unsigned long long attr_done = 0;   // one bit per device
    if (dev < 64 && !(attr_done >> dev & 1ull)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kTotal) != cudaSuccess)
            return 3;
        attr_done |= 1ull << dev;
    }
    CUtensorMap tq, tk, tv;
    const uint32_t box[4] = {64, 1, kPfRows, 1};
    {
        const uint64_t dims[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(h), static_cast<uint64_t>(S_q),
                                  static_cast<uint64_t>(B)};
        const uint64_t strides[3] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(h) * D * 2,
                                     static_cast<uint64_t>(S_q) * h * D * 2};
        if (!gqa_host::encode_tensor_map(&tq, q, 4, dims, strides, box)) return 3;
    }
    {
        const uint64_t dims[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(n_kv), static_cast<uint64_t>(S_kv),
                                  static_cast<uint64_t>(B)};
        const uint64_t strides[3] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(n_kv) * D * 2,
                                     static_cast<uint64_t>(S_kv) * n_kv * D * 2};
        if (!gqa_host::encode_tensor_map(&tk, k, 4, dims, strides, box)) return 3;
        if (!gqa_host::encode_tensor_map(&tv, v, 4, dims, strides, box)) return 3;
    }
    PrefillParams prm;
    prm.out = static_cast<__nv_bfloat16 *>(out);
    prm.B = B;
    prm.S_q = S_q;
    prm.S_kv = S_kv;
    prm.h = h;
    prm.n_kv = n_kv;
    prm.G = h / n_kv;
    prm.n_pairs = (S_q + 2 * kPfRows - 1) / (2 * kPfRows);
    prm.causal = causal ? 1 : 0;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.status = gqa_host::device_status();
    if (!prm.status) return 3;
    const long ctas = static_cast<long>(prm.n_pairs) * B * h;
    if (ctas > 0x7fffffffL) return 1;
    gqa_prefill_kernel<D><<<static_cast<unsigned>(ctas), kPfThreads, SM::kTotal, stream>>>(tq, tk, tv, prm);
    return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

int launch_prefill(const void *q, const void *k, const void *v, void *out, int B, int S_q, int S_kv, int h, int n_kv,
                   int d, int causal, float scale, cudaStream_t stream) {
    if (d == 128) return launch_prefill_t<128>(q, k, v, out, B, S_q, S_kv, h, n_kv, causal, scale, stream);
    return launch_prefill_t<64>(q, k, v, out, B, S_q, S_kv, h, n_kv, causal, scale, stream);
}

}  // namespace gqa
