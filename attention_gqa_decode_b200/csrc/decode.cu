// Decode: one query token per sequence against its KV cache.  The cache is
// packed (sequence b's tokens contiguous, one after another) or paged (fixed
// pages placed anywhere, found through a block table), and its elements are
// bf16 or 8-bit E4M3 floats with one fp32 scale per KV head for K and for V.
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
//
// 8-bit caches ("Multi-Query Attention (MQA)" (inferensys glossary), "KV
// cache quantization"; "Multi-query attention" (pranaymahendrakar),
// "Interaction with other techniques": fp8 halves the bytes per element):
// a stage holds 128 tokens (the same bytes as 64 bf16 tokens).  The codes are
// widened exactly to f16 in registers (one cvt per pair) and the products run
// on f16 m16n8k16 MMAs: Q is re-encoded as f16, P is rounded to f16.  The K
// scale of the head is folded into the softmax scale and the V scale into
// the final 1 / l.  Fragment layouts:
//   - Q K^T: a non-transposed ldmatrix gives each lane 4 consecutive channels
//     of one token; the MMA's k index is permuted to match (k 2c+e <-> channel
//     4c+e, k 2c+8+e <-> channel 4c+2+e), and Q is loaded with the same
//     permutation, which leaves the dot products unchanged;
//   - P V: a transposed ldmatrix of the byte pairs gives each lane, for two
//     tokens, the codes of two adjacent channels; one byte permute splits
//     them into an even-channel and an odd-channel B fragment, so each
//     16-channel chunk is computed as two interleaved 8-channel n-tiles,
//     un-interleaved when the partials are written.
//
// Paged caches ("Multi-Query Attention (MQA)" (inferensys glossary),
// "PagedAttention": the cache is cut into fixed-size pages placed anywhere):
// token t of sequence b is slot t % page_size of page
// block_table[b][t / page_size]; a stage loads one TMA box per page piece.
// The producer warp reads the page ids of the next stage one stage ahead.  A
// page id outside [0, num_pages) is recorded as GQA_ERR_INVALID_ARG in the
// status word and read as zeros (an out-of-range TMA coordinate).  Slots past
// a sequence's end are masked: their scores by selection, their V codes in
// registers (0 * NaN would otherwise leak into the sums).
#include <cooperative_groups.h>

#include <algorithm>
#include <type_traits>

#include "common.cuh"

#ifndef GQA_DECODE_MAX_SPLIT
#define GQA_DECODE_MAX_SPLIT 8     // splits per (sequence, KV head) = thread-block cluster size
#endif

namespace cg = cooperative_groups;

namespace gqa {

constexpr int kDecWarps = 4;       // consumer warps
constexpr int kDecThreads = (kDecWarps + 1) * 32;
constexpr int kDecMaxHeads = 64;   // query heads one CTA serves (4 m-tiles of 16)
// bf16 caches: the softmax weights reach the tensor cores as bf16.  For a
// sequence of at most this many tokens, where a few keys can carry most of a
// row's weight (and the weights' rounding does not average out), they also
// go as the bf16 remainder p - bf16(p) in a second product, so they are
// carried to about 16 bits.
constexpr int kSplitAllBelow = 256;

enum class KvFmt { kBf16, kE4m3 };

// Shared-memory geometry of one stage's K (or V) tile.  A bf16 tile is stored
// as 64-dim panels of 128-byte token rows; an E4M3 tile as one panel of
// D-byte rows.  TMA writes each panel with the swizzle of its row width.
template <int D, KvFmt F>
struct DecGeom {
    static constexpr bool kFp8 = (F == KvFmt::kE4m3);
    static constexpr int kTok = kFp8 ? 128 : 64;         // tokens per pipeline stage (16 KB of K at d = 128)
    static constexpr int kRowBytes = kFp8 ? D : 128;     // one token's bytes in a panel
    static constexpr int kPanels = kFp8 ? 1 : D / 64;
    static constexpr int kBoxInner = kFp8 ? D : 64;      // TMA box, innermost extent in elements
    static constexpr int kPanelBytes = kTok * kRowBytes;
    static constexpr int kTileBytes = kPanels * kPanelBytes;
    static_assert(kRowBytes == 128 || kRowBytes == 64, "row width must be a TMA swizzle span");
    // XOR term of the swizzle for a row r with r % 8 == lane % 8:
    // 128-byte rows XOR the chunk with r % 8, 64-byte rows with (r / 2) % 4.
    __device__ static __forceinline__ uint32_t swz(uint32_t lane) {
        return kRowBytes == 128 ? (lane & 7u) : ((lane & 7u) >> 1);
    }
};

struct DecodeParams {
    const __nv_bfloat16 *q;
    const int32_t *seqlens;
    __nv_bfloat16 *out;
    const float *k_scale, *v_scale;   // E4M3 caches: one scale per KV head
    const int32_t *block_table;       // paged caches: [B, max_blocks]
    int max_blocks, page_size, num_pages;
    int B, h, n_kv, G, slices;        // slices = ceil(G / kDecMaxHeads)
    long long cache_rows;             // packed caches: rows the caches hold (the tensor maps' extent)
    float scale_log2;                 // scale * log2(e), >= 0
    int *status;                      // the library's device status word
    GQA_TEST_STALL_FIELD
};

template <int D, KvFmt F, int STAGES, bool TR>
struct DecodeSmem {
    static constexpr uint32_t kTileBytes = DecGeom<D, F>::kTileBytes;   // K or V of one stage
    static constexpr uint32_t kStageBytes = 2 * kTileBytes;
    static constexpr uint32_t kRingBytes = STAGES * kStageBytes;
    static constexpr uint32_t kCtrlBytes = 256;                       // barriers, flags
    static constexpr uint32_t kTotal = kRingBytes + kCtrlBytes + 1024;  // + alignment slack
    // After the ring has drained it is reused for the partial results:
    //   per-warp partials  part[WT][HS][D], pm[WT][HS], pl[WT][HS]
    //   per-CTA partial    co[HS][D], cm[HS], cl[HS]
    // (WT * HS <= 64 rows, HS <= 64; the transposed path has HS <= 8, WT = 4)
    static constexpr uint32_t kPartRows = TR ? 32 : 64;
    static constexpr uint32_t kCoRows = TR ? 8 : 64;
    static constexpr uint32_t kPartBytes = kPartRows * D * 4;
    static_assert(kPartBytes + 4 * 64 * 2 + kCoRows * D * 4 + 4 * 64 * 2 <= kRingBytes,
                  "partials must fit in the drained ring");
};

// Consumer of a group of at most 8 query heads, with the products transposed so
// that no tensor-core row is padding: tokens are the M rows and the heads the
// N = 8 columns.  S^T = K Q^T (K from shared memory as the A operand, Q as the
// B operand in registers), online softmax per column, then O^T += V^T P^T
// (V^T from a transposed ldmatrix as the A operand; P^T, the B operand, is
// the S^T accumulator packed to 16 bits and transposed in registers with
// movmatrix).  Per 16 tokens: D / 16 MMAs for each product.  Warp w takes
// tokens [w * TOK / WT, (w + 1) * TOK / WT) of every stage.
// O^T m-tile mt holds channels 16 mt + {g, g + 8} (bf16) or, for E4M3
// caches, 16 mt + {2g, 2g + 1} (the even/odd channel split of the byte
// pairs), g = lane / 4, for heads 2 (lane % 4) and 2 (lane % 4) + 1.
template <int D, int STAGES, int WT, KvFmt F, bool PAGED>
__device__ __forceinline__ void consume_transposed(const DecodeParams &p, uint8_t *smem, uint64_t *full,
                                                   uint64_t *empty, volatile int *abort_flag, int b, int head0,
                                                   int HS, int L, int first, int n_stages, float k_scale,
                                                   float (&o)[D / 8][4], float (&m_run)[2], float (&l_run)[2]) {
    using Geo = DecGeom<D, F>;
    using SM = DecodeSmem<D, F, STAGES, true>;
    constexpr bool FP8 = Geo::kFp8;
    constexpr int TOK = Geo::kTok;
    constexpr int RB = Geo::kRowBytes;
    constexpr int KSTEPS = D / 16;
    constexpr int TWARP = TOK / WT;      // tokens of a stage this warp handles
    constexpr int TT = TWARP / 16;       // 16-token tiles of them
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g8 = lane >> 2, q4 = lane & 3;

    // Q^T as the B operand: b0 = Q[head g8][k 2j, 2j+1], b1 = Q[head g8][k 2j+8, 2j+9]
    // (E4M3: k 2j+e <-> channel 4j+e, k 2j+8+e <-> channel 4j+2+e, as the K fragments)
    const __nv_bfloat16 *qrow = p.q + (static_cast<size_t>(b) * p.h + head0 + g8) * D;
    uint32_t qb[KSTEPS][2];
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
        if constexpr (!FP8) {
            const int c = ks * 16 + 2 * q4;
            qb[ks][0] = g8 < HS ? *reinterpret_cast<const uint32_t *>(qrow + c) : 0u;
            qb[ks][1] = g8 < HS ? *reinterpret_cast<const uint32_t *>(qrow + c + 8) : 0u;
        } else {
            const uint2 x = g8 < HS ? *reinterpret_cast<const uint2 *>(qrow + ks * 16 + 4 * q4) : make_uint2(0u, 0u);
            qb[ks][0] = bf16x2_to_f16x2(x.x);
            qb[ks][1] = bf16x2_to_f16x2(x.y);
        }
    }
    const float cl2 = p.scale_log2 * k_scale;
    const uint32_t sw = Geo::swz(lane);
    // ldmatrix lane roles (lane group m = lane / 8 addresses matrix m)
    const uint32_t arow = ((lane >> 3) & 1) * 8 + (lane & 7);   // K (A of S^T), E4M3 V: token within 16
    const uint32_t achk = lane >> 4;                            //   chunk within a pair
    const uint32_t vrow = ((lane >> 4) & 1) * 8 + (lane & 7);   // bf16 V (A of O^T): token within 16
    const uint32_t vchk = (lane >> 3) & 1;                      //   8-channel half of an m-tile
    const int tw0 = (warp % WT) * TWARP;

    for (int i = 0; i < n_stages; ++i) {
        const int slot = i % STAGES, use = i / STAGES;
        const bool landed = mbar_wait(&full[slot], use & 1, abort_flag, p.status);
        if (!__all_sync(0xffffffffu, landed)) break;   // warp-uniform: the mma/ldmatrix below are .aligned
        const int t0 = (first + i) * TOK;
        const int row_lo = PAGED ? 0 : max(0, t0 - (L - TOK));
        const int row_hi = PAGED ? min(TOK, L - t0) : TOK;
        if (row_lo >= tw0 + TWARP || row_hi <= tw0) {   // none of this warp's rows are valid
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
            continue;
        }
        const bool partial = row_lo > tw0 || row_hi < tw0 + TWARP;
        const bool split = !FP8 && L <= kSplitAllBelow;   // warp-uniform
        const uint32_t kbase = smem_u32(smem + slot * SM::kStageBytes) + tw0 * RB;
        const uint32_t vbase = kbase + SM::kTileBytes;

        // S^T = K Q^T: tile tt rows = tokens tw0 + 16 tt + {g8, g8 + 8}, columns = heads 2 q4, 2 q4 + 1
        float s[TT][4];
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
            s[tt][0] = s[tt][1] = s[tt][2] = s[tt][3] = 0.f;
            const uint32_t rowaddr = kbase + (tt * 16 + arow) * RB;
            if constexpr (!FP8) {
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks) {
                    const uint32_t chunk = 2 * ks + achk;
                    uint32_t a[4];
                    ldmatrix_x4(a[0], a[1], a[2], a[3],
                                rowaddr + (chunk >> 3) * Geo::kPanelBytes + (((chunk & 7) ^ (lane & 7)) << 4));
                    mma_bf16_16816(s[tt], a, qb[ks][0], qb[ks][1]);
                }
            } else {
#pragma unroll
                for (int kp = 0; kp < KSTEPS / 2; ++kp) {
                    // x0: tokens 0-7 of k-step 2kp; x1: tokens 8-15; x2, x3: the same for k-step 2kp+1
                    uint32_t x0, x1, x2, x3;
                    ldmatrix_x4(x0, x1, x2, x3, rowaddr + (((2 * kp + achk) ^ sw) << 4));
                    const uint32_t a0[4] = {e4m3x2_to_f16x2_lo(x0), e4m3x2_to_f16x2_lo(x1), e4m3x2_to_f16x2_hi(x0),
                                            e4m3x2_to_f16x2_hi(x1)};
                    mma_f16_16816(s[tt], a0, qb[2 * kp][0], qb[2 * kp][1]);
                    const uint32_t a1[4] = {e4m3x2_to_f16x2_lo(x2), e4m3x2_to_f16x2_lo(x3), e4m3x2_to_f16x2_hi(x2),
                                            e4m3x2_to_f16x2_hi(x3)};
                    mma_f16_16816(s[tt], a1, qb[2 * kp + 1][0], qb[2 * kp + 1][1]);
                }
            }
        }
        if (partial) {
#pragma unroll
            for (int tt = 0; tt < TT; ++tt) {
                const int row = tw0 + tt * 16 + g8;
                if (row < row_lo || row >= row_hi) s[tt][0] = s[tt][1] = -INFINITY;
                if (row + 8 < row_lo || row + 8 >= row_hi) s[tt][2] = s[tt][3] = -INFINITY;
            }
        }
        // online softmax per column (head): reduce over this lane's rows, then over the 8 lanes of a column
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
            mx[0] = fmax3(mx[0], s[tt][0], s[tt][2]);
            mx[1] = fmax3(mx[1], s[tt][1], s[tt][3]);
        }
        float alpha[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            mx[c] = fmaxf(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], 4));
            mx[c] = fmaxf(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], 8));
            mx[c] = fmaxf(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], 16));
            const float m_new = fmaxf(m_run[c], mx[c] * cl2);   // mx is finite: >= 1 valid token
            alpha[c] = exp2f(m_run[c] - m_new);
            m_run[c] = m_new;
            l_run[c] *= alpha[c];
        }
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            o[mt][0] *= alpha[0];
            o[mt][1] *= alpha[1];
            o[mt][2] *= alpha[0];
            o[mt][3] *= alpha[1];
        }
        // P^T B fragments: pack a row (token) of two heads, transpose the 8x8 blocks
        uint32_t pb[TT][2], pr[TT][2];   // the weights (bf16) and, on split stages, their bf16 remainders
        float2 ls = make_float2(0.f, 0.f);
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
            const float2 y0 = ffma2_bcast(s[tt][0], s[tt][1], cl2, 0.f);
            const float2 y1 = ffma2_bcast(s[tt][2], s[tt][3], cl2, 0.f);
            float e0 = exp2f(y0.x - m_run[0]), e1 = exp2f(y0.y - m_run[1]);
            float e2 = exp2f(y1.x - m_run[0]), e3 = exp2f(y1.y - m_run[1]);
            if (partial) {   // masked tokens add nothing (also when the scale is 0)
                const int row = tw0 + tt * 16 + g8;
                if (row < row_lo || row >= row_hi) e0 = e1 = 0.f;
                if (row + 8 < row_lo || row + 8 >= row_hi) e2 = e3 = 0.f;
            }
            uint32_t lo, hi;
            if constexpr (FP8) {
                lo = pack_f16x2(e0, e1);
                hi = pack_f16x2(e2, e3);
                ls = fadd2(ls, fadd2(unpack_f16x2(lo), unpack_f16x2(hi)));
            } else {
                lo = pack_bf16x2(e0, e1);
                hi = pack_bf16x2(e2, e3);
                const float2 ul = unpack_bf16x2(lo), uh = unpack_bf16x2(hi);
                ls = fadd2(ls, fadd2(ul, uh));
                if (split) {   // remainders (exact in fp32), rounded to bf16 for the second product
                    const uint32_t rl = pack_bf16x2(e0 - ul.x, e1 - ul.y), rh = pack_bf16x2(e2 - uh.x, e3 - uh.y);
                    ls = fadd2(ls, fadd2(unpack_bf16x2(rl), unpack_bf16x2(rh)));
                    pr[tt][0] = movmatrix_trans(rl);
                    pr[tt][1] = movmatrix_trans(rh);
                }
            }
            pb[tt][0] = movmatrix_trans(lo);   // P[head g8][tokens 2 q4, 2 q4 + 1]
            pb[tt][1] = movmatrix_trans(hi);   // P[head g8][tokens 2 q4 + 8, 2 q4 + 9]
        }
        l_run[0] += ls.x;
        l_run[1] += ls.y;
        // O^T += V^T P^T.  On edge stages the V values of invalid rows are zeroed in
        // registers: each half of a transposed fragment register is one token.
        auto pv = [&](auto masked) {
          constexpr bool MASKED = decltype(masked)::value;
#pragma unroll
          for (int tt = 0; tt < TT; ++tt) {
            uint32_t mlo = 0xFFFFFFFFu, mhi = 0xFFFFFFFFu;
            if constexpr (MASKED) {
                const int row = tw0 + tt * 16 + 2 * q4;
                auto ok = [&](int r) { return r >= row_lo && r < row_hi; };
                mlo = (ok(row) ? 0x0000FFFFu : 0u) | (ok(row + 1) ? 0xFFFF0000u : 0u);
                mhi = (ok(row + 8) ? 0x0000FFFFu : 0u) | (ok(row + 9) ? 0xFFFF0000u : 0u);
            }
            if constexpr (!FP8) {
                const uint32_t rowaddr = vbase + (tt * 16 + vrow) * RB;
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    // matrices: (tokens 0-7, channels 0-7), (0-7, 8-15), (8-15, 0-7), (8-15, 8-15) of m-tile mt
                    const uint32_t chunk = 2 * mt + vchk;
                    uint32_t a[4];
                    ldmatrix_x4_trans(a[0], a[1], a[2], a[3],
                                      rowaddr + (chunk >> 3) * Geo::kPanelBytes + (((chunk & 7) ^ (lane & 7)) << 4));
                    if constexpr (MASKED) {
                        a[0] &= mlo;
                        a[1] &= mlo;
                        a[2] &= mhi;
                        a[3] &= mhi;
                    }
                    mma_bf16_16816(o[mt], a, pb[tt][0], pb[tt][1]);
                    if (split) mma_bf16_16816(o[mt], a, pr[tt][0], pr[tt][1]);
                }
            } else {
                const uint32_t rowaddr = vbase + (tt * 16 + arow) * RB;
#pragma unroll
                for (int cp = 0; cp < D / 32; ++cp) {
                    // x0: tokens 0-7 of chunk 2cp; x1: tokens 8-15; x2, x3: the same for chunk 2cp+1.
                    // The permute puts the even channel's token pair in the low half, the odd's in the high.
                    uint32_t x0, x1, x2, x3;
                    ldmatrix_x4_trans(x0, x1, x2, x3, rowaddr + (((2 * cp + achk) ^ sw) << 4));
                    if constexpr (MASKED) {
                        x0 &= mlo;
                        x1 &= mhi;
                        x2 &= mlo;
                        x3 &= mhi;
                    }
                    x0 = __byte_perm(x0, 0, 0x3120);
                    x1 = __byte_perm(x1, 0, 0x3120);
                    x2 = __byte_perm(x2, 0, 0x3120);
                    x3 = __byte_perm(x3, 0, 0x3120);
                    const uint32_t a0[4] = {e4m3x2_to_f16x2_lo(x0), e4m3x2_to_f16x2_hi(x0), e4m3x2_to_f16x2_lo(x1),
                                            e4m3x2_to_f16x2_hi(x1)};
                    mma_f16_16816(o[2 * cp], a0, pb[tt][0], pb[tt][1]);
                    const uint32_t a1[4] = {e4m3x2_to_f16x2_lo(x2), e4m3x2_to_f16x2_hi(x2), e4m3x2_to_f16x2_lo(x3),
                                            e4m3x2_to_f16x2_hi(x3)};
                    mma_f16_16816(o[2 * cp + 1], a1, pb[tt][0], pb[tt][1]);
                }
            }
          }
        };
        if (partial)
            pv(std::true_type{});
        else
            pv(std::false_type{});
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
    }
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        l_run[c] += __shfl_xor_sync(0xffffffffu, l_run[c], 4);
        l_run[c] += __shfl_xor_sync(0xffffffffu, l_run[c], 8);
        l_run[c] += __shfl_xor_sync(0xffffffffu, l_run[c], 16);
    }
}

// WT = token sub-ranges per stage (4, 2 or 1): consumer warp w serves m-tile
// w / WT (16 query heads) on tokens [(w % WT) * TOK / WT, ...) of every stage,
// in passes of at most 32 (d = 128) or 64 (d = 64) tokens.
template <int D, int STAGES, int WT, KvFmt F, bool PAGED, bool TR, int MINB>
__global__ void __launch_bounds__(kDecThreads, MINB)
    gqa_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const DecodeParams p) {
    using Geo = DecGeom<D, F>;
    using SM = DecodeSmem<D, F, STAGES, TR>;
    constexpr bool FP8 = Geo::kFp8;
    constexpr int TOK = Geo::kTok;
    constexpr int RB = Geo::kRowBytes;
    constexpr int KSTEPS = D / 16;          // k-steps of Q K^T
    constexpr int NT_O = D / 8;             // n-tiles of O (dims)
    constexpr int TWARP = TOK / WT;         // tokens of a stage one warp handles
    constexpr int TCAP = D == 128 ? 32 : 64;       // register budget: O takes D / 2 registers
    constexpr int TPW = TWARP < TCAP ? TWARP : TCAP;   // tokens per pass
    constexpr int NPASS = TWARP / TPW;
    constexpr int NTS = TPW / 8;            // n-tiles of the scores of a pass
    constexpr int KKS = TPW / 16;           // k-steps of its P V

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + SM::kRingBytes);
    uint64_t *empty = full + STAGES;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + STAGES);
    long long *red = reinterpret_cast<long long *>(empty + STAGES + 1);   // [kDecWarps + 1] partial sums

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

    // packed caches: first cache row of sequence b = sum of the earlier (non-negative) lengths (64-bit)
    long long acc = 0;
    if (!PAGED)
        for (int i = threadIdx.x; i < b; i += kDecThreads) acc += max(p.seqlens[i], 0);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) red[warp] = acc;
    __syncthreads();
    long long off64 = 0;
#pragma unroll
    for (int w = 0; w <= kDecWarps; ++w) off64 += red[w];
    int L = max(p.seqlens[b], 0);
    if (PAGED && L > p.max_blocks * p.page_size) {   // longer than its block-table row
        if (threadIdx.x == 0) record_status(p.status, kStatusInvalid);
        L = p.max_blocks * p.page_size;
    }
    if (!PAGED && off64 + L > p.cache_rows) {   // the lengths ask for rows the caches do not hold
        if (threadIdx.x == 0) record_status(p.status, kStatusInvalid);
        L = static_cast<int>(max(0LL, p.cache_rows - off64));
    }
    // off + L <= cache_rows <= INT32_MAX whenever a row is read (the host bounds cache_rows)
    const int off = static_cast<int>(min(off64, p.cache_rows));

    // this split's stages: stage i covers tokens [t0, min(t0 + TOK, L)), t0 = TOK * (first + i)
    const int n_total = (L + TOK - 1) / TOK;
    const int per_split = (n_total + P - 1) / P;
    const int first = split * per_split;
    const int n_stages = max(0, min(n_total, first + per_split) - first);

    if (warp == kDecWarps) {
        // ------------------------------------------------------------ producer
        const int pb = PAGED ? min(p.page_size, TOK) : TOK;   // tokens per TMA box
        const int pieces = TOK / pb;                           // boxes per stage
        // paged: box k of stage i is piece n = i * pieces + k of this split; lane l
        // holds the page id of piece 32 * batch + l, the next batch loaded a batch ahead
        auto batch_of = [&](int batch) -> int {
            const int t = first * TOK + (batch * 32 + lane) * pb;
            int page = 0;
            if (PAGED && t < L) {
                page = p.block_table[static_cast<size_t>(b) * p.max_blocks + t / p.page_size];
                if (page < 0 || page >= p.num_pages) {   // read as zeros, reported
                    record_status(p.status, kStatusInvalid);
                    page = p.num_pages;
                }
            }
            return page;
        };
        int cur_batch = 0;
        int ids = (PAGED && n_stages > 0) ? batch_of(0) : 0;
        int ids_next = (PAGED && n_stages * pieces > 32) ? batch_of(1) : 0;
        int issued = 0;
        const int first_loaded = GQA_STALLED(p) ? 1 : 0;   // wait-test build: stage 0 never arrives
        for (int i = 0; i < n_stages; ++i) {
            const int slot = i % STAGES, use = i / STAGES;
            int ok = 1;
            if (lane == 0 && use > 0) ok = mbar_wait(&empty[slot], (use - 1) & 1, abort_flag, p.status);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            if (i < first_loaded) {
                ++issued;
                continue;
            }
            const int t0 = (first + i) * TOK;
            uint8_t *kdst = smem + slot * SM::kStageBytes;
            uint8_t *vdst = kdst + SM::kTileBytes;
            if constexpr (!PAGED) {
                if (lane == 0) {
                    // The last stage of a sequence is shifted back so it ends at the
                    // sequence end: the box never reads past the packed cache.
                    const int z = off + min(t0, L - TOK);
                    mbar_arrive_expect_tx(&full[slot], SM::kStageBytes);
#pragma unroll
                    for (int pp = 0; pp < Geo::kPanels; ++pp) {
                        tma_load_3d(kdst + pp * Geo::kPanelBytes, &tm_k, &full[slot], pp * 64, g, z);
                        tma_load_3d(vdst + pp * Geo::kPanelBytes, &tm_v, &full[slot], pp * 64, g, z);
                    }
                }
            } else {
                const int nb = (min(TOK, L - t0) + pb - 1) / pb;   // boxes of this stage
                if (lane == 0)
                    mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(nb * pb * RB * Geo::kPanels * 2));
                for (int j = 0; j < nb; ++j) {
                    const int n = i * pieces + j;
                    if (n / 32 != cur_batch) {   // warp-uniform
                        cur_batch = n / 32;
                        ids = ids_next;
                        if ((cur_batch + 1) * 32 < n_stages * pieces) ids_next = batch_of(cur_batch + 1);
                    }
                    const int page = __shfl_sync(0xffffffffu, ids, n % 32);
                    if (lane == 0) {
                        const int slot_in_page = (t0 + j * pb) % p.page_size;
#pragma unroll
                        for (int pp = 0; pp < Geo::kPanels; ++pp) {
                            const int dst = pp * Geo::kPanelBytes + j * pb * RB;
                            tma_load_4d(kdst + dst, &tm_k, &full[slot], pp * 64, g, slot_in_page, page);
                            tma_load_4d(vdst + dst, &tm_v, &full[slot], pp * 64, g, slot_in_page, page);
                        }
                    }
                }
            }
            ++issued;
        }
        if (lane == 0 && *abort_flag) {   // let the copies in flight land before the CTA moves on
            for (int i = max(first_loaded, issued - STAGES); i < issued; ++i)
                mbar_wait_drain(&full[i % STAGES], (i / STAGES) & 1, p.status);
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
    float k_scale = 1.f, v_scale = 1.f;
    if (FP8) {
        k_scale = p.k_scale[g];
        v_scale = p.v_scale[g];
        if (!(k_scale >= 0.f && k_scale <= 3.0e38f) || !(v_scale >= 0.f && v_scale <= 3.0e38f)) {
            if (threadIdx.x == 0) record_status(p.status, kStatusInvalid);   // negative, infinite or NaN
            k_scale = 0.f;
            v_scale = 0.f;
        }
    }

    if constexpr (TR) {
        if (consumer) consume_transposed<D, STAGES, WT, F, PAGED>(p, smem, full, empty, abort_flag, b, head0, HS, L,
                                                                   first, n_stages, k_scale, o, m_run, l_run);
    } else if (consumer) {
        // ------------------------------------------------------------ consumers
        // Q fragments of m-tile mi (rows = query heads of the group), kept in registers
        const int r0 = mi * 16 + (lane >> 2), r1 = r0 + 8;
        const int cq = 2 * (lane & 3);
        const __nv_bfloat16 *qb = p.q + (static_cast<size_t>(b) * p.h + head0) * D;
        uint32_t qa[KSTEPS][4];
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
            if constexpr (!FP8) {
                const int c = ks * 16 + cq;
                qa[ks][0] = r0 < HS ? *reinterpret_cast<const uint32_t *>(qb + r0 * D + c) : 0u;
                qa[ks][1] = r1 < HS ? *reinterpret_cast<const uint32_t *>(qb + r1 * D + c) : 0u;
                qa[ks][2] = r0 < HS ? *reinterpret_cast<const uint32_t *>(qb + r0 * D + c + 8) : 0u;
                qa[ks][3] = r1 < HS ? *reinterpret_cast<const uint32_t *>(qb + r1 * D + c + 8) : 0u;
            } else {   // k index 2c+e <-> channel 4c+e, 2c+8+e <-> 4c+2+e
                const int c = ks * 16 + 2 * cq;
                const uint2 x0 = r0 < HS ? *reinterpret_cast<const uint2 *>(qb + r0 * D + c) : make_uint2(0u, 0u);
                const uint2 x1 = r1 < HS ? *reinterpret_cast<const uint2 *>(qb + r1 * D + c) : make_uint2(0u, 0u);
                qa[ks][0] = bf16x2_to_f16x2(x0.x);
                qa[ks][1] = bf16x2_to_f16x2(x1.x);
                qa[ks][2] = bf16x2_to_f16x2(x0.y);
                qa[ks][3] = bf16x2_to_f16x2(x1.y);
            }
        }
        const float cl2 = p.scale_log2 * k_scale;
        const uint32_t sw = Geo::swz(lane);
        // ldmatrix lane roles
        const uint32_t lrow = ((lane >> 4) & 1) * 8 + (lane & 7);   // bf16 QK: token within a 16-token pair
        const uint32_t lchk = (lane >> 3) & 1;                      // bf16 QK: low/high 8 dims of a k-step
        const uint32_t frow = ((lane >> 3) & 1) * 8 + (lane & 7);   // fp8 QK and PV: token within 16 tokens
        const uint32_t fchk = lane >> 4;                            // chunk within a pair of chunks

        for (int i = 0; i < n_stages; ++i) {
            const int slot = i % STAGES, use = i / STAGES;
            const bool landed = mbar_wait(&full[slot], use & 1, abort_flag, p.status);
            if (!__all_sync(0xffffffffu, landed)) break;   // warp-uniform: the mma/ldmatrix below are .aligned
            const int t0 = (first + i) * TOK;
            // valid rows of the stage's box: [row_lo, row_hi)
            const int row_lo = PAGED ? 0 : max(0, t0 - (L - TOK));
            const int row_hi = PAGED ? min(TOK, L - t0) : TOK;
            const uint32_t stage = smem_u32(smem + slot * SM::kStageBytes);
#pragma unroll
            for (int pass = 0; pass < NPASS; ++pass) {
                const int tw0 = ti * TWARP + pass * TPW;              // first row of this pass
                if (row_lo >= tw0 + TPW || row_hi <= tw0) continue;  // no valid row here
                const bool partial = row_lo > tw0 || row_hi < tw0 + TPW;
                const bool split = !FP8 && L <= kSplitAllBelow;   // warp-uniform
                const uint32_t kbase = stage + tw0 * RB;
                const uint32_t vbase = kbase + SM::kTileBytes;

                // S = Q K^T  (16 heads x TPW tokens)
                float s[NTS][4];
#pragma unroll
                for (int nt = 0; nt < NTS; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
                if constexpr (!FP8) {
#pragma unroll
                    for (int ks = 0; ks < KSTEPS; ++ks) {
                        const uint32_t chunk = 2 * ks + lchk;
                        const uint32_t hbase =
                            kbase + (chunk >> 3) * Geo::kPanelBytes + ((((chunk & 7) ^ (lane & 7))) << 4);
#pragma unroll
                        for (int np = 0; np < NTS / 2; ++np) {
                            uint32_t b0, b1, b2, b3;
                            ldmatrix_x4(b0, b1, b2, b3, hbase + (np * 16 + lrow) * RB);
                            mma_bf16_16816(s[2 * np], qa[ks], b0, b1);
                            mma_bf16_16816(s[2 * np + 1], qa[ks], b2, b3);
                        }
                    }
                } else {
#pragma unroll
                    for (int kp = 0; kp < KSTEPS / 2; ++kp) {
                        const uint32_t cbase = kbase + (((2 * kp + fchk) ^ sw) << 4);
#pragma unroll
                        for (int np = 0; np < NTS / 2; ++np) {
                            // x0: tokens 0-7, k-step 2kp; x1: tokens 8-15, 2kp; x2: 0-7, 2kp+1; x3: 8-15, 2kp+1
                            uint32_t x0, x1, x2, x3;
                            ldmatrix_x4(x0, x1, x2, x3, cbase + (np * 16 + frow) * RB);
                            mma_f16_16816(s[2 * np], qa[2 * kp], e4m3x2_to_f16x2_lo(x0), e4m3x2_to_f16x2_hi(x0));
                            mma_f16_16816(s[2 * np + 1], qa[2 * kp], e4m3x2_to_f16x2_lo(x1), e4m3x2_to_f16x2_hi(x1));
                            mma_f16_16816(s[2 * np], qa[2 * kp + 1], e4m3x2_to_f16x2_lo(x2), e4m3x2_to_f16x2_hi(x2));
                            mma_f16_16816(s[2 * np + 1], qa[2 * kp + 1], e4m3x2_to_f16x2_lo(x3),
                                          e4m3x2_to_f16x2_hi(x3));
                        }
                    }
                }
                // online softmax over these tokens (rows r0 and r1 of the m-tile)
                if (partial) {
#pragma unroll
                    for (int nt = 0; nt < NTS; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int row = tw0 + nt * 8 + cq + (e & 1);
                            if (row < row_lo || row >= row_hi) s[nt][e] = -INFINITY;
                        }
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
                // P as bf16 (f16 for 8-bit caches) A fragments; the running sums add the rounded weights
                uint32_t pa[KKS][4], par[KKS][4];   // the weights and, on split stages, their bf16 remainders
                float2 ls0 = make_float2(0.f, 0.f), ls1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int nt = 0; nt < NTS; ++nt) {
                    const float2 y0 = ffma2_bcast(s[nt][0], s[nt][1], cl2, -m_run[0]);
                    const float2 y1 = ffma2_bcast(s[nt][2], s[nt][3], cl2, -m_run[1]);
                    float e0 = exp2f(y0.x), e1 = exp2f(y0.y), e2 = exp2f(y1.x), e3 = exp2f(y1.y);
                    if (partial) {   // masked tokens add nothing (also when the scale is 0)
                        const int row = tw0 + nt * 8 + cq;
                        if (row < row_lo || row >= row_hi) {
                            e0 = 0.f;
                            e2 = 0.f;
                        }
                        if (row + 1 < row_lo || row + 1 >= row_hi) {
                            e1 = 0.f;
                            e3 = 0.f;
                        }
                    }
                    uint32_t lo, hi;
                    if constexpr (FP8) {
                        lo = pack_f16x2(e0, e1);
                        hi = pack_f16x2(e2, e3);
                        ls0 = fadd2(ls0, unpack_f16x2(lo));
                        ls1 = fadd2(ls1, unpack_f16x2(hi));
                    } else {
                        lo = pack_bf16x2(e0, e1);
                        hi = pack_bf16x2(e2, e3);
                        const float2 ul = unpack_bf16x2(lo), uh = unpack_bf16x2(hi);
                        ls0 = fadd2(ls0, ul);
                        ls1 = fadd2(ls1, uh);
                        if (split) {   // remainders (exact in fp32), rounded to bf16 for the second product
                            const uint32_t rl = pack_bf16x2(e0 - ul.x, e1 - ul.y);
                            const uint32_t rh = pack_bf16x2(e2 - uh.x, e3 - uh.y);
                            ls0 = fadd2(ls0, unpack_bf16x2(rl));
                            ls1 = fadd2(ls1, unpack_bf16x2(rh));
                            par[nt >> 1][(nt & 1) * 2 + 0] = rl;
                            par[nt >> 1][(nt & 1) * 2 + 1] = rh;
                        }
                    }
                    pa[nt >> 1][(nt & 1) * 2 + 0] = lo;
                    pa[nt >> 1][(nt & 1) * 2 + 1] = hi;
                }
                l_run[0] += ls0.x + ls0.y;
                l_run[1] += ls1.x + ls1.y;
                // O += P V.  On edge passes the V values of invalid rows are zeroed in
                // registers: each half of a transposed fragment register is one token.
                auto pv = [&](auto masked) {
                  constexpr bool MASKED = decltype(masked)::value;
#pragma unroll
                  for (int kk = 0; kk < KKS; ++kk) {
                    uint32_t mlo = 0xFFFFFFFFu, mhi = 0xFFFFFFFFu;
                    if constexpr (MASKED) {
                        const int row = tw0 + kk * 16 + cq;   // this lane's tokens: row, row + 1 (and + 8)
                        auto ok = [&](int r) { return r >= row_lo && r < row_hi; };
                        mlo = (ok(row) ? 0x0000FFFFu : 0u) | (ok(row + 1) ? 0xFFFF0000u : 0u);
                        mhi = (ok(row + 8) ? 0x0000FFFFu : 0u) | (ok(row + 9) ? 0xFFFF0000u : 0u);
                    }
                    const uint32_t rowaddr = vbase + (kk * 16 + frow) * RB;
                    if constexpr (!FP8) {
#pragma unroll
                        for (int dp = 0; dp < NT_O / 2; ++dp) {
                            const uint32_t chunk = 2 * dp + fchk;
                            uint32_t b0, b1, b2, b3;
                            ldmatrix_x4_trans(b0, b1, b2, b3,
                                              rowaddr + (chunk >> 3) * Geo::kPanelBytes +
                                                  (((chunk & 7) ^ (lane & 7)) << 4));
                            if constexpr (MASKED) {
                                b0 &= mlo;
                                b1 &= mhi;
                                b2 &= mlo;
                                b3 &= mhi;
                            }
                            mma_bf16_16816(o[2 * dp], pa[kk], b0, b1);
                            mma_bf16_16816(o[2 * dp + 1], pa[kk], b2, b3);
                            if (split) {
                                mma_bf16_16816(o[2 * dp], par[kk], b0, b1);
                                mma_bf16_16816(o[2 * dp + 1], par[kk], b2, b3);
                            }
                        }
                    } else {
#pragma unroll
                        for (int cp = 0; cp < D / 32; ++cp) {
                            // x0: tokens 0-7 of chunk 2cp; x1: tokens 8-15; x2, x3: the same for chunk 2cp+1.
                            // Bytes of a register: (token, channel) = (2c, 2n), (2c, 2n+1), (2c+1, 2n), (2c+1, 2n+1);
                            // the permute makes the low half the even channel's pair and the high half the odd's.
                            uint32_t x0, x1, x2, x3;
                            ldmatrix_x4_trans(x0, x1, x2, x3, rowaddr + (((2 * cp + fchk) ^ sw) << 4));
                            if constexpr (MASKED) {
                                x0 &= mlo;
                                x1 &= mhi;
                                x2 &= mlo;
                                x3 &= mhi;
                            }
                            x0 = __byte_perm(x0, 0, 0x3120);
                            x1 = __byte_perm(x1, 0, 0x3120);
                            x2 = __byte_perm(x2, 0, 0x3120);
                            x3 = __byte_perm(x3, 0, 0x3120);
                            mma_f16_16816(o[4 * cp + 0], pa[kk], e4m3x2_to_f16x2_lo(x0), e4m3x2_to_f16x2_lo(x1));
                            mma_f16_16816(o[4 * cp + 1], pa[kk], e4m3x2_to_f16x2_hi(x0), e4m3x2_to_f16x2_hi(x1));
                            mma_f16_16816(o[4 * cp + 2], pa[kk], e4m3x2_to_f16x2_lo(x2), e4m3x2_to_f16x2_lo(x3));
                            mma_f16_16816(o[4 * cp + 3], pa[kk], e4m3x2_to_f16x2_hi(x2), e4m3x2_to_f16x2_hi(x3));
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
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
            l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
        }
    }

    // ---------------------------------------------------------------- combine
    __syncthreads();   // the ring has drained: reuse it for the partials
    float *part = reinterpret_cast<float *>(smem);               // [WT][HS][D]
    float *pm = part + SM::kPartRows * D;                        // [WT][HS]
    float *pl = pm + 64;                                         // [WT][HS]
    float *co = reinterpret_cast<float *>(smem + SM::kPartBytes + 4 * 64 * 2);   // [HS][D]
    float *cm = co + SM::kCoRows * D;                            // [HS]
    float *cl = cm + 64;                                         // [HS]
    if (consumer && TR) {
        // O^T m-tile mt: rows = channels, columns = heads 2j, 2j+1 (j = lane % 4)
        const int g8 = lane >> 2, h0 = 2 * (lane & 3), h1 = h0 + 1;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            const int c0 = FP8 ? mt * 16 + 2 * g8 : mt * 16 + g8;   // row g8
            const int c1 = FP8 ? c0 + 1 : c0 + 8;                    // row g8 + 8
            if (h0 < HS) {
                part[(ti * HS + h0) * D + c0] = o[mt][0];
                part[(ti * HS + h0) * D + c1] = o[mt][2];
            }
            if (h1 < HS) {
                part[(ti * HS + h1) * D + c0] = o[mt][1];
                part[(ti * HS + h1) * D + c1] = o[mt][3];
            }
        }
        if (g8 == 0) {
            if (h0 < HS) { pm[ti * HS + h0] = m_run[0]; pl[ti * HS + h0] = l_run[0]; }
            if (h1 < HS) { pm[ti * HS + h1] = m_run[1]; pl[ti * HS + h1] = l_run[1]; }
        }
    } else if (consumer) {
        const int r0 = mi * 16 + (lane >> 2), r1 = r0 + 8;
        const int cq = 2 * (lane & 3);
        if constexpr (!FP8) {
#pragma unroll
            for (int nt = 0; nt < NT_O; ++nt) {
                if (r0 < HS) *reinterpret_cast<float2 *>(&part[(ti * HS + r0) * D + nt * 8 + cq]) = make_float2(o[nt][0], o[nt][1]);
                if (r1 < HS) *reinterpret_cast<float2 *>(&part[(ti * HS + r1) * D + nt * 8 + cq]) = make_float2(o[nt][2], o[nt][3]);
            }
        } else {   // n-tile 2c holds channels 16c + 4j + {0, 2}, n-tile 2c+1 channels 16c + 4j + {1, 3}
#pragma unroll
            for (int c = 0; c < D / 16; ++c) {
                const int ch = c * 16 + 2 * cq;
                if (r0 < HS)
                    *reinterpret_cast<float4 *>(&part[(ti * HS + r0) * D + ch]) =
                        make_float4(o[2 * c][0], o[2 * c + 1][0], o[2 * c][1], o[2 * c + 1][1]);
                if (r1 < HS)
                    *reinterpret_cast<float4 *>(&part[(ti * HS + r1) * D + ch]) =
                        make_float4(o[2 * c][2], o[2 * c + 1][2], o[2 * c][3], o[2 * c + 1][3]);
            }
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
            const float inv = cl[r] > 0.f ? v_scale / cl[r] : 0.f;
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
        const float inv = sl > 0.f ? v_scale / sl : 0.f;
        if (ok) *reinterpret_cast<__nv_bfloat162 *>(ob + r * D + c) = __floats2bfloat162_rn(s0 * inv, s1 * inv);
    }
    cluster.sync();   // no CTA leaves while a peer may still read its shared memory
}

// ---------------------------------------------------------------------------
// host launcher

struct DecodeCall {
    const void *q, *k, *v;
    const float *k_scale, *v_scale;
    const int32_t *seqlens, *block_table;
    void *out;
    int B, h, n_kv, max_blocks, page_size, num_pages;
    long long cache_rows;   // packed caches: rows the caches hold (0 < rows <= INT32_MAX, or open: 2^30)
    float scale;
    cudaStream_t stream;
};

template <int D, int STAGES, int WT, KvFmt F, bool PAGED, bool TR, int MINB = 2>
static int launch_decode_t(const DecodeCall &c) {
    using Geo = DecGeom<D, F>;
    using SM = DecodeSmem<D, F, STAGES, TR>;
    auto kern = gqa_decode_kernel<D, STAGES, WT, F, PAGED, TR, MINB>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 3;
    static std::atomic<unsigned long long> attr_done{0};
    if (!gqa_host::once_per_device(attr_done, dev, [&] {
            return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kTotal) == cudaSuccess &&
                   (GQA_DECODE_MAX_SPLIT <= 8 ||
                    cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess);
        }))
        return 3;
    constexpr uint64_t E = Geo::kFp8 ? 1 : 2;   // bytes per element
    const CUtensorMapDataType dt = Geo::kFp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapSwizzle swz = Geo::kRowBytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUtensorMap tk, tv;
    if (!PAGED) {
        // [tokens, n_kv, D]; the token extent is the caches' row count (the kernel cuts
        // lengths that ask for more rows and reports them)
        const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(c.n_kv),
                                  static_cast<uint64_t>(std::max(c.cache_rows, 1LL))};
        const uint64_t strides[2] = {D * E, static_cast<uint64_t>(c.n_kv) * D * E};
        const uint32_t box[3] = {static_cast<uint32_t>(Geo::kBoxInner), 1, static_cast<uint32_t>(Geo::kTok)};
        if (!gqa_host::encode_tensor_map_ex(&tk, dt, swz, c.k, 3, dims, strides, box)) return 3;
        if (!gqa_host::encode_tensor_map_ex(&tv, dt, swz, c.v, 3, dims, strides, box)) return 3;
    } else {
        // [num_pages, page_size, n_kv, D]; page ids past num_pages read as zeros
        const uint64_t dims[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(c.n_kv),
                                  static_cast<uint64_t>(c.page_size), static_cast<uint64_t>(c.num_pages)};
        const uint64_t strides[3] = {D * E, static_cast<uint64_t>(c.n_kv) * D * E,
                                     static_cast<uint64_t>(c.page_size) * c.n_kv * D * E};
        const uint32_t box[4] = {static_cast<uint32_t>(Geo::kBoxInner), 1,
                                 static_cast<uint32_t>(std::min(c.page_size, Geo::kTok)), 1};
        if (!gqa_host::encode_tensor_map_ex(&tk, dt, swz, c.k, 4, dims, strides, box)) return 3;
        if (!gqa_host::encode_tensor_map_ex(&tv, dt, swz, c.v, 4, dims, strides, box)) return 3;
    }

    const int G = c.h / c.n_kv;
    const int slices = (G + kDecMaxHeads - 1) / kDecMaxHeads;
    const long units = static_cast<long>(c.B) * c.n_kv * slices;
    const int sms = gqa_host::sm_count();
    // Splits per (sequence, KV head): as many as fit in one wave of resident
    // CTAs (two per SM), at most the cluster limit.  Longer CTAs amortise their
    // start and merge; a second, partial wave would leave SMs idle at the end.
    // (MINB resident CTAs per SM: 2 with a 3-stage ring, 3 with a 2-stage ring.)
    const long slots = static_cast<long>(MINB) * sms;
    const int P = static_cast<int>(std::max(1L, std::min(static_cast<long>(GQA_DECODE_MAX_SPLIT), slots / units)));

    DecodeParams prm;
    prm.q = static_cast<const __nv_bfloat16 *>(c.q);
    prm.seqlens = c.seqlens;
    prm.out = static_cast<__nv_bfloat16 *>(c.out);
    prm.k_scale = c.k_scale;
    prm.v_scale = c.v_scale;
    prm.block_table = c.block_table;
    prm.max_blocks = c.max_blocks;
    prm.page_size = c.page_size;
    prm.num_pages = c.num_pages;
    prm.B = c.B;
    prm.h = c.h;
    prm.n_kv = c.n_kv;
    prm.G = G;
    prm.slices = slices;
    prm.cache_rows = c.cache_rows;
    prm.scale_log2 = c.scale * 1.4426950408889634f;
    prm.status = gqa_host::device_status();
    if (!prm.status) return 3;
    GQA_SET_TEST_STALL(prm);

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P, c.n_kv * slices, c.B);
    cfg.blockDim = dim3(kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = SM::kTotal;
    cfg.stream = c.stream;
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

template <int D, int STAGES, KvFmt F, bool PAGED>
static int launch_decode_d(const DecodeCall &c) {
    const int HS = std::min(c.h / c.n_kv, kDecMaxHeads);   // query heads per CTA
    if (HS <= 8) return launch_decode_t<D, STAGES, 4, F, PAGED, true>(c);
    if (HS <= 16) return launch_decode_t<D, STAGES, 4, F, PAGED, false>(c);
    if (HS <= 32) return launch_decode_t<D, STAGES, 2, F, PAGED, false>(c);
    return launch_decode_t<D, STAGES, 1, F, PAGED, false>(c);
}

// Ring depth: 96 KB of stages per CTA, two CTAs per SM.
template <KvFmt F, bool PAGED>
static int launch_decode_f(const DecodeCall &c, int d) {
    if (d == 128) return launch_decode_d<128, 3, F, PAGED>(c);
    return launch_decode_d<64, 6, F, PAGED>(c);
}

int launch_decode(const void *q, const void *k, const void *v, const int32_t *seqlens, void *out, int B, int h,
                  int n_kv, int d, float scale, long long cache_rows, cudaStream_t stream) {
    const DecodeCall c{q, k, v, nullptr, nullptr, seqlens, nullptr, out, B, h, n_kv, 0, 0, 0, cache_rows, scale,
                       stream};
    return launch_decode_f<KvFmt::kBf16, false>(c, d);
}

int launch_decode_ex(const void *q, const void *k, const void *v, const float *k_scale, const float *v_scale,
                     const int32_t *seqlens, const int32_t *block_table, int max_blocks, int page_size,
                     int num_pages, void *out, int B, int h, int n_kv, int d, float scale, long long cache_rows,
                     cudaStream_t stream) {
    const DecodeCall c{q,   k,         v,         k_scale, v_scale, seqlens, block_table, out,  B,
                       h,   n_kv,      max_blocks, page_size, num_pages, cache_rows, scale, stream};
    const bool fp8 = k_scale != nullptr, paged = block_table != nullptr;
    if (fp8 && paged) return launch_decode_f<KvFmt::kE4m3, true>(c, d);
    if (fp8) return launch_decode_f<KvFmt::kE4m3, false>(c, d);
    if (paged) return launch_decode_f<KvFmt::kBf16, true>(c, d);
    return launch_decode_f<KvFmt::kBf16, false>(c, d);
}

}  // namespace gqa
