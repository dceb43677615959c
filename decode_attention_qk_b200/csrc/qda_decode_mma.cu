// Tensor-core attention step for the larger Qwen3 sizes -- 32, 40 or 64 query
// heads over 8 kv heads of 128 (nnterp qwen3, "Grouped-query attention, with
// 128-wide heads on every size"), i.e. G = 4, 5 or 8 query heads per kv head --
// and for T > 1 new tokens per sequence at any size with T*G <= 8. Same
// computation as the 16-head decode kernel (Qwen3-0.6B Model Spec,
// "Compute-graph nodes": attn.qk_norm, attn.rope, attn.core, and the append
// to the 16-token paged cache); query head h reads kv head h / G. With T new
// tokens, token t sits in cache slot L - T + t and attends over slots up to
// its own (Model Spec, "What to watch for": every layer is full causal
// attention).
//
// Why tensor cores here. Per kv head and page the scores and the value sums
// are a [G x 128] x [128 x 16] and a [G x 16] x [16 x 128] product: 2G flops
// per byte of K/V, 16 at G = 8, above what the CUDA cores sustain at HBM
// speed. Warp j (kv head j) runs them as mma.sync m16n8k16 bf16 products with
// float accumulators. Query row r < T*G stands for new token r / G and head
// G*j + r % G; the 16 rows of the A operand hold, for row r, row r = the bf16
// value of q (or of the probabilities) and row r + 8 = the bf16 of the
// remainder, so the products carry ~16 significant bits of q and p; the two
// rows are added back in float. The score accumulator fragment of lane
// (r = lane/4, t = lane%4) holds row r at page tokens 2t, 2t+1, 8+2t, 9+2t,
// which is exactly its A fragment for the value product, so probabilities
// never leave registers. Each row masks the tokens after its own slot.
//
// Staging. A producer warp bulk-copies each token row (2 KiB, all 8 kv heads)
// into a stage whose rows are 2064 bytes apart, so that the 8 rows an
// ldmatrix phase reads start in 8 different 16-byte bank groups (at the
// cache's own 2048-byte pitch they would all hit the same banks). Each
// sequence piece's T qkv rows go to one slot of their own, released by the
// consumers once they have formed q. Only cache rows older than the new
// tokens are copied; the new tokens' k (formed in double, rounded once to
// bf16) and v are appended to the cache by the CTA holding their page and
// patched into its staged page.
//
// Split sequences. The work split is the 16-head kernel's (equal page ranges
// per CTA, scratch slot g + b per piece). A piece that covers its whole
// sequence writes o; a piece of a split sequence writes its partial, and a
// second launch (one CTA per sequence and kv head, one warp per query row)
// combines them with the log-sum-exp rule (Supported models, "Facts proved
// about the specs": flashAttn_eq, softmax_shift), spreading long merges over
// many SMs. Both launches are programmatic dependent launches: the combine
// launch starts while the attention launch ends, and the attention launch
// while the previous step's last launch ends; each waits for its predecessor
// to complete before it touches global memory.
#include <cuda_bf16.h>
#include <cstdint>

#include "qda_device.cuh"
#include "qda_internal.h"
#include "qwen3_decode_attn.h"

namespace qda {
namespace {

constexpr int kConsumerWarps = kNumKvHeads;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kRowPitch = kRowBytes + 16;           // staged token-row pitch: 2064 bytes
constexpr int kStageK = 0;
constexpr int kStageV = kPage * kRowPitch;
constexpr int kStageBytes = 2 * kPage * kRowPitch;  // 66048

// Row stride (float2 entries) of the rotation table: one more than the 64
// pairs, so that lanes reading the same pair for different tokens fall in
// different banks.
constexpr int kRotStride = 65;

template <int G, int T>
struct Layout {
    static constexpr int kHq = G * kNumKvHeads;
    static constexpr int kQkvW = (kHq + 2 * kNumKvHeads) * kHeadDim;     // elements in one token's qkv row
    static constexpr int kQkvBytes = kQkvW * 2;
    static constexpr int kSlotBytes = T * kQkvBytes;                     // a sequence's T rows
    static constexpr int kQRowBytes = kHq * kHeadDim * 2;                // the q part of one row
    static constexpr int kRows = G * T;                                  // query rows per kv head
    static constexpr bool kWide = kRows > 8;
    // Up to 8 query rows per kv head the rows are staged in a shared-memory
    // slot next to three K/V stages: whole when they take up to 24 KiB, else
    // (16 heads x 4 tokens: 32 KiB) their q parts only, the new k and v words
    // being read from global memory (prefetched to L2) by the CTA appending
    // them. Wide instances read the rows from global memory.
    static constexpr bool kDirectQkv = kWide;
    static constexpr bool kStageQOnly = !kWide && kSlotBytes > 24576;
    static constexpr int kStagedBytes = kWide ? 0 : (kStageQOnly ? T * kQRowBytes : kSlotBytes);
    static constexpr int kStages = 3;
    static constexpr int kSmemQkv = kStages * kStageBytes;
    // wide instances: the new tokens' k words, [warp][token][64] (formed when a sequence starts)
    static constexpr int kSmemNewK = kSmemQkv + kStagedBytes;
    static constexpr int kNewKBytes = (kRows > 8) ? kConsumerWarps * T * 64 * 4 : 0;
    static constexpr int kSmemSeg = kSmemNewK + kNewKBytes;                   // int [kMaxBatch + 4]
    static constexpr int kSmemLens = kSmemSeg + (kMaxBatch + 4) * 4;        // int [kMaxBatch]
    static constexpr int kSmemInvFreq = kSmemLens + kMaxBatch * 4;          // double [64]
    // (cos f_i, sin f_i) in double, the step of pair i from one position to the next
    static constexpr int kSmemStep = kSmemInvFreq + 64 * 8;                 // double2 [64]
    // (cos, sin) of u * f_i in float for the later new tokens u = 1..T-1
    static constexpr int kSmemRot = kSmemStep + 64 * 16;                    // float2 [T - 1][kRotStride]
    static constexpr int kSmemGains = kSmemRot + (T - 1) * kRotStride * 8;  // bf16 [2][128]
    static constexpr int kSmemMeta = kSmemGains + 2 * kHeadDim * 2;         // StageMeta [kStages] + qkv position
    static constexpr int kSmemBars = kSmemMeta + (kStages + 1) * 16;        // full, empty, qkv_full, qkv_empty, never
    static constexpr int kSmemFlags = kSmemBars + (2 * kStages + 3) * 8;
    static constexpr int kSmemTotal = kSmemFlags + 16;
    // Up to 8 query rows per kv head, q and the probabilities enter the tensor
    // cores as two bf16 terms (value and remainder, rows r and r + 8 of the
    // A operand); with 9 to 16 rows ("wide"), the 16 rows are 16 query rows
    // and q and the probabilities enter as bf16.
    static_assert(kRows <= 16, "at most 16 query rows per kv head");
    static_assert(kStagedBytes <= 24576, "the staged rows leave room for three K/V stages");
    static_assert(kSmemQkv % 16 == 0 && kSmemInvFreq % 16 == 0 && kSmemBars % 8 == 0, "alignment");
    static_assert(kSmemTotal <= 227 * 1024, "fits one CTA per SM");
};

// Row of a split piece's partial: query row r (new token r / G, head
// G*j + r % G) of kv head j in scratch slot `slot`.
template <int G, int T>
__device__ __forceinline__ size_t part_row(int j, int slot, int r) {
    return (size_t)slot * kPartRows + (size_t)(r / G) * Layout<G, T>::kHq + G * j + r % G;
}

// Row of qkv (and of o) holding new token u of sequence b: a call may cover
// tokens [tok_offset, tok_offset + T) of blocks of tok_stride tokens per
// sequence (a long block of new tokens runs as several such launches).
__device__ __forceinline__ size_t token_row(const Params& p, int b, int u) {
    return (size_t)b * p.tok_stride + p.tok_offset + u;
}

// RoPE position of the first new token of this launch for sequence b of
// (trimmed) length L with T new tokens in this launch.
__device__ __forceinline__ int first_position(const Params& p, int b, int L, int T) {
    return p.positions != nullptr ? __ldg(p.positions + b) + p.tok_offset : L - T;
}

// Prefetch `bytes` (a multiple of 16, 16-byte aligned) from global memory to L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

struct Shared {
    uint8_t* stages;
    uint32_t* new_k;      // wide instances: [warp][token][64] k words of the new tokens
    uint8_t* qkv;         // the current sequence piece's T qkv rows
    int* seg;
    int* lens;
    double* inv_freq;
    double2* step;        // [64] (cos f_i, sin f_i)
    float2* rot;          // [T - 1][kRotStride] (cos, sin) of u * f_i, u = 1..T-1
    const uint16_t* gains;
    volatile StageMeta* meta;
    volatile int* qkv_pos;
    uint64_t* full_bar;
    uint64_t* empty_bar;
    uint64_t* qkv_full;
    uint64_t* qkv_empty;
    uint64_t* never_bar;
    volatile int* abort_flag;
};

// ---------------------------------------------------------------------------
// Producer warp.

template <int G, int T>
__device__ __forceinline__ void run_producer(const Params& p, const Shared& s, int B, int start, int end, int lane) {
    using Lay = Layout<G, T>;
    constexpr int kStages = Lay::kStages;
    const int count = end - start;
    int slot = 0;
    uint32_t phase = 0, qphase = 0;
    uint32_t armed = 0, armed_parity = 0;
    bool qarmed = false;
    uint32_t qarmed_parity = 0;
    bool aborted = false;
    for (int base = 0; base < count && !aborted; base += 32) {
        const int gp = start + base + lane;
        int id = 0, rows = 0, qkv_b = -1, pos = 0;
        if (gp < end) {
            const int b = find_seq(s.seg, B, gp);
            const int i = gp - s.seg[b];
            id = __ldg(p.block_table + (size_t)b * p.bt_stride + i);
            // only the rows older than the T new tokens are read from the cache
            rows = min(kPage, max(0, (s.lens[b] - T) - kPage * i));
            if (gp == start || i == 0) {
                qkv_b = b;
                pos = first_position(p, b, s.lens[b], T);
            }
        }
        const int n = min(32, count - base);
        for (int kk = 0; kk < n; ++kk) {
            const int page_id = __shfl_sync(kFull, id, kk);
            const int page_rows = __shfl_sync(kFull, rows, kk);
            const int seq_qkv = __shfl_sync(kFull, qkv_b, kk);
            const int seq_pos = __shfl_sync(kFull, pos, kk);
            int ok = 1;
            uint32_t kv_bytes = 0;
            if (lane == 0) {
                if (Lay::kDirectQkv && seq_qkv >= 0) {
                    // the consumers read these rows from global memory: have them in L2 first
                    bulk_prefetch_l2(p.qkv + token_row(p, seq_qkv, 0) * Lay::kQkvW, (uint32_t)Lay::kSlotBytes);
                } else if (seq_qkv >= 0) {
                    // the qkv slot frees once every consumer has formed q from it
                    ok = mbar_try_wait(s.qkv_empty, qphase ^ 1u) ||
                         mbar_wait(s.qkv_empty, qphase ^ 1u, p.timeout_ns, s.abort_flag);
                    if (ok) {
                        *s.qkv_pos = seq_pos;
                        const uint16_t* src = p.qkv + token_row(p, seq_qkv, 0) * Lay::kQkvW;
                        mbar_arrive_expect_tx(s.qkv_full, (uint32_t)Lay::kStagedBytes);
                        if constexpr (Lay::kStageQOnly) {
                            // each token's q part; the k and v words to L2 for the appending CTA
#pragma unroll
                            for (int u = 0; u < T; ++u)
                                bulk_g2s(s.qkv + u * Lay::kQRowBytes, src + (size_t)u * Lay::kQkvW,
                                         (uint32_t)Lay::kQRowBytes, s.qkv_full);
                            bulk_prefetch_l2(src, (uint32_t)Lay::kSlotBytes);
                        } else {
                            bulk_g2s(s.qkv, src, (uint32_t)Lay::kSlotBytes, s.qkv_full);
                        }
                        qarmed = true;
                        qarmed_parity = qphase;
                        qphase ^= 1u;
                    }
                }
                if (ok)
                    ok = mbar_try_wait(&s.empty_bar[slot], phase ^ 1u) ||
                         mbar_wait(&s.empty_bar[slot], phase ^ 1u, p.timeout_ns, s.abort_flag);
                if (ok) {
                    const bool bad = page_id < 0 || page_id >= p.num_pages;
                    s.meta[slot].page = page_id;
                    s.meta[slot].bad = bad ? 1 : 0;
                    if (bad) record_error(p.status, QDA_ERR_BOUNDS);
                    kv_bytes = bad ? 0u : (uint32_t)page_rows * kRowBytes;
                    if (kv_bytes != 0) {
                        mbar_arrive_expect_tx(&s.full_bar[slot], 2u * kv_bytes);
                        armed |= 1u << slot;
                        armed_parity = (armed_parity & ~(1u << slot)) | (phase << slot);
                    } else {
                        mbar_arrive(&s.full_bar[slot]);
                    }
                } else {
                    *s.abort_flag = 1;
                    record_error(p.status, QDA_ERR_TIMEOUT);
                }
            }
            ok = __shfl_sync(kFull, ok, 0);
            if (!ok) {
                aborted = true;
                break;
            }
            // one row copy per lane: lanes 0..15 the K rows, 16..31 the V rows
            kv_bytes = __shfl_sync(kFull, kv_bytes, 0);
            if (kv_bytes != 0 && (lane & 15) < page_rows) {
                const int r = lane & 15;
                const bool is_v = lane >= 16;
                uint8_t* dst = s.stages + slot * kStageBytes + (is_v ? kStageV : kStageK) + r * kRowPitch;
                const uint8_t* src = reinterpret_cast<const uint8_t*>(is_v ? p.v_cache : p.k_cache) +
                                     (size_t)page_id * kPageBytes + (size_t)r * kRowBytes;
                bulk_g2s(dst, src, (uint32_t)kRowBytes, &s.full_bar[slot]);
            }
            if (++slot == kStages) {
                slot = 0;
                phase ^= 1u;
            }
        }
    }
    if (lane == 0 && *s.abort_flag != 0) {
        for (int k = 0; k < kStages; ++k)
            if (armed & (1u << k)) (void)mbar_wait(&s.full_bar[k], (armed_parity >> k) & 1u, p.timeout_ns, nullptr);
        if (qarmed) (void)mbar_wait(s.qkv_full, qarmed_parity, p.timeout_ns, nullptr);
    }
}

// ---------------------------------------------------------------------------
// Consumer warps.

// x - n * 2*pi for the integer n nearest x / (2*pi), in double: 2*pi is split
// into a 32-bit head (n * head and x - n * head are exact for the |x| < 2^20
// here) and its double remainder, so the result carries about one ulp of x.
__device__ __forceinline__ double reduce_two_pi(double x) {
    constexpr double kTwoPiHi = 6.2831853069365025;      // 2*pi rounded to 32 significant bits
    constexpr double kTwoPiLo = 2.430840202602477e-10;   // 2*pi - kTwoPiHi
    constexpr double kInvTwoPi = 0.15915494309189535;
    const double n = rint(x * kInvTwoPi);
    return fma(-n, kTwoPiLo, fma(-n, kTwoPiHi, x));
}

template <int T>
struct State {
    uint32_t qa[8][4];    // A fragments of q per 16-dim step: rows r (bf16 of q) and r+8 (remainder)
    float o[16][4];       // value accumulators: 16 tiles of 8 dims, rows r and r+8
    float m;              // running max of row r (log2 units)
    float lsum;           // partial softmax sum of this lane's tokens
    uint32_t k_lo[T], k_hi[T], v_lo[T], v_hi[T];   // this lane's words of the appended k/v rows
};

// Start a sequence piece from its T qkv rows (staged in shared memory, or
// their q parts staged and the rest read from global memory): q of row r = lane/4 (new
// token r / G, head G*j + r % G) at dims 8m + 2t, 8m + 2t + 1 (t = lane%4,
// m = 0..15), i.e. both halves of the rotation pairs 8m' + 2t + e, m' < 8.
// Lane l forms the first new token's angles of pairs 2l, 2l+1 (reduced
// modulo 2*pi in double, then float sin/cos); a lane fetches those of its
// pairs by shuffles and turns them to its row's token tt by the tabled
// rotation of tt positions. When this CTA holds a page with new tokens, their
// k is formed in double. Every load from the rows is issued first, so that
// rows read from global memory cost one round trip.
template <int G, int T>
__device__ __forceinline__ void begin_sequence(const Params& p, const Shared& s, const uint8_t* qrows, int q_stride,
                                               const uint8_t* rows, int pos0, int j, int lane, bool appends,
                                               State<T>& st) {
    using Lay = Layout<G, T>;
    const int r = lane >> 2, t = lane & 3;
    const bool active = r < Lay::kRows;
    const int tt = active ? r / G : 0;          // this row's new token
    const int head = G * j + (active ? r % G : 0);

    // the loads: this row's q words (token u's q part at qrows + u * q_stride),
    // and the new tokens' k and v words (from the whole rows `rows`)
    const uint32_t* xq = reinterpret_cast<const uint32_t*>(qrows + tt * q_stride + head * (kHeadDim * 2));
    uint32_t xw[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) xw[m] = xq[4 * m + t];
    uint32_t kx_lo[T], kx_hi[T];
    if (appends) {
#pragma unroll
        for (int u = 0; u < T; ++u) {
            const uint8_t* row = rows + u * Lay::kQkvBytes;
            const uint32_t* xk = reinterpret_cast<const uint32_t*>(row + (Lay::kHq + j) * (kHeadDim * 2));
            const uint32_t* xv = reinterpret_cast<const uint32_t*>(row + (Lay::kHq + kNumKvHeads + j) * (kHeadDim * 2));
            kx_lo[u] = xk[lane];
            kx_hi[u] = xk[32 + lane];
            st.v_lo[u] = xv[lane];
            st.v_hi[u] = xv[32 + lane];
        }
    }

    // the first new token's angles of pairs 2*lane + e
    float c0[2], s0[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const double ang = (double)pos0 * s.inv_freq[2 * lane + e];
        sincosf((float)reduce_two_pi(ang), &s0[e], &c0[e]);
    }
    const uint32_t* gq = reinterpret_cast<const uint32_t*>(s.gains);
    float ss = 0.f;
#pragma unroll
    for (int m = 0; m < 16; ++m) ss = fmaf(bf_lo(xw[m]), bf_lo(xw[m]), fmaf(bf_hi(xw[m]), bf_hi(xw[m]), ss));
    ss += __shfl_xor_sync(kFull, ss, 1);
    ss += __shfl_xor_sync(kFull, ss, 2);
    const float inv_r = rsqrtf(ss * (1.f / 128.f) + (float)p.rms_eps);
    const float scale = (float)kQScale;
#pragma unroll
    for (int mp = 0; mp < 8; ++mp) {
        float qa[2], qb[2];
        const uint32_t wlo = gq[4 * mp + t], whi = gq[32 + 4 * mp + t];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            // the angle of pair 8*mp + 2t + e at the first new token, then at this row's
            float cs = __shfl_sync(kFull, c0[e], 4 * mp + t);
            float sn = __shfl_sync(kFull, s0[e], 4 * mp + t);
            if (T > 1 && tt > 0) {
                const float2 rt = s.rot[(tt - 1) * kRotStride + 8 * mp + 2 * t + e];
                const float c = fmaf(cs, rt.x, -sn * rt.y);
                sn = fmaf(sn, rt.x, cs * rt.y);
                cs = c;
            }
            const float ya = (e ? bf_hi(xw[mp]) : bf_lo(xw[mp])) * inv_r * (e ? bf_hi(wlo) : bf_lo(wlo));
            const float yb = (e ? bf_hi(xw[mp + 8]) : bf_lo(xw[mp + 8])) * inv_r * (e ? bf_hi(whi) : bf_lo(whi));
            qa[e] = fmaf(ya, cs, -yb * sn) * scale;   // dim 8*mp + 2t + e
            qb[e] = fmaf(yb, cs, ya * sn) * scale;    // dim 64 + 8*mp + 2t + e
        }
        uint16_t ha0, la0, ha1, la1, hb0, lb0, hb1, lb1;
        split_bf16(qa[0], ha0, la0);
        split_bf16(qa[1], ha1, la1);
        split_bf16(qb[0], hb0, lb0);
        split_bf16(qb[1], hb1, lb1);
        const int part = (mp & 1) ? 2 : 0;   // dims 16s + 2t (+1) or 16s + 8 + 2t (+1)
        st.qa[mp >> 1][part] = active ? ((uint32_t)ha1 << 16 | ha0) : 0u;
        st.qa[mp >> 1][part + 1] = active ? ((uint32_t)la1 << 16 | la0) : 0u;
        st.qa[4 + (mp >> 1)][part] = active ? ((uint32_t)hb1 << 16 | hb0) : 0u;
        st.qa[4 + (mp >> 1)][part + 1] = active ? ((uint32_t)lb1 << 16 | lb0) : 0u;
    }

    if (appends) {
        // lane l: dims 2l, 2l+1 (word l of the head) and 64+2l, 65+2l (word 32+l), all in double.
        // The angle of token u is pos0*f + u*f: token 0's sine and cosine (argument
        // reduced modulo 2*pi first), then u rotations by the tabled step f (error
        // ~u ulp of double, far below k's bf16 rounding).
        const uint32_t* gk = reinterpret_cast<const uint32_t*>(s.gains + kHeadDim);
        const uint32_t wk_lo = gk[lane], wk_hi = gk[32 + lane];
        double sn0, cs0, sn1, cs1;
        sincos(reduce_two_pi((double)pos0 * s.inv_freq[2 * lane]), &sn0, &cs0);
        sincos(reduce_two_pi((double)pos0 * s.inv_freq[2 * lane + 1]), &sn1, &cs1);
        const double2 st0 = s.step[2 * lane], st1 = s.step[2 * lane + 1];
        double ssq[T];
        double a0[T], a1[T], b0[T], b1[T];
#pragma unroll
        for (int u = 0; u < T; ++u) {
            a0[u] = bf_to_d(kx_lo[u] & 0xFFFFu);
            a1[u] = bf_to_d(kx_lo[u] >> 16);
            b0[u] = bf_to_d(kx_hi[u] & 0xFFFFu);
            b1[u] = bf_to_d(kx_hi[u] >> 16);
            ssq[u] = a0[u] * a0[u] + a1[u] * a1[u] + b0[u] * b0[u] + b1[u] * b1[u];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int u = 0; u < T; ++u) ssq[u] += __shfl_xor_sync(kFull, ssq[u], off);
#pragma unroll
        for (int u = 0; u < T; ++u) {
            const double inv_rr = 1.0 / sqrt(ssq[u] / 128.0 + p.rms_eps);
            const double x0 = a0[u] * inv_rr * bf_to_d(wk_lo & 0xFFFFu);
            const double x1 = a1[u] * inv_rr * bf_to_d(wk_lo >> 16);
            const double y0 = b0[u] * inv_rr * bf_to_d(wk_hi & 0xFFFFu);
            const double y1 = b1[u] * inv_rr * bf_to_d(wk_hi >> 16);
            const double ra0 = x0 * cs0 - y0 * sn0, rb0 = y0 * cs0 + x0 * sn0;
            const double ra1 = x1 * cs1 - y1 * sn1, rb1 = y1 * cs1 + x1 * sn1;
            st.k_lo[u] = d_to_bf(ra0) | (d_to_bf(ra1) << 16);
            st.k_hi[u] = d_to_bf(rb0) | (d_to_bf(rb1) << 16);
            if (u + 1 < T) {   // advance both angles by one position
                const double c0n = cs0 * st0.x - sn0 * st0.y, s0n = sn0 * st0.x + cs0 * st0.y;
                const double c1n = cs1 * st1.x - sn1 * st1.y, s1n = sn1 * st1.x + cs1 * st1.y;
                cs0 = c0n; sn0 = s0n; cs1 = c1n; sn1 = s1n;
            }
        }
    }

#pragma unroll
    for (int n = 0; n < 16; ++n)
#pragma unroll
        for (int k = 0; k < 4; ++k) st.o[n][k] = 0.f;
    st.m = -INFINITY;
    st.lsum = 0.f;
}

// Scores, online softmax and value accumulation over one staged page. Unless
// kFullPage, this lane's row sees page tokens 0..limit only (its causal
// limit, which also excludes rows past the sequence).
template <int G, int T, bool kFullPage>
__device__ __forceinline__ void attend_page(const uint8_t* stage, int limit, int j, int lane, State<T>& st) {
    const int r = lane >> 2, t = lane & 3;
    // K rows as the column-major B operand: matrix l/8 = (tokens 0-7 | 8-15) x (dims +0 | +8)
    const uint32_t kaddr = smem_addr(stage + kStageK) + j * (kHeadDim * 2) +
                           ((lane & 7) + ((lane >> 4) << 3)) * kRowPitch + ((lane >> 3) & 1) * 16;
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kaddr + s * 32, b0, b1, b2, b3);
        mma_bf16_16816(c0, st.qa[s], b0, b1);
        mma_bf16_16816(c1, st.qa[s], b2, b3);
    }
    // row r's scores at tokens 2t, 2t+1, 8+2t, 9+2t (accumulator row r plus row r+8)
    float sc[4] = {c0[0] + c0[2], c0[1] + c0[3], c1[0] + c1[2], c1[1] + c1[3]};
    if (!kFullPage) {
        sc[0] = (2 * t <= limit) ? sc[0] : -INFINITY;
        sc[1] = (2 * t + 1 <= limit) ? sc[1] : -INFINITY;
        sc[2] = (8 + 2 * t <= limit) ? sc[2] : -INFINITY;
        sc[3] = (9 + 2 * t <= limit) ? sc[3] : -INFINITY;
    }
    float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
    const bool grow = mx > st.m + kRescaleThreshold;
    if (__any_sync(kFull, grow)) {
        const float nm = grow ? mx : st.m;
        const float a = grow ? exp2_approx(st.m - nm) : 1.f;   // exp2(-inf) = 0 on the first page
#pragma unroll
        for (int n = 0; n < 16; ++n)
#pragma unroll
            for (int k = 0; k < 4; ++k) st.o[n][k] *= a;
        st.lsum *= a;
        st.m = nm;
    }
    float pr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        pr[i] = (sc[i] == -INFINITY || r >= Layout<G, T>::kRows) ? 0.f : exp2_approx(sc[i] - st.m);
    st.lsum += (pr[0] + pr[1]) + (pr[2] + pr[3]);
    uint32_t pa[4];
    {
        uint16_t h0, l0, h1, l1, h2, l2, h3, l3;
        split_bf16(pr[0], h0, l0);
        split_bf16(pr[1], h1, l1);
        split_bf16(pr[2], h2, l2);
        split_bf16(pr[3], h3, l3);
        pa[0] = (uint32_t)h1 << 16 | h0;   // row r, tokens 2t, 2t+1
        pa[1] = (uint32_t)l1 << 16 | l0;   // row r+8
        pa[2] = (uint32_t)h3 << 16 | h2;   // row r, tokens 8+2t, 9+2t
        pa[3] = (uint32_t)l3 << 16 | l2;   // row r+8
    }
    // V rows as the column-major B operand (transposed load): matrix l/8 =
    // (tokens 0-7 | 8-15) x (dims +0 | +8)
    const uint32_t vaddr = smem_addr(stage + kStageV) + j * (kHeadDim * 2) +
                           ((lane & 7) + (((lane >> 3) & 1) << 3)) * kRowPitch + ((lane >> 4) & 1) * 16;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_trans(vaddr + u * 32, b0, b1, b2, b3);
        mma_bf16_16816(st.o[2 * u], pa, b0, b1);
        mma_bf16_16816(st.o[2 * u + 1], pa, b2, b3);
    }
}

__device__ __forceinline__ bool wait_full(const Params& p, const Shared& s, uint64_t* bar, uint32_t phase, int lane) {
    bool ok = mbar_try_wait(bar, phase);
    if (__all_sync(kFull, ok)) return true;
    ok = ok || mbar_wait(bar, phase, p.timeout_ns, s.abort_flag);
    ok = __all_sync(kFull, ok || mbar_try_wait(bar, phase));
    if (!ok && lane == 0) {
        *s.abort_flag = 1;
        record_error(p.status, QDA_ERR_TIMEOUT);
    }
    return ok;
}

// Attend over the staged page in `slot`: page i of a sequence of length L
// whose last T slots are the new tokens. New tokens on this page are written
// to the cache and patched into the staged page first.
template <int G, int T>
__device__ __forceinline__ void consume_page(const Params& p, const Shared& s, int slot, int i, int L, int j,
                                             int lane, State<T>& st) {
    uint8_t* stage = s.stages + slot * kStageBytes;
    const int first_new = L - T;                    // slot of the first new token
    const int ntok = min(kPage, L - kPage * i);     // rows of this page inside the sequence
    if (s.meta[slot].bad == 0) {
        if (kPage * i + kPage > first_new) {
            // new tokens on this page: to the cache and into the staged page
            const int page = s.meta[slot].page;
#pragma unroll
            for (int u = 0; u < T; ++u) {
                const int row = first_new + u - kPage * i;
                if (row < 0 || row >= kPage) continue;
                const size_t off =
                    (size_t)page * (kPageBytes / 2) + (size_t)row * (kRowBytes / 2) + (size_t)j * kHeadDim;
                uint32_t* kd = reinterpret_cast<uint32_t*>(p.k_cache + off);
                uint32_t* vd = reinterpret_cast<uint32_t*>(p.v_cache + off);
                kd[lane] = st.k_lo[u];
                kd[32 + lane] = st.k_hi[u];
                vd[lane] = st.v_lo[u];
                vd[32 + lane] = st.v_hi[u];
                uint32_t* kr = reinterpret_cast<uint32_t*>(stage + kStageK + row * kRowPitch + j * kHeadDim * 2);
                uint32_t* vr = reinterpret_cast<uint32_t*>(stage + kStageV + row * kRowPitch + j * kHeadDim * 2);
                kr[lane] = st.k_lo[u];
                kr[32 + lane] = st.k_hi[u];
                vr[lane] = st.v_lo[u];
                vr[32 + lane] = st.v_hi[u];
            }
            // rows after the sequence hold stale bytes; the value product would
            // turn a stale NaN into NaN even at probability 0, so clear them
            for (int rr = ntok; rr < kPage; ++rr) {
                uint32_t* z = reinterpret_cast<uint32_t*>(stage + kStageV + rr * kRowPitch + j * kHeadDim * 2);
                z[lane] = 0u;
                z[32 + lane] = 0u;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
        }
        // this lane's row (new token tt) sees slots <= first_new + tt
        const int r = lane >> 2;
        const int tt = r < Layout<G, T>::kRows ? r / G : 0;
        const int limit = first_new + tt - kPage * i;
        if (first_new - kPage * i >= kPage) attend_page<G, T, true>(stage, limit, j, lane, st);
        else attend_page<G, T, false>(stage, limit, j, lane, st);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty_bar[slot]);
}

// End of a sequence piece: o directly when the piece is the whole sequence,
// else this piece's partial at scratch slot blockIdx.x + b, row t*Hq + head of
// the slot's kPartRows.
template <int G, int T>
__device__ __forceinline__ bool finish_piece(const Params& p, const Shared& s, int b, int j, int lane, int per_cta,
                                             State<T>& st) {
    using Lay = Layout<G, T>;
    const int r = lane >> 2, t = lane & 3;
    float l = st.lsum;
    l += __shfl_xor_sync(kFull, l, 1);
    l += __shfl_xor_sync(kFull, l, 2);
    const int part_first = s.seg[b] / per_cta;
    const int part_last = (s.seg[b + 1] - 1) / per_cta;
    if (r >= Lay::kRows) return part_first != part_last;
    const int tt = r / G;
    const int head = G * j + r % G;
    if (part_first == part_last) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint32_t* dst = reinterpret_cast<uint32_t*>(p.o + (token_row(p, b, tt) * Lay::kHq + head) * kHeadDim);
#pragma unroll
        for (int n = 0; n < 16; ++n)
            dst[4 * n + t] = pack_bf2((st.o[n][0] + st.o[n][2]) * inv, (st.o[n][1] + st.o[n][3]) * inv);
        return false;
    }
    const size_t prow = part_row<G, T>(j, (int)blockIdx.x + b, r);
    float2* pa = reinterpret_cast<float2*>(p.part_acc + prow * kHeadDim);
#pragma unroll
    for (int n = 0; n < 16; ++n) __stcg(pa + 4 * n + t, make_float2(st.o[n][0] + st.o[n][2], st.o[n][1] + st.o[n][3]));
    if (t == 0) __stcg(p.part_ml + prow, make_float2(st.m, l));
    return true;
}

// ---------------------------------------------------------------------------
// Wide instances: 9 to 16 query rows per kv head, one row per accumulator row.

struct WState {
    uint32_t qa[8][4];    // A fragments of q per 16-dim step: rows g (regs 0, 2) and g + 8 (regs 1, 3), bf16
    float o[16][4];       // value accumulators: 16 tiles of 8 dims, rows g (0, 1) and g + 8 (2, 3)
    float m[2];           // running max of rows g and g + 8 (log2 units)
    float lsum[2];        // partial softmax sums of this lane's tokens, rows g and g + 8
};

// The new tokens' k for kv head j, normed and rotated in double and rounded
// once to bf16, into this warp's words of s.new_k. Lane l handles dims 2l,
// 2l+1 (word l) and 64+2l, 65+2l (word 32+l); the angle of token u is token
// 0's rotated by the step u times (error ~u ulp of double, far below k's bf16
// rounding).
template <int G, int T>
__device__ __forceinline__ void form_new_k(const Params& p, const Shared& s, const uint8_t* rows, int pos0, int j,
                                           int lane) {
    using Lay = Layout<G, T>;
    const uint32_t* gk = reinterpret_cast<const uint32_t*>(s.gains + kHeadDim);
    const uint32_t wk_lo = gk[lane], wk_hi = gk[32 + lane];
    double sn0, cs0, sn1, cs1;
    sincos(reduce_two_pi((double)pos0 * s.inv_freq[2 * lane]), &sn0, &cs0);
    sincos(reduce_two_pi((double)pos0 * s.inv_freq[2 * lane + 1]), &sn1, &cs1);
    const double dc0 = s.step[2 * lane].x, ds0 = s.step[2 * lane].y;
    const double dc1 = s.step[2 * lane + 1].x, ds1 = s.step[2 * lane + 1].y;
    uint32_t* dst = s.new_k + (size_t)j * T * 64;
    // every token's words first (one round trip to L2), then the arithmetic
    uint32_t xlo[T], xhi[T];
#pragma unroll
    for (int u = 0; u < T; ++u) {
        const uint32_t* xk =
            reinterpret_cast<const uint32_t*>(rows + u * Lay::kQkvBytes + (Lay::kHq + j) * (kHeadDim * 2));
        xlo[u] = xk[lane];
        xhi[u] = xk[32 + lane];
    }
#pragma unroll
    for (int u = 0; u < T; ++u) {
        double a0 = bf_to_d(xlo[u] & 0xFFFFu), a1 = bf_to_d(xlo[u] >> 16);
        double b0 = bf_to_d(xhi[u] & 0xFFFFu), b1 = bf_to_d(xhi[u] >> 16);
        const double inv_rr = 1.0 / sqrt(warp_sum(a0 * a0 + a1 * a1 + b0 * b0 + b1 * b1) / 128.0 + p.rms_eps);
        a0 = a0 * inv_rr * bf_to_d(wk_lo & 0xFFFFu);
        a1 = a1 * inv_rr * bf_to_d(wk_lo >> 16);
        b0 = b0 * inv_rr * bf_to_d(wk_hi & 0xFFFFu);
        b1 = b1 * inv_rr * bf_to_d(wk_hi >> 16);
        const double ra0 = a0 * cs0 - b0 * sn0, rb0 = b0 * cs0 + a0 * sn0;
        const double ra1 = a1 * cs1 - b1 * sn1, rb1 = b1 * cs1 + a1 * sn1;
        dst[u * 64 + lane] = d_to_bf(ra0) | (d_to_bf(ra1) << 16);
        dst[u * 64 + 32 + lane] = d_to_bf(rb0) | (d_to_bf(rb1) << 16);
        const double c0n = cs0 * dc0 - sn0 * ds0, s0n = sn0 * dc0 + cs0 * ds0;   // one position on
        const double c1n = cs1 * dc1 - sn1 * ds1, s1n = sn1 * dc1 + cs1 * ds1;
        cs0 = c0n; sn0 = s0n; cs1 = c1n; sn1 = s1n;
    }
    __syncwarp();
}

// Start a sequence piece: q of rows g and g + 8 (g = lane/4; row r is new
// token r / G, head G*j + r % G) at dims 8m + 2t, 8m + 2t + 1 (t = lane%4),
// normed and rotated in float as in begin_sequence, then rounded to bf16.
template <int G, int T>
__device__ __forceinline__ void begin_sequence_wide(const Params& p, const Shared& s, const uint8_t* rows, int pos0,
                                                    int j, int lane, bool appends, WState& st) {
    using Lay = Layout<G, T>;
    if (appends) form_new_k<G, T>(p, s, rows, pos0, j, lane);
    const int g = lane >> 2, t = lane & 3;
    float c0[2], s0[2];   // the first new token's angles of pairs 2*lane + e
#pragma unroll
    for (int e = 0; e < 2; ++e) sincosf((float)reduce_two_pi((double)pos0 * s.inv_freq[2 * lane + e]), &s0[e], &c0[e]);
    const uint32_t* gq = reinterpret_cast<const uint32_t*>(s.gains);
    const float scale = (float)kQScale;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int r = g + 8 * h;
        const bool active = r < Lay::kRows;
        const int tt = active ? r / G : 0;
        const int head = G * j + (active ? r % G : 0);
        const uint32_t* xq = reinterpret_cast<const uint32_t*>(rows + tt * Lay::kQkvBytes + head * (kHeadDim * 2));
        uint32_t xw[16];
        float ss = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            xw[m] = xq[4 * m + t];
            ss = fmaf(bf_lo(xw[m]), bf_lo(xw[m]), fmaf(bf_hi(xw[m]), bf_hi(xw[m]), ss));
        }
        ss += __shfl_xor_sync(kFull, ss, 1);
        ss += __shfl_xor_sync(kFull, ss, 2);
        const float inv_r = rsqrtf(ss * (1.f / 128.f) + (float)p.rms_eps);
#pragma unroll
        for (int mp = 0; mp < 8; ++mp) {
            float qa[2], qb[2];
            const uint32_t wlo = gq[4 * mp + t], whi = gq[32 + 4 * mp + t];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                // the angle of pair 8*mp + 2t + e at the first new token, then at this row's
                float cs = __shfl_sync(kFull, c0[e], 4 * mp + t);
                float sn = __shfl_sync(kFull, s0[e], 4 * mp + t);
                if (tt > 0) {
                    const float2 rt = s.rot[(tt - 1) * kRotStride + 8 * mp + 2 * t + e];
                    const float c = fmaf(cs, rt.x, -sn * rt.y);
                    sn = fmaf(sn, rt.x, cs * rt.y);
                    cs = c;
                }
                const float ya = (e ? bf_hi(xw[mp]) : bf_lo(xw[mp])) * inv_r * (e ? bf_hi(wlo) : bf_lo(wlo));
                const float yb = (e ? bf_hi(xw[mp + 8]) : bf_lo(xw[mp + 8])) * inv_r * (e ? bf_hi(whi) : bf_lo(whi));
                qa[e] = fmaf(ya, cs, -yb * sn) * scale;   // dim 8*mp + 2t + e
                qb[e] = fmaf(yb, cs, ya * sn) * scale;    // dim 64 + 8*mp + 2t + e
            }
            const int part = ((mp & 1) ? 2 : 0) + h;   // dims 16s + 2t (+1) or 16s + 8 + 2t (+1); row g or g + 8
            st.qa[mp >> 1][part] = active ? pack_bf2(qa[0], qa[1]) : 0u;
            st.qa[4 + (mp >> 1)][part] = active ? pack_bf2(qb[0], qb[1]) : 0u;
        }
    }
#pragma unroll
    for (int n = 0; n < 16; ++n)
#pragma unroll
        for (int k = 0; k < 4; ++k) st.o[n][k] = 0.f;
    st.m[0] = st.m[1] = -INFINITY;
    st.lsum[0] = st.lsum[1] = 0.f;
}

// Scores, online softmax and value accumulation over one staged page for rows
// g and g + 8, which see page tokens up to lim0 and lim1 (unless kFullPage).
// The probabilities enter the value product as bf16, and the sums add the
// same rounded values, so o stays a convex combination of the v rows.
template <int G, int T, bool kFullPage>
__device__ __forceinline__ void attend_page_wide(const uint8_t* stage, int lim0, int lim1, int j, int lane,
                                                 WState& st) {
    using Lay = Layout<G, T>;
    const int g = lane >> 2, t = lane & 3;
    const bool act0 = g < Lay::kRows, act1 = g + 8 < Lay::kRows;
    const uint32_t kaddr = smem_addr(stage + kStageK) + j * (kHeadDim * 2) +
                           ((lane & 7) + ((lane >> 4) << 3)) * kRowPitch + ((lane >> 3) & 1) * 16;
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kaddr + s * 32, b0, b1, b2, b3);
        mma_bf16_16816(c0, st.qa[s], b0, b1);
        mma_bf16_16816(c1, st.qa[s], b2, b3);
    }
    // rows g and g + 8 at page tokens 2t, 2t+1, 8+2t, 9+2t
    float s0[4] = {c0[0], c0[1], c1[0], c1[1]};
    float s1[4] = {c0[2], c0[3], c1[2], c1[3]};
    if (!kFullPage) {
        const int tok[4] = {2 * t, 2 * t + 1, 8 + 2 * t, 9 + 2 * t};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            s0[i] = tok[i] <= lim0 ? s0[i] : -INFINITY;
            s1[i] = tok[i] <= lim1 ? s1[i] : -INFINITY;
        }
    }
    float mx0 = fmaxf(fmaxf(s0[0], s0[1]), fmaxf(s0[2], s0[3]));
    float mx1 = fmaxf(fmaxf(s1[0], s1[1]), fmaxf(s1[2], s1[3]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, 2));
    const bool grow0 = mx0 > st.m[0] + kRescaleThreshold;
    const bool grow1 = mx1 > st.m[1] + kRescaleThreshold;
    if (__any_sync(kFull, grow0 || grow1)) {
        const float n0 = grow0 ? mx0 : st.m[0], n1 = grow1 ? mx1 : st.m[1];
        const float a0 = grow0 ? exp2_approx(st.m[0] - n0) : 1.f;   // exp2(-inf) = 0 on the first page
        const float a1 = grow1 ? exp2_approx(st.m[1] - n1) : 1.f;
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            st.o[n][0] *= a0;
            st.o[n][1] *= a0;
            st.o[n][2] *= a1;
            st.o[n][3] *= a1;
        }
        st.lsum[0] *= a0;
        st.lsum[1] *= a1;
        st.m[0] = n0;
        st.m[1] = n1;
    }
    float p0[4], p1[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        p0[i] = (s0[i] == -INFINITY || !act0) ? 0.f : exp2_approx(s0[i] - st.m[0]);
        p1[i] = (s1[i] == -INFINITY || !act1) ? 0.f : exp2_approx(s1[i] - st.m[1]);
    }
    uint32_t pa[4];
    pa[0] = pack_bf2(p0[0], p0[1]);   // row g, tokens 2t, 2t+1
    pa[1] = pack_bf2(p1[0], p1[1]);   // row g + 8
    pa[2] = pack_bf2(p0[2], p0[3]);   // row g, tokens 8+2t, 9+2t
    pa[3] = pack_bf2(p1[2], p1[3]);   // row g + 8
    st.lsum[0] += (bf_lo(pa[0]) + bf_hi(pa[0])) + (bf_lo(pa[2]) + bf_hi(pa[2]));
    st.lsum[1] += (bf_lo(pa[1]) + bf_hi(pa[1])) + (bf_lo(pa[3]) + bf_hi(pa[3]));
    const uint32_t vaddr = smem_addr(stage + kStageV) + j * (kHeadDim * 2) +
                           ((lane & 7) + (((lane >> 3) & 1) << 3)) * kRowPitch + ((lane >> 4) & 1) * 16;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_trans(vaddr + u * 32, b0, b1, b2, b3);
        mma_bf16_16816(st.o[2 * u], pa, b0, b1);
        mma_bf16_16816(st.o[2 * u + 1], pa, b2, b3);
    }
}

template <int G, int T>
__device__ __forceinline__ void consume_page_wide(const Params& p, const Shared& s, int slot, int i, int L, int j,
                                                  int lane, const uint8_t* rows, WState& st) {
    using Lay = Layout<G, T>;
    uint8_t* stage = s.stages + slot * kStageBytes;
    const int first_new = L - T;                    // slot of the first new token
    const int ntok = min(kPage, L - kPage * i);     // rows of this page inside the sequence
    if (s.meta[slot].bad == 0) {
        if (kPage * i + kPage > first_new) {
            // the new tokens on this page: k (formed when the sequence started)
            // and v bits, to the cache and into the staged page
            const int page = s.meta[slot].page;
            const int u_lo = max(0, kPage * i - first_new), u_hi = min(T, kPage * i + kPage - first_new);
            const uint32_t* nk = s.new_k + (size_t)j * T * 64;
            // the v words of every token on the page first (one round trip to L2)
            uint32_t vw_lo[T], vw_hi[T];
#pragma unroll
            for (int u = 0; u < T; ++u) {
                if (u < u_lo || u >= u_hi) continue;
                const uint32_t* xv = reinterpret_cast<const uint32_t*>(
                    rows + u * Lay::kQkvBytes + (Lay::kHq + kNumKvHeads + j) * (kHeadDim * 2));
                vw_lo[u] = xv[lane];
                vw_hi[u] = xv[32 + lane];
            }
#pragma unroll
            for (int u = 0; u < T; ++u) {
                if (u < u_lo || u >= u_hi) continue;
                const uint32_t k_lo = nk[u * 64 + lane], k_hi = nk[u * 64 + 32 + lane];
                const uint32_t v_lo = vw_lo[u], v_hi = vw_hi[u];
                const int r = first_new + u - kPage * i;
                const size_t off =
                    (size_t)page * (kPageBytes / 2) + (size_t)r * (kRowBytes / 2) + (size_t)j * kHeadDim;
                uint32_t* kd = reinterpret_cast<uint32_t*>(p.k_cache + off);
                uint32_t* vd = reinterpret_cast<uint32_t*>(p.v_cache + off);
                kd[lane] = k_lo;
                kd[32 + lane] = k_hi;
                vd[lane] = v_lo;
                vd[32 + lane] = v_hi;
                uint32_t* kr = reinterpret_cast<uint32_t*>(stage + kStageK + r * kRowPitch + j * kHeadDim * 2);
                uint32_t* vr = reinterpret_cast<uint32_t*>(stage + kStageV + r * kRowPitch + j * kHeadDim * 2);
                kr[lane] = k_lo;
                kr[32 + lane] = k_hi;
                vr[lane] = v_lo;
                vr[32 + lane] = v_hi;
            }
            // rows after the sequence hold stale bytes; a stale NaN would survive a
            // zero probability in the tensor-core sum, so clear them
            for (int rr = ntok; rr < kPage; ++rr) {
                uint32_t* z = reinterpret_cast<uint32_t*>(stage + kStageV + rr * kRowPitch + j * kHeadDim * 2);
                z[lane] = 0u;
                z[32 + lane] = 0u;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
        }
        const int g = lane >> 2;
        const int tt0 = g < Lay::kRows ? g / G : 0;
        const int tt1 = g + 8 < Lay::kRows ? (g + 8) / G : 0;
        const int lim0 = first_new + tt0 - kPage * i, lim1 = first_new + tt1 - kPage * i;
        if (first_new - kPage * i >= kPage) attend_page_wide<G, T, true>(stage, lim0, lim1, j, lane, st);
        else attend_page_wide<G, T, false>(stage, lim0, lim1, j, lane, st);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty_bar[slot]);
}

// End of a sequence piece (wide): o, or the piece's partial, for rows g and g + 8.
template <int G, int T>
__device__ __forceinline__ bool finish_piece_wide(const Params& p, const Shared& s, int b, int j, int lane,
                                                  int per_cta, WState& st) {
    using Lay = Layout<G, T>;
    const int g = lane >> 2, t = lane & 3;
    float l[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l[h] = st.lsum[h];
        l[h] += __shfl_xor_sync(kFull, l[h], 1);
        l[h] += __shfl_xor_sync(kFull, l[h], 2);
    }
    const int part_first = s.seg[b] / per_cta;
    const int part_last = (s.seg[b + 1] - 1) / per_cta;
    const bool split = part_first != part_last;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int r = g + 8 * h;
        if (r >= Lay::kRows) continue;
        const int tt = r / G;
        const int head = G * j + r % G;
        if (!split) {
            const float inv = l[h] > 0.f ? 1.f / l[h] : 0.f;
            uint32_t* dst = reinterpret_cast<uint32_t*>(p.o + (token_row(p, b, tt) * Lay::kHq + head) * kHeadDim);
#pragma unroll
            for (int n = 0; n < 16; ++n) dst[4 * n + t] = pack_bf2(st.o[n][2 * h] * inv, st.o[n][2 * h + 1] * inv);
        } else {
            const size_t prow = part_row<G, T>(j, (int)blockIdx.x + b, r);
            float2* pa = reinterpret_cast<float2*>(p.part_acc + prow * kHeadDim);
#pragma unroll
            for (int n = 0; n < 16; ++n) __stcg(pa + 4 * n + t, make_float2(st.o[n][2 * h], st.o[n][2 * h + 1]));
            if (t == 0) __stcg(p.part_ml + prow, make_float2(st.m[h], l[h]));
        }
    }
    return split;
}

// Consumer warp j of a wide instance: as run_consumer, with the query rows'
// qkv and the new tokens read from global memory.
template <int G, int T>
__device__ __forceinline__ void run_consumer_wide(const Params& p, const Shared& s, int B, int start, int end,
                                                  int per_cta, int warp, int lane) {
    using Lay = Layout<G, T>;
    const int j = warp;
    WState st;
    int b = find_seq(s.seg, B, start);
    int i0 = start - s.seg[b];
    int slot = 0;
    uint32_t phase = 0;
    const int count = end - start;
    int k = 0;
    bool aborted = false;
    while (k < count && !aborted) {
        const int nb = s.seg[b + 1] - s.seg[b];
        const int L = s.lens[b];
        const int n_here = min(nb - i0, count - k);
        const int pos0 = first_position(p, b, L, T);
        const uint8_t* rows = reinterpret_cast<const uint8_t*>(p.qkv + token_row(p, b, 0) * Lay::kQkvW);
        // this CTA appends when it holds a page with one of the new tokens
        const bool appends = s.seg[b] + (L - T) / kPage < end;
        begin_sequence_wide<G, T>(p, s, rows, pos0, j, lane, appends, st);
        for (int u = 0; u < n_here; ++u) {
            if (!wait_full(p, s, &s.full_bar[slot], phase, lane)) {
                aborted = true;
                break;
            }
            consume_page_wide<G, T>(p, s, slot, i0 + u, L, j, lane, rows, st);
            if (++slot == Lay::kStages) {
                slot = 0;
                phase ^= 1u;
            }
        }
        if (aborted) break;
        k += n_here;
        (void)finish_piece_wide<G, T>(p, s, b, j, lane, per_cta, st);
        if (k < count) {
            do { ++b; } while (b < B && s.seg[b + 1] == s.seg[b]);
            i0 = 0;
        }
    }
}

template <int G, int T>
__device__ __forceinline__ void run_consumer(const Params& p, const Shared& s, int B, int start, int end, int per_cta,
                                             int warp, int lane) {
    constexpr int kStages = Layout<G, T>::kStages;
    const int j = warp;
    State<T> st;
#pragma unroll
    for (int u = 0; u < T; ++u) st.k_lo[u] = st.k_hi[u] = st.v_lo[u] = st.v_hi[u] = 0u;
    int b = find_seq(s.seg, B, start);
    int i0 = start - s.seg[b];
    int slot = 0;
    uint32_t phase = 0, qphase = 0;
    const int count = end - start;
    int k = 0;
    bool aborted = false;
    while (k < count && !aborted) {
        const int nb = s.seg[b + 1] - s.seg[b];
        const int L = s.lens[b];
        const int n_here = min(nb - i0, count - k);
        // this CTA appends when it holds a page with one of the new tokens
        const bool appends = s.seg[b] + (L - T) / kPage < end;
        {
            using Lay = Layout<G, T>;
            if (!wait_full(p, s, s.qkv_full, qphase, lane)) {
                aborted = true;
                break;
            }
            const uint8_t* rows = Lay::kStageQOnly
                                      ? reinterpret_cast<const uint8_t*>(p.qkv + token_row(p, b, 0) * Lay::kQkvW)
                                      : s.qkv;
            begin_sequence<G, T>(p, s, s.qkv, Lay::kStageQOnly ? Lay::kQRowBytes : Lay::kQkvBytes, rows,
                                 *s.qkv_pos, j, lane, appends, st);
            __syncwarp();
            if (lane == 0) mbar_arrive(s.qkv_empty);
            qphase ^= 1u;
        }
        for (int u = 0; u < n_here; ++u) {
            if (!wait_full(p, s, &s.full_bar[slot], phase, lane)) {
                aborted = true;
                break;
            }
            consume_page<G, T>(p, s, slot, i0 + u, L, j, lane, st);
            if (++slot == kStages) {
                slot = 0;
                phase ^= 1u;
            }
        }
        if (aborted) break;
        k += n_here;
        (void)finish_piece<G, T>(p, s, b, j, lane, per_cta, st);
        if (k < count) {
            do { ++b; } while (b < B && s.seg[b + 1] == s.seg[b]);
            i0 = 0;
        }
    }
}

template <int G, int T>
__global__ void __launch_bounds__(kThreads, 1) grouped_attention_kernel(const Params p) {
    using Lay = Layout<G, T>;
    constexpr int kStages = Lay::kStages;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    Shared s;
    s.stages = smem;
    s.qkv = smem + Lay::kSmemQkv;
    s.new_k = reinterpret_cast<uint32_t*>(smem + Lay::kSmemNewK);
    s.seg = reinterpret_cast<int*>(smem + Lay::kSmemSeg);
    s.lens = reinterpret_cast<int*>(smem + Lay::kSmemLens);
    s.inv_freq = reinterpret_cast<double*>(smem + Lay::kSmemInvFreq);
    s.step = reinterpret_cast<double2*>(smem + Lay::kSmemStep);
    s.rot = reinterpret_cast<float2*>(smem + Lay::kSmemRot);
    s.gains = reinterpret_cast<const uint16_t*>(smem + Lay::kSmemGains);
    s.meta = reinterpret_cast<volatile StageMeta*>(smem + Lay::kSmemMeta);
    s.qkv_pos = reinterpret_cast<volatile int*>(smem + Lay::kSmemMeta + kStages * 16);
    s.full_bar = reinterpret_cast<uint64_t*>(smem + Lay::kSmemBars);
    s.empty_bar = s.full_bar + kStages;
    s.qkv_full = s.empty_bar + kStages;
    s.qkv_empty = s.qkv_full + 1;
    s.never_bar = s.qkv_empty + 1;
    s.abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kSmemFlags);

    // Launched as a programmatic dependent launch: the prologue below touches
    // no global memory, and griddepcontrol.wait holds until the previous
    // launch on the stream has completed and its writes are visible.
    if (threadIdx.x >= 64 && threadIdx.x < 128) {
        // the frequencies, and the angles every sequence start reuses: one
        // position's step (double, for k) and the offsets of the later new
        // tokens (float, for q); small arguments, so one sincos each
        const int i = threadIdx.x - 64;
        const double f = pow(p.rope_theta, -2.0 * i / 128.0);
        s.inv_freq[i] = f;
        double sn, cs;
        sincos(f, &sn, &cs);
        s.step[i] = make_double2(cs, sn);
#pragma unroll
        for (int u = 1; u < T; ++u) {
            sincos((double)u * f, &sn, &cs);
            s.rot[(u - 1) * kRotStride + i] = make_float2((float)cs, (float)sn);
        }
    }
    if (threadIdx.x == 0) {
        for (int k = 0; k < kStages; ++k) {
            mbar_init(&s.full_bar[k], 1);
            mbar_init(&s.empty_bar[k], kConsumerWarps);
        }
        mbar_init(s.qkv_full, 1);
        mbar_init(s.qkv_empty, kConsumerWarps);
        mbar_init(s.never_bar, 1);
        *s.abort_flag = 0;
        s.seg[0] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    pdl_wait();

    const int B = p.batch;
    for (int b = threadIdx.x; b < B; b += kThreads) {
        // the sequence's length counts its whole block of tok_stride new tokens;
        // this launch sees it without the block's tokens after its own
        const int L_all = p.seq_lens[b];
        const bool ok = L_all >= p.tok_stride && L_all <= p.max_seq_len && L_all <= kPage * p.bt_stride;
        if (!ok && blockIdx.x == 0) record_error(p.status, QDA_ERR_BOUNDS);
        const int L = ok ? L_all - p.len_trim : 0;
        s.lens[b] = L;
        s.seg[b + 1] = ok ? (L + kPage - 1) / kPage : 0;
    }
    if (threadIdx.x < 128) {
        // one 4-byte word per thread (the gain pointers are only 4-byte aligned)
        const uint16_t* src = threadIdx.x < 64 ? p.q_norm_w : p.k_norm_w;
        reinterpret_cast<uint32_t*>(smem + Lay::kSmemGains)[threadIdx.x] =
            *reinterpret_cast<const uint32_t*>(src + 2 * (threadIdx.x & 63));
    }
    __syncthreads();
    if (warp == 0) {  // inclusive scan of the page counts
        int v[8];
        int run = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int idx = 1 + 8 * lane + k;
            run += (idx <= B) ? s.seg[idx] : 0;
            v[k] = run;
        }
        int incl = run;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int t = __shfl_up_sync(kFull, incl, off);
            if (lane >= off) incl += t;
        }
        const int excl = incl - run;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int idx = 1 + 8 * lane + k;
            if (idx <= B) s.seg[idx] = excl + v[k];
        }
    }
    __syncthreads();
    if (blockIdx.x == 0)   // page offsets for the combine launch
        for (int b = threadIdx.x; b <= B; b += kThreads) p.seg[b] = s.seg[b];

    const int total = s.seg[B];
    const int per_cta = (total + (int)gridDim.x - 1) / (int)gridDim.x;
    const int start = (int)blockIdx.x * per_cta;
    const int end = min(start + per_cta, total);
    if (start < end) {
        if (warp == kConsumerWarps) run_producer<G, T>(p, s, B, start, end, lane);
        else if constexpr (Lay::kWide) run_consumer_wide<G, T>(p, s, B, start, end, per_cta, warp, lane);
        else run_consumer<G, T>(p, s, B, start, end, per_cta, warp, lane);
    }
    if ((p.flags & QDA_FLAG_INJECT_WAIT_TIMEOUT) != 0u && blockIdx.x == 0 && warp == 0) {
        if (!mbar_wait(s.never_bar, 0u, p.timeout_ns, nullptr) && lane == 0) record_error(p.status, QDA_ERR_TIMEOUT);
    }
    pdl_launch_dependents();
}

// Combine the partials of one split sequence (blockIdx.x) for the query rows
// of one kv head (blockIdx.y): warp w handles query row w (new token w / G,
// head G*y + w % G), and lane l its dims 4l..4l+3; o = sum_t 2^(m_t - M)
// acc_t / sum_t 2^(m_t - M) l_t with M = max_t m_t (log-sum-exp rule;
// Supported models, "Facts proved about the specs": flashAttn_eq,
// softmax_shift). Sequences held whole by one CTA were written by the first
// launch and are skipped. Spreading the merges over a CTA per (sequence, kv
// head) keeps each SM's share of the partials' reads small.
template <int G, int T>
__global__ void __launch_bounds__(32 * G * T, 1) combine_kernel(const Params p, int main_grid) {
    using Lay = Layout<G, T>;
    pdl_wait();   // the first launch has finished and its writes are visible
    pdl_launch_dependents();   // the next step's attention launch may be scheduled
    const int b = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tt = warp / G;
    const int h = G * blockIdx.y + warp % G;
    const int lo = p.seg[b], hi = p.seg[b + 1], total = p.seg[p.batch];
    if (hi == lo) return;   // a sequence the first launch skipped
    const int per_cta = (total + main_grid - 1) / main_grid;
    const int first = lo / per_cta, n = (hi - 1) / per_cta - first + 1;
    if (n == 1) return;
    const size_t row0 = part_row<G, T>((int)blockIdx.y, first + b, warp);   // piece t at row0 + t*kPartRows
    const float2* ml = p.part_ml + row0;
    float M = -INFINITY;
    for (int t = lane; t < n; t += 32) M = fmaxf(M, __ldcg(ml + (size_t)t * kPartRows).x);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
    const float4* src = reinterpret_cast<const float4*>(p.part_acc + row0 * kHeadDim) + lane;
    constexpr size_t kSlotStride = (size_t)kPartRows * kHeadDim / 4;   // float4 per scratch slot
    float Ls = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int t0 = 0; t0 < n; t0 += 32) {
        float wt = 0.f;
        if (t0 + lane < n) {
            const float2 v = __ldcg(ml + (size_t)(t0 + lane) * kPartRows);
            wt = (v.x == -INFINITY) ? 0.f : exp2_approx(v.x - M);   // a piece whose pages were all skipped
            Ls = fmaf(wt, v.y, Ls);
        }
        const int m = min(32, n - t0);
        for (int u0 = 0; u0 < m; u0 += 8) {
            float4 x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (u0 + u < m) x[u] = __ldcg(src + (size_t)(t0 + u0 + u) * kSlotStride);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float w = __shfl_sync(kFull, wt, (u0 + u) & 31);
                if (u0 + u < m) {
                    acc.x = fmaf(w, x[u].x, acc.x);
                    acc.y = fmaf(w, x[u].y, acc.y);
                    acc.z = fmaf(w, x[u].z, acc.z);
                    acc.w = fmaf(w, x[u].w, acc.w);
                }
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) Ls += __shfl_xor_sync(kFull, Ls, off);
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    uint2 out;
    out.x = pack_bf2(acc.x * inv, acc.y * inv);
    out.y = pack_bf2(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(p.o + (token_row(p, b, tt) * Lay::kHq + h) * kHeadDim)[lane] = out;
}

template <int G, int T>
cudaError_t prepare_one() {
    return cudaFuncSetAttribute(grouped_attention_kernel<G, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Layout<G, T>::kSmemTotal);
}

template <int G, int T>
cudaError_t launch_one(const Params& p, int grid, cudaStream_t stream) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t main = {};
    main.gridDim = dim3((unsigned)grid, 1, 1);
    main.blockDim = dim3(kThreads, 1, 1);
    main.dynamicSmemBytes = Layout<G, T>::kSmemTotal;
    main.stream = stream;
    main.attrs = attr;
    main.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&main, grouped_attention_kernel<G, T>, p);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.batch, (unsigned)kNumKvHeads, 1);
    cfg.blockDim = dim3(32 * G * T, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, combine_kernel<G, T>, p, grid);
}

}  // namespace

// The compiled (G, T) instances: every pair with T*G <= 16 query rows per kv
// head, T = 1 at G = 2 being the 16-head decode kernel's.
#define QDA_GROUPED_INSTANCES(X) \
    X(4, 1) X(5, 1) X(8, 1) X(2, 2) X(2, 3) X(2, 4) X(2, 5) X(2, 6) X(2, 7) X(2, 8) \
    X(4, 2) X(4, 3) X(4, 4) X(5, 2) X(5, 3) X(8, 2)

cudaError_t prepare_grouped() {
    cudaError_t e = cudaSuccess;
#define QDA_PREPARE(G, T) \
    if (e == cudaSuccess) e = prepare_one<G, T>();
    QDA_GROUPED_INSTANCES(QDA_PREPARE)
#undef QDA_PREPARE
    return e;
}

int grouped_max_tokens(int num_q_heads) {
    const int G = num_q_heads / kNumKvHeads;
    int best = 0;
#define QDA_MAX_T(GG, TT) \
    if (G == GG && TT > best) best = TT;
    QDA_GROUPED_INSTANCES(QDA_MAX_T)
#undef QDA_MAX_T
    return G == 2 && best < 1 ? 1 : best;
}

bool grouped_supported(int num_q_heads, int new_tokens) {
    const int G = num_q_heads / kNumKvHeads;
#define QDA_MATCH(GG, TT) \
    if (G == GG && new_tokens == TT) return true;
    QDA_GROUPED_INSTANCES(QDA_MATCH)
#undef QDA_MATCH
    return false;
}

cudaError_t launch_grouped(const Params& p, int grid, cudaStream_t stream) {
    const int G = p.num_q_heads / kNumKvHeads;
#define QDA_LAUNCH(GG, TT) \
    if (G == GG && p.new_tokens == TT) return launch_one<GG, TT>(p, grid, stream);
    QDA_GROUPED_INSTANCES(QDA_LAUNCH)
#undef QDA_LAUNCH
    return cudaErrorInvalidValue;
}

}  // namespace qda
