// Fused Qwen3-0.6B decode-attention step for sm_100a: per-head q/k RMSNorm,
// RoPE, paged KV-cache append and split-KV decodeGQA in one launch.
//
// What is computed (Qwen3-0.6B Model Spec, "Compute-graph nodes"):
//   attn.qk_norm  y = x / sqrt(sum x^2 / 128 + eps) * w, per head, shared gain
//   attn.rope     pairs (i, i+64) rotated by pos * theta^(-2i/128)
//   attn.core     o[b,h] = sum_{s<L_b} softmax_s(<q[b,h], k[b,s,h/2]>/sqrt(128)) v[b,s,h/2]
// plus the append of the new token's k/v at cache slot L_b - 1 (pages of 16
// tokens, "At a glance" shape domain).
//
// Work split. The pages of all sequences, concatenated in batch order, form
// one list of P = sum_b ceil(L_b/16) pages (each page costs the same 64 KiB of
// K+V). CTA g of G takes the contiguous range [g*W, (g+1)*W), W = ceil(P/G),
// so every SM streams the same number of bytes whatever the length mix. A
// range may cut a sequence; each CTA produces one partial (running max, sum,
// un-normalised output) per sequence piece it holds, and the last CTA to
// finish a piece of a cut sequence merges the partials (log-sum-exp combine;
// exact by the online-softmax theorem flashAttn_eq and softmax_shift on the
// Supported models page, "Facts proved about the specs"), bulk-copying them
// into its then idle staging ring so that the merge costs one round trip to
// L2 per 24 pieces rather than one per few pieces. The piece of
// sequence b held by CTA g gets scratch slot g + b; these slots are distinct
// because ranges and sequences are both ordered.
//
// Inside a CTA. Warp 8 is the producer: lane 0 issues one bulk copy of the
// K rows and one of the V rows of a page (up to 32 KiB each, all 8 kv heads)
// into a 3-stage shared-memory ring, completed on an mbarrier; with the first
// page of each sequence piece it also copies that sequence's 8 KiB qkv row,
// so consumers never wait on a global load of their own. Warps 0..7 are
// consumers; warp j serves kv head j and both query heads 2j, 2j+1 that read
// it (nnterp qwen3, "Grouped-query attention"), so every K/V byte is read from
// HBM once. Lane (grp = lane/8, c = lane%8) owns head dims [8c, 8c+8) and
// [64+8c, 64+8c+8) -- the two halves of the rotation pairs 8c..8c+7 -- and
// the tokens 4i + grp of each page; each of the 4 token groups keeps its own
// running max per head, so the only cross-lane work per page is a 3-step
// reduce-scatter of 8 partial dot products, a 3-step max and an 8-way gather
// of probabilities. Products use the packed two-float FMA of sm_100.
//
// Numbers. q and the new k are normed and rotated in double precision; q is
// kept in float, pre-multiplied by log2(e)/sqrt(128) so scores are in log2
// units; the new k is rounded once to bf16 (nearest-even) and both written to
// the cache and patched into the staged page, so it never makes a round trip
// through HBM. Every wait is bounded in time; on expiry the kernel records
// QDA_ERR_TIMEOUT, stops issuing work, drains its own copies and returns.
#include <cuda_bf16.h>
#include <cstdint>

#include "qda_device.cuh"
#include "qda_internal.h"
#include "qwen3_decode_attn.h"

namespace qda {
namespace {

constexpr int kStages = 3;
constexpr int kConsumerWarps = kNumKvHeads;           // one warp per kv head
constexpr int kThreads = (kConsumerWarps + 1) * 32;   // + the producer warp
constexpr int kQkvBytes = kQkvWidth * 2;              // one bf16 qkv row: 8 KiB

// Shared-memory layout (bytes). A stage holds the K rows and V rows of one
// page and, for the first page of a sequence piece, the sequence's qkv row.
constexpr int kStageK = 0;
constexpr int kStageV = kPageBytes;
constexpr int kStageQkv = 2 * kPageBytes;
constexpr int kStageBytes = 2 * kPageBytes + kQkvBytes;
constexpr int kSmemSeg = kStages * kStageBytes;                            // int [kMaxBatch + 4]
constexpr int kSmemLens = kSmemSeg + (kMaxBatch + 4) * 4;                  // int [kMaxBatch]
constexpr int kSmemInvFreq = kSmemLens + kMaxBatch * 4;                    // double [64]
constexpr int kSmemGains = kSmemInvFreq + 64 * 8;                          // bf16 [2][128]
constexpr int kSmemMeta = kSmemGains + 2 * kHeadDim * 2;                   // StageMeta [kStages]
constexpr int kSmemBars = kSmemMeta + kStages * 16;                        // uint64 [2*kStages + 1]
constexpr int kSmemMergeBars = kSmemBars + (2 * kStages + 1) * 8;          // uint64 [kConsumerWarps + 1]
constexpr int kSmemFlags = kSmemMergeBars + (kConsumerWarps + 1) * 8;      // abort flag
constexpr int kSmemTotal = kSmemFlags + 16;
static_assert(kStageBytes % 128 == 0 && kSmemInvFreq % 8 == 0 && kSmemBars % 8 == 0, "alignment");
static_assert(kSmemTotal <= 227 * 1024, "fits one CTA per SM");

// Merging split sequences. Once every consumer warp is past its last page the
// ring is free: warp j merges in its own 1/8 of it, copying up to kMergeBatch
// pieces' partials (1 KiB of un-normalised output for heads 2j, 2j+1, and 16 B
// of running max and sum per piece). The scratch holds kv head j's rows of
// consecutive slots next to each other (part_row), so a batch of pieces is two
// bulk copies: the output rows and the (max, sum) pairs.
constexpr int kMergeRegion = kStages * kStageBytes / kConsumerWarps;
constexpr int kMergeRowBytes = kGroup * kHeadDim * 4;                      // 1 KiB
constexpr int kMergeBatch = 24;
constexpr int kMergeMlOff = kMergeBatch * kMergeRowBytes;
static_assert(kMergeBatch <= 32 && kMergeMlOff + kMergeBatch * 16 <= kMergeRegion && kMergeRegion % 16 == 0,
              "merge region");

// Partial dot products of one staged k row (this lane's 16 dims: words 0..3
// are dims 8c..8c+7, words 4..7 dims 64+8c..64+8c+7) with both query heads.
__device__ __forceinline__ void dot_row(const f32x2* q0, const f32x2* q1, const uint4& lo, const uint4& hi,
                                        float& d0, float& d1) {
    const f32x2 k0 = bf2(lo.x), k1 = bf2(lo.y), k2 = bf2(lo.z), k3 = bf2(lo.w);
    const f32x2 k4 = bf2(hi.x), k5 = bf2(hi.y), k6 = bf2(hi.z), k7 = bf2(hi.w);
    f32x2 a0 = mul2(q0[0], k0), b0 = mul2(q0[4], k4);
    f32x2 a1 = mul2(q1[0], k0), b1 = mul2(q1[4], k4);
    a0 = fma2(q0[1], k1, a0);
    b0 = fma2(q0[5], k5, b0);
    a1 = fma2(q1[1], k1, a1);
    b1 = fma2(q1[5], k5, b1);
    a0 = fma2(q0[2], k2, a0);
    b0 = fma2(q0[6], k6, b0);
    a1 = fma2(q1[2], k2, a1);
    b1 = fma2(q1[6], k6, b1);
    a0 = fma2(q0[3], k3, a0);
    b0 = fma2(q0[7], k7, b0);
    a1 = fma2(q1[3], k3, a1);
    b1 = fma2(q1[7], k7, b1);
    const float2 r0 = unpack2(add2(a0, b0));
    const float2 r1 = unpack2(add2(a1, b1));
    d0 = r0.x + r0.y;
    d1 = r1.x + r1.y;
}

// acc_h += p_h * v for one staged v row (same dim layout as dot_row).
__device__ __forceinline__ void axpy_row(f32x2* acc0, f32x2* acc1, float p0, float p1, const uint4& lo,
                                         const uint4& hi) {
    const f32x2 pp0 = pack2(p0, p0), pp1 = pack2(p1, p1);
    const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const f32x2 v = bf2(w[k]);
        acc0[k] = fma2(pp0, v, acc0[k]);
        acc1[k] = fma2(pp1, v, acc1[k]);
    }
}

struct Shared {
    uint8_t* stages;
    int* seg;        // seg[b] = first global page of sequence b; seg[B] = P
    int* lens;       // seq_lens as read
    double* inv_freq;
    const uint16_t* gains;  // q_norm_w then k_norm_w
    volatile StageMeta* meta;
    uint64_t* full_bar;
    uint64_t* empty_bar;
    uint64_t* never_bar;
    uint64_t* merge_bar;    // [kConsumerWarps]: the merge copies of warp j
    uint64_t* done_bar;     // every consumer warp is past its last page
    volatile int* abort_flag;
};

// ---------------------------------------------------------------------------
// Producer warp: stream the CTA's pages (and each piece's qkv row) into the ring.

__device__ __forceinline__ void run_producer(const Params& p, const Shared& s, int B, int start, int end, int lane) {
    const int count = end - start;
    int slot = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_parity = 0;   // lane 0: slots with a phase armed, and its parity
    bool aborted = false;
    // When this launch depends on the one producing qkv (programmatic
    // dependent launch), the first round of stages gets its K/V copies at
    // once and its qkv copies only after griddepcontrol.wait.
    bool qkv_ready = p.qkv_after_wait == 0;
    int deferred_seq[kStages];
    uint32_t deferred = 0;   // slots of the first round whose qkv copy waits
    int issued = 0;
    auto release_qkv = [&]() {
        pdl_wait();
        asm volatile("fence.proxy.async.global;" ::: "memory");   // the bulk copies read what it wrote
        for (int k = 0; k < kStages; ++k)
            if (deferred & (1u << k))
                bulk_g2s(s.stages + k * kStageBytes + kStageQkv, p.qkv + (size_t)deferred_seq[k] * kQkvWidth,
                         (uint32_t)kQkvBytes, &s.full_bar[k]);
        deferred = 0;
        qkv_ready = true;
    };
    for (int base = 0; base < count && !aborted; base += 32) {
        // 32 pages' descriptions fetched at once, one per lane.
        const int gp = start + base + lane;
        int id = 0, rows = 0, qkv_b = -1, pos = 0;
        if (gp < end) {
            const int b = find_seq(s.seg, B, gp);
            const int i = gp - s.seg[b];
            const int nb = s.seg[b + 1] - s.seg[b];
            id = __ldg(p.block_table + (size_t)b * p.bt_stride + i);
            // the sequence's last page holds the new token at row (L-1)%16; only
            // the rows before it are read from the cache
            rows = (i == nb - 1) ? (s.lens[b] - 1) - kPage * i : kPage;
            if (gp == start || i == 0) {
                qkv_b = b;
                pos = p.positions != nullptr ? __ldg(p.positions + b) : s.lens[b] - 1;
            }
        }
        const int n = min(32, count - base);
        for (int kk = 0; kk < n; ++kk) {
            const int page_id = __shfl_sync(kFull, id, kk);
            const int page_rows = __shfl_sync(kFull, rows, kk);
            const int seq_qkv = __shfl_sync(kFull, qkv_b, kk);
            const int seq_pos = __shfl_sync(kFull, pos, kk);
            int ok = 1;
            if (lane == 0) {
                if (!qkv_ready && issued == kStages) release_qkv();   // before the ring's second round
                ok = mbar_try_wait(&s.empty_bar[slot], phase ^ 1u) ||
                     mbar_wait(&s.empty_bar[slot], phase ^ 1u, p.timeout_ns, s.abort_flag);
                if (ok) {
                    const bool bad = page_id < 0 || page_id >= p.num_pages;
                    s.meta[slot].page = page_id;
                    s.meta[slot].bad = bad ? 1 : 0;
                    s.meta[slot].pos = seq_pos;
                    if (bad) record_error(p.status, QDA_ERR_BOUNDS);
                    const uint32_t kv_bytes = bad ? 0u : (uint32_t)page_rows * kRowBytes;
                    const uint32_t qkv_bytes = seq_qkv >= 0 ? (uint32_t)kQkvBytes : 0u;
                    if (kv_bytes + qkv_bytes != 0) {
                        uint8_t* dst = s.stages + slot * kStageBytes;
                        const size_t off = (size_t)page_id * kPageBytes;
                        mbar_arrive_expect_tx(&s.full_bar[slot], 2u * kv_bytes + qkv_bytes);
                        if (kv_bytes != 0) {
                            bulk_g2s(dst + kStageK, reinterpret_cast<const uint8_t*>(p.k_cache) + off, kv_bytes,
                                     &s.full_bar[slot]);
                            bulk_g2s(dst + kStageV, reinterpret_cast<const uint8_t*>(p.v_cache) + off, kv_bytes,
                                     &s.full_bar[slot]);
                        }
                        if (qkv_bytes != 0) {
                            if (qkv_ready) {
                                bulk_g2s(dst + kStageQkv, p.qkv + (size_t)seq_qkv * kQkvWidth, qkv_bytes,
                                         &s.full_bar[slot]);
                            } else {
                                deferred |= 1u << slot;
                                deferred_seq[slot] = seq_qkv;
                            }
                        }
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
            ++issued;
            if (++slot == kStages) {
                slot = 0;
                phase ^= 1u;
            }
        }
    }
    if (lane == 0 && !qkv_ready) release_qkv();   // a range shorter than one round of the ring
    // After an abort, copies this warp issued may still be landing in shared
    // memory: wait (bounded) for each before the CTA may exit.
    if (lane == 0 && *s.abort_flag != 0) {
        for (int k = 0; k < kStages; ++k)
            if (armed & (1u << k)) (void)mbar_wait(&s.full_bar[k], (armed_parity >> k) & 1u, p.timeout_ns, nullptr);
    }
}

// ---------------------------------------------------------------------------
// Consumer warps.

struct HeadState {
    f32x2 q0[8], q1[8];         // query heads 2j, 2j+1 at this lane's 16 dims (log2-scaled), in pairs
    f32x2 acc0[8], acc1[8];     // un-normalised outputs of this lane's token group, in pairs
    float m0, m1;               // running max of the token group (log2 units)
    float lsum;                 // partial softmax sum of this lane's (token, head) slot
    uint32_t k_lo, k_hi, v_lo, v_hi;  // this lane's words of the appended k/v row
};

// Start sequence b from its staged qkv row. q is normed and rotated in float:
// each rotation angle pos * theta^(-2i/128) is formed and reduced modulo 2*pi
// in double (Cody-Waite, two-part 2*pi) before its float sine and cosine, so
// q keeps float accuracy at any position. When this CTA holds the sequence's
// last page, the new k is normed and rotated entirely in double and rounded
// once to bf16. Lane l computes the angles of pairs 2l and 2l+1; lane (grp, c)
// gathers those of pairs 8c..8c+7, whose two halves are exactly its q dims.
__device__ __forceinline__ void begin_sequence(const Params& p, const Shared& s, const uint8_t* qkv_row, int pos,
                                               int j, int lane, int c, bool appends, HeadState& st) {
    constexpr double kTwoPiHi = 6.2831853069365025;      // 2*pi rounded to 32 significant bits
    constexpr double kTwoPiLo = 2.430840202602477e-10;   // 2*pi - kTwoPiHi
    constexpr double kInvTwoPi = 0.15915494309189535;
    const double ang0 = (double)pos * s.inv_freq[2 * lane];
    const double ang1 = (double)pos * s.inv_freq[2 * lane + 1];
    float cf0, sf0, cf1, sf1;
    {
        const double n0 = rint(ang0 * kInvTwoPi), n1 = rint(ang1 * kInvTwoPi);
        const double r0 = fma(-n0, kTwoPiLo, fma(-n0, kTwoPiHi, ang0));
        const double r1 = fma(-n1, kTwoPiLo, fma(-n1, kTwoPiHi, ang1));
        sincosf((float)r0, &sf0, &cf0);
        sincosf((float)r1, &sf1, &cf1);
    }
    // this lane's 16 dims of heads 2j, 2j+1: words 0..3 dims 8c..8c+7, 4..7 dims 64+8c..
    uint32_t x0[8], x1[8];
    {
        const uint8_t* xh = qkv_row + (kGroup * j) * (kHeadDim * 2);
        const uint4 a0 = *reinterpret_cast<const uint4*>(xh + 16 * c);
        const uint4 b0 = *reinterpret_cast<const uint4*>(xh + 128 + 16 * c);
        const uint4 a1 = *reinterpret_cast<const uint4*>(xh + kHeadDim * 2 + 16 * c);
        const uint4 b1 = *reinterpret_cast<const uint4*>(xh + kHeadDim * 2 + 128 + 16 * c);
        x0[0] = a0.x; x0[1] = a0.y; x0[2] = a0.z; x0[3] = a0.w; x0[4] = b0.x; x0[5] = b0.y; x0[6] = b0.z; x0[7] = b0.w;
        x1[0] = a1.x; x1[1] = a1.y; x1[2] = a1.z; x1[3] = a1.w; x1[4] = b1.x; x1[5] = b1.y; x1[6] = b1.z; x1[7] = b1.w;
    }
    float ss0 = 0.f, ss1 = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        ss0 = fmaf(bf_lo(x0[w]), bf_lo(x0[w]), fmaf(bf_hi(x0[w]), bf_hi(x0[w]), ss0));
        ss1 = fmaf(bf_lo(x1[w]), bf_lo(x1[w]), fmaf(bf_hi(x1[w]), bf_hi(x1[w]), ss1));
    }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {   // over the 8 lanes of the token group
        ss0 += __shfl_xor_sync(kFull, ss0, off);
        ss1 += __shfl_xor_sync(kFull, ss1, off);
    }
    const float eps = (float)p.rms_eps;
    const float inv_r0 = rsqrtf(ss0 * (1.f / 128.f) + eps);
    const float inv_r1 = rsqrtf(ss1 * (1.f / 128.f) + eps);
    const uint4 wa = *reinterpret_cast<const uint4*>(s.gains + 8 * c);        // q gains, dims 8c..
    const uint4 wb = *reinterpret_cast<const uint4*>(s.gains + 64 + 8 * c);   // dims 64+8c..
    const uint32_t wq[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
    const float scale = (float)kQScale;
    // pair 8c + k: dims 8c+k (word k/2 of the low half) and 64+8c+k (word 4 + k/2)
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        float q0a[2], q0b[2], q1a[2], q1b[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int src = 4 * c + m;   // lane holding pairs 8c + 2m and 8c + 2m + 1
            const float cs = __shfl_sync(kFull, e ? cf1 : cf0, src);
            const float sn = __shfl_sync(kFull, e ? sf1 : sf0, src);
            const float wlo = e ? bf_hi(wq[m]) : bf_lo(wq[m]);
            const float whi = e ? bf_hi(wq[4 + m]) : bf_lo(wq[4 + m]);
            const float ya0 = (e ? bf_hi(x0[m]) : bf_lo(x0[m])) * inv_r0 * wlo;
            const float yb0 = (e ? bf_hi(x0[4 + m]) : bf_lo(x0[4 + m])) * inv_r0 * whi;
            const float ya1 = (e ? bf_hi(x1[m]) : bf_lo(x1[m])) * inv_r1 * wlo;
            const float yb1 = (e ? bf_hi(x1[4 + m]) : bf_lo(x1[4 + m])) * inv_r1 * whi;
            q0a[e] = fmaf(ya0, cs, -yb0 * sn) * scale;
            q0b[e] = fmaf(yb0, cs, ya0 * sn) * scale;
            q1a[e] = fmaf(ya1, cs, -yb1 * sn) * scale;
            q1b[e] = fmaf(yb1, cs, ya1 * sn) * scale;
        }
        st.q0[m] = pack2(q0a[0], q0a[1]);
        st.q0[4 + m] = pack2(q0b[0], q0b[1]);
        st.q1[m] = pack2(q1a[0], q1a[1]);
        st.q1[4 + m] = pack2(q1b[0], q1b[1]);
    }

    if (appends) {
        // lane l: dims 2l, 2l+1 (word l of the head) and 64+2l, 65+2l (word 32+l), all in double
        double cs0, sn0, cs1, sn1;
        sincos(ang0, &sn0, &cs0);
        sincos(ang1, &sn1, &cs1);
        const uint32_t* xk = reinterpret_cast<const uint32_t*>(qkv_row + (kNumQHeads + j) * (kHeadDim * 2));
        const uint32_t* xv = reinterpret_cast<const uint32_t*>(qkv_row + (kNumQHeads + kNumKvHeads + j) * (kHeadDim * 2));
        const uint32_t* gk = reinterpret_cast<const uint32_t*>(s.gains + kHeadDim);
        const uint32_t xlo = xk[lane], xhi = xk[32 + lane];
        const uint32_t wk_lo = gk[lane], wk_hi = gk[32 + lane];
        double a0 = bf_to_d(xlo & 0xFFFFu), a1 = bf_to_d(xlo >> 16);
        double b0 = bf_to_d(xhi & 0xFFFFu), b1 = bf_to_d(xhi >> 16);
        const double r = sqrt(warp_sum(a0 * a0 + a1 * a1 + b0 * b0 + b1 * b1) / 128.0 + p.rms_eps);
        a0 = a0 / r * bf_to_d(wk_lo & 0xFFFFu);
        a1 = a1 / r * bf_to_d(wk_lo >> 16);
        b0 = b0 / r * bf_to_d(wk_hi & 0xFFFFu);
        b1 = b1 / r * bf_to_d(wk_hi >> 16);
        const double ra0 = a0 * cs0 - b0 * sn0, rb0 = b0 * cs0 + a0 * sn0;
        const double ra1 = a1 * cs1 - b1 * sn1, rb1 = b1 * cs1 + a1 * sn1;
        st.k_lo = d_to_bf(ra0) | (d_to_bf(ra1) << 16);
        st.k_hi = d_to_bf(rb0) | (d_to_bf(rb1) << 16);
        st.v_lo = xv[lane];
        st.v_hi = xv[32 + lane];
    }

#pragma unroll
    for (int k = 0; k < 8; ++k) {
        st.acc0[k] = 0ull;  // +0.0f, +0.0f
        st.acc1[k] = 0ull;
    }
    st.m0 = -INFINITY;
    st.m1 = -INFINITY;
    st.lsum = 0.f;
}

// Scores, online softmax and value accumulation over one staged page. With
// kFull every one of the 16 rows is a token of the sequence; otherwise the
// rows >= ntok are skipped.
template <bool kFull>
__device__ __forceinline__ void attend_page(const uint8_t* kst, const uint8_t* vst, int ntok, int j, int grp,
                                            int c, int lane, HeadState& st) {
    const uint8_t* kb = kst + j * (kHeadDim * 2) + c * 16;
    const uint8_t* vb = vst + j * (kHeadDim * 2) + c * 16;

    // 8 partial dot products: index 2*ii + h for token 4*ii + grp, head h.
    float sc[8];
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
        const int t = 4 * ii + grp;
        float d0 = 0.f, d1 = 0.f;
        if (kFull || t < ntok) {
            const uint4 lo = *reinterpret_cast<const uint4*>(kb + t * kRowBytes);
            const uint4 hi = *reinterpret_cast<const uint4*>(kb + t * kRowBytes + 128);
            dot_row(st.q0, st.q1, lo, hi, d0, d1);
        }
        sc[2 * ii] = d0;
        sc[2 * ii + 1] = d1;
    }
    // Reduce-scatter over the 8 lanes of the group: lane c ends with the full
    // score of index c (token 4*(c>>1) + grp, head c&1).
    float r4[4], r2[2];
    {
        const bool up = (c & 4) != 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float send = up ? sc[k] : sc[k + 4];
            const float keep = up ? sc[k + 4] : sc[k];
            r4[k] = keep + __shfl_xor_sync(kFull, send, 4);
        }
    }
    {
        const bool up = (c & 2) != 0;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const float send = up ? r4[k] : r4[k + 2];
            const float keep = up ? r4[k + 2] : r4[k];
            r2[k] = keep + __shfl_xor_sync(kFull, send, 2);
        }
    }
    float score;
    {
        const bool up = (c & 1) != 0;
        const float send = up ? r2[0] : r2[1];
        const float keep = up ? r2[1] : r2[0];
        score = keep + __shfl_xor_sync(kFull, send, 1);
    }
    const bool valid = kFull || (4 * (c >> 1) + grp) < ntok;
    if (!kFull) score = valid ? score : -INFINITY;

    // Page max per head within the group, then the lazy rescale.
    float mx = fmaxf(score, __shfl_xor_sync(kFull, score, 2));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
    const float mx_other = __shfl_xor_sync(kFull, mx, 1);
    const float mp0 = (c & 1) ? mx_other : mx;
    const float mp1 = (c & 1) ? mx : mx_other;
    const bool grow0 = mp0 > st.m0 + kRescaleThreshold;
    const bool grow1 = mp1 > st.m1 + kRescaleThreshold;
    if (__any_sync(kFull, grow0 || grow1)) {
        const float n0 = grow0 ? mp0 : st.m0;
        const float n1 = grow1 ? mp1 : st.m1;
        const float a0 = grow0 ? exp2_approx(st.m0 - n0) : 1.f;   // exp2(-inf) = 0 on the first page
        const float a1 = grow1 ? exp2_approx(st.m1 - n1) : 1.f;
        const f32x2 aa0 = pack2(a0, a0), aa1 = pack2(a1, a1);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            st.acc0[k] = mul2(st.acc0[k], aa0);
            st.acc1[k] = mul2(st.acc1[k], aa1);
        }
        st.lsum *= (c & 1) ? a1 : a0;
        st.m0 = n0;
        st.m1 = n1;
    }
    const float pr = valid ? exp2_approx(score - ((c & 1) ? st.m1 : st.m0)) : 0.f;
    st.lsum += pr;

    // Gather the group's 8 probabilities and accumulate V.
    float pv[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) pv[k] = __shfl_sync(kFull, pr, (lane & 24) | k);
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
        const int t = 4 * ii + grp;
        if (kFull || t < ntok) {
            const uint4 lo = *reinterpret_cast<const uint4*>(vb + t * kRowBytes);
            const uint4 hi = *reinterpret_cast<const uint4*>(vb + t * kRowBytes + 128);
            axpy_row(st.acc0, st.acc1, pv[2 * ii], pv[2 * ii + 1], lo, hi);
        }
    }
}

__device__ __forceinline__ void store_bf16x8(uint16_t* dst, const float* v, float scale) {
    uint4 w;
    w.x = pack_bf2(v[0] * scale, v[1] * scale);
    w.y = pack_bf2(v[2] * scale, v[3] * scale);
    w.z = pack_bf2(v[4] * scale, v[5] * scale);
    w.w = pack_bf2(v[6] * scale, v[7] * scale);
    *reinterpret_cast<uint4*>(dst) = w;
}

// Row of the split-piece scratch for kv head j, scratch slot `slot` and query
// head 2j + hb: kv head major, then slot, then the head pair, so that one kv
// head's rows of consecutive slots are contiguous. The slot stride is grid +
// batch (slots are CTA + sequence), within the workspace's grid + max_batch.
__device__ __forceinline__ size_t part_row(const Params& p, int j, int slot, int hb) {
    const size_t stride = (size_t)gridDim.x + (size_t)p.batch;
    return ((size_t)j * stride + (size_t)slot) * kGroup + (size_t)hb;
}

// End of a sequence piece: merge the 4 token groups, then write o directly
// when this CTA holds the whole sequence, else write this piece's partial
// (un-normalised output and its running max and sum) to scratch slot
// blockIdx.x + b. Returns whether a partial was written.
__device__ __forceinline__ bool finish_piece(const Params& p, const Shared& s, int b, int j, int grp, int c,
                                             int per_cta, HeadState& st) {
    const int hb = grp & 1;    // this lane writes head 2j + hb ...
    const int hf = grp >> 1;   // ... dims [64*hf + 8c, 64*hf + 8c + 8)
    float M0 = st.m0, M1 = st.m1;
    M0 = fmaxf(M0, __shfl_xor_sync(kFull, M0, 8));
    M0 = fmaxf(M0, __shfl_xor_sync(kFull, M0, 16));
    M1 = fmaxf(M1, __shfl_xor_sync(kFull, M1, 8));
    M1 = fmaxf(M1, __shfl_xor_sync(kFull, M1, 16));
    const float f0 = (st.m0 == -INFINITY) ? 0.f : exp2_approx(st.m0 - M0);
    const float f1 = (st.m1 == -INFINITY) ? 0.f : exp2_approx(st.m1 - M1);

    float l = st.lsum;
    l += __shfl_xor_sync(kFull, l, 2);
    l += __shfl_xor_sync(kFull, l, 4);
    l *= (c & 1) ? f1 : f0;
    l += __shfl_xor_sync(kFull, l, 8);
    l += __shfl_xor_sync(kFull, l, 16);
    const float l_other = __shfl_xor_sync(kFull, l, 1);
    const float l0 = (c & 1) ? l_other : l;
    const float l1 = (c & 1) ? l : l_other;

    float acc0[16], acc1[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float2 x0 = unpack2(st.acc0[k]), x1 = unpack2(st.acc1[k]);
        acc0[2 * k] = x0.x;
        acc0[2 * k + 1] = x0.y;
        acc1[2 * k] = x1.x;
        acc1[2 * k + 1] = x1.y;
    }
    float r[16], out[8];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float send = hb ? acc0[k] * f0 : acc1[k] * f1;
        const float keep = hb ? acc1[k] * f1 : acc0[k] * f0;
        r[k] = keep + __shfl_xor_sync(kFull, send, 8);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float send = hf ? r[k] : r[k + 8];
        const float keep = hf ? r[k + 8] : r[k];
        out[k] = keep + __shfl_xor_sync(kFull, send, 16);
    }
    const float Mh = hb ? M1 : M0;
    const float Lh = hb ? l1 : l0;
    const int head = kGroup * j + hb;
    const int dim0 = 64 * hf + 8 * c;

    const int part_first = s.seg[b] / per_cta;
    const int part_last = (s.seg[b + 1] - 1) / per_cta;
    if (part_first == part_last) {
        store_bf16x8(p.o + ((size_t)b * kNumQHeads + head) * kHeadDim + dim0, out, Lh > 0.f ? 1.f / Lh : 0.f);
        return false;
    }
    const size_t row = part_row(p, j, (int)blockIdx.x + b, hb);
    float4* pa = reinterpret_cast<float4*>(p.part_acc + row * kHeadDim + dim0);
    __stcg(pa, make_float4(out[0], out[1], out[2], out[3]));
    __stcg(pa + 1, make_float4(out[4], out[5], out[6], out[7]));
    if (c == 0 && hf == 0) __stcg(p.part_ml + row, make_float2(Mh, Lh));
    return true;
}

// Bounded wait of a whole warp on `bar`; on expiry records QDA_ERR_TIMEOUT and
// sets the CTA's abort flag.
__device__ __forceinline__ bool warp_wait(const Params& p, const Shared& s, uint64_t* bar, uint32_t phase, int lane) {
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

// Pieces of sequence b: scratch slots first + b .. first + b + n - 1.
__device__ __forceinline__ int pieces_of(const Shared& s, int b, int per_cta, int& first) {
    first = s.seg[b] / per_cta;
    return (s.seg[b + 1] - 1) / per_cta - first + 1;
}

// Merge every piece's partial of sequence b for heads 2j, 2j+1 and write o
// (this warp was the last to arrive). Pieces come in batches of kMergeBatch
// through this warp's merge region; o = sum_t 2^(m_t - M) acc_t / sum_t
// 2^(m_t - M) l_t with M the running maximum, rescaled between batches.
// Returns false when a wait ran out.
__device__ __forceinline__ bool merge_sequence(const Params& p, const Shared& s, int b, int j, int lane, int issuer,
                                               int grp, int c, int per_cta, uint32_t& mphase) {
    const int hb = grp & 1;
    const int hf = grp >> 1;
    const int head = kGroup * j + hb;
    const int dim0 = 64 * hf + 8 * c;
    int first = 0;
    const int n = pieces_of(s, b, per_cta, first);
    uint8_t* region = s.stages + j * kMergeRegion;
    uint64_t* bar = &s.merge_bar[j];
    float M0 = -INFINITY, M1 = -INFINITY, L0 = 0.f, L1 = 0.f, A[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) A[k] = 0.f;
    for (int t0 = 0; t0 < n; t0 += kMergeBatch) {
        const int nb = min(kMergeBatch, n - t0);
        // earlier reads of the region come before the copies that overwrite it
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == issuer) {
            mbar_arrive_expect_tx(bar, (uint32_t)nb * (kMergeRowBytes + 16));
            // rows of slots first + b + t0 .. + nb - 1 for heads 2j, 2j+1: contiguous
            const size_t row = part_row(p, j, first + b + t0, 0);
            bulk_g2s(region, p.part_acc + row * kHeadDim, (uint32_t)nb * kMergeRowBytes, bar);
            bulk_g2s(region + kMergeMlOff, p.part_ml + row, (uint32_t)nb * 16u, bar);
        }
        if (!warp_wait(p, s, bar, mphase, lane)) {
            // the copies may still be landing: wait once more (bounded) before leaving
            if (lane == 0) (void)mbar_wait(bar, mphase, p.timeout_ns, nullptr);
            __syncwarp();
            return false;
        }
        mphase ^= 1u;
        // lane t < nb holds piece t's (max, sum) of both heads
        const float4 ml = lane < nb ? *reinterpret_cast<const float4*>(region + kMergeMlOff + lane * 16)
                                    : make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
        float bm0 = ml.x, bm1 = ml.z;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            bm0 = fmaxf(bm0, __shfl_xor_sync(kFull, bm0, off));
            bm1 = fmaxf(bm1, __shfl_xor_sync(kFull, bm1, off));
        }
        const float nM0 = fmaxf(M0, bm0), nM1 = fmaxf(M1, bm1);
        // what the earlier batches summed, rescaled to the new maximum (nothing on the first)
        const float r0 = (M0 == -INFINITY) ? 0.f : exp2_approx(M0 - nM0);
        const float r1 = (M1 == -INFINITY) ? 0.f : exp2_approx(M1 - nM1);
        const float rh = hb ? r1 : r0;
#pragma unroll
        for (int k = 0; k < 8; ++k) A[k] *= rh;
        // a piece whose pages were all skipped has max -inf and weight 0
        const float w0 = (ml.x == -INFINITY) ? 0.f : exp2_approx(ml.x - nM0);
        const float w1 = (ml.z == -INFINITY) ? 0.f : exp2_approx(ml.z - nM1);
        L0 = fmaf(w0, ml.y, L0 * r0);
        L1 = fmaf(w1, ml.w, L1 * r1);
        const uint8_t* src = region + (hb * kHeadDim + dim0) * 4;
        for (int t = 0; t < nb; ++t) {
            const float wa = __shfl_sync(kFull, w0, t);
            const float wb = __shfl_sync(kFull, w1, t);
            const float w = hb ? wb : wa;
            const float4 x0 = *reinterpret_cast<const float4*>(src + t * kMergeRowBytes);
            const float4 x1 = *reinterpret_cast<const float4*>(src + t * kMergeRowBytes + 16);
            A[0] = fmaf(w, x0.x, A[0]);
            A[1] = fmaf(w, x0.y, A[1]);
            A[2] = fmaf(w, x0.z, A[2]);
            A[3] = fmaf(w, x0.w, A[3]);
            A[4] = fmaf(w, x1.x, A[4]);
            A[5] = fmaf(w, x1.y, A[5]);
            A[6] = fmaf(w, x1.z, A[6]);
            A[7] = fmaf(w, x1.w, A[7]);
        }
        M0 = nM0;
        M1 = nM1;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        L0 += __shfl_xor_sync(kFull, L0, off);
        L1 += __shfl_xor_sync(kFull, L1, off);
    }
    const float Ls = hb ? L1 : L0;
    store_bf16x8(p.o + ((size_t)b * kNumQHeads + head) * kHeadDim + dim0, A, Ls > 0.f ? 1.f / Ls : 0.f);
    if (lane == 0) p.counters[b * kNumKvHeads + j] = 0;  // ready for the next call
    return true;
}

// Wait for the page in `slot`; returns false when the wait ran out (the
// kernel is then aborting).
__device__ __forceinline__ bool wait_full(const Params& p, const Shared& s, int slot, uint32_t phase, int lane) {
    return warp_wait(p, s, &s.full_bar[slot], phase, lane);
}

// Attend over the staged page in `slot` (page i of a sequence of nb pages and
// length L), appending the new token first when it is the last page, then
// release the slot.
__device__ __forceinline__ void consume_page(const Params& p, const Shared& s, int slot, int i, int nb, int L, int j,
                                             int grp, int c, int lane, HeadState& st) {
    uint8_t* stage = s.stages + slot * kStageBytes;
    const bool last = (i == nb - 1);
    const int new_row = (L - 1) - kPage * i;   // row of the new token on the last page
    const int ntok = last ? new_row + 1 : kPage;
    if (s.meta[slot].bad == 0) {
        if (last) {
            // the new token: written to the cache, and patched into the staged
            // page (this warp's head slice of the row the copy left out)
            const int page = s.meta[slot].page;
            const size_t off =
                (size_t)page * (kPageBytes / 2) + (size_t)new_row * (kRowBytes / 2) + (size_t)j * kHeadDim;
            uint32_t* kd = reinterpret_cast<uint32_t*>(p.k_cache + off);
            uint32_t* vd = reinterpret_cast<uint32_t*>(p.v_cache + off);
            kd[lane] = st.k_lo;
            kd[32 + lane] = st.k_hi;
            vd[lane] = st.v_lo;
            vd[32 + lane] = st.v_hi;
            uint32_t* kr = reinterpret_cast<uint32_t*>(stage + kStageK + new_row * kRowBytes + j * kHeadDim * 2);
            uint32_t* vr = reinterpret_cast<uint32_t*>(stage + kStageV + new_row * kRowBytes + j * kHeadDim * 2);
            kr[lane] = st.k_lo;
            kr[32 + lane] = st.k_hi;
            vr[lane] = st.v_lo;
            vr[32 + lane] = st.v_hi;
            // order these generic writes before the next bulk copy into the slot
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
        }
        if (ntok == kPage) attend_page<true>(stage + kStageK, stage + kStageV, ntok, j, grp, c, lane, st);
        else attend_page<false>(stage + kStageK, stage + kStageV, ntok, j, grp, c, lane, st);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty_bar[slot]);
}

// Consumer warp j: walk the CTA's pages piece by piece (a piece = the pages of
// one sequence inside the CTA's range). Only the first and the last piece can
// be split with other CTAs; their arrivals (and any merge) wait for the end.
__device__ __forceinline__ void run_consumer(const Params& p, const Shared& s, int B, int start, int end, int per_cta,
                                             int warp, int lane) {
    const int j = warp;
    const int grp = lane >> 3;
    const int c = lane & 7;
    HeadState st;
    st.k_lo = st.k_hi = st.v_lo = st.v_hi = 0u;

    int b = find_seq(s.seg, B, start);
    int i0 = start - s.seg[b];       // first page of the piece within its sequence
    int slot = 0;
    uint32_t phase = 0;
    int pending0 = -1, pending1 = -1;  // split pieces whose arrival waits for the end
    const int count = end - start;
    bool aborted = false;
    int k = 0;
    while (k < count && !aborted) {
        const int nb = s.seg[b + 1] - s.seg[b];
        const int L = s.lens[b];
        const int n_here = min(nb - i0, count - k);
        // first page of the piece: it carries the sequence's qkv row
        if (!wait_full(p, s, slot, phase, lane)) {
            aborted = true;
            break;
        }
        begin_sequence(p, s, s.stages + slot * kStageBytes + kStageQkv, s.meta[slot].pos, j, lane, c,
                       /*appends=*/s.seg[b + 1] <= end, st);
        consume_page(p, s, slot, i0, nb, L, j, grp, c, lane, st);
        if (++slot == kStages) { slot = 0; phase ^= 1u; }
        for (int u = 1; u < n_here; ++u) {
            if (!wait_full(p, s, slot, phase, lane)) {
                aborted = true;
                break;
            }
            consume_page(p, s, slot, i0 + u, nb, L, j, grp, c, lane, st);
            if (++slot == kStages) { slot = 0; phase ^= 1u; }
        }
        if (aborted) break;
        k += n_here;
        if (finish_piece(p, s, b, j, grp, c, per_cta, st)) {
            if (pending0 < 0) pending0 = b;
            else pending1 = b;
        }
        if (k < count) {
            do { ++b; } while (b < B && s.seg[b + 1] == s.seg[b]);
            i0 = 0;
        }
    }
    // this warp no longer reads the ring
    __syncwarp();
    if (lane == 0) mbar_arrive(s.done_bar);
    if (aborted || pending0 < 0) return;

    // Count this CTA's split pieces as done (lane 0: pending0, lane 1:
    // pending1); the last piece of a sequence to arrive merges it.
    __threadfence();   // this warp's partial stores before its arrivals
    asm volatile("fence.proxy.async.global;" ::: "memory");
    const int npend = pending1 >= 0 ? 2 : 1;
    const int mine = lane == 0 ? pending0 : pending1;
    int first = 0, prev = -1, need = 0;
    if (lane < npend) {
        need = pieces_of(s, mine, per_cta, first) - 1;
        // acquire: the last to arrive sees every other piece's released partial
        prev = atomic_add_acquire(p.counters + mine * kNumKvHeads + j, 1);
    }
    const bool last0 = __shfl_sync(kFull, prev == need, 0);
    const bool last1 = __shfl_sync(kFull, prev == need, 1) && npend == 2;
    if (!last0 && !last1) return;
    // The other pieces' partials are read through the async proxy by bulk
    // copies, each batch issued by the lane whose acquiring increment found
    // the sequence complete (lane 0 for pending0, lane 1 for pending1).
    asm volatile("fence.proxy.async.global;" ::: "memory");
    if (!warp_wait(p, s, s.done_bar, 0u, lane)) return;
    uint32_t mphase = 0;
    if (last0 && !merge_sequence(p, s, pending0, j, lane, 0, grp, c, per_cta, mphase)) return;
    if (last1) (void)merge_sequence(p, s, pending1, j, lane, 1, grp, c, per_cta, mphase);
}

__global__ void __launch_bounds__(kThreads, 1) decode_attention_kernel(const Params p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    Shared s;
    s.stages = smem;
    s.seg = reinterpret_cast<int*>(smem + kSmemSeg);
    s.lens = reinterpret_cast<int*>(smem + kSmemLens);
    s.inv_freq = reinterpret_cast<double*>(smem + kSmemInvFreq);
    s.gains = reinterpret_cast<const uint16_t*>(smem + kSmemGains);
    s.meta = reinterpret_cast<volatile StageMeta*>(smem + kSmemMeta);
    s.full_bar = reinterpret_cast<uint64_t*>(smem + kSmemBars);
    s.empty_bar = s.full_bar + kStages;
    s.never_bar = s.empty_bar + kStages;
    s.merge_bar = reinterpret_cast<uint64_t*>(smem + kSmemMergeBars);
    s.done_bar = s.merge_bar + kConsumerWarps;
    s.abort_flag = reinterpret_cast<volatile int*>(smem + kSmemFlags);

    // Every launch is a programmatic dependent launch: the next launch on the
    // stream may be scheduled now (its CTAs take an SM as one of these ends),
    // and this one may have started before the previous launch finished. The
    // prologue below touches no global memory; griddepcontrol.wait then holds
    // until the previous launch has completed and its writes are visible
    // (in the mode where that launch only writes qkv, the wait comes later,
    // before the qkv copies).
    pdl_launch_dependents();
    if (threadIdx.x >= 64 && threadIdx.x < 128) {
        const int i = threadIdx.x - 64;
        s.inv_freq[i] = pow(p.rope_theta, -2.0 * i / 128.0);
    }
    if (threadIdx.x == 0) {
        for (int k = 0; k < kStages; ++k) {
            mbar_init(&s.full_bar[k], 1);
            mbar_init(&s.empty_bar[k], kConsumerWarps);
        }
        mbar_init(s.never_bar, 1);
        for (int k = 0; k < kConsumerWarps; ++k) mbar_init(&s.merge_bar[k], 1);
        mbar_init(s.done_bar, kConsumerWarps);
        *s.abort_flag = 0;
        s.seg[0] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (p.qkv_after_wait == 0) pdl_wait();

    // Pages per sequence (0 for a sequence whose length is out of range).
    const int B = p.batch;
    for (int b = threadIdx.x; b < B; b += kThreads) {
        const int L = p.seq_lens[b];
        const bool ok = L >= 1 && L <= p.max_seq_len && L <= kPage * p.bt_stride;
        if (!ok && blockIdx.x == 0) record_error(p.status, QDA_ERR_BOUNDS);
        s.lens[b] = L;
        s.seg[b + 1] = ok ? (L + kPage - 1) / kPage : 0;
    }
    if (threadIdx.x < 128) {
        // both gain vectors, one 4-byte word per thread (the pointers are only
        // 4-byte aligned)
        const uint16_t* src = threadIdx.x < 64 ? p.q_norm_w : p.k_norm_w;
        reinterpret_cast<uint32_t*>(smem + kSmemGains)[threadIdx.x] =
            *reinterpret_cast<const uint32_t*>(src + 2 * (threadIdx.x & 63));
    }
    __syncthreads();
    if (warp == 0) {  // inclusive scan of the page counts: seg[b] becomes the first page of b
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

    const int total = s.seg[B];
    const int per_cta = (total + (int)gridDim.x - 1) / (int)gridDim.x;
    const int start = (int)blockIdx.x * per_cta;
    const int end = min(start + per_cta, total);
    if (start < end) {
        if (warp == kConsumerWarps) run_producer(p, s, B, start, end, lane);
        else run_consumer(p, s, B, start, end, per_cta, warp, lane);
    }
    if ((p.flags & QDA_FLAG_INJECT_WAIT_TIMEOUT) != 0u && blockIdx.x == 0 && warp == 0) {
        // test hook: a barrier nothing arrives at; the wait must end by itself
        if (!mbar_wait(s.never_bar, 0u, p.timeout_ns, nullptr) && lane == 0) record_error(p.status, QDA_ERR_TIMEOUT);
    }
}

}  // namespace

size_t smem_bytes() { return (size_t)kSmemTotal; }

cudaError_t prepare_device() {
    return cudaFuncSetAttribute(decode_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotal);
}

cudaError_t launch(const Params& p, int grid, cudaStream_t stream, bool after_producer) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemTotal;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    Params q = p;
    q.qkv_after_wait = after_producer ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode_attention_kernel, q);
}

}  // namespace qda
