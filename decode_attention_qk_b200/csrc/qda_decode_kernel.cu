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
// Supported models page, "Facts proved about the specs"). The piece of
// sequence b held by CTA g gets scratch slot g + b; these slots are distinct
// because ranges and sequences are both ordered.
//
// Inside a CTA. Warp 8 is the producer: lane 0 issues one bulk copy of the
// K rows and one of the V rows of a page (up to 32 KiB each, all 8 kv heads)
// into a 3-stage shared-memory ring, completed on an mbarrier. Warps 0..7 are
// consumers; warp j serves kv head j and both query heads 2j, 2j+1 that read
// it (nnterp qwen3, "Grouped-query attention"), so every K/V byte is read from
// HBM once. Lane (grp = lane/8, c = lane%8) owns head dims [8c, 8c+8) and
// [64+8c, 64+8c+8) and the tokens 4i + grp of each page; each of the 4 token
// groups keeps its own running max per head, so the only cross-lane work per
// page is a 3-step reduce-scatter of 8 partial dot products, a 3-step max and
// an 8-way gather of probabilities.
//
// q and the new k are normed and rotated in double precision; q is kept in
// float, pre-multiplied by log2(e)/sqrt(128) so scores are in log2 units; the
// new k is rounded once to bf16 (nearest-even) and both written to the cache
// and patched into the staged page, so it never makes a round trip through
// HBM. Every wait is bounded in time; on expiry the kernel records
// QDA_ERR_TIMEOUT, stops issuing work, drains its own copies and returns.
#include <cuda_bf16.h>
#include <cstdint>

#include "qda_internal.h"
#include "qwen3_decode_attn.h"

namespace qda {
namespace {

constexpr int kStages = 3;
constexpr int kConsumerWarps = kNumKvHeads;           // one warp per kv head
constexpr int kThreads = (kConsumerWarps + 1) * 32;   // + the producer warp
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr float kRescaleThreshold = 8.0f;             // log2 units: rescale only when the max grows by > 2^8
constexpr double kQScale = 1.4426950408889634 * 0.088388347648318441;  // log2(e) / sqrt(128)

// Shared-memory layout (bytes).
constexpr int kStageBytes = 2 * kPageBytes;           // K rows, then V rows
constexpr int kSmemQ = kStages * kStageBytes;         // per consumer warp: float [2][128]
constexpr int kSmemSeg = kSmemQ + kConsumerWarps * kGroup * kHeadDim * 4;  // int [kMaxBatch + 4]
constexpr int kSmemLens = kSmemSeg + (kMaxBatch + 4) * 4;                  // int [kMaxBatch]
constexpr int kSmemInvFreq = kSmemLens + kMaxBatch * 4;                    // double [64]
constexpr int kSmemBars = kSmemInvFreq + 64 * 8;                           // uint64 [2*kStages + 1]
constexpr int kSmemFlags = kSmemBars + (2 * kStages + 1) * 8;              // int [kStages] + abort
constexpr int kSmemTotal = kSmemFlags + 8 * 4;
static_assert(kSmemInvFreq % 8 == 0 && kSmemBars % 8 == 0, "8-byte alignment");
static_assert(kSmemTotal <= 227 * 1024, "fits one CTA per SM");

// ---------------------------------------------------------------------------
// PTX wrappers: mbarrier, bulk copy, timer, exp2

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of `bar` with parity `parity` to complete, for at most
// `timeout_ns` (and at most 2^30 polls). Gives up early when `abort_flag` is
// set. Returns whether the phase completed.
__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int64_t timeout_ns,
                                       const volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1; it < (1u << 30); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31u) == 0) {
            if (abort_flag != nullptr && *abort_flag != 0) return false;
            if (static_cast<int64_t>(global_ns() - t0) > timeout_ns) return false;
        }
    }
    return false;
}

// One bulk copy global -> shared, completing `bytes` of transaction on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void record_error(int* status, int code) { atomicCAS(status, 0, code); }

// ---------------------------------------------------------------------------
// bf16 helpers

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ double bf_to_d(uint32_t bits16) { return (double)__uint_as_float(bits16 << 16); }

// double -> bf16, nearest-even, without double rounding: truncate to float and
// set the last bit when the truncation was inexact (round-to-odd at 24 bits);
// rounding that to nearest-even at 8 bits gives the correctly rounded result
// of the double (rounding to odd with >= 2 spare bits is innocuous; Boldo and
// Melquiond, IEEE Trans. Computers 57(4), 2008).
__device__ __forceinline__ uint32_t d_to_bf(double x) {
    float f = __double2float_rz(x);
    if ((double)f != x) f = __uint_as_float(__float_as_uint(f) | 1u);
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ uint32_t pack_bf2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
    return v;
}

// Partial dot product of 16 q values with 16 bf16 k values (two 16-byte rows).
__device__ __forceinline__ float dot16(const float* q, const uint4& lo, const uint4& hi) {
    float a = q[0] * bf_lo(lo.x);
    float b = q[8] * bf_lo(hi.x);
    a = fmaf(q[1], bf_hi(lo.x), a);
    b = fmaf(q[9], bf_hi(hi.x), b);
    a = fmaf(q[2], bf_lo(lo.y), a);
    b = fmaf(q[10], bf_lo(hi.y), b);
    a = fmaf(q[3], bf_hi(lo.y), a);
    b = fmaf(q[11], bf_hi(hi.y), b);
    a = fmaf(q[4], bf_lo(lo.z), a);
    b = fmaf(q[12], bf_lo(hi.z), b);
    a = fmaf(q[5], bf_hi(lo.z), a);
    b = fmaf(q[13], bf_hi(hi.z), b);
    a = fmaf(q[6], bf_lo(lo.w), a);
    b = fmaf(q[14], bf_lo(hi.w), b);
    a = fmaf(q[7], bf_hi(lo.w), a);
    b = fmaf(q[15], bf_hi(hi.w), b);
    return a + b;
}

__device__ __forceinline__ void axpy16(float* acc, float p, const uint4& lo, const uint4& hi) {
    acc[0] = fmaf(p, bf_lo(lo.x), acc[0]);
    acc[1] = fmaf(p, bf_hi(lo.x), acc[1]);
    acc[2] = fmaf(p, bf_lo(lo.y), acc[2]);
    acc[3] = fmaf(p, bf_hi(lo.y), acc[3]);
    acc[4] = fmaf(p, bf_lo(lo.z), acc[4]);
    acc[5] = fmaf(p, bf_hi(lo.z), acc[5]);
    acc[6] = fmaf(p, bf_lo(lo.w), acc[6]);
    acc[7] = fmaf(p, bf_hi(lo.w), acc[7]);
    acc[8] = fmaf(p, bf_lo(hi.x), acc[8]);
    acc[9] = fmaf(p, bf_hi(hi.x), acc[9]);
    acc[10] = fmaf(p, bf_lo(hi.y), acc[10]);
    acc[11] = fmaf(p, bf_hi(hi.y), acc[11]);
    acc[12] = fmaf(p, bf_lo(hi.z), acc[12]);
    acc[13] = fmaf(p, bf_hi(hi.z), acc[13]);
    acc[14] = fmaf(p, bf_lo(hi.w), acc[14]);
    acc[15] = fmaf(p, bf_hi(hi.w), acc[15]);
}

// Largest b in [0, B) with seg[b] <= page: the sequence holding global page
// `page` (zero-page sequences are skipped because their successor starts at
// the same offset).
__device__ __forceinline__ int find_seq(const int* seg, int B, int page) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (seg[mid] <= page) lo = mid; else hi = mid - 1;
    }
    return lo;
}

struct Shared {
    uint8_t* stages;
    float* q;
    int* seg;        // seg[b] = first global page of sequence b; seg[B] = P
    int* lens;       // seq_lens as read
    double* inv_freq;
    uint64_t* full_bar;
    uint64_t* empty_bar;
    uint64_t* never_bar;
    volatile int* slot_bad;
    volatile int* abort_flag;
};

// ---------------------------------------------------------------------------
// Producer warp: stream the CTA's pages into the ring.

__device__ __forceinline__ void run_producer(const Params& p, const Shared& s, int B, int start, int end, int lane) {
    const int count = end - start;
    int slot = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_parity = 0;   // lane 0: slots with a phase armed, and its parity
    bool aborted = false;
    for (int base = 0; base < count && !aborted; base += 32) {
        // 32 pages' ids fetched at once, one per lane.
        const int gp = start + base + lane;
        int id = 0, rows = 0;
        if (gp < end) {
            const int b = find_seq(s.seg, B, gp);
            const int i = gp - s.seg[b];
            const int nb = s.seg[b + 1] - s.seg[b];
            id = __ldg(p.block_table + (size_t)b * p.bt_stride + i);
            // the sequence's last page holds the new token at row (L-1)%16; only
            // the rows before it are read from the cache
            rows = (i == nb - 1) ? (s.lens[b] - 1) - kPage * i : kPage;
        }
        const int n = min(32, count - base);
        for (int kk = 0; kk < n; ++kk) {
            const int page_id = __shfl_sync(kFull, id, kk);
            const int page_rows = __shfl_sync(kFull, rows, kk);
            int ok = 1;
            if (lane == 0) {
                ok = mbar_wait(&s.empty_bar[slot], phase ^ 1u, p.timeout_ns, s.abort_flag);
                if (ok) {
                    const bool bad = page_id < 0 || page_id >= p.num_pages;
                    s.slot_bad[slot] = bad ? 1 : 0;
                    if (bad) record_error(p.status, QDA_ERR_BOUNDS);
                    const uint32_t bytes = bad ? 0u : (uint32_t)page_rows * kRowBytes;
                    if (bytes != 0) {
                        uint8_t* dst = s.stages + slot * kStageBytes;
                        const size_t off = (size_t)page_id * kPageBytes;
                        mbar_arrive_expect_tx(&s.full_bar[slot], 2u * bytes);
                        bulk_g2s(dst, reinterpret_cast<const uint8_t*>(p.k_cache) + off, bytes, &s.full_bar[slot]);
                        bulk_g2s(dst + kPageBytes, reinterpret_cast<const uint8_t*>(p.v_cache) + off, bytes,
                                 &s.full_bar[slot]);
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
            if (++slot == kStages) {
                slot = 0;
                phase ^= 1u;
            }
        }
    }
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
    float q0[16], q1[16];       // query heads 2j, 2j+1 at this lane's 16 dims (log2-scaled)
    float acc0[16], acc1[16];   // un-normalised outputs of this lane's token group
    float m0, m1;               // running max of the token group (log2 units)
    float lsum;                 // partial softmax sum of this lane's (token, head) slot
    uint32_t k_lo, k_hi, v_lo, v_hi;  // this lane's words of the appended k/v row
};

// Norm and rotate q (and, when this CTA appends for sequence b, k), in double.
// Lane l handles the rotation pairs 2l and 2l+1: dims 2l, 2l+1, 64+2l, 65+2l.
__device__ __forceinline__ void begin_sequence(const Params& p, const Shared& s, int b, int j, int lane, int c,
                               bool appends, HeadState& st) {
    const int L = s.lens[b];
    const double pos = (double)(p.positions != nullptr ? p.positions[b] : L - 1);
    double sn0, cs0, sn1, cs1;
    sincos(pos * s.inv_freq[2 * lane], &sn0, &cs0);
    sincos(pos * s.inv_freq[2 * lane + 1], &sn1, &cs1);

    const uint16_t* row = p.qkv + (size_t)b * kQkvWidth;
    float* qs = s.q + j * (kGroup * kHeadDim);
    const uint32_t wq_lo = *reinterpret_cast<const uint32_t*>(p.q_norm_w + 2 * lane);
    const uint32_t wq_hi = *reinterpret_cast<const uint32_t*>(p.q_norm_w + 64 + 2 * lane);
    __syncwarp();  // the previous sequence's q may still be being read
#pragma unroll
    for (int h = 0; h < kGroup; ++h) {
        const uint16_t* x = row + (kGroup * j + h) * kHeadDim;
        const uint32_t xlo = *reinterpret_cast<const uint32_t*>(x + 2 * lane);
        const uint32_t xhi = *reinterpret_cast<const uint32_t*>(x + 64 + 2 * lane);
        double a0 = bf_to_d(xlo & 0xFFFFu), a1 = bf_to_d(xlo >> 16);
        double b0 = bf_to_d(xhi & 0xFFFFu), b1 = bf_to_d(xhi >> 16);
        const double r = sqrt(warp_sum(a0 * a0 + a1 * a1 + b0 * b0 + b1 * b1) / 128.0 + p.rms_eps);
        a0 = a0 / r * bf_to_d(wq_lo & 0xFFFFu);
        a1 = a1 / r * bf_to_d(wq_lo >> 16);
        b0 = b0 / r * bf_to_d(wq_hi & 0xFFFFu);
        b1 = b1 / r * bf_to_d(wq_hi >> 16);
        const double ra0 = a0 * cs0 - b0 * sn0, rb0 = b0 * cs0 + a0 * sn0;
        const double ra1 = a1 * cs1 - b1 * sn1, rb1 = b1 * cs1 + a1 * sn1;
        float2* qh = reinterpret_cast<float2*>(qs + h * kHeadDim);
        qh[lane] = make_float2((float)(ra0 * kQScale), (float)(ra1 * kQScale));
        qh[32 + lane] = make_float2((float)(rb0 * kQScale), (float)(rb1 * kQScale));
    }
    __syncwarp();
    {
        const float4* q0 = reinterpret_cast<const float4*>(qs + 8 * c);
        const float4* q0h = reinterpret_cast<const float4*>(qs + 64 + 8 * c);
        const float4* q1 = reinterpret_cast<const float4*>(qs + kHeadDim + 8 * c);
        const float4* q1h = reinterpret_cast<const float4*>(qs + kHeadDim + 64 + 8 * c);
        float4 v;
        v = q0[0];  st.q0[0] = v.x;  st.q0[1] = v.y;  st.q0[2] = v.z;  st.q0[3] = v.w;
        v = q0[1];  st.q0[4] = v.x;  st.q0[5] = v.y;  st.q0[6] = v.z;  st.q0[7] = v.w;
        v = q0h[0]; st.q0[8] = v.x;  st.q0[9] = v.y;  st.q0[10] = v.z; st.q0[11] = v.w;
        v = q0h[1]; st.q0[12] = v.x; st.q0[13] = v.y; st.q0[14] = v.z; st.q0[15] = v.w;
        v = q1[0];  st.q1[0] = v.x;  st.q1[1] = v.y;  st.q1[2] = v.z;  st.q1[3] = v.w;
        v = q1[1];  st.q1[4] = v.x;  st.q1[5] = v.y;  st.q1[6] = v.z;  st.q1[7] = v.w;
        v = q1h[0]; st.q1[8] = v.x;  st.q1[9] = v.y;  st.q1[10] = v.z; st.q1[11] = v.w;
        v = q1h[1]; st.q1[12] = v.x; st.q1[13] = v.y; st.q1[14] = v.z; st.q1[15] = v.w;
    }

    if (appends) {
        const uint16_t* x = row + kNumQHeads * kHeadDim + j * kHeadDim;
        const uint32_t xlo = *reinterpret_cast<const uint32_t*>(x + 2 * lane);
        const uint32_t xhi = *reinterpret_cast<const uint32_t*>(x + 64 + 2 * lane);
        const uint32_t wk_lo = *reinterpret_cast<const uint32_t*>(p.k_norm_w + 2 * lane);
        const uint32_t wk_hi = *reinterpret_cast<const uint32_t*>(p.k_norm_w + 64 + 2 * lane);
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
        const uint16_t* v = row + (kNumQHeads + kNumKvHeads) * kHeadDim + j * kHeadDim;
        st.v_lo = *reinterpret_cast<const uint32_t*>(v + 2 * lane);
        st.v_hi = *reinterpret_cast<const uint32_t*>(v + 64 + 2 * lane);

        const int nb = s.seg[b + 1] - s.seg[b];
        const int page = p.block_table[(size_t)b * p.bt_stride + nb - 1];
        if (page >= 0 && page < p.num_pages) {
            const size_t off = (size_t)page * (kPageBytes / 2) + (size_t)((L - 1) % kPage) * (kRowBytes / 2) +
                               (size_t)j * kHeadDim;
            uint32_t* kd = reinterpret_cast<uint32_t*>(p.k_cache + off);
            uint32_t* vd = reinterpret_cast<uint32_t*>(p.v_cache + off);
            kd[lane] = st.k_lo;
            kd[32 + lane] = st.k_hi;
            vd[lane] = st.v_lo;
            vd[32 + lane] = st.v_hi;
        }
    }

#pragma unroll
    for (int k = 0; k < 16; ++k) {
        st.acc0[k] = 0.f;
        st.acc1[k] = 0.f;
    }
    st.m0 = -INFINITY;
    st.m1 = -INFINITY;
    st.lsum = 0.f;
}

// Scores, online softmax and value accumulation over one staged page.
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
        if (t < ntok) {
            const uint4 lo = *reinterpret_cast<const uint4*>(kb + t * kRowBytes);
            const uint4 hi = *reinterpret_cast<const uint4*>(kb + t * kRowBytes + 128);
            d0 = dot16(st.q0, lo, hi);
            d1 = dot16(st.q1, lo, hi);
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
    const bool valid = (4 * (c >> 1) + grp) < ntok;
    score = valid ? score : -INFINITY;

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
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            st.acc0[k] *= a0;
            st.acc1[k] *= a1;
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
        if (t < ntok) {
            const uint4 lo = *reinterpret_cast<const uint4*>(vb + t * kRowBytes);
            const uint4 hi = *reinterpret_cast<const uint4*>(vb + t * kRowBytes + 128);
            axpy16(st.acc0, pv[2 * ii], lo, hi);
            axpy16(st.acc1, pv[2 * ii + 1], lo, hi);
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

// Merge the 4 token groups; write o directly when this CTA holds the whole
// sequence, else write a partial and let the last CTA of the sequence combine.
__device__ __forceinline__ void end_sequence(const Params& p, const Shared& s, int b, int j, int lane, int grp, int c,
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

    float r[16], out[8];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float send = hb ? st.acc0[k] * f0 : st.acc1[k] * f1;
        const float keep = hb ? st.acc1[k] * f1 : st.acc0[k] * f0;
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
    uint16_t* o = p.o + ((size_t)b * kNumQHeads + head) * kHeadDim + dim0;

    const int part_first = s.seg[b] / per_cta;
    const int part_last = (s.seg[b + 1] - 1) / per_cta;
    const int nparts = part_last - part_first + 1;
    if (nparts == 1) {
        store_bf16x8(o, out, Lh > 0.f ? 1.f / Lh : 0.f);
        return;
    }

    const int slot = blockIdx.x + b;
    float4* pa = reinterpret_cast<float4*>(p.part_acc + ((size_t)slot * kNumQHeads + head) * kHeadDim + dim0);
    __stcg(pa, make_float4(out[0], out[1], out[2], out[3]));
    __stcg(pa + 1, make_float4(out[4], out[5], out[6], out[7]));
    if (c == 0 && hf == 0) __stcg(p.part_ml + (size_t)slot * kNumQHeads + head, make_float2(Mh, Lh));
    __threadfence();
    __syncwarp();
    int prev = 0;
    if (lane == 0) prev = atomicAdd(p.counters + b * kNumKvHeads + j, 1);
    prev = __shfl_sync(kFull, prev, 0);
    if (prev != nparts - 1) return;

    // Last arrival: combine every piece of this sequence for heads 2j, 2j+1.
    __threadfence();
    float M = -INFINITY, Ls = 0.f, A[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) A[k] = 0.f;
    for (int t = 0; t < nparts; ++t) {
        const int sid = part_first + t + b;
        const float2 ml = __ldcg(p.part_ml + (size_t)sid * kNumQHeads + head);
        const float4* src =
            reinterpret_cast<const float4*>(p.part_acc + ((size_t)sid * kNumQHeads + head) * kHeadDim + dim0);
        const float4 x0 = __ldcg(src), x1 = __ldcg(src + 1);
        if (ml.x == -INFINITY) continue;  // a piece whose pages were all skipped
        const float Mn = fmaxf(M, ml.x);
        const float sa = exp2_approx(M - Mn);
        const float sb = exp2_approx(ml.x - Mn);
        Ls = Ls * sa + ml.y * sb;
        A[0] = A[0] * sa + x0.x * sb;
        A[1] = A[1] * sa + x0.y * sb;
        A[2] = A[2] * sa + x0.z * sb;
        A[3] = A[3] * sa + x0.w * sb;
        A[4] = A[4] * sa + x1.x * sb;
        A[5] = A[5] * sa + x1.y * sb;
        A[6] = A[6] * sa + x1.z * sb;
        A[7] = A[7] * sa + x1.w * sb;
        M = Mn;
    }
    store_bf16x8(o, A, Ls > 0.f ? 1.f / Ls : 0.f);
    if (lane == 0) p.counters[b * kNumKvHeads + j] = 0;  // ready for the next call
}

__device__ __forceinline__ void run_consumer(const Params& p, const Shared& s, int B, int start, int end, int per_cta, int warp,
                             int lane) {
    const int j = warp;
    const int grp = lane >> 3;
    const int c = lane & 7;
    HeadState st;
    st.k_lo = st.k_hi = st.v_lo = st.v_hi = 0u;

    int b = find_seq(s.seg, B, start);
    int i = start - s.seg[b];
    int slot = 0;
    uint32_t phase = 0;
    const int count = end - start;
    for (int k = 0; k < count; ++k) {
        const int nb = s.seg[b + 1] - s.seg[b];
        const int L = s.lens[b];
        const bool last = (i == nb - 1);
        if (k == 0 || i == 0) begin_sequence(p, s, b, j, lane, c, /*appends=*/s.seg[b + 1] <= end, st);
        const int new_row = (L - 1) - kPage * i;   // row of the new token on the last page
        const int ntok = last ? new_row + 1 : kPage;

        bool ok = mbar_wait(&s.full_bar[slot], phase, p.timeout_ns, s.abort_flag);
        ok = __all_sync(kFull, ok || mbar_try_wait(&s.full_bar[slot], phase));
        if (!ok) {
            if (lane == 0) {
                *s.abort_flag = 1;
                record_error(p.status, QDA_ERR_TIMEOUT);
            }
            return;
        }
        uint8_t* kst = s.stages + slot * kStageBytes;
        uint8_t* vst = kst + kPageBytes;
        if (s.slot_bad[slot] == 0) {
            if (last) {
                // the new token: this warp's head slice of the row the copy left out
                uint32_t* kr = reinterpret_cast<uint32_t*>(kst + new_row * kRowBytes + j * kHeadDim * 2);
                uint32_t* vr = reinterpret_cast<uint32_t*>(vst + new_row * kRowBytes + j * kHeadDim * 2);
                kr[lane] = st.k_lo;
                kr[32 + lane] = st.k_hi;
                vr[lane] = st.v_lo;
                vr[32 + lane] = st.v_hi;
                // order these generic writes before the next bulk copy into the slot
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
            }
            attend_page(kst, vst, ntok, j, grp, c, lane, st);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.empty_bar[slot]);
        if (++slot == kStages) {
            slot = 0;
            phase ^= 1u;
        }
        if (last || k == count - 1) end_sequence(p, s, b, j, lane, grp, c, per_cta, st);
        if (++i == nb) {
            i = 0;
            do { ++b; } while (b < B && s.seg[b + 1] == s.seg[b]);
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1) decode_attention_kernel(const Params p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    Shared s;
    s.stages = smem;
    s.q = reinterpret_cast<float*>(smem + kSmemQ);
    s.seg = reinterpret_cast<int*>(smem + kSmemSeg);
    s.lens = reinterpret_cast<int*>(smem + kSmemLens);
    s.inv_freq = reinterpret_cast<double*>(smem + kSmemInvFreq);
    s.full_bar = reinterpret_cast<uint64_t*>(smem + kSmemBars);
    s.empty_bar = s.full_bar + kStages;
    s.never_bar = s.empty_bar + kStages;
    s.slot_bad = reinterpret_cast<volatile int*>(smem + kSmemFlags);
    s.abort_flag = s.slot_bad + kStages;

    // Pages per sequence (0 for a sequence whose length is out of range).
    const int B = p.batch;
    for (int b = threadIdx.x; b < B; b += kThreads) {
        const int L = p.seq_lens[b];
        const bool ok = L >= 1 && L <= p.max_seq_len && L <= kPage * p.bt_stride;
        if (!ok && blockIdx.x == 0) record_error(p.status, QDA_ERR_BOUNDS);
        s.lens[b] = L;
        s.seg[b + 1] = ok ? (L + kPage - 1) / kPage : 0;
    }
    if (threadIdx.x < 64) s.inv_freq[threadIdx.x] = pow(p.rope_theta, -2.0 * threadIdx.x / 128.0);
    if (threadIdx.x == 0) {
        for (int k = 0; k < kStages; ++k) {
            mbar_init(&s.full_bar[k], 1);
            mbar_init(&s.empty_bar[k], kConsumerWarps);
            s.slot_bad[k] = 0;
        }
        mbar_init(s.never_bar, 1);
        *s.abort_flag = 0;
        s.seg[0] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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

cudaError_t launch(const Params& p, int grid, cudaStream_t stream) {
    decode_attention_kernel<<<grid, kThreads, kSmemTotal, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace qda
