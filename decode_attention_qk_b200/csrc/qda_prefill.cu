// Blocks of many new tokens per sequence: a chunked prefill whose launches
// each take up to 128 query rows per kv head (Qwen3-0.6B Model Spec, "At a
// glance": T new tokens per sequence; "What to watch for": every layer is full
// causal attention; query head h reads kv head h / G, nnterp qwen3,
// "Grouped-query attention"). Token t of a block of T sits in cache slot
// L - T + t and attends over slots up to its own.
//
// The decode-shaped kernels take at most 16 query rows per kv head, so a long
// block run through them reads the whole cache once per 16 rows. Here one
// launch covers a chunk of n tokens with n * G <= 128 rows per kv head and
// reads the cache once:
//
//   1. prefill_append_kernel: one warp per (sequence, kv head, 32 tokens)
//      forms the chunk's new k (RMSNorm and RoPE in double, rounded once to
//      bf16) and writes k and v to their cache slots.
//   2. prefill_kernel: the units (sequence b, kv head j) in order, each the
//      pages of sequence b for kv head j, form one list of page-heads; CTA g
//      takes an equal range of it (whatever the length mix). A producer
//      thread fetches each page's 16 K rows and 16 V rows of kv head j with
//      four tiled copies (a 3-D tensor map over the cache, boxes of 16 rows x
//      64 dims with the 128-byte swizzle, so that the 8 rows an ldmatrix phase
//      reads fall in 8 different bank groups; per-row copies of 256 bytes were
//      bound by the copy engine's per-copy cost). Consumer warp w
//      holds query rows 16w..16w+15 of the unit (row r: token r / G, head
//      G*j + r % G) as one 16-row tile: mma.sync m16n8k16 bf16 products with
//      float accumulators, q and the probabilities in bf16 (the running sums
//      add the same rounded probabilities, so o stays a convex combination of
//      the v rows), an online softmax with lazy rescaling, and each row's
//      causal limit. A unit held whole by one CTA writes o; a split unit writes
//      partials (running max, sum, un-normalised output) to its CTA's slot
//      2g (the CTA's first unit) or 2g + 1 (its last).
//   3. prefill_combine_kernel: one CTA per unit merges the partials of split
//      units with the log-sum-exp rule (Supported models, "Facts proved about
//      the specs": flashAttn_eq, softmax_shift).
//
// All three are programmatic dependent launches; each waits for its
// predecessor to complete before it touches global memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <mutex>

#include "qda_device.cuh"
#include "qda_internal.h"
#include "qda_prefill.h"
#include "qwen3_decode_attn.h"

namespace qda {
namespace {

constexpr int kPfWarps = 8;                          // consumer warps, 16 query rows each
constexpr int kPfThreads = (kPfWarps + 1) * 32;
// A stage: K dims 0-63, K dims 64-127, V dims 0-63, V dims 64-127 of one
// page and kv head, each 16 rows x 128 bytes in the 128-byte swizzled layout
// (row r's 16-byte piece c at piece c ^ (r % 8)).
constexpr int kPfBoxBytes = kPage * 128;             // 2 KiB
constexpr int kPfStageK = 0;
constexpr int kPfStageV = 2 * kPfBoxBytes;
constexpr int kPfStageBytes = 4 * kPfBoxBytes;       // 8 KiB
constexpr int kPfStages = 16;
constexpr int kPfSmemSeg = kPfStages * kPfStageBytes;            // int [kMaxBatch + 4]
constexpr int kPfSmemLens = kPfSmemSeg + (kMaxBatch + 4) * 4;    // int [kMaxBatch]
constexpr int kPfSmemInvFreq = kPfSmemLens + kMaxBatch * 4;      // double [64]
constexpr int kPfSmemGains = kPfSmemInvFreq + 64 * 8;            // bf16 [128], the q gains
constexpr int kPfSmemMeta = kPfSmemGains + kHeadDim * 2;         // StageMeta [kPfStages]
constexpr int kPfSmemBars = kPfSmemMeta + kPfStages * 16;        // full [S], empty [S], never
constexpr int kPfSmemFlags = kPfSmemBars + (2 * kPfStages + 1) * 8;
constexpr int kPfSmemTotal = kPfSmemFlags + 16;
constexpr int kPfSmemAlloc = kPfSmemTotal + 1024;   // slack to align the stages to 1024 bytes
static_assert(kPfStageBytes % 1024 == 0 && kPfSmemInvFreq % 8 == 0 && kPfSmemBars % 8 == 0, "alignment");
static_assert(kPfSmemAlloc <= 227 * 1024, "fits one CTA per SM");
static_assert(kPfWarps * 16 == kPrefillRows, "one 16-row tile per consumer warp");

// x - n * 2*pi for the integer n nearest x / (2*pi), in double: 2*pi is split
// into a 32-bit head (n * head and x - n * head are exact for the |x| < 2^20
// here) and its double remainder, so the result carries about one ulp of x.
__device__ __forceinline__ double reduce_angle(double x) {
    constexpr double kTwoPiHi = 6.2831853069365025;      // 2*pi rounded to 32 significant bits
    constexpr double kTwoPiLo = 2.430840202602477e-10;   // 2*pi - kTwoPiHi
    constexpr double kInvTwoPi = 0.15915494309189535;
    const double m = rint(x * kInvTwoPi);
    return fma(-m, kTwoPiLo, fma(-m, kTwoPiHi, x));
}

// One tiled copy of a 3-D box (16 rows x 1 head x 64 dims of the cache) into
// this CTA's shared memory at dst (1024-byte aligned), completing its bytes
// on `bar`. x (the dim) is 0 or 64: 128-byte aligned.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
        : "memory");
}

// The sequence's length counts its whole block of tok_stride new tokens; a
// launch sees it without the block's tokens after its own (len_trim).
__device__ __forceinline__ bool length_ok(const Params& p, int L_all) {
    return L_all >= p.tok_stride && L_all <= p.max_seq_len && L_all <= kPage * p.bt_stride;
}

__device__ __forceinline__ size_t pf_token_row(const Params& p, int b, int u) {
    return (size_t)b * p.tok_stride + p.tok_offset + u;
}

__device__ __forceinline__ int pf_first_position(const Params& p, int b, int L, int n) {
    return p.positions != nullptr ? __ldg(p.positions + b) + p.tok_offset : L - n;
}

// ---------------------------------------------------------------------------
// 1. The append.

template <int G>
__global__ void __launch_bounds__(32) prefill_append_kernel(const Params p) {
    constexpr int kHq = G * kNumKvHeads;
    constexpr int kQkvW = (kHq + 2 * kNumKvHeads) * kHeadDim;
    pdl_wait();
    pdl_launch_dependents();
    const int b = blockIdx.x, j = blockIdx.y, lane = threadIdx.x;
    const int n = p.new_tokens;
    const int L_all = p.seq_lens[b];
    if (!length_ok(p, L_all)) return;   // the attention launch records it and skips the sequence
    const int L = L_all - p.len_trim;
    const int pos0 = pf_first_position(p, b, L, n);
    // lane l: dims 2l, 2l+1 (word l of the head) and 64+2l, 65+2l (word 32+l), all in double
    const uint32_t* gk = reinterpret_cast<const uint32_t*>(p.k_norm_w);
    const uint32_t wk_lo = gk[lane], wk_hi = gk[32 + lane];
    const double f0 = pow(p.rope_theta, -2.0 * (2 * lane) / 128.0);
    const double f1 = pow(p.rope_theta, -2.0 * (2 * lane + 1) / 128.0);
    const int u_end = min(n, (int)(blockIdx.z + 1) * 32);
    for (int u = (int)blockIdx.z * 32; u < u_end; ++u) {
        const int slot = L - n + u;
        const int page = __ldg(p.block_table + (size_t)b * p.bt_stride + slot / kPage);
        if (page < 0 || page >= p.num_pages) continue;   // recorded by the attention launch
        const uint32_t* row = reinterpret_cast<const uint32_t*>(p.qkv + pf_token_row(p, b, u) * kQkvW);
        const uint32_t* xk = row + (kHq + j) * (kHeadDim / 2);
        const uint32_t* xv = row + (kHq + kNumKvHeads + j) * (kHeadDim / 2);
        const uint32_t xlo = xk[lane], xhi = xk[32 + lane];
        const uint32_t vlo = xv[lane], vhi = xv[32 + lane];
        double a0 = bf_to_d(xlo & 0xFFFFu), a1 = bf_to_d(xlo >> 16);
        double b0 = bf_to_d(xhi & 0xFFFFu), b1 = bf_to_d(xhi >> 16);
        const double inv_rr = 1.0 / sqrt(warp_sum(a0 * a0 + a1 * a1 + b0 * b0 + b1 * b1) / 128.0 + p.rms_eps);
        a0 = a0 * inv_rr * bf_to_d(wk_lo & 0xFFFFu);
        a1 = a1 * inv_rr * bf_to_d(wk_lo >> 16);
        b0 = b0 * inv_rr * bf_to_d(wk_hi & 0xFFFFu);
        b1 = b1 * inv_rr * bf_to_d(wk_hi >> 16);
        const double pos = (double)(pos0 + u);
        double sn0, cs0, sn1, cs1;
        sincos(reduce_angle(pos * f0), &sn0, &cs0);
        sincos(reduce_angle(pos * f1), &sn1, &cs1);
        const double ra0 = a0 * cs0 - b0 * sn0, rb0 = b0 * cs0 + a0 * sn0;
        const double ra1 = a1 * cs1 - b1 * sn1, rb1 = b1 * cs1 + a1 * sn1;
        const size_t off =
            (size_t)page * (kPageBytes / 2) + (size_t)(slot % kPage) * (kRowBytes / 2) + (size_t)j * kHeadDim;
        uint32_t* kd = reinterpret_cast<uint32_t*>(p.k_cache + off);
        uint32_t* vd = reinterpret_cast<uint32_t*>(p.v_cache + off);
        kd[lane] = d_to_bf(ra0) | (d_to_bf(ra1) << 16);
        kd[32 + lane] = d_to_bf(rb0) | (d_to_bf(rb1) << 16);
        vd[lane] = vlo;
        vd[32 + lane] = vhi;
    }
}

// ---------------------------------------------------------------------------
// 2. The attention.

struct PfShared {
    uint8_t* stages;
    int* seg;
    int* lens;
    double* inv_freq;
    const uint16_t* gains;
    volatile StageMeta* meta;
    uint64_t* full_bar;
    uint64_t* empty_bar;
    uint64_t* never_bar;
    volatile int* abort_flag;
};

// The unit holding global page-head x: sequence b, kv head j, page i of b.
__device__ __forceinline__ void pf_locate(const PfShared& s, int B, int x, int& b, int& j, int& i) {
    b = find_seq(s.seg, B, x >> 3);
    const int np = s.seg[b + 1] - s.seg[b];
    const int r = x - 8 * s.seg[b];
    j = r / np;
    i = r % np;
}

__device__ __forceinline__ void pf_producer(const Params& p, const PfShared& s, const CUtensorMap* tm_k,
                                            const CUtensorMap* tm_v, int B, int start, int end, int lane) {
    const int count = end - start;
    int slot = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_parity = 0;
    bool aborted = false;
    for (int base = 0; base < count && !aborted; base += 32) {
        const int x = start + base + lane;
        int id = 0, head = 0;
        if (x < end) {
            int b, i;
            pf_locate(s, B, x, b, head, i);
            id = __ldg(p.block_table + (size_t)b * p.bt_stride + i);
        }
        const int m = min(32, count - base);
        for (int kk = 0; kk < m; ++kk) {
            const int page_id = __shfl_sync(kFull, id, kk);
            const int page_head = __shfl_sync(kFull, head, kk);
            int ok = 1;
            if (lane == 0) {
                ok = mbar_try_wait(&s.empty_bar[slot], phase ^ 1u) ||
                     mbar_wait(&s.empty_bar[slot], phase ^ 1u, p.timeout_ns, s.abort_flag);
                if (ok) {
                    const bool bad = page_id < 0 || page_id >= p.num_pages;
                    s.meta[slot].page = page_id;
                    s.meta[slot].bad = bad ? 1 : 0;
                    if (bad) record_error(p.status, QDA_ERR_BOUNDS);
                    if (!bad) {
                        // the page's 16 rows of kv head page_head, K and V, dims 0-63 and 64-127
                        const uint32_t dst = smem_addr(s.stages + slot * kPfStageBytes);
                        mbar_arrive_expect_tx(&s.full_bar[slot], (uint32_t)kPfStageBytes);
                        for (int h = 0; h < 2; ++h) {
                            tma_load_3d(dst + kPfStageK + h * kPfBoxBytes, tm_k, 64 * h, page_head, page_id * kPage,
                                        &s.full_bar[slot]);
                            tma_load_3d(dst + kPfStageV + h * kPfBoxBytes, tm_v, 64 * h, page_head, page_id * kPage,
                                        &s.full_bar[slot]);
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
            if (++slot == kPfStages) {
                slot = 0;
                phase ^= 1u;
            }
        }
    }
    if (lane == 0 && *s.abort_flag != 0) {
        // copies still landing in this CTA's shared memory: wait (bounded) for each
        for (int k = 0; k < kPfStages; ++k)
            if (armed & (1u << k)) (void)mbar_wait(&s.full_bar[k], (armed_parity >> k) & 1u, p.timeout_ns, nullptr);
    }
}

struct PfState {
    uint32_t qa[8][4];    // A fragments of q per 16-dim step: rows g (regs 0, 2) and g + 8 (regs 1, 3), bf16
    float o[16][4];       // value accumulators: 16 tiles of 8 dims, rows g (0, 1) and g + 8 (2, 3)
    float m[2];           // running max of rows g and g + 8 (log2 units)
    float lsum[2];        // partial softmax sums of this lane's tokens, rows g and g + 8
};

// q of this warp's rows 16w + g and 16w + g + 8 of unit (b, j): RMSNorm and
// RoPE in float (each row's angles from its token's position, the argument
// reduced modulo 2*pi in double), scaled by log2(e)/sqrt(128) and rounded to
// bf16, at dims 8m + 2t, 8m + 2t + 1.
template <int G>
__device__ __forceinline__ void pf_begin(const Params& p, const PfShared& s, int b, int j, int w, int lane, int L,
                                         PfState& st) {
    constexpr int kHq = G * kNumKvHeads;
    constexpr int kQkvW = (kHq + 2 * kNumKvHeads) * kHeadDim;
    const int g = lane >> 2, t = lane & 3;
    const int n = p.new_tokens, R = n * G;
    const int pos0 = pf_first_position(p, b, L, n);
    const uint32_t* gq = reinterpret_cast<const uint32_t*>(s.gains);
    const float scale = (float)kQScale;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int r = 16 * w + g + 8 * h;
        const bool active = r < R;
        const int tt = active ? r / G : 0;
        const int head = G * j + (active ? r % G : 0);
        const uint32_t* xq =
            reinterpret_cast<const uint32_t*>(p.qkv + pf_token_row(p, b, tt) * kQkvW + head * kHeadDim);
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
        const double pos = (double)(pos0 + tt);
#pragma unroll
        for (int mp = 0; mp < 8; ++mp) {
            float qa[2], qb[2];
            const uint32_t wlo = gq[4 * mp + t], whi = gq[32 + 4 * mp + t];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float sn, cs;
                sincosf((float)reduce_angle(pos * s.inv_freq[8 * mp + 2 * t + e]), &sn, &cs);
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
    for (int nn = 0; nn < 16; ++nn)
#pragma unroll
        for (int k = 0; k < 4; ++k) st.o[nn][k] = 0.f;
    st.m[0] = st.m[1] = -INFINITY;
    st.lsum[0] = st.lsum[1] = 0.f;
}

// Scores, online softmax and value accumulation over one staged page for rows
// g and g + 8, which see page tokens up to lim0 and lim1 (unless kFullPage).
// In a swizzled box, row r's 16-byte piece c sits at r * 128 + ((c ^ (r % 8)) * 16).
template <bool kFullPage>
__device__ __forceinline__ void pf_attend(const uint8_t* stage, int lim0, int lim1, bool act0, bool act1, int lane,
                                          PfState& st) {
    const int t = lane & 3;
    const int x7 = lane & 7;   // = row % 8 for every row this lane addresses
    // K rows as the column-major B operand: matrix lane/8 = (tokens 0-7 | 8-15) x (dims +0 | +8)
    const uint32_t krow = smem_addr(stage + kPfStageK) + (x7 + ((lane >> 4) << 3)) * 128;
    const int kc = (lane >> 3) & 1;
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(krow + (k >> 2) * kPfBoxBytes + ((((2 * (k & 3)) + kc) ^ x7) << 4), b0, b1, b2, b3);
        mma_bf16_16816(c0, st.qa[k], b0, b1);
        mma_bf16_16816(c1, st.qa[k], b2, b3);
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
        for (int nn = 0; nn < 16; ++nn) {
            st.o[nn][0] *= a0;
            st.o[nn][1] *= a0;
            st.o[nn][2] *= a1;
            st.o[nn][3] *= a1;
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
    // V rows as the column-major B operand (transposed load): matrix lane/8 =
    // (tokens 0-7 | 8-15) x (dims +0 | +8)
    const uint32_t vrow = smem_addr(stage + kPfStageV) + (x7 + (((lane >> 3) & 1) << 3)) * 128;
    const int vc = (lane >> 4) & 1;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_trans(vrow + (u >> 2) * kPfBoxBytes + ((((2 * (u & 3)) + vc) ^ x7) << 4), b0, b1, b2, b3);
        mma_bf16_16816(st.o[2 * u], pa, b0, b1);
        mma_bf16_16816(st.o[2 * u + 1], pa, b2, b3);
    }
}

__device__ __forceinline__ bool pf_wait_full(const Params& p, const PfShared& s, int slot, uint32_t phase,
                                             int lane) {
    uint64_t* bar = &s.full_bar[slot];
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

// End of a unit piece: o for the warp's active rows when the unit is held
// whole by this CTA, else the partials in scratch slot `slot`.
template <int G>
__device__ __forceinline__ void pf_finish(const Params& p, const PrefillScratch& sc, int b, int j, int w, int lane,
                                          bool whole, int slot, PfState& st) {
    constexpr int kHq = G * kNumKvHeads;
    const int g = lane >> 2, t = lane & 3;
    const int R = p.new_tokens * G;
    float l[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l[h] = st.lsum[h];
        l[h] += __shfl_xor_sync(kFull, l[h], 1);
        l[h] += __shfl_xor_sync(kFull, l[h], 2);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int r = 16 * w + g + 8 * h;
        if (r >= R) continue;
        if (whole) {
            const int tt = r / G, head = G * j + r % G;
            const float inv = l[h] > 0.f ? 1.f / l[h] : 0.f;
            uint32_t* dst = reinterpret_cast<uint32_t*>(p.o + (pf_token_row(p, b, tt) * kHq + head) * kHeadDim);
#pragma unroll
            for (int nn = 0; nn < 16; ++nn) dst[4 * nn + t] = pack_bf2(st.o[nn][2 * h] * inv, st.o[nn][2 * h + 1] * inv);
        } else {
            const size_t prow = (size_t)slot * kPrefillRows + r;
            float2* pa = reinterpret_cast<float2*>(sc.acc + prow * kHeadDim);
#pragma unroll
            for (int nn = 0; nn < 16; ++nn) __stcg(pa + 4 * nn + t, make_float2(st.o[nn][2 * h], st.o[nn][2 * h + 1]));
            if (t == 0) __stcg(sc.ml + prow, make_float2(st.m[h], l[h]));
        }
    }
}

template <int G>
__device__ __forceinline__ void pf_consumer(const Params& p, const PrefillScratch& sc, const PfShared& s, int B,
                                            int start, int end, int per_cta, int w, int lane) {
    const int n = p.new_tokens, R = n * G;
    const bool active_warp = 16 * w < R;
    const int g = lane >> 2;
    const int r0 = 16 * w + g, r1 = r0 + 8;
    const bool act0 = r0 < R, act1 = r1 < R;
    const int tt0 = act0 ? r0 / G : 0, tt1 = act1 ? r1 / G : 0;
    PfState st;
    int b, j, i0;
    pf_locate(s, B, start, b, j, i0);
    int slot = 0;
    uint32_t phase = 0;
    const int count = end - start;
    int k = 0;
    bool aborted = false;
    while (k < count && !aborted) {
        const int np = s.seg[b + 1] - s.seg[b];
        const int L = s.lens[b];
        const int n_here = min(np - i0, count - k);
        if (active_warp) pf_begin<G>(p, s, b, j, w, lane, L, st);
        for (int u = 0; u < n_here; ++u) {
            if (!pf_wait_full(p, s, slot, phase, lane)) {
                aborted = true;
                break;
            }
            uint8_t* stage = s.stages + slot * kPfStageBytes;
            const int i = i0 + u;
            if (active_warp && s.meta[slot].bad == 0) {
                const int rows = min(kPage, L - kPage * i);
                if (rows < kPage) {
                    // rows after the sequence hold stale bytes; a stale NaN times a
                    // zero probability would still give NaN in the value product
                    for (int rr = rows; rr < kPage; ++rr) {   // row rr of both halves (the swizzle stays in the row)
                        reinterpret_cast<uint32_t*>(stage + kPfStageV + rr * 128)[lane] = 0u;
                        reinterpret_cast<uint32_t*>(stage + kPfStageV + kPfBoxBytes + rr * 128)[lane] = 0u;
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                }
                // row r (token tt) sees slots <= L - n + tt
                const int lim0 = (L - n + tt0) - kPage * i, lim1 = (L - n + tt1) - kPage * i;
                if (kPage * i + kPage - 1 <= L - n) pf_attend<true>(stage, lim0, lim1, act0, act1, lane, st);
                else pf_attend<false>(stage, lim0, lim1, act0, act1, lane, st);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.empty_bar[slot]);
            if (++slot == kPfStages) {
                slot = 0;
                phase ^= 1u;
            }
        }
        if (aborted) break;
        // the unit's page-head range; a unit held whole by one CTA writes o
        const int ustart = 8 * s.seg[b] + j * np;
        const bool whole = ustart / per_cta == (ustart + np - 1) / per_cta;
        const int pslot = 2 * (int)blockIdx.x + (k == 0 ? 0 : 1);   // the CTA's first piece, else its last
        if (active_warp) pf_finish<G>(p, sc, b, j, w, lane, whole, pslot, st);
        k += n_here;
        if (k < count) {
            if (++j == kNumKvHeads) {
                j = 0;
                do { ++b; } while (b < B && s.seg[b + 1] == s.seg[b]);
            }
            i0 = 0;
        }
    }
}

template <int G>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, const Params p,
                   const PrefillScratch sc) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    // the stages start on a 1024-byte boundary (the swizzle atom)
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    PfShared s;
    s.stages = smem;
    s.seg = reinterpret_cast<int*>(smem + kPfSmemSeg);
    s.lens = reinterpret_cast<int*>(smem + kPfSmemLens);
    s.inv_freq = reinterpret_cast<double*>(smem + kPfSmemInvFreq);
    s.gains = reinterpret_cast<const uint16_t*>(smem + kPfSmemGains);
    s.meta = reinterpret_cast<volatile StageMeta*>(smem + kPfSmemMeta);
    s.full_bar = reinterpret_cast<uint64_t*>(smem + kPfSmemBars);
    s.empty_bar = s.full_bar + kPfStages;
    s.never_bar = s.empty_bar + kPfStages;
    s.abort_flag = reinterpret_cast<volatile int*>(smem + kPfSmemFlags);

    // The prologue touches no global memory; griddepcontrol.wait then holds
    // until the append launch has completed and its cache writes are visible.
    if (threadIdx.x >= 64 && threadIdx.x < 128) {
        const int i = threadIdx.x - 64;
        s.inv_freq[i] = pow(p.rope_theta, -2.0 * i / 128.0);
    }
    if (threadIdx.x == 0) {
        for (int k = 0; k < kPfStages; ++k) {
            mbar_init(&s.full_bar[k], 1);
            mbar_init(&s.empty_bar[k], kPfWarps);
        }
        mbar_init(s.never_bar, 1);
        *s.abort_flag = 0;
        s.seg[0] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_v)) : "memory");
    }
    pdl_wait();

    const int B = p.batch;
    for (int b = threadIdx.x; b < B; b += kPfThreads) {
        const int L_all = p.seq_lens[b];
        const bool ok = length_ok(p, L_all);
        if (!ok && blockIdx.x == 0) record_error(p.status, QDA_ERR_BOUNDS);
        const int L = ok ? L_all - p.len_trim : 0;
        s.lens[b] = L;
        s.seg[b + 1] = ok ? (L + kPage - 1) / kPage : 0;
    }
    if (threadIdx.x < kHeadDim / 2) {   // the q gains, one 4-byte word per thread
        reinterpret_cast<uint32_t*>(smem + kPfSmemGains)[threadIdx.x] =
            reinterpret_cast<const uint32_t*>(p.q_norm_w)[threadIdx.x];
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
    if (blockIdx.x == 0)   // page offsets for the combine launch
        for (int b = threadIdx.x; b <= B; b += kPfThreads) p.seg[b] = s.seg[b];

    const int total = kNumKvHeads * s.seg[B];   // page-heads
    const int per_cta = (total + (int)gridDim.x - 1) / (int)gridDim.x;
    const int start = (int)blockIdx.x * per_cta;
    const int end = min(start + per_cta, total);
    if (start < end) {
        if (warp == kPfWarps) pf_producer(p, s, &tm_k, &tm_v, B, start, end, lane);
        else pf_consumer<G>(p, sc, s, B, start, end, per_cta, warp, lane);
    }
    pdl_launch_dependents();
}

// ---------------------------------------------------------------------------
// 3. The combine: CTA (b, j), warp w merges rows w, w + 8, ... of the unit;
// lane l dims 4l..4l+3. The unit's pieces sit in consecutive CTAs g0..gk of
// the attention launch: slot 2*g0 + 1 when the unit starts inside g0's range
// (it is g0's last piece), else 2*g0; slot 2*g in the later CTAs.
template <int G>
__global__ void __launch_bounds__(256) prefill_combine_kernel(const Params p, const PrefillScratch sc) {
    constexpr int kHq = G * kNumKvHeads;
    pdl_wait();
    pdl_launch_dependents();
    const int b = blockIdx.x, j = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int np = p.seg[b + 1] - p.seg[b];
    if (np == 0) return;   // a sequence the attention launch skipped
    const int total = kNumKvHeads * p.seg[p.batch];
    const int per_cta = (total + sc.grid - 1) / sc.grid;
    const int ustart = kNumKvHeads * p.seg[b] + j * np;
    const int g0 = ustart / per_cta, gk = (ustart + np - 1) / per_cta;
    if (g0 == gk) return;   // held whole by one CTA, which wrote o
    const int R = p.new_tokens * G;
    for (int r = warp; r < R; r += 8) {
        float M = -INFINITY;
        for (int g = g0; g <= gk; ++g) {
            const int slot = (g == g0 && ustart % per_cta != 0) ? 2 * g + 1 : 2 * g;
            M = fmaxf(M, __ldcg(sc.ml + (size_t)slot * kPrefillRows + r).x);
        }
        float Ls = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int g = g0; g <= gk; ++g) {
            const int slot = (g == g0 && ustart % per_cta != 0) ? 2 * g + 1 : 2 * g;
            const size_t prow = (size_t)slot * kPrefillRows + r;
            const float2 ml = __ldcg(sc.ml + prow);
            const float wt = (ml.x == -INFINITY) ? 0.f : exp2_approx(ml.x - M);   // a piece that saw no slot
            Ls = fmaf(wt, ml.y, Ls);
            const float4 x = __ldcg(reinterpret_cast<const float4*>(sc.acc + prow * kHeadDim) + lane);
            acc.x = fmaf(wt, x.x, acc.x);
            acc.y = fmaf(wt, x.y, acc.y);
            acc.z = fmaf(wt, x.z, acc.z);
            acc.w = fmaf(wt, x.w, acc.w);
        }
        const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
        uint2 out;
        out.x = pack_bf2(acc.x * inv, acc.y * inv);
        out.y = pack_bf2(acc.z * inv, acc.w * inv);
        const int tt = r / G, head = G * j + r % G;
        reinterpret_cast<uint2*>(p.o + (pf_token_row(p, b, tt) * kHq + head) * kHeadDim)[lane] = out;
    }
}

PFN_cuTensorMapEncodeTiled_v12000 pf_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        else
            cudaGetLastError();
    });
    return fn;
}

// The cache [num_pages * 16 rows][8 heads][128 dims] bf16 as a 3-D tensor,
// read in boxes of 16 rows x 1 head x 64 dims with the 128-byte swizzle.
bool encode_cache(CUtensorMap* map, const void* cache, int num_pages) {
    const PFN_cuTensorMapEncodeTiled_v12000 fn = pf_encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)kNumKvHeads, (cuuint64_t)num_pages * kPage};
    const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)kRowBytes};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kPage};
    const cuuint32_t elem[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(cache), dims, strides, box, elem,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int G>
cudaError_t launch_prefill_g(const Params& p, const PrefillScratch& sc, cudaStream_t stream) {
    CUtensorMap tk, tv;
    if (!encode_cache(&tk, p.k_cache, p.num_pages) || !encode_cache(&tv, p.v_cache, p.num_pages))
        return cudaErrorInvalidValue;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((unsigned)p.batch, (unsigned)kNumKvHeads, (unsigned)((p.new_tokens + 31) / 32));
    cfg.blockDim = dim3(32, 1, 1);
    cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_append_kernel<G>, p);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)sc.grid, 1, 1);
    cfg.blockDim = dim3(kPfThreads, 1, 1);
    cfg.dynamicSmemBytes = kPfSmemAlloc;
    e = cudaLaunchKernelEx(&cfg, prefill_kernel<G>, tk, tv, p, sc);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)p.batch, (unsigned)kNumKvHeads, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, prefill_combine_kernel<G>, p, sc);
}

}  // namespace

cudaError_t prepare_prefill() {
    if (pf_encode_fn() == nullptr) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPfSmemAlloc);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(prefill_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPfSmemAlloc);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(prefill_kernel<5>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPfSmemAlloc);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(prefill_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPfSmemAlloc);
    return e;
}

int prefill_max_tokens(int num_q_heads) { return kPrefillRows / (num_q_heads / kNumKvHeads); }

cudaError_t launch_prefill(const Params& p, const PrefillScratch& sc, cudaStream_t stream) {
    const int G = p.num_q_heads / kNumKvHeads;
    if (p.new_tokens < 1 || p.new_tokens * G > kPrefillRows || sc.grid < 1) return cudaErrorInvalidValue;
    switch (G) {
        case 2: return launch_prefill_g<2>(p, sc, stream);
        case 4: return launch_prefill_g<4>(p, sc, stream);
        case 5: return launch_prefill_g<5>(p, sc, stream);
        case 8: return launch_prefill_g<8>(p, sc, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace qda
