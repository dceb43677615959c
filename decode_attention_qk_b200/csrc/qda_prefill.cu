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
//   1. prefill_prep_kernel: one warp per (sequence, kv head, token) forms the
//      token's new k and writes k and v to their cache slots, and forms its G
//      query rows of the kv head into the unit's 128-row query tile (scratch,
//      already in the tensor cores' swizzled layout).
//   2. prefill_kernel: the units (sequence b, kv head j) in order, each the
//      pages of sequence b for kv head j, form one list of page-heads; CTA g
//      takes an equal range of it (whatever the length mix). Per unit piece
//      the query tile is one 128-row operand of the 5th-generation tensor
//      cores: S = Q K^T and O += P V with accumulators in tensor memory, the
//      K and V tiles copied by the tensor memory accelerator (a 3-D tensor map
//      over the cache, boxes of 16 rows x 64 dims with the 128-byte swizzle),
//      the softmax one thread per row. A unit held whole by one CTA writes o;
//      a split unit writes partials (running max, sum, un-normalised output)
//      to its CTA's slot 2g (the CTA's first unit) or 2g + 1 (its last).
//   3. prefill_combine_kernel: one warp per row of a split unit merges its
//      partials with the log-sum-exp rule (Supported models, "Facts proved
//      about the specs": flashAttn_eq, softmax_shift).
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
#include "qda_tc.cuh"
#include "qwen3_decode_attn.h"

namespace qda {
namespace {


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
// 1. The prep: warp w of CTA (b, j, z) takes token u = 4z + w of the chunk.
// It forms the token's new k (RMSNorm and RoPE in double, rounded once to
// bf16) and writes k and v to their cache slots, and forms the token's G query
// rows of kv head j (RMSNorm and RoPE in float, the angle reduced modulo 2*pi
// in double, scaled by log2(e)/sqrt(128), rounded to bf16) into the unit's
// query tile in the attention's layout. Lane l holds dims 2l, 2l+1 (word l of
// a head) and 64+2l, 65+2l (word 32+l), the RoPE pairs (i, i+64).

template <int G>
__global__ void __launch_bounds__(128) prefill_prep_kernel(const Params p, const PrefillScratch sc) {
    constexpr int kHq = G * kNumKvHeads;
    constexpr int kQkvW = (kHq + 2 * kNumKvHeads) * kHeadDim;
    pdl_wait();
    pdl_launch_dependents();
    const int b = blockIdx.x, j = blockIdx.y, lane = threadIdx.x & 31;
    const int u = 4 * (int)blockIdx.z + (int)(threadIdx.x >> 5);
    const int n = p.new_tokens;
    if (u >= n) return;
    const int L_all = p.seq_lens[b];
    if (!length_ok(p, L_all)) return;   // the attention launch records it and skips the sequence
    const int L = L_all - p.len_trim;
    const double pos = (double)(pf_first_position(p, b, L, n) + u);
    const double ang0 = reduce_angle(pos * pow(p.rope_theta, -2.0 * (2 * lane) / 128.0));
    const double ang1 = reduce_angle(pos * pow(p.rope_theta, -2.0 * (2 * lane + 1) / 128.0));
    const uint32_t* row = reinterpret_cast<const uint32_t*>(p.qkv + pf_token_row(p, b, u) * kQkvW);

    const int slot = L - n + u;
    const int page = __ldg(p.block_table + (size_t)b * p.bt_stride + slot / kPage);
    if (page >= 0 && page < p.num_pages) {   // else recorded by the attention launch
        const uint32_t* gk = reinterpret_cast<const uint32_t*>(p.k_norm_w);
        const uint32_t wk_lo = gk[lane], wk_hi = gk[32 + lane];
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
        double sn0, cs0, sn1, cs1;
        sincos(ang0, &sn0, &cs0);
        sincos(ang1, &sn1, &cs1);
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

    float sn0, cs0, sn1, cs1;
    sincosf((float)ang0, &sn0, &cs0);
    sincosf((float)ang1, &sn1, &cs1);
    const uint32_t* gq = reinterpret_cast<const uint32_t*>(p.q_norm_w);
    const uint32_t wq_lo = gq[lane], wq_hi = gq[32 + lane];
    const float scale = (float)kQScale;
    uint8_t* tile = reinterpret_cast<uint8_t*>(sc.q) + (size_t)(b * kNumKvHeads + j) * kPrefillQTileBytes;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
        const int r = u * G + hh;
        const uint32_t* xq = row + (G * j + hh) * (kHeadDim / 2);
        const uint32_t xlo = xq[lane], xhi = xq[32 + lane];
        float ss = bf_lo(xlo) * bf_lo(xlo) + bf_hi(xlo) * bf_hi(xlo) + bf_lo(xhi) * bf_lo(xhi) + bf_hi(xhi) * bf_hi(xhi);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(kFull, ss, o);
        const float inv_r = rsqrtf(ss * (1.f / 128.f) + (float)p.rms_eps);
        const float ya0 = bf_lo(xlo) * inv_r * bf_lo(wq_lo), ya1 = bf_hi(xlo) * inv_r * bf_hi(wq_lo);
        const float yb0 = bf_lo(xhi) * inv_r * bf_lo(wq_hi), yb1 = bf_hi(xhi) * inv_r * bf_hi(wq_hi);
        const uint32_t qa = pack_bf2(fmaf(ya0, cs0, -yb0 * sn0) * scale, fmaf(ya1, cs1, -yb1 * sn1) * scale);
        const uint32_t qb = pack_bf2(fmaf(yb0, cs0, ya0 * sn0) * scale, fmaf(yb1, cs1, ya1 * sn1) * scale);
        // row r of each 64-dim half: 128 bytes, 16-byte piece c at piece c ^ (r % 8)
        const uint32_t off = (uint32_t)r * 128u + ((((uint32_t)lane >> 2) ^ ((uint32_t)r & 7u)) << 4) + (lane & 3) * 4;
        *reinterpret_cast<uint32_t*>(tile + off) = qa;
        *reinterpret_cast<uint32_t*>(tile + kPrefillQTileBytes / 2 + off) = qb;
    }
}

// ---------------------------------------------------------------------------
// 2. The attention, on the 5th-generation tensor cores.
//
// A unit piece is (sequence b, kv head j, a range of b's pages). Its query
// tile Q, 128 rows x 128 dims in bf16 (row r < R = n * G: token r / G, head
// G*j + r % G; the rows from R on are never read out), is copied from the
// prep launch's scratch into one of two shared-memory buffers, so that the
// next piece's tile lands while this one runs. The cache arrives in stages of
// 64 rows (4 pages) of K and V, and for each stage
//   S = Q K^T     tcgen05.mma, M = 128 rows, N = 64 keys, K = 128 dims, into
//                 one of two S buffers in tensor memory (S of the next stage
//                 forms while this stage's softmax runs);
//   softmax       one thread per row: the causal and length mask, the running
//                 max with lazy rescaling of O, P = exp2(S - m) rounded to bf16
//                 into shared memory (the running sum adds the same rounded
//                 values, so o stays a convex combination of v rows);
//   O += P V      M = 128 rows, N = 128 dims, K = 64 keys, V read MN-major
//                 from its copied tile;
// and O, accumulated in tensor memory over the piece, is read out once at the
// piece's end.
//
// Warp roles (256 threads): warp 0 issues the copies; one thread of warp 1
// issues the tensor-core instructions (warp 1 also allocates tensor memory);
// warps 4-7 run the softmax and write o (warp 4 + w reads tensor-memory lanes
// 32w..32w+31, the rows it owns). Every wait is bounded: a timeout records
// QDA_ERR_TIMEOUT, sets the CTA's abort flag and every role leaves its loop;
// tensor memory is freed after every issued instruction has completed.

constexpr int kTcKeys = 64;                          // cache rows per stage
constexpr int kTcPages = kTcKeys / kPage;            // 4
constexpr int kTcStages = 4;
constexpr int kTcThreads = 8 * 32;
constexpr int kTcHalf = kTcKeys * 128;               // 64 dims of a stage's rows: 8 KiB
constexpr int kTcStageK = 0;                         // K dims 0-63 | K dims 64-127
constexpr int kTcStageV = 2 * kTcHalf;               // V dims 0-63 | V dims 64-127
constexpr int kTcStageBytes = 4 * kTcHalf;           // 32 KiB
constexpr int kTcBoxBytes = kPage * 128;             // one copied box: 16 rows x 64 dims
constexpr int kTcTile = kPrefillRows * 128;          // 64 columns of a 128-row operand: 16 KiB
constexpr int kTcSmemQ = kTcStages * kTcStageBytes;  // 2 buffers: Q dims 0-63 | Q dims 64-127
constexpr int kTcSmemP = kTcSmemQ + 4 * kTcTile;     // P: 128 rows x 64 keys
constexpr int kTcSmemSeg = kTcSmemP + kTcTile;                       // int [kMaxBatch + 4]
constexpr int kTcSmemLens = kTcSmemSeg + (kMaxBatch + 4) * 4;        // int [kMaxBatch]
constexpr int kTcSmemMask = kTcSmemLens + kMaxBatch * 4;             // int [kTcStages]: pages not copied
constexpr int kTcSmemBars = kTcSmemMask + kTcStages * 4;
// kv_full[S], kv_empty[S], s_full[2], p_full, pv_done, q_full[2], q_free[2], fin
constexpr int kTcNumBars = 2 * kTcStages + 9;
constexpr int kTcSmemTmem = kTcSmemBars + kTcNumBars * 8;            // tensor-memory address, abort flag
constexpr int kTcSmemTotal = kTcSmemTmem + 16;
constexpr int kTcSmemAlloc = kTcSmemTotal + 1024;   // slack to align the tiles to 1024 bytes
constexpr uint32_t kTcTmemCols = 256;               // S buffers at columns 0 and 64, O at 128
constexpr uint32_t kTcTmemO = 128;
static_assert(kTcStageBytes % 1024 == 0 && kTcSmemSeg % 1024 == 0, "swizzle atoms are 1024-byte aligned");
static_assert(kTcSmemBars % 8 == 0 && 2 * kTcTile == kPrefillQTileBytes, "layout");
static_assert(kTcSmemAlloc <= 227 * 1024, "fits one CTA per SM");
static_assert(kTcKeys == 64, "a P row is one 128-byte swizzled row");

struct TcShared {
    uint8_t* stages;
    uint8_t* q;
    uint8_t* p;
    int* seg;
    int* lens;
    volatile int* mask;
    uint64_t* kv_full;
    uint64_t* kv_empty;
    uint64_t* s_full;
    uint64_t* p_full;
    uint64_t* pv_done;
    uint64_t* q_full;   // [2]
    uint64_t* q_free;   // [2]
    uint64_t* fin;
    volatile int* abort_flag;
};

// The unit pieces of a CTA's page-head range [start, end), in order; every
// role walks the same sequence.
struct PieceWalk {
    int b, j, i0, n;   // sequence b, kv head j, pages i0 .. i0 + n - 1 of b
    int k;             // pages of the range before this piece
    int count;
    __device__ __forceinline__ void begin(const int* seg, int B, int start, int end) {
        count = end - start;
        k = 0;
        b = find_seq(seg, B, start >> 3);
        const int np = seg[b + 1] - seg[b];
        const int r = start - 8 * seg[b];
        j = r / np;
        i0 = r % np;
        n = min(np - i0, count);
    }
    __device__ __forceinline__ bool next(const int* seg, int B) {
        k += n;
        if (k >= count) return false;
        if (++j == kNumKvHeads) {
            j = 0;
            do { ++b; } while (b < B && seg[b + 1] == seg[b]);
        }
        i0 = 0;
        n = min(seg[b + 1] - seg[b], count - k);
        return true;
    }
};

// One thread's bounded wait; a failure aborts the CTA.
__device__ __forceinline__ bool tc_wait1(const Params& p, const TcShared& s, uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    if (mbar_wait(bar, parity, p.timeout_ns, s.abort_flag)) return true;
    *s.abort_flag = 1;
    record_error(p.status, QDA_ERR_TIMEOUT);
    return false;
}

// A whole warp's bounded wait, with one verdict for all its lanes.
__device__ __forceinline__ bool tc_wait_warp(const Params& p, const TcShared& s, uint64_t* bar, uint32_t parity,
                                             int lane) {
    bool ok = mbar_try_wait(bar, parity);
    if (__all_sync(kFull, ok)) return true;
    ok = ok || mbar_wait(bar, parity, p.timeout_ns, s.abort_flag);
    ok = __all_sync(kFull, ok || mbar_try_wait(bar, parity));
    if (!ok && lane == 0) {
        *s.abort_flag = 1;
        record_error(p.status, QDA_ERR_TIMEOUT);
    }
    return ok;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void fence_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Warp 0: the page ids (32 page-heads looked up at a time), then per stage
// four tiled copies per page: K and V of kv head j, dims 0-63 and 64-127,
// into the stage's halves at 2 KiB per page. Pages whose block-table entry is
// out of range are not copied; the stage's mask tells the softmax.
__device__ __forceinline__ void tc_producer(const Params& p, const PrefillScratch& sc, const TcShared& s,
                                            const CUtensorMap* tm_k, const CUtensorMap* tm_v, int B, int start,
                                            int end, int lane) {
    const uint32_t q_bytes = (uint32_t)(p.new_tokens * (p.num_q_heads / kNumKvHeads)) * 128u;   // R rows per half
    int wbase = 0x40000000, id = -1;
    uint32_t g = 0, u = 0, armed = 0, armed_parity = 0, q_armed = 0;
    bool ok = true;
    asm volatile("fence.proxy.async.global;" ::: "memory");   // the copies read what the prep launch wrote
    PieceWalk w;
    w.begin(s.seg, B, start, end);
    do {
        // the piece's query tile, into buffer u % 2 once the piece two back has
        // finished reading it
        {
            int good = 1;
            if (lane == 0) {
                if (u >= 2) good = tc_wait1(p, s, &s.q_free[u & 1u], ((u >> 1) - 1) & 1u) ? 1 : 0;
                if (good) {
                    const uint8_t* src = reinterpret_cast<const uint8_t*>(sc.q) +
                                         (size_t)(w.b * kNumKvHeads + w.j) * kPrefillQTileBytes;
                    uint8_t* dst = s.q + (u & 1u) * 2 * kTcTile;
                    mbar_arrive_expect_tx(&s.q_full[u & 1u], 2 * q_bytes);
                    bulk_g2s(dst, src, q_bytes, &s.q_full[u & 1u]);
                    bulk_g2s(dst + kTcTile, src + kTcTile, q_bytes, &s.q_full[u & 1u]);
                    q_armed = (q_armed & ~(3u << (2 * (u & 1u)))) | ((2u | ((u >> 1) & 1u)) << (2 * (u & 1u)));
                }
            }
            if (!__shfl_sync(kFull, good, 0)) break;
            ++u;
        }
        const int np_b = s.seg[w.b + 1] - s.seg[w.b];
        const int x_piece = 8 * s.seg[w.b] + w.j * np_b + w.i0;
        for (int q = 0; q < w.n; q += kTcPages, ++g) {
            const int npg = min(kTcPages, w.n - q);
            const int x0 = x_piece + q;
            if (x0 < wbase || x0 + npg > wbase + 32) {
                wbase = x0;
                const int x = x0 + lane;
                id = -1;
                if (x < end) {
                    const int bb = find_seq(s.seg, B, x >> 3);
                    const int np = s.seg[bb + 1] - s.seg[bb];
                    const int r = x - 8 * s.seg[bb];
                    id = __ldg(p.block_table + (size_t)bb * p.bt_stride + r % np);
                }
            }
            const int st = (int)(g % kTcStages);
            int good = 1;
            if (lane == 0 && g >= (uint32_t)kTcStages)
                good = tc_wait1(p, s, &s.kv_empty[st], ((g / kTcStages) - 1) & 1u) ? 1 : 0;
            if (!__shfl_sync(kFull, good, 0)) {
                ok = false;
                break;
            }
            const int my = __shfl_sync(kFull, id, (x0 - wbase + lane) & 31);
            const uint32_t bad = __ballot_sync(kFull, lane < npg && (my < 0 || my >= p.num_pages));
            if (lane == 0) {
                s.mask[st] = (int)bad;
                if (bad != 0) record_error(p.status, QDA_ERR_BOUNDS);
                const int copied = npg - __popc(bad);
                if (copied > 0) {
                    mbar_arrive_expect_tx(&s.kv_full[st], (uint32_t)(copied * 4 * kTcBoxBytes));
                    armed |= 1u << st;
                    armed_parity = (armed_parity & ~(1u << st)) | (((g / kTcStages) & 1u) << st);
                } else {
                    mbar_arrive(&s.kv_full[st]);
                }
            }
            const uint32_t dst = smem_addr(s.stages + st * kTcStageBytes);
            for (int k = 0; k < npg; ++k) {
                const int page = __shfl_sync(kFull, my, k);
                if (lane == 0 && ((bad >> k) & 1u) == 0) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        tma_load_3d(dst + kTcStageK + h * kTcHalf + k * kTcBoxBytes, tm_k, 64 * h, w.j, page * kPage,
                                    &s.kv_full[st]);
                        tma_load_3d(dst + kTcStageV + h * kTcHalf + k * kTcBoxBytes, tm_v, 64 * h, w.j, page * kPage,
                                    &s.kv_full[st]);
                    }
                }
            }
        }
    } while (ok && w.next(s.seg, B));
    if (lane == 0 && *s.abort_flag != 0) {
        // copies still landing in this CTA's shared memory: wait (bounded) for each
        for (int k = 0; k < kTcStages; ++k)
            if (armed & (1u << k)) (void)mbar_wait(&s.kv_full[k], (armed_parity >> k) & 1u, p.timeout_ns, nullptr);
        for (int k = 0; k < 2; ++k)
            if ((q_armed >> (2 * k)) & 2u)
                (void)mbar_wait(&s.q_full[k], (q_armed >> (2 * k)) & 1u, p.timeout_ns, nullptr);
    }
}

// One thread of warp 1: per stage g, S_g = Q K_g^T into S buffer g % 2, then
// O += P_{g-1} V_{g-1} once the softmax has written P_{g-1}. S_g overwrites
// the buffer the softmax of stage g - 2 read, which it had finished before
// writing P_{g-2}.
__device__ __forceinline__ void tc_issuer(const Params& p, const TcShared& s, int B, int start, int end,
                                          uint32_t tmem) {
    const uint32_t idesc_s = umma_idesc_bf16_m128(kTcKeys);
    const uint32_t idesc_o = umma_idesc_bf16_m128_bmn(kHeadDim);
    const uint32_t p_base = smem_addr(s.p), st_base = smem_addr(s.stages);
    auto pv = [&](uint32_t x, bool first) -> bool {
        if (!tc_wait1(p, s, s.p_full, x & 1u)) return false;
        tc_fence_after();
        const uint32_t v = st_base + (x % kTcStages) * kTcStageBytes + kTcStageV;
#pragma unroll
        for (int kk = 0; kk < kTcKeys / 16; ++kk)
            umma_bf16(tmem + kTcTmemO, umma_desc_sw128(p_base + 32 * kk),
                      umma_desc_sw128_mn(v + 2 * 1024 * kk, kTcHalf, 1024), idesc_o, (first && kk == 0) ? 0u : 1u);
        umma_commit(s.pv_done);
        umma_commit(&s.kv_empty[x % kTcStages]);   // K and V of the stage have been read
        return true;
    };
    uint32_t g = 0, u = 0;
    bool prev_first = false, ok = true;
    PieceWalk w;
    w.begin(s.seg, B, start, end);
    do {
        if (!tc_wait1(p, s, &s.q_full[u & 1u], (u >> 1) & 1u)) {
            ok = false;
            break;
        }
        tc_fence_after();
        const uint32_t q_base = smem_addr(s.q) + (u & 1u) * 2 * kTcTile;
        for (int q = 0; q < w.n; q += kTcPages, ++g) {
            const int st = (int)(g % kTcStages);
            if (!tc_wait1(p, s, &s.kv_full[st], (g / kTcStages) & 1u)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t kb = st_base + st * kTcStageBytes + kTcStageK;
            const uint32_t sd = tmem + (g & 1u) * kTcKeys;
#pragma unroll
            for (int kk = 0; kk < kHeadDim / 16; ++kk)
                umma_bf16(sd, umma_desc_sw128(q_base + (kk >> 2) * kTcTile + (kk & 3) * 32),
                          umma_desc_sw128(kb + (kk >> 2) * kTcHalf + (kk & 3) * 32), idesc_s, kk != 0 ? 1u : 0u);
            umma_commit(&s.s_full[g & 1u]);
            if (q + kTcPages >= w.n) umma_commit(&s.q_free[u & 1u]);   // the piece's last product reading Q
            if (g > 0 && !pv(g - 1, prev_first)) {
                ok = false;
                break;
            }
            prev_first = q == 0;
        }
        ++u;
    } while (ok && w.next(s.seg, B));
    if (ok && g > 0) (void)pv(g - 1, prev_first);
    umma_commit(s.fin);   // every instruction issued above has completed
}

// Warps 4-7, thread = row r = 32 * (warp - 4) + lane.
template <int G>
__device__ __forceinline__ void tc_softmax(const Params& p, const PrefillScratch& sc, const TcShared& s, int B,
                                           int start, int end, int per_cta, int r, uint32_t tmem) {
    constexpr int kHq = G * kNumKvHeads;
    const int lane = r & 31;
    const int n = p.new_tokens, R = n * G;
    const bool active = r < R;
    const bool warp_active = (r & ~31) < R;
    const int tt = active ? r / G : 0;
    const uint32_t lanes = tmem + ((uint32_t)(r & ~31) << 16);
    const uint32_t p_row = smem_addr(s.p) + r * 128;
    uint32_t g = 0, pv_seen = 0;
    bool ok = true;
    auto pv_wait = [&](uint32_t x) -> bool {   // O += P_x V_x has completed
        if (pv_seen > x) return true;
        if (!tc_wait_warp(p, s, s.pv_done, x & 1u, lane)) return false;
        pv_seen = x + 1;
        return true;
    };
    PieceWalk w;
    w.begin(s.seg, B, start, end);
    do {
        const int np_b = s.seg[w.b + 1] - s.seg[w.b];
        const int L = s.lens[w.b];
        const int lim = active ? L - n + tt : -1;   // the last cache slot this row sees
        float m = -INFINITY, lsum = 0.f;
        for (int q = 0; q < w.n; q += kTcPages, ++g) {
            const int npg = min(kTcPages, w.n - q);
            const int slot0 = kPage * (w.i0 + q);
            const int st = (int)(g % kTcStages);
            if (!tc_wait_warp(p, s, &s.kv_full[st], (g / kTcStages) & 1u, lane)) {
                ok = false;
                break;
            }
            const uint32_t bad = (uint32_t)s.mask[st];
            {
                // cache rows of the stage that hold nothing valid (after the
                // sequence, past the piece, not copied) may hold any bytes: a
                // NaN there times a zero probability would still give NaN, so
                // their V rows are zeroed (thread r: row r % 64, half r / 64)
                const int kr = r & 63, pg = kr >> 4;
                if (pg >= npg || ((bad >> pg) & 1u) != 0 || slot0 + kr >= L) {
                    const uint32_t row = smem_addr(s.stages + st * kTcStageBytes + kTcStageV + (r >> 6) * kTcHalf) +
                                         kr * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) st_shared_v4(row + 16 * c, 0u, 0u, 0u, 0u);
                }
            }
            uint32_t pw[kTcKeys / 2];
            if (warp_active) {
                if (!tc_wait_warp(p, s, &s.s_full[g & 1u], (g >> 1) & 1u, lane)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t raw[4][16];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld16(lanes + (g & 1u) * kTcKeys + 16 * c, raw[c]);
                tmem_ld_wait();
                float sv[kTcKeys];
                // keys c <= climit are inside this row's causal window and the piece's pages
                const int climit = min(lim - slot0, kPage * npg - 1);
                float mx = -INFINITY;
                if (bad == 0 && climit >= kTcKeys - 1) {
#pragma unroll
                    for (int c = 0; c < kTcKeys; ++c) {
                        sv[c] = __uint_as_float(raw[c >> 4][c & 15]);
                        mx = fmaxf(mx, sv[c]);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < kTcKeys; ++c) {
                        const bool keep = c <= climit && ((bad >> (c >> 4)) & 1u) == 0;
                        sv[c] = keep ? __uint_as_float(raw[c >> 4][c & 15]) : -INFINITY;
                        mx = fmaxf(mx, sv[c]);
                    }
                }
                const bool grow = mx > m + kRescaleThreshold;
                const bool rescale = grow && m != -INFINITY;   // O holds earlier stages of this piece
                if (__any_sync(kFull, rescale)) {
                    if (!pv_wait(g - 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const float a = rescale ? exp2_approx(m - mx) : 1.f;
#pragma unroll 1
                    for (int c = 0; c < kHeadDim / 16; ++c) {
                        uint32_t v[16];
                        tmem_ld16(lanes + kTcTmemO + 16 * c, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * a);
                        tmem_st16(lanes + kTcTmemO + 16 * c, v);
                    }
                    tmem_st_wait();
                    lsum *= a;
                }
                if (grow) m = mx;
                const float mb = m == -INFINITY ? 0.f : m;
#pragma unroll
                for (int c = 0; c < kTcKeys / 2; ++c) {
                    pw[c] = pack_bf2(exp2_approx(sv[2 * c] - mb), exp2_approx(sv[2 * c + 1] - mb));
                    lsum += bf_lo(pw[c]) + bf_hi(pw[c]);
                }
            }
            // The previous stage's product has read the P tile. Every warp
            // waits for it before arriving: p_full counts arrivals, and a warp
            // must not arrive for stage g + 1 before stage g's phase is over.
            if (g > 0 && !pv_wait(g - 1)) {
                ok = false;
                break;
            }
            if (warp_active) {
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    st_shared_v4(p_row + ((c ^ (r & 7)) << 4), pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
            }
            fence_async_shared();
            tc_fence_before();
            mbar_arrive(s.p_full);
        }
        if (!ok) break;
        if (warp_active) {
            // the piece's last product, then o (whole unit) or the partials
            if (!pv_wait(g - 1)) break;
            tc_fence_after();
            const int ustart = 8 * s.seg[w.b] + w.j * np_b;
            const bool whole = ustart / per_cta == (ustart + np_b - 1) / per_cta;
            const int pslot = 2 * (int)blockIdx.x + (w.k == 0 ? 0 : 1);   // the CTA's first piece, else its last
            const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
            uint4* orow = reinterpret_cast<uint4*>(p.o + (pf_token_row(p, w.b, tt) * kHq + G * w.j + r % G) * kHeadDim);
            const size_t prow = (size_t)pslot * kPrefillRows + r;
            float4* arow = reinterpret_cast<float4*>(sc.acc + prow * kHeadDim);
#pragma unroll 1
            for (int c = 0; c < kHeadDim / 16; ++c) {
                uint32_t v[16];
                tmem_ld16(lanes + kTcTmemO + 16 * c, v);
                tmem_ld_wait();
                if (!active) {
                } else if (whole) {
                    uint32_t o8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        o8[e] = pack_bf2(__uint_as_float(v[2 * e]) * inv, __uint_as_float(v[2 * e + 1]) * inv);
                    orow[2 * c] = make_uint4(o8[0], o8[1], o8[2], o8[3]);
                    orow[2 * c + 1] = make_uint4(o8[4], o8[5], o8[6], o8[7]);
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        __stcg(arow + 4 * c + e, make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                                             __uint_as_float(v[4 * e + 2]),
                                                             __uint_as_float(v[4 * e + 3])));
                }
                __syncwarp();
            }
            if (active && !whole) __stcg(sc.ml + prow, make_float2(m, lsum));
        }
    } while (ok && w.next(s.seg, B));
}

template <int G>
__global__ void __launch_bounds__(kTcThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, const Params p,
                   const PrefillScratch sc) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    // the tiles start on a 1024-byte boundary (the swizzle atom)
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    TcShared s;
    s.stages = smem;
    s.q = smem + kTcSmemQ;
    s.p = smem + kTcSmemP;
    s.seg = reinterpret_cast<int*>(smem + kTcSmemSeg);
    s.lens = reinterpret_cast<int*>(smem + kTcSmemLens);
    s.mask = reinterpret_cast<volatile int*>(smem + kTcSmemMask);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTcSmemBars);
    s.kv_full = bars;
    s.kv_empty = bars + kTcStages;
    s.s_full = bars + 2 * kTcStages;
    s.p_full = s.s_full + 2;
    s.pv_done = s.p_full + 1;
    s.q_full = s.pv_done + 1;
    s.q_free = s.q_full + 2;
    s.fin = s.q_free + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kTcSmemTmem);
    s.abort_flag = reinterpret_cast<volatile int*>(smem + kTcSmemTmem + 4);

    // The prologue touches no global memory; griddepcontrol.wait then holds
    // until the prep launch has completed and its writes are visible.
    if (threadIdx.x == 0) {
        for (int k = 0; k < kTcStages; ++k) {
            mbar_init(&s.kv_full[k], 1);
            mbar_init(&s.kv_empty[k], 1);
        }
        mbar_init(&s.s_full[0], 1);
        mbar_init(&s.s_full[1], 1);
        mbar_init(s.p_full, 4 * 32);
        mbar_init(s.pv_done, 1);
        for (int k = 0; k < 2; ++k) {
            mbar_init(&s.q_full[k], 1);
            mbar_init(&s.q_free[k], 1);
        }
        mbar_init(s.fin, 1);
        *s.abort_flag = 0;
        s.seg[0] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTcTmemCols);
    pdl_wait();
    const int B = p.batch;
    for (int b = threadIdx.x; b < B; b += kTcThreads) {
        const int L_all = p.seq_lens[b];
        const bool ok = length_ok(p, L_all);
        if (!ok && blockIdx.x == 0) record_error(p.status, QDA_ERR_BOUNDS);
        const int L = ok ? L_all - p.len_trim : 0;
        s.lens[b] = L;
        s.seg[b + 1] = ok ? (L + kPage - 1) / kPage : 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
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
        for (int b = threadIdx.x; b <= B; b += kTcThreads) p.seg[b] = s.seg[b];

    const int total = kNumKvHeads * s.seg[B];   // page-heads
    const int per_cta = (total + (int)gridDim.x - 1) / (int)gridDim.x;
    const int start = (int)blockIdx.x * per_cta;
    const int end = min(start + per_cta, total);
    if (start < end) {
        if (warp == 0) {
            tc_producer(p, sc, s, &tm_k, &tm_v, B, start, end, lane);
        } else if (warp == 1) {
            if (lane == 0) {
                tc_issuer(p, s, B, start, end, tmem);
                // nothing may still write tensor memory when it is freed
                (void)mbar_wait(s.fin, 0u, p.timeout_ns, nullptr);
            }
        } else if (warp >= 4) {
            tc_softmax<G>(p, sc, s, B, start, end, per_cta, threadIdx.x - 128, tmem);
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTcTmemCols);
    }
    pdl_launch_dependents();
}

// ---------------------------------------------------------------------------
// 3. The combine: warp w of CTA (b, j, z) merges row 8z + w of unit (b, j)
// when the unit was split across CTAs; lane l holds dims 4l..4l+3. The unit's
// pieces sit in consecutive CTAs g0..gk of the attention launch: slot 2*g0 + 1
// when the unit starts inside g0's range (it is g0's last piece), else 2*g0;
// slot 2*g in the later CTAs.
template <int G>
__global__ void __launch_bounds__(256) prefill_combine_kernel(const Params p, const PrefillScratch sc) {
    constexpr int kHq = G * kNumKvHeads;
    pdl_wait();
    pdl_launch_dependents();
    const int b = blockIdx.x, j = blockIdx.y, lane = threadIdx.x & 31;
    const int r = 8 * (int)blockIdx.z + (int)(threadIdx.x >> 5);
    if (r >= p.new_tokens * G) return;
    const int np = p.seg[b + 1] - p.seg[b];
    if (np == 0) return;   // a sequence the attention launch skipped
    const int total = kNumKvHeads * p.seg[p.batch];
    const int per_cta = (total + sc.grid - 1) / sc.grid;
    const int ustart = kNumKvHeads * p.seg[b] + j * np;
    const int g0 = ustart / per_cta, gk = (ustart + np - 1) / per_cta;
    if (g0 == gk) return;   // held whole by one CTA, which wrote o
    const int first = ustart % per_cta != 0 ? 2 * g0 + 1 : 2 * g0;   // slot of piece 0; piece k > 0: 2 * (g0 + k)
    const int pieces = gk - g0 + 1;
    float M = -INFINITY;
    for (int k = lane; k < pieces; k += 32) {
        const int slot = k == 0 ? first : 2 * (g0 + k);
        M = fmaxf(M, __ldcg(sc.ml + (size_t)slot * kPrefillRows + r).x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
    float Ls = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int k = 0; k < pieces; ++k) {
        const size_t prow = (size_t)(k == 0 ? first : 2 * (g0 + k)) * kPrefillRows + r;
        const float2 ml = __ldcg(sc.ml + prow);
        const float4 x = __ldcg(reinterpret_cast<const float4*>(sc.acc + prow * kHeadDim) + lane);
        const float wt = (ml.x == -INFINITY) ? 0.f : exp2_approx(ml.x - M);   // a piece that saw no slot
        Ls = fmaf(wt, ml.y, Ls);
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
    cfg.gridDim = dim3((unsigned)p.batch, (unsigned)kNumKvHeads, (unsigned)((p.new_tokens + 3) / 4));
    cfg.blockDim = dim3(128, 1, 1);
    cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_prep_kernel<G>, p, sc);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)sc.grid, 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = kTcSmemAlloc;
    e = cudaLaunchKernelEx(&cfg, prefill_kernel<G>, tk, tv, p, sc);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)p.batch, (unsigned)kNumKvHeads, (unsigned)((p.new_tokens * G + 7) / 8));
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, prefill_combine_kernel<G>, p, sc);
}

}  // namespace

cudaError_t prepare_prefill() {
    if (pf_encode_fn() == nullptr) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemAlloc);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(prefill_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemAlloc);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(prefill_kernel<5>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemAlloc);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(prefill_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemAlloc);
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
