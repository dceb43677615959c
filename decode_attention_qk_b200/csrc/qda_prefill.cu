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
//      takes a range of it of equal cost (pages plus a fixed cost per unit
//      piece), whatever the length mix. Per unit piece
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
// 1. The prep: warp w of CTA (b, j, z) takes token u = 8z + w of the chunk.
// It forms the token's new k (RMSNorm and RoPE in double, rounded once to
// bf16) and writes k and v to their cache slots, and forms the token's G query
// rows of kv head j (RMSNorm and RoPE in float, the angle reduced modulo 2*pi
// in double, scaled by log2(e)/sqrt(128), rounded to bf16) into the unit's
// query tile in the attention's layout. Lane l holds dims 2l, 2l+1 (word l of
// a head) and 64+2l, 65+2l (word 32+l), the RoPE pairs (i, i+64).

template <int G>
__global__ void __launch_bounds__(256) prefill_prep_kernel(const Params p, const PrefillScratch sc) {
    constexpr int kHq = G * kNumKvHeads;
    constexpr int kQkvW = (kHq + 2 * kNumKvHeads) * kHeadDim;
    __shared__ double inv_freq[kHeadDim / 2];   // theta^(-2i/128), shared by the CTA's tokens
    if (threadIdx.x < kHeadDim / 2) inv_freq[threadIdx.x] = pow(p.rope_theta, -2.0 * (int)threadIdx.x / 128.0);
    pdl_wait();
    pdl_launch_dependents();
    __syncthreads();
    const int b = blockIdx.x, j = blockIdx.y, lane = threadIdx.x & 31;
    const int u = 8 * (int)blockIdx.z + (int)(threadIdx.x >> 5);
    const int n = p.new_tokens;
    if (u >= n) return;
    const int L_all = p.seq_lens[b];
    if (!length_ok(p, L_all)) return;   // the attention launch records it and skips the sequence
    const int L = L_all - p.len_trim;
    const double pos = (double)(pf_first_position(p, b, L, n) + u);
    const double ang0 = reduce_angle(pos * inv_freq[2 * lane]);
    const double ang1 = reduce_angle(pos * inv_freq[2 * lane + 1]);
    // every load first (the token's k, v and G query rows, the gains, the
    // page), so that their latencies overlap
    const uint32_t* row = reinterpret_cast<const uint32_t*>(p.qkv + pf_token_row(p, b, u) * kQkvW);
    const uint32_t* xk = row + (kHq + j) * (kHeadDim / 2);
    const uint32_t* xv = row + (kHq + kNumKvHeads + j) * (kHeadDim / 2);
    const uint32_t klo = xk[lane], khi = xk[32 + lane];
    const uint32_t vlo = xv[lane], vhi = xv[32 + lane];
    uint32_t qlo[G], qhi[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
        qlo[hh] = row[(G * j + hh) * (kHeadDim / 2) + lane];
        qhi[hh] = row[(G * j + hh) * (kHeadDim / 2) + 32 + lane];
    }
    const uint32_t* gk = reinterpret_cast<const uint32_t*>(p.k_norm_w);
    const uint32_t wk_lo = gk[lane], wk_hi = gk[32 + lane];
    const uint32_t* gq = reinterpret_cast<const uint32_t*>(p.q_norm_w);
    const uint32_t wq_lo = gq[lane], wq_hi = gq[32 + lane];
    const int slot = L - n + u;
    const int page = __ldg(p.block_table + (size_t)b * p.bt_stride + slot / kPage);

    {
        double a0 = bf_to_d(klo & 0xFFFFu), a1 = bf_to_d(klo >> 16);
        double b0 = bf_to_d(khi & 0xFFFFu), b1 = bf_to_d(khi >> 16);
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
        if (page >= 0 && page < p.num_pages) {   // else recorded by the attention launch
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

    float sn0, cs0, sn1, cs1;
    sincosf((float)ang0, &sn0, &cs0);
    sincosf((float)ang1, &sn1, &cs1);
    const float scale = (float)kQScale;
    uint8_t* tile = reinterpret_cast<uint8_t*>(sc.q) + (size_t)(b * kNumKvHeads + j) * kPrefillQTileBytes;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
        const int r = u * G + hh;
        const uint32_t xlo = qlo[hh], xhi = qhi[hh];
        float ss =
            bf_lo(xlo) * bf_lo(xlo) + bf_hi(xlo) * bf_hi(xlo) + bf_lo(xhi) * bf_lo(xhi) + bf_hi(xhi) * bf_hi(xhi);
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
//   softmax       one thread per row and half of the stage's keys (two
//                 warpgroups): the causal and length mask, the running max
//                 with lazy rescaling of O, P = exp2(S - m) rounded to bf16
//                 into tensor memory (the running sum adds the same rounded
//                 values, so o stays a convex combination of v rows);
//   O += P V      M = 128 rows, N = 128 dims, K = 64 keys, P read from
//                 tensor memory and V MN-major from its copied tile;
// and O, accumulated in tensor memory over the piece, is read out once at the
// piece's end.
//
// Warp roles (384 threads): warps 0 and 3 issue the copies of K (and Q) and
// of V; one thread of warp 1 issues S and one of warp 2 issues O += P V (warp
// 1 also allocates tensor memory); warps 4-11 run the softmax in two
// warpgroups, each over half of a stage's keys with an accumulator of its
// own, and write o. Every wait is bounded: a timeout records QDA_ERR_TIMEOUT,
// sets the CTA's abort flag and every role leaves its loop; tensor memory is
// freed after every issued instruction has completed.

constexpr int kTcKeys = 64;                          // cache rows per stage
constexpr int kTcPages = kTcKeys / kPage;            // 4
// K and V sit in rings of their own: a K slot is free once S has read it, a V
// slot only once O += P V has. A stage stays in a V slot from its copy through
// S, the softmax and the product, so the V ring is the deeper one: with about
// three stages held in processing it still keeps two or more in flight.
constexpr int kTcKSlots = 4;
constexpr int kTcVSlots = 6;
constexpr int kTcThreads = 12 * 32;
constexpr int kTcHalf = kTcKeys * 128;               // 64 dims of a stage's rows: 8 KiB
constexpr int kTcSlotBytes = 2 * kTcHalf;            // a K or V slot: dims 0-63 | dims 64-127
constexpr int kTcBoxBytes = kPage * 128;             // one copied box: 16 rows x 64 dims
constexpr int kTcTile = kPrefillRows * 128;          // 64 columns of a 128-row operand: 16 KiB
// Shared memory: the small items first, then the tiles on the next 1024-byte
// boundary (the swizzle atom).
// k_full[K], k_empty[K], v_full[V], v_empty[V], s_full[2], p_full[2],
// pv_done[2], q_full[2], q_free[2], ml_ready[2], fin, never (the test hook's)
constexpr int kTcNumBars = 2 * kTcKSlots + 2 * kTcVSlots + 14;
constexpr int kTcSmemTmem = kTcNumBars * 8;                          // tensor-memory address, abort flag
constexpr int kTcSmemMask = kTcSmemTmem + 16;                        // int [kTcVSlots]: pages not copied
constexpr int kTcSmemSeg = kTcSmemMask + kTcVSlots * 4;              // int [kMaxBatch + 4]
constexpr int kTcSmall = (kTcSmemSeg + (kMaxBatch + 4) * 4 + 15) / 16 * 16;
constexpr int kTcTileV = kTcKSlots * kTcSlotBytes;   // from the tiles' start: K ring, V ring,
constexpr int kTcTileQ = kTcTileV + kTcVSlots * kTcSlotBytes;   // 2 buffers of Q dims 0-63 | 64-127
constexpr int kTcTiles = kTcTileQ + 4 * kTcTile;
constexpr int kTcSmemAlloc = kTcSmall + 1024 + kTcTiles;   // with up to 1023 bytes of padding
// tensor-memory columns: S buffers at 0 and 64, O_0 at 128, O_1 at 256, the
// (m, l) swap at 384, P buffers (64 bf16 keys in 32 columns) at 416 and 448
constexpr uint32_t kTcTmemCols = 512;
constexpr uint32_t kTcTmemO = 128;
constexpr uint32_t kTcTmemMl = 384;
constexpr uint32_t kTcTmemP = 416;
static_assert(kTcSlotBytes % 1024 == 0 && kTcTile % 1024 == 0, "swizzle atoms are 1024-byte aligned");
static_assert(kTcSmall % 16 == 0 && 2 * kTcTile == kPrefillQTileBytes, "layout");
static_assert(kTcSmemAlloc <= 227 * 1024, "fits one CTA per SM");
static_assert(kTcKeys == 64, "a P row is one 128-byte swizzled row");

struct TcShared {
    uint8_t* k;          // K ring
    uint8_t* v;          // V ring
    uint8_t* q;
    int* seg;
    volatile int* mask;  // [kTcVSlots]: pages of the stage in V slot i that were not copied
    uint64_t* k_full;
    uint64_t* k_empty;
    uint64_t* v_full;
    uint64_t* v_empty;
    uint64_t* s_full;    // [2]: S of stage g in S buffer g % 2
    uint64_t* p_full;    // [2]: P of stage g written into P buffer g % 2
    uint64_t* pv_done;   // [2]: O += P V of stage g (g % 2) completed
    uint64_t* q_full;    // [2]
    uint64_t* q_free;    // [2]
    uint64_t* ml_ready;  // [2]: both warpgroups have posted (m, l) of piece u (u % 2)
    uint64_t* fin;
    uint64_t* never;
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

// The split of the page-head list over the CTAs. Besides its pages, every
// unit (b, j) costs kPieceCost page equivalents of fixed work where a CTA
// holds a piece of it (the pipeline's drain, the merge of the halves, the
// output; 12 was the best of the settings measured, 3 to 24). CTA g takes
// page-heads [pf_split(g), pf_split(g + 1)): the points where the running
// cost, units in order with each unit's fixed cost before its pages, crosses
// g * w, w the total over the grid. seg is the page prefix of the sequences.
constexpr int kPieceCost = 12;

__device__ __forceinline__ int pf_cost_before(const int* seg, int b) { return 8 * (seg[b] + kPieceCost * b); }

__device__ __forceinline__ int pf_split(const int* seg, int B, int grid, int g) {
    const int W = pf_cost_before(seg, B);
    const int w = (W + grid - 1) / grid;
    const long long t = (long long)g * w;
    if (t >= W) return 8 * seg[B];
    int lo = 0, hi = B - 1;   // the sequence whose cost range holds t
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pf_cost_before(seg, mid) <= t) lo = mid; else hi = mid - 1;
    }
    const int np = seg[lo + 1] - seg[lo];
    const int r = (int)t - pf_cost_before(seg, lo);          // < 8 * (np + kPieceCost)
    const int j = min(kNumKvHeads - 1, r / (np + kPieceCost));
    const int off = r - j * (np + kPieceCost) - kPieceCost;   // pages into unit (lo, j); < np
    return 8 * seg[lo] + j * np + max(0, off);
}

// One thread's bounded wait; a failure aborts the CTA.
__device__ __forceinline__ bool tc_wait1(const Params& p, const TcShared& s, uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    if (mbar_wait(bar, parity, p.timeout_ns, s.abort_flag)) return true;
    *s.abort_flag = 1;
    record_error(p.status, QDA_ERR_TIMEOUT);
    return false;
}

// A whole warp's bounded wait, with one outcome for all its lanes.
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

// The copies, one warp per ring: warp 0 fills the K ring (and copies each
// piece's query tile), warp 3 the V ring. Each looks the page ids up 32
// page-heads at a time, then per stage issues two tiled copies per page (kv
// head j, dims 0-63 and 64-127) into the slot's halves at 2 KiB per page.
// Pages whose block-table entry is out of range are not copied; the V warp's
// mask of them tells the softmax.
template <bool kIsV>
__device__ __forceinline__ void tc_producer(const Params& p, const PrefillScratch& sc, const TcShared& s,
                                            const CUtensorMap* tm, int B, int start, int end, int lane) {
    constexpr int kSlots = kIsV ? kTcVSlots : kTcKSlots;
    uint64_t* full = kIsV ? s.v_full : s.k_full;
    uint64_t* empty = kIsV ? s.v_empty : s.k_empty;
    uint8_t* ring = kIsV ? s.v : s.k;
    const uint32_t q_bytes = (uint32_t)(p.new_tokens * (p.num_q_heads / kNumKvHeads)) * 128u;   // R rows per half
    int wbase = 0x40000000, id = -1;
    uint32_t g = 0, u = 0, armed = 0, armed_parity = 0, q_armed = 0;
    bool ok = true;
    asm volatile("fence.proxy.async.global;" ::: "memory");   // the copies read what the prep launch wrote
    PieceWalk w;
    w.begin(s.seg, B, start, end);
    do {
        if (!kIsV) {
            // the piece's query tile, into buffer u % 2 once the piece two back
            // has finished reading it
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
        if (!kIsV && lane == 0) {
            // for the combine launch: the slot of the unit's first piece, the CTA of its last
            int2* unit = sc.unit + w.b * kNumKvHeads + w.j;
            if (w.i0 == 0) unit->x = 2 * (int)blockIdx.x + (w.k == 0 ? 0 : 1);
            if (w.i0 + w.n == np_b) unit->y = (int)blockIdx.x;
        }
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
            const int st = (int)(g % kSlots);
            int good = 1;
            if (lane == 0 && g >= (uint32_t)kSlots) good = tc_wait1(p, s, &empty[st], ((g / kSlots) - 1) & 1u) ? 1 : 0;
            if (!__shfl_sync(kFull, good, 0)) {
                ok = false;
                break;
            }
            const int my = __shfl_sync(kFull, id, (x0 - wbase + lane) & 31);
            const uint32_t bad = __ballot_sync(kFull, lane < npg && (my < 0 || my >= p.num_pages));
            if (lane == 0) {
                if (kIsV) {
                    s.mask[st] = (int)bad;
                    if (bad != 0) record_error(p.status, QDA_ERR_BOUNDS);
                }
                const int copied = npg - __popc(bad);
                if (copied > 0) {
                    mbar_arrive_expect_tx(&full[st], (uint32_t)(copied * 2 * kTcBoxBytes));
                    armed |= 1u << st;
                    armed_parity = (armed_parity & ~(1u << st)) | (((g / kSlots) & 1u) << st);
                } else {
                    mbar_arrive(&full[st]);
                }
            }
            const uint32_t dst = smem_addr(ring + st * kTcSlotBytes);
            for (int k = 0; k < npg; ++k) {
                const int page = __shfl_sync(kFull, my, k);
                if (lane == 0 && ((bad >> k) & 1u) == 0) {
                    tma_load_3d(dst + k * kTcBoxBytes, tm, 0, w.j, page * kPage, &full[st]);
                    tma_load_3d(dst + kTcHalf + k * kTcBoxBytes, tm, 64, w.j, page * kPage, &full[st]);
                }
            }
        }
    } while (ok && w.next(s.seg, B));
    if (lane == 0 && *s.abort_flag != 0) {
        // copies still landing in this CTA's shared memory: wait (bounded) for each
        for (int k = 0; k < kSlots; ++k)
            if (armed & (1u << k)) (void)mbar_wait(&full[k], (armed_parity >> k) & 1u, p.timeout_ns, nullptr);
        for (int k = 0; k < 2; ++k)
            if ((q_armed >> (2 * k)) & 2u)
                (void)mbar_wait(&s.q_full[k], (q_armed >> (2 * k)) & 1u, p.timeout_ns, nullptr);
    }
}

// The tensor-core instructions come from two threads, so that their issue
// (about 0.05 us per instruction and thread, whatever its size) runs in two
// streams: one issues S, the other O += P V.
//
// Lane 0 of warp 1: per stage g, S_g = Q K_g^T into S buffer g % 2, once K_g
// has landed and the softmax of stage g - 2 has finished reading that buffer
// (it read S before writing P_{g-2}); the K slot is free once S_g completes.
__device__ __forceinline__ void tc_issue_s(const Params& p, const TcShared& s, int B, int start, int end,
                                           uint32_t tmem) {
    const uint32_t idesc_s = umma_idesc_bf16_m128(kTcKeys);
    const uint32_t k_base = smem_addr(s.k);
    uint32_t g = 0, u = 0;
    bool ok = true;
    PieceWalk w;
    w.begin(s.seg, B, start, end);
    do {
        if (!tc_wait1(p, s, &s.q_full[u & 1u], (u >> 1) & 1u)) break;
        tc_fence_after();
        const uint32_t q_base = smem_addr(s.q) + (u & 1u) * 2 * kTcTile;
        for (int q = 0; q < w.n; q += kTcPages, ++g) {
            const int st = (int)(g % kTcKSlots);
            if (!tc_wait1(p, s, &s.k_full[st], (g / kTcKSlots) & 1u) ||
                (g >= 2 && !tc_wait1(p, s, &s.p_full[g & 1u], ((g - 2) >> 1) & 1u))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t kb = k_base + st * kTcSlotBytes;
            const uint32_t sd = tmem + (g & 1u) * kTcKeys;
#pragma unroll
            for (int kk = 0; kk < kHeadDim / 16; ++kk)
                umma_bf16(sd, umma_desc_sw128(q_base + (kk >> 2) * kTcTile + (kk & 3) * 32),
                          umma_desc_sw128(kb + (kk >> 2) * kTcHalf + (kk & 3) * 32), idesc_s, kk != 0 ? 1u : 0u);
            umma_commit(&s.s_full[g & 1u]);
            umma_commit(&s.k_empty[st]);
            if (q + kTcPages >= w.n) umma_commit(&s.q_free[u & 1u]);   // the piece's last product reading Q
        }
        ++u;
    } while (ok && w.next(s.seg, B));
    umma_commit(s.fin);   // counts once every instruction issued above has completed
}

// Lane 0 of warp 2: per stage x, once both softmax warpgroups have written
// P_x into tensor-memory P buffer x % 2, O_0 += P_x[:, 0:32] V_x[0:32] and
// O_1 += P_x[:, 32:64] V_x[32:64], each accumulator starting afresh at its
// piece's first stage; the V slot and the P buffer are free once these
// complete.
__device__ __forceinline__ void tc_issue_pv(const Params& p, const TcShared& s, int B, int start, int end,
                                            uint32_t tmem) {
    const uint32_t idesc_o = umma_idesc_bf16_m128_bmn(kHeadDim);
    const uint32_t v_base = smem_addr(s.v);
    uint32_t x = 0;
    bool ok = true;
    PieceWalk w;
    w.begin(s.seg, B, start, end);
    do {
        for (int q = 0; q < w.n; q += kTcPages, ++x) {
            if (!tc_wait1(p, s, &s.p_full[x & 1u], (x >> 1) & 1u)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t v = v_base + (x % kTcVSlots) * kTcSlotBytes;
            const uint32_t pa = tmem + kTcTmemP + (x & 1u) * (kTcKeys / 2);
#pragma unroll
            for (int kk = 0; kk < kTcKeys / 16; ++kk)   // 16 keys (8 columns) per instruction; keys 32h.. go to O_h
                umma_bf16_ts(tmem + kTcTmemO + (kk >> 1) * kHeadDim, pa + 8 * kk,
                             umma_desc_sw128_mn(v + 2 * 1024 * kk, kTcHalf, 1024), idesc_o,
                             (q == 0 && (kk & 1) == 0) ? 0u : 1u);
            umma_commit(&s.pv_done[x & 1u]);
            umma_commit(&s.v_empty[x % kTcVSlots]);
        }
    } while (ok && w.next(s.seg, B));
    umma_commit(s.fin);
}

// Warps 4-11, two warpgroups: thread t owns row r = t % 128 and keys 32h ..
// 32h + 31 of every stage, h = t / 128 (warp 4 + 4h + q reads tensor-memory
// lanes 32q..32q+31), with its own running max m_h, sum l_h and accumulator
// O_h. At a piece's end the halves are merged (the log-sum-exp rule):
//   M = max(m_0, m_1), a_h = exp2(m_h - M),
//   o = (a_0 O_0 + a_1 O_1) / (a_0 l_0 + a_1 l_1),
// warpgroup h writing dims 64h .. 64h + 63, after the two have swapped (m, l)
// through tensor memory.
template <int G>
__device__ __forceinline__ void tc_softmax(const Params& p, const PrefillScratch& sc, const TcShared& s, int B,
                                           int start, int end, int t, uint32_t tmem) {
    constexpr int kHq = G * kNumKvHeads;
    const int r = t & 127, h = t >> 7, lane = t & 31;
    const int n = p.new_tokens, R = n * G;
    const bool active = r < R;
    const bool warp_active = (r & ~31) < R;
    const int tt = active ? r / G : 0;
    const uint32_t lanes = tmem + ((uint32_t)(r & ~31) << 16);
    const uint32_t o_own = lanes + kTcTmemO + (uint32_t)h * kHeadDim;
    uint32_t g = 0, u = 0, pv_seen[2] = {0u, 0u};
    bool ok = true;
    // O += P_x V_x has completed: completion x / 2 of pv_done[x % 2]. The
    // phases of each barrier are waited for in order, and none can complete
    // two ahead of this warp (P_{x+2} is written after this wait).
    auto pv_wait = [&](uint32_t x) -> bool {
        const uint32_t k = x & 1u, c = x >> 1;
        if (pv_seen[k] > c) return true;
        if (!tc_wait_warp(p, s, &s.pv_done[k], c & 1u, lane)) return false;
        pv_seen[k] = c + 1;
        return true;
    };
    PieceWalk w;
    w.begin(s.seg, B, start, end);
    do {
        const int np_b = s.seg[w.b + 1] - s.seg[w.b];
        const int L = p.seq_lens[w.b] - p.len_trim;   // the piece's sequence passed the length checks
        const int lim = active ? L - n + tt : -1;     // the last cache slot this row sees
        float m = -INFINITY, lsum = 0.f;
        for (int q = 0; q < w.n; q += kTcPages, ++g) {
            const int npg = min(kTcPages, w.n - q);
            const int slot0 = kPage * (w.i0 + q);
            const int st = (int)(g % kTcVSlots);
            if (!tc_wait_warp(p, s, &s.v_full[st], (g / kTcVSlots) & 1u, lane)) {
                ok = false;
                break;
            }
            const uint32_t bad = (uint32_t)s.mask[st];
            if (h == 0) {
                // cache rows of the stage that hold nothing valid (after the
                // sequence, past the piece, not copied) may hold any bytes: a
                // NaN there times a zero probability would still give NaN, so
                // their V rows are zeroed (thread r: row r % 64, half r / 64)
                const int kr = r & 63, pg = kr >> 4;
                if (pg >= npg || ((bad >> pg) & 1u) != 0 || slot0 + kr >= L) {
                    const uint32_t row = smem_addr(s.v + st * kTcSlotBytes + (r >> 6) * kTcHalf) + kr * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) st_shared_v4(row + 16 * c, 0u, 0u, 0u, 0u);
                    fence_async_shared();   // visible to the tensor cores' proxy before the arrival below
                }
            }
            uint32_t pw[8];
            if (warp_active) {
                if (!tc_wait_warp(p, s, &s.s_full[g & 1u], (g >> 1) & 1u, lane)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t raw[2][16];
                tmem_ld16(lanes + (g & 1u) * kTcKeys + 32 * h, raw[0]);
                tmem_ld16(lanes + (g & 1u) * kTcKeys + 32 * h + 16, raw[1]);
                tmem_ld_wait();
                float sv[32];
                // key 32h + c is inside this row's causal window and the piece's pages when c <= climit
                const int climit = min(lim - slot0, kPage * npg - 1) - 32 * h;
                const uint32_t badh = (bad >> (2 * h)) & 3u;   // pages 2h, 2h + 1 of the stage
                float mx = -INFINITY;
                if (badh == 0 && climit >= 31) {
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        sv[c] = __uint_as_float(raw[c >> 4][c & 15]);
                        mx = fmaxf(mx, sv[c]);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const bool keep = c <= climit && ((badh >> (c >> 4)) & 1u) == 0;
                        sv[c] = keep ? __uint_as_float(raw[c >> 4][c & 15]) : -INFINITY;
                        mx = fmaxf(mx, sv[c]);
                    }
                }
                const bool grow = mx > m + kRescaleThreshold;
                const bool rescale = grow && m != -INFINITY;   // O_h holds earlier stages of this piece
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
                        tmem_ld16(o_own + 16 * c, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * a);
                        tmem_st16(o_own + 16 * c, v);
                    }
                    tmem_st_wait();
                    lsum *= a;
                }
                if (grow) m = mx;
                const float mb = m == -INFINITY ? 0.f : m;
                const f32x2 nmb = pack2(-mb, -mb);
                f32x2 ls2 = pack2(0.f, 0.f);   // even and odd keys' sums, one packed add per pair
                uint32_t pw2[8];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float2 d = unpack2(add2(pack2(sv[2 * c], sv[2 * c + 1]), nmb));
                    const uint32_t wv = pack_bf2(exp2_approx(d.x), exp2_approx(d.y));
                    if (c < 8) pw[c] = wv;
                    else pw2[c - 8] = wv;
                    ls2 = add2(ls2, bf2(wv));
                }
                const float2 lsp = unpack2(ls2);
                lsum += lsp.x + lsp.y;
                // the product of stage g - 2 has read P buffer g % 2
                if (g > 1 && !pv_wait(g - 2)) {
                    ok = false;
                    break;
                }
                uint32_t pcol[16];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    pcol[c] = pw[c];
                    pcol[8 + c] = pw2[c];
                }
                tmem_st16(lanes + kTcTmemP + (g & 1u) * (kTcKeys / 2) + 16 * h, pcol);
                tmem_st_wait();
            } else if (g > 1 && !pv_wait(g - 2)) {
                // every warp waits before arriving: p_full[g % 2] counts
                // arrivals, and none may arrive for stage g + 2 before stage
                // g's phase is over
                ok = false;
                break;
            }
            // one arrival per warp, once every lane's P (and V zeroing) is in place
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.p_full[g & 1u]);
        }
        if (!ok) break;
        // The piece's last products, then the merge of the two halves: o
        // (unit held whole) or the partials.
        const uint32_t ml_col = kTcTmemMl + 4 * (u & 1u);
        if (warp_active) {
            if (!pv_wait(g - 1)) break;
            tc_fence_after();
            const uint32_t mine[2] = {__float_as_uint(m), __float_as_uint(lsum)};
            tmem_st2(lanes + ml_col + 2 * h, mine);
            tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.ml_ready[u & 1u]);
        if (!tc_wait_warp(p, s, &s.ml_ready[u & 1u], (u >> 1) & 1u, lane)) break;
        if (warp_active) {
            tc_fence_after();
            uint32_t other[2];
            tmem_ld2(lanes + ml_col + 2 * (1 - h), other);
            tmem_ld_wait();
            const float m0 = h == 0 ? m : __uint_as_float(other[0]), l0 = h == 0 ? lsum : __uint_as_float(other[1]);
            const float m1 = h == 0 ? __uint_as_float(other[0]) : m, l1 = h == 0 ? __uint_as_float(other[1]) : lsum;
            const float M = fmaxf(m0, m1);
            const float a0 = m0 == -INFINITY ? 0.f : exp2_approx(m0 - M);
            const float a1 = m1 == -INFINITY ? 0.f : exp2_approx(m1 - M);
            const float Lt = a0 * l0 + a1 * l1;
            const bool whole = w.i0 == 0 && w.n == np_b;   // this CTA holds the whole unit
            const int pslot = 2 * (int)blockIdx.x + (w.k == 0 ? 0 : 1);   // the CTA's first piece, else its last
            const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
            uint4* orow = reinterpret_cast<uint4*>(p.o + (pf_token_row(p, w.b, tt) * kHq + G * w.j + r % G) * kHeadDim);
            const size_t prow = (size_t)pslot * kPrefillRows + r;
            float4* arow = reinterpret_cast<float4*>(sc.acc + prow * kHeadDim);
#pragma unroll 1
            for (int c = 4 * h; c < 4 * h + 4; ++c) {   // dims 16c .. 16c + 15
                uint32_t v0[16], v1[16];
                tmem_ld16(lanes + kTcTmemO + 16 * c, v0);
                tmem_ld16(lanes + kTcTmemO + kHeadDim + 16 * c, v1);
                tmem_ld_wait();
                float x[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) x[e] = a0 * __uint_as_float(v0[e]) + a1 * __uint_as_float(v1[e]);
                if (!active) {
                } else if (whole) {
                    uint32_t o8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) o8[e] = pack_bf2(x[2 * e] * inv, x[2 * e + 1] * inv);
                    orow[2 * c] = make_uint4(o8[0], o8[1], o8[2], o8[3]);
                    orow[2 * c + 1] = make_uint4(o8[4], o8[5], o8[6], o8[7]);
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        __stcg(arow + 4 * c + e, make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]));
                }
                __syncwarp();
            }
            if (active && !whole && h == 0) __stcg(sc.ml + prow, make_float2(M, Lt));
        }
        ++u;
    } while (ok && w.next(s.seg, B));
}

template <int G>
__global__ void __launch_bounds__(kTcThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, const Params p,
                   const PrefillScratch sc) {
    extern __shared__ __align__(16) uint8_t smem[];
    // the tiles start on the first 1024-byte boundary after the small items
    uint8_t* tiles = smem + kTcSmall + ((1024u - ((smem_addr(smem) + kTcSmall) & 1023u)) & 1023u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    TcShared s;
    s.k = tiles;
    s.v = tiles + kTcTileV;
    s.q = tiles + kTcTileQ;
    s.seg = reinterpret_cast<int*>(smem + kTcSmemSeg);
    s.mask = reinterpret_cast<volatile int*>(smem + kTcSmemMask);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    s.k_full = bars;
    s.k_empty = s.k_full + kTcKSlots;
    s.v_full = s.k_empty + kTcKSlots;
    s.v_empty = s.v_full + kTcVSlots;
    s.s_full = s.v_empty + kTcVSlots;
    s.p_full = s.s_full + 2;
    s.pv_done = s.p_full + 2;
    s.q_full = s.pv_done + 2;
    s.q_free = s.q_full + 2;
    s.ml_ready = s.q_free + 2;
    s.fin = s.ml_ready + 2;
    s.never = s.fin + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kTcSmemTmem);
    s.abort_flag = reinterpret_cast<volatile int*>(smem + kTcSmemTmem + 4);

    // The prologue touches no global memory; griddepcontrol.wait then holds
    // until the prep launch has completed and its writes are visible.
    if (threadIdx.x == 0) {
        for (int k = 0; k < kTcKSlots; ++k) {
            mbar_init(&s.k_full[k], 1);
            mbar_init(&s.k_empty[k], 1);
        }
        for (int k = 0; k < kTcVSlots; ++k) {
            mbar_init(&s.v_full[k], 1);
            mbar_init(&s.v_empty[k], 1);
        }
        mbar_init(&s.s_full[0], 1);
        mbar_init(&s.s_full[1], 1);
        for (int k = 0; k < 2; ++k) {
            mbar_init(&s.p_full[k], 8);     // one arrival per softmax warp
            mbar_init(&s.pv_done[k], 1);
            mbar_init(&s.ml_ready[k], 8);
            mbar_init(&s.q_full[k], 1);
            mbar_init(&s.q_free[k], 1);
        }
        mbar_init(s.fin, 2);
        mbar_init(s.never, 1);
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
    const int start = pf_split(s.seg, B, (int)gridDim.x, (int)blockIdx.x);
    const int end = min(pf_split(s.seg, B, (int)gridDim.x, (int)blockIdx.x + 1), total);
    if (start < end) {
        if (warp == 0 || warp == 3) {
            if (warp == 0) tc_producer<false>(p, sc, s, &tm_k, B, start, end, lane);
            else tc_producer<true>(p, sc, s, &tm_v, B, start, end, lane);
        } else if (warp == 1 || warp == 2) {
            if (lane == 0) {
                if (warp == 1) tc_issue_s(p, s, B, start, end, tmem);
                else tc_issue_pv(p, s, B, start, end, tmem);
                // nothing may still write tensor memory when it is freed
                (void)mbar_wait(s.fin, 0u, p.timeout_ns, nullptr);
            }
        } else if (warp >= 4) {
            tc_softmax<G>(p, sc, s, B, start, end, threadIdx.x - 128, tmem);
        }
    }
    if ((p.flags & QDA_FLAG_INJECT_WAIT_TIMEOUT) != 0u && blockIdx.x == 0 && warp == 0) {
        // test hook: a barrier nothing arrives at; the wait must end by itself
        if (!mbar_wait(s.never, 0u, p.timeout_ns, nullptr) && lane == 0) record_error(p.status, QDA_ERR_TIMEOUT);
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
// pieces sit in consecutive CTAs g0..gk of the attention launch, which
// recorded the slot of the first (2*g0 + 1 when the unit starts inside g0's
// range, as g0's last piece; else 2*g0) and gk; the later pieces are in slots
// 2*g.
template <int G>
__global__ void __launch_bounds__(256) prefill_combine_kernel(const Params p, const PrefillScratch sc) {
    constexpr int kHq = G * kNumKvHeads;
    pdl_wait();
    pdl_launch_dependents();
    const int b = blockIdx.x, j = blockIdx.y, lane = threadIdx.x & 31;
    const int r = 8 * (int)blockIdx.z + (int)(threadIdx.x >> 5);
    if (r >= p.new_tokens * G) return;
    if (p.seg[b + 1] == p.seg[b]) return;   // a sequence the attention launch skipped
    const int2 info = sc.unit[b * kNumKvHeads + j];
    const int first = info.x, g0 = info.x >> 1, gk = info.y;
    if (g0 == gk) return;   // held whole by one CTA, which wrote o
    if (g0 < 0 || gk < g0 || gk >= sc.grid) return;   // not recorded (an attention launch that gave up)
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
    cfg.gridDim = dim3((unsigned)p.batch, (unsigned)kNumKvHeads, (unsigned)((p.new_tokens + 7) / 8));
    cfg.blockDim = dim3(256, 1, 1);
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
