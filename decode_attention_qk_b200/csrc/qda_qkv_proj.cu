// The two nodes that produce the attention step's input, fused: input_norm
// (RMSNorm over the hidden size H with a gain per feature) and attn.qkv_proj
// (a linear map with no bias), Qwen3-0.6B Model Spec, "Compute-graph nodes":
//   qkv[b, n] = sum_k ( x[b, k] / r_b * g[k] ) * W[n, k],
//   r_b = sqrt(sum_k x[b, k]^2 / H + eps),  K = H = 1024, N = 4096 for 0.6B.
//
// Numbers. Nothing is rounded before the bf16 qkv row. Since x and g are bf16,
// their product has at most 16 significant bits and splits exactly into two
// bf16 values, x*g = hi + lo; the tensor cores form hi*W and lo*W exactly and
// sum them in float. 1/r_b (from float sums of the exact squares x^2, finished
// in double) scales the float sums just before the one rounding to bf16.
//
// Work split. The product is cut along N into 128-column tiles and along K
// into 4 quarters: CTA (n-tile, quarter, row block) reads the 128 weight rows'
// quarter (64 KiB at H = 1024) and its rows' quarter of the split, and writes
// a float partial tile into its own shared memory. The four quarters of a tile
// form a thread-block cluster: after a cluster barrier, quarter q adds the
// four partials of columns [32q, 32q + 32) in quarter order, reading its peers'
// shared memory directly (so the result does not depend on timing and no
// partial goes through L2), scales by 1/r_b and writes bf16 qkv. With 4 warps
// of 32 columns each, a CTA needs no reduction of its own.
//
// Operands reach shared memory by 16-byte asynchronous copies (cp.async)
// through a 3-stage ring of 128-wide K chunks (64-wide for the 64-row blocks
// of large batches, so that two CTAs share an SM), in rows 16 bytes longer
// than the chunk so that the 8 rows an ldmatrix phase reads fall in 8
// different bank groups. (One
// bulk copy per short row slice was tried first: at about one copy every
// 45 ns per SM the copy count, not the bytes, set the time.)
//
// The split of x*g. For up to 32 rows each CTA forms it for its own quarter of
// K from raw x staged next to the weight (4x less repeated work than forming
// it for all of K, and no second launch). For more rows a first launch forms
// it once per row (with 1/r_b) into workspace and the product launch starts
// with programmatic dependent launch: it issues the weight copies of its first
// stages before it waits for the first launch.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "qda_device.cuh"
#include "qda_internal.h"
#include "qwen3_decode_attn.h"

namespace qda {
namespace {

constexpr int kNT = kProjNTile;                // output columns per CTA
constexpr int kKS = kProjKSplits;              // K quarters
constexpr int kStages = 3;
constexpr int kWarps = 4;
constexpr int kThreadsP = kWarps * 32;
constexpr int kPrepThreads = 128;

// kConvert: the CTA forms the split itself from raw x (up to 32 rows); else it
// copies the split formed by the first launch.
//
// Operand tiles are stored K-major in the tensor cores' canonical layout
// without swizzle: core matrices of 8 rows x 16 bytes (8 bf16 along K), rows
// 16 bytes apart; the core matrices of a row group follow one another along K
// (128 bytes apart) and row groups follow at kKC * 16 bytes. That order is
// simply 16-byte piece i = (row group, piece along K, row within the group),
// so copy i lands at byte 16 i.
template <int MT, bool kConvert>
struct PLayout {
    // K per chunk: 128, or 64 for the 64-row blocks of large batches, whose
    // CTAs then fit two to an SM
    static constexpr int kKC = kConvert ? 128 : 64;
    static constexpr int kPieces = kKC / 8;                          // 16-byte pieces per row slice
    static constexpr uint32_t kLBO = 128;                            // next core matrix along K
    static constexpr uint32_t kSBO = kKC * 16;                       // next group of 8 rows
    static constexpr int kCtasPerSm = kConvert ? 1 : 2;
    static constexpr int kWBytes = kNT * kKC * 2;                    // the weight tile
    static constexpr int kABytes = MT * kKC * 2;                     // one tile of MT rows
    static constexpr int kStageBytes = kWBytes + (kConvert ? 1 : 2) * kABytes;   // + raw x, or hi and lo
    static constexpr int kSmemHiLo = kStages * kStageBytes;          // convert: 2 buffers of (hi, lo)
    static constexpr int kSmemGain = kSmemHiLo + (kConvert ? 4 * kABytes : 0);   // bf16 [hidden / 4]
    static constexpr int kSmemSq = kSmemGain + (kConvert ? kMaxHidden / kKS * 2 : 0);   // float [MT][kPieces]
    static constexpr int kSmemInvR = kSmemSq + (kConvert ? MT * kPieces * 4 : 0);      // float [MT]
    static constexpr int kSmemBars = kSmemInvR + MT * 4;                               // uint64 [kStages]
    static constexpr int kSmemTmem = kSmemBars + kStages * 8;                          // TMEM address
    static constexpr int kSmemTotal = kSmemTmem + 16;
    // the accumulator: 128 TMEM lanes (output columns) x MT columns (rows)
    static constexpr uint32_t kTmemCols = MT < 32 ? 32 : MT;
    // after the K loop the ring holds this quarter's partial tile and sums of x^2
    static_assert((MT * kNT + MT) * 4 <= kStages * kStageBytes, "partial tile fits in the ring");
    static_assert(kCtasPerSm * (kSmemTotal + 1024) <= 228 * 1024, "CTAs per SM fit in shared memory");
    static_assert(kStageBytes % 1024 == 0 && kSmemBars % 8 == 0, "alignment");
    static_assert(MT % 16 == 0 && MT >= 16 && MT <= 256, "N of one tensor-core instruction");
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ---------------------------------------------------------------------------
// The 5th-generation tensor cores (tcgen05): descriptors and instructions.

// Shared-memory matrix descriptor of a K-major operand in the canonical layout
// without swizzle: start address >> 4 in bits [0,14), leading byte offset
// (between the two core matrices of a 16-element K step) >> 4 in [16,30),
// stride byte offset (between groups of 8 rows) >> 4 in [32,46), descriptor
// version 1 in [46,48), base offset 0, layout 0 (no swizzle) in [61,64).
__host__ __device__ constexpr uint64_t umma_smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// Instruction descriptor of kind::f16: f32 accumulator (bits [4,6) = 1), bf16
// A and B (bits [7,10) = 1, [10,13) = 1), both K-major (bits 15, 16 = 0),
// N >> 3 in [17,23), M >> 4 in [24,29); M = 128.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_m128(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
static_assert(umma_idesc_bf16_m128(64) == 0x08100490u, "instruction descriptor bits");
static_assert(umma_smem_desc(0x400u, 128u, 1024u) == ((0x40ull) | (8ull << 16) | (64ull << 32) | (1ull << 46)),
              "matrix descriptor bits");

// D[tmem] (+)= A * B^T for one K step of 16, issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}
// The mbarrier gets one arrival once every tensor-core instruction this thread
// issued before has completed (and read its shared-memory operands).
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Warp-wide: allocate `cols` TMEM columns (a power of two >= 32), address to *dst.
__device__ __forceinline__ void tmem_alloc(void* dst, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)), "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
// Warp-wide: 16 consecutive columns of this warp's 32 TMEM lanes, one lane per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, "
        "[%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
    return v;
}

// The exact split of the products x*g of one 16-byte piece (8 values): hi, lo
// words, and the squares of x added to ss.
__device__ __forceinline__ void split_piece(const uint4& xv, const uint32_t* gw, uint4& hv, uint4& lv, float& ss) {
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float x0 = bf_lo(xw[e]), x1 = bf_hi(xw[e]);
        ss = fmaf(x0, x0, fmaf(x1, x1, ss));     // squares of bf16 values: exact in float
        uint16_t h0, l0, h1, l1;
        split_bf16(x0 * bf_lo(gw[e]), h0, l0);   // the product has <= 16 significant bits: exact
        split_bf16(x1 * bf_hi(gw[e]), h1, l1);
        hw[e] = (uint32_t)h1 << 16 | h0;
        lw[e] = (uint32_t)l1 << 16 | l0;
    }
    hv = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    lv = make_uint4(lw[0], lw[1], lw[2], lw[3]);
}

// ---------------------------------------------------------------------------
// First launch (more than 32 rows): per row b, the split of x[b, k] * g[k] and 1 / r_b.

__global__ void __launch_bounds__(kPrepThreads) input_norm_split_kernel(const QkvProjParams p) {
    pdl_launch_dependents();   // the product may start streaming the weight now
    const int b = blockIdx.x;
    const uint4* xr = reinterpret_cast<const uint4*>(p.x + (size_t)b * p.hidden);
    const uint4* gr = reinterpret_cast<const uint4*>(p.norm_w);
    uint4* hr = reinterpret_cast<uint4*>(p.xg_hi + (size_t)b * p.hidden);
    uint4* lr = reinterpret_cast<uint4*>(p.xg_lo + (size_t)b * p.hidden);
    float ss = 0.f;
    for (int v = threadIdx.x; v < p.hidden / 8; v += kPrepThreads) {
        const uint4 gv = __ldg(gr + v);
        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
        uint4 hv, lv;
        split_piece(__ldg(xr + v), gw, hv, lv, ss);
        hr[v] = hv;
        lr[v] = lv;
    }
    __shared__ float part[kPrepThreads / 32];
    ss = warp_sum_f(ss);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
        double sum = 0.0;
        for (int w = 0; w < kPrepThreads / 32; ++w) sum += (double)part[w];
        p.inv_r[b] = (float)(1.0 / sqrt(sum / (double)p.hidden + p.eps));
    }
}

// ---------------------------------------------------------------------------
// The product, split along K.

template <int MT, bool kConvert>
__global__ void __launch_bounds__(kThreadsP, PLayout<MT, kConvert>::kCtasPerSm) qkv_proj_kernel(const QkvProjParams p) {
    using Lay = PLayout<MT, kConvert>;
    constexpr int kKC = Lay::kKC;
    constexpr int kPieces = Lay::kPieces;
    extern __shared__ __align__(1024) uint8_t smem[];
    pdl_launch_dependents();   // an attention launch after this one may start its K/V streaming
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int nt = (int)blockIdx.x, ks = (int)blockIdx.y, mb = (int)blockIdx.z;
    const int n0 = nt * kNT;
    const int m0 = mb * MT;
    const int rows = min(MT, p.batch - m0);
    const int kq = p.hidden / kKS;           // this CTA's K range: [ks*kq, ks*kq + kq)
    const int kbase = ks * kq;
    const int chunks = kq / kKC;
    const uint32_t ring = smem_addr(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kSmemBars);   // [s]: the products of a chunk in stage s

    // piece i of a tile: row ((i / (8 kPieces)) * 8 + i % 8), piece (i / 8) % kPieces along K, at byte 16 i
    auto piece_row = [](int i) { return ((i / (8 * kPieces)) << 3) | (i & 7); };
    auto piece_k = [](int i) { return (i >> 3) % kPieces; };
    auto weight_rows = [&](int c) {   // 128 rows x kKC: needs nothing from a first launch
        const uint32_t stage = ring + (c % kStages) * Lay::kStageBytes;
        for (int i = tid; i < kNT * kPieces; i += kThreadsP)
            cp_async16(stage + i * 16, p.w + (size_t)(n0 + piece_row(i)) * p.hidden + (size_t)(kbase + c * kKC) +
                                           piece_k(i) * 8);
    };
    auto a_rows = [&](int c) {        // raw x rows, or hi and lo rows (rows past the batch are left as they are)
        const uint32_t stage = ring + (c % kStages) * Lay::kStageBytes + Lay::kWBytes;
        for (int i = tid; i < MT * kPieces; i += kThreadsP) {
            const int r = piece_row(i);
            if (r >= rows) continue;
            const size_t src = (size_t)(m0 + r) * p.hidden + (size_t)(kbase + c * kKC) + piece_k(i) * 8;
            if (kConvert) {
                cp_async16(stage + i * 16, p.x + src);
            } else {
                cp_async16(stage + i * 16, p.xg_hi + src);
                cp_async16(stage + Lay::kABytes + i * 16, p.xg_lo + src);
            }
        }
    };

    // the accumulator in tensor memory, and one mbarrier per stage
    if (warp == 0) tmem_alloc(smem + Lay::kSmemTmem, Lay::kTmemCols);
    if (tid == 0) {
        for (int k = 0; k < kStages; ++k) mbar_init(&bars[k], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // Groups, oldest first: {gain quarter and weight of chunks 0..S-2}, {A of
    // chunk 0}, ..., {A of chunk S-2}, then one group per later chunk.
    const int pre = min(kStages - 1, chunks);
    if (kConvert)
        for (int i = tid; i < kq / 8; i += kThreadsP) cp_async16(ring + Lay::kSmemGain + i * 16, p.norm_w + kbase + i * 8);
    for (int c = 0; c < pre; ++c) weight_rows(c);
    cp_async_commit();
    if (!kConvert) pdl_wait();   // hi, lo and 1/r are complete and visible from here on
    for (int c = 0; c < kStages - 1; ++c) {
        if (c < pre) a_rows(c);
        cp_async_commit();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + Lay::kSmemTmem);
    constexpr uint32_t kIdesc = umma_idesc_bf16_m128(MT);

    // kConvert: thread tid splits pieces tid + 128 m of the raw x tile
    constexpr int kConvPerThread = kConvert ? MT * kPieces / kThreadsP : 1;
    float ss[kConvPerThread];
#pragma unroll
    for (int m = 0; m < kConvPerThread; ++m) ss[m] = 0.f;
    bool ok = true;   // every wait so far completed
    for (int c = 0; c < chunks; ++c) {
        cp_async_wait<kStages - 2>();   // this thread's copies of chunk c have landed
        uint32_t b_hi;
        if (kConvert) {
            __syncthreads();            // ... and everyone's raw x
            const uint8_t* raw = smem + (c % kStages) * Lay::kStageBytes + Lay::kWBytes;
            // buffer c % 2: the products of chunk c - 2 that read it are complete
            uint8_t* hilo = smem + Lay::kSmemHiLo + (c & 1) * 2 * Lay::kABytes;
            const uint32_t* gw = reinterpret_cast<const uint32_t*>(smem + Lay::kSmemGain) + (c * kKC) / 2;
#pragma unroll
            for (int m = 0; m < kConvPerThread; ++m) {
                const int i = tid + kThreadsP * m;
                uint4 hv, lv;
                split_piece(*reinterpret_cast<const uint4*>(raw + i * 16), gw + 4 * piece_k(i), hv, lv, ss[m]);
                *reinterpret_cast<uint4*>(hilo + i * 16) = hv;
                *reinterpret_cast<uint4*>(hilo + Lay::kABytes + i * 16) = lv;
            }
            b_hi = smem_addr(hilo);
        } else {
            b_hi = ring + (c % kStages) * Lay::kStageBytes + Lay::kWBytes;
        }
        // the staged and split operands are read by the tensor cores (async proxy)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        if (tid == 0 && ok) {
            tc_fence_after();
            const uint32_t a = ring + (c % kStages) * Lay::kStageBytes;
            const uint32_t b_lo = b_hi + Lay::kABytes;
#pragma unroll
            for (int k = 0; k < kKC / 16; ++k) {   // 16 along K = 2 core matrices = 256 bytes
                const uint64_t da = umma_smem_desc(a + k * 256, Lay::kLBO, Lay::kSBO);
                umma_bf16(tmem, da, umma_smem_desc(b_hi + k * 256, Lay::kLBO, Lay::kSBO), kIdesc, (c | k) != 0);
                umma_bf16(tmem, da, umma_smem_desc(b_lo + k * 256, Lay::kLBO, Lay::kSBO), kIdesc, 1u);
            }
            umma_commit(&bars[c % kStages]);
        }
        // refill the stage of chunk c - 1 once its products are complete
        if (c >= 1 && ok) {
            ok = mbar_wait(&bars[(c - 1) % kStages], (uint32_t)(((c - 1) / kStages) & 1), p.timeout_ns, nullptr);
            if (!ok && tid == 0) record_error(p.status, QDA_ERR_TIMEOUT);
        }
        if (c + kStages - 1 < chunks && ok) {
            weight_rows(c + kStages - 1);
            a_rows(c + kStages - 1);
        }
        cp_async_commit();
    }
    cp_async_wait<0>();
    if (ok) {
        ok = mbar_wait(&bars[(chunks - 1) % kStages], (uint32_t)(((chunks - 1) / kStages) & 1), p.timeout_ns, nullptr);
        if (!ok && tid == 0) record_error(p.status, QDA_ERR_TIMEOUT);
    }
    tc_fence_after();

    // This quarter's partial tile (float) and, when converting, its sums of x^2,
    // in shared memory for the cluster.
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    float* tile = reinterpret_cast<float*>(smem);   // [MT][kNT], the ring is drained
    float* tss = tile + MT * kNT;                   // [MT]
    if (kConvert) {
        float* sq = reinterpret_cast<float*>(smem + Lay::kSmemSq);   // [MT][kPieces]
#pragma unroll
        for (int m = 0; m < kConvPerThread; ++m) {
            const int i = tid + kThreadsP * m;
            sq[piece_row(i) * kPieces + piece_k(i)] = ss[m];
        }
    }
    // warp w holds TMEM lanes 32w..32w+31 = output columns; TMEM column r = row r
#pragma unroll
    for (int r0 = 0; r0 < MT; r0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)r0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) tile[(r0 + j) * kNT + 32 * warp + lane] = __uint_as_float(v[j]);
    }
    tc_fence_before();
    __syncthreads();
    if (kConvert && tid < MT) {
        const float* sq = reinterpret_cast<const float*>(smem + Lay::kSmemSq) + tid * kPieces;
        float v = 0.f;
#pragma unroll
        for (int q = 0; q < kPieces; ++q) v += sq[q];
        tss[tid] = v;
    }
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, Lay::kTmemCols);
    }
    cluster.sync();   // all four quarters' partials are in place
    const int q = (int)cluster.block_rank();   // = ks
    const float* peer[kKS];
    const float* peer_ss[kKS];
#pragma unroll
    for (int r = 0; r < kKS; ++r) {
        peer[r] = cluster.map_shared_rank(tile, r);
        peer_ss[r] = cluster.map_shared_rank(tss, r);
    }
    float* inv_r = reinterpret_cast<float*>(smem + Lay::kSmemInvR);
    for (int r = tid; r < rows; r += kThreadsP) {
        if (kConvert) {
            double sum = 0.0;
#pragma unroll
            for (int k = 0; k < kKS; ++k) sum += (double)peer_ss[k][r];
            inv_r[r] = (float)(1.0 / sqrt(sum / (double)p.hidden + p.eps));
        } else {
            inv_r[r] = __ldg(p.inv_r + m0 + r);
        }
    }
    __syncthreads();
    // columns [32q, 32q + 32) of the tile: 16 column pairs per row
    for (int e = tid; e < rows * 16; e += kThreadsP) {
        const int r = e / 16, col = 32 * q + 2 * (e % 16);
        float2 sum = *reinterpret_cast<const float2*>(peer[0] + r * kNT + col);
#pragma unroll
        for (int k = 1; k < kKS; ++k) {
            const float2 v = *reinterpret_cast<const float2*>(peer[k] + r * kNT + col);
            sum.x += v.x;
            sum.y += v.y;
        }
        const float f = inv_r[r];
        *reinterpret_cast<uint32_t*>(p.y + (size_t)(m0 + r) * p.qkv_width + n0 + col) = pack_bf2(sum.x * f, sum.y * f);
    }
    cluster.sync();   // peers may still be reading this CTA's partial
}

template <int MT, bool kConvert>
cudaError_t prepare_proj_one() {
    return cudaFuncSetAttribute(qkv_proj_kernel<MT, kConvert>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                PLayout<MT, kConvert>::kSmemTotal);
}

template <int MT, bool kConvert>
cudaError_t launch_proj_one(const QkvProjParams& p, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.qkv_width / kNT), (unsigned)kKS, (unsigned)((p.batch + MT - 1) / MT));
    cfg.blockDim = dim3(kThreadsP, 1, 1);
    cfg.dynamicSmemBytes = PLayout<MT, kConvert>::kSmemTotal;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;   // the 4 K quarters of a tile
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = kKS;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = kConvert ? 1 : 2;   // dependent launch only after the split's own launch
    return cudaLaunchKernelEx(&cfg, qkv_proj_kernel<MT, kConvert>, p);
}

}  // namespace

cudaError_t prepare_qkv_proj() {
    cudaError_t e = prepare_proj_one<16, true>();
    if (e == cudaSuccess) e = prepare_proj_one<32, true>();
    if (e == cudaSuccess) e = prepare_proj_one<64, false>();
    return e;
}

cudaError_t launch_qkv_proj(const QkvProjParams& p, cudaStream_t stream) {
    if (p.batch <= 16) return launch_proj_one<16, true>(p, stream);
    if (p.batch <= 32) return launch_proj_one<32, true>(p, stream);
    input_norm_split_kernel<<<p.batch, kPrepThreads, 0, stream>>>(p);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_proj_one<64, false>(p, stream);
}

}  // namespace qda
