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
template <int MT, bool kConvert>
struct PLayout {
    // K per chunk: 128, or 64 for the 64-row blocks of large batches, whose
    // CTAs then fit two to an SM
    static constexpr int kKC = kConvert ? 128 : 64;
    static constexpr int kPitch = kKC * 2 + 16;                      // staged row pitch (bytes)
    static constexpr int kPieces = kKC / 8;                          // 16-byte pieces per row slice
    static constexpr int kCtasPerSm = kConvert ? 1 : 2;
    static constexpr int kARows = kConvert ? MT : 2 * MT;            // raw x, or hi and lo
    static constexpr int kStageBytes = (kNT + kARows) * kPitch;
    static constexpr int kSmemHiLo = kStages * kStageBytes;          // convert: hi, lo of the current chunk
    static constexpr int kSmemGain = kSmemHiLo + (kConvert ? 2 * MT * kPitch : 0);   // bf16 [hidden / 4]
    static constexpr int kSmemInvR = kSmemGain + (kConvert ? kMaxHidden / kKS * 2 : 0);  // float [MT]
    static constexpr int kSmemTotal = kSmemInvR + MT * 4;
    // after the K loop the ring holds this quarter's partial tile and sums of x^2
    static_assert((MT * kNT + MT) * 4 <= kStages * kStageBytes, "partial tile fits in the ring");
    static_assert(kCtasPerSm * (kSmemTotal + 1024) <= 228 * 1024, "CTAs per SM fit in shared memory");
    static_assert(kStageBytes % 16 == 0 && kPitch % 128 == 16, "alignment, conflict-free rows");
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

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
    constexpr int kMTiles = MT / 16;
    constexpr int kKC = Lay::kKC;
    constexpr int kPitch = Lay::kPitch;
    constexpr int kPieces = Lay::kPieces;
    extern __shared__ __align__(128) uint8_t smem[];
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

    auto weight_rows = [&](int c) {   // 128 rows x 128: needs nothing from a first launch
        const uint32_t stage = ring + (c % kStages) * Lay::kStageBytes;
        for (int i = tid; i < kNT * kPieces; i += kThreadsP) {
            const int r = i / kPieces, q = i % kPieces;
            cp_async16(stage + r * kPitch + q * 16,
                       p.w + (size_t)(n0 + r) * p.hidden + (size_t)(kbase + c * kKC) + q * 8);
        }
    };
    auto a_rows = [&](int c) {        // raw x rows, or hi and lo rows
        const uint32_t stage = ring + (c % kStages) * Lay::kStageBytes + kNT * kPitch;
        for (int i = tid; i < rows * kPieces; i += kThreadsP) {
            const int r = i / kPieces, q = i % kPieces;
            const size_t src = (size_t)(m0 + r) * p.hidden + (size_t)(kbase + c * kKC) + q * 8;
            if (kConvert) {
                cp_async16(stage + r * kPitch + q * 16, p.x + src);
            } else {
                cp_async16(stage + r * kPitch + q * 16, p.xg_hi + src);
                cp_async16(stage + (MT + r) * kPitch + q * 16, p.xg_lo + src);
            }
        }
    };
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

    const int g = lane >> 2, t = lane & 3;
    // kConvert: thread tid splits pieces tid + 128 m (row (tid + 128 m) / 16,
    // piece tid % 16); the 16 threads of a half-warp share a row
    constexpr int kConvPerThread = kConvert ? MT * kPieces / kThreadsP : 1;
    float ss[kConvPerThread];
#pragma unroll
    for (int m = 0; m < kConvPerThread; ++m) ss[m] = 0.f;
    float acc[kMTiles][4][4];
#pragma unroll
    for (int i = 0; i < kMTiles; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
    for (int c = 0; c < chunks; ++c) {
        if (c + kStages - 1 < chunks) {
            weight_rows(c + kStages - 1);
            a_rows(c + kStages - 1);
        }
        cp_async_commit();
        cp_async_wait<kStages - 1>();   // this thread's copies of chunk c have landed ...
        __syncthreads();                // ... and everyone's
        const uint32_t stage = ring + (c % kStages) * Lay::kStageBytes;
        uint32_t abase_hi, abase_lo;
        if (kConvert) {
            const uint8_t* raw = smem + (c % kStages) * Lay::kStageBytes + kNT * kPitch;
            const uint32_t* gw = reinterpret_cast<const uint32_t*>(smem + Lay::kSmemGain) + (c * kKC) / 2;
#pragma unroll
            for (int m = 0; m < kConvPerThread; ++m) {
                const int i = tid + kThreadsP * m;
                const int r = i / kPieces, q = i % kPieces;
                uint4 hv, lv;
                split_piece(*reinterpret_cast<const uint4*>(raw + r * kPitch + q * 16), gw + 4 * q, hv, lv, ss[m]);
                *reinterpret_cast<uint4*>(smem + Lay::kSmemHiLo + r * kPitch + q * 16) = hv;
                *reinterpret_cast<uint4*>(smem + Lay::kSmemHiLo + (MT + r) * kPitch + q * 16) = lv;
            }
            __syncthreads();
            abase_hi = ring + Lay::kSmemHiLo;
        } else {
            abase_hi = stage + kNT * kPitch;
        }
        abase_lo = abase_hi + MT * kPitch;
        // ldmatrix row addresses: this warp's 32 weight rows as the column-major
        // B operand, hi and lo rows as the row-major A operand
        const uint32_t wbase =
            stage + (32 * warp + (lane & 7) + ((lane >> 4) << 3)) * kPitch + ((lane >> 3) & 1) * 16;
        const uint32_t aoff = ((lane & 7) + ((lane >> 3) & 1) * 8) * kPitch + ((lane >> 4) & 1) * 16;
#pragma unroll
        for (int kstep = 0; kstep < kKC / 16; ++kstep) {
            const int k0 = kstep * 16;
            uint32_t b[4][2];
            ldsm_x4(wbase + k0 * 2, b[0][0], b[0][1], b[1][0], b[1][1]);
            ldsm_x4(wbase + 16 * kPitch + k0 * 2, b[2][0], b[2][1], b[3][0], b[3][1]);
#pragma unroll
            for (int i = 0; i < kMTiles; ++i) {
                uint32_t ahi[4], alo[4];
                ldsm_x4(abase_hi + aoff + i * 16 * kPitch + k0 * 2, ahi[0], ahi[1], ahi[2], ahi[3]);
                ldsm_x4(abase_lo + aoff + i * 16 * kPitch + k0 * 2, alo[0], alo[1], alo[2], alo[3]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    mma_bf16_16816(acc[i][j], ahi, b[j][0], b[j][1]);
                    mma_bf16_16816(acc[i][j], alo, b[j][0], b[j][1]);
                }
            }
        }
        __syncthreads();                // the stage (and the hi/lo buffer) may be refilled
    }
    cp_async_wait<0>();

    // This quarter's partial tile (float) and, when converting, its sums of x^2,
    // in shared memory for the cluster.
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    float* tile = reinterpret_cast<float*>(smem);   // [MT][kNT], the ring is drained
    float* tss = tile + MT * kNT;                   // [MT]
#pragma unroll
    for (int i = 0; i < kMTiles; ++i) {
        const int r0 = 16 * i + g;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int col = 32 * warp + 8 * j + 2 * t;
            *reinterpret_cast<float2*>(tile + r0 * kNT + col) = make_float2(acc[i][j][0], acc[i][j][1]);
            *reinterpret_cast<float2*>(tile + (r0 + 8) * kNT + col) = make_float2(acc[i][j][2], acc[i][j][3]);
        }
    }
    if (kConvert) {
#pragma unroll
        for (int m = 0; m < kConvPerThread; ++m) {
            float v = ss[m];
            v += __shfl_xor_sync(kFull, v, 1);
            v += __shfl_xor_sync(kFull, v, 2);
            v += __shfl_xor_sync(kFull, v, 4);
            v += __shfl_xor_sync(kFull, v, 8);
            if ((lane & 15) == 0) tss[(tid + kThreadsP * m) / kPieces] = v;
        }
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
