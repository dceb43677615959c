// The dense products around the attention step on the 5th-generation tensor
// cores: attn.o_proj (after it) and, first, the two nodes that produce the
// step's input, fused: input_norm
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
// Two launches. The first forms hi, lo and 1/r_b once per row into the
// handle's workspace (the product reads each row many times). The second is
// a dense product on the 5th-generation tensor cores (linear_tc_kernel):
//
//   CTA (n-tile, k-part, batch group) computes a 128 x C tile of the result
//   transposed, D[n][b] = sum_k W[n][k] (hi[b][k] + lo[b][k]), with the 128
//   weight rows as the A operand (M = 128) and C <= 64 batch rows as the B
//   operand (N = C). A producer thread streams 128 x 64 weight boxes and the
//   matching C x 64 boxes of hi and lo into a 4-stage shared ring by tiled
//   copies with the 128-byte swizzle; four threads issue tcgen05.mma, thread
//   t taking every chunk of stage t into its own accumulator in tensor memory
//   (two products per 16-wide K step: hi, then lo), and free the stage with
//   tcgen05.commit; four warps read the accumulators back (tcgen05.ld) and
//   add them in order for the epilogue. (One issuing thread stalls on the
//   products it issues; four keep four chains in flight.)
//
//   The work split fills the SMs at any batch: the batch is cut in groups
//   of at most 64 rows, and the K range in P = 1, 2, 4 or 8 parts, the
//   fewest that keep at least 80% of the SMs busy (at 0.6B: P = 4 for
//   qkv_proj up to 64 rows, giving 128 CTAs; P = 1 at 256 rows). The P parts
//   of a tile form a thread-block cluster. CTA q of the cluster owns rows
//   [q * 128/P, (q+1) * 128/P) of the tile: after the products every CTA
//   sends its partial values of those rows into CTA q's shared memory with
//   asynchronous stores that complete on CTA q's tile barrier, and CTA q,
//   once its barrier has seen all their bytes, adds the P parts in part
//   order, so the result does not depend on timing.
//
// Both launches are programmatic dependents of the launch before them. The
// first waits for its predecessor before it reads x; the product allocates
// tensor memory and issues its first weight copies before it waits for the
// first launch's hi, lo and 1/r.
//
// attn.o_proj (Model Spec, "Compute-graph nodes": linear, K = 2048,
// N = 1024 for 0.6B) is the same product with one term: the attention output
// o [B][Hq][128], read as rows of Hq * 128, is the B operand as it is (bf16
// products are exact in float), no row scale; it is launched as a
// programmatic dependent of the attention, whose o it waits for after its
// first weight copies.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <mutex>

#include "qda_device.cuh"
#include "qda_internal.h"
#include "qda_tc.cuh"
#include "qwen3_decode_attn.h"

namespace qda {
namespace {

constexpr int kPrepThreads = 128;

constexpr int kLinThreads = 256;                      // 8 warps: producer, scales, 4 MMA issuers; warps 0-3 the epilogue
constexpr int kLinIssuers = 4;                        // MMA-issuing threads (lane 0 of warps 4-7), one accumulator each
constexpr int kLinM = 128;                            // weight rows per CTA (the instruction's M)
constexpr int kLinKC = 64;                            // K per stage: one 128-byte swizzle row
constexpr int kLinStages = 4;
// Issuer t consumes every chunk of stage t, in order: a thread waiting on a
// stage's full barrier is then never more than one phase ahead of it (a wait
// on a parity two phases ahead would pass at once).
static_assert(kLinStages == kLinIssuers, "each MMA issuer owns one stage of the ring");
constexpr int kLinMaxCols = 64;                       // batch rows per CTA (the instruction's N)
constexpr int kLinABytes = kLinM * kLinKC * 2;        // 16 KiB of weight per stage
constexpr int kLinBBytes = 2 * kLinMaxCols * kLinKC * 2;   // hi and lo boxes: up to 16 KiB
constexpr int kLinStageBytes = kLinABytes + kLinBBytes;
// After the ring: the output tile [K part][cols][rows of the part] (float)
// that the cluster's CTAs write into the owner of the rows, the row scales,
// then the barriers.
constexpr int kLinSmemTile = kLinStages * kLinStageBytes;
constexpr int kLinTileBytes = kLinMaxCols * kLinM * 4;      // 32 KiB: every part's share of one CTA's rows
constexpr int kLinSmemScale = kLinSmemTile + kLinTileBytes;  // float [kLinMaxCols]
constexpr int kLinSmemBars = kLinSmemScale + kLinMaxCols * 4;   // full[S], empty[S], acc, tile, tmem address, abort
constexpr int kLinSmemUsed = kLinSmemBars + (2 * kLinStages + 2) * 8 + 16;
constexpr int kLinSmemTotal = kLinSmemUsed + 1024;    // slack to align the ring to 1024 bytes
constexpr uint32_t kLinTmemCols = kLinIssuers * kLinMaxCols;   // one accumulator of up to 64 columns per issuer
static_assert(kLinStageBytes % 1024 == 0 && kLinABytes % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
static_assert(kLinSmemTotal <= 227 * 1024, "fits one CTA per SM");

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

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
    return v;
}

// ---------------------------------------------------------------------------
// First launch: per row b, the split of x[b, k] * g[k] and 1 / r_b.

__global__ void __launch_bounds__(kPrepThreads) input_norm_split_kernel(const QkvProjParams p) {
    pdl_launch_dependents();   // the product may start streaming the weight now
    pdl_wait();                // x may come from the launch before this one
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
// The dense product on tcgen05.

// Bounded wait of one thread; on expiry records QDA_ERR_TIMEOUT and sets the
// CTA's abort flag.
__device__ __forceinline__ bool lin_wait(uint64_t* bar, uint32_t parity, const LinearParams& p,
                                         volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    if (mbar_wait(bar, parity, p.timeout_ns, abort_flag)) return true;
    *abort_flag = 1;
    record_error(p.status, QDA_ERR_TIMEOUT);
    return false;
}

// Columns [j0, j0 + 16) of this warp's 32 tensor-memory lanes, summed over the
// first `naccs` accumulators (64 columns apart) in accumulator order; all the
// loads are in flight before the one wait.
__device__ __forceinline__ void load_acc_sum(uint32_t lane_base, int j0, int naccs, uint32_t (&v)[16]) {
    uint32_t w[kLinIssuers][16];
#pragma unroll
    for (int a = 0; a < kLinIssuers; ++a)
        if (a < naccs) tmem_ld16(lane_base + (uint32_t)(kLinMaxCols * a + j0), w[a]);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float sum = __uint_as_float(w[0][i]);
#pragma unroll
        for (int a = 1; a < kLinIssuers; ++a)
            if (a < naccs) sum += __uint_as_float(w[a][i]);
        v[i] = __float_as_uint(sum);
    }
}

__global__ void __launch_bounds__(kLinThreads, 1)
    linear_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_hi,
                     const __grid_constant__ CUtensorMap tm_lo, const LinearParams p) {
    extern __shared__ uint8_t smem_raw[];
    // the ring must start on a 1024-byte boundary (the swizzle atom)
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const uint32_t ring = smem_addr(smem);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kLinSmemBars);
    uint64_t* empty = full + kLinStages;
    uint64_t* acc_bar = empty + kLinStages;
    uint64_t* tile_bar = acc_bar + 1;   // the cluster peers' partial values have landed in the tile
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tile_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    pdl_launch_dependents();   // a launch consuming this result may be scheduled now
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = (int)blockIdx.x * kLinM;
    const int part = (int)blockIdx.y;               // K part = rank in the cluster when k_split > 1
    const int b0 = (int)blockIdx.z * p.cols;
    const int chunks = p.k / kLinKC / p.k_split;    // K stages of this CTA
    const int c0 = part * chunks;
    const uint32_t term_bytes = (uint32_t)p.cols * kLinKC * 2;
    const uint32_t stage_tx = (uint32_t)kLinABytes + (p.two_terms ? 2u : 1u) * term_bytes;
    const int rows = kLinM / p.k_split;   // the rows of the tile this CTA owns

    float* scale_s = reinterpret_cast<float*>(smem + kLinSmemScale);
    const int pre = min(kLinStages, chunks);
    if (threadIdx.x == 0) {
        // the barriers, then at once the weight boxes of the first round (they
        // need nothing from the previous launch), while warp 1 allocates the
        // accumulator
        for (int s = 0; s < kLinStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_bar, kLinIssuers);
        mbar_init(tile_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        // the bytes the other K parts will store into this CTA's tile
        if (p.k_split > 1) mbar_arrive_expect_tx(tile_bar, (uint32_t)((p.k_split - 1) * p.cols * rows * 4));
        tma_prefetch_desc(&tm_w);
        for (int c = 0; c < pre; ++c) {
            mbar_arrive_expect_tx(&full[c], stage_tx);
            tma_load_2d(ring + c * kLinStageBytes, &tm_w, (c0 + c) * kLinKC, n0, &full[c]);
        }
    }
    if (warp == 1) tmem_alloc(tmem_slot, kLinTmemCols);
    // the peers may store into this CTA's tile once their wait on this arrival ends
    if (p.k_split > 1) cluster_arrive_relaxed();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

    if (warp == 0 && lane == 0) {
        // Producer: the activation boxes wait for the previous launch.
        tma_prefetch_desc(&tm_hi);
        if (p.two_terms) tma_prefetch_desc(&tm_lo);
        if (p.wait_acts) {
            pdl_wait();
            asm volatile("fence.proxy.async.global;" ::: "memory");   // the copies read what it wrote
        }
        auto acts = [&](int c, int s) {
            const uint32_t b = ring + s * kLinStageBytes + kLinABytes;
            tma_load_2d(b, &tm_hi, (c0 + c) * kLinKC, b0, &full[s]);
            if (p.two_terms) tma_load_2d(b + term_bytes, &tm_lo, (c0 + c) * kLinKC, b0, &full[s]);
        };
        for (int c = 0; c < pre; ++c) acts(c, c);
        int issued = pre;
        for (int c = pre; c < chunks; ++c) {
            const int s = c % kLinStages;
            if (!lin_wait(&empty[s], (uint32_t)((c / kLinStages - 1) & 1), p, abort_flag)) break;
            mbar_arrive_expect_tx(&full[s], stage_tx);
            tma_load_2d(ring + s * kLinStageBytes, &tm_w, (c0 + c) * kLinKC, n0, &full[s]);
            acts(c, s);
            issued = c + 1;
        }
        if (*abort_flag != 0) {
            // copies still landing in this CTA's shared memory: wait (bounded) for the last round
            for (int c = max(0, issued - kLinStages); c < issued; ++c)
                (void)mbar_wait(&full[c % kLinStages], (uint32_t)((c / kLinStages) & 1), p.timeout_ns, nullptr);
        }
    } else if (warp >= 4 && lane == 0) {
        // MMA issuer t (of 4) takes chunks t, t + 4, ... (all in stage t) into
        // its own accumulator (columns 64t..): two products per 16-wide K step
        // (hi, then lo). An issuing thread stalls on the products it issues
        // (about 0.45 us per 64-wide chunk at the small N here, measured), so
        // four of them keep four chains in flight.
        const int t = warp - 4;
        const uint32_t idesc = umma_idesc_bf16_m128(p.cols);
        const uint32_t acc = tmem + (uint32_t)(kLinMaxCols * t);
        for (int c = t; c < chunks; c += kLinIssuers) {
            const int s = c % kLinStages;
            if (!lin_wait(&full[s], (uint32_t)((c / kLinStages) & 1), p, abort_flag)) break;
            tc_fence_after();
            const uint32_t a = ring + s * kLinStageBytes;
            const uint32_t b = a + kLinABytes;
#pragma unroll
            for (int kk = 0; kk < kLinKC / 16; ++kk) {
                const uint64_t da = umma_desc_sw128(a + 32 * kk);
                umma_bf16(acc, da, umma_desc_sw128(b + 32 * kk), idesc, (c != t || kk != 0) ? 1u : 0u);
                if (p.two_terms) umma_bf16(acc, da, umma_desc_sw128(b + term_bytes + 32 * kk), idesc, 1u);
            }
            umma_commit(&empty[s]);   // the stage is free once these products have read it
        }
        umma_commit(acc_bar);         // every product issued above has completed
    } else if (warp == 1) {
        // the row scales of this CTA's batch rows (from the previous launch)
        if (p.wait_acts) pdl_wait();
        for (int j = lane; j < p.cols; j += 32) {
            const int b = b0 + j;
            scale_s[j] = (p.row_scale != nullptr && b < p.batch) ? __ldg(p.row_scale + b) : 1.f;
        }
    }
    __syncwarp();

    // Epilogue: warp w < 4 holds tensor-memory lanes 32w..32w+31 = weight rows
    // n0 + 32w + lane, and adds the issuers' accumulators in issuer order.
    // Each CTA owns rows [part*R, part*R + R) of the tile,
    // R = 128 / k_split, laid out [part][cols][R]; every CTA of the cluster
    // stores its partial values of those rows into the owner's tile with
    // asynchronous stores that complete their bytes on the owner's tile
    // barrier (a CTA that gave up stores zeros, so that no owner waits in
    // vain). Each owner waits on its own barrier only, then adds the parts in
    // part order, scales, rounds and stores 8 rows (16 bytes) at a time.
    // (warp-uniform: tcgen05.ld is a whole-warp instruction)
    const bool ok = __all_sync(kFull, lin_wait(acc_bar, 0u, p, abort_flag) && *abort_flag == 0);
    tc_fence_after();
    const int naccs = min(kLinIssuers, chunks);   // accumulators that received products
    if (p.k_split == 1) {
        // No K parts: each thread scales and stores its weight row's outputs from
        // registers (a warp's 32 lanes write 32 consecutive outputs per batch row).
        __syncthreads();   // the row scales
        if (warp < 4 && ok) {
            const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
            const int n = n0 + 32 * warp + lane;
            for (int j0 = 0; j0 < p.cols; j0 += 16) {
                uint32_t v[16];
                load_acc_sum(lane_base, j0, naccs, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int b = b0 + j0 + i;
                    if (b < p.batch)
                        p.y[(size_t)b * p.n_out + n] =
                            __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[i]) * scale_s[j0 + i]));
                }
            }
        }
    } else {   // K parts
        cluster_wait();   // every peer's tile barrier is initialised (warps converged here)
        if (warp < 4) {
            const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
            const int r = 32 * warp + lane;
            const int owner = r / rows, rr = r % rows;
            float* tile = reinterpret_cast<float*>(smem + kLinSmemTile);
            const uint32_t elem = smem_addr(tile + (size_t)part * p.cols * rows + rr);
            const bool local = owner == part;
            const uint32_t dst = local ? elem : cluster_map(elem, (uint32_t)owner);
            const uint32_t dst_bar = local ? 0u : cluster_map(smem_addr(tile_bar), (uint32_t)owner);
            for (int j0 = 0; j0 < p.cols; j0 += 16) {
                uint32_t v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = 0u;
                if (ok) load_acc_sum(lane_base, j0, naccs, v);
                if (local) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) tile[((size_t)part * p.cols + j0 + i) * rows + rr] = __uint_as_float(v[i]);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        st_async_f32(dst + (uint32_t)((j0 + i) * rows * 4), __uint_as_float(v[i]), dst_bar);
                }
            }
        }
        __syncthreads();   // this CTA's own part is in the tile
        {
            // the other parts: a bounded wait that does not give up on this CTA's
            // abort flag, since their stores land here whatever this CTA did
            if (threadIdx.x == 0 && !mbar_wait(tile_bar, 0u, p.timeout_ns, nullptr)) {
                *abort_flag = 1;
                record_error(p.status, QDA_ERR_TIMEOUT);
            }
            __syncthreads();
        }
        {
            const float* tile = reinterpret_cast<const float*>(smem + kLinSmemTile);
            const int oct = rows / 8;
            for (int e = threadIdx.x; e < oct * p.cols; e += kLinThreads) {
                const int j = e / oct, rr = 8 * (e % oct);
                const int b = b0 + j;
                float acc[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) acc[k] = 0.f;
                for (int q = 0; q < p.k_split; ++q) {
                    const float4* src = reinterpret_cast<const float4*>(tile + ((size_t)q * p.cols + j) * rows + rr);
                    const float4 x0 = src[0], x1 = src[1];
                    acc[0] += x0.x; acc[1] += x0.y; acc[2] += x0.z; acc[3] += x0.w;
                    acc[4] += x1.x; acc[5] += x1.y; acc[6] += x1.z; acc[7] += x1.w;
                }
                if (b < p.batch && *abort_flag == 0) {
                    const float sc = scale_s[j];
                    uint4 w;
                    w.x = pack_bf2(acc[0] * sc, acc[1] * sc);
                    w.y = pack_bf2(acc[2] * sc, acc[3] * sc);
                    w.z = pack_bf2(acc[4] * sc, acc[5] * sc);
                    w.w = pack_bf2(acc[6] * sc, acc[7] * sc);
                    *reinterpret_cast<uint4*>(p.y + (size_t)b * p.n_out + n0 + part * rows + rr) = w;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kLinTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launches.

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// A row-major bf16 matrix [rows][cols] (cols contiguous, row pitch cols * 2
// bytes) read in boxes of 64 x box_rows with the 128-byte swizzle; rows past
// the end read as zeros.
bool encode_rows(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
    const PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kLinKC, (cuuint32_t)box_rows};
    const cuuint32_t elem[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, elem,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

void linear_split(int batch, int n_out, int k, int sms, int& cols, int& k_split, int& groups) {
    cols = batch <= kLinMaxCols ? (batch + 15) / 16 * 16 : kLinMaxCols;
    groups = (batch + cols - 1) / cols;
    // K parts (a cluster of at most 8): the fewest that give about one CTA
    // per SM (at least 80% of the SMs busy), so that no CTA waits for a
    // second wave and no more partial tiles are added up than needed
    const int tiles = n_out / kLinM * groups;
    k_split = 1;
    while (k_split < 8 && tiles * k_split * 5 < sms * 4 && (k / kLinKC) % (2 * k_split) == 0) k_split *= 2;
}

cudaError_t launch_linear(const LinearOperands& ops, const LinearParams& p0, cudaStream_t stream) {
    LinearParams p = p0;
    int device = 0, sms = 0, groups = 1;
    if (cudaGetDevice(&device) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || sms < 1)
        return cudaErrorInvalidDevice;
    linear_split(p.batch, p.n_out, p.k, sms, p.cols, p.k_split, groups);
    if (p.k % (kLinKC * p.k_split) != 0 || p.n_out % kLinM != 0) return cudaErrorInvalidValue;
    CUtensorMap tw, th, tl;
    if (!encode_rows(&tw, ops.w, p.n_out, p.k, kLinM) || !encode_rows(&th, ops.act_hi, p.batch, p.k, p.cols) ||
        !encode_rows(&tl, ops.act_lo != nullptr ? ops.act_lo : ops.act_hi, p.batch, p.k, p.cols))
        return cudaErrorInvalidValue;
    p.two_terms = ops.act_lo != nullptr ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.n_out / kLinM), (unsigned)p.k_split, (unsigned)groups);
    cfg.blockDim = dim3(kLinThreads, 1, 1);
    cfg.dynamicSmemBytes = kLinSmemTotal;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (p.k_split > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;   // the K parts of a tile
        attr[n].val.clusterDim.x = 1;
        attr[n].val.clusterDim.y = (unsigned)p.k_split;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, linear_tc_kernel, tw, th, tl, p);
}

cudaError_t prepare_qkv_proj() {
    if (encode_fn() == nullptr) return cudaErrorNotSupported;
    return cudaFuncSetAttribute(linear_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kLinSmemTotal);
}

cudaError_t launch_o_proj(const OProjParams& p, cudaStream_t stream) {
    LinearOperands ops{p.w, p.x, nullptr};
    LinearParams lp{};
    lp.y = p.y;
    lp.row_scale = nullptr;
    lp.batch = p.batch;
    lp.k = p.in_features;
    lp.n_out = p.hidden;
    lp.wait_acts = 1;
    lp.status = p.status;
    lp.timeout_ns = p.timeout_ns;
    return launch_linear(ops, lp, stream);
}

cudaError_t launch_qkv_proj(const QkvProjParams& p, cudaStream_t stream) {
    // a programmatic dependent of the launch before it: its launch overlaps that one's end
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.batch, 1, 1);
    cfg.blockDim = dim3(kPrepThreads, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, input_norm_split_kernel, p);
    if (e != cudaSuccess) return e;
    LinearOperands ops{p.w, p.xg_hi, p.xg_lo};
    LinearParams lp{};
    lp.y = p.y;
    lp.row_scale = p.inv_r;
    lp.batch = p.batch;
    lp.k = p.hidden;
    lp.n_out = p.qkv_width;
    lp.wait_acts = 1;
    lp.status = p.status;
    lp.timeout_ns = p.timeout_ns;
    return launch_linear(ops, lp, stream);
}

}  // namespace qda
