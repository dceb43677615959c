// The two nodes that produce the attention step's input, fused: input_norm
// (RMSNorm over the hidden size H with a gain per feature) and attn.qkv_proj
// (a linear map with no bias), Qwen3-0.6B Model Spec, "Compute-graph nodes":
//   qkv[b, n] = sum_k ( x[b, k] / r_b * g[k] ) * W[n, k],
//   r_b = sqrt(sum_k x[b, k]^2 / H + eps),  K = H = 1024, N = 4096 for 0.6B.
//
// Numbers. Nothing is rounded before the bf16 qkv row. Since x and g are bf16,
// their product has at most 16 significant bits and splits exactly into two
// bf16 values, x*g = hi + lo; the tensor cores then form hi*W and lo*W exactly
// and sum them in float. The factor 1/r_b (from float sums of the exact
// squares x^2, finished in double) is applied to the float sums before the one
// rounding to bf16. So qkv equals the correctly rounded value except where the
// float sums land within ~2^-19 of a rounding midpoint.
//
// Work split. CTA (nb, mb) owns output columns [32 nb, 32 nb + 32) for the
// batch rows [MT mb, MT mb + MT) and the whole K. A producer warp streams K in
// chunks of 256 through a 4-stage ring: each chunk brings the 32 weight rows'
// 512-byte slices and the MT rows' slices of x, one bulk copy per row, into
// rows 528 bytes apart (so that the 8 rows an ldmatrix phase reads fall in 8
// different bank groups). Four consumer warps split each chunk's 16 k-steps
// between them (k-step s goes to warp s % 4); warp w accumulates every row
// and column of the tile over its k-steps with mma.sync m16n8k16 (bf16 in,
// float accumulate), and the four partial tiles and squared sums are added
// through shared memory at the end. For B <= 64 the grid is N / 32 = 128 CTAs
// whose 4 stages together hold the whole weight in flight.
#include <cuda_bf16.h>
#include <cstdint>

#include "qda_device.cuh"
#include "qda_internal.h"
#include "qwen3_decode_attn.h"

namespace qda {
namespace {

constexpr int kNT = 32;                        // output columns per CTA
constexpr int kKC = 256;                       // K per chunk
constexpr int kStagesP = 4;
constexpr int kPitch = kKC * 2 + 16;           // 528-byte staged row pitch
constexpr int kConsumers = 4;
constexpr int kThreadsP = (kConsumers + 1) * 32;

template <int MT>
struct PLayout {
    static constexpr int kRowsPerStage = kNT + MT;                 // weight rows, then x rows
    static constexpr int kStageBytes = kRowsPerStage * kPitch;
    static constexpr int kSmemGain = kStagesP * kStageBytes;       // bf16 [kMaxHidden]
    static constexpr int kSmemBars = kSmemGain + kMaxHidden * 2;   // full[4], empty[4], gain
    static constexpr int kSmemFlags = kSmemBars + (2 * kStagesP + 1) * 8;
    static constexpr int kSmemTotal = kSmemFlags + 16;
    // the end-of-loop reduction reuses the ring: 4 partial tiles and row sums
    static constexpr int kRedBytes = kConsumers * MT * kNT * 4 + kConsumers * MT * 4 + MT * 4;
    static_assert(kRedBytes <= kStagesP * kStageBytes, "reduction fits in the ring");
    static_assert(kStageBytes % 16 == 0 && kSmemBars % 8 == 0, "alignment");
    static_assert(kSmemTotal <= 227 * 1024, "fits one CTA per SM");
};

struct PShared {
    uint8_t* stages;
    const uint16_t* gain;
    uint64_t* full_bar;
    uint64_t* empty_bar;
    uint64_t* gain_bar;
    volatile int* abort_flag;
};

// Producer warp: the gain once, then K / 256 chunks of the tile's weight and x rows.
template <int MT>
__device__ __forceinline__ void proj_producer(const QkvProjParams& p, const PShared& s, int n0, int m0, int rows,
                                              int lane) {
    using Lay = PLayout<MT>;
    const int chunks = p.hidden / kKC;
    if (lane == 0) {
        mbar_arrive_expect_tx(s.gain_bar, (uint32_t)p.hidden * 2u);
        bulk_g2s(const_cast<uint16_t*>(s.gain), p.norm_w, (uint32_t)p.hidden * 2u, s.gain_bar);
    }
    uint32_t armed = 0, armed_parity = 0;
    bool aborted = false;
    for (int c = 0; c < chunks; ++c) {
        const int slot = c % kStagesP;
        const uint32_t phase = (uint32_t)(c / kStagesP) & 1u;
        int ok = 1;
        if (lane == 0) {
            ok = mbar_try_wait(&s.empty_bar[slot], phase ^ 1u) ||
                 mbar_wait(&s.empty_bar[slot], phase ^ 1u, p.timeout_ns, s.abort_flag);
            if (ok) {
                mbar_arrive_expect_tx(&s.full_bar[slot], (uint32_t)(kNT + rows) * (kKC * 2));
                armed |= 1u << slot;
                armed_parity = (armed_parity & ~(1u << slot)) | (phase << slot);
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
        uint8_t* stage = s.stages + slot * Lay::kStageBytes;
        const size_t koff = (size_t)c * kKC;
        // lane l: weight row n0 + l, and x rows l and l + 32 of the tile
        bulk_g2s(stage + lane * kPitch, p.w + (size_t)(n0 + lane) * p.hidden + koff, kKC * 2, &s.full_bar[slot]);
#pragma unroll
        for (int r = lane; r < MT; r += 32)
            if (r < rows)
                bulk_g2s(stage + (kNT + r) * kPitch, p.x + (size_t)(m0 + r) * p.hidden + koff, kKC * 2,
                         &s.full_bar[slot]);
    }
    if (lane == 0 && (aborted || *s.abort_flag != 0)) {
        for (int k = 0; k < kStagesP; ++k)
            if (armed & (1u << k)) (void)mbar_wait(&s.full_bar[k], (armed_parity >> k) & 1u, p.timeout_ns, nullptr);
        (void)mbar_wait(s.gain_bar, 0u, p.timeout_ns, nullptr);
    }
}

// Split the exact product a*b of two bf16 values (at most 16 significant bits)
// into hi + lo, both bf16, with nothing lost.
__device__ __forceinline__ void split_product(float a, float b, uint16_t& hi, uint16_t& lo) {
    const float prod = a * b;   // exact in float: 8-bit by 8-bit significands
    const __nv_bfloat16 h = __float2bfloat16_rn(prod);
    hi = __bfloat16_as_ushort(h);
    lo = __bfloat16_as_ushort(__float2bfloat16_rn(prod - __bfloat162float(h)));   // exact remainder
}

__device__ __forceinline__ bool proj_wait(const QkvProjParams& p, const PShared& s, uint64_t* bar, uint32_t phase,
                                          int lane) {
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

template <int MT>
__global__ void __launch_bounds__(kThreadsP, 1) qkv_proj_kernel(const QkvProjParams p) {
    using Lay = PLayout<MT>;
    constexpr int kMTiles = MT / 16;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    PShared s;
    s.stages = smem;
    s.gain = reinterpret_cast<const uint16_t*>(smem + Lay::kSmemGain);
    s.full_bar = reinterpret_cast<uint64_t*>(smem + Lay::kSmemBars);
    s.empty_bar = s.full_bar + kStagesP;
    s.gain_bar = s.empty_bar + kStagesP;
    s.abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kSmemFlags);

    const int n0 = (int)blockIdx.x * kNT;
    const int m0 = (int)blockIdx.y * MT;
    const int rows = min(MT, p.batch - m0);
    if (threadIdx.x == 0) {
        for (int k = 0; k < kStagesP; ++k) {
            mbar_init(&s.full_bar[k], 1);
            mbar_init(&s.empty_bar[k], kConsumers);
        }
        mbar_init(s.gain_bar, 1);
        *s.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (warp == kConsumers) {
        proj_producer<MT>(p, s, n0, m0, rows, lane);
        return;
    }

    // Consumer warp `warp`: k-steps warp, warp + 4, ... of every chunk.
    const int g = lane >> 2, t = lane & 3;
    float acc[kMTiles][4][4];
    float ss[kMTiles][2];   // this lane's squares of rows g and g + 8 of each m-tile
#pragma unroll
    for (int i = 0; i < kMTiles; ++i) {
        ss[i][0] = ss[i][1] = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
    }
    bool ok = proj_wait(p, s, s.gain_bar, 0u, lane);
    const uint32_t* gain_w = reinterpret_cast<const uint32_t*>(s.gain);
    const int chunks = p.hidden / kKC;
    for (int c = 0; c < chunks && ok; ++c) {
        const int slot = c % kStagesP;
        if (!proj_wait(p, s, &s.full_bar[slot], (uint32_t)(c / kStagesP) & 1u, lane)) {
            ok = false;
            break;
        }
        const uint8_t* stage = s.stages + slot * Lay::kStageBytes;
        // ldmatrix row addresses: weight rows as the column-major B operand,
        // x rows as the row-major A operand
        const uint32_t wbase = smem_addr(stage) + ((lane & 7) + ((lane >> 4) << 3)) * kPitch + ((lane >> 3) & 1) * 16;
        const uint32_t xbase =
            smem_addr(stage) + (kNT + (lane & 7) + ((lane >> 3) & 1) * 8) * kPitch + ((lane >> 4) & 1) * 16;
#pragma unroll
        for (int q = 0; q < kKC / 16 / kConsumers; ++q) {
            const int k0 = (q * kConsumers + warp) * 16;   // within the chunk
            uint32_t b[4][2];
            ldsm_x4(wbase + k0 * 2, b[0][0], b[0][1], b[1][0], b[1][1]);
            ldsm_x4(wbase + 16 * kPitch + k0 * 2, b[2][0], b[2][1], b[3][0], b[3][1]);
            // gains of this lane's k columns: 2t, 2t+1 and 2t+8, 2t+9
            const int kg = c * kKC + k0;
            const uint32_t g01 = gain_w[(kg >> 1) + t], g89 = gain_w[(kg >> 1) + 4 + t];
#pragma unroll
            for (int i = 0; i < kMTiles; ++i) {
                uint32_t a[4];
                ldsm_x4(xbase + i * 16 * kPitch + k0 * 2, a[0], a[1], a[2], a[3]);
                uint32_t ahi[4], alo[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const uint32_t gw = (r & 2) ? g89 : g01;
                    const float x0 = bf_lo(a[r]), x1 = bf_hi(a[r]);
                    ss[i][r & 1] = fmaf(x0, x0, fmaf(x1, x1, ss[i][r & 1]));
                    uint16_t h0, l0, h1, l1;
                    split_product(x0, bf_lo(gw), h0, l0);
                    split_product(x1, bf_hi(gw), h1, l1);
                    ahi[r] = (uint32_t)h1 << 16 | h0;
                    alo[r] = (uint32_t)l1 << 16 | l0;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    mma_bf16_16816(acc[i][j], ahi, b[j][0], b[j][1]);
                    mma_bf16_16816(acc[i][j], alo, b[j][0], b[j][1]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.empty_bar[slot]);
    }

    // All four consumer warps meet here whatever happened (no early return),
    // so the named barrier always completes.
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
    if (*s.abort_flag != 0) return;
    // Partial tiles and squared sums to shared memory (the ring is drained).
    float* red = reinterpret_cast<float*>(s.stages);                    // [4][MT][32]
    float* red_ss = red + kConsumers * MT * kNT;                        // [4][MT]
    float* inv_r = red_ss + kConsumers * MT;                            // [MT]
#pragma unroll
    for (int i = 0; i < kMTiles; ++i) {
        float s0 = ss[i][0], s1 = ss[i][1];
        s0 += __shfl_xor_sync(kFull, s0, 1);
        s0 += __shfl_xor_sync(kFull, s0, 2);
        s1 += __shfl_xor_sync(kFull, s1, 1);
        s1 += __shfl_xor_sync(kFull, s1, 2);
        if (t == 0) {
            red_ss[warp * MT + 16 * i + g] = s0;
            red_ss[warp * MT + 16 * i + g + 8] = s1;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float* r0 = red + ((size_t)warp * MT + 16 * i + g) * kNT + 8 * j + 2 * t;
            float* r1 = r0 + 8 * kNT;
            *reinterpret_cast<float2*>(r0) = make_float2(acc[i][j][0], acc[i][j][1]);
            *reinterpret_cast<float2*>(r1) = make_float2(acc[i][j][2], acc[i][j][3]);
        }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
    const int tid = threadIdx.x;
    for (int r = tid; r < MT; r += kConsumers * 32) {
        const double sum = (double)red_ss[r] + (double)red_ss[MT + r] + (double)red_ss[2 * MT + r] +
                           (double)red_ss[3 * MT + r];
        inv_r[r] = (float)(1.0 / sqrt(sum / (double)p.hidden + p.eps));
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
    // two adjacent columns per thread: one 4-byte store each
    for (int e = tid; e < MT * kNT / 2; e += kConsumers * 32) {
        const int r = e / (kNT / 2), col = 2 * (e % (kNT / 2));
        if (r >= rows) continue;
        float v0 = 0.f, v1 = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) {
            const float2 v = *reinterpret_cast<const float2*>(red + ((size_t)w * MT + r) * kNT + col);
            v0 += v.x;
            v1 += v.y;
        }
        const float f = inv_r[r];
        *reinterpret_cast<uint32_t*>(p.y + (size_t)(m0 + r) * p.qkv_width + n0 + col) = pack_bf2(v0 * f, v1 * f);
    }
}

template <int MT>
cudaError_t prepare_proj_one() {
    return cudaFuncSetAttribute(qkv_proj_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                PLayout<MT>::kSmemTotal);
}

template <int MT>
cudaError_t launch_proj_one(const QkvProjParams& p, cudaStream_t stream) {
    const dim3 grid((unsigned)(p.qkv_width / kNT), (unsigned)((p.batch + MT - 1) / MT), 1);
    qkv_proj_kernel<MT><<<grid, kThreadsP, PLayout<MT>::kSmemTotal, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t prepare_qkv_proj() {
    cudaError_t e = prepare_proj_one<16>();
    if (e == cudaSuccess) e = prepare_proj_one<32>();
    if (e == cudaSuccess) e = prepare_proj_one<64>();
    return e;
}

cudaError_t launch_qkv_proj(const QkvProjParams& p, cudaStream_t stream) {
    if (p.batch <= 16) return launch_proj_one<16>(p, stream);
    if (p.batch <= 32) return launch_proj_one<32>(p, stream);
    return launch_proj_one<64>(p, stream);
}

}  // namespace qda
