// Device helpers shared by the decode-attention kernels: mbarrier and
// bulk-copy wrappers, bounded waits, bf16 conversions, packed two-float
// arithmetic. Internal to the library.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace qda {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr float kRescaleThreshold = 8.0f;             // log2 units: rescale only when the max grows by > 2^8
constexpr double kQScale = 1.4426950408889634 * 0.088388347648318441;  // log2(e) / sqrt(128)

// What a producer warp tells the consumer warps about a staged page.
struct StageMeta {
    int page;   // cache page id of the staged page
    int bad;    // the block-table entry was out of range: nothing was copied
    int pos;    // RoPE position of the sequence (valid when a qkv row was staged)
    int pad;
};

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
static __device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int64_t timeout_ns,
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

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue, and wait for the previous kernel's results.
// atomicAdd with acquire semantics at GPU scope: what other threads released
// before their own increments is visible to this thread after it.
__device__ __forceinline__ int atomic_add_acquire(int* addr, int v) {
    int old;
    asm volatile("atom.acquire.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Tensor-core fragments (warp-level mma.sync, m16n8k16, bf16 in, float out)

// Four 8x8 b16 matrices from shared memory; lane l supplies the address of row
// l%8 of matrix l/8. Register r of each lane holds row (lane/4), columns
// 2*(lane%4) and +1 of matrix r (transposed: column lane/4, rows 2*(lane%4), +1).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}

// c += A(16x16, row-major) * B(16x8, column-major); bf16 operands, float accumulators.
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

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

// A float split into two bf16 whose sum carries ~16 significant bits:
// hi = bf16(x), lo = bf16(x - hi). Returns hi in the low half, lo in the high half.
__device__ __forceinline__ void split_bf16(float x, uint16_t& hi, uint16_t& lo) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi = __bfloat16_as_ushort(h);
    lo = __bfloat16_as_ushort(__float2bfloat16_rn(x - __bfloat162float(h)));
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

// Two floats in one 64-bit register pair (low word first), for the packed
// f32x2 arithmetic of sm_100: one instruction does two float FMAs.
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 pack2(float lo, float hi) {
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ float2 unpack2(f32x2 v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}

__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
    f32x2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// A word holding two bf16 (first element in the low half) as two floats.
__device__ __forceinline__ f32x2 bf2(uint32_t w) { return pack2(bf_lo(w), bf_hi(w)); }

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

}  // namespace qda
