// The 5th-generation tensor cores (tcgen05, accumulators in tensor memory)
// and the tensor memory accelerator's tiled copies, as used by the dense
// products of this library (the input and output projections of the
// attention block). Internal to the library.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "qda_device.cuh"

namespace qda {

// Shared-memory matrix descriptor of a K-major bf16 operand stored in the
// 128-byte swizzled layout that a tiled copy with CU_TENSOR_MAP_SWIZZLE_128B
// writes: rows of 64 elements (128 bytes), groups of 8 rows 1024 bytes apart,
// the 16-byte pieces of row r permuted by r % 8. Fields: start address >> 4 in
// bits [0,14), leading byte offset >> 4 in [16,30) (unused by this layout,
// 1 by convention), stride byte offset >> 4 in [32,46) (1024 bytes between
// 8-row groups), version 1 in [46,48), base offset 0 (the atom is 1024-byte
// aligned), layout 2 (128-byte swizzle) in [61,64). One K step of 16 elements
// (32 bytes) inside the atom is addressed by adding 32 * step to the start.
__host__ __device__ constexpr uint64_t umma_desc_sw128(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | (1ull << 16) | ((uint64_t)(1024u >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}

// Instruction descriptor of tcgen05.mma kind::f16: f32 accumulator (bits
// [4,6) = 1), bf16 A and B (bits [7,10) = 1, [10,13) = 1), both K-major (bits
// 15, 16 = 0), N >> 3 in [17,23), M >> 4 in [24,29); M = 128.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_m128(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
static_assert(umma_idesc_bf16_m128(64) == 0x08100490u, "instruction descriptor bits");

// The same with B MN-major (bit 16): B stored with its N index contiguous,
// as rows of K.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_m128_bmn(int n) {
    return umma_idesc_bf16_m128(n) | (1u << 16);
}

// Shared-memory matrix descriptor of an MN-major bf16 operand in the 128-byte
// swizzled layout: each K index is a 128-byte row of 64 consecutive MN
// elements, 8 such rows form a 1024-byte swizzle atom; the atoms of the next 8
// K indices are `sbo` bytes on, those of the next 64 MN elements `lbo` bytes
// on. Same fields as umma_desc_sw128; one K step of 16 rows is 2 atoms, so it
// advances the start by 2 * sbo.
__host__ __device__ constexpr uint64_t umma_desc_sw128_mn(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
static_assert(umma_desc_sw128(0x400u) == (0x40ull | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61)),
              "matrix descriptor bits");

// D[tmem] (+)= A * B^T for one K step of 16, issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The same with A (M x 16, K-major) in tensor memory at a_tmem: row i in lane
// i, two consecutive bf16 elements per 32-bit column (the lower-numbered one in
// the low half), 8 columns per instruction.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The mbarrier receives one arrival once every tensor-core instruction this
// thread issued before has completed (and has read its shared operands).
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Warp-wide: allocate `cols` tensor-memory columns (a power of two >= 32);
// the address goes to the shared word *dst.
__device__ __forceinline__ void tmem_alloc(void* dst, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)),
                 "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}

// Warp-wide: 16 consecutive columns of this warp's 32 tensor-memory lanes,
// lane i of the warp receiving lane (base + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Warp-wide: store 16 consecutive columns of this warp's 32 lanes (the
// inverse of tmem_ld16); tmem_st_wait() orders them before later accesses.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Warp-wide: 2 consecutive columns of this warp's 32 lanes, in or out.
__device__ __forceinline__ void tmem_ld2(uint32_t taddr, uint32_t (&v)[2]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(v[0]), "=r"(v[1]) : "r"(taddr));
}
__device__ __forceinline__ void tmem_st2(uint32_t taddr, const uint32_t (&v)[2]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(taddr), "r"(v[0]), "r"(v[1])
                 : "memory");
}

// One tiled copy of a 2-D box from global memory (described by `map`, a
// kernel parameter) into this CTA's shared memory at `dst`, completing its
// bytes on `bar`. (x, y) is the box's first element: x along the contiguous
// dimension (a multiple of 64 elements here, so 128-byte aligned), y the row.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// The whole thread-block cluster: release this thread's shared-memory writes,
// then wait for every thread of every CTA of the cluster.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The two halves of a cluster barrier, for a thread that arrives early (after
// initialising mbarriers, whose fence.mbarrier_init orders the
// initialisation) and waits only when it first touches a peer.
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// The shared::cluster address of the same shared-memory location in the
// cluster's CTA `rank`.
__device__ __forceinline__ uint32_t cluster_map(uint32_t local_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
    return r;
}

// An asynchronous 4-byte store into a peer CTA's shared memory (addresses from
// cluster_map) that completes 4 bytes of transaction on the peer's mbarrier
// `remote_bar`: the peer learns of the data's arrival from its own barrier.
__device__ __forceinline__ void st_async_f32(uint32_t remote_addr, float v, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(remote_addr),
                 "r"(__float_as_uint(v)), "r"(remote_bar)
                 : "memory");
}

}  // namespace qda
