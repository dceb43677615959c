// Stage-in of the host-buffer entry point: one launch that reads a step's
// per-step inputs (qkv, seq_lens, positions, block table) from page-locked
// host memory mapped into the device's address space and writes them to the
// handle's device staging buffers.
//
// A copy-engine transfer pays a fixed start-up cost per buffer, and a kernel
// that reads its small inputs across the host link itself stalls on one
// link round trip after another (every CTA of the attention step reads every
// sequence length before it can start). Here all CTAs issue 16-byte loads at
// once, so the link's latency is paid about once per launch and the transfer
// runs at the link's bandwidth.
//
// Overlap with the step before. The entry point alternates between two sets
// of staging buffers, so this launch never writes what the previous step's
// attention reads. It is then launched as a programmatic dependent of that
// attention: its CTAs (no shared memory, 256 threads) fit beside the
// attention's on the same SMs and bring the next step's inputs across the
// link while the previous step's pages stream. It waits for the previous
// launch to complete only at its end, so that its own completion (which the
// next attention launch waits for) still implies the previous step's.
#include <cstdint>

#include <cuda_runtime.h>

#include "qda_device.cuh"
#include "qda_internal.h"

namespace qda {
namespace {

constexpr int kStageThreads = 256;

__global__ void __launch_bounds__(kStageThreads) stage_in_kernel(StageParams sp) {
    // the attention launch that follows may be scheduled now; it waits for
    // this launch to complete before it reads anything
    pdl_launch_dependents();
    const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t nthreads = (size_t)gridDim.x * blockDim.x;
#pragma unroll
    for (int r = 0; r < kMaxStageRanges; ++r) {
        if (r >= sp.n) break;
        const StageRange rg = sp.r[r];
        const size_t words = rg.bytes / 4;
        size_t done_words = 0;
        if (((reinterpret_cast<uintptr_t>(rg.src) | reinterpret_cast<uintptr_t>(rg.dst)) & 15) == 0) {
            // 16-byte body, four loads in flight per thread before the stores
            const size_t vecs = rg.bytes / 16;
            const uint4* src = static_cast<const uint4*>(rg.src);
            uint4* dst = static_cast<uint4*>(rg.dst);
            size_t i = tid;
            for (; i + 3 * nthreads < vecs; i += 4 * nthreads) {
                uint4 a = src[i], b = src[i + nthreads], c = src[i + 2 * nthreads], d = src[i + 3 * nthreads];
                dst[i] = a;
                dst[i + nthreads] = b;
                dst[i + 2 * nthreads] = c;
                dst[i + 3 * nthreads] = d;
            }
            for (; i < vecs; i += nthreads) dst[i] = src[i];
            done_words = vecs * 4;
        }
        // 4-byte words: the tail of the 16-byte body, or a range not 16-byte aligned
        const uint32_t* src = static_cast<const uint32_t*>(rg.src);
        uint32_t* dst = static_cast<uint32_t*>(rg.dst);
        for (size_t i = done_words + tid; i < words; i += nthreads) dst[i] = src[i];
    }
    // complete only once the previous launch has (it may still be running when
    // this one is a programmatic dependent of it)
    pdl_wait();
}

}  // namespace

cudaError_t launch_stage_in(const StageParams& sp, int max_ctas, cudaStream_t stream) {
    if (sp.n <= 0) return cudaSuccess;
    size_t vecs = 0;
    for (int r = 0; r < sp.n; ++r) vecs += (sp.r[r].bytes + 15) / 16;
    // one 16-byte load per thread, up to max_ctas CTAs (the rest loop)
    const size_t want = (vecs + kStageThreads - 1) / kStageThreads;
    const int grid = (int)(want < 1 ? 1 : (want > (size_t)max_ctas ? (size_t)max_ctas : want));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(kStageThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, stage_in_kernel, sp);
}

}  // namespace qda
