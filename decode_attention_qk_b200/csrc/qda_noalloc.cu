// Handle-free entry point whose scratch lives in a fixed device array, for
// callers that must not allocate device memory (see
// qwen3_decode_attn_append_and_attend_noalloc in include/qwen3_decode_attn.h).
//
// The decode-attention kernel needs scratch beyond its inputs and outputs:
// partial results of sequences whose pages are split across CTAs, one merge
// counter per (sequence, kv head), and a status word. Here that scratch is one
// statically sized __device__ array, created when the library's module is
// loaded on a device and kept until the process exits; no call allocates or
// frees anything.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "qda_internal.h"
#include "qwen3_decode_attn.h"

namespace {

// Largest grid this entry point launches: min(SM count, 160). With the
// largest batch (256) that is 160 + 256 = 416 partial slots.
constexpr int kNoAllocMaxGrid = 160;
constexpr int kNoAllocSlots = kNoAllocMaxGrid + qda::kMaxBatch;
constexpr size_t kPartAccBytes = (size_t)kNoAllocSlots * qda::kNumQHeads * qda::kHeadDim * sizeof(float);
constexpr size_t kPartMlBytes = (size_t)kNoAllocSlots * qda::kNumQHeads * sizeof(float2);
constexpr size_t kCounterBytes = (size_t)qda::kMaxBatch * qda::kNumKvHeads * sizeof(int);
constexpr size_t kStatusBytes = 256;
constexpr size_t kOffPartMl = kPartAccBytes;
constexpr size_t kOffCounters = kOffPartMl + kPartMlBytes;
constexpr size_t kOffStatus = kOffCounters + kCounterBytes;
// 3,469,568 bytes (about 3.3 MiB) on every device that loads the library.
constexpr size_t kScratchBytes = kOffStatus + kStatusBytes;
static_assert(kScratchBytes == 3469568, "the size the header states");
static_assert(kOffPartMl % 256 == 0 && kOffCounters % 256 == 0 && kOffStatus % 256 == 0, "256-byte sections");

static __device__ __align__(256) unsigned char g_qda_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
constexpr int64_t kTimeoutNs = 1000000000;  // 1 s per device-side wait

struct DeviceSetup {
    std::mutex mu;
    bool ready = false;                // set only by a set-up that succeeded
    unsigned char* scratch = nullptr;  // device address of g_qda_noalloc_scratch
    int grid = 0;
};
DeviceSetup g_setup[kMaxDevices];

// Once per device, with that device current: look up the device address of
// the scratch array (its name is only a host-side stand-in), raise the
// kernel's shared-memory limit, and size the grid. A set-up that fails (for
// instance when the first call is made during a stream capture, where the
// lookup may not run) leaves the device not ready and clears the CUDA error,
// so a later call tries again.
cudaError_t setup_device(int device, DeviceSetup& s) {
    std::lock_guard<std::mutex> lock(s.mu);
    if (s.ready) return cudaSuccess;
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_qda_noalloc_scratch);
    if (e == cudaSuccess) e = qda::prepare_device();
    int sms = 0;
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
    if (e == cudaSuccess && sms < 1) e = cudaErrorInvalidDevice;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return e;
    }
    s.scratch = static_cast<unsigned char*>(ptr);
    s.grid = sms < kNoAllocMaxGrid ? sms : kNoAllocMaxGrid;
    s.ready = true;
    return cudaSuccess;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" int qwen3_decode_attn_append_and_attend_noalloc(const void* qkv, const void* q_norm_w,
                                                           const void* k_norm_w, const int32_t* seq_lens,
                                                           const int32_t* positions, const int32_t* block_table,
                                                           int block_table_stride, void* k_cache, void* v_cache,
                                                           int num_pages, void* o, int batch, void* cuda_stream) {
    if (qkv == nullptr || q_norm_w == nullptr || k_norm_w == nullptr || seq_lens == nullptr ||
        block_table == nullptr || k_cache == nullptr || v_cache == nullptr || o == nullptr)
        return QDA_ERR_INVALID_ARG;
    // batch beyond the scratch's maximum (256 sequences) is refused here
    if (batch < 1 || batch > qda::kMaxBatch || block_table_stride < 1 || num_pages < 1) return QDA_ERR_INVALID_ARG;
    if (!aligned(qkv, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) ||
        !aligned(q_norm_w, 4) || !aligned(k_norm_w, 4) || !aligned(seq_lens, 4) || !aligned(block_table, 4) ||
        (positions != nullptr && !aligned(positions, 4)))
        return QDA_ERR_INVALID_ARG;

    int device = 0;
    if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDevices) return QDA_ERR_CUDA;
    DeviceSetup& s = g_setup[device];
    if (setup_device(device, s) != cudaSuccess) return QDA_ERR_CUDA;

    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    // The array keeps the previous call's contents: the merge counters must
    // start at zero, and the status word is cleared with them.
    if (cudaMemsetAsync(s.scratch + kOffCounters, 0, kCounterBytes + kStatusBytes, stream) != cudaSuccess)
        return QDA_ERR_CUDA;

    qda::Params p{};
    p.qkv = static_cast<const uint16_t*>(qkv);
    p.q_norm_w = static_cast<const uint16_t*>(q_norm_w);
    p.k_norm_w = static_cast<const uint16_t*>(k_norm_w);
    p.seq_lens = seq_lens;
    p.positions = positions;
    p.block_table = block_table;
    p.k_cache = static_cast<uint16_t*>(k_cache);
    p.v_cache = static_cast<uint16_t*>(v_cache);
    p.o = static_cast<uint16_t*>(o);
    p.num_q_heads = qda::kNumQHeads;
    p.new_tokens = 1;
    p.tok_stride = 1;
    p.bt_stride = block_table_stride;
    p.num_pages = num_pages;
    p.batch = batch;
    p.max_seq_len = QDA_MAX_SEQ_LEN;
    p.rope_theta = 1.0e6;
    p.rms_eps = 1.0e-6;
    p.part_acc = reinterpret_cast<float*>(s.scratch);
    p.part_ml = reinterpret_cast<float2*>(s.scratch + kOffPartMl);
    p.counters = reinterpret_cast<int*>(s.scratch + kOffCounters);
    p.status = reinterpret_cast<int*>(s.scratch + kOffStatus);
    p.timeout_ns = kTimeoutNs;
    p.flags = 0u;
    return qda::launch(p, s.grid, stream) == cudaSuccess ? QDA_OK : QDA_ERR_CUDA;
}
