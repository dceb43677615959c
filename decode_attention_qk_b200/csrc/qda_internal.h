// Internal interface between the C-ABI host code and the decode-attention
// kernel. Not installed; the public boundary is include/qwen3_decode_attn.h.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace qda {

// Geometry of Qwen3-0.6B attention (Model Spec, "Published configuration").
// The larger Qwen3 sizes keep 8 kv heads of 128 and have 32, 40 or 64 query
// heads (nnterp qwen3, "Grouped-query attention, with 128-wide heads on every
// size"); kNumQHeads and kGroup are the 0.6B values.
constexpr int kNumQHeads = 16;
constexpr int kNumKvHeads = 8;
constexpr int kGroup = kNumQHeads / kNumKvHeads;   // query heads per kv head
constexpr int kHeadDim = 128;
constexpr int kPage = 16;                          // tokens per cache page
constexpr int kQkvWidth = 4096;                    // 2048 q | 1024 k | 1024 v
constexpr int kMaxBatch = 256;
constexpr int kMaxSeqLen = 40960;
constexpr int kMaxGridCtas = 4096;

// One token row of a page holds every kv head: 8 x 128 bf16 = 2 KiB; a page of
// one cache is 16 rows = 32 KiB, contiguous.
constexpr int kRowBytes = kNumKvHeads * kHeadDim * 2;
constexpr int kPageBytes = kPage * kRowBytes;

// Everything one launch needs. Pointers are device pointers.
struct Params {
    const uint16_t* qkv;          // bf16 [B][(num_q_heads + 16) * 128]
    const uint16_t* q_norm_w;     // bf16 [128]
    const uint16_t* k_norm_w;     // bf16 [128]
    const int32_t* seq_lens;      // [B]
    const int32_t* positions;     // [B] or nullptr
    const int32_t* block_table;   // [B][bt_stride]
    uint16_t* k_cache;            // bf16 [num_pages][16][8][128]
    uint16_t* v_cache;
    uint16_t* o;                  // bf16 [B][new_tokens][num_q_heads][128]
    int num_q_heads;              // 16, 32, 40 or 64
    int new_tokens;               // new tokens per sequence (qkv is [B][new_tokens][...])
    int bt_stride;
    int num_pages;
    int batch;
    int max_seq_len;
    double rope_theta;
    double rms_eps;
    // workspace
    float* part_acc;              // [num_slots][rows][128] un-normalised partial sums; rows = 16 for the
                                  // 16-head kernel (ordered kv head, slot, head pair there), kPartRows
                                  // for the tensor-core kernel
    float2* part_ml;              // [num_slots][rows] (running max in log2 units, sum), same row order
    int* seg;                     // [kMaxBatch + 1] page offsets of the sequences (written for the combine
                                  // launch of the 32/40/64-head kernels; unused at 16 heads)
    int* counters;                // [kMaxBatch][8] merge arrival counters, zero between calls
    int* status;                  // sticky device error (0 = none)
    int64_t timeout_ns;           // limit of every device-side wait
    unsigned flags;
    int qkv_after_wait;           // 16-head kernel: launched to depend on the launch writing qkv
};

// Partial rows per scratch slot of the tensor-core kernel: new tokens x query
// heads, at most 8 rows per kv head.
constexpr int kPartRows = 8 * kNumKvHeads;

// Scratch slots a launch with `grid` CTAs and batches up to `max_batch` needs.
inline int64_t num_slots(int grid, int max_batch) { return (int64_t)grid + max_batch; }

// Dynamic shared memory of one CTA.
size_t smem_bytes();

// Prepare the kernel for launch on the current device (raises its dynamic
// shared-memory limit). Returns the first CUDA error.
cudaError_t prepare_device();

// Launch one decode-attention step with `grid` CTAs on `stream` (16 query
// heads), as a programmatic dependent launch: its CTAs may be scheduled while
// the previous launch on the stream ends, and they read and write global
// memory only after it has completed. after_producer: that previous launch
// writes qkv and nothing else this step reads, so K/V streaming starts at
// once and only qkv waits for it to complete.
cudaError_t launch(const Params& p, int grid, cudaStream_t stream, bool after_producer = false);

// The tensor-core step (32, 40 or 64 query heads with one new token; 16
// heads with 2..4 new tokens, 32 heads with 2): the attention launch, then a
// launch that combines the partials of sequences split across CTAs.
cudaError_t launch_grouped(const Params& p, int grid, cudaStream_t stream);

// input_norm + attn.qkv_proj (qda_qkv_proj.cu): hidden size a multiple of 512,
// at most kMaxHidden (the Qwen3 sizes: 1024, 2048, 2560, 4096, 5120). The
// product is split over kProjKSplits CTAs along K (a thread-block cluster).
constexpr int kMaxHidden = 8192;
constexpr int kProjKSplits = 4;
constexpr int kProjNTile = 128;     // output columns per CTA

struct QkvProjParams {
    const uint16_t* x;        // bf16 [batch][hidden]
    const uint16_t* norm_w;   // bf16 [hidden], input_norm gain
    const uint16_t* w;        // bf16 [qkv_width][hidden], row n = output feature n
    uint16_t* y;              // bf16 [batch][qkv_width]
    int batch;
    int hidden;
    int qkv_width;            // (num_q_heads + 16) * 128, a multiple of 32
    double eps;
    // workspace: the exact split x*g = hi + lo, and 1 / r per row (batches
    // above 32 rows, formed by a first launch)
    uint16_t* xg_hi;          // bf16 [batch][hidden]
    uint16_t* xg_lo;          // bf16 [batch][hidden]
    float* inv_r;             // [batch]
    int* status;
    int64_t timeout_ns;
};

cudaError_t prepare_qkv_proj();
cudaError_t launch_qkv_proj(const QkvProjParams& p, cudaStream_t stream);

// Stage-in of the host-buffer entry point (qda_host_stage.cu): copy up to
// kMaxStageRanges ranges from device-addressable host memory (page-locked and
// mapped) to device memory in one launch. Every range is 4-byte aligned at
// both ends and a multiple of 4 bytes long.
constexpr int kMaxStageRanges = 4;
struct StageRange {
    const void* src;   // the device's address of the host buffer
    void* dst;         // device memory
    size_t bytes;
};
struct StageParams {
    StageRange r[kMaxStageRanges];
    int n;
};
cudaError_t launch_stage_in(const StageParams& sp, int max_ctas, cudaStream_t stream);

// Whether the tensor-core kernel has an instance for this head and token count.
bool grouped_supported(int num_q_heads, int new_tokens);

// Prepare the tensor-core kernels on the current device.
cudaError_t prepare_grouped();

}  // namespace qda
