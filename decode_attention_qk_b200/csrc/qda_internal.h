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
    int new_tokens;               // new tokens per sequence in this launch
    // A block of tok_stride new tokens per sequence (qkv [B][tok_stride][...],
    // o [B][tok_stride][...]) may run as several launches: this one covers
    // tokens [tok_offset, tok_offset + new_tokens) and sees each sequence
    // without the len_trim block tokens after them (seq_lens count them all).
    // The 16-head decode kernel runs only whole one-token blocks.
    int tok_stride;
    int tok_offset;
    int len_trim;
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
                                  // launch of the tensor-core kernel; unused at 16 heads)
    int* counters;                // [kMaxBatch][8] merge arrival counters, zero between calls
    int* status;                  // sticky device error (0 = none)
    int64_t timeout_ns;           // limit of every device-side wait
    unsigned flags;
    int qkv_after_wait;           // 16-head kernel: launched to depend on the launch writing qkv
};

// Partial rows per scratch slot of the tensor-core kernel: new tokens x query
// heads, at most 16 rows per kv head.
constexpr int kPartRows = 16 * kNumKvHeads;

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

// The tensor-core step (32, 40 or 64 query heads with one new token; T new
// tokens with T * Hq / 8 <= 16 query rows per kv head): the attention launch,
// then a launch that combines the partials of sequences split across CTAs.
cudaError_t launch_grouped(const Params& p, int grid, cudaStream_t stream);

// input_norm + attn.qkv_proj (qda_qkv_proj.cu): hidden size a multiple of 512,
// at most kMaxHidden (the Qwen3 sizes: 1024, 2048, 2560, 4096, 5120).
constexpr int kMaxHidden = 8192;

struct QkvProjParams {
    const uint16_t* x;        // bf16 [batch][hidden]
    const uint16_t* norm_w;   // bf16 [hidden], input_norm gain
    const uint16_t* w;        // bf16 [qkv_width][hidden], row n = output feature n
    uint16_t* y;              // bf16 [batch][qkv_width]
    int batch;
    int hidden;
    int qkv_width;            // (num_q_heads + 16) * 128, a multiple of 128
    double eps;
    // workspace: the exact split x*g = hi + lo, and 1 / r per row, formed by
    // the first launch
    uint16_t* xg_hi;          // bf16 [batch][hidden]
    uint16_t* xg_lo;          // bf16 [batch][hidden]
    float* inv_r;             // [batch]
    int* status;
    int64_t timeout_ns;
};

// A dense product on the 5th-generation tensor cores (qda_qkv_proj.cu):
//   y[b][n] = row_scale[b] * sum_k w[n][k] * (act_hi[b][k] + act_lo[b][k])
// with bf16 operands (row-major, k contiguous, 16-byte aligned rows), float
// sums and one rounding to bf16. act_lo may be null (one term); row_scale may
// be null (scale 1). k is a multiple of 256, n_out a multiple of 128.
struct LinearOperands {
    const void* w;            // bf16 [n_out][k]
    const void* act_hi;       // bf16 [batch][k]
    const void* act_lo;       // bf16 [batch][k] or nullptr
};
struct LinearParams {
    uint16_t* y;              // bf16 [batch][n_out]
    const float* row_scale;   // [batch] or nullptr
    int batch;
    int k;
    int n_out;
    int wait_acts;            // the activations and row scales come from the previous launch on the stream
    int* status;
    int64_t timeout_ns;
    // set by launch_linear
    int cols;                 // batch rows per CTA (a multiple of 16, <= 64)
    int k_split;              // K parts per tile (a thread-block cluster when > 1)
    int two_terms;
};
// How a product is cut: batch rows per CTA, K parts, batch groups, for a GPU
// of `sms` SMs.
void linear_split(int batch, int n_out, int k, int sms, int& cols, int& k_split, int& groups);

// attn.o_proj: y[b][n] = sum_k x[b][k] * w[n][k], x = the attention output
// o [batch][Hq][128] read as rows of in_features = Hq * 128.
struct OProjParams {
    const uint16_t* x;        // bf16 [batch][in_features]
    const uint16_t* w;        // bf16 [hidden][in_features]
    uint16_t* y;              // bf16 [batch][hidden]
    int batch;
    int in_features;
    int hidden;               // a multiple of 128
    int* status;
    int64_t timeout_ns;
};
cudaError_t launch_o_proj(const OProjParams& p, cudaStream_t stream);
cudaError_t launch_linear(const LinearOperands& ops, const LinearParams& p, cudaStream_t stream);

cudaError_t prepare_qkv_proj();
cudaError_t launch_qkv_proj(const QkvProjParams& p, cudaStream_t stream);

// Stage-in of the host-buffer entry point (qda_host_stage.cu): copy up to
// kMaxStageRanges ranges from device-addressable host memory (page-locked and
// mapped) to device memory in one launch. Every range is 4-byte aligned at
// both ends and a multiple of 4 bytes long. The launch is a programmatic
// dependent of the previous launch on the stream: it reads and writes while
// that launch may still run (so neither may touch these ranges), and it
// completes only after that launch has.
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

// The largest count of new tokens one tensor-core launch takes at this head
// count (at most 16 query rows per kv head).
int grouped_max_tokens(int num_q_heads);

// Prepare the tensor-core kernels on the current device.
cudaError_t prepare_grouped();

}  // namespace qda
