// C-ABI entry points of the decode-attention library (declared in
// include/qwen3_decode_attn.h): argument checks, workspace ownership and the
// launch. All arithmetic of the step runs in the kernel (qda_decode_kernel.cu).
#include <cstdint>
#include <cstring>
#include <new>

#include <cuda_runtime.h>

#include "qda_internal.h"
#include "qda_prefill.h"
#include "qwen3_decode_attn.h"

struct qda_handle {
    int device = 0;
    qda_config cfg{};
    int grid = 0;
    float* part_acc = nullptr;
    float2* part_ml = nullptr;
    int* counters = nullptr;
    int* seg = nullptr;
    // the chunked prefill: query tiles [max_batch][8], partials (2 slots per
    // CTA of its attention launch)
    uint16_t* pf_q = nullptr;
    int2* pf_unit = nullptr;
    float* pf_acc = nullptr;
    float2* pf_ml = nullptr;
    int pf_grid = 0;
    int* status = nullptr;
    // input_norm + qkv_proj: the exact split of x*g, and 1/r per row
    uint16_t* xg_hi = nullptr;
    uint16_t* xg_lo = nullptr;
    float* inv_r = nullptr;
    // staging of the host-buffer entry point: two sets, used by alternate
    // calls, so that one call's stage-in overlaps the previous call's attention
    uint16_t* st_qkv[2] = {nullptr, nullptr};
    int32_t* st_seq_lens[2] = {nullptr, nullptr};
    int32_t* st_positions[2] = {nullptr, nullptr};
    int32_t* st_block_table[2] = {nullptr, nullptr};
    uint16_t* st_o[2] = {nullptr, nullptr};
    unsigned host_calls = 0;
};

namespace {

constexpr int64_t kDefaultTimeoutNs = 1000000000;  // 1 s

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// The query-head counts of the Qwen3 sizes: 16 (0.6B, 1.7B), 32 (4B, 8B),
// 40 (14B), 64 (32B), all over 8 kv heads of 128.
bool supported_q_heads(int n) { return n == 16 || n == 32 || n == 40 || n == 64; }

size_t qkv_elems(int num_q_heads) { return (size_t)(num_q_heads + 2 * qda::kNumKvHeads) * qda::kHeadDim; }

// Makes `device` current for the lifetime of the guard, then restores the
// caller's device.
class DeviceGuard {
  public:
    explicit DeviceGuard(int device) {
        ok_ = cudaGetDevice(&prev_) == cudaSuccess && cudaSetDevice(device) == cudaSuccess;
    }
    ~DeviceGuard() {
        if (ok_) cudaSetDevice(prev_);
    }
    bool ok() const { return ok_; }

  private:
    int prev_ = 0;
    bool ok_ = false;
};

void free_workspace(qda_handle* h) {
    cudaFree(h->part_acc);
    cudaFree(h->part_ml);
    cudaFree(h->counters);
    cudaFree(h->seg);
    cudaFree(h->pf_q);
    cudaFree(h->pf_unit);
    cudaFree(h->pf_acc);
    cudaFree(h->pf_ml);
    cudaFree(h->status);
    cudaFree(h->xg_hi);
    cudaFree(h->xg_lo);
    cudaFree(h->inv_r);
    for (int k = 0; k < 2; ++k) {
        cudaFree(h->st_qkv[k]);
        cudaFree(h->st_seq_lens[k]);
        cudaFree(h->st_positions[k]);
        cudaFree(h->st_block_table[k]);
        cudaFree(h->st_o[k]);
    }
}

template <typename T>
bool alloc(T** p, size_t bytes) {
    return cudaMalloc(reinterpret_cast<void**>(p), bytes) == cudaSuccess;
}

int check_call(const qda_handle* h, const void* qkv, const void* q_norm_w, const void* k_norm_w,
               const int32_t* seq_lens, const int32_t* positions, const int32_t* block_table,
               int block_table_stride, const void* k_cache, const void* v_cache, int num_pages, const void* o,
               int batch) {
    if (h == nullptr || qkv == nullptr || q_norm_w == nullptr || k_norm_w == nullptr || seq_lens == nullptr ||
        block_table == nullptr || k_cache == nullptr || v_cache == nullptr || o == nullptr)
        return QDA_ERR_INVALID_ARG;
    if (batch < 1 || batch > h->cfg.max_batch || block_table_stride < 1 || num_pages < 1)
        return QDA_ERR_INVALID_ARG;
    if (!aligned(qkv, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) ||
        !aligned(q_norm_w, 4) || !aligned(k_norm_w, 4) || !aligned(seq_lens, 4) || !aligned(block_table, 4) ||
        (positions != nullptr && !aligned(positions, 4)))
        return QDA_ERR_INVALID_ARG;
    return QDA_OK;
}

qda::Params make_params(const qda_handle* h, const void* qkv, const void* q_norm_w, const void* k_norm_w,
                        const int32_t* seq_lens, const int32_t* positions, const int32_t* block_table,
                        int block_table_stride, void* k_cache, void* v_cache, int num_pages, void* o, int batch) {
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
    p.num_q_heads = h->cfg.num_q_heads;
    p.new_tokens = 1;
    p.tok_stride = 1;
    p.tok_offset = 0;
    p.len_trim = 0;
    p.bt_stride = block_table_stride;
    p.num_pages = num_pages;
    p.batch = batch;
    p.max_seq_len = h->cfg.max_seq_len;
    p.rope_theta = h->cfg.rope_theta;
    p.rms_eps = h->cfg.rms_eps;
    p.part_acc = h->part_acc;
    p.part_ml = h->part_ml;
    p.counters = h->counters;
    p.seg = h->seg;
    p.status = h->status;
    p.timeout_ns = h->cfg.wait_timeout_ns > 0 ? h->cfg.wait_timeout_ns : kDefaultTimeoutNs;
    p.flags = h->cfg.flags;
    return p;
}

cudaError_t launch_step(const qda_handle* h, const qda::Params& p, cudaStream_t stream,
                        bool after_producer = false) {
    return p.num_q_heads == qda::kNumQHeads && p.new_tokens == 1 ? qda::launch(p, h->grid, stream, after_producer)
                                                                 : qda::launch_grouped(p, h->grid, stream);
}

// Whether the device can access `p` where it lies (page-locked host memory
// mapped into the current device's address space); *dev receives the address
// the device uses. Pageable or unknown memory answers no.
bool mapped_host(const void* p, void** dev) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();   // not a pointer CUDA knows: clear the error
        return false;
    }
    if (a.type != cudaMemoryTypeHost || a.devicePointer == nullptr) return false;
    *dev = a.devicePointer;
    return true;
}

// Host checks of the input_norm + qkv_proj arguments.
int check_proj(const qda_handle* h, const void* x, const void* input_norm_w, const void* w_qkv, int hidden,
               const void* qkv, int batch) {
    if (h == nullptr || x == nullptr || input_norm_w == nullptr || w_qkv == nullptr || qkv == nullptr)
        return QDA_ERR_INVALID_ARG;
    if (batch < 1 || batch > h->cfg.max_batch || hidden < 512 || hidden > qda::kMaxHidden || hidden % 512 != 0)
        return QDA_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(input_norm_w, 16) || !aligned(w_qkv, 16) || !aligned(qkv, 16))
        return QDA_ERR_INVALID_ARG;
    return QDA_OK;
}

qda::QkvProjParams make_proj_params(const qda_handle* h, const void* x, const void* input_norm_w, const void* w_qkv,
                                    int hidden, void* qkv, int batch) {
    qda::QkvProjParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.norm_w = static_cast<const uint16_t*>(input_norm_w);
    p.w = static_cast<const uint16_t*>(w_qkv);
    p.y = static_cast<uint16_t*>(qkv);
    p.batch = batch;
    p.hidden = hidden;
    p.qkv_width = (int)qkv_elems(h->cfg.num_q_heads);
    p.eps = h->cfg.rms_eps;
    p.xg_hi = h->xg_hi;
    p.xg_lo = h->xg_lo;
    p.inv_r = h->inv_r;
    p.status = h->status;
    p.timeout_ns = h->cfg.wait_timeout_ns > 0 ? h->cfg.wait_timeout_ns : kDefaultTimeoutNs;
    return p;
}

}  // namespace

extern "C" {

void qwen3_decode_attn_default_config(qda_config* cfg) {
    if (cfg == nullptr) return;
    std::memset(cfg, 0, sizeof(*cfg));
    cfg->num_q_heads = QDA_NUM_Q_HEADS;
    cfg->num_kv_heads = QDA_NUM_KV_HEADS;
    cfg->head_dim = QDA_HEAD_DIM;
    cfg->page_size = QDA_PAGE_SIZE;
    cfg->max_batch = QDA_MAX_BATCH;
    cfg->max_seq_len = QDA_MAX_SEQ_LEN;
    cfg->max_pages_per_seq = QDA_MAX_SEQ_LEN / QDA_PAGE_SIZE;
    cfg->rope_theta = 1.0e6;
    cfg->rms_eps = 1.0e-6;
    cfg->grid_ctas = 0;
    cfg->flags = 0u;
    cfg->wait_timeout_ns = 0;
}

int qwen3_decode_attn_create(const qda_config* cfg, int device, qda_handle** out) {
    if (out == nullptr) return QDA_ERR_INVALID_ARG;
    *out = nullptr;
    if (cfg == nullptr) return QDA_ERR_INVALID_ARG;
    if (!supported_q_heads(cfg->num_q_heads) || cfg->num_kv_heads != QDA_NUM_KV_HEADS ||
        cfg->head_dim != QDA_HEAD_DIM || cfg->page_size != QDA_PAGE_SIZE)
        return QDA_ERR_UNSUPPORTED;
    if (cfg->max_batch < 1 || cfg->max_batch > QDA_MAX_BATCH || cfg->max_seq_len < 1 ||
        cfg->max_seq_len > QDA_MAX_SEQ_LEN ||
        cfg->max_pages_per_seq < (cfg->max_seq_len + QDA_PAGE_SIZE - 1) / QDA_PAGE_SIZE ||
        !(cfg->rope_theta > 0.0) || !(cfg->rms_eps >= 0.0) || cfg->grid_ctas < 0 ||
        cfg->grid_ctas > qda::kMaxGridCtas || cfg->wait_timeout_ns < 0 ||
        (cfg->flags & ~QDA_FLAG_INJECT_WAIT_TIMEOUT) != 0u)
        return QDA_ERR_INVALID_ARG;
    if (device < 0) return QDA_ERR_INVALID_ARG;

    DeviceGuard guard(device);
    if (!guard.ok()) return QDA_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || sms < 1)
        return QDA_ERR_CUDA;
    if (qda::prepare_device() != cudaSuccess || qda::prepare_grouped() != cudaSuccess ||
        qda::prepare_qkv_proj() != cudaSuccess || qda::prepare_prefill() != cudaSuccess)
        return QDA_ERR_CUDA;

    qda_handle* h = new (std::nothrow) qda_handle();
    if (h == nullptr) return QDA_ERR_CUDA;
    h->device = device;
    h->cfg = *cfg;
    h->grid = cfg->grid_ctas > 0 ? cfg->grid_ctas : sms;
    h->pf_grid = sms;

    const size_t slots = (size_t)qda::num_slots(h->grid, cfg->max_batch);
    const size_t B = (size_t)cfg->max_batch;
    const size_t Hq = (size_t)cfg->num_q_heads;
    // partial rows per slot: 16 for the 16-head decode kernel, kPartRows (new
    // tokens x query heads) for the tensor-core kernel; size for the larger
    const size_t rows = (size_t)qda::kPartRows;
    bool ok = alloc(&h->part_acc, slots * rows * qda::kHeadDim * sizeof(float)) &&
              alloc(&h->part_ml, slots * rows * sizeof(float2)) &&
              alloc(&h->counters, (size_t)qda::kMaxBatch * qda::kNumKvHeads * sizeof(int)) &&
              alloc(&h->status, sizeof(int)) && alloc(&h->seg, (size_t)(qda::kMaxBatch + 1) * sizeof(int)) &&
              alloc(&h->pf_q, qda::prefill_q_bytes(cfg->max_batch)) &&
              alloc(&h->pf_unit, qda::prefill_unit_bytes(cfg->max_batch)) &&
              alloc(&h->pf_acc, qda::prefill_acc_bytes(sms)) && alloc(&h->pf_ml, qda::prefill_ml_bytes(sms)) &&
              alloc(&h->xg_hi, B * (size_t)qda::kMaxHidden * sizeof(uint16_t)) &&
              alloc(&h->xg_lo, B * (size_t)qda::kMaxHidden * sizeof(uint16_t)) &&
              alloc(&h->inv_r, B * sizeof(float));
    for (int k = 0; k < 2 && ok; ++k)
        ok = alloc(&h->st_qkv[k], B * qkv_elems(cfg->num_q_heads) * sizeof(uint16_t)) &&
             alloc(&h->st_seq_lens[k], B * sizeof(int32_t)) && alloc(&h->st_positions[k], B * sizeof(int32_t)) &&
             alloc(&h->st_block_table[k], B * (size_t)cfg->max_pages_per_seq * sizeof(int32_t)) &&
             alloc(&h->st_o[k], B * Hq * qda::kHeadDim * sizeof(uint16_t));
    ok = ok && cudaMemset(h->counters, 0, (size_t)qda::kMaxBatch * qda::kNumKvHeads * sizeof(int)) == cudaSuccess &&
         cudaMemset(h->pf_unit, 0, qda::prefill_unit_bytes(cfg->max_batch)) == cudaSuccess &&
         cudaMemset(h->status, 0, sizeof(int)) == cudaSuccess && cudaDeviceSynchronize() == cudaSuccess;
    if (!ok) {
        free_workspace(h);
        delete h;
        cudaGetLastError();  // clear the sticky-free allocation error
        return QDA_ERR_CUDA;
    }
    *out = h;
    return QDA_OK;
}

int qwen3_decode_attn_append_and_attend(qda_handle* h, const void* qkv, const void* q_norm_w, const void* k_norm_w,
                                        const int32_t* seq_lens, const int32_t* positions,
                                        const int32_t* block_table, int block_table_stride, void* k_cache,
                                        void* v_cache, int num_pages, void* o, int batch, void* cuda_stream) {
    int rc = check_call(h, qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table, block_table_stride, k_cache,
                        v_cache, num_pages, o, batch);
    if (rc != QDA_OK) return rc;
    DeviceGuard guard(h->device);
    if (!guard.ok()) return QDA_ERR_CUDA;
    const qda::Params p = make_params(h, qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table,
                                      block_table_stride, k_cache, v_cache, num_pages, o, batch);
    return launch_step(h, p, static_cast<cudaStream_t>(cuda_stream)) == cudaSuccess ? QDA_OK : QDA_ERR_CUDA;
}

int qwen3_decode_attn_append_and_attend_tokens(qda_handle* h, const void* qkv, const void* q_norm_w,
                                               const void* k_norm_w, const int32_t* seq_lens,
                                               const int32_t* positions, const int32_t* block_table,
                                               int block_table_stride, void* k_cache, void* v_cache, int num_pages,
                                               void* o, int batch, int new_tokens, void* cuda_stream) {
    int rc = check_call(h, qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table, block_table_stride, k_cache,
                        v_cache, num_pages, o, batch);
    if (rc != QDA_OK) return rc;
    if (new_tokens < 1 || new_tokens > QDA_MAX_NEW_TOKENS || new_tokens > h->cfg.max_seq_len)
        return QDA_ERR_INVALID_ARG;
    DeviceGuard guard(h->device);
    if (!guard.ok()) return QDA_ERR_CUDA;
    qda::Params p = make_params(h, qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table, block_table_stride,
                                k_cache, v_cache, num_pages, o, batch);
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    p.tok_stride = new_tokens;
    if (new_tokens == 1) return launch_step(h, p, st) == cudaSuccess ? QDA_OK : QDA_ERR_CUDA;
    if (new_tokens <= qda::grouped_max_tokens(h->cfg.num_q_heads)) {
        // up to 16 query rows per kv head: one launch of the decode-shaped
        // tensor-core kernel (and its combine)
        p.new_tokens = new_tokens;
        if (!qda::grouped_supported(h->cfg.num_q_heads, new_tokens)) return QDA_ERR_UNSUPPORTED;
        return qda::launch_grouped(p, h->grid, st) == cudaSuccess ? QDA_OK : QDA_ERR_CUDA;
    }
    // Longer blocks: the chunked prefill, up to kPrefillRows query rows per kv
    // head per chunk (the cache read once per chunk). Chunk [c0, c0 + n) sees
    // the cache plus the block's tokens up to its own (its launches trim the
    // later ones from seq_lens), so each token still attends over exactly the
    // slots up to its own.
    const qda::PrefillScratch sc{h->pf_q, h->pf_acc, h->pf_ml, h->pf_unit, h->pf_grid};
    const int max_t = qda::prefill_max_tokens(h->cfg.num_q_heads);
    for (int c0 = 0; c0 < new_tokens;) {
        const int n = new_tokens - c0 < max_t ? new_tokens - c0 : max_t;
        p.new_tokens = n;
        p.tok_offset = c0;
        p.len_trim = new_tokens - c0 - n;
        if (qda::launch_prefill(p, sc, st) != cudaSuccess) return QDA_ERR_CUDA;
        c0 += n;
    }
    return QDA_OK;
}

int qwen3_decode_attn_qkv_proj(qda_handle* h, const void* x, const void* input_norm_w, const void* w_qkv, int hidden,
                               void* qkv, int batch, void* cuda_stream) {
    int rc = check_proj(h, x, input_norm_w, w_qkv, hidden, qkv, batch);
    if (rc != QDA_OK) return rc;
    DeviceGuard guard(h->device);
    if (!guard.ok()) return QDA_ERR_CUDA;
    const qda::QkvProjParams p = make_proj_params(h, x, input_norm_w, w_qkv, hidden, qkv, batch);
    return qda::launch_qkv_proj(p, static_cast<cudaStream_t>(cuda_stream)) == cudaSuccess ? QDA_OK : QDA_ERR_CUDA;
}

int qwen3_decode_attn_o_proj(qda_handle* h, const void* x, const void* w_o, int hidden, void* y, int batch,
                             void* cuda_stream) {
    if (h == nullptr || x == nullptr || w_o == nullptr || y == nullptr) return QDA_ERR_INVALID_ARG;
    if (batch < 1 || batch > h->cfg.max_batch || hidden < 128 || hidden > qda::kMaxHidden || hidden % 128 != 0)
        return QDA_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w_o, 16) || !aligned(y, 16)) return QDA_ERR_INVALID_ARG;
    DeviceGuard guard(h->device);
    if (!guard.ok()) return QDA_ERR_CUDA;
    qda::OProjParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.w = static_cast<const uint16_t*>(w_o);
    p.y = static_cast<uint16_t*>(y);
    p.batch = batch;
    p.in_features = h->cfg.num_q_heads * qda::kHeadDim;
    p.hidden = hidden;
    p.status = h->status;
    p.timeout_ns = h->cfg.wait_timeout_ns > 0 ? h->cfg.wait_timeout_ns : kDefaultTimeoutNs;
    return qda::launch_o_proj(p, static_cast<cudaStream_t>(cuda_stream)) == cudaSuccess ? QDA_OK : QDA_ERR_CUDA;
}

int qwen3_decode_attn_from_hidden(qda_handle* h, const void* x, const void* input_norm_w, const void* w_qkv,
                                  int hidden, void* qkv, const void* q_norm_w, const void* k_norm_w,
                                  const int32_t* seq_lens, const int32_t* positions, const int32_t* block_table,
                                  int block_table_stride, void* k_cache, void* v_cache, int num_pages, void* o,
                                  int batch, void* cuda_stream) {
    int rc = check_proj(h, x, input_norm_w, w_qkv, hidden, qkv, batch);
    if (rc != QDA_OK) return rc;
    rc = check_call(h, qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table, block_table_stride, k_cache,
                    v_cache, num_pages, o, batch);
    if (rc != QDA_OK) return rc;
    DeviceGuard guard(h->device);
    if (!guard.ok()) return QDA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    const qda::QkvProjParams pp = make_proj_params(h, x, input_norm_w, w_qkv, hidden, qkv, batch);
    if (qda::launch_qkv_proj(pp, st) != cudaSuccess) return QDA_ERR_CUDA;
    const qda::Params p = make_params(h, qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table,
                                      block_table_stride, k_cache, v_cache, num_pages, o, batch);
    // the attention starts while the projection finishes; it reads qkv only after
    return launch_step(h, p, st, /*after_producer=*/true) == cudaSuccess ? QDA_OK : QDA_ERR_CUDA;
}

int qwen3_decode_attn_append_and_attend_host(qda_handle* h, const void* qkv_host, const void* q_norm_w,
                                             const void* k_norm_w, const int32_t* seq_lens_host,
                                             const int32_t* positions_host, const int32_t* block_table_host,
                                             int block_table_stride, void* k_cache, void* v_cache, int num_pages,
                                             void* o_host, int batch, void* cuda_stream) {
    if (h == nullptr) return QDA_ERR_INVALID_ARG;
    int rc = check_call(h, qkv_host, q_norm_w, k_norm_w, seq_lens_host, positions_host, block_table_host,
                        block_table_stride, k_cache, v_cache, num_pages, h->st_o[0], batch);
    if (rc != QDA_OK) return rc;
    if (o_host == nullptr || block_table_stride > h->cfg.max_pages_per_seq) return QDA_ERR_INVALID_ARG;
    DeviceGuard guard(h->device);
    if (!guard.ok()) return QDA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    const size_t B = (size_t)batch;
    // Alternate calls use alternate staging sets, so this call's stage-in
    // may run while the previous call's attention still reads its own set.
    const int k = (int)(h->host_calls++ & 1u);
    // Inputs in page-locked host memory that the device can address are
    // brought over by one stage-in launch; any other host memory by a copy
    // of its own. o in such memory is written by the attention kernel where
    // it is; otherwise it is copied out of the staging buffer.
    qda::StageParams sp{};
    auto bring = [&](const void* src, void* dst, size_t bytes) {
        void* dev = nullptr;
        if (mapped_host(src, &dev)) {
            sp.r[sp.n++] = qda::StageRange{dev, dst, bytes};
            return true;
        }
        return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, st) == cudaSuccess;
    };
    const bool ok = bring(qkv_host, h->st_qkv[k], B * qkv_elems(h->cfg.num_q_heads) * sizeof(uint16_t)) &&
                    bring(seq_lens_host, h->st_seq_lens[k], B * sizeof(int32_t)) &&
                    bring(block_table_host, h->st_block_table[k], B * (size_t)block_table_stride * sizeof(int32_t)) &&
                    (positions_host == nullptr || bring(positions_host, h->st_positions[k], B * sizeof(int32_t)));
    if (!ok || qda::launch_stage_in(sp, 2 * h->grid, st) != cudaSuccess) return QDA_ERR_CUDA;
    void* o_dev = nullptr;
    const bool o_mapped = mapped_host(o_host, &o_dev) && aligned(o_dev, 16);
    const qda::Params p = make_params(h, h->st_qkv[k], q_norm_w, k_norm_w, h->st_seq_lens[k],
                                      positions_host != nullptr ? h->st_positions[k] : nullptr, h->st_block_table[k],
                                      block_table_stride, k_cache, v_cache, num_pages, o_mapped ? o_dev : h->st_o[k],
                                      batch);
    if (launch_step(h, p, st) != cudaSuccess) return QDA_ERR_CUDA;
    if (!o_mapped && cudaMemcpyAsync(o_host, h->st_o[k], B * (size_t)h->cfg.num_q_heads * qda::kHeadDim * sizeof(uint16_t),
                                     cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return QDA_ERR_CUDA;
    return QDA_OK;
}

int qwen3_decode_attn_check(qda_handle* h, void* cuda_stream) {
    if (h == nullptr) return QDA_ERR_INVALID_ARG;
    DeviceGuard guard(h->device);
    if (!guard.ok()) return QDA_ERR_CUDA;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess) return QDA_ERR_CUDA;
    int status = 0;
    if (cudaMemcpy(&status, h->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return QDA_ERR_CUDA;
    if (status != 0) {
        // an aborted launch may leave merge counters mid-count: start them over
        if (cudaMemset(h->status, 0, sizeof(int)) != cudaSuccess ||
            cudaMemset(h->counters, 0, (size_t)qda::kMaxBatch * qda::kNumKvHeads * sizeof(int)) != cudaSuccess ||
            cudaDeviceSynchronize() != cudaSuccess)
            return QDA_ERR_CUDA;
    }
    return status;
}

int qwen3_decode_attn_grid_ctas(const qda_handle* h) { return h == nullptr ? 0 : h->grid; }

void qwen3_decode_attn_destroy(qda_handle* h) {
    if (h == nullptr) return;
    {
        DeviceGuard guard(h->device);
        free_workspace(h);
    }
    delete h;
}

const char* qwen3_decode_attn_strerror(int code) {
    switch (code) {
        case QDA_OK: return "success";
        case QDA_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, or a size outside its range)";
        case QDA_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
        case QDA_ERR_UNSUPPORTED:
            return "configuration differs from the compiled head geometry (16/32/40/64 query heads, 8 kv heads, "
                   "head dim 128, page 16) or has no kernel for this count of new tokens";
        case QDA_ERR_BOUNDS: return "a seq_len or block-table entry was out of range on the device";
        case QDA_ERR_TIMEOUT: return "a device-side wait ran out of time";
        default: return "unknown error code";
    }
}

}  // extern "C"
