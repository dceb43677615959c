/*
 * qwen3_decode_attn.h -- C ABI of the Qwen3-0.6B decode-attention step for
 * NVIDIA B200 (sm_100a).
 *
 * One call performs, for every sequence b of a decode batch, the attention
 * nodes of the Qwen3-0.6B Model Spec (docs.theformalera.com/models/qwen3-0-6b,
 * table "Compute-graph nodes"):
 *
 *   attn.qk_norm  per-head RMSNorm of the 16 query and 8 key heads over their
 *                 128 dims, eps = 1e-6, one gain vector shared by every head
 *                 (also: nnterp encyclopedia, qwen3, "Queries and keys are
 *                 normed per head, before the rotary");
 *   attn.rope     rotation of each pair (x_i, x_{i+64}), i < 64, by the angle
 *                 pos * theta^(-2i/128), theta = 1e6, counter-clockwise:
 *                 (a, b) -> (a cos - b sin, b cos + a sin);
 *   cache append  the new key (rounded once to bf16, nearest-even) and the new
 *                 value (its bits) are written to cache slot seq_lens[b]-1 of a
 *                 paged cache with 16-token pages (Model Spec, "At a glance",
 *                 shape domain);
 *   attn.core     decodeGQA: o[b,h] = sum_{s < seq_lens[b]} softmax_s(
 *                 <q[b,h], k[b,s,h/2]> / sqrt(128)) v[b,s,h/2], 16 query heads
 *                 over 8 kv heads (Supported models page, "What every spec
 *                 covers": one new query per sequence over seq_lens[b] cached
 *                 positions; nnterp qwen3, "Grouped-query attention").
 *
 * The larger Qwen3 sizes have the same attention with 32 (4B, 8B), 40 (14B)
 * or 64 (32B) query heads over the same 8 kv heads of 128 (nnterp qwen3,
 * "Grouped-query attention, with 128-wide heads on every size"); a handle
 * created with num_q_heads = Hq serves that size, and query head h then reads
 * kv head h / (Hq / 8). Below, Hq = 16 for Qwen3-0.6B.
 *
 * Tensor layouts (all little-endian, row-major, no padding):
 *
 *   qkv          bf16 [B][(Hq + 16) * 128]: Hq q heads x 128 | 8 k heads x 128 |
 *                8 v heads x 128, the attn.qkv_proj output row (N = 4096 at Hq = 16).
 *   q_norm_w     bf16 [128]; k_norm_w bf16 [128].
 *   seq_lens     int32 [B]. Counts the new token: 1 <= seq_lens[b] <= the
 *                handle's max_seq_len (<= 40960) and <= 16 * block_table_stride.
 *   positions    int32 [B] RoPE positions, or NULL for seq_lens[b]-1. The cache
 *                slot is seq_lens[b]-1 either way.
 *   block_table  int32 [B][block_table_stride]; logical slot t of sequence b
 *                lives in page block_table[b][t/16], row t%16. Entries past
 *                ceil(seq_lens[b]/16) are never read.
 *   k_cache,     bf16 [num_pages][16][8][128] each: page, token row, kv head,
 *   v_cache      dim. One page of one cache is 32 KiB, contiguous.
 *   o            bf16 [B][Hq][128].
 *
 * Numbers: the new k is normed and rotated in double precision and rounded
 * once to bf16 (nearest-even) when stored; q is normed and rotated in float,
 * its rotation angle formed and reduced modulo 2*pi in double, and is never
 * rounded to bf16; the scores, the softmax and the value accumulation are
 * float; o is rounded once to bf16 (nearest-even).
 *
 * Ownership: every tensor is caller-owned memory. The handle owns only its
 * workspace (device scratch for split partials, merge counters and the status
 * word, and the staging buffers of the host-buffer entry point), allocated by
 * qwen3_decode_attn_create and freed by qwen3_decode_attn_destroy.
 *
 * Streams: the attention entry points are asynchronous on the given stream
 * (a cudaStream_t passed as void*, NULL for the legacy default stream) and do
 * not synchronize. A handle's workspace serves one call at a time: calls that
 * share a handle must be ordered (same stream, or explicit events).
 *
 * Errors: functions return QDA_OK (0) or a negative QDA_ERR_* code; nothing
 * aborts, traps or prints. Argument errors are found on the host before any
 * launch. Errors found on the device (an index out of range, a bounded wait
 * that ran out) are recorded in the handle's sticky status word and returned
 * by qwen3_decode_attn_check.
 *
 * Preconditions the library relies on and does not check: the page that
 * receives a sequence's new token is not read or written by another sequence
 * of the same call; tensors do not overlap one another.
 */
#ifndef QWEN3_DECODE_ATTN_H
#define QWEN3_DECODE_ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Geometry of Qwen3-0.6B (Model Spec, "Published configuration":
 * num_attention_heads 16, num_key_value_heads 8, head_dim 128; "At a glance":
 * page size 16, B <= 256, S <= 40960; attn.qkv_proj N = 4096). The kernels are
 * also compiled for 32, 40 and 64 query heads over the same 8 kv heads. */
#define QDA_NUM_Q_HEADS   16
#define QDA_NUM_KV_HEADS  8
#define QDA_HEAD_DIM      128
#define QDA_PAGE_SIZE     16
#define QDA_QKV_WIDTH     4096
#define QDA_MAX_BATCH     256
#define QDA_MAX_SEQ_LEN   40960
#define QDA_MAX_NEW_TOKENS 40960 /* new tokens per sequence of one call (also <= max_seq_len) */

/* Return codes. */
#define QDA_OK               0
#define QDA_ERR_INVALID_ARG  (-1) /* null/misaligned pointer, size outside the domain */
#define QDA_ERR_CUDA         (-2) /* a CUDA runtime call or a launch failed */
#define QDA_ERR_UNSUPPORTED  (-3) /* config geometry differs from the compiled one */
#define QDA_ERR_BOUNDS       (-4) /* device: a seq_len or a block-table entry out of range */
#define QDA_ERR_TIMEOUT      (-5) /* device: a bounded wait ran out */

/* Create-time flags. */
#define QDA_FLAG_INJECT_WAIT_TIMEOUT 0x1u /* test only: every launch makes one warp
                                             wait on a barrier that nothing completes,
                                             until wait_timeout_ns runs out; the call
                                             still computes its result and records
                                             QDA_ERR_TIMEOUT */

typedef struct qda_handle qda_handle; /* opaque */

typedef struct {
    int num_q_heads;        /* 16 (Qwen3-0.6B, 1.7B), 32 (4B, 8B), 40 (14B) or 64 (32B) */
    int num_kv_heads;       /* must be 8 */
    int head_dim;           /* must be 128 */
    int page_size;          /* must be 16 */
    int max_batch;          /* 1..256: largest B a call may pass */
    int max_seq_len;        /* 1..40960: largest seq_lens[b] accepted */
    int max_pages_per_seq;  /* block-table row capacity of the host-buffer entry
                               point's staging; >= ceil(max_seq_len/16) */
    double rope_theta;      /* RoPE base, > 0 (1e6 for Qwen3-0.6B) */
    double rms_eps;         /* RMSNorm epsilon, >= 0 (1e-6 for Qwen3-0.6B) */
    int grid_ctas;          /* 0: one CTA per SM. > 0: exactly that many CTAs
                               (<= 4096), which changes how the key range of a
                               sequence is split; the result must not change */
    unsigned flags;         /* QDA_FLAG_* */
    int64_t wait_timeout_ns;/* limit of every device-side wait; 0: 1 second */
} qda_config;

/* Fill *cfg with the Qwen3-0.6B values: 16/8/128/16, max_batch 256,
 * max_seq_len 40960, max_pages_per_seq 2560, theta 1e6, eps 1e-6, grid 0,
 * flags 0, timeout 0. */
void qwen3_decode_attn_default_config(qda_config *cfg);

/* Create a handle bound to CUDA device `device` (made current during the
 * call). Allocates the workspace on that device. On success *out receives the
 * handle; on failure *out is set to NULL.
 * Errors: INVALID_ARG (null pointer, a size outside its range),
 *         UNSUPPORTED (query heads not 16/32/40/64, or kv heads, head_dim or
 *         page_size not 8/128/16),
 *         CUDA (no such device, allocation failure). */
int qwen3_decode_attn_create(const qda_config *cfg, int device, qda_handle **out);

/* The decode-attention step on device buffers (layouts above, with the
 * handle's Hq). At 16 query heads it is one kernel launch (sequences whose
 * pages are split across CTAs are combined inside it); at 32, 40 or 64 a
 * second launch combines them. Every pointer is a
 * device pointer. qkv, k_cache, v_cache and o must be 16-byte aligned;
 * q_norm_w, k_norm_w, seq_lens, positions and block_table 4-byte aligned.
 * `batch` is B (1..max_batch); `num_pages` (>= 1) bounds every block-table
 * entry the call reads; `block_table_stride` (>= 1) is the row pitch in
 * entries.
 * On return the work is queued on `cuda_stream`. When it has run: k_cache and
 * v_cache hold the appended tokens (no other cache byte changes) and o holds
 * the attention output.
 * Errors: INVALID_ARG (found on the host; nothing is launched), CUDA (the
 * launch failed). Device-side errors go to the status word: a seq_len outside
 * [1, min(max_seq_len, 16*block_table_stride)] makes the call skip that
 * sequence (its o rows and cache are left untouched); a block-table entry
 * outside [0, num_pages) is not dereferenced (that page is skipped, the
 * sequence's o rows are then unspecified, and no append goes to it). */
int qwen3_decode_attn_append_and_attend(qda_handle *h,
                                        const void *qkv,
                                        const void *q_norm_w,
                                        const void *k_norm_w,
                                        const int32_t *seq_lens,
                                        const int32_t *positions,
                                        const int32_t *block_table,
                                        int block_table_stride,
                                        void *k_cache,
                                        void *v_cache,
                                        int num_pages,
                                        void *o,
                                        int batch,
                                        void *cuda_stream);

/* The step with T = new_tokens new tokens per sequence (several tokens
 * decoded at once, e.g. draft tokens to verify). Model Spec, "Compute-graph
 * nodes" (attn.qk_norm, attn.rope, attn.core, the paged append) applied to T
 * tokens, under "What to watch for": every layer is full causal attention.
 * Layouts: qkv is bf16 [B][T][(Hq + 16) * 128] (token t of sequence b at row
 * b*T + t); o is bf16 [B][T][Hq][128]. seq_lens[b] = L counts the T new
 * tokens, and L >= T. Token t is appended at cache slot L - T + t, with RoPE
 * position positions[b] + t (or L - T + t when positions is NULL), and its
 * query attends over slots 0 .. L - T + t: the cache before the call plus the
 * new tokens up to and including itself.
 * new_tokens = 1 is exactly qwen3_decode_attn_append_and_attend. For T > 1
 * with up to 16 query rows per kv head (T * Hq / 8 <= 16: T <= 8 at 16 query
 * heads, 4 at 32, 3 at 40, 2 at 64) one launch of the decode-shaped
 * tensor-core kernel takes the block, followed by one that combines the
 * sequences split across CTAs. Up to 8 query rows per kv head q and the
 * probabilities enter the tensor cores as two bf16 terms (about 16
 * significant bits); with 9 to 16 rows they enter as bf16 (8 bits), with
 * float sums either way. A longer block runs as a chunked prefill: chunks of
 * 128 / G tokens (G = Hq / 8; 64 tokens at 16 query heads, 32 at 32, 25 at
 * 40, 16 at 64), each chunk attending over the cache plus the block's tokens
 * up to its own, so the result is the same causal attention. A chunk is three
 * launches: its k and v appended and its query rows formed, the attention
 * (each kv head's query rows of the chunk as one 128-row tile on the tensor
 * cores, so the cache is read once per chunk; q and the probabilities in bf16,
 * float sums), and the combine.
 * Errors as for qwen3_decode_attn_append_and_attend, plus INVALID_ARG for
 * new_tokens outside [1, min(QDA_MAX_NEW_TOKENS, max_seq_len)]; on the
 * device, a seq_len below T is out of range like one above the limits. */
int qwen3_decode_attn_append_and_attend_tokens(qda_handle *h,
                                               const void *qkv,
                                               const void *q_norm_w,
                                               const void *k_norm_w,
                                               const int32_t *seq_lens,
                                               const int32_t *positions,
                                               const int32_t *block_table,
                                               int block_table_stride,
                                               void *k_cache,
                                               void *v_cache,
                                               int num_pages,
                                               void *o,
                                               int batch,
                                               int new_tokens,
                                               void *cuda_stream);

/* The step's input, from the hidden state: input_norm then attn.qkv_proj
 * (Model Spec, "Compute-graph nodes": rmsnorm over H = hidden with a gain
 * per feature and eps = the handle's rms_eps; then y[t,n] = sum_k x[t,k]
 * w[n,k], no bias):
 *   qkv[b,n] = sum_k (x[b,k] / sqrt(sum_j x[b,j]^2 / hidden + eps) * g[k]) * w_qkv[n,k]
 * Two launches on `cuda_stream`: one forms the normalised rows into the
 * handle's workspace, the second is the product on the tensor cores.
 * Layouts (device pointers, 16-byte aligned): x bf16 [B][hidden] (row
 * stride hidden); input_norm_w bf16 [hidden]; w_qkv bf16 [N][hidden] with
 * N = (num_q_heads + 16) * 128 of the handle (row n = output feature n, the
 * layout of a torch Linear weight; q rows, then k rows, then v rows); qkv
 * bf16 [B][N] (output). hidden is a multiple of 512 in [512, 8192]
 * (Qwen3: 1024 for 0.6B, 2048, 2560, 4096, 5120 for the larger sizes).
 * Nothing is rounded before qkv, which is rounded once to bf16: the products
 * x*g are split exactly into two bf16 terms for the tensor cores and summed
 * in float, so qkv is the correctly rounded value except where the float sum
 * lies within about 2^-19 (relative) of a rounding midpoint, where it may be
 * the neighbouring bf16 value.
 * Errors: INVALID_ARG (null or misaligned pointer, batch outside
 * [1, max_batch], hidden not a multiple of 512 in range), CUDA (a launch
 * failed). Device-side errors (a bounded wait that ran out) go to the status
 * word read by qwen3_decode_attn_check. */
int qwen3_decode_attn_qkv_proj(qda_handle *h,
                               const void *x,
                               const void *input_norm_w,
                               const void *w_qkv,
                               int hidden,
                               void *qkv,
                               int batch,
                               void *cuda_stream);

/* The step's consumer, attn.o_proj (Model Spec, "Compute-graph nodes":
 * linear, y[t,n] = sum_k x[t,k] w[n,k], K = 2048, N = 1024 for Qwen3-0.6B, no
 * bias), on the tensor cores, one launch:
 *   y[b,n] = sum_k o[b,k] * w_o[n,k]
 * Layouts (device pointers, 16-byte aligned): x bf16 [B][Hq * 128], the
 * attention output o [B][Hq][128] of this handle's head count read as rows
 * (the "Tensors of the main nodes" table gives attn.core's o [B, 16, 128]
 * and attn.o_proj's x [T, 2048]); w_o bf16 [hidden][Hq * 128] (row n =
 * output feature n, a torch Linear weight); y bf16 [B][hidden] (output).
 * hidden is a multiple of 128 in [128, 8192] (Qwen3: 1024 for 0.6B; 2048,
 * 2560, 4096, 5120 for the larger sizes). The products of two bf16 values are
 * exact and summed in float; y is rounded once to bf16. The launch is a
 * programmatic dependent of the previous launch on the stream: its first
 * weight copies overlap that launch's end, and it reads x only after that
 * launch has completed, so it may directly follow the attention call that
 * writes o.
 * Errors: INVALID_ARG (null or misaligned pointer, batch outside
 * [1, max_batch], hidden not a multiple of 128 in range), CUDA (the launch
 * failed). Device-side errors (a bounded wait that ran out) go to the status
 * word read by qwen3_decode_attn_check. */
int qwen3_decode_attn_o_proj(qda_handle *h,
                             const void *x,
                             const void *w_o,
                             int hidden,
                             void *y,
                             int batch,
                             void *cuda_stream);

/* qwen3_decode_attn_qkv_proj into `qkv` (caller-owned, bf16 [B][N], it
 * holds the step's qkv afterwards), then qwen3_decode_attn_append_and_attend
 * on it: the layer's attention from the hidden state, three or four launches
 * on `cuda_stream`. Arguments and errors as for those two calls. */
int qwen3_decode_attn_from_hidden(qda_handle *h,
                                  const void *x,
                                  const void *input_norm_w,
                                  const void *w_qkv,
                                  int hidden,
                                  void *qkv,
                                  const void *q_norm_w,
                                  const void *k_norm_w,
                                  const int32_t *seq_lens,
                                  const int32_t *positions,
                                  const int32_t *block_table,
                                  int block_table_stride,
                                  void *k_cache,
                                  void *v_cache,
                                  int num_pages,
                                  void *o,
                                  int batch,
                                  void *cuda_stream);

/* The same step for a caller whose per-step tensors are in HOST memory:
 * qkv_host, seq_lens_host, positions_host (or NULL) and block_table_host are
 * host pointers, and o_host is the host destination of o. q_norm_w, k_norm_w,
 * k_cache and v_cache stay device pointers (weights and cache are
 * device-resident state). qkv, seq_lens, positions and the block table are
 * brought into the handle's device staging buffers: those in page-locked host
 * memory that the device can address (from cudaHostAlloc / cudaMallocHost or
 * registered with cudaHostRegister, as cudaPointerGetAttributes reports it)
 * by one library launch that reads them across the host link, any others by
 * a copy each. o in such memory (16-byte aligned) is written by the attention
 * kernel where it lies; otherwise it is copied out of the staging buffer.
 * All of it is queued on `cuda_stream` and the call returns; o_host is valid after
 * the stream is synchronized, and the host buffers must not change before
 * then. The stage-in launch may start while the previous launch on the stream
 * still runs (alternate calls use alternate staging buffers): it reads the
 * host inputs at once, so they must be final when the call is made, and must
 * not be written by work queued before it. Requires block_table_stride <=
 * max_pages_per_seq. Errors as for qwen3_decode_attn_append_and_attend. */
int qwen3_decode_attn_append_and_attend_host(qda_handle *h,
                                             const void *qkv_host,
                                             const void *q_norm_w,
                                             const void *k_norm_w,
                                             const int32_t *seq_lens_host,
                                             const int32_t *positions_host,
                                             const int32_t *block_table_host,
                                             int block_table_stride,
                                             void *k_cache,
                                             void *v_cache,
                                             int num_pages,
                                             void *o_host,
                                             int batch,
                                             void *cuda_stream);

/* The same step for callers that must not allocate device memory. The pages
 * have no counterpart of this entry point; it exists for users of this
 * library who cannot call cudaMalloc: code embedded in a framework or server
 * that owns all device memory through its own pool and forbids allocations on
 * the side, plugins that are handed only pre-allocated buffers, and
 * latency-critical loops where an allocation (which can synchronize the
 * device, or fail for lack of memory at call time) is not acceptable. It needs
 * no handle, and it allocates and frees nothing.
 *
 * It computes what qwen3_decode_attn_append_and_attend computes, with the
 * Qwen3-0.6B constants (theta 1e6, eps 1e-6, max_seq_len 40960), on the
 * calling thread's current device; every pointer is a device pointer of that
 * device, with the layouts and alignment stated above. The caller still
 * passes every input and output. The kernel's scratch (partials of sequences
 * split across CTAs, merge counters, a status word) is one fixed device
 * array of 3,469,568 bytes that every GPU which loads the library holds until the
 * process exits. It is sized for at most 256 sequences per call (a larger
 * batch returns QDA_ERR_INVALID_ARG) and at most 160 CTAs per launch (the call
 * launches min(SM count, 160)).
 *
 * The first call on each device performs a one-time set-up there (it looks up
 * the array's device address and raises the kernel's shared-memory limit);
 * make that first call before any stream capture. A first call whose set-up
 * fails returns QDA_ERR_CUDA and leaves the device to be set up again by the
 * next call. Each call then zeroes the merge counters and the status word on
 * `cuda_stream` before it launches (a memset, so the launch does not overlap
 * the end of the work queued before it the way the handle entry point's
 * launches do). All
 * calls share the one array, which keeps the last call's contents: calls that
 * overlap on the GPU (different streams or threads without ordering between
 * them) race on it and produce wrong results. Device-side errors (an
 * out-of-range seq_len or page id, a wait that ran out) are not reported by
 * this entry point: the kernel still never reads or writes out of range, but
 * o is then undefined for the sequences concerned and nothing tells the
 * caller; callers who need that report use the handle entry points.
 * Errors: INVALID_ARG (as for qwen3_decode_attn_append_and_attend, or batch
 * > 256), CUDA (the set-up, the memset or the launch failed). */
int qwen3_decode_attn_append_and_attend_noalloc(const void *qkv,
                                                const void *q_norm_w,
                                                const void *k_norm_w,
                                                const int32_t *seq_lens,
                                                const int32_t *positions,
                                                const int32_t *block_table,
                                                int block_table_stride,
                                                void *k_cache,
                                                void *v_cache,
                                                int num_pages,
                                                void *o,
                                                int batch,
                                                void *cuda_stream);

/* Synchronize `cuda_stream`, read and clear the status word, and return the
 * first device error recorded since the last check (QDA_OK if none;
 * QDA_ERR_BOUNDS or QDA_ERR_TIMEOUT otherwise). After an error the handle's
 * merge counters are reset, so the handle stays usable. CUDA if a runtime call
 * fails. */
int qwen3_decode_attn_check(qda_handle *h, void *cuda_stream);

/* Number of CTAs one call launches (the grid size). */
int qwen3_decode_attn_grid_ctas(const qda_handle *h);

/* Free the workspace and the handle. NULL is ignored. The caller must ensure
 * no work that uses the handle is still queued. */
void qwen3_decode_attn_destroy(qda_handle *h);

/* Static, human-readable text for a return code. */
const char *qwen3_decode_attn_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* QWEN3_DECODE_ATTN_H */
