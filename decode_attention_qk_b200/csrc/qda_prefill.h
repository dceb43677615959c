// Blocks of many new tokens per sequence (a chunked prefill) with query
// tiles of their own: up to 128 query rows per kv head per launch, the cache
// read once per launch. Internal to the library.
#pragma once

#include <cuda_runtime.h>

#include "qda_internal.h"

namespace qda {

// Query rows per kv head one prefill launch takes (8 warps x 16 rows).
constexpr int kPrefillRows = 128;
// Blocks with at least this many query rows per kv head (T * Hq / 8) run as
// the prefill; shorter ones as launches of up to 16 rows of the
// decode-shaped tensor-core kernel.
constexpr int kPrefillFrom = 64;

// Partial scratch of the prefill attention: 2 slots per CTA (its first and
// its last unit piece), kPrefillRows rows each.
struct PrefillScratch {
    float* acc;     // [2 * grid][kPrefillRows][128]
    float2* ml;     // [2 * grid][kPrefillRows]
    int grid;       // CTAs of the attention launch
};
inline size_t prefill_acc_bytes(int grid) { return (size_t)2 * grid * kPrefillRows * kHeadDim * sizeof(float); }
inline size_t prefill_ml_bytes(int grid) { return (size_t)2 * grid * kPrefillRows * sizeof(float2); }

// Raise the attention kernel's shared-memory limit on the current device.
cudaError_t prepare_prefill();

// New tokens a prefill launch takes at this head count (kPrefillRows / G).
int prefill_max_tokens(int num_q_heads);

// One launch's worth of the chunked prefill: tokens [p.tok_offset,
// p.tok_offset + p.new_tokens) of blocks of p.tok_stride per sequence, with
// p.new_tokens * num_q_heads / 8 <= kPrefillRows. Three programmatic
// dependent launches: the append of the tokens' k and v to the cache, the
// attention, and the combine of units split across CTAs.
cudaError_t launch_prefill(const Params& p, const PrefillScratch& s, cudaStream_t stream);

}  // namespace qda
