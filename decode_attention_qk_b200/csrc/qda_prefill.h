// Blocks of many new tokens per sequence (a chunked prefill) with query
// tiles of their own: up to 128 query rows per kv head per launch, the cache
// read once per launch. Internal to the library.
#pragma once

#include <cuda_runtime.h>

#include "qda_internal.h"

namespace qda {

// Query rows per kv head one prefill chunk takes: the M of one tensor-core
// tile. Blocks of more than 16 query rows per kv head (T * Hq / 8) run as the
// prefill; shorter ones as one launch of the decode-shaped tensor-core kernel.
constexpr int kPrefillRows = 128;

// One unit's query tile: kPrefillRows rows x 128 dims in bf16, as two 64-dim
// halves of 128-byte rows, the 16-byte pieces of row r permuted by r % 8 (the
// tensor cores' 128-byte swizzled layout).
constexpr int kPrefillQTileBytes = kPrefillRows * kHeadDim * 2;

// Scratch of the prefill: the query tiles the prep launch forms, and the
// partials of the attention, 2 slots per CTA (its first and its last unit
// piece), kPrefillRows rows each.
struct PrefillScratch {
    uint16_t* q;    // [max_batch][8][kPrefillQTileBytes / 2]
    float* acc;     // [2 * grid][kPrefillRows][128]
    float2* ml;     // [2 * grid][kPrefillRows]
    int2* unit;     // [max_batch][8]: per unit, the slot of its first piece and the CTA of its last
    int grid;       // CTAs of the attention launch
};
inline size_t prefill_q_bytes(int max_batch) { return (size_t)max_batch * kNumKvHeads * kPrefillQTileBytes; }
inline size_t prefill_unit_bytes(int max_batch) { return (size_t)max_batch * kNumKvHeads * sizeof(int2); }
inline size_t prefill_acc_bytes(int grid) { return (size_t)2 * grid * kPrefillRows * kHeadDim * sizeof(float); }
inline size_t prefill_ml_bytes(int grid) { return (size_t)2 * grid * kPrefillRows * sizeof(float2); }

// Raise the attention kernel's shared-memory limit on the current device.
cudaError_t prepare_prefill();

// New tokens a prefill launch takes at this head count (kPrefillRows / G).
int prefill_max_tokens(int num_q_heads);

// One launch's worth of the chunked prefill: tokens [p.tok_offset,
// p.tok_offset + p.new_tokens) of blocks of p.tok_stride per sequence, with
// p.new_tokens * num_q_heads / 8 <= kPrefillRows and p.batch at most the
// max_batch s.q was sized for. Three programmatic dependent launches: the prep
// (the tokens' k and v appended to the cache, their query tiles formed), the
// attention, and the combine of units split across CTAs.
cudaError_t launch_prefill(const Params& p, const PrefillScratch& s, cudaStream_t stream);

}  // namespace qda
