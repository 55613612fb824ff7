// append_check.cuh -- the opt-in check behind PKV_LAUNCH_CHECK_APPENDS.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace pkv {

// Records PKV_ERR_APPEND_CONFLICT in `err` when the appends of one call
// (position seq_lens[b] - 1 of each sequence b, through the block-table slab
// `bt` [batch][max_blocks]) race: two of them name one slot, or -- when
// `fused` -- one names a slot that a context of the same call reads.  Reads
// only bt and seq_lens; launched without programmatic dependent launch.
cudaError_t launch_append_check(const int32_t* bt, const int32_t* seq_lens, int32_t* err,
                                int32_t batch, int32_t max_blocks, int32_t num_pages,
                                bool fused, cudaStream_t stream);

// Bytes of the slot bitmap launch_fill_check needs for a pool of num_pages.
size_t fill_check_bitmap_bytes(int32_t num_pages);

// Records PKV_ERR_APPEND_CONFLICT in `err` when two rows of one pkv_fill call
// (same arguments as pkv_fill) write the same slot.  `bits`: device scratch
// of fill_check_bitmap_bytes(num_pages), cleared here on `stream`.
cudaError_t launch_fill_check(const int32_t* bt, const int32_t* cu, const int32_t* start,
                              uint32_t* bits, int32_t* err, int32_t batch, int32_t max_blocks,
                              int32_t num_pages, int32_t total_tokens, cudaStream_t stream);

}  // namespace pkv
