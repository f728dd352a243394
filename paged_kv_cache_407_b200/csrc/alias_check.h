// Host checks of the check build (PKV_CHECK): the caller guarantees that the
// cache write and the block copy rely on, verified before anything is queued.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pkv.h"

namespace pkv {

// PKV_ERR_ALIAS if a non-negative slot occurs twice among the num_tokens
// device-resident slots (copied to the host; the stream is synchronised).
// PKV_ERR_CUDA if the copy fails or the stream is capturing;
// PKV_ERR_TOO_LARGE if the host copy cannot be allocated.
pkv_status check_unique_slots(const int64_t *slot_mapping, int32_t num_tokens, cudaStream_t stream);

// PKV_ERR_ALIAS if, among the (src, dst) pairs with both ids in
// [0, num_blocks) (the ones the kernel copies), a dst occurs twice or also
// occurs as a src.  Same host copy and synchronisation.
pkv_status check_copy_pairs(const int64_t *block_pairs, int32_t num_pairs, int64_t num_blocks,
                            cudaStream_t stream);

}  // namespace pkv
