// Launch interface of the BlockMask build kernel.
#pragma once

#include <cuda_runtime.h>

#include "mask_eval.cuh"

namespace fa {

struct BlockMaskLaunch {
    MaskParams mask;
    int64_t q_len, kv_len;
    int32_t H, nq, nkv;
    int32_t* kv_num_blocks;
    int32_t* kv_indices;
    int32_t* full_kv_num_blocks;
    int32_t* full_kv_indices;
    int32_t split_full;  // 0: full tiles go to the partial lists too (full lists left empty)
};

// Grid (nq, H, B): one CTA per BlockMask row.
cudaError_t launch_block_mask(const BlockMaskLaunch& p, int B, cudaStream_t stream);

} // namespace fa
