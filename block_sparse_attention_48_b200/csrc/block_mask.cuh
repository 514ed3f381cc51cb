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

// The transposed view from the lists of launch_block_mask (same stream, after it).
struct TransposeLaunch {
    int32_t H, nq, nkv, has_full;
    const int32_t* kv_num_blocks;
    const int32_t* kv_indices;
    const int32_t* full_kv_num_blocks;
    const int32_t* full_kv_indices;
    int32_t* q_num_blocks;
    int32_t* q_indices;
    int32_t* full_q_num_blocks;
    int32_t* full_q_indices;
};

// Grid (nkv, H, B): one warp per transposed row.
cudaError_t launch_block_mask_transpose(const TransposeLaunch& p, int B, cudaStream_t stream);

} // namespace fa
