// Launch interface of the block-sparse FlexAttention forward kernel.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "mask_eval.cuh"

namespace fa {

// Device status bits written into the workspace status word.
enum : int { STATUS_TIMEOUT = 1, STATUS_BAD_BLOCKMASK = 2 };

struct FwdParams {
    CUtensorMap tm_q;     // Q  [B, Hq, q_len, D]   box 64 x 128
    CUtensorMap tm_k;     // K  [B, Hkv, kv_len, D] box 64 x 128
    CUtensorMap tm_v;     // V  [B, Hkv, kv_len, D] box 64 x 128
    CUtensorMap tm_bias;  // bias [B, Hq, q_len, kv_len] box 64 x 128 (BIAS only)

    int32_t B, Hq, Hkv, G;          // G = Hq / Hkv
    int64_t q_len, kv_len;
    int32_t nq, nkv;
    int32_t num_items;              // B * Hq * nq

    // BlockMask (read only)
    const int32_t* kv_num;
    const int32_t* kv_idx;
    const int32_t* full_num;
    const int32_t* full_idx;
    int32_t bm_B, bm_H;
    int32_t has_full;
    int32_t num_rows;               // rows to rank by tile count (bm_B * bm_H * nq), 0 = keep query-block order
    MaskParams mask;

    // score_mod
    float scale_log2;               // scale * log2(e)
    float softcap;                  // cap
    float softcap_in;               // scale / cap
    float softcap_inv;              // 1 / cap (BIAS_SOFTCAP: multiplies the bias)
    float softcap_out;              // cap * log2(e)
    const float* slopes;            // [Hq]

    // outputs
    uint16_t* o;                    // bf16 bits
    int64_t o_stride_b, o_stride_h, o_stride_s;
    float* lse;                     // [B, Hq, q_len] or null
    int32_t bias_b_bcast, bias_h_bcast;  // bias read at batch / head coordinate 0 (broadcast)

    // paged KV cache: K / V tiles of logical kv block kb of batch b come from page
    // page_table[b * pt_stride + kb] of the pools [num_pages, Hkv, 128, D]
    const int32_t* page_table;      // null: K / V are [B, Hkv, kv_len, D]
    int64_t pt_stride;
    int32_t num_pages;

    int* status;                    // device status word
    uint64_t watchdog_ns;
    int32_t selftest_stall;         // nonzero: the producer waits on a barrier nothing completes
};

// Launch on `stream` with `grid` persistent CTAs.  D in {64, 128}; score_kind an
// fa_score_kind; ext selects the instances with the work-order ranking and paged
// K / V compiled in (needed for a DOCUMENT leaf's ranking and for a page table).
// Code compiled into a set of kernel instances besides the base path: the
// longest-first ranking of BlockMask rows (masks with a DOCUMENT leaf) and the
// page-table read of paged K / V.
constexpr int kExtRank = 1, kExtPage = 2;
cudaError_t launch_flex_forward(const FwdParams& p, int D, int score_kind, int ext, int grid, cudaStream_t stream);
cudaError_t launch_flex_forward_base(const FwdParams& p, int D, int score_kind, int grid, cudaStream_t stream);
cudaError_t launch_flex_forward_ext(const FwdParams& p, int D, int score_kind, int grid, cudaStream_t stream);
cudaError_t launch_flex_forward_paged(const FwdParams& p, int D, int score_kind, int grid, cudaStream_t stream);

// Dynamic shared memory the kernel variant needs.
int flex_forward_smem_bytes(int D, int score_kind);

} // namespace fa
