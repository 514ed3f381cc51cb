// Launch interface of the FlexDecoding kernels (split-KV decode and the merge of
// the partial results).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "mask_eval.cuh"

namespace fa {

constexpr int kDecodeMaxRows = 16;  // query rows of one kv head's group: G * q_len

struct DecParams {
    CUtensorMap tm_k;  // K [B, Hkv, kv_len, D]  box 64 x 128
    CUtensorMap tm_v;  // V [B, Hkv, kv_len, D]  box 64 x 128

    const uint16_t* q;  // Q [B, Hq, q_len, D] bf16
    int64_t q_st0, q_st1, q_st2;
    uint16_t* o;        // O [B, Hq, q_len, D] bf16
    int64_t o_st0, o_st1, o_st2;
    float* lse;         // [B, Hq, q_len] or null

    int32_t B, Hq, Hkv, G, q_len;
    int64_t kv_len;
    int32_t nkv;
    int32_t rows;       // G * q_len query rows per kv head (<= kDecodeMaxRows)

    // BlockMask row of query block 0 (one row per batch when bm_B > 1; head-independent)
    const int32_t* kv_num;
    const int32_t* kv_idx;
    const int32_t* full_num;
    const int32_t* full_idx;
    int32_t bm_B, has_full;
    MaskParams mask;

    int32_t score_kind;
    float scale;        // natural-units multiplier of Q.K
    float softcap, softcap_in, softcap_inv;
    const float* slopes;
    const uint16_t* bias;
    int64_t bias_st0, bias_st1, bias_st2;

    // Work split: the kv blocks of all (batch, kv head) segments as one list,
    // CTA c of `grid` taking the c-th equal share.  Each CTA writes, per compute
    // warp, one partial result for every piece of a segment it holds, as
    // partial number (segment + c), segment = b * Hkv + hk:
    int32_t grid;
    float* part_o;      // [B * Hkv + grid][8 warps][rows][D] fp32, unnormalised
    float* part_ml;     // [B * Hkv + grid][8 warps][rows][2]: running max (log2 units), sum
    int32_t* seg_first; // [B * Hkv]: the first and last CTA holding blocks of a segment
    int32_t* seg_last;
    long long* total;   // the list's length, written by CTA 0 for the merge

    int* status;
    uint64_t watchdog_ns;
};

constexpr int kDecodeWarps = 8;  // compute warps of a decode CTA, one partial result each

cudaError_t launch_flex_decode(const DecParams& p, int D, cudaStream_t stream);
// Merge of the partial results into O and LSE.
cudaError_t launch_decode_merge(const DecParams& p, int D, cudaStream_t stream);

} // namespace fa
