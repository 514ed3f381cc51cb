// Launch interface of the FlexDecoding kernels (split-KV decode and the merge of
// the splits).
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

    int32_t splits;     // kv splits per (batch, kv head)
    float* part_o;      // [splits][B * Hq * q_len][D] fp32, unnormalised (splits > 1)
    float* part_ml;     // [splits][B * Hq * q_len][2]: running max (log2 units), sum

    int* status;
    uint64_t watchdog_ns;
};

// Number of kv splits fa_decode uses for a problem (a function of the grid it
// would otherwise launch and of the kv blocks available).
int decode_splits(int64_t B, int64_t Hkv, int32_t nkv, int sms);

cudaError_t launch_flex_decode(const DecParams& p, int D, cudaStream_t stream);
// Merge of the splits into O and LSE (splits > 1).
cudaError_t launch_decode_merge(const DecParams& p, int D, cudaStream_t stream);

} // namespace fa
