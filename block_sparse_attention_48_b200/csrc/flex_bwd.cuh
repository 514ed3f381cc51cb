// Launch interface of the block-sparse FlexAttention backward pass.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "mask_eval.cuh"

namespace fa {

struct BwdParams {
    CUtensorMap tm_q;   // Q  [B, Hq, q_len, D]    box 64 x 128
    CUtensorMap tm_do;  // dO [B, Hq, q_len, D]    box 64 x 128
    CUtensorMap tm_k;   // K  [B, Hkv, kv_len, D]  box 64 x 128
    CUtensorMap tm_v;   // V  [B, Hkv, kv_len, D]  box 64 x 128
    CUtensorMap tm_dq;  // dQ accumulator, fp32 [B * Hq * nq * 128, D]  box 32 x 32 (reduction target)

    int32_t B, Hq, Hkv, G;
    int64_t q_len, kv_len;
    int32_t nq, nkv;
    int32_t num_units;              // B * Hkv * nkv work units (batch, kv head, kv block)
    int32_t num_sms;                // SMs of the device (persistent grids)

    // transposed BlockMask (read only)
    const int32_t* q_num;
    const int32_t* q_idx;
    const int32_t* full_q_num;
    const int32_t* full_q_idx;
    int32_t bm_B, bm_H;
    int32_t has_full;
    MaskParams mask;

    // score_mod
    int32_t score_kind;
    float scale;
    float softcap;                  // cap
    float softcap_in;               // scale / cap
    float softcap_inv;              // 1 / cap
    const float* slopes;            // [Hq]
    const uint16_t* bias;           // bf16 [B, Hq, q_len, kv_len] with strides below
    int64_t bias_st0, bias_st1, bias_st2;

    // per-row inputs (written by the prologue) and outputs
    const float* ld;                // [B * Hq * nq][2][128]: per query block, nl (the negated LSE in
                                    // log2 units, less the ALiBi column term; -inf for a row that
                                    // admits nothing or lies past q_len), then Delta
    uint16_t* dk;                   // bf16
    int64_t dk_st0, dk_st1, dk_st2;
    uint16_t* dv;                   // bf16
    int64_t dv_st0, dv_st1, dv_st2;

    int* status;
    uint64_t watchdog_ns;
};

// Per query row, padded to whole 128-row blocks: nl and Delta = rowsum(dO * O)
// in fp32 (the [2][128] blocks of BwdParams::ld), and a zeroed dQ accumulator
// row; one warp per row.
struct BwdPrepParams {
    const uint16_t* o;
    int64_t o_st0, o_st1, o_st2;
    const uint16_t* dout;
    int64_t do_st0, do_st1, do_st2;
    const float* lse;               // [B, Hq, q_len] natural log (forward output)
    const float* slopes;            // [Hq] ALiBi slopes, or null
    float* ld;
    float* dq_acc;                  // [B * Hq * nq * 128, D]
    int32_t Hq, D, nq;
    int64_t q_len, rows_pad;        // rows_pad = B * Hq * nq * 128
};

// dQ = scale * accumulator, converted to bf16.
struct BwdDqParams {
    const float* dq_acc;            // [B * Hq * nq * 128, D]
    uint16_t* dq;
    int64_t dq_st0, dq_st1, dq_st2;
    int32_t Hq, D, nq;
    int64_t q_len, rows;            // rows = B * Hq * q_len
    float scale;
};

cudaError_t launch_bwd_prep(const BwdPrepParams& p, cudaStream_t stream);
cudaError_t launch_flex_backward(const BwdParams& p, int D, cudaStream_t stream);
cudaError_t launch_bwd_dq(const BwdDqParams& p, cudaStream_t stream);

} // namespace fa
