// Device-side evaluation of the enumerated mask_mod: per element, per tile
// (all-true / all-false / mixed summaries) and per row as 128-bit column masks.
//
// Leaves ("Concepts", sections mask_mod and Composing masks; paper review
// sec. 4.4 and 5.3):
//   causal    q >= kv
//   sliding   q - kv <= W
//   document  doc[b][q] == doc[b][kv]
//   prefix    kv < P
// combined by a single AND or OR.
#pragma once

#include <cstdint>

#include "flexattn.h"

namespace fa {

struct MaskParams {
    int32_t n_leaves;
    int32_t op;
    int32_t kind[FA_MAX_LEAVES];
    int64_t param[FA_MAX_LEAVES];
    const int32_t* doc_ids;
    int64_t doc_stride;
    int32_t has_doc;
    int64_t q_offset;  // position of query row 0
};

enum : int { SUM_FALSE = 0, SUM_TRUE = 1, SUM_MIXED = 2 };

// Summary of one leaf over the rectangle q in [q0, q1], kv in [k0, k1] (in-range,
// inclusive).  Interval leaves are decided exactly; the document leaf is decided
// from the id ranges of the two sides (qmin..qmax, kmin..kmax) where possible.
__device__ __forceinline__ int leaf_summary(const MaskParams& m, int i, int64_t q0, int64_t q1, int64_t k0,
                                            int64_t k1, int32_t qmin, int32_t qmax, int32_t kmin, int32_t kmax)
{
    switch (m.kind[i]) {
    case FA_LEAF_CAUSAL:
        if (k1 <= q0) return SUM_TRUE;
        if (k0 > q1) return SUM_FALSE;
        return SUM_MIXED;
    case FA_LEAF_SLIDING:
        if (q1 - k0 <= m.param[i]) return SUM_TRUE;
        if (q0 - k1 > m.param[i]) return SUM_FALSE;
        return SUM_MIXED;
    case FA_LEAF_PREFIX:
        if (k1 < m.param[i]) return SUM_TRUE;
        if (k0 >= m.param[i]) return SUM_FALSE;
        return SUM_MIXED;
    case FA_LEAF_DOCUMENT:
        if (qmax < kmin || kmax < qmin) return SUM_FALSE;
        if (qmin == qmax && kmin == kmax && qmin == kmin) return SUM_TRUE;
        return SUM_MIXED;
    default:
        return SUM_FALSE;
    }
}

// Combined summary: decided when the operator's absorbing value appears or all
// leaves agree; otherwise SUM_MIXED (the tile must be counted element by element).
__device__ __forceinline__ int mask_summary(const MaskParams& m, int64_t q0, int64_t q1, int64_t k0, int64_t k1,
                                            int32_t qmin, int32_t qmax, int32_t kmin, int32_t kmax)
{
    if (m.n_leaves == 0) return SUM_TRUE;
    int n_true = 0, n_false = 0;
    for (int i = 0; i < m.n_leaves; ++i) {
        int s = leaf_summary(m, i, q0, q1, k0, k1, qmin, qmax, kmin, kmax);
        n_true += (s == SUM_TRUE);
        n_false += (s == SUM_FALSE);
    }
    if (m.op == FA_MASK_OR) {
        if (n_true > 0) return SUM_TRUE;
        if (n_false == m.n_leaves) return SUM_FALSE;
    } else {
        if (n_false > 0) return SUM_FALSE;
        if (n_true == m.n_leaves) return SUM_TRUE;
    }
    return SUM_MIXED;
}

// Document-leaf words of one row: bit c of word j is doc[k0 + 32 j + c] == qdoc,
// for the in-range columns (k0 + c < kv_len).  Reads the tile's ids with 16-byte
// loads when the whole tile lies inside the id row and starts on a 16-byte
// boundary (id rows are 16-byte aligned; k0 is a multiple of 4).
__device__ __forceinline__ void doc_bits(const int32_t* doc_row, int64_t k0, int64_t kv_len, int32_t qdoc,
                                         uint32_t (&d)[4])
{
#pragma unroll
    for (int j = 0; j < 4; ++j) d[j] = 0u;
    if (k0 + 128 <= kv_len && (k0 & 3) == 0) {
        const int4* src = reinterpret_cast<const int4*>(doc_row + k0);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
            const int4 v = __ldg(src + c);
            const int j = (4 * c) >> 5, b = (4 * c) & 31;
            d[j] |= ((uint32_t)(v.x == qdoc) << b) | ((uint32_t)(v.y == qdoc) << (b + 1)) |
                    ((uint32_t)(v.z == qdoc) << (b + 2)) | ((uint32_t)(v.w == qdoc) << (b + 3));
        }
    } else {
        for (int c = 0; c < 128 && k0 + c < kv_len; ++c)
            d[c >> 5] |= (uint32_t)(__ldg(doc_row + k0 + c) == qdoc) << (c & 31);
    }
}

// Bits of the 32 columns [base, base + 32) that lie in [lo, hi] (tile-local
// columns; lo, hi already clamped to [-1, 128]).
__device__ __forceinline__ uint32_t range_bits32(int lo, int hi, int base)
{
    const int a = lo - base, b = hi - base;
    if (b < 0 || a > 31 || a > b) return 0u;
    const uint32_t ua = a < 0 ? 0u : (uint32_t)a;
    const uint32_t ub = b > 31 ? 31u : (uint32_t)b;
    return (0xFFFFFFFFu >> (31u - ub)) & (0xFFFFFFFFu << ua);
}

__device__ __forceinline__ int clamp_col(int64_t c)
{
    return c < -1 ? -1 : (c > 128 ? 128 : (int)c);
}

// The 128 columns of one row (query q) of the tile starting at kv = k0 as four
// 32-bit words: bit c of word w is the mask at kv = k0 + 32 w + c, ANDed with
// kv < kv_len.  `dbits` holds the DOCUMENT leaf's words (doc[q] == doc[kv]) when
// that leaf is present.  Interval leaves become column ranges of the tile, clamped
// to [-1, 128] so that the arithmetic is 32-bit.
__device__ __forceinline__ void row_mask_words(const MaskParams& m, int64_t q, int64_t k0, int64_t kv_len,
                                               const uint32_t (&dbits)[4], uint32_t (&w)[4])
{
    const bool is_or = (m.op == FA_MASK_OR);
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] = (m.n_leaves == 0 || !is_or) ? 0xFFFFFFFFu : 0u;
    const int64_t d = q - k0;  // the causal diagonal's column
    for (int i = 0; i < m.n_leaves; ++i) {
        uint32_t lw[4];
        const int kind = m.kind[i];
        if (kind == FA_LEAF_DOCUMENT) {
#pragma unroll
            for (int j = 0; j < 4; ++j) lw[j] = dbits[j];
        } else {
            int lo = 1, hi = 0;
            if (kind == FA_LEAF_CAUSAL) { lo = 0; hi = clamp_col(d); }
            else if (kind == FA_LEAF_SLIDING) { lo = clamp_col(d - m.param[i]); hi = 127; }
            else if (kind == FA_LEAF_PREFIX) { lo = 0; hi = clamp_col(m.param[i] - 1 - k0); }
#pragma unroll
            for (int j = 0; j < 4; ++j) lw[j] = range_bits32(lo, hi, 32 * j);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = is_or ? (w[j] | lw[j]) : (w[j] & lw[j]);
    }
    if (k0 + 128 > kv_len) {
        const int last = clamp_col(kv_len - 1 - k0);
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] &= range_bits32(0, last, 32 * j);
    }
}

// The transposed view for the backward pass: the 128 query columns of one key
// row (key kv) of the tile starting at q = q0, as four 32-bit words: bit c of
// word w is the mask at q = q0 + 32 w + c, ANDed with q < q_len.  `dbits` holds
// the DOCUMENT leaf's words (doc[q] == doc[kv]) when that leaf is present.
//   causal  q >= kv       -> columns from kv - q0 on
//   sliding q - kv <= W   -> columns up to kv - q0 + W
//   prefix  kv < P        -> every column or none
__device__ __forceinline__ void col_mask_words(const MaskParams& m, int64_t kv, int64_t q0, int64_t q_len,
                                               const uint32_t (&dbits)[4], uint32_t (&w)[4])
{
    const bool is_or = (m.op == FA_MASK_OR);
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] = (m.n_leaves == 0 || !is_or) ? 0xFFFFFFFFu : 0u;
    const int64_t d = kv - q0;  // the causal diagonal's column
    for (int i = 0; i < m.n_leaves; ++i) {
        uint32_t lw[4];
        const int kind = m.kind[i];
        if (kind == FA_LEAF_DOCUMENT) {
#pragma unroll
            for (int j = 0; j < 4; ++j) lw[j] = dbits[j];
        } else {
            int lo = 1, hi = 0;
            if (kind == FA_LEAF_CAUSAL) { lo = clamp_col(d); hi = 127; }
            else if (kind == FA_LEAF_SLIDING) {
                const int64_t W = m.param[i];
                lo = 0;
                hi = W > (int64_t(1) << 40) ? 128 : (W < -(int64_t(1) << 40) ? -1 : clamp_col(d + W));
            }
            else if (kind == FA_LEAF_PREFIX) { lo = 0; hi = kv < m.param[i] ? 127 : -1; }
#pragma unroll
            for (int j = 0; j < 4; ++j) lw[j] = range_bits32(lo, hi, 32 * j);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = is_or ? (w[j] | lw[j]) : (w[j] & lw[j]);
    }
    if (q0 + 128 > q_len) {
        const int last = clamp_col(q_len - 1 - q0);
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] &= range_bits32(0, last, 32 * j);
    }
}

} // namespace fa
