// Block-sparse FlexAttention backward pass for sm_100a.
//
// Gradients of out = softmax(mod(Q K^T * scale)) V with respect to Q, K and V
// ("Flex Attention" paper review sec. 3.1: the backward template; attention-gym
// "Concepts", BlockMask Internals: the transposed q_num_blocks / q_indices lists
// are "used in backward").  With P the probabilities (recomputed from the
// forward pass's LSE) and dO the upstream gradient:
//
//   dP = dO V^T,  Delta = rowsum(dO * O),  dS = P * (dP - Delta) * mod'(s)
//   dV = P^T dO,  dK = scale dS^T Q,       dQ = scale dS K
//
// One CTA per (batch, kv head, kv block): it keeps K and V of its block in shared
// memory and dK, dV in tensor memory, and walks the query blocks of the kv
// block's transposed BlockMask row for every query head of the kv head's group
// (partial tiles, where the mask is evaluated per element, then full ones).  Per
// tile the five products run on the tensor core:
//   S^T  = K Q^T      (TMEM, fp32)        dP^T = V dO^T   (TMEM, fp32)
//   dV  += P^T dO     (P^T bf16 in TMEM)  dK  += dS^T Q   (dS^T bf16 in TMEM)
//   dQ   = dS K       (dS bf16 in shared memory, fp32 result in TMEM)
// and dQ is added into an fp32 accumulator with vector reductions (several kv
// blocks contribute to one query row).
//
// Warps: 0-7 compute (thread = key row = TMEM lane; warps w and w + 4 share the
// rows of lane quadrant w and split the 128 query columns, and D, in halves),
// 8 TMA producer, 9 MMA issue.
#include <mutex>
#include <vector>

#include <cuda_runtime.h>

#include "context.cuh"
#include "flex_bwd.cuh"
#include "flex_fwd.cuh"
#include "ptx.cuh"
#include "score_math.cuh"

namespace fa {

namespace {

constexpr int kBwdThreads = 320;
constexpr int kComputeWarps = 8;
constexpr int kProdWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kBox = 16384;  // bytes of one 128-row x 64-column bf16 TMA box
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BCfg {
    static constexpr int TILE = 128 * D * 2;
    static constexpr int NSLOT = D == 64 ? 2 : 1;  // Q / dO slots
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = TILE;
    static constexpr int OFF_Q = 2 * TILE;
    static constexpr int OFF_DO = OFF_Q + NSLOT * TILE;
    static constexpr int OFF_DS = OFF_DO + NSLOT * TILE;  // dS [kv][q] bf16, 128-byte swizzle, two 64-column chunks
    static constexpr int OFF_LD = OFF_DS + 2 * kBox;       // [2 buffers][LSE log2, Delta][128] fp32
    static constexpr int SMEM = OFF_LD + 2 * 2 * 128 * 4 + 1024;
    // TMEM columns: S^T (P^T over its first 64), dP^T (dS^T over its first 64),
    // dV, dK; dQ in its own columns at D = 64 and over S^T at D = 128
    static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + D;
    static constexpr bool DQ_OVER_S = D == 128;
    static constexpr uint32_t COL_DQ = DQ_OVER_S ? 0u : 384u;
};

struct __align__(16) BShared {
    uint64_t kv_full;
    uint64_t qd_full[2], qd_empty[2];
    uint64_t sdp_full, pds_full, dq_full, dq_free;
    uint64_t ld_ready[2];  // the compute warps staged a tile's LSE / Delta (one arrival per warp)
    uint64_t s_read;       // the first column half read all of S^T, dP^T it needs (one arrival per warp)
    uint64_t drain;
    uint32_t tmem_base;
};

struct BTile {
    int hq, qb;
    bool partial;
};

// The tiles of one CTA, in the same order for every role: for each query head of
// the group, the partial then the full query blocks of the kv block's transposed
// row.  Counts and indices are clamped (a corrupt BlockMask is reported, never
// read out of bounds).
struct BwdWalk {
    int b, hk, kb;
    int g, t, np, n;
    const int32_t* plist;
    const int32_t* flist;

    __device__ __forceinline__ void load_row(const BwdParams& p, bool& bad)
    {
        const int hq = hk * p.G + g;
        const int mb = p.bm_B == 1 ? 0 : b, mh = p.bm_H == 1 ? 0 : hq;
        const int64_t r = ((int64_t)mb * p.bm_H + mh) * p.nkv + kb;
        int a = __ldg(p.q_num + r), f = p.has_full ? __ldg(p.full_q_num + r) : 0;
        if (a < 0 || a > p.nq) { bad = true; a = a < 0 ? 0 : p.nq; }
        if (f < 0 || f > p.nq) { bad = true; f = f < 0 ? 0 : p.nq; }
        np = a;
        n = a + f;
        plist = p.q_idx + r * p.nq;
        flist = p.has_full ? p.full_q_idx + r * p.nq : nullptr;
        t = 0;
    }

    __device__ __forceinline__ void init(const BwdParams& p, int b_, int hk_, int kb_, bool& bad)
    {
        b = b_;
        hk = hk_;
        kb = kb_;
        g = 0;
        load_row(p, bad);
    }

    __device__ __forceinline__ bool next(const BwdParams& p, BTile& out, bool& bad)
    {
        while (t >= n) {
            if (++g >= p.G) return false;
            load_row(p, bad);
        }
        int qb = t < np ? __ldg(plist + t) : __ldg(flist + (t - np));
        if (qb < 0 || qb >= p.nq) { bad = true; qb = qb < 0 ? 0 : p.nq - 1; }
        out.hq = hk * p.G + g;
        out.qb = qb;
        out.partial = t < np;
        ++t;
        return true;
    }
};

__device__ __forceinline__ void unit_coords(const BwdParams& p, int& b, int& hk, int& kb)
{
    // kv block slowest: under causal-like masks the first kv blocks have the most
    // query blocks, so the longest CTAs start first
    const int u = blockIdx.x;
    const int bh = p.B * p.Hkv;
    kb = u / bh;
    const int r = u - kb * bh;
    b = r / p.Hkv;
    hk = r - b * p.Hkv;
}

__device__ __forceinline__ uint64_t desc64(uint32_t hi, uint32_t lo)
{
    return ((uint64_t)hi << 32) | lo;
}

template <int D>
__device__ __forceinline__ void bwd_producer(const BwdParams& p, BShared& sh, uint8_t* smem, Watchdog& wd,
                                             bool& bad)
{
    using C = BCfg<D>;
    int b, hk, kb;
    unit_coords(p, b, hk, kb);
    if (elect_one_sync()) {
        mbar_arrive_expect_tx(&sh.kv_full, 2 * C::TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
            tma_load_4d(smem + C::OFF_K + c * kBox, &p.tm_k, &sh.kv_full, c * 64, kb * 128, hk, b);
            tma_load_4d(smem + C::OFF_V + c * kBox, &p.tm_v, &sh.kv_full, c * 64, kb * 128, hk, b);
        }
    }
    __syncwarp();
    BwdWalk w;
    w.init(p, b, hk, kb, bad);
    BTile tl;
    uint32_t i = 0;
    bool ok = true;
    while (ok && w.next(p, tl, bad)) {
        const uint32_t slot = i % C::NSLOT, use = i / C::NSLOT;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.qd_empty[slot], (use & 1) ^ 1, wd));
        if (!ok) break;
        if (elect_one_sync()) {
            mbar_arrive_expect_tx(&sh.qd_full[slot], 2 * C::TILE);
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                tma_load_4d(smem + C::OFF_Q + slot * C::TILE + c * kBox, &p.tm_q, &sh.qd_full[slot], c * 64,
                            tl.qb * 128, tl.hq, b);
                tma_load_4d(smem + C::OFF_DO + slot * C::TILE + c * kBox, &p.tm_do, &sh.qd_full[slot], c * 64,
                            tl.qb * 128, tl.hq, b);
            }
        }
        __syncwarp();
        ++i;
    }
    // Copies still in flight land before the CTA exits: wait (bounded) for the
    // last issued phase of every slot and for K / V.
    Watchdog dw{wd.failed ? 1000000ull : wd.limit_ns, false};
    mbar_wait(&sh.kv_full, 0, dw);
    for (uint32_t j = 0; j < (uint32_t)C::NSLOT && j < i; ++j) {
        const uint32_t last = i - 1 - j;
        dw.failed = false;
        mbar_wait(&sh.qd_full[last % C::NSLOT], (last / C::NSLOT) & 1, dw);
    }
    if ((threadIdx.x & 31) == 0 && (wd.failed || !ok)) atomicOr(p.status, STATUS_TIMEOUT);
}

template <int D>
__device__ __forceinline__ void bwd_mma(const BwdParams& p, BShared& sh, uint8_t* smem, uint32_t tmem, Watchdog& wd,
                                        bool& bad)
{
    using C = BCfg<D>;
    int b, hk, kb;
    unit_coords(p, b, hk, kb);
    const uint32_t hi_k = (uint32_t)(sdesc_sw128(0, 16, 1024) >> 32);
    const uint32_t hi_mn = (uint32_t)(sdesc_sw128(0, kBox, 1024) >> 32);
    const uint32_t k_desc = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_K), 16, 1024);
    const uint32_t v_desc = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_V), 16, 1024);
    const uint32_t k_mn = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_K), kBox, 1024);
    const uint32_t ds_mn = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_DS), kBox, 1024);
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
    constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, false, true);  // P^T dO, dS^T Q
    constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, true, true);    // dS K
    bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.kv_full, 0, wd));
    BwdWalk w;
    w.init(p, b, hk, kb, bad);
    BTile tl;
    uint32_t i = 0;
    while (ok && w.next(p, tl, bad)) {
        const uint32_t slot = i % C::NSLOT, use = i / C::NSLOT;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.qd_full[slot], use & 1, wd));
        if (ok && C::DQ_OVER_S && i > 0) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.dq_free, (i - 1) & 1, wd));
        if (!ok) break;
        const uint32_t q_k = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_Q + slot * C::TILE), 16, 1024);
        const uint32_t do_k = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_DO + slot * C::TILE), 16, 1024);
        tc_fence_after();
        if (elect_one_sync()) {
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint32_t off = (uint32_t)(((k / 4) * kBox + (k % 4) * 32) >> 4);
                umma_ss(tmem + C::COL_S, desc64(hi_k, k_desc + off), desc64(hi_k, q_k + off), idesc_s, k > 0);
            }
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint32_t off = (uint32_t)(((k / 4) * kBox + (k % 4) * 32) >> 4);
                umma_ss(tmem + C::COL_DP, desc64(hi_k, v_desc + off), desc64(hi_k, do_k + off), idesc_s, k > 0);
            }
            umma_commit(&sh.sdp_full);
        }
        __syncwarp();
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.pds_full, i & 1, wd));
        if (ok && !C::DQ_OVER_S && i > 0) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.dq_free, (i - 1) & 1, wd));
        if (!ok) break;
        const uint32_t q_mn = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_Q + slot * C::TILE), kBox, 1024);
        const uint32_t do_mn = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_DO + slot * C::TILE), kBox, 1024);
        tc_fence_after();
        if (elect_one_sync()) {
            // 16 rows of the K dimension (query rows, or key rows for dQ) per step: 2 KB
#pragma unroll
            for (int k = 0; k < 8; ++k)
                umma_ts(tmem + C::COL_DV, tmem + C::COL_S + 8 * k, desc64(hi_mn, do_mn + ((k * 2048) >> 4)),
                        idesc_acc, (i > 0 || k > 0) ? 1u : 0u);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                umma_ts(tmem + C::COL_DK, tmem + C::COL_DP + 8 * k, desc64(hi_mn, q_mn + ((k * 2048) >> 4)),
                        idesc_acc, (i > 0 || k > 0) ? 1u : 0u);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                umma_ss(tmem + C::COL_DQ, desc64(hi_mn, ds_mn + ((k * 2048) >> 4)),
                        desc64(hi_mn, k_mn + ((k * 2048) >> 4)), idesc_dq, k > 0);
            umma_commit(&sh.dq_full);
            umma_commit(&sh.qd_empty[slot]);
        }
        __syncwarp();
        ++i;
    }
    // every issued MMA completes before TMEM is released
    if (elect_one_sync()) umma_commit(&sh.drain);
    __syncwarp();
    Watchdog dw{wd.failed ? 1000000ull : wd.limit_ns, false};
    const bool drained = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.drain, 0, dw));
    if ((threadIdx.x & 31) == 0 && (wd.failed || !ok || !drained)) atomicOr(p.status, STATUS_TIMEOUT);
}

// Modified score and its derivative for one element: u = mod(s * scale) (natural
// units), g = d mod / d s_scaled.
template <int SCORE>
__device__ __forceinline__ void score_and_grad(const BwdParams& p, float s, float slope, float dist, float bias,
                                               float& u, float& g)
{
    if constexpr (SCORE == FA_SCORE_SOFTCAP || SCORE == FA_SCORE_BIAS_SOFTCAP) {
        const float y = SCORE == FA_SCORE_SOFTCAP ? s * p.softcap_in : fmaf(s, p.softcap_in, bias * p.softcap_inv);
        const float t = tanh_accurate(y);
        u = p.softcap * t;
        g = fmaf(-t, t, 1.0f);
    } else {
        u = s * p.scale;
        if constexpr (SCORE == FA_SCORE_ALIBI) u = fmaf(slope, dist, u);
        if constexpr (SCORE == FA_SCORE_BIAS) u += bias;
        g = 1.0f;
    }
}

template <int D, int SCORE>
__device__ __forceinline__ void bwd_compute(const BwdParams& p, BShared& sh, uint8_t* smem, uint32_t tmem,
                                            Watchdog& wd, bool& bad)
{
    using C = BCfg<D>;
    constexpr bool HAS_BIAS = SCORE == FA_SCORE_BIAS || SCORE == FA_SCORE_BIAS_SOFTCAP;
    int b, hk, kb;
    unit_coords(p, b, hk, kb);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int quad = warp & 3, half = warp >> 2;  // TMEM lane quadrant; column half
    const int row = quad * 32 + lane;             // key row of the tile = TMEM lane
    const int64_t kv = (int64_t)kb * 128 + row;
    const bool row_ok = kv < p.kv_len;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    float* ld = reinterpret_cast<float*>(smem + C::OFF_LD);
    const uint32_t ds_row = smem_u32(smem + C::OFF_DS) + row * 128;
    const int32_t* doc_row = p.mask.has_doc ? p.mask.doc_ids + (int64_t)b * p.mask.doc_stride : nullptr;
    const int32_t kvdoc = (doc_row && row_ok) ? __ldg(doc_row + kv) : 0;

    BwdWalk w;
    w.init(p, b, hk, kb, bad);
    BTile tl;
    uint32_t i = 0;
    bool ok = true;
    while (ok && w.next(p, tl, bad)) {
        const int64_t q0 = (int64_t)tl.qb * 128;
        const int64_t rowbase = ((int64_t)b * p.Hq + tl.hq) * p.q_len;
        // this tile's 128 query rows: LSE (log2 units; +inf for a row that admits
        // nothing, so that its probabilities are 0) and Delta, staged in shared memory
        float* lse2 = ld + (i & 1) * 256;
        float* dlt = lse2 + 128;
        const uint32_t ld_s = smem_u32(lse2);  // dlt is 512 bytes further
        if (half == 0) {
            const int64_t qm = q0 + row;
            float l2 = 0.f, dl = 0.f;
            if (qm < p.q_len) {
                const float l = __ldg(p.lse + rowbase + qm);
                l2 = l == -INFINITY ? INFINITY : l * kLog2e;
                dl = __ldg(p.delta + rowbase + qm);
            }
            lse2[row] = l2;
            dlt[row] = dl;
        }
        // every compute warp's values are in before any is read (a bounded wait:
        // the buffers alternate, and a warp is at most one tile ahead)
        mbar_arrive_warp(&sh.ld_ready[i & 1]);
        ok = mbar_wait(&sh.ld_ready[i & 1], (i >> 1) & 1, wd);
        if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }

        // column mask words: partial tiles, the ragged last query block, ragged key rows
        uint32_t mw[4] = {0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu};
        if (!row_ok) {
#pragma unroll
            for (int j = 0; j < 4; ++j) mw[j] = 0u;
        } else if (tl.partial) {
            // the mask sees query positions: rows plus the offset
            const int64_t off = p.mask.q_offset;
            uint32_t db[4] = {0u, 0u, 0u, 0u};
            if (doc_row) doc_bits(doc_row, q0 + off, p.q_len + off, kvdoc, db);
            col_mask_words(p.mask, kv, q0 + off, p.q_len + off, db, mw);
        } else if (q0 + 128 > p.q_len) {
            const int last = clamp_col(p.q_len - 1 - q0);
#pragma unroll
            for (int j = 0; j < 4; ++j) mw[j] = range_bits32(0, last, 32 * j);
        }
        const float slope = SCORE == FA_SCORE_ALIBI ? __ldg(p.slopes + tl.hq) : 0.f;
        const float dist0 = (float)(kv - q0 - p.mask.q_offset);  // kv - q position at column 0
        const uint16_t* bias_row = nullptr;
        if (HAS_BIAS) bias_row = p.bias + (int64_t)b * p.bias_st0 + (int64_t)tl.hq * p.bias_st1 + kv;

        ok = mbar_wait(&sh.sdp_full, i & 1, wd);
        if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
        tc_fence_after();
        // this warp's two 32-column chunks of the query columns (the chunk's mask word
        // is selected, not indexed, so the words stay in registers)
        const uint32_t mw_lo = half ? mw[2] : mw[0], mw_hi = half ? mw[3] : mw[1];
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * half + cc;
            const uint32_t mwc = cc ? mw_hi : mw_lo;
            uint32_t sv[32], dv[32];
            tmem_ld32(tmem + lane_base + C::COL_S + 32 * c, sv);
            tmem_ld32(tmem + lane_base + C::COL_DP + 32 * c, dv);
            tmem_ld_wait();
            if (half == 0 && cc == 1) {
                // the second half's P / dS chunks land in these columns
                tc_fence_before();
                mbar_arrive_warp(&sh.s_read);
            }
            uint32_t pk[16], dk[16];
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                // the four columns' LSE and Delta as 16-byte shared loads (the same
                // address in every lane: broadcast)
                const uint4 l4 = lds128(ld_s + (uint32_t)(32 * c + j) * 4u);
                const uint4 d4 = lds128(ld_s + 512u + (uint32_t)(32 * c + j) * 4u);
                const float lv[4] = {__uint_as_float(l4.x), __uint_as_float(l4.y), __uint_as_float(l4.z),
                                     __uint_as_float(l4.w)};
                const float dl[4] = {__uint_as_float(d4.x), __uint_as_float(d4.y), __uint_as_float(d4.z),
                                     __uint_as_float(d4.w)};
                float pr[4], dr[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int col = 32 * c + j + e;
                    const bool adm = (mwc >> (j + e)) & 1u;
                    float bias = 0.f;
                    if (HAS_BIAS && adm) bias = __uint_as_float((uint32_t)__ldg(bias_row + (q0 + col) * p.bias_st2) << 16);
                    float u, g;
                    score_and_grad<SCORE>(p, __uint_as_float(sv[j + e]), slope, dist0 - (float)col, bias, u, g);
                    const float pe = adm ? ex2_approx(fmaf(u, kLog2e, -lv[e])) : 0.f;
                    pr[e] = pe;
                    dr[e] = pe * (__uint_as_float(dv[j + e]) - dl[e]) * g;
                }
                pk[j / 2] = pack_bf16x2(pr[0], pr[1]);
                pk[j / 2 + 1] = pack_bf16x2(pr[2], pr[3]);
                dk[j / 2] = pack_bf16x2(dr[0], dr[1]);
                dk[j / 2 + 1] = pack_bf16x2(dr[2], dr[3]);
            }
            // P^T over S^T and dS^T over dP^T (columns already read), dS to shared memory
            if (half == 1 && cc == 0) {
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.s_read, i & 1, wd))) { ok = false; break; }
                tc_fence_after();
            }
            tmem_st16(tmem + lane_base + C::COL_S + 16 * c, pk);
            tmem_st16(tmem + lane_base + C::COL_DP + 16 * c, dk);
#pragma unroll
            for (int u4 = 0; u4 < 4; ++u4) {
                const int unit = (c & 1) * 4 + u4;
                sts128(ds_row + (c >> 1) * kBox + ((unit ^ (row & 7)) * 16), dk[4 * u4], dk[4 * u4 + 1],
                       dk[4 * u4 + 2], dk[4 * u4 + 3]);
            }
        }
        if (!ok) break;
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive_warp(&sh.pds_full);

        // dQ rows of this tile (thread = query row): add into the fp32 accumulator
        ok = mbar_wait(&sh.dq_full, i & 1, wd);
        if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
        tc_fence_after();
        const int64_t qr = q0 + row;
        float* acc = p.dq_acc + (rowbase + qr) * D;
#pragma unroll 1
        for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + C::COL_DQ + 32 * c, v);
            tmem_ld_wait();
            if (qr < p.q_len) {
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    red_add_v4(acc + 32 * c + j, __uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                               __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
            }
        }
        tc_fence_before();
        mbar_arrive_warp(&sh.dq_free);
        ++i;
    }
    if (!ok) {
        if (lane == 0) atomicOr(p.status, STATUS_TIMEOUT);
        return;
    }
    // dK = scale * (dS^T Q), dV = P^T dO of this kv block (zero if no query block
    // attends to it).  Every lane runs the (warp-collective) TMEM loads; only the
    // stores of key rows past kv_len are skipped.
    uint16_t* dk_row = p.dk + (int64_t)b * p.dk_st0 + (int64_t)hk * p.dk_st1 + kv * p.dk_st2;
    uint16_t* dv_row = p.dv + (int64_t)b * p.dv_st0 + (int64_t)hk * p.dv_st1 + kv * p.dv_st2;
#pragma unroll 1
    for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
        uint32_t a[32], v[32];
        if (i > 0) {  // uniform over the CTA
            tmem_ld32(tmem + lane_base + C::COL_DK + 32 * c, a);
            tmem_ld32(tmem + lane_base + C::COL_DV + 32 * c, v);
            tmem_ld_wait();
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) a[j] = v[j] = 0u;
        }
        uint32_t pa[16], pv[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            pa[j] = pack_bf16x2(__uint_as_float(a[2 * j]) * p.scale, __uint_as_float(a[2 * j + 1]) * p.scale);
            pv[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
        }
        if (row_ok) {
            uint4* dka = reinterpret_cast<uint4*>(dk_row + 32 * c);
            uint4* dva = reinterpret_cast<uint4*>(dv_row + 32 * c);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                dka[j] = make_uint4(pa[4 * j], pa[4 * j + 1], pa[4 * j + 2], pa[4 * j + 3]);
                dva[j] = make_uint4(pv[4 * j], pv[4 * j + 1], pv[4 * j + 2], pv[4 * j + 3]);
            }
        }
    }
}

template <int D, int SCORE>
__global__ void __launch_bounds__(kBwdThreads, 1) flex_bwd_kernel(const __grid_constant__ BwdParams p)
{
    using C = BCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ BShared sh;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x / 32;

    if (warp == kMmaWarp) {
        tmem_alloc(&sh.tmem_base, 512);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        mbar_init(&sh.kv_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh.qd_full[s], 1);
            mbar_init(&sh.qd_empty[s], 1);
        }
        mbar_init(&sh.sdp_full, 1);
        mbar_init(&sh.pds_full, kComputeWarps);
        mbar_init(&sh.dq_full, 1);
        mbar_init(&sh.dq_free, kComputeWarps);
        mbar_init(&sh.ld_ready[0], kComputeWarps);
        mbar_init(&sh.ld_ready[1], kComputeWarps);
        mbar_init(&sh.s_read, 4);
        mbar_init(&sh.drain, 1);
        mbar_fence_init();
    }
    if (warp == kProdWarp && (threadIdx.x & 31) == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_do);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    Watchdog wd{p.watchdog_ns, false};
    bool bad = false;
    if (warp == kProdWarp) bwd_producer<D>(p, sh, smem, wd, bad);
    else if (warp == kMmaWarp) bwd_mma<D>(p, sh, smem, tmem, wd, bad);
    else bwd_compute<D, SCORE>(p, sh, smem, tmem, wd, bad);
    if (bad) atomicOr(p.status, STATUS_BAD_BLOCKMASK);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// Delta and the zeroed accumulator: one warp per query row.
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdPrepParams p)
{
    const int64_t r = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (r >= p.rows) return;
    const int64_t q = r % p.q_len, bh = r / p.q_len;
    const int64_t hq = bh % p.Hq, b = bh / p.Hq;
    const uint16_t* o = p.o + b * p.o_st0 + hq * p.o_st1 + q * p.o_st2;
    const uint16_t* d = p.dout + b * p.do_st0 + hq * p.do_st1 + q * p.do_st2;
    float s = 0.f;
    for (int j = lane * 2; j < p.D; j += 64) {
        const uint32_t a = *reinterpret_cast<const uint32_t*>(o + j);
        const uint32_t c = *reinterpret_cast<const uint32_t*>(d + j);
        s = fmaf(__uint_as_float(a << 16), __uint_as_float(c << 16), s);
        s = fmaf(__uint_as_float(a & 0xFFFF0000u), __uint_as_float(c & 0xFFFF0000u), s);
    }
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o2);
    if (lane == 0) p.delta[r] = s;
    float4* acc = reinterpret_cast<float4*>(p.dq_acc + r * p.D);
    for (int j = lane; j < p.D / 4; j += 32) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dQ = scale * accumulator in bf16: one thread per 8 elements of a row.
__global__ void __launch_bounds__(256) bwd_dq_kernel(const BwdDqParams p)
{
    const int64_t e = ((int64_t)blockIdx.x * 256 + threadIdx.x) * 8;
    if (e >= p.rows * p.D) return;
    const int64_t r = e / p.D;
    const int j = (int)(e - r * p.D);
    const int64_t q = r % p.q_len, bh = r / p.q_len;
    const int64_t hq = bh % p.Hq, b = bh / p.Hq;
    const float4 a = *reinterpret_cast<const float4*>(p.dq_acc + e);
    const float4 c = *reinterpret_cast<const float4*>(p.dq_acc + e + 4);
    uint4 out;
    out.x = pack_bf16x2(a.x * p.scale, a.y * p.scale);
    out.y = pack_bf16x2(a.z * p.scale, a.w * p.scale);
    out.z = pack_bf16x2(c.x * p.scale, c.y * p.scale);
    out.w = pack_bf16x2(c.z * p.scale, c.w * p.scale);
    *reinterpret_cast<uint4*>(p.dq + b * p.dq_st0 + hq * p.dq_st1 + q * p.dq_st2 + j) = out;
}

template <int D, int SCORE>
cudaError_t launch_bwd_variant(const BwdParams& p, cudaStream_t stream)
{
    static_assert(BCfg<D>::SMEM + sizeof(BShared) <= 232448, "shared memory beyond 227 KB per CTA");
    static std::mutex mu;
    static std::vector<CtxKey> done;
    auto kern = flex_bwd_kernel<D, SCORE>;
    {
        CtxKey key;
        std::lock_guard<std::mutex> lock(mu);
        bool have = false;
        if (current_ctx(&key))
            for (const CtxKey& k : done) have |= k == key;
        if (!have) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, BCfg<D>::SMEM);
            if (e != cudaSuccess) return e;
            if (current_ctx(&key)) done.push_back(key);
        }
    }
    kern<<<p.num_units, kBwdThreads, BCfg<D>::SMEM, stream>>>(p);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_bwd_prep(const BwdPrepParams& p, cudaStream_t stream)
{
    if (p.rows == 0) return cudaSuccess;
    const int64_t blocks = (p.rows + 7) / 8;
    bwd_prep_kernel<<<(unsigned)blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_bwd_dq(const BwdDqParams& p, cudaStream_t stream)
{
    if (p.rows == 0) return cudaSuccess;
    const int64_t threads = p.rows * p.D / 8;
    bwd_dq_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_flex_backward(const BwdParams& p, int D, cudaStream_t stream)
{
    if (p.num_units == 0) return cudaSuccess;
#define FA_BWD_CASE(DD, SS) \
    if (D == DD && p.score_kind == SS) return launch_bwd_variant<DD, SS>(p, stream);
    FA_BWD_CASE(64, FA_SCORE_NONE) FA_BWD_CASE(64, FA_SCORE_ALIBI) FA_BWD_CASE(64, FA_SCORE_SOFTCAP)
    FA_BWD_CASE(64, FA_SCORE_BIAS) FA_BWD_CASE(64, FA_SCORE_BIAS_SOFTCAP)
    FA_BWD_CASE(128, FA_SCORE_NONE) FA_BWD_CASE(128, FA_SCORE_ALIBI) FA_BWD_CASE(128, FA_SCORE_SOFTCAP)
    FA_BWD_CASE(128, FA_SCORE_BIAS) FA_BWD_CASE(128, FA_SCORE_BIAS_SOFTCAP)
#undef FA_BWD_CASE
    return cudaErrorInvalidValue;
}

} // namespace fa
