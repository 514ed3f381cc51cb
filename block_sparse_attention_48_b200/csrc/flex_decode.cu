// FlexDecoding for sm_100a: the forward pass for a few query tokens against a
// long KV cache ("Flex Attention" paper review sec. 3.1, the decoding template;
// rocketrecap talk: decoding splits the work along the KV dimension and reduces
// the partial results at the end).
//
// With one to a few query tokens per sequence the contraction is tiny and the
// pass is bound by reading K and V from HBM, so this kernel does not use the
// 128-row tcgen05 tiles of the prefill kernel: the G query heads that share a
// kv head (GQA) and their q_len tokens are packed as the (at most 16) rows of
// warp-level m16n8k16 MMAs, and the kv blocks of the BlockMask row are split
// over CTAs (grid: split x kv head x batch).  Each CTA streams its kv blocks
// through a TMA ring; each of its eight compute warps takes 16 keys of every
// block and keeps its own online softmax (running max, sum, O); the warps are
// merged in shared memory, and the splits by a second kernel.
#include <mutex>
#include <vector>

#include <cuda_runtime.h>

#include "context.cuh"
#include "flex_decode.cuh"
#include "flex_fwd.cuh"
#include "ptx.cuh"
#include "score_math.cuh"

namespace fa {

namespace {

constexpr int kDecWarps = 8;                     // compute warps, 16 keys of each block each
constexpr int kDecThreads = 32 * (kDecWarps + 1);  // plus the TMA producer warp
constexpr int kDecProdWarp = kDecWarps;
constexpr int kBox = 16384;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
struct DCfg {
    static constexpr int TILE = 128 * D * 2;           // one K or V block
    // ring stages: about 192 KB of copies in flight per SM (two CTAs per SM at D = 64)
    static constexpr int NS = 3;
    static constexpr int STAGE = 2 * TILE;             // K then V
    static constexpr int SMEM = NS * STAGE + 1024;
    static constexpr int MIN_CTAS = 1;
    // warp-merge scratch (reuses the ring once every block is consumed)
    static constexpr int MERGE = kDecWarps * kDecodeMaxRows * (D + 2) * 4;
    static_assert(MERGE <= NS * STAGE, "merge scratch exceeds the ring");
};

struct __align__(16) DShared {
    uint64_t full[3], empty[3];
    uint64_t consumed;  // every compute warp consumed its last block (one arrival per warp)
    uint64_t written;   // every compute warp wrote its partial result
};

// Address of element row `key`, 16-byte unit `unit` (8 bf16 of D) of a tile
// loaded by TMA with the 128-byte swizzle (64-column chunks of 16 KB).
__device__ __forceinline__ uint32_t swz(uint32_t base, int key, int unit)
{
    return base + (uint32_t)((unit >> 3) * kBox + key * 128 + (((unit & 7) ^ (key & 7)) << 4));
}

// One mask element at query position q and key kv (the DOCUMENT leaf compares
// the query's id qdoc with the key's).
__device__ __forceinline__ bool mask_elem(const MaskParams& m, int32_t qdoc, const int32_t* doc_row, int64_t q,
                                          int64_t kv)
{
    if (m.n_leaves == 0) return true;
    const bool is_or = m.op == FA_MASK_OR;
    bool acc = !is_or;
    for (int i = 0; i < m.n_leaves; ++i) {
        bool x;
        switch (m.kind[i]) {
        case FA_LEAF_CAUSAL: x = q >= kv; break;
        case FA_LEAF_SLIDING: x = q - kv <= m.param[i]; break;
        case FA_LEAF_PREFIX: x = kv < m.param[i]; break;
        case FA_LEAF_DOCUMENT: x = __ldg(doc_row + kv) == qdoc; break;
        default: x = false;
        }
        acc = is_or ? (acc || x) : (acc && x);
    }
    return acc;
}

// Tiles [t0, t1) of the split within the BlockMask row: partial blocks first,
// then full ones.  Counts and indices are clamped.
struct DecList {
    const int32_t* part;
    const int32_t* full;
    int np, n, t0, t1;
};

__device__ __forceinline__ DecList dec_list(const DecParams& p, int b, int split, bool& bad)
{
    DecList L;
    const int64_t r = p.bm_B == 1 ? 0 : b;  // query block 0 of the batch's row
    int a = __ldg(p.kv_num + r), f = p.has_full ? __ldg(p.full_num + r) : 0;
    if (a < 0 || a > p.nkv) { bad = true; a = a < 0 ? 0 : p.nkv; }
    if (f < 0 || f > p.nkv) { bad = true; f = f < 0 ? 0 : p.nkv; }
    L.part = p.kv_idx + r * p.nkv;
    L.full = p.has_full ? p.full_idx + r * p.nkv : nullptr;
    L.np = a;
    L.n = a + f;
    L.t0 = (int)((int64_t)L.n * split / p.splits);
    L.t1 = (int)((int64_t)L.n * (split + 1) / p.splits);
    return L;
}

__device__ __forceinline__ int dec_block(const DecParams& p, const DecList& L, int t, bool& bad)
{
    int kb = t < L.np ? __ldg(L.part + t) : __ldg(L.full + (t - L.np));
    if (kb < 0 || kb >= p.nkv) { bad = true; kb = kb < 0 ? 0 : p.nkv - 1; }
    return kb;
}

template <int D, int SCORE>
__global__ void __launch_bounds__(kDecThreads, DCfg<D>::MIN_CTAS) flex_decode_kernel(const __grid_constant__ DecParams p)
{
    using C = DCfg<D>;
    constexpr bool HAS_BIAS = SCORE == FA_SCORE_BIAS || SCORE == FA_SCORE_BIAS_SOFTCAP;
    constexpr int KD = D / 16;  // k16 steps of Q.K
    constexpr int ND = D / 8;   // n8 tiles of O
    extern __shared__ uint8_t smem_raw[];
    __shared__ DShared sh;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    bool bad = false;
    Watchdog wd{p.watchdog_ns, false};

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NS; ++i) {
            mbar_init(&sh.full[i], 1);
            mbar_init(&sh.empty[i], kDecWarps);
        }
        mbar_init(&sh.consumed, kDecWarps);
        mbar_init(&sh.written, kDecWarps);
        mbar_fence_init();
    }
    __syncthreads();
    const DecList L = dec_list(p, b, split, bad);

    if (warp == kDecProdWarp) {
        // TMA producer: K and V of every block of the split
        uint32_t issued = 0;
        bool ok = true;
        for (int t = L.t0; t < L.t1 && ok; ++t, ++issued) {
            const uint32_t slot = issued % C::NS, use = issued / C::NS;
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.empty[slot], (use & 1) ^ 1, wd));
            if (!ok) break;
            const int kb = dec_block(p, L, t, bad);
            if (elect_one_sync()) {
                uint8_t* dst = smem + slot * C::STAGE;
                mbar_arrive_expect_tx(&sh.full[slot], C::STAGE);
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    tma_load_4d(dst + c * kBox, &p.tm_k, &sh.full[slot], c * 64, kb * 128, hk, b);
                    tma_load_4d(dst + C::TILE + c * kBox, &p.tm_v, &sh.full[slot], c * 64, kb * 128, hk, b);
                }
            }
            __syncwarp();
        }
        // copies in flight land before the CTA exits (bounded)
        Watchdog dw{wd.failed ? 1000000ull : wd.limit_ns, false};
        for (uint32_t j = 0; j < (uint32_t)C::NS && j < issued; ++j) {
            const uint32_t last = issued - 1 - j;
            dw.failed = false;
            mbar_wait(&sh.full[last % C::NS], (last / C::NS) & 1, dw);
        }
        if (lane == 0 && (wd.failed || !ok)) atomicOr(p.status, STATUS_TIMEOUT);
        if (bad && lane == 0) atomicOr(p.status, STATUS_BAD_BLOCKMASK);
        return;
    }

    // ---- compute warps: rows g and g + 8 of the packed (head, token) rows
    const int g = lane >> 2, tq = lane & 3;
    int rr[2] = {g, g + 8};
    bool rvalid[2];
    int hq_r[2];
    int64_t qpos[2], qrow[2];
    float slope[2] = {0.f, 0.f};
    int32_t qdoc[2] = {0, 0};
    const int32_t* doc_row = p.mask.has_doc ? p.mask.doc_ids + (int64_t)b * p.mask.doc_stride : nullptr;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        rvalid[h] = rr[h] < p.rows;
        const int rv = rvalid[h] ? rr[h] : 0;
        hq_r[h] = hk * p.G + rv / p.q_len;
        qrow[h] = rv % p.q_len;
        qpos[h] = qrow[h] + p.mask.q_offset;
        if (SCORE == FA_SCORE_ALIBI) slope[h] = __ldg(p.slopes + hq_r[h]) * kLog2e;
        if (doc_row) qdoc[h] = __ldg(doc_row + qpos[h]);
    }
    // Q fragments (A operand of S = Q K^T): rows g / g + 8, columns 16 kk + 2 tq (+1, +8, +9)
    uint32_t qa[KD][4];
#pragma unroll
    for (int kk = 0; kk < KD; ++kk)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int h = e & 1, col = 16 * kk + 2 * tq + 8 * (e >> 1);
            const uint16_t* src = p.q + (int64_t)b * p.q_st0 + (int64_t)hq_r[h] * p.q_st1 + qrow[h] * p.q_st2 + col;
            qa[kk][e] = rvalid[h] ? *reinterpret_cast<const uint32_t*>(src) : 0u;
        }
    float oacc[ND][4];
#pragma unroll
    for (int n = 0; n < ND; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[n][e] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};  // log2 units; per-thread partial sums
    const float F = SCORE == FA_SCORE_SOFTCAP || SCORE == FA_SCORE_BIAS_SOFTCAP ? p.softcap * kLog2e : p.scale * kLog2e;

    uint32_t used = 0;
    bool ok = true;
    // kv block of the next tile, read one tile ahead (off the per-tile chain)
    int kb_next = L.t0 < L.t1 ? dec_block(p, L, L.t0, bad) : 0;
    for (int t = L.t0; t < L.t1; ++t, ++used) {
        const int kb = kb_next;
        if (t + 1 < L.t1) kb_next = dec_block(p, L, t + 1, bad);
        const uint32_t slot = used % C::NS, use = used / C::NS;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.full[slot], use & 1, wd));
        if (!ok) break;
        const bool partial = t < L.np;
        const uint32_t kbase = smem_u32(smem + slot * C::STAGE), vbase = kbase + C::TILE;
        const int key0 = 16 * warp;  // this warp's keys within the block

        // S = Q K^T for the warp's 16 keys (two n8 tiles)
        float sacc[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[j][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KD; ++kk) {
            const int m = lane >> 3;
            uint32_t r[4];
            ldsm_x4(swz(kbase, key0 + 8 * (m >> 1) + (lane & 7), 2 * kk + (m & 1)), r);
            mma_bf16_16816(sacc[0], qa[kk], r[0], r[1]);
            mma_bf16_16816(sacc[1], qa[kk], r[2], r[3]);
        }

        // score_mod, mask, in log2 units; row maxima
        float mt[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int h = e >> 1;
                const int64_t kv = (int64_t)kb * 128 + key0 + 8 * j + 2 * tq + (e & 1);
                bool adm = rvalid[h] && kv < p.kv_len;
                if (adm && partial) adm = mask_elem(p.mask, qdoc[h], doc_row, qpos[h], kv);
                float x = -INFINITY;
                if (adm) {
                    const float s = sacc[j][e];
                    float bias = 0.f;
                    if (HAS_BIAS)
                        bias = __uint_as_float((uint32_t)__ldg(p.bias + (int64_t)b * p.bias_st0 +
                                                               (int64_t)hq_r[h] * p.bias_st1 + qrow[h] * p.bias_st2 +
                                                               kv)
                                               << 16);
                    if constexpr (SCORE == FA_SCORE_SOFTCAP) x = tanh_accurate(s * p.softcap_in) * F;
                    else if constexpr (SCORE == FA_SCORE_BIAS_SOFTCAP)
                        x = tanh_accurate(fmaf(s, p.softcap_in, bias * p.softcap_inv)) * F;
                    else if constexpr (SCORE == FA_SCORE_BIAS) x = fmaf(bias, kLog2e, s * F);
                    else if constexpr (SCORE == FA_SCORE_ALIBI) x = fmaf(slope[h], (float)(kv - qpos[h]), s * F);
                    else x = s * F;
                }
                sacc[j][e] = x;
                mt[h] = fmaxf(mt[h], x);
            }
        // the four threads of a quad share rows g and g + 8
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            mt[h] = fmaxf(mt[h], __shfl_xor_sync(0xFFFFFFFFu, mt[h], 1));
            mt[h] = fmaxf(mt[h], __shfl_xor_sync(0xFFFFFFFFu, mt[h], 2));
        }
        float alpha[2], m_use[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float m_new = fmaxf(m_run[h], mt[h]);
            m_use[h] = m_new == -INFINITY ? 0.f : m_new;
            alpha[h] = ex2_approx(m_run[h] - m_use[h]);  // 0 while nothing was admitted
            m_run[h] = m_new;
            l_run[h] *= alpha[h];
        }
        // P = 2^(x - m), as the bf16 A fragment of O += P V (one k16 step of 16 keys)
        uint32_t pa[4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float pv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                pv[e] = ex2_approx(sacc[j][e] - m_use[e >> 1]);
                l_run[e >> 1] += pv[e];
            }
            pa[2 * j] = pack_bf16x2(pv[0], pv[1]);
            pa[2 * j + 1] = pack_bf16x2(pv[2], pv[3]);
        }
#pragma unroll
        for (int n = 0; n < ND; ++n) {
            oacc[n][0] *= alpha[0];
            oacc[n][1] *= alpha[0];
            oacc[n][2] *= alpha[1];
            oacc[n][3] *= alpha[1];
        }
        // O += P V: V fragments by transposed 8x8 loads (keys x 8 columns of D)
#pragma unroll
        for (int n = 0; n < ND; n += 2) {
            const int m = lane >> 3;
            uint32_t r[4];
            ldsm_x4_trans(swz(vbase, key0 + 8 * (m & 1) + (lane & 7), n + (m >> 1)), r);
            mma_bf16_16816(oacc[n], pa, r[0], r[1]);
            mma_bf16_16816(oacc[n + 1], pa, r[2], r[3]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[slot]);
    }
    if (bad && lane == 0) atomicOr(p.status, STATUS_BAD_BLOCKMASK);
    if (!ok || wd.failed) {
        // copies may still be in flight into the ring: leave without the merge
        if (lane == 0) atomicOr(p.status, STATUS_TIMEOUT);
        return;
    }

    // row sums over the quad
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l_run[h] += __shfl_xor_sync(0xFFFFFFFFu, l_run[h], 1);
        l_run[h] += __shfl_xor_sync(0xFFFFFFFFu, l_run[h], 2);
    }
    // Merge of the four warps through shared memory (the ring is free: every
    // block was consumed and the producer's copies have landed).
    float* mo = reinterpret_cast<float*>(smem);                   // [warps][16][D]
    float* mml = mo + kDecWarps * kDecodeMaxRows * D;             // [warps][16][2]
    // wait until every warp consumed its last block before overwriting the ring
    // (the ring holds the last blocks other warps may still read); bounded
    if (lane == 0) mbar_arrive(&sh.consumed);
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.consumed, 0, wd))) {
        if (lane == 0) atomicOr(p.status, STATUS_TIMEOUT);
        return;
    }
#pragma unroll
    for (int n = 0; n < ND; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int row = e < 2 ? g : g + 8;
            mo[(warp * kDecodeMaxRows + row) * D + 8 * n + 2 * tq + (e & 1)] = oacc[n][e];
        }
    if (tq == 0) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            mml[(warp * kDecodeMaxRows + rr[h]) * 2] = m_run[h];
            mml[(warp * kDecodeMaxRows + rr[h]) * 2 + 1] = l_run[h];
        }
    }
    // every partial result is in shared memory before the merge reads it (bounded)
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.written);
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.written, 0, wd))) {
        if (lane == 0) atomicOr(p.status, STATUS_TIMEOUT);
        return;
    }
    // thread -> (row, 8 columns)
    for (int idx = threadIdx.x; idx < p.rows * (D / 8); idx += 32 * kDecWarps) {
        const int row = idx / (D / 8), c8 = (idx % (D / 8)) * 8;
        float M = -INFINITY;
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, mml[(w * kDecodeMaxRows + row) * 2]);
        const float Mu = M == -INFINITY ? 0.f : M;
        float Ls = 0.f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int w = 0; w < kDecWarps; ++w) {
            const float sc = ex2_approx(mml[(w * kDecodeMaxRows + row) * 2] - Mu);
            Ls += mml[(w * kDecodeMaxRows + row) * 2 + 1] * sc;
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] += mo[(w * kDecodeMaxRows + row) * D + c8 + j] * sc;
        }
        const int hq = hk * p.G + row / p.q_len;
        const int64_t qr = row % p.q_len;
        const int64_t orow = ((int64_t)b * p.Hq + hq) * p.q_len + qr;
        if (p.splits == 1) {
            const float inv = (Ls > 0.f && M != -INFINITY) ? 1.0f / Ls : 0.f;
            uint4 v;
            v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
            v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
            v.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
            v.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
            *reinterpret_cast<uint4*>(p.o + (int64_t)b * p.o_st0 + (int64_t)hq * p.o_st1 + qr * p.o_st2 + c8) = v;
            if (c8 == 0 && p.lse)
                p.lse[orow] = (Ls > 0.f && M != -INFINITY) ? (M + __log2f(Ls)) * kLn2 : -INFINITY;
        } else {
            float* po = p.part_o + ((int64_t)split * p.B * p.Hq * p.q_len + orow) * D + c8;
            reinterpret_cast<float4*>(po)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            reinterpret_cast<float4*>(po)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
            if (c8 == 0) {
                float* pml = p.part_ml + ((int64_t)split * p.B * p.Hq * p.q_len + orow) * 2;
                pml[0] = M;
                pml[1] = Ls;
            }
        }
    }
}

// Merge of the splits: one warp per output row (b, hq, q); lane j owns columns
// [D/32 * j, D/32 * (j + 1)).
template <int D>
__global__ void __launch_bounds__(256) decode_merge_kernel(const __grid_constant__ DecParams p)
{
    const int64_t rows = (int64_t)p.B * p.Hq * p.q_len;
    const int64_t r = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (r >= rows) return;
    constexpr int PER = D / 32;
    float M = -INFINITY;
    for (int s = 0; s < p.splits; ++s) M = fmaxf(M, p.part_ml[((int64_t)s * rows + r) * 2]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float Ls = 0.f, acc[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) acc[j] = 0.f;
    for (int s = 0; s < p.splits; ++s) {
        const float* ml = p.part_ml + ((int64_t)s * rows + r) * 2;
        const float sc = ex2_approx(ml[0] - Mu);
        Ls += ml[1] * sc;
        const float* po = p.part_o + ((int64_t)s * rows + r) * D + PER * lane;
#pragma unroll
        for (int j = 0; j < PER; ++j) acc[j] += po[j] * sc;
    }
    const float inv = (Ls > 0.f && M != -INFINITY) ? 1.0f / Ls : 0.f;
    const int64_t q = r % p.q_len, bh = r / p.q_len;
    const int64_t hq = bh % p.Hq, b = bh / p.Hq;
    uint16_t* o = p.o + b * p.o_st0 + hq * p.o_st1 + q * p.o_st2 + PER * lane;
#pragma unroll
    for (int j = 0; j < PER; j += 2) reinterpret_cast<uint32_t*>(o)[j / 2] = pack_bf16x2(acc[j] * inv, acc[j + 1] * inv);
    if (lane == 0 && p.lse) p.lse[r] = (Ls > 0.f && M != -INFINITY) ? (M + __log2f(Ls)) * kLn2 : -INFINITY;
}

template <int D, int SCORE>
cudaError_t launch_dec_variant(const DecParams& p, cudaStream_t stream)
{
    static std::mutex mu;
    static std::vector<CtxKey> done;
    auto kern = flex_decode_kernel<D, SCORE>;
    {
        CtxKey key;
        std::lock_guard<std::mutex> lock(mu);
        bool have = false;
        if (current_ctx(&key))
            for (const CtxKey& k : done) have |= k == key;
        if (!have) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DCfg<D>::SMEM);
            if (e != cudaSuccess) return e;
            if (current_ctx(&key)) done.push_back(key);
        }
    }
    dim3 grid((unsigned)p.splits, (unsigned)p.Hkv, (unsigned)p.B);
    kern<<<grid, kDecThreads, DCfg<D>::SMEM, stream>>>(p);
    return cudaGetLastError();
}

} // namespace

int decode_splits(int64_t B, int64_t Hkv, int32_t nkv, int sms)
{
    // about four CTAs per SM over the whole grid, at most one kv block per split
    const int64_t units = B * Hkv;
    int64_t s = units > 0 ? (4 * (int64_t)sms + units - 1) / units : 1;
    if (s > nkv) s = nkv;
    if (s > 64) s = 64;
    return s < 1 ? 1 : (int)s;
}

cudaError_t launch_flex_decode(const DecParams& p, int D, cudaStream_t stream)
{
#define FA_DEC_CASE(DD, SS) \
    if (D == DD && p.score_kind == SS) return launch_dec_variant<DD, SS>(p, stream);
    FA_DEC_CASE(64, FA_SCORE_NONE) FA_DEC_CASE(64, FA_SCORE_ALIBI) FA_DEC_CASE(64, FA_SCORE_SOFTCAP)
    FA_DEC_CASE(64, FA_SCORE_BIAS) FA_DEC_CASE(64, FA_SCORE_BIAS_SOFTCAP)
    FA_DEC_CASE(128, FA_SCORE_NONE) FA_DEC_CASE(128, FA_SCORE_ALIBI) FA_DEC_CASE(128, FA_SCORE_SOFTCAP)
    FA_DEC_CASE(128, FA_SCORE_BIAS) FA_DEC_CASE(128, FA_SCORE_BIAS_SOFTCAP)
#undef FA_DEC_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode_merge(const DecParams& p, int D, cudaStream_t stream)
{
    const int64_t rows = (int64_t)p.B * p.Hq * p.q_len;
    if (rows == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((rows + 7) / 8);
    if (D == 64) decode_merge_kernel<64><<<blocks, 256, 0, stream>>>(p);
    else decode_merge_kernel<128><<<blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

} // namespace fa
