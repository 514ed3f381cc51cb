// FlexDecoding for sm_100a: the forward pass for a few query tokens against a
// long KV cache ("Flex Attention" paper review sec. 3.1, the decoding template;
// rocketrecap talk: decoding splits the work along the KV dimension and reduces
// the partial results at the end).
//
// With one to a few query tokens per sequence the contraction is tiny and the
// pass is bound by reading K and V from HBM, so this kernel does not use the
// 128-row tcgen05 tiles of the prefill kernel: the G query heads that share a
// kv head (GQA) and their q_len tokens (at most 16 rows) are packed as the n = 8
// side of warp-level m16n8k16 MMAs, the keys (and D) as the m = 16 side.
//
// Work split: the kv blocks of all (batch, kv head) segments form one list —
// segments in (batch, kv head) order, each its batch's BlockMask row, partial
// blocks first — and the grid is one CTA per SM, CTA c streaming the list's
// c-th equal share (whole segments or pieces of them).  Every SM therefore
// reads the same number of bytes, with no wave tail and one ring ramp per SM.
// Each CTA finds where its share starts by a scan of the rows' block counts.
// It streams its blocks through a TMA ring; each of its eight compute warps
// takes 16 keys of every block with its own online softmax (running max, sum,
// O), and at the end of every piece of a segment writes that state as a
// partial result.  A second kernel merges the partials of each segment.
#include <mutex>
#include <vector>

#include <cuda_runtime.h>

#include "context.cuh"
#include "decode_walk.cuh"
#include "flex_decode.cuh"
#include "flex_fwd.cuh"
#include "ptx.cuh"
#include "score_math.cuh"

namespace fa {

namespace {

constexpr int kDecWarps = kDecodeWarps;          // compute warps, 16 keys of each block each
constexpr int kDecThreads = 32 * (kDecWarps + 1);  // plus the TMA producer warp
constexpr int kDecProdWarp = kDecWarps;
constexpr int kBox = 16384;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
struct DCfg {
    static constexpr int TILE = 128 * D * 2;           // one K or V block
    // ring stages: 128 KB of copies in flight per SM (one CTA per SM).  With 192 KB
    // the SMs streamed at more unequal rates and the slowest share ended later
    // (D = 128: 199.9 -> 181.2 us, D = 64: 119.7 -> 113.7 us on a 32k cache)
    static constexpr int NS = D == 128 ? 2 : 4;
    static constexpr int STAGE = 2 * TILE;             // K then V
    static constexpr int SMEM = NS * STAGE + 1024;
    static constexpr int MIN_CTAS = 1;
    static_assert(NS <= 6, "ring barriers");
};

struct __align__(16) DShared {
    uint64_t full[6], empty[6];
    long long scan[kDecThreads / 32];  // per-warp sums of the block-count scan
    long long count;                   // blocks of this CTA's share
    int start_b, start_hk, start_t;    // where the share starts
};

// Transpose of an 8x8 b16 matrix held as a warp fragment (thread l: row l / 4,
// columns 2 (l % 4), 2 (l % 4) + 1, one 32-bit register).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

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

// Every thread of the CTA: the list's length T from a scan of the rows' block
// counts, this CTA's share [floor(c T / G), floor((c + 1) T / G)) and the
// position where it starts, left in shared memory.
__device__ __forceinline__ void dec_locate(const DecParams& p, DShared& sh, bool& bad)
{
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int nrow = p.bm_B == 1 ? 1 : p.B;
    const int per = (nrow + kDecThreads - 1) / kDecThreads;
    const int lo = min(nrow, tid * per), hi = min(nrow, lo + per);
    long long mine = 0;
    for (int r = lo; r < hi; ++r) {
        int np, n;
        dec_counts(p, r, np, n, bad);
        mine += n;
    }
    long long inc = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xFFFFFFFFu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) sh.scan[warp] = inc;
    if (tid == 0) sh.count = 0;
    __syncthreads();
    long long before = 0, total = 0;
    for (int w = 0; w < kDecThreads / 32; ++w) {
        before += w < warp ? sh.scan[w] : 0;
        total += sh.scan[w];
    }
    const long long excl = before + inc - mine;  // blocks of the rows before this thread's
    const long long T = (long long)p.Hkv * (p.bm_B == 1 ? total * p.B : total);
    const long long x0 = share_start(T, blockIdx.x, gridDim.x), x1 = share_start(T, blockIdx.x + 1, gridDim.x);
    if (tid == 0 && blockIdx.x == 0) *p.total = T;  // for the merge
    if (x0 < x1) {
        DecWalk w0{};
        bool found = false;
        if (p.bm_B == 1) {
            if (tid == 0) {
                w0 = dec_find_shared(p, x0, total, bad);  // every segment has `total` blocks
                found = true;
            }
        } else if ((long long)p.Hkv * excl <= x0 && x0 < (long long)p.Hkv * (excl + mine)) {
            found = dec_find(p, x0, lo, hi, excl, w0, bad);  // this thread's rows hold x0
        }
        if (found) {
            sh.start_b = w0.b;
            sh.start_hk = w0.hk;
            sh.start_t = w0.t;
            sh.count = x1 - x0;
        }
    }
    __syncthreads();
}

template <int D, int SCORE, int NR>
__global__ void __launch_bounds__(kDecThreads, DCfg<D>::MIN_CTAS) flex_decode_kernel(const __grid_constant__ DecParams p)
{
    using C = DCfg<D>;
    constexpr bool HAS_BIAS = SCORE == FA_SCORE_BIAS || SCORE == FA_SCORE_BIAS_SOFTCAP;
    constexpr int KD = D / 16;  // k16 steps of Q.K
    extern __shared__ uint8_t smem_raw[];
    __shared__ DShared sh;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    bool bad = false;
    Watchdog wd{p.watchdog_ns, false};

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NS; ++i) {
            mbar_init(&sh.full[i], 1);
            mbar_init(&sh.empty[i], kDecWarps);
        }
        mbar_fence_init();
    }
    dec_locate(p, sh, bad);  // ends with a CTA barrier
    // the merge grid may be scheduled now; it waits for this grid's completion
    if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const long long count = sh.count;
    DecWalk w0{sh.start_b, sh.start_hk, sh.start_t, 0, 0};
    if (count > 0) dec_counts(p, dec_row(p, w0.b), w0.np, w0.n, bad);

    if (warp == kDecProdWarp) {
        // TMA producer: K and V of every block of the share
        uint32_t issued = 0;
        bool ok = true;
        DecWalk w = w0;
        for (long long i = 0; i < count && ok; ++i, ++issued) {
            const uint32_t slot = issued % C::NS, use = issued / C::NS;
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.empty[slot], (use & 1) ^ 1, wd));
            if (!ok) break;
            const int kb = dec_block(p, w, bad);
            if (elect_one_sync()) {
                uint8_t* dst = smem + slot * C::STAGE;
                mbar_arrive_expect_tx(&sh.full[slot], C::STAGE);
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    tma_load_4d(dst + c * kBox, &p.tm_k, &sh.full[slot], c * 64, kb * 128, w.hk, w.b);
                    tma_load_4d(dst + C::TILE + c * kBox, &p.tm_v, &sh.full[slot], c * 64, kb * 128, w.hk, w.b);
                }
            }
            __syncwarp();
            if (i + 1 < count) dec_advance(p, w, bad);
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

    // ---- compute warps.  Transposed products, so that the few query rows are the
    // n = 8 side of the m16n8k16 MMAs (NR tiles of 8 rows): S^T = K Q^T for the
    // warp's 16 keys, then O^T += V^T P^T.  Thread (g, tq) = (lane / 4, lane % 4)
    // holds S^T at keys g, g + 8 and query rows 2 tq, 2 tq + 1 (+ 8 per row tile).
    const int g = lane >> 2, tq = lane & 3;
    int rr[NR][2];
    bool rvalid[NR][2];
#pragma unroll
    for (int nt = 0; nt < NR; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            rr[nt][j] = 8 * nt + 2 * tq + j;
            rvalid[nt][j] = rr[nt][j] < p.rows;
        }
    // per-segment state: query heads, positions, ALiBi slopes, document ids, Q^T fragments
    int hq_r[NR][2], qrow[NR][2];  // query head and token of each of the thread's rows
    float slope[NR][2];
    int32_t qdoc[NR][2];
    const int32_t* doc_row = nullptr;
    uint32_t qb[NR][KD][2];  // B operand of S^T: Q[row 8 nt + g][16 kk + 2 tq (+1)], [.. + 8 (+9)]
    auto load_segment = [&](int b, int hk) {
        doc_row = p.mask.has_doc ? p.mask.doc_ids + (int64_t)b * p.mask.doc_stride : nullptr;
#pragma unroll
        for (int nt = 0; nt < NR; ++nt) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int rv = rvalid[nt][j] ? rr[nt][j] : 0;
                hq_r[nt][j] = hk * p.G + rv / p.q_len;
                qrow[nt][j] = rv % p.q_len;
                slope[nt][j] = SCORE == FA_SCORE_ALIBI ? __ldg(p.slopes + hq_r[nt][j]) * kLog2e : 0.f;
                qdoc[nt][j] = doc_row ? __ldg(doc_row + qrow[nt][j] + p.mask.q_offset) : 0;
            }
            // the B fragment's column is query row 8 nt + g (not this thread's S^T rows)
            const int rb = 8 * nt + g;
            const bool vb = rb < p.rows;
            const int rvb = vb ? rb : 0;
            const uint16_t* qsrc = p.q + (int64_t)b * p.q_st0 + (int64_t)(hk * p.G + rvb / p.q_len) * p.q_st1 +
                                   (int64_t)(rvb % p.q_len) * p.q_st2 + 2 * tq;
#pragma unroll
            for (int kk = 0; kk < KD; ++kk) {
                qb[nt][kk][0] = vb ? *reinterpret_cast<const uint32_t*>(qsrc + 16 * kk) : 0u;
                qb[nt][kk][1] = vb ? *reinterpret_cast<const uint32_t*>(qsrc + 16 * kk + 8) : 0u;
            }
        }
    };
    float oacc[D / 16][NR][4];  // O^T: d = 16 mt + g (+8), query rows 8 nt + 2 tq (+1)
    float m_run[NR][2], l_run[NR][2];  // log2 units; l: this thread's keys only
    auto reset = [&]() {
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
            for (int nt = 0; nt < NR; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) oacc[mt][nt][e] = 0.f;
#pragma unroll
        for (int nt = 0; nt < NR; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                m_run[nt][j] = -INFINITY;
                l_run[nt][j] = 0.f;
            }
    };
    // the warp's state for its piece of segment (b, hk) as partial result number
    // (segment + CTA); the first and last CTAs of a segment are recorded for the merge
    auto write_partial = [&](const DecWalk& w) {
        const int64_t seg = (int64_t)w.b * p.Hkv + w.hk;
        const int64_t base = ((seg + blockIdx.x) * kDecWarps + warp) * p.rows;
#pragma unroll
        for (int nt = 0; nt < NR; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float l = l_run[nt][j];  // sum over the eight key groups g
                l += __shfl_xor_sync(0xFFFFFFFFu, l, 4);
                l += __shfl_xor_sync(0xFFFFFFFFu, l, 8);
                l += __shfl_xor_sync(0xFFFFFFFFu, l, 16);
                if (!rvalid[nt][j]) continue;
                float* po = p.part_o + (base + rr[nt][j]) * D + g;
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    po[16 * mt] = oacc[mt][nt][j];
                    po[16 * mt + 8] = oacc[mt][nt][2 + j];
                }
                if (g == 0) *reinterpret_cast<float2*>(p.part_ml + (base + rr[nt][j]) * 2) = make_float2(m_run[nt][j], l);
            }
        if (warp == 0 && lane == 0 && w.t + 1 == w.n) p.seg_last[seg] = (int)blockIdx.x;
    };
    const float F = SCORE == FA_SCORE_SOFTCAP || SCORE == FA_SCORE_BIAS_SOFTCAP ? p.softcap * kLog2e : p.scale * kLog2e;

    DecWalk w = w0;
    if (count > 0) load_segment(w.b, w.hk);
    reset();
    uint32_t used = 0;
    bool ok = true;
    // kv block of the next tile, read one tile ahead (off the per-tile chain)
    int kb_next = count > 0 ? dec_block(p, w, bad) : 0;
    for (long long i = 0; i < count; ++i, ++used) {
        const int kb = kb_next;
        DecWalk wn = w;
        if (i + 1 < count) {
            dec_advance(p, wn, bad);
            kb_next = dec_block(p, wn, bad);
        }
        if (w.t == 0 && warp == 0 && lane == 0) p.seg_first[(int64_t)w.b * p.Hkv + w.hk] = (int)blockIdx.x;
        const uint32_t slot = used % C::NS, use = used / C::NS;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.full[slot], use & 1, wd));
        if (!ok) break;
        const bool partial = w.t < w.np;
        const uint32_t kbase = smem_u32(smem + slot * C::STAGE), vbase = kbase + C::TILE;
        const int key0 = 16 * warp;  // this warp's keys within the block
        const int m4 = lane >> 3;    // the 8x8 matrix whose row address this lane gives

        // Where the registers allow (not at D = 128 with two row tiles) the warp's K and
        // V^T fragments are all read first and the stage is released before any
        // arithmetic, so the ring refills while the products run.
        constexpr bool kEarly = !(D == 128 && NR == 2);
        uint32_t ka[kEarly ? KD : 1][4], va[kEarly ? D / 16 : 1][4];
        if constexpr (kEarly) {
#pragma unroll
            for (int kk = 0; kk < KD; ++kk)
                ldsm_x4(swz(kbase, key0 + 8 * (m4 & 1) + (lane & 7), 2 * kk + (m4 >> 1)), ka[kk]);
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt)
                ldsm_x4_trans(swz(vbase, key0 + 8 * (m4 >> 1) + (lane & 7), 2 * mt + (m4 & 1)), va[mt]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.empty[slot]);
        }
        // S^T = K Q^T: A = K (keys x d, ldmatrix), B = Q^T (registers)
        float sacc[NR][4];
#pragma unroll
        for (int nt = 0; nt < NR; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KD; ++kk) {
            if constexpr (!kEarly) ldsm_x4(swz(kbase, key0 + 8 * (m4 & 1) + (lane & 7), 2 * kk + (m4 >> 1)), ka[0]);
#pragma unroll
            for (int nt = 0; nt < NR; ++nt) mma_bf16_16816(sacc[nt], ka[kEarly ? kk : 0], qb[nt][kk][0], qb[nt][kk][1]);
        }

        // score_mod, mask, in log2 units; maxima over the 16 keys per query row
        float mt_[NR][2];
#pragma unroll
        for (int nt = 0; nt < NR; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) mt_[nt][j] = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < NR; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = e & 1;
                const int64_t kv = (int64_t)kb * 128 + key0 + g + 8 * (e >> 1);
                bool adm = rvalid[nt][j] && kv < p.kv_len;
                const int64_t qpos = qrow[nt][j] + p.mask.q_offset;
                if (adm && partial) adm = mask_elem(p.mask, qdoc[nt][j], doc_row, qpos, kv);
                float x = -INFINITY;
                if (adm) {
                    const float s = sacc[nt][e];
                    float bias = 0.f;
                    if (HAS_BIAS)
                        bias = __uint_as_float((uint32_t)__ldg(p.bias + (int64_t)w.b * p.bias_st0 +
                                                               (int64_t)hq_r[nt][j] * p.bias_st1 +
                                                               (int64_t)qrow[nt][j] * p.bias_st2 + kv)
                                               << 16);
                    if constexpr (SCORE == FA_SCORE_SOFTCAP) x = tanh_accurate(s * p.softcap_in) * F;
                    else if constexpr (SCORE == FA_SCORE_BIAS_SOFTCAP)
                        x = tanh_accurate(fmaf(s, p.softcap_in, bias * p.softcap_inv)) * F;
                    else if constexpr (SCORE == FA_SCORE_BIAS) x = fmaf(bias, kLog2e, s * F);
                    else if constexpr (SCORE == FA_SCORE_ALIBI) x = fmaf(slope[nt][j], (float)(kv - qpos), s * F);
                    else x = s * F;
                }
                sacc[nt][e] = x;
                mt_[nt][j] = fmaxf(mt_[nt][j], x);
            }
        // the eight key groups g (lanes tq, tq + 4, ..) share query rows 2 tq, 2 tq + 1
        float alpha[NR][2], m_use[NR][2];
#pragma unroll
        for (int nt = 0; nt < NR; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float m = mt_[nt][j];
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 8));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 16));
                const float m_new = fmaxf(m_run[nt][j], m);
                m_use[nt][j] = m_new == -INFINITY ? 0.f : m_new;
                alpha[nt][j] = ex2_approx(m_run[nt][j] - m_use[nt][j]);  // 0 while nothing was admitted
                m_run[nt][j] = m_new;
                l_run[nt][j] *= alpha[nt][j];
            }
        // P^T = 2^(x - m) in bf16; the B fragment of O^T += V^T P^T (keys 2 tq (+1), 2 tq + 8 (+9)
        // at query row g) is the transpose of the 8x8 blocks this thread holds
        uint32_t pb[NR][2];
#pragma unroll
        for (int nt = 0; nt < NR; ++nt) {
            float pv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                pv[e] = ex2_approx(sacc[nt][e] - m_use[nt][e & 1]);
                l_run[nt][e & 1] += pv[e];
            }
            pb[nt][0] = movmatrix_trans(pack_bf16x2(pv[0], pv[1]));  // keys 0-7
            pb[nt][1] = movmatrix_trans(pack_bf16x2(pv[2], pv[3]));  // keys 8-15
        }
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
            for (int nt = 0; nt < NR; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) oacc[mt][nt][e] *= alpha[nt][e & 1];
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            if constexpr (!kEarly)
                ldsm_x4_trans(swz(vbase, key0 + 8 * (m4 >> 1) + (lane & 7), 2 * mt + (m4 & 1)), va[0]);
#pragma unroll
            for (int nt = 0; nt < NR; ++nt) mma_bf16_16816(oacc[mt][nt], va[kEarly ? mt : 0], pb[nt][0], pb[nt][1]);
        }
        if constexpr (!kEarly) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.empty[slot]);
        }
        // the piece ends with the segment or with the share
        if (i + 1 == count || wn.b != w.b || wn.hk != w.hk) {
            write_partial(w);
            if (i + 1 < count) {
                load_segment(wn.b, wn.hk);
                reset();
            }
        }
        w = wn;
    }
    if (bad && lane == 0) atomicOr(p.status, STATUS_BAD_BLOCKMASK);
    if ((!ok || wd.failed) && lane == 0) atomicOr(p.status, STATUS_TIMEOUT);
}

// Merge of the partial results: one warp per output row (b, hq, q).  The
// segment's partials are those of CTAs seg_first..seg_last whose share is not
// empty (with fewer blocks than CTAs some shares are), eight (one per compute
// warp) each.  They are taken 32 at a time: lane k reads partial k's running
// max and sum, the warp forms the common maximum and the weights, then every
// lane accumulates its D/32 columns of the 32 partials (loads issued together).
// Launched as a programmatic dependent of the decode kernel: it waits for that
// grid's completion before reading anything.
template <int D>
__global__ void __launch_bounds__(256) decode_merge_kernel(const __grid_constant__ DecParams p)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t rows = (int64_t)p.B * p.Hq * p.q_len;
    const int64_t r = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (r >= rows) return;
    constexpr int PER = D / 32;
    static_assert(PER == 2 || PER == 4, "D is 64 or 128");
    const int64_t q = r % p.q_len, bh = r / p.q_len;
    const int hq = (int)(bh % p.Hq), b = (int)(bh / p.Hq);
    const int hk = hq / p.G, row = (hq % p.G) * p.q_len + (int)q;
    const int64_t seg = (int64_t)b * p.Hkv + hk;
    bool bad = false;
    int np, n;
    dec_counts(p, dec_row(p, b), np, n, bad);
    const int first = p.seg_first[seg], last = p.seg_last[seg];
    const long long T = *p.total;
    int c_lo = 0, c_hi = -1;  // no kv block: O = 0, LSE = -inf
    if (n > 0) {
        c_lo = max(0, first);
        c_hi = min(p.grid - 1, last);
    }
    const int K = (c_hi - c_lo + 1) * kDecWarps;  // partials, some of empty shares
    float M = -INFINITY, Ls = 0.f, acc[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) acc[j] = 0.f;
    for (int k0 = 0; k0 < K; k0 += 32) {
        // lane k: partial k0 + k
        const int k = k0 + lane, c = c_lo + k / kDecWarps;
        float2 ml = make_float2(-INFINITY, 0.f);
        if (k < K && share_start(T, c, p.grid) < share_start(T, c + 1, p.grid))
            ml = *reinterpret_cast<const float2*>(p.part_ml + (((seg + c) * kDecWarps + k % kDecWarps) * p.rows + row) * 2);
        float Mn = fmaxf(M, ml.x);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) Mn = fmaxf(Mn, __shfl_xor_sync(0xFFFFFFFFu, Mn, o));
        const float Mu = Mn == -INFINITY ? 0.f : Mn;
        const float a = ex2_approx(M - Mu);  // 0 while nothing was merged
        const float sc = ex2_approx(ml.x - Mu);  // 0 for an empty partial
        float lsum = ml.y * sc;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xFFFFFFFFu, lsum, o);
        Ls = Ls * a + lsum;
#pragma unroll
        for (int j = 0; j < PER; ++j) acc[j] *= a;
        M = Mn;
        // columns: partials with a zero weight are skipped (empty shares, past K)
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) {
            const float w = __shfl_sync(0xFFFFFFFFu, sc, kk);
            if (w == 0.f) continue;
            const int kq = k0 + kk, cq = c_lo + kq / kDecWarps;
            const float* src = p.part_o + (((seg + cq) * kDecWarps + kq % kDecWarps) * p.rows + row) * D + PER * lane;
            if constexpr (PER == 4) {
                const float4 x = *reinterpret_cast<const float4*>(src);
                acc[0] += x.x * w; acc[1] += x.y * w; acc[2] += x.z * w; acc[3] += x.w * w;
            } else {
                const float2 x = *reinterpret_cast<const float2*>(src);
                acc[0] += x.x * w; acc[1] += x.y * w;
            }
        }
    }
    const float inv = (Ls > 0.f && M != -INFINITY) ? 1.0f / Ls : 0.f;
    uint16_t* o = p.o + (int64_t)b * p.o_st0 + (int64_t)hq * p.o_st1 + q * p.o_st2 + PER * lane;
#pragma unroll
    for (int j = 0; j < PER; j += 2) reinterpret_cast<uint32_t*>(o)[j / 2] = pack_bf16x2(acc[j] * inv, acc[j + 1] * inv);
    if (lane == 0 && p.lse) p.lse[r] = (Ls > 0.f && M != -INFINITY) ? (M + __log2f(Ls)) * kLn2 : -INFINITY;
}

template <int D, int SCORE, int NR>
cudaError_t launch_dec_variant(const DecParams& p, cudaStream_t stream)
{
    static std::mutex mu;
    static std::vector<CtxKey> done;
    auto kern = flex_decode_kernel<D, SCORE, NR>;
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
    kern<<<(unsigned)p.grid, kDecThreads, DCfg<D>::SMEM, stream>>>(p);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_flex_decode(const DecParams& p, int D, cudaStream_t stream)
{
    // one tile of eight query rows, or two for groups of 9 to 16 rows
#define FA_DEC_CASE(DD, SS)                                                                      \
    if (D == DD && p.score_kind == SS)                                                           \
        return p.rows > 8 ? launch_dec_variant<DD, SS, 2>(p, stream) : launch_dec_variant<DD, SS, 1>(p, stream);
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
    // a programmatic dependent launch: the merge grid is scheduled while the decode
    // grid drains and waits (griddepcontrol.wait) for its completion
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((rows + 7) / 8));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if (D == 64) return cudaLaunchKernelEx(&cfg, decode_merge_kernel<64>, p);
    return cudaLaunchKernelEx(&cfg, decode_merge_kernel<128>, p);
}

} // namespace fa
