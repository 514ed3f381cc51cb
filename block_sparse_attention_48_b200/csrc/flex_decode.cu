// FlexDecoding for sm_100a: the forward pass for a few query tokens against a
// long KV cache ("Flex Attention" paper review sec. 3.1, the decoding template;
// rocketrecap talk: decoding splits the work along the KV dimension and reduces
// the partial results at the end).
//
// With one to a few query tokens per sequence the contraction is tiny and the
// pass is bound by reading K and V from HBM, so this kernel does not use the
// 128-row tcgen05 tiles of the prefill kernel: the G query heads that share a
// kv head (GQA) and their q_len tokens are packed as the (at most 16) rows of
// warp-level m16n8k16 MMAs.
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
    // ring stages: 192 KB of copies in flight per SM at D = 128, 96 KB at D = 64
    static constexpr int NS = 3;
    static constexpr int STAGE = 2 * TILE;             // K then V
    static constexpr int SMEM = NS * STAGE + 1024;
    static constexpr int MIN_CTAS = 1;
};

struct __align__(16) DShared {
    uint64_t full[3], empty[3];
    long long scan[kDecThreads / 32];  // per-warp sums of the block-count scan
    long long count;                   // blocks of this CTA's share
    int start_b, start_hk, start_t;    // where the share starts
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

// Block counts of BlockMask row r (query block 0 of a batch): partial and
// partial + full, each clamped to [0, nkv] (a corrupt count sets `bad`).
__device__ __forceinline__ void dec_counts(const DecParams& p, int64_t r, int& np, int& n, bool& bad)
{
    int a = __ldg(p.kv_num + r), f = p.has_full ? __ldg(p.full_num + r) : 0;
    if (a < 0 || a > p.nkv) { bad = true; a = a < 0 ? 0 : p.nkv; }
    if (f < 0 || f > p.nkv) { bad = true; f = f < 0 ? 0 : p.nkv; }
    np = a;
    n = a + f;
}

// Position in the list of (batch, kv head, block): segment (b, hk), block t of
// the batch's row, which has np partial and n blocks in all.
struct DecWalk {
    int b, hk, t, np, n;
};

__device__ __forceinline__ int64_t dec_row(const DecParams& p, int b) { return p.bm_B == 1 ? 0 : b; }

__device__ __forceinline__ int dec_block(const DecParams& p, const DecWalk& w, bool& bad)
{
    const int64_t r = dec_row(p, w.b) * p.nkv;
    int kb = w.t < w.np ? __ldg(p.kv_idx + r + w.t) : __ldg(p.full_idx + r + (w.t - w.np));
    if (kb < 0 || kb >= p.nkv) { bad = true; kb = kb < 0 ? 0 : p.nkv - 1; }
    return kb;
}

// The next position (called only while the CTA's share has blocks left, so a
// non-empty segment follows; the batch index never passes B - 1).
__device__ __forceinline__ void dec_advance(const DecParams& p, DecWalk& w, bool& bad)
{
    if (++w.t < w.n) return;
    w.t = 0;
    if (++w.hk < p.Hkv) return;
    w.hk = 0;
    do {
        if (w.b + 1 >= p.B) { w.n = 0; return; }
        ++w.b;
        dec_counts(p, dec_row(p, w.b), w.np, w.n, bad);
    } while (w.n == 0);
}

// floor(c * T / G) without overflowing the product.
__device__ __forceinline__ long long share_start(long long T, int c, int G)
{
    return (T / G) * c + (T % G) * c / G;
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
        if (p.bm_B == 1) {
            if (tid == 0) {
                const long long seg = x0 / total;  // every segment has `total` blocks
                sh.start_b = (int)(seg / p.Hkv);
                sh.start_hk = (int)(seg % p.Hkv);
                sh.start_t = (int)(x0 % total);
                sh.count = x1 - x0;
            }
        } else if ((long long)p.Hkv * excl <= x0 && x0 < (long long)p.Hkv * (excl + mine)) {
            long long acc = excl;
            for (int r = lo; r < hi; ++r) {
                int np, n;
                dec_counts(p, r, np, n, bad);
                if (x0 < (long long)p.Hkv * (acc + n)) {
                    const long long off = x0 - (long long)p.Hkv * acc;
                    sh.start_b = r;
                    sh.start_hk = (int)(off / n);
                    sh.start_t = (int)(off % n);
                    sh.count = x1 - x0;
                    break;
                }
                acc += n;
            }
        }
    }
    __syncthreads();
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

    // ---- compute warps: rows g and g + 8 of the packed (head, token) rows
    const int g = lane >> 2, tq = lane & 3;
    const int rr[2] = {g, g + 8};
    bool rvalid[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) rvalid[h] = rr[h] < p.rows;
    // per-segment state: query heads, positions, ALiBi slopes, document ids, Q fragments
    int hq_r[2];
    int64_t qpos[2], qrow[2];
    float slope[2] = {0.f, 0.f};
    int32_t qdoc[2] = {0, 0};
    const int32_t* doc_row = nullptr;
    uint32_t qa[KD][4];  // A operand of S = Q K^T: rows g / g + 8, columns 16 kk + 2 tq (+1, +8, +9)
    auto load_segment = [&](int b, int hk) {
        doc_row = p.mask.has_doc ? p.mask.doc_ids + (int64_t)b * p.mask.doc_stride : nullptr;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int rv = rvalid[h] ? rr[h] : 0;
            hq_r[h] = hk * p.G + rv / p.q_len;
            qrow[h] = rv % p.q_len;
            qpos[h] = qrow[h] + p.mask.q_offset;
            if (SCORE == FA_SCORE_ALIBI) slope[h] = __ldg(p.slopes + hq_r[h]) * kLog2e;
            if (doc_row) qdoc[h] = __ldg(doc_row + qpos[h]);
        }
#pragma unroll
        for (int kk = 0; kk < KD; ++kk)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int h = e & 1, col = 16 * kk + 2 * tq + 8 * (e >> 1);
                const uint16_t* src = p.q + (int64_t)b * p.q_st0 + (int64_t)hq_r[h] * p.q_st1 + qrow[h] * p.q_st2 + col;
                qa[kk][e] = rvalid[h] ? *reinterpret_cast<const uint32_t*>(src) : 0u;
            }
    };
    float oacc[ND][4];
    float m_run[2], l_run[2];  // log2 units; per-thread partial sums
    auto reset = [&]() {
#pragma unroll
        for (int n = 0; n < ND; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) oacc[n][e] = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            m_run[h] = -INFINITY;
            l_run[h] = 0.f;
        }
    };
    // the warp's state for its piece of segment (b, hk) as partial result number
    // (segment + CTA); the first and last CTAs of a segment are recorded for the merge
    auto write_partial = [&](const DecWalk& w) {
        float l[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            l[h] = l_run[h] + __shfl_xor_sync(0xFFFFFFFFu, l_run[h], 1);
            l[h] += __shfl_xor_sync(0xFFFFFFFFu, l[h], 2);
        }
        const int64_t seg = (int64_t)w.b * p.Hkv + w.hk;
        const int64_t base = ((seg + blockIdx.x) * kDecWarps + warp) * p.rows;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (!rvalid[h]) continue;
            float* po = p.part_o + (base + rr[h]) * D + 2 * tq;
#pragma unroll
            for (int n = 0; n < ND; ++n)
                *reinterpret_cast<float2*>(po + 8 * n) = make_float2(oacc[n][2 * h], oacc[n][2 * h + 1]);
            if (tq == 0) *reinterpret_cast<float2*>(p.part_ml + (base + rr[h]) * 2) = make_float2(m_run[h], l[h]);
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
                        bias = __uint_as_float((uint32_t)__ldg(p.bias + (int64_t)w.b * p.bias_st0 +
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
    kern<<<(unsigned)p.grid, kDecThreads, DCfg<D>::SMEM, stream>>>(p);
    return cudaGetLastError();
}

} // namespace

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
