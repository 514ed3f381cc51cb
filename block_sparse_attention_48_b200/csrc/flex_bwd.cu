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
// Work unit: (batch, kv head, kv block).  Its CTA keeps K and V of the block in
// shared memory and dK, dV in tensor memory, and walks the query blocks of the kv
// block's transposed BlockMask row for every query head of the kv head's group
// (partial tiles, where the mask is evaluated per element, then full ones).  At
// D = 64 the grid is persistent (one CTA per SM takes a unit of every round of
// gridDim.x units, in snake order): the next unit's K and V load into a second buffer while this
// unit's tiles run, and the epilogue warps store each unit's dK and dV; at D = 128
// (no room for a second buffer) there is one CTA per unit.  Per
// tile the five products run on the tensor core:
//   S^T  = K Q^T,  dP^T = V dO^T                 (TMEM, fp32)
//   dV  += P^T dO, dK  += dS^T Q,  dQ = dS K     (dS bf16 in shared memory; P^T bf16
//                                                 in TMEM at D = 64, in shared memory
//                                                 at D = 128)
// and dQ is added into an fp32 accumulator (several kv blocks contribute to one
// query row) by TMA reductions: a warp stages 32 rows x 32 columns in shared
// memory and one lane issues the reduce-add.  Each query block's nl (the negated
// log2 LSE, less the ALiBi column term) and Delta rows come in by bulk copy with
// its Q and dO tiles.
//
// At D = 64 consecutive tiles overlap: S^T and dP^T of tile i + 1 are computed as
// soon as the compute warps have read those of tile i, while they still turn them
// into P and dS, and the dQ of tile i is reduced while tile i + 1 runs.  At D = 128
// dV, dK, S^T and dP^T fill the 512 TMEM columns and dQ is computed over dP^T: the
// next tile's S^T follows as soon as its Q has landed (Q and dO have barriers of
// their own there, released after dK and dV), its dP^T once dQ has been read.
//
// Warps: 0-7 compute (thread = key row = TMEM lane; warps w and w + 4 share the
// rows of lane quadrant w and split the 128 query columns, and D, in halves),
// 8-11 dQ, dK and dV epilogue at D = 64 (warp 8 + q reads lane quadrant q), 12 TMA producer,
// 13 MMA issue, 14-15 idle (they complete the fourth warpgroup).  At D = 128 the
// compute warps read dQ themselves: it is on the way to the next tile, and they
// would otherwise wait.  Launched at 128 registers per thread, the compute
// warpgroups run at 168 and the other two at 88.
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

constexpr int kBwdThreads = 512;
constexpr int kComputeWarps = 8;
constexpr int kDqWarp0 = 8;  // warps 8-11
constexpr int kDqWarps = 4;
constexpr int kProdWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kLaunchRegs = 128;
constexpr int kComputeRegs = 168;
constexpr int kOtherRegs = 88;
static_assert(2 * 128 * kComputeRegs + 2 * 128 * kOtherRegs <= kBwdThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
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
    // P and dS, [kv][q] bf16 in the 128-byte swizzle, two 64-column boxes each: the
    // A operands of dV = P^T dO and dK = dS^T Q (K-major) and of dQ = dS K (MN-major).
    // At D = 64 P^T is in TMEM instead and the P space is unused.
    static constexpr int OFF_P = OFF_DO + NSLOT * TILE;
    static constexpr int OFF_DS = OFF_P + 2 * kBox;
    static constexpr int OFF_LD = OFF_DS + 2 * kBox;  // [NSLOT][nl, Delta][128] fp32
    // TMEM columns: S^T, dP^T, dV, dK; dQ in its own columns at D = 64 and over
    // dP^T at D = 128; at D = 64 also P^T (COL_PT)
    static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + D;
    static constexpr bool DQ_OVER_DP = D == 128;
    static constexpr uint32_t COL_DQ = DQ_OVER_DP ? COL_DP : 384u;
    // D = 64: P^T as bf16 in the last 64 TMEM columns, the A operand (TS form) of
    // dV += P^T dO; at D = 128 the 512 columns are taken
    static constexpr bool PT_TMEM = !DQ_OVER_DP;
    static constexpr uint32_t COL_PT = 448u;
    static_assert(!PT_TMEM || (COL_DQ + D <= COL_PT && COL_PT + 64 <= 512), "TMEM columns overlap");
    // Overlapped tiles (dQ in its own columns), whose dQ the epilogue warps read and
    // stage in two 32-row x 32-column fp32 boxes each (8 KB per warp).  Over dP^T the
    // compute warps stage it in the 4 KB of dS and of P each of them writes.
    static constexpr bool PIPE = !DQ_OVER_DP;
    // One Q and one dO slot (D = 128): separate barriers, qd_*[0] for Q and the nl /
    // Delta rows, qd_*[1] for dO, so that each refills as soon as its last reader
    // (dK, dV) is done.  With two slots (D = 64) Q and dO of a slot share qd_*[slot].
    static constexpr bool SPLIT_QD = NSLOT == 1;
    // Persistent CTAs (D = 64), K / V double-buffered: the second buffer is the P
    // space, unused with P^T in TMEM.
    static constexpr bool PERSIST = PIPE;
    static constexpr int NKV = PERSIST ? 2 : 1;
    static constexpr int off_k(uint32_t s) { return s ? OFF_P : OFF_K; }
    static constexpr int off_v(uint32_t s) { return s ? OFF_P + TILE : OFF_V; }
    static_assert(!PERSIST || (PT_TMEM && 2 * TILE <= 2 * kBox), "second K / V buffer does not fit the P space");
    static constexpr int OFF_STG = OFF_LD + NSLOT * 1024;
    static constexpr int SMEM = OFF_STG + (PIPE ? kDqWarps * 8192 : 0) + 1024;
};

struct __align__(16) BShared {
    uint64_t kv_full[2], kv_empty[2];  // K, V of a unit in buffer kvc % NKV; the unit's MMAs are done with them
    uint64_t qd_full[2], qd_empty[2];
    uint64_t sdp_full;  // S^T, dP^T of a tile are in TMEM
    uint64_t s_free;    // the compute warps have read them (one arrival per warp)
    uint64_t pds_full;  // P, dS of a tile are in shared memory (one arrival per warp)
    uint64_t pds_free;  // the gradient products have read them
    uint64_t dq_full, dq_free;  // dQ in TMEM; it has been read (one arrival per reading warp)
    uint64_t dkv_full, dkv_free;  // PERSIST: a unit's dK, dV are final in TMEM; the epilogue warps read them
    uint64_t drain;
    uint32_t tmem_base;
};

struct BTile {
    int hq, qb;
    bool partial;
    int b, hk, kb;  // its unit
    uint32_t kvc;   // index of its unit among this CTA's units that have tiles
    bool first;     // first tile of its unit
};

// The tiles of one CTA, in the same order for every role: for each query head of
// the group, the partial then the full query blocks of the kv block's transposed
// row.  The next entry is read one call ahead, so that its global-memory latency
// overlaps a tile's work.  Counts and indices are clamped (a corrupt BlockMask is
// reported, never read out of bounds).
struct BwdWalk {
    int b, hk, kb;
    int g, t, np, n, ahead;
    const int32_t* plist;
    const int32_t* flist;

    __device__ __forceinline__ int entry(int k) const { return ldg_now(k < np ? plist + k : flist + (k - np)); }

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
        ahead = n > 0 ? entry(0) : 0;
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
        int qb = ahead;
        if (qb < 0 || qb >= p.nq) { bad = true; qb = qb < 0 ? 0 : p.nq - 1; }
        out.hq = hk * p.G + g;
        out.qb = qb;
        out.partial = t < np;
        ++t;
        if (t < n) ahead = entry(t);
        return true;
    }
};

__device__ __forceinline__ void unit_coords(const BwdParams& p, int u, int& b, int& hk, int& kb)
{
    // kv block slowest: under causal-like masks the first kv blocks have the most
    // query blocks, so the longest units start first
    const int bh = p.B * p.Hkv;
    kb = u / bh;
    const int r = u - kb * bh;
    b = r / p.Hkv;
    hk = r - b * p.Hkv;
}

// Unit of this CTA in round r: units are dealt in rounds of gridDim.x, in
// alternating (snake) order, so that with units numbered longest first every CTA
// gets a similar amount of work; a CTA's units increase with r (none past the first
// one out of range).
__device__ __forceinline__ int unit_of(int r)
{
    const int g = gridDim.x, c = blockIdx.x;
    return r * g + ((r & 1) ? g - 1 - c : c);
}

// The tiles of all units of this CTA, in the same order for every role; units
// without tiles are passed over.
struct UnitWalk {
    BwdWalk w;
    int u, r;
    uint32_t kvc;  // units with tiles begun so far
    bool begun;    // the current unit has given a tile

    __device__ __forceinline__ void start(const BwdParams& p, bool& bad)
    {
        int b, hk, kb;
        unit_coords(p, u, b, hk, kb);
        w.init(p, b, hk, kb, bad);
        begun = false;
    }

    __device__ __forceinline__ void init(const BwdParams& p, bool& bad)
    {
        r = 0;
        u = unit_of(0);
        kvc = 0;
        begun = false;
        if (u < p.num_units) start(p, bad);
    }

    __device__ __forceinline__ bool next(const BwdParams& p, BTile& out, bool& bad)
    {
        while (u < p.num_units) {
            if (w.next(p, out, bad)) {
                out.b = w.b;
                out.hk = w.hk;
                out.kb = w.kb;
                out.first = !begun;
                if (!begun) {
                    begun = true;
                    ++kvc;
                }
                out.kvc = kvc - 1;
                return true;
            }
            u = unit_of(++r);
            if (u < p.num_units) start(p, bad);
        }
        return false;
    }
};

__device__ __forceinline__ uint64_t desc64(uint32_t hi, uint32_t lo)
{
    return ((uint64_t)hi << 32) | lo;
}

// descriptor offset (16-byte units) of the 16-wide K step k of a K-major operand
// held as 64-column boxes in the 128-byte swizzle
__device__ __forceinline__ uint32_t kstep(int k)
{
    return (uint32_t)(((k / 4) * kBox + (k % 4) * 32) >> 4);
}

template <int D>
__device__ __forceinline__ void bwd_producer(const BwdParams& p, BShared& sh, uint8_t* smem, Watchdog& wd,
                                             bool& bad)
{
    using C = BCfg<D>;
    UnitWalk w;
    w.init(p, bad);
    BTile tl;
    uint32_t i = 0, kvn = 0;  // tiles, units with tiles
    bool ok = true;
    while (ok && w.next(p, tl, bad)) {
        const int b = tl.b;
        if (tl.first) {
            // K, V of the unit, once the MMAs of the unit that last used the buffer are done
            const uint32_t kvs = tl.kvc % C::NKV;
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.kv_empty[kvs], ((tl.kvc / C::NKV) & 1) ^ 1, wd));
            if (!ok) break;
            if (elect_one_sync()) {
                mbar_arrive_expect_tx(&sh.kv_full[kvs], 2 * C::TILE);
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    tma_load_4d(smem + C::off_k(kvs) + c * kBox, &p.tm_k, &sh.kv_full[kvs], c * 64, tl.kb * 128, tl.hk,
                                b);
                    tma_load_4d(smem + C::off_v(kvs) + c * kBox, &p.tm_v, &sh.kv_full[kvs], c * 64, tl.kb * 128, tl.hk,
                                b);
                }
            }
            __syncwarp();
            kvn = tl.kvc + 1;
        }
        const uint32_t slot = i % C::NSLOT, use = i / C::NSLOT;
        if constexpr (C::SPLIT_QD) {
            const int64_t blk = ((int64_t)b * p.Hq + tl.hq) * p.nq + tl.qb;
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.qd_empty[0], (i & 1) ^ 1, wd));
            if (!ok) break;
            if (elect_one_sync()) {
                mbar_arrive_expect_tx(&sh.qd_full[0], C::TILE + 1024);
#pragma unroll
                for (int c = 0; c < D / 64; ++c)
                    tma_load_4d(smem + C::OFF_Q + c * kBox, &p.tm_q, &sh.qd_full[0], c * 64, tl.qb * 128, tl.hq, b);
                bulk_load(smem + C::OFF_LD, p.ld + blk * 256, 1024, &sh.qd_full[0]);
            }
            __syncwarp();
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.qd_empty[1], (i & 1) ^ 1, wd));
            if (!ok) break;
            if (elect_one_sync()) {
                mbar_arrive_expect_tx(&sh.qd_full[1], C::TILE);
#pragma unroll
                for (int c = 0; c < D / 64; ++c)
                    tma_load_4d(smem + C::OFF_DO + c * kBox, &p.tm_do, &sh.qd_full[1], c * 64, tl.qb * 128, tl.hq, b);
            }
            __syncwarp();
            ++i;
            continue;
        }
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.qd_empty[slot], (use & 1) ^ 1, wd));
        if (!ok) break;
        if (elect_one_sync()) {
            mbar_arrive_expect_tx(&sh.qd_full[slot], 2 * C::TILE + 1024);
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                tma_load_4d(smem + C::OFF_Q + slot * C::TILE + c * kBox, &p.tm_q, &sh.qd_full[slot], c * 64,
                            tl.qb * 128, tl.hq, b);
                tma_load_4d(smem + C::OFF_DO + slot * C::TILE + c * kBox, &p.tm_do, &sh.qd_full[slot], c * 64,
                            tl.qb * 128, tl.hq, b);
            }
            const int64_t blk = ((int64_t)b * p.Hq + tl.hq) * p.nq + tl.qb;
            bulk_load(smem + C::OFF_LD + slot * 1024, p.ld + blk * 256, 1024, &sh.qd_full[slot]);
        }
        __syncwarp();
        ++i;
    }
    // Copies still in flight land before the CTA exits: wait (bounded) for the
    // last issued phase of every slot and K / V buffer.
    Watchdog dw{wd.failed ? 1000000ull : wd.limit_ns, false};
    for (uint32_t j = 0; j < (uint32_t)C::NKV && j < kvn; ++j) {
        const uint32_t last = kvn - 1 - j;
        dw.failed = false;
        mbar_wait(&sh.kv_full[last % C::NKV], (last / C::NKV) & 1, dw);
    }
    if constexpr (C::SPLIT_QD) {
        for (int j = 0; j < 2 && i > 0; ++j) {
            dw.failed = false;
            mbar_wait(&sh.qd_full[j], (i - 1) & 1, dw);
        }
    } else {
        for (uint32_t j = 0; j < (uint32_t)C::NSLOT && j < i; ++j) {
            const uint32_t last = i - 1 - j;
            dw.failed = false;
            mbar_wait(&sh.qd_full[last % C::NSLOT], (last / C::NSLOT) & 1, dw);
        }
    }
    if ((threadIdx.x & 31) == 0 && (wd.failed || !ok)) atomicOr(p.status, STATUS_TIMEOUT);
}

template <int D>
__device__ __forceinline__ void bwd_mma(const BwdParams& p, BShared& sh, uint8_t* smem, uint32_t tmem, Watchdog& wd,
                                        bool& bad)
{
    using C = BCfg<D>;
    const uint32_t hi_k = (uint32_t)(sdesc_sw128(0, 16, 1024) >> 32);
    const uint32_t hi_mn = (uint32_t)(sdesc_sw128(0, kBox, 1024) >> 32);
    // K, V of each buffer (K-major for S^T and dP^T, K MN-major for dQ)
    uint32_t k_desc[C::NKV], v_desc[C::NKV], k_mn[C::NKV];
#pragma unroll
    for (int s2 = 0; s2 < C::NKV; ++s2) {
        k_desc[s2] = (uint32_t)sdesc_sw128(smem_u32(smem + C::off_k(s2)), 16, 1024);
        v_desc[s2] = (uint32_t)sdesc_sw128(smem_u32(smem + C::off_v(s2)), 16, 1024);
        k_mn[s2] = (uint32_t)sdesc_sw128(smem_u32(smem + C::off_k(s2)), kBox, 1024);
    }
    // the first tile of a unit waits for the unit's K and V
    auto wait_kv = [&](const BTile& t) -> bool {
        if (!t.first) return true;
        return __all_sync(0xFFFFFFFFu, mbar_wait(&sh.kv_full[t.kvc % C::NKV], (t.kvc / C::NKV) & 1, wd));
    };
    const uint32_t p_k = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_P), 16, 1024);
    const uint32_t ds_k = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_DS), 16, 1024);
    const uint32_t ds_mn = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_DS), kBox, 1024);
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
    constexpr uint32_t idesc_kv = idesc_bf16_f32(128, D, false, true);  // P^T dO, dS^T Q
    constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, true, true);   // dS K

    // SPLIT_QD: S^T = K Q^T, then (separately) dP^T = V dO^T of tile j, whose
    // commit signals both
    auto issue_s_only = [&](uint32_t j, const BTile& t) -> bool {
        const uint32_t kvs = t.kvc % C::NKV;
        if (!wait_kv(t)) return false;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.qd_full[0], j & 1, wd))) return false;
        const uint32_t q_k = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_Q), 16, 1024);
        tc_fence_after();
        if (elect_one_sync()) {
#pragma unroll
            for (int k = 0; k < D / 16; ++k)
                umma_ss(tmem + C::COL_S, desc64(hi_k, k_desc[kvs] + kstep(k)), desc64(hi_k, q_k + kstep(k)),
                        idesc_s, k > 0);
        }
        __syncwarp();
        return true;
    };
    auto issue_dp_only = [&](uint32_t j, const BTile& t) -> bool {
        const uint32_t kvs = t.kvc % C::NKV;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.qd_full[1], j & 1, wd))) return false;
        const uint32_t do_k = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_DO), 16, 1024);
        tc_fence_after();
        if (elect_one_sync()) {
#pragma unroll
            for (int k = 0; k < D / 16; ++k)
                umma_ss(tmem + C::COL_DP, desc64(hi_k, v_desc[kvs] + kstep(k)), desc64(hi_k, do_k + kstep(k)),
                        idesc_s, k > 0);
            umma_commit(&sh.sdp_full);
        }
        __syncwarp();
        return true;
    };
    // S^T = K Q^T and dP^T = V dO^T of tile j (Q and dO in slot j % NSLOT)
    auto issue_s = [&](uint32_t j, const BTile& t) -> bool {
        if constexpr (C::SPLIT_QD) return issue_s_only(j, t) && issue_dp_only(j, t);
        const uint32_t slot = j % C::NSLOT, kvs = t.kvc % C::NKV;
        if (!wait_kv(t)) return false;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.qd_full[slot], (j / C::NSLOT) & 1, wd))) return false;
        const uint32_t q_k = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_Q + slot * C::TILE), 16, 1024);
        const uint32_t do_k = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_DO + slot * C::TILE), 16, 1024);
        tc_fence_after();
        if (elect_one_sync()) {
#pragma unroll
            for (int k = 0; k < D / 16; ++k)
                umma_ss(tmem + C::COL_S, desc64(hi_k, k_desc[kvs] + kstep(k)), desc64(hi_k, q_k + kstep(k)),
                        idesc_s, k > 0);
#pragma unroll
            for (int k = 0; k < D / 16; ++k)
                umma_ss(tmem + C::COL_DP, desc64(hi_k, v_desc[kvs] + kstep(k)), desc64(hi_k, do_k + kstep(k)),
                        idesc_s, k > 0);
            umma_commit(&sh.sdp_full);
        }
        __syncwarp();
        return true;
    };
    // dK += dS^T Q, dV += P^T dO, dQ = dS K of tile j, 16 query (or key, for dQ)
    // rows of the K dimension per step; `last`: the last tile of its unit
    auto issue_grads = [&](uint32_t j, const BTile& t, bool last) -> bool {
        const uint32_t slot = j % C::NSLOT, kvs = t.kvc % C::NKV;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.pds_full, j & 1, wd))) return false;
        // a new unit's dK, dV start over in TMEM once the previous unit's were read
        if (C::PERSIST && t.first && t.kvc > 0 &&
            !__all_sync(0xFFFFFFFFu, mbar_wait(&sh.dkv_free, (t.kvc - 1) & 1, wd)))
            return false;
        const uint32_t q_mn = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_Q + slot * C::TILE), kBox, 1024);
        const uint32_t do_mn = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_DO + slot * C::TILE), kBox, 1024);
        tc_fence_after();
        if (elect_one_sync()) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                umma_ss(tmem + C::COL_DK, desc64(hi_k, ds_k + kstep(k)), desc64(hi_mn, q_mn + ((k * 2048) >> 4)),
                        idesc_kv, (!t.first || k > 0) ? 1u : 0u);
            if (C::SPLIT_QD) umma_commit(&sh.qd_empty[0]);  // Q read for the last time
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                if constexpr (C::PT_TMEM)
                    umma_ts(tmem + C::COL_DV, tmem + C::COL_PT + 8 * k, desc64(hi_mn, do_mn + ((k * 2048) >> 4)),
                            idesc_kv, (!t.first || k > 0) ? 1u : 0u);
                else
                    umma_ss(tmem + C::COL_DV, desc64(hi_k, p_k + kstep(k)), desc64(hi_mn, do_mn + ((k * 2048) >> 4)),
                            idesc_kv, (!t.first || k > 0) ? 1u : 0u);
            }
            if (C::SPLIT_QD) umma_commit(&sh.qd_empty[1]);  // dO read for the last time
        }
        __syncwarp();
        // the previous tile's dQ has been read from its columns
        if (C::PIPE && j > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait(&sh.dq_free, (j - 1) & 1, wd))) return false;
        tc_fence_after();
        if (elect_one_sync()) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                umma_ss(tmem + C::COL_DQ, desc64(hi_mn, ds_mn + ((k * 2048) >> 4)),
                        desc64(hi_mn, k_mn[kvs] + ((k * 2048) >> 4)), idesc_dq, k > 0);
            umma_commit(&sh.dq_full);
            if (!C::SPLIT_QD) umma_commit(&sh.qd_empty[slot]);
            umma_commit(&sh.pds_free);
            if (last) {
                umma_commit(&sh.kv_empty[kvs]);       // the unit's K, V are no longer read
                if (C::PERSIST) umma_commit(&sh.dkv_full);  // its dK, dV are final
            }
        }
        __syncwarp();
        return true;
    };

    bool ok = true;
    UnitWalk w;
    w.init(p, bad);
    BTile cur, nx;
    bool have = w.next(p, cur, bad);
    if (have) ok = issue_s(0, cur);
    uint32_t i = 0;
    while (ok && have) {
        const bool more = w.next(p, nx, bad);
        const bool last = !more || nx.first;  // the next tile, if any, begins another unit
        if (C::PIPE && more) {
            // the next tile's scores as soon as this tile's have been read
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.s_free, i & 1, wd)) && issue_s(i + 1, nx);
            if (!ok) break;
        }
        if (!(ok = issue_grads(i, cur, last))) break;
        if (!C::PIPE && more) {
            // the next S^T as soon as its Q has landed (this tile's S^T was read before
            // P and dS were formed); the next dP^T once dQ over dP^T has been read
            ok = issue_s_only(i + 1, nx) && __all_sync(0xFFFFFFFFu, mbar_wait(&sh.dq_free, i & 1, wd)) &&
                 issue_dp_only(i + 1, nx);
            if (!ok) break;
        }
        cur = nx;
        have = more;
        ++i;
    }
    // every issued MMA completes before TMEM is released
    if (elect_one_sync()) umma_commit(&sh.drain);
    __syncwarp();
    Watchdog dw{wd.failed ? 1000000ull : wd.limit_ns, false};
    const bool drained = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.drain, 0, dw));
    if ((threadIdx.x & 31) == 0 && (wd.failed || !ok || !drained)) atomicOr(p.status, STATUS_TIMEOUT);
}

// P and dS of one 32-column chunk of a key row, packed to bf16 pairs.  The score
// in log2 units is s * scale * log2e + r + nl[col], with nl the negated log2 LSE
// of the query row (minus the ALiBi column term when r holds the row's ALiBi
// term, see bwd_prep_kernel); soft-capping and bias enter as in score_and_grad.
// MASKED applies the chunk's mask word; without it every column is admitted.
template <int SCORE, bool MASKED>
__device__ __forceinline__ void pds_chunk(const BwdParams& p, const uint32_t (&sv)[32], const uint32_t (&dv)[32],
                                          uint32_t ld_s, int c, uint32_t mwc, uint64_t r2,
                                          const uint16_t* bias_row, int64_t q0, uint32_t (&pk)[16],
                                          uint32_t (&dk)[16])
{
    constexpr bool HAS_BIAS = SCORE == FA_SCORE_BIAS || SCORE == FA_SCORE_BIAS_SOFTCAP;
    constexpr bool CAP = SCORE == FA_SCORE_SOFTCAP || SCORE == FA_SCORE_BIAS_SOFTCAP;
    const float sl = p.scale * kLog2e;
    const uint64_t c2 = f2_pack(sl, sl);
    const uint64_t l2e2 = f2_pack(kLog2e, kLog2e);
    const float capl = p.softcap * kLog2e;
    const uint64_t capl2 = f2_pack(capl, capl);
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
        // the four columns' nl and Delta as 16-byte shared loads (the same address
        // in every lane: broadcast)
        const uint4 n4 = lds128(ld_s + (uint32_t)(32 * c + j) * 4u);
        const uint4 d4 = lds128(ld_s + 512u + (uint32_t)(32 * c + j) * 4u);
        const uint64_t nl[2] = {((uint64_t)n4.y << 32) | n4.x, ((uint64_t)n4.w << 32) | n4.z};
        const uint64_t dl[2] = {((uint64_t)d4.y << 32) | d4.x, ((uint64_t)d4.w << 32) | d4.z};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = j + 2 * h;
            const bool adm0 = !MASKED || ((mwc >> e) & 1u), adm1 = !MASKED || ((mwc >> (e + 1)) & 1u);
            float b0 = 0.f, b1 = 0.f;
            if constexpr (HAS_BIAS) {
                const int col = 32 * c + e;
                if (adm0) b0 = __uint_as_float((uint32_t)__ldg(bias_row + (q0 + col) * p.bias_st2) << 16);
                if (adm1) b1 = __uint_as_float((uint32_t)__ldg(bias_row + (q0 + col + 1) * p.bias_st2) << 16);
            }
            const float s0 = __uint_as_float(sv[e]), s1 = __uint_as_float(sv[e + 1]);
            uint64_t a2, g2 = 0;
            if constexpr (CAP) {
                const float y0 = SCORE == FA_SCORE_SOFTCAP ? s0 * p.softcap_in : fmaf(s0, p.softcap_in, b0 * p.softcap_inv);
                const float y1 = SCORE == FA_SCORE_SOFTCAP ? s1 * p.softcap_in : fmaf(s1, p.softcap_in, b1 * p.softcap_inv);
                const float t0 = tanh_accurate(y0), t1 = tanh_accurate(y1);
                a2 = f2_fma(f2_pack(t0, t1), capl2, nl[h]);
                g2 = f2_pack(fmaf(-t0, t0, 1.0f), fmaf(-t1, t1, 1.0f));
            } else {
                uint64_t base = nl[h];
                if constexpr (SCORE == FA_SCORE_ALIBI) base = f2_add(base, r2);
                if constexpr (HAS_BIAS) base = f2_fma(f2_pack(b0, b1), l2e2, base);
                a2 = f2_fma(f2_pack(s0, s1), c2, base);
            }
            float a0, a1;
            f2_unpack(a2, a0, a1);
            float e0 = ex2_approx(a0), e1 = ex2_approx(a1);
            if (MASKED) {
                e0 = adm0 ? e0 : 0.f;
                e1 = adm1 ? e1 : 0.f;
            }
            const uint64_t p2 = f2_pack(e0, e1);
            uint64_t d2 = f2_mul(p2, f2_sub(f2_pack(__uint_as_float(dv[e]), __uint_as_float(dv[e + 1])), dl[h]));
            if constexpr (CAP) d2 = f2_mul(d2, g2);
            float x0, x1;
            f2_unpack(d2, x0, x1);
            pk[e / 2] = pack_bf16x2(e0, e1);
            dk[e / 2] = pack_bf16x2(x0, x1);
        }
    }
}

template <int D, int SCORE>
__device__ __forceinline__ void bwd_compute(const BwdParams& p, BShared& sh, uint8_t* smem, uint32_t tmem,
                                            Watchdog& wd, bool& bad)
{
    using C = BCfg<D>;
    constexpr bool HAS_BIAS = SCORE == FA_SCORE_BIAS || SCORE == FA_SCORE_BIAS_SOFTCAP;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int quad = warp & 3, half = warp >> 2;  // TMEM lane quadrant; column half
    const int row = quad * 32 + lane;             // key row of the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t p_row = smem_u32(smem + C::OFF_P) + row * 128;
    const uint32_t ds_row = smem_u32(smem + C::OFF_DS) + row * 128;
    // D = 128: this warp's dQ staging, the 4 KB of dS and of P it writes (its 32 key
    // rows of one box)
    const uint32_t stage0 = smem_u32(smem + C::OFF_DS + half * kBox + quad * 4096);
    const uint32_t stage1 = smem_u32(smem + C::OFF_P + half * kBox + quad * 4096);
    // the current unit's key row and its document
    int64_t kv = 0;
    bool row_ok = false;
    const int32_t* doc_row = nullptr;
    int32_t kvdoc = 0;

    UnitWalk w;
    w.init(p, bad);
    BTile tl;
    uint32_t i = 0;
    float slope = 0.f;
    int slope_hq = -1;
    bool ok = true;
    while (ok && w.next(p, tl, bad)) {
        const int b = tl.b;
        if (tl.first) {
            kv = (int64_t)tl.kb * 128 + row;
            row_ok = kv < p.kv_len;
            doc_row = p.mask.has_doc ? p.mask.doc_ids + (int64_t)b * p.mask.doc_stride : nullptr;
            kvdoc = (doc_row && row_ok) ? __ldg(doc_row + kv) : 0;
        }
        const uint32_t slot = i % C::NSLOT;
        const int64_t q0 = (int64_t)tl.qb * 128;
        // the tile's 128 query rows: nl (the negated log2 LSE, -inf for a row that
        // admits nothing, so that its probabilities are 0), then Delta 512 bytes further
        const uint32_t ld_s = smem_u32(smem + C::OFF_LD + slot * 1024);

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
        // ALiBi: slope * log2e * (kv - q position at column 0); the column term is
        // folded into nl
        if (SCORE == FA_SCORE_ALIBI && tl.hq != slope_hq) {  // read once per query head
            slope = __ldg(p.slopes + tl.hq);
            slope_hq = tl.hq;
        }
        const float rterm = slope * kLog2e * (float)(kv - q0 - p.mask.q_offset);
        const uint64_t r2 = f2_pack(rterm, rterm);
        const uint16_t* bias_row = nullptr;
        if (HAS_BIAS) bias_row = p.bias + (int64_t)b * p.bias_st0 + (int64_t)tl.hq * p.bias_st1 + kv;

        // LSE / Delta arrived with Q and dO
        ok = mbar_wait(&sh.qd_full[slot], (i / C::NSLOT) & 1, wd);
        ok = ok && mbar_wait(&sh.sdp_full, i & 1, wd);
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
            if (cc == 1) {
                // this warp has read its S^T, dP^T columns of the tile
                tc_fence_before();
                mbar_arrive_warp(&sh.s_free);
            }
            uint32_t pk[16], dk[16];
            if (__all_sync(0xFFFFFFFFu, mwc == 0xFFFFFFFFu))
                pds_chunk<SCORE, false>(p, sv, dv, ld_s, c, mwc, r2, bias_row, q0, pk, dk);
            else
                pds_chunk<SCORE, true>(p, sv, dv, ld_s, c, mwc, r2, bias_row, q0, pk, dk);
            if (cc == 0) {
                // the previous tile's gradient products have read P and dS (and, at
                // D = 128, its dQ reductions the staging over them)
                if (i > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait(&sh.pds_free, (i - 1) & 1, wd))) {
                    ok = false;
                    break;
                }
                if (!C::PIPE) {
                    if (lane == 0) bulk_wait_read0();
                    __syncwarp();
                }
            }
            if constexpr (C::PT_TMEM) tmem_st16(tmem + lane_base + C::COL_PT + 16 * c, pk);
#pragma unroll
            for (int u4 = 0; u4 < 4; ++u4) {
                const uint32_t off = (c >> 1) * kBox + ((((c & 1) * 4 + u4) ^ (row & 7)) * 16);
                if constexpr (!C::PT_TMEM) sts128(p_row + off, pk[4 * u4], pk[4 * u4 + 1], pk[4 * u4 + 2], pk[4 * u4 + 3]);
                sts128(ds_row + off, dk[4 * u4], dk[4 * u4 + 1], dk[4 * u4 + 2], dk[4 * u4 + 3]);
            }
        }
        if (!ok) break;
        if constexpr (C::PT_TMEM) {
            tmem_st_wait();
            tc_fence_before();
        }
        fence_proxy_async_smem();
        mbar_arrive_warp(&sh.pds_full);
        if constexpr (!C::PIPE) {
            // dQ of this tile (thread = query row): each warp stages its 32 rows x 32
            // columns at a time and one lane adds them into the accumulator with TMA
            // reductions (rows past q_len land in the padding)
            if (!(ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.dq_full, i & 1, wd)))) break;
            tc_fence_after();
#pragma unroll 1
            for (int k = 0; k < 2; ++k) {
                const uint32_t stage = (k == 0 ? stage0 : stage1) + lane * 128;
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + C::COL_DQ + 32 * (2 * half + k), v);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    sts128(stage + ((u ^ (lane & 7)) * 16), v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
            }
            tc_fence_before();
            mbar_arrive_warp(&sh.dq_free);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const int y = (int)((((int64_t)b * p.Hq + tl.hq) * p.nq + tl.qb) * 128 + quad * 32);
                tma_reduce_add_2d(&p.tm_dq, stage0, 64 * half, y);
                tma_reduce_add_2d(&p.tm_dq, stage1, 64 * half + 32, y);
                bulk_commit();
            }
            __syncwarp();
        }
        ++i;
    }
    // the reductions complete before the CTA's shared memory is released
    if (!C::PIPE) {
        if (lane == 0) bulk_wait0();
        __syncwarp();
    }
    if (!ok) {
        if (lane == 0) atomicOr(p.status, STATUS_TIMEOUT);
        return;
    }
    if constexpr (C::PERSIST) return;  // the epilogue warps store dK, dV
    // One unit per CTA: the last gradient products (the last MMAs of the CTA) have completed
    if (i > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait(&sh.pds_free, (i - 1) & 1, wd))) {
        if (lane == 0) atomicOr(p.status, STATUS_TIMEOUT);
        return;
    }
    tc_fence_after();
    // dK = scale * (dS^T Q), dV = P^T dO of this kv block (zero if no query block
    // attends to it).  Every lane runs the (warp-collective) TMEM loads; only the
    // stores of key rows past kv_len are skipped.
    int b, hk, kb;
    unit_coords(p, blockIdx.x, b, hk, kb);
    kv = (int64_t)kb * 128 + row;
    row_ok = kv < p.kv_len;
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

// dQ of every tile (thread = query row = TMEM lane of its warp's quadrant): the
// warp stages its 32 rows, 32 columns at a time, in the 128-byte swizzle (two
// boxes, used in turn) and one lane adds each box into the fp32 accumulator with
// a TMA reduction; rows past q_len land in the padding.  After a unit's last
// tile, its dK = scale dS^T Q and dV = P^T dO (thread = key row; zero for a unit
// no query block attends to), converted to bf16 and stored.
template <int D>
__device__ __forceinline__ void bwd_dq_role(const BwdParams& p, BShared& sh, uint8_t* smem, uint32_t tmem,
                                            Watchdog& wd, bool& bad)
{
    using C = BCfg<D>;
    const int lane = threadIdx.x % 32, quad = (threadIdx.x / 32) & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t stage = smem_u32(smem + C::OFF_STG + quad * 8192);
    uint32_t i = 0, kvn = 0;  // tiles, units with tiles
    bool ok = true;
    for (int r = 0, u = unit_of(0); ok && u < p.num_units; u = unit_of(++r)) {
        int b, hk, kb;
        unit_coords(p, u, b, hk, kb);
        BwdWalk w;
        w.init(p, b, hk, kb, bad);
        BTile tl;
        bool any = false;
        while (ok && w.next(p, tl, bad)) {
            any = true;
            const int y = (int)((((int64_t)b * p.Hq + tl.hq) * p.nq + tl.qb) * 128 + quad * 32);
            if (!(ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.dq_full, i & 1, wd)))) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                const uint32_t box = stage + (c & 1) * 4096;
                if ((c & 1) == 0) {
                    // the reductions issued from these boxes have read them
                    if (lane == 0) bulk_wait_read0();
                    __syncwarp();
                }
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + C::COL_DQ + 32 * c, v);
                tmem_ld_wait();
#pragma unroll
                for (int uu = 0; uu < 8; ++uu)
                    sts128(box + lane * 128 + ((uu ^ (lane & 7)) * 16), v[4 * uu], v[4 * uu + 1], v[4 * uu + 2],
                           v[4 * uu + 3]);
                if (c == D / 32 - 1) {
                    // all of this warp's dQ columns are read
                    tc_fence_before();
                    mbar_arrive_warp(&sh.dq_free);
                }
                if (c & 1) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_reduce_add_2d(&p.tm_dq, stage, 32 * (c - 1), y);
                        tma_reduce_add_2d(&p.tm_dq, stage + 4096, 32 * c, y);
                        bulk_commit();
                    }
                    __syncwarp();
                }
            }
            ++i;
        }
        if (!ok) break;
        // the unit's dK, dV: every lane runs the (warp-collective) TMEM loads; only
        // the stores of key rows past kv_len are skipped
        if (any) {
            if (!(ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.dkv_full, kvn & 1, wd)))) break;
            tc_fence_after();
        }
        const int64_t kv = (int64_t)kb * 128 + row;
        const bool row_ok = kv < p.kv_len;
        uint16_t* dk_row = p.dk + (int64_t)b * p.dk_st0 + (int64_t)hk * p.dk_st1 + kv * p.dk_st2;
        uint16_t* dv_row = p.dv + (int64_t)b * p.dv_st0 + (int64_t)hk * p.dv_st1 + kv * p.dv_st2;
#pragma unroll 1
        for (int c = 0; c < 2 * (D / 32); ++c) {
            const bool is_k = c < D / 32;  // dK chunks, then dV chunks
            const int cc = is_k ? c : c - D / 32;
            uint32_t v[32];
            if (any) {
                tmem_ld32(tmem + lane_base + (is_k ? C::COL_DK : C::COL_DV) + 32 * cc, v);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = 0u;
            }
            const float sc = is_k ? p.scale : 1.0f;
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]) * sc, __uint_as_float(v[2 * j + 1]) * sc);
            if (row_ok) {
                uint4* dst = reinterpret_cast<uint4*>((is_k ? dk_row : dv_row) + 32 * cc);
#pragma unroll
                for (int j = 0; j < 4; ++j) dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            }
        }
        if (any) {
            tc_fence_before();
            mbar_arrive_warp(&sh.dkv_free);
            ++kvn;
        }
    }
    // the reductions complete before the CTA's shared memory is released
    if (lane == 0) bulk_wait0();
    __syncwarp();
    if (lane == 0 && !ok) atomicOr(p.status, STATUS_TIMEOUT);
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
        for (int s2 = 0; s2 < 2; ++s2) {
            mbar_init(&sh.kv_full[s2], 1);
            mbar_init(&sh.kv_empty[s2], 1);
        }
        mbar_init(&sh.dkv_full, 1);
        mbar_init(&sh.dkv_free, kDqWarps);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh.qd_full[s], 1);
            mbar_init(&sh.qd_empty[s], 1);
        }
        mbar_init(&sh.sdp_full, 1);
        mbar_init(&sh.s_free, kComputeWarps);
        mbar_init(&sh.pds_full, kComputeWarps);
        mbar_init(&sh.pds_free, 1);
        mbar_init(&sh.dq_full, 1);
        mbar_init(&sh.dq_free, C::PIPE ? kDqWarps : kComputeWarps);
        mbar_init(&sh.drain, 1);
        mbar_fence_init();
    }
    if (warp == kProdWarp && (threadIdx.x & 31) == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_do);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_v);
        tma_prefetch_desc(&p.tm_dq);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    Watchdog wd{p.watchdog_ns, false};
    bool bad = false;
    if (warp >= kComputeWarps) {
        regs_dec<kOtherRegs>();
        if (warp >= kDqWarp0 && warp < kDqWarp0 + kDqWarps) {
            if constexpr (C::PIPE) bwd_dq_role<D>(p, sh, smem, tmem, wd, bad);
        }
        else if (warp == kProdWarp) bwd_producer<D>(p, sh, smem, wd, bad);
        else if (warp == kMmaWarp) bwd_mma<D>(p, sh, smem, tmem, wd, bad);
    } else {
        regs_inc<kComputeRegs>();
        bwd_compute<D, SCORE>(p, sh, smem, tmem, wd, bad);
    }
    if (bad) atomicOr(p.status, STATUS_BAD_BLOCKMASK);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// nl, Delta and the zeroed accumulator over the padded rows.  D / 8 lanes share a
// row, each with one 16-byte piece of its O and dO rows; a warp covers 32 / (D / 8)
// rows per step and takes kPrepSteps steps, issuing every load first.  One step
// at eight blocks per SM (measured): occupancy keeps more loads in flight than
// longer steps per warp.
// nl = -(LSE * log2e + slope * log2e * (q mod 128)) with the ALiBi slope of the
// row's head (0 without ALiBi): the kernel adds the key row's term
// slope * log2e * (kv - q position of the block's first row).  Rows past q_len, and
// rows whose LSE is -inf, get nl = -inf (probability 0) and Delta 0.
constexpr int kPrepSteps = 1;

__device__ __forceinline__ float dot_bf16x8(uint4 a, uint4 b)
{
    const uint32_t x[4] = {a.x, a.y, a.z, a.w}, y[4] = {b.x, b.y, b.z, b.w};
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        s = fmaf(__uint_as_float(x[i] << 16), __uint_as_float(y[i] << 16), s);
        s = fmaf(__uint_as_float(x[i] & 0xFFFF0000u), __uint_as_float(y[i] & 0xFFFF0000u), s);
    }
    return s;
}

__global__ void __launch_bounds__(256, 8) bwd_prep_kernel(const BwdPrepParams p)
{
    const int lpr = p.D / 8;  // lanes per row: 8 or 16
    const int lane = threadIdx.x & 31, piece = lane % lpr, rpw = 32 / lpr;
    const int64_t warp = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;
    const int64_t span = (int64_t)p.nq * 128;
    uint4 ov[kPrepSteps], dv[kPrepSteps];
    float lv[kPrepSteps];
#pragma unroll
    for (int it = 0; it < kPrepSteps; ++it) {
        const int64_t r = (warp * kPrepSteps + it) * rpw + lane / lpr;
        const int64_t bh = r / span, q = r - bh * span;
        ov[it] = dv[it] = make_uint4(0u, 0u, 0u, 0u);
        lv[it] = -INFINITY;
        if (r < p.rows_pad && q < p.q_len) {
            const int64_t hq = bh % p.Hq, b = bh / p.Hq;
            ov[it] = __ldg(reinterpret_cast<const uint4*>(p.o + b * p.o_st0 + hq * p.o_st1 + q * p.o_st2) + piece);
            dv[it] = __ldg(reinterpret_cast<const uint4*>(p.dout + b * p.do_st0 + hq * p.do_st1 + q * p.do_st2) + piece);
            lv[it] = __ldg(p.lse + bh * p.q_len + q);
        }
    }
#pragma unroll
    for (int it = 0; it < kPrepSteps; ++it) {
        const int64_t r = (warp * kPrepSteps + it) * rpw + lane / lpr;
        float s = dot_bf16x8(ov[it], dv[it]);
        for (int o2 = 1; o2 < lpr; o2 <<= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o2);  // within the row's lanes
        if (r >= p.rows_pad) continue;
        const int64_t bh = r / span, q = r - bh * span;
        if (piece == 0) {
            float nl = -INFINITY;
            if (lv[it] != -INFINITY) {
                const float col = p.slopes ? __ldg(p.slopes + bh % p.Hq) * kLog2e * (float)(q % 128) : 0.f;
                nl = -fmaf(lv[it], kLog2e, col);
            }
            float* blk = p.ld + (bh * p.nq + q / 128) * 256;
            blk[q % 128] = nl;
            blk[128 + q % 128] = q < p.q_len ? s : 0.f;
        }
        float4* acc = reinterpret_cast<float4*>(p.dq_acc + r * p.D) + 2 * piece;
        acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
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
    const float* src = p.dq_acc + (bh * p.nq * 128 + q) * p.D + j;
    const float4 a = *reinterpret_cast<const float4*>(src);
    const float4 c = *reinterpret_cast<const float4*>(src + 4);
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
            // the register split assumes the launch allocation: refuse anything else
            // rather than launch a kernel whose setmaxnreg.inc could never be served
            cudaFuncAttributes attr;
            cudaError_t e = cudaFuncGetAttributes(&attr, kern);
            if (e != cudaSuccess) return e;
            if (attr.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, BCfg<D>::SMEM);
            if (e != cudaSuccess) return e;
            if (current_ctx(&key)) done.push_back(key);
        }
    }
    // persistent CTAs: one per SM (at most one unit each when there are fewer units)
    const int grid = BCfg<D>::PERSIST ? (p.num_units < p.num_sms ? p.num_units : (p.num_sms > 0 ? p.num_sms : 1))
                                      : p.num_units;
    kern<<<grid, kBwdThreads, BCfg<D>::SMEM, stream>>>(p);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_bwd_prep(const BwdPrepParams& p, cudaStream_t stream)
{
    if (p.rows_pad == 0) return cudaSuccess;
    const int64_t rows_per_block = 8 * kPrepSteps * (32 / (p.D / 8));
    const int64_t blocks = (p.rows_pad + rows_per_block - 1) / rows_per_block;
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
