// Block-sparse FlexAttention forward pass for sm_100a.
//
//   out = softmax(mod(Q K^T * scale)) V,  LSE = logsumexp of the modified scores
//
// ("Flex Attention" paper review sec. 2.1; attention-gym "Concepts".)  The KV loop
// of each 128-row query tile walks only the kv blocks its BlockMask row lists
// (paper review sec. 4.3, indirect memory access): first the full blocks, where
// no mask is evaluated, then the partial blocks, where the mask is evaluated per
// element (sec. 4.2).  score_mod is applied to every admitted score.  Softmax is
// computed online (sec. 3.3): a running row maximum and sum with rescaling.
//
// Structure of one persistent CTA (384 threads, one CTA per SM):
//   warps 0-3  softmax warpgroup of stream 0 (thread = query row)
//   warps 4-7  softmax warpgroup of stream 1
//   warp  8    MMA issue for stream 0 (one elected lane issues): S = Q K^T and O += P V
//   warp  9    TMA producer (one elected lane issues): Q, K, V and bias tiles of both streams
//   warp  10   counts each stream's tiles at start-up, then issues stream 1's MMAs (elected lane)
//   warp  11   idle (completes the third warpgroup for register reallocation)
// The softmax warpgroups take registers from the third warpgroup (setmaxnreg):
// launched at 168 per thread, they run at 208 and the third at 88.
//
// Each CTA runs two independent streams of work items (b, hq, query block), so
// that the tensor core works for one stream while the other stream's softmax
// runs.  Accumulators live in tensor memory (TMEM).  At D = 64 every stream has
// its own S (fp32 scores, 128 columns), P (bf16 probabilities, 64 columns) and O
// (64 columns): S of the next tile is computed while the softmax of the current
// tile runs, as soon as the softmax has copied S into registers.  At D = 128 the
// 512 columns hold only S and O of both streams, so P is written over S and the
// next S waits for the P V product that reads P.
// K and V tiles stream through shared-memory rings shared by both streams and
// filled in a fixed interleaved order (round r: stream 0's r-th tile, then
// stream 1's), so every role can compute which slot holds which tile.  Each
// stream's MMAs are issued in a fixed order by its own thread.  Every role reads
// the BlockMask one step ahead of use.
//
// O is rescaled only when a row maximum grows by more than 2^8 (log2 domain):
// the final O / l and LSE are the same for any choice of the running maximum.
#pragma once

#include <mutex>
#include <vector>

#include <cuda_runtime.h>

#include "context.cuh"
#include "flex_fwd.cuh"
#include "ptx.cuh"
#include "score_math.cuh"

namespace fa {

namespace {

constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 208;
constexpr int kOtherRegs = 88;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kMmaWarp0 = 8;
constexpr int kLoadWarp = 9;
constexpr int kMmaWarp1 = 10;  // also counts the streams' tiles at start-up
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kBox = 16384;  // bytes of one 128-row x 64-column bf16 TMA box
constexpr int kMaxSlots = 6;  // deepest K / V ring

template <int D, int SCORE>
struct Cfg {
    static constexpr bool SEP_P = D == 64;  // P in its own TMEM columns
    // The two softmax warps on one SM sub-partition (warp w of stream 0, warp
    // w + 4 of stream 1) take turns on the exponential pass, so that one runs
    // its exponentials on the sub-partition's MUFU while the other does the
    // rest of its tile.  Measured faster at D = 64 without a bias tensor; at
    // D = 128 (twice the MMA time per tile) and with a bias it was not.
    static constexpr bool TURNS = D == 64 && (SCORE == FA_SCORE_NONE || SCORE == FA_SCORE_ALIBI);
    static constexpr bool HAS_BIAS = SCORE == FA_SCORE_BIAS || SCORE == FA_SCORE_BIAS_SOFTCAP;
    static constexpr bool HAS_CAP = SCORE == FA_SCORE_SOFTCAP || SCORE == FA_SCORE_BIAS_SOFTCAP;
    static constexpr int TILE = 128 * D * 2;
    // ring depths (slots) within the 227 KB of shared memory
    static constexpr int NK = D == 64 ? (HAS_BIAS ? 2 : 3) : 2;
    static constexpr int NV = D == 64 ? (HAS_BIAS ? 3 : 6) : 2;
    static constexpr int NB = HAS_BIAS ? (D == 64 ? 3 : 1) : 0;
    static constexpr int BIAS_TILE = 128 * 128 * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 2 * TILE;
    static constexpr int OFF_V = OFF_K + NK * TILE;
    static constexpr int OFF_B = OFF_V + NV * TILE;
    static constexpr int SMEM = OFF_B + NB * BIAS_TILE + 1024;
    // TMEM columns of stream s
    static constexpr uint32_t s_col(int s) { return 128u * s; }
    static constexpr uint32_t p_col(int s) { return SEP_P ? 256u + 64u * s : 128u * s; }
    static constexpr uint32_t o_col(int s) { return SEP_P ? 384u + 64u * s : 256u + (uint32_t)D * s; }
};

struct __align__(16) Shared {  // barriers and small shared state
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[kMaxSlots], k_empty[kMaxSlots];
    uint64_t v_full[kMaxSlots], v_empty[kMaxSlots];
    uint64_t b_full[3], b_empty[3];
    uint64_t s_full[2], s_free[2], p_full[2], p_free[2], o_full[2], o_empty[2];
    uint64_t drain[2];
    uint64_t turn[2][4];  // stream s's warp w finished an exponential pass
    uint64_t never;  // completed by nothing (watchdog self-test)
    uint32_t tmem_base;
    int total[2];  // tiles of each stream
    int bad;       // a count read by the counting warp was out of range
};

// A work item: query block qb of (b, hq), and its BlockMask row.
struct Item {
    int b, hq, qb;
    int row;       // BlockMask row
    int npart, n;  // tiles: [0, npart) from the partial list, [npart, n) from the full list
    const int32_t* full_list;
    const int32_t* part_list;
};

// Work item of stream s, k-th in that stream.  Items are numbered longest first
// (see row_at_rank); rounds of 2 * grid items are dealt to CTAs in alternating
// (snake) order, so that every CTA gets a mix of long and short items.
__device__ __forceinline__ long long item_index(int s, int k, int grid, int cta)
{
    int pos = (k & 1) ? 2 * (grid - 1 - cta) + s : 2 * cta + s;
    return (long long)k * 2 * grid + pos;
}

// BlockMask rows (r = (mb * bm_H + mh) * nq + qb) ordered by their tile count,
// most tiles first, ranked by every CTA at start-up when the host asks for it
// (num_rows > 0, at most kMaxOrderRows rows); ties, and the other cases, keep the
// query-block-descending order (which is the tile-count order of causal-like
// masks).
constexpr int kMaxOrderRows = 256;
__shared__ uint16_t s_row_order[kMaxOrderRows];

// Row at position k of the query-block-descending order.
__device__ __forceinline__ int fallback_row(const FwdParams& p, int k)
{
    const int bmh = p.bm_B * p.bm_H;
    const int qb = p.nq - 1 - k / bmh;
    return (k % bmh) * p.nq + qb;
}

__device__ __forceinline__ bool rows_ranked(const FwdParams& p)
{
    return p.num_rows > 0 && p.num_rows <= kMaxOrderRows;
}

__device__ __forceinline__ int row_at_rank(const FwdParams& p, int k)
{
    return rows_ranked(p) ? (int)s_row_order[k] : fallback_row(p, k);
}

// Rank the BlockMask rows (all threads of the CTA, before the pipeline starts):
// key = (65535 - tiles) << 16 | fallback position, rank = number of smaller keys.
// `scratch` is kMaxOrderRows words of shared memory free until the pipeline runs.
__device__ __forceinline__ void rank_rows(const FwdParams& p, uint32_t* scratch)
{
    const int R = p.num_rows;
    if (!rows_ranked(p)) return;
    const int bmh = p.bm_B * p.bm_H;
    for (int r = threadIdx.x; r < R; r += blockDim.x) {
        int a = __ldg(p.kv_num + r), f = p.has_full ? __ldg(p.full_num + r) : 0;
        a = min(max(a, 0), p.nkv);  // corrupt counts are reported by the walks
        f = min(max(f, 0), p.nkv);
        const int qb = r % p.nq;
        const uint32_t pos = (uint32_t)((p.nq - 1 - qb) * bmh + r / p.nq);
        scratch[r] = ((uint32_t)(65535 - min(a + f, 65535)) << 16) | pos;
    }
    __syncthreads();
    for (int r = threadIdx.x; r < R; r += blockDim.x) {
        const uint32_t key = scratch[r];
        int rank = 0;
        for (int j = 0; j < R; ++j) rank += scratch[j] < key;
        s_row_order[rank] = (uint16_t)r;
    }
    __syncthreads();
}

// Coordinates and BlockMask lists of work item idx (counts left unset).  Each
// BlockMask row serves M = (B / bm_B) * (Hq / bm_H) items (its broadcast batch and
// heads), numbered consecutively.
template <int EXT>
__device__ __forceinline__ Item item_at(const FwdParams& p, int idx)
{
    Item it;
    if constexpr (!(EXT & kExtRank)) {
        // query block descending, then (b, hq): two divisions
        const int bh_count = p.B * p.Hq;
        const int qb_rank = idx / bh_count;
        const int bh = idx - qb_rank * bh_count;
        it.qb = p.nq - 1 - qb_rank;
        it.b = bh / p.Hq;
        it.hq = bh - it.b * p.Hq;
        const int r = ((p.bm_B == 1 ? 0 : it.b) * p.bm_H + (p.bm_H == 1 ? 0 : it.hq)) * p.nq + it.qb;
        it.full_list = p.has_full ? p.full_idx + (int64_t)r * p.nkv : nullptr;
        it.part_list = p.kv_idx + (int64_t)r * p.nkv;
        it.row = r;
        it.npart = it.n = 0;
        return it;
    }
    const int inst_h = p.bm_H == 1 ? p.Hq : 1;
    const int M = (p.bm_B == 1 ? p.B : 1) * inst_h;
    const int rank = idx / M;
    const int inst = idx - rank * M;
    const int r = row_at_rank(p, rank);
    it.qb = r % p.nq;
    const int mbh = r / p.nq;
    const int ih = inst % inst_h, ib = inst / inst_h;
    it.b = p.bm_B == 1 ? ib : mbh / p.bm_H;
    it.hq = p.bm_H == 1 ? ih : mbh % p.bm_H;
    it.full_list = p.has_full ? p.full_idx + (int64_t)r * p.nkv : nullptr;
    it.part_list = p.kv_idx + (int64_t)r * p.nkv;
    it.row = r;
    it.npart = it.n = 0;
    return it;
}

// An item's BlockMask reads in flight (only raw values are held): item_finish()
// validates them, so the loads are waited for only when the item is used.
struct ItemLoad {
    int idx;
    int nf_raw, np_raw;
    int f0_raw, p0_raw;  // first entries of the two lists
    float slope;         // ALiBi slope of the head (ALIBI only)
    int qdoc;            // document id of this thread's query row (softmax, DOCUMENT only)
    bool valid;          // an item exists at this stream position
};

template <int EXT>
__device__ __forceinline__ void item_issue(const FwdParams& p, long long idx, ItemLoad& L, bool want_first,
                                           bool want_slope, int row)
{
    L.valid = idx < p.num_items;
    L.f0_raw = L.p0_raw = 0;
    if (!L.valid) return;
    L.idx = (int)idx;
    const Item it = item_at<EXT>(p, L.idx);
    const int64_t r = it.row;
    // read one item ahead (ldg_now: issued here, not at the first use)
    L.nf_raw = p.has_full ? ldg_now(p.full_num + r) : 0;
    L.np_raw = ldg_now(p.kv_num + r);
    if (want_first && p.nkv > 0) {
        L.f0_raw = p.has_full ? ldg_now(it.full_list) : 0;
        L.p0_raw = ldg_now(it.part_list);
    }
    if (want_slope) L.slope = ldg_now(p.slopes + it.hq);
    if (row >= 0 && p.mask.has_doc) {
        const int64_t q = (int64_t)it.qb * 128 + row;
        L.qdoc = q < p.q_len ? ldg_now(p.mask.doc_ids + (int64_t)it.b * p.mask.doc_stride + q + p.mask.q_offset)
                             : INT32_MIN;
    }
}

__device__ __forceinline__ int clamp_count(int v, int nkv, bool& bad)
{
    if (v < 0 || v > nkv) {
        bad = true;
        return v < 0 ? 0 : nkv;
    }
    return v;
}

__device__ __forceinline__ int clamp_kb(int kb, int nkv, bool& bad)
{
    if (kb < 0 || kb >= nkv) {
        bad = true;
        return kb < 0 ? 0 : nkv - 1;
    }
    return kb;
}

template <int EXT>
__device__ __forceinline__ Item item_finish(const FwdParams& p, const ItemLoad& L, bool& bad)
{
    Item it = item_at<EXT>(p, L.idx);
    it.npart = clamp_count(L.np_raw, p.nkv, bad);
    it.n = it.npart + clamp_count(L.nf_raw, p.nkv, bad);
    return it;
}

// Raw (unvalidated) kv block of tile t of an item.  A row's partial blocks come
// first, then its full blocks (each list ascending): under causal-like masks the
// diagonal block, whose scores carry the largest position biases, is seen first,
// so the running maximum rarely moves afterwards.
__device__ __forceinline__ int list_raw(const Item& it, int t)
{
    return ldg_now(t < it.npart ? it.part_list + t : it.full_list + (t - it.npart));
}

// kv block of an item's first tile from the prefetched list heads.
__device__ __forceinline__ int first_kb_raw(const Item& it, int f0_raw, int p0_raw)
{
    return it.npart > 0 ? p0_raw : f0_raw;
}

// Position of stream s's r-th tile in the interleaved production order.
__device__ __forceinline__ uint32_t tile_seq(int s, int r, int T0, int T1)
{
    return (uint32_t)(min(r, T0) + min(r, T1) + ((s == 1 && r < T0) ? 1 : 0));
}

// Cursor over the tiles of one stream's non-empty items, run by a whole warp:
// lane i holds the kv block of tile 32 c + i of the current item (c the current
// chunk of 32 tiles), read with one load per lane, and each tile takes its kv
// block with a shuffle.  The next item's counts are read one item ahead.
template <int EXT>
struct TileWalk {
    Item it;
    int t;
    int kb;       // kv block of tile t
    int kb_lane;  // raw kv block of tile (t & ~31) + lane
    int k;        // stream position of the next item to read
    ItemLoad nx;
    bool done;

    __device__ __forceinline__ void fetch(const FwdParams& p, int s)
    {
        item_issue<EXT>(p, item_index(s, k++, gridDim.x, blockIdx.x), nx, false, false, -1);
    }

    __device__ __forceinline__ void load_chunk(int base)
    {
        const int tt = base + (int)(threadIdx.x & 31);
        kb_lane = tt < it.n ? list_raw(it, tt) : 0;
    }

    __device__ __forceinline__ void next_item(const FwdParams& p, int s, bool& bad)
    {
        for (;;) {
            if (!nx.valid) {
                done = true;
                return;
            }
            it = item_finish<EXT>(p, nx, bad);
            if (it.n > 0) break;
            fetch(p, s);
        }
        t = 0;
        load_chunk(0);
        fetch(p, s);
        kb = clamp_kb(__shfl_sync(0xFFFFFFFFu, kb_lane, 0), p.nkv, bad);
    }

    __device__ __forceinline__ void init(const FwdParams& p, int s, bool& bad)
    {
        k = 0;
        done = false;
        fetch(p, s);
        next_item(p, s, bad);
    }

    __device__ __forceinline__ void advance(const FwdParams& p, int s, bool& bad)
    {
        if (++t == it.n) {
            next_item(p, s, bad);
            return;
        }
        if ((t & 31) == 0) load_chunk(t);
        kb = clamp_kb(__shfl_sync(0xFFFFFFFFu, kb_lane, t & 31), p.nkv, bad);
    }
};

// The MMA threads need only each item's tile count: a slim cursor with the next
// item's counts read one item ahead.
template <int EXT>
struct CountWalk {
    int n, t;  // tiles of the current item, tile within it
    int k;     // stream position of the next item to read
    int nf_raw, np_raw;
    bool nx_valid;

    __device__ __forceinline__ void fetch(const FwdParams& p, int s)
    {
        const long long idx = item_index(s, k++, gridDim.x, blockIdx.x);
        nx_valid = idx < p.num_items;
        if (!nx_valid) return;
        const int64_t r = item_at<EXT>(p, (int)idx).row;
        nf_raw = p.has_full ? __ldg(p.full_num + r) : 0;
        np_raw = __ldg(p.kv_num + r);
    }

    __device__ __forceinline__ void next_item(const FwdParams& p, int s, bool& bad)
    {
        for (;;) {
            if (!nx_valid) return;
            n = clamp_count(nf_raw, p.nkv, bad) + clamp_count(np_raw, p.nkv, bad);
            fetch(p, s);
            if (n > 0) break;
        }
        t = 0;
    }

    __device__ __forceinline__ void init(const FwdParams& p, int s, bool& bad)
    {
        k = 0;
        n = 0;
        t = 0;
        fetch(p, s);
        next_item(p, s, bad);
    }

    __device__ __forceinline__ void advance(const FwdParams& p, int s, bool& bad)
    {
        if (++t == n) next_item(p, s, bad);
    }
};

__device__ __forceinline__ void report(const FwdParams& p, int bits)
{
    atomicOr(p.status, bits);
}

// ---------------------------------------------------------------- math

// P = exp2(u * F + b + g * j) of one row (128 scores, column j) as bf16 to TMEM at
// p_addr, and its sum in two packed fp32 accumulators; the column term g * j only
// when COLTERM (ALiBi), carried as a running pair and recomputed exactly every 16
// columns.  The exponentials run on MUFU (ex2.approx).
template <bool COLTERM>
__device__ __forceinline__ void exp_pass(const float (&x)[128], uint64_t F2, float b, float g, uint32_t p_addr,
                                         uint64_t& la, uint64_t& lb)
{
    const uint64_t step2 = f2_pack(2.0f * g, 2.0f * g);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint32_t pk[8];
        uint64_t b2;
        if (COLTERM) {
            const float bc = fmaf(g, (float)(16 * c), b);
            b2 = f2_pack(bc, bc + g);
        } else {
            b2 = f2_pack(b, b);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = 16 * c + 2 * j;
            float a0, a1, e0, e1;
            f2_unpack(f2_fma(f2_pack(x[e], x[e + 1]), F2, b2), a0, a1);
            if (COLTERM && j < 7) b2 = f2_add(b2, step2);
            e0 = ex2_approx(a0);
            e1 = ex2_approx(a1);
            if (j & 1) lb = f2_add(lb, f2_pack(e0, e1));
            else la = f2_add(la, f2_pack(e0, e1));
            pk[j] = pack_bf16x2(e0, e1);
        }
        tmem_st8(p_addr + 8 * c, pk);
    }
}

// ---------------------------------------------------------------- MMA issue

// Shared-memory descriptors of every operand buffer, built once.  All K-major
// ones share one high word, the MN-major ones another; a K step of an MMA adds a
// small constant to the start-address field in the low word.
struct MmaDescs {
    uint32_t q;   // Q tile of this stream (K-major)
    uint32_t k0;  // K ring slot 0 (K-major); slot i starts TILE bytes further
    uint32_t v0;  // V ring slot 0 (MN-major, 64-column chunks 16 KB apart)
    uint32_t hi_k, hi_mn;
};

__device__ __forceinline__ uint64_t desc64(uint32_t hi, uint32_t lo)
{
    return ((uint64_t)hi << 32) | lo;
}

// Tile r of a stream as the MMA thread sees it.
struct MmaTile {
    uint32_t seq;
    bool first, last;  // first / last tile of its item
};

// O (+)= P V of one tile of stream S: P (128 x 128 bf16) from TMEM, V from its
// ring slot (operands ready: P signalled, V landed, O read out if first).
template <int D, int SCORE>
__device__ __forceinline__ void issue_pv(Shared& sh, int S, const MmaTile& tl, uint32_t tmem, const MmaDescs& dd)
{
    using C = Cfg<D, SCORE>;
    const uint32_t slot = tl.seq % C::NV;
    tc_fence_after();
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
    const uint32_t vd = dd.v0 + slot * (uint32_t)(C::TILE >> 4);
    const uint32_t o_tmem = tmem + C::o_col(S), p_tmem = tmem + C::p_col(S);
    if (elect_one_sync()) {
#pragma unroll
        for (int k = 0; k < 8; ++k)  // 16 kv rows (2 KB of V) per K step
            umma_ts(o_tmem, p_tmem + 8 * k, desc64(dd.hi_mn, vd + (uint32_t)((k * 2048) >> 4)), idesc_o,
                    (!tl.first || k > 0) ? 1u : 0u);
        umma_commit(&sh.v_empty[slot]);
        if (C::SEP_P) umma_commit(&sh.p_free[S]);
        if (tl.last) umma_commit(&sh.o_full[S]);
    }
    __syncwarp();
}

// S(r) = Q K^T of one tile of stream S (operands ready).
template <int D, int SCORE>
__device__ __forceinline__ void issue_s(Shared& sh, int S, const MmaTile& tl, uint32_t tmem, const MmaDescs& dd)
{
    using C = Cfg<D, SCORE>;
    const uint32_t slot = tl.seq % C::NK;
    tc_fence_after();
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
    const uint32_t kd = dd.k0 + slot * (uint32_t)(C::TILE >> 4);
    if (elect_one_sync()) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
            // start address advances 32 bytes per K step inside a 128-byte row, 16 KB per 64 columns
            const uint32_t off = (uint32_t)(((k / 4) * kBox + (k % 4) * 32) >> 4);
            umma_ss(tmem + C::s_col(S), desc64(dd.hi_k, dd.q + off), desc64(dd.hi_k, kd + off), idesc_s, k > 0);
        }
        umma_commit(&sh.k_empty[slot]);
        umma_commit(&sh.s_full[S]);
        if (tl.last) umma_commit(&sh.q_empty[S]);
    }
    __syncwarp();
}

// Blocking form of the P V step: wait for its operands, then issue.
template <int D, int SCORE>
__device__ __forceinline__ bool mma_pv(Shared& sh, int S, const MmaTile& tl, uint32_t r, uint32_t& ocount,
                                       uint32_t tmem, const MmaDescs& dd, Watchdog& wd)
{
    using C = Cfg<D, SCORE>;
    const uint32_t slot = tl.seq % C::NV;
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.p_full[S], r & 1, wd))) return false;
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.v_full[slot], (tl.seq / C::NV) & 1, wd))) return false;
    if (tl.first) {
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.o_empty[S], (ocount & 1) ^ 1, wd))) return false;
        ocount++;
    }
    issue_pv<D, SCORE>(sh, S, tl, tmem, dd);
    return true;
}

// All MMAs of stream S, in a fixed order.  At D = 64: S(r), then P V of tile r - 1
// (S(r) needs only that the softmax has read S(r - 1)).  At D = 128: P V of tile
// r - 1, then S(r) (S(r) overwrites P(r - 1)).  One code path serves both streams.
template <int D, int SCORE, int EXT>
__device__ __forceinline__ void mma_role(const FwdParams& p, Shared& sh, uint8_t* smem, uint32_t tmem, int S,
                                         int T0, int T1, Watchdog& wd, bool& bad)
{
    using C = Cfg<D, SCORE>;
    const int T = S == 0 ? T0 : T1;
    MmaDescs dd;
    dd.hi_k = (uint32_t)(sdesc_sw128(0, 16, 1024) >> 32);
    dd.hi_mn = (uint32_t)(sdesc_sw128(0, kBox, 1024) >> 32);
    dd.q = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_Q + S * C::TILE), 16, 1024);
    dd.k0 = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_K), 16, 1024);
    dd.v0 = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_V), kBox, 1024);
    CountWalk<EXT> w;
    w.init(p, S, bad);
    uint32_t qcount = 0, ocount = 0;
    MmaTile prev{0, false, false};
    bool ok = true;
    for (int r = 0; r <= T && ok; ++r) {
        MmaTile cur{0, false, false};
        if (r < T) {
            cur.seq = tile_seq(S, r, T0, T1);
            cur.first = w.t == 0;
            cur.last = w.t == w.n - 1;
        }
        if constexpr (C::SEP_P) {
            // S(r) and P V(r - 1) use different TMEM columns: issue whichever has
            // its operands first (polling; a short sleep when neither is ready).
            bool need_s = r < T, need_pv = r > 0;
            uint64_t t_idle = 0;
            while (need_s || need_pv) {
                bool progressed = false;
                if (need_s) {
                    const uint32_t ks = cur.seq % C::NK;
                    bool rdy = (r == 0 || mbar_test_wait(&sh.s_free[S], (r - 1) & 1)) &&
                               (!cur.first || mbar_test_wait(&sh.q_full[S], qcount & 1)) &&
                               mbar_test_wait(&sh.k_full[ks], (cur.seq / C::NK) & 1);
                    if (__all_sync(0xFFFFFFFFu, rdy)) {
                        if (cur.first) qcount++;
                        issue_s<D, SCORE>(sh, S, cur, tmem, dd);
                        need_s = false;
                        progressed = true;
                    }
                }
                if (need_pv) {
                    const uint32_t vs = prev.seq % C::NV;
                    bool rdy = mbar_test_wait(&sh.p_full[S], (r - 1) & 1) &&
                               mbar_test_wait(&sh.v_full[vs], (prev.seq / C::NV) & 1) &&
                               (!prev.first || mbar_test_wait(&sh.o_empty[S], (ocount & 1) ^ 1));
                    if (__all_sync(0xFFFFFFFFu, rdy)) {
                        if (prev.first) ocount++;
                        issue_pv<D, SCORE>(sh, S, prev, tmem, dd);
                        need_pv = false;
                        progressed = true;
                    }
                }
                if (progressed) {
                    t_idle = 0;
                } else {
                    const uint64_t now = globaltimer_ns();
                    if (t_idle == 0) t_idle = now;
                    else if (now - t_idle > wd.limit_ns) { wd.failed = true; ok = false; break; }
                    __nanosleep(32);
                }
            }
        } else {
            // P V(r - 1) first: S(r) overwrites P(r - 1)
            if (r > 0) ok = mma_pv<D, SCORE>(sh, S, prev, (uint32_t)(r - 1), ocount, tmem, dd, wd);
            if (ok && r < T) {
                const uint32_t ks = cur.seq % C::NK;
                if (cur.first) {
                    ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.q_full[S], qcount & 1, wd));
                    qcount++;
                }
                ok = ok && __all_sync(0xFFFFFFFFu, mbar_wait(&sh.k_full[ks], (cur.seq / C::NK) & 1, wd));
                if (ok) issue_s<D, SCORE>(sh, S, cur, tmem, dd);
            }
        }
        if (r < T) {
            prev = cur;
            w.advance(p, S, bad);
        }
    }
    // All issued MMAs complete before the CTA tears down TMEM.
    if (elect_one_sync()) umma_commit(&sh.drain[S]);
    __syncwarp();
    Watchdog dw{wd.failed ? 1000000ull : wd.limit_ns, false};
    const bool drained = __all_sync(0xFFFFFFFFu, mbar_wait(&sh.drain[S], 0, dw));
    if ((threadIdx.x & 31) == 0 && (wd.failed || !drained || !ok)) report(p, STATUS_TIMEOUT);
}

// ---------------------------------------------------------------- producers

struct LoadState {
    uint32_t seq, qcount[2];
    uint32_t k_issued, v_issued, b_issued;
};

// Load the current tile of stream S: the item's Q tile before its first tile, then
// K, the bias tile and V.  (One thread issues all of them, in this order; letting
// separate threads run the K and V rings independently measured slower: the far-
// ahead K copies delay the V copies that are needed first.)  Returns false if a
// wait for a free slot timed out.
template <int D, int SCORE, int EXT>
__device__ __forceinline__ bool produce_tile(const FwdParams& p, Shared& sh, uint8_t* smem, int S,
                                             TileWalk<EXT>& w, LoadState& st, Watchdog& wd, bool& bad)
{
    using C = Cfg<D, SCORE>;
    const Item& I = w.it;
    const int kb = w.kb;
    const int hk = I.hq / p.G;
    const uint32_t seq = st.seq;
    // K / V tile coordinates (rows, batch): the kv block of the batch, or its page
    int kv_row = kb * 128, kv_b = I.b;
    if ((EXT & kExtPage) && p.page_table) {
        int page = __ldg(p.page_table + (int64_t)I.b * p.pt_stride + kb);
        if (page < 0 || page >= p.num_pages) {
            bad = true;
            page = page < 0 ? 0 : p.num_pages - 1;
        }
        kv_row = 0;
        kv_b = page;
    }
    {
        if (w.t == 0) {
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.q_empty[S], (st.qcount[S] & 1) ^ 1, wd))) return false;
            uint8_t* dst = smem + C::OFF_Q + S * C::TILE;
            if (elect_one_sync()) {
                mbar_arrive_expect_tx(&sh.q_full[S], C::TILE);
#pragma unroll
                for (int c = 0; c < D / 64; ++c)
                    tma_load_4d(dst + c * kBox, &p.tm_q, &sh.q_full[S], c * 64, I.qb * 128, I.hq, I.b);
            }
            __syncwarp();
            st.qcount[S]++;
        }
        {
            const uint32_t slot = seq % C::NK;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.k_empty[slot], ((seq / C::NK) & 1) ^ 1, wd))) return false;
            uint8_t* dst = smem + C::OFF_K + slot * C::TILE;
            if (elect_one_sync()) {
                mbar_arrive_expect_tx(&sh.k_full[slot], C::TILE);
#pragma unroll
                for (int c = 0; c < D / 64; ++c)
                    tma_load_4d(dst + c * kBox, &p.tm_k, &sh.k_full[slot], c * 64, kv_row, hk, kv_b);
            }
            __syncwarp();
            st.k_issued++;
        }
        if constexpr (C::HAS_BIAS) {
            const uint32_t slot = seq % C::NB;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.b_empty[slot], ((seq / C::NB) & 1) ^ 1, wd))) return false;
            uint8_t* dst = smem + C::OFF_B + slot * C::BIAS_TILE;
            if (elect_one_sync()) {
                mbar_arrive_expect_tx(&sh.b_full[slot], C::BIAS_TILE);
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    tma_load_4d(dst + c * kBox, &p.tm_bias, &sh.b_full[slot], kb * 128 + c * 64, I.qb * 128,
                                p.bias_h_bcast ? 0 : I.hq, p.bias_b_bcast ? 0 : I.b);
            }
            __syncwarp();
            st.b_issued++;
        }
    }
    {
        const uint32_t slot = seq % C::NV;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.v_empty[slot], ((seq / C::NV) & 1) ^ 1, wd))) return false;
        uint8_t* dst = smem + C::OFF_V + slot * C::TILE;
        if (elect_one_sync()) {
            mbar_arrive_expect_tx(&sh.v_full[slot], C::TILE);
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
                tma_load_4d(dst + c * kBox, &p.tm_v, &sh.v_full[slot], c * 64, kv_row, hk, kv_b);
        }
        __syncwarp();
        st.v_issued++;
    }
    st.seq++;
    w.advance(p, S, bad);
    return true;
}

template <int D, int SCORE, int EXT>
__device__ __forceinline__ void producer_role(const FwdParams& p, Shared& sh, uint8_t* smem, int T0, int T1,
                                              Watchdog& wd, bool& bad)
{
    using C = Cfg<D, SCORE>;
    TileWalk<EXT> w[2];  // one cursor per stream (one code path serves both)
    w[0].init(p, 0, bad);
    w[1].init(p, 1, bad);
    LoadState st;
    st.seq = 0;
    st.qcount[0] = st.qcount[1] = 0;
    st.k_issued = st.v_issued = st.b_issued = 0;
    const int rounds = max(T0, T1);
    // watchdog self-test: wait for a phase that never completes; the wait gives up
    // after the limit and every later wait of this thread returns at once
    bool ok = !p.selftest_stall || __all_sync(0xFFFFFFFFu, mbar_wait(&sh.never, 0, wd));
    for (int r = 0; r < rounds && ok; ++r)
        for (int S = 0; S < 2 && ok; ++S)
            if (r < (S == 0 ? T0 : T1)) ok = produce_tile<D, SCORE, EXT>(p, sh, smem, S, w[S], st, wd, bad);
    if (wd.failed) {
        if ((threadIdx.x & 31) == 0) report(p, STATUS_TIMEOUT);
        // Let copies already in flight land before the CTA exits: wait (briefly,
        // bounded) for the latest issued phase of every slot.
        Watchdog dw{1000000ull, false};
        auto drain = [&](uint64_t* full, uint32_t issued, uint32_t n) {
            for (uint32_t i = 0; i < n && i < issued; ++i) {
                const uint32_t last = issued - 1 - i;
                dw.failed = false;
                mbar_wait(&full[last % n], (last / n) & 1, dw);
            }
        };
        drain(sh.k_full, st.k_issued, C::NK);
        drain(sh.v_full, st.v_issued, C::NV);
        if (C::NB > 0) drain(sh.b_full, st.b_issued, C::NB > 0 ? C::NB : 1);
        for (int s = 0; s < 2; ++s)
            if (st.qcount[s] > 0) {
                dw.failed = false;
                mbar_wait(&sh.q_full[s], (st.qcount[s] - 1) & 1, dw);
            }
    }
}

// ---------------------------------------------------------------- softmax

// One stream's softmax warpgroup: for every tile, S from TMEM -> score_mod and
// mask -> running maximum -> P = exp2(x' - m) in bf16 to TMEM, row sum in fp32;
// per item, the epilogue O / l and LSE.
template <int D, int SCORE, int EXT>
__device__ __forceinline__ void softmax_role(const FwdParams& p, Shared& sh, uint8_t* smem, uint32_t tmem, int s,
                                             int T0, int T1, Watchdog& wd, bool& bad)
{
    using C = Cfg<D, SCORE>;
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int wq = warp % 4;
    const int row = wq * 32 + lane;
    // turns (Cfg::TURNS): stream 1's pass r follows stream 0's pass r, and stream
    // 0's pass r follows stream 1's pass r - 1, while the other stream has one
    const int turn_lo = s == 0 ? 1 : 0;
    const int turn_hi = (s == 0 ? T1 : T0) + turn_lo;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + C::s_col(s);
    const uint32_t p_addr = tmem + lane_base + C::p_col(s);
    const uint32_t o_addr = tmem + lane_base + C::o_col(s);

    // Frame of the transformed scores u: the modified score in log2 units is
    // u * F + shift, and p = exp2(u * F + shift - m).
    float F;
    if constexpr (SCORE == FA_SCORE_NONE) F = p.scale_log2;
    else if constexpr (SCORE == FA_SCORE_BIAS) F = kLog2e;
    else if constexpr (C::HAS_CAP) F = p.softcap_out;  // u = tanh(s * scale / cap), tanh((s * scale + bias) / cap)
    else F = p.scale_log2;                                            // ALIBI: u = s, column term separate
    const uint64_t F2 = f2_pack(F, F);
    const float bias_scale = p.scale_log2 / kLog2e;  // BIAS: u = s * scale + bias (natural units)

    uint32_t ocount = 0;
    int r = 0;
    bool dead = false;
    ItemLoad nxt;
    item_issue<EXT>(p, item_index(s, 0, gridDim.x, blockIdx.x), nxt, true, SCORE == FA_SCORE_ALIBI, row);
    int k = 0;
    Item I;
    int f0 = 0, p0 = 0;
    float slope = 0.f;
    int32_t qdoc = 0;
    int64_t q = 0;
    int qpos = 0;
    bool q_in = false;
    // Advance to the stream's next non-empty item (empty ones get O = 0 and
    // LSE = -inf here) and start the reads of the one after it.
    auto next_item = [&]() -> bool {
        while (nxt.valid) {
            I = item_finish<EXT>(p, nxt, bad);
            f0 = nxt.f0_raw;
            p0 = nxt.p0_raw;
            slope = SCORE == FA_SCORE_ALIBI ? nxt.slope : 0.f;
            qdoc = nxt.qdoc;
            item_issue<EXT>(p, item_index(s, ++k, gridDim.x, blockIdx.x), nxt, true, SCORE == FA_SCORE_ALIBI, row);
            q = (int64_t)I.qb * 128 + row;
            q_in = q < p.q_len;
            qpos = (int)(q + p.mask.q_offset);  // the row's position (< 2^31)
            if (I.n > 0) return true;
            uint16_t* orow = p.o + I.b * p.o_stride_b + I.hq * p.o_stride_h + q * p.o_stride_s;
            float* lse_ptr = p.lse ? p.lse + ((int64_t)I.b * p.Hq + I.hq) * p.q_len + q : nullptr;
            if (q_in) {
#pragma unroll
                for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(orow)[c] = make_uint4(0, 0, 0, 0);
                if (lse_ptr) *lse_ptr = -INFINITY;
            }
        }
        return false;
    };
    bool more = next_item();
    while (more && !dead) {
        const int32_t* doc_row = p.mask.has_doc ? p.mask.doc_ids + (int64_t)I.b * p.mask.doc_stride : nullptr;
        const float slope2 = slope * kLog2e;  // ALiBi term per column, log2 units
        // The chunk bound below exceeds the true maximum by at most 31 |slope2|;
        // for slopes too steep for that, the column term is applied up front.
        const bool alibi_exact = SCORE == FA_SCORE_ALIBI && fabsf(slope2) * 31.f > 60.f;
        const float g_col = alibi_exact ? 0.f : slope2;  // column term left for the exponential pass
        const float hi_off = slope2 > 0.f ? 31.f : 0.f;   // chunk column with the largest term

        float m_run = -INFINITY;
        uint64_t l2 = f2_pack(0.f, 0.f);
        int kb = clamp_kb(first_kb_raw(I, f0, p0), p.nkv, bad);
        int kb_next_raw = I.n > 1 ? list_raw(I, 1) : 0;
        for (int t = 0; t < I.n; ++t, ++r) {
            const int64_t k0 = (int64_t)kb * 128;
            const bool partial = t < I.npart;
            const bool ragged = (kb == p.nkv - 1) && (p.kv_len % 128 != 0);

            // per-row mask words (partial tiles and the ragged last kv tile)
            uint32_t mw[4] = {0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu};
            if (partial) {
                uint32_t db[4] = {0u, 0u, 0u, 0u};
                if (p.mask.has_doc) doc_bits(doc_row, k0, p.kv_len, qdoc, db);
                row_mask_words(p.mask, qpos, k0, p.kv_len, db, mw);
            } else if (ragged) {
                const int lastc = clamp_col(p.kv_len - 1 - k0);
#pragma unroll
                for (int j = 0; j < 4; ++j) mw[j] = range_bits32(0, lastc, 32 * j);
            }
            const bool masked = partial || ragged;
            float shift = 0.f;
            if constexpr (SCORE == FA_SCORE_ALIBI) shift = slope2 * (float)((int)k0 - qpos);

            bool ok = mbar_wait(&sh.s_full[s], r & 1, wd);
            if (!__all_sync(0xFFFFFFFFu, ok)) { dead = true; break; }
            tc_fence_after();

            float x[128];
            {
                uint32_t raw[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + 32 * c, raw[c]);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int j = 0; j < 32; ++j) x[32 * c + j] = __uint_as_float(raw[c][j]);
            }
            if constexpr (C::SEP_P) {
                // S is in registers: the next tile's S may overwrite it
                tc_fence_before();
                mbar_arrive_warp(&sh.s_free[s]);
            }

            // score_mod: u in the frame above (ALiBi's column term is added in the
            // exponential pass; its row maximum is bounded per 32-column chunk)
            if constexpr (SCORE == FA_SCORE_ALIBI) {
                if (alibi_exact) {
                    const uint64_t js2 = f2_pack(slope / bias_scale, slope / bias_scale);
#pragma unroll
                    for (int j = 0; j < 128; j += 2)
                        f2_unpack(f2_fma(f2_pack((float)j, (float)(j + 1)), js2, f2_pack(x[j], x[j + 1])), x[j],
                                  x[j + 1]);
                }
            }
            if constexpr (C::HAS_BIAS) {
                // BIAS: u = s * scale + bias; BIAS_SOFTCAP: u = (s * scale + bias) / cap
                const uint32_t seq = tile_seq(s, r, T0, T1);
                const uint32_t slot = seq % C::NB;
                bool okb = mbar_wait(&sh.b_full[slot], (seq / C::NB) & 1, wd);
                if (!__all_sync(0xFFFFFFFFu, okb)) { dead = true; break; }
                const uint32_t brow = smem_u32(smem + C::OFF_B + slot * C::BIAS_TILE + row * 128);
                const float s_mul = SCORE == FA_SCORE_BIAS ? bias_scale : p.softcap_in;
                const float b_mul = SCORE == FA_SCORE_BIAS ? 1.0f : p.softcap_inv;
                const uint64_t sc2 = f2_pack(s_mul, s_mul), bm2 = f2_pack(b_mul, b_mul);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 v4 = lds128(brow + h * kBox + ((c ^ (row & 7)) * 16));
                        const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = h * 64 + c * 8 + 2 * e;
                            uint64_t bb = f2_pack(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xFFFF0000u));
                            if (SCORE == FA_SCORE_BIAS_SOFTCAP) bb = f2_mul(bb, bm2);
                            f2_unpack(f2_fma(f2_pack(x[j], x[j + 1]), sc2, bb), x[j], x[j + 1]);
                        }
                    }
                }
                mbar_arrive_warp(&sh.b_empty[slot]);
            }
            if constexpr (C::HAS_CAP) {
                if constexpr (SCORE == FA_SCORE_SOFTCAP) {
                    const uint64_t in2 = f2_pack(p.softcap_in, p.softcap_in);
#pragma unroll
                    for (int j = 0; j < 128; j += 2) f2_unpack(f2_mul(f2_pack(x[j], x[j + 1]), in2), x[j], x[j + 1]);
                }
                // u = tanh(y): the polynomial where every |y| of the warp's 32-column
                // chunk is small, else per element the exponential form beyond 0.625
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    bool far = false;
#pragma unroll
                    for (int j = 32 * c; j < 32 * c + 32; ++j) far |= fabsf(x[j]) > 0.625f;
                    if (__any_sync(0xFFFFFFFFu, far)) {
#pragma unroll
                        for (int j = 32 * c; j < 32 * c + 32; j += 2) {
                            float t0, t1;
                            f2_unpack(tanh_poly2(f2_pack(x[j], x[j + 1])), t0, t1);
                            if (fabsf(x[j]) > 0.625f) t0 = tanh_far(x[j]);
                            if (fabsf(x[j + 1]) > 0.625f) t1 = tanh_far(x[j + 1]);
                            x[j] = t0;
                            x[j + 1] = t1;
                        }
                    } else {
#pragma unroll
                        for (int j = 32 * c; j < 32 * c + 32; j += 2)
                            f2_unpack(tanh_poly2(f2_pack(x[j], x[j + 1])), x[j], x[j + 1]);
                    }
                }
            }

            if (masked) {
#pragma unroll
                for (int j = 0; j < 128; ++j)
                    if (!((mw[j >> 5] >> (j & 31)) & 1u)) x[j] = -INFINITY;
            }

            // maximum of each 32-column chunk c (one chain per chunk)
            float mx[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float* xc = x + 32 * c;
                float m0 = max3(xc[0], xc[1], xc[2]), m1 = max3(xc[3], xc[4], xc[5]);
#pragma unroll
                for (int j = 6; j < 30; j += 4) {
                    m0 = max3(m0, xc[j], xc[j + 1]);
                    m1 = max3(m1, xc[j + 2], xc[j + 3]);
                }
                mx[c] = max3(m0, m1, fmaxf(xc[30], xc[31]));
            }
            float m_tile;
            if constexpr (SCORE == FA_SCORE_ALIBI) {
                // upper bound of the row maximum: each chunk's largest column term
                // (at most 31 columns' worth of slope above the true maximum)
                m_tile = fmaxf(fmaxf(fmaf(mx[0], F, hi_off * g_col), fmaf(mx[1], F, (32.f + hi_off) * g_col)),
                               fmaxf(fmaf(mx[2], F, (64.f + hi_off) * g_col), fmaf(mx[3], F, (96.f + hi_off) * g_col))) +
                         shift;
            } else {
                m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * F + shift;
            }

            // running maximum: moved only when the tile maximum exceeds it by
            // more than the threshold (first tile: always set)
            float alpha = 1.0f;
            bool rescale = false;
            if (t == 0) {
                m_run = m_tile;
            } else if (m_tile > m_run + kRescaleThreshold) {
                alpha = ex2_approx(m_run - m_tile);
                m_run = m_tile;
                l2 = f2_mul(l2, f2_pack(alpha, alpha));
                rescale = true;
            }

            if (C::TURNS && r >= turn_lo && r < turn_hi) {
                // a timeout marks the watchdog, and the next wait ends the loop
                mbar_wait_lean(&sh.turn[s ^ 1][wq], (r - turn_lo) & 1, wd);
            }
            if constexpr (C::SEP_P) {
                // P(r - 1) has been consumed and O is stable once P V of tile r - 1 is done
                if (r > 0) {
                    ok = mbar_wait(&sh.p_free[s], (r - 1) & 1, wd);
                    if (!__all_sync(0xFFFFFFFFu, ok)) { dead = true; break; }
                    tc_fence_after();
                }
            }
            const float m_use = m_run == -INFINITY ? 0.f : m_run;
            const float b_row = shift - m_use;
            uint64_t la = f2_pack(0.f, 0.f), lb = la;
            exp_pass<SCORE == FA_SCORE_ALIBI>(x, F2, b_row, g_col, p_addr, la, lb);
            if (C::TURNS) mbar_arrive_warp(&sh.turn[s][wq]);
            l2 = f2_add(l2, f2_add(la, lb));
            // next tile's kv block (read one tile ahead)
            if (t + 1 < I.n) {
                kb = clamp_kb(kb_next_raw, p.nkv, bad);
                kb_next_raw = t + 2 < I.n ? list_raw(I, t + 2) : 0;
            }
            if (__any_sync(0xFFFFFFFFu, rescale)) {
                // O is stable here: P V of the previous tile is done (at D = 64
                // waited for above; at D = 128 S of this tile was issued after it),
                // and this tile's P V waits for p_full.
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(o_addr + 32 * c, ov);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
                    tmem_st32(o_addr + 32 * c, ov);
                }
            }

            tmem_st_wait();
            tc_fence_before();
            mbar_arrive_warp(&sh.p_full[s]);
        }
        if (dead) break;

        // epilogue: O / l -> bf16, LSE = ln(2) * (m + log2 l).  The next item's
        // reads and index arithmetic go first: they overlap the last P V.
        float l_lo, l_hi;
        f2_unpack(l2, l_lo, l_hi);
        const float l_run = l_lo + l_hi;
        uint16_t* orow = p.o + I.b * p.o_stride_b + I.hq * p.o_stride_h + q * p.o_stride_s;
        float* lse_ptr = p.lse ? p.lse + ((int64_t)I.b * p.Hq + I.hq) * p.q_len + q : nullptr;
        const bool row_in = q_in;
        more = next_item();
        bool ok = mbar_wait(&sh.o_full[s], ocount & 1, wd);
        if (!__all_sync(0xFFFFFFFFu, ok)) { dead = true; break; }
        ocount++;
        tc_fence_after();
        // no admitted position in the whole row: O = 0, LSE = -inf
        const bool empty_row = m_run == -INFINITY;
        const float inv_l = (l_run > 0.f && !empty_row) ? 1.0f / l_run : 0.f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(o_addr + 32 * c, ov);
            tmem_ld_wait();
            if (c == D / 32 - 1) {
                tc_fence_before();
                mbar_arrive_warp(&sh.o_empty[s]);
            }
            if (row_in) {
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    pk[j] = pack_bf16x2(__uint_as_float(ov[2 * j]) * inv_l, __uint_as_float(ov[2 * j + 1]) * inv_l);
                uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
                for (int j = 0; j < 4; ++j) dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            }
        }
        if (row_in && lse_ptr) *lse_ptr = (l_run > 0.f && !empty_row) ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
    }
    if (dead || wd.failed) {
        if (lane == 0) report(p, STATUS_TIMEOUT);
    }
}

// ---------------------------------------------------------------- kernel

template <int D, int SCORE, int EXT>
__global__ void __launch_bounds__(kThreads, 1) flex_fwd_kernel(const __grid_constant__ FwdParams p)
{
    using C = Cfg<D, SCORE>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ Shared sh;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (warp == kMmaWarp0) {
        tmem_alloc(&sh.tmem_base, 512);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh.q_full[s], 1);
            mbar_init(&sh.q_empty[s], 1);
            mbar_init(&sh.s_full[s], 1);
            mbar_init(&sh.s_free[s], 4);
            mbar_init(&sh.p_full[s], 4);
            mbar_init(&sh.p_free[s], 1);
            mbar_init(&sh.o_full[s], 1);
            mbar_init(&sh.o_empty[s], 4);
            mbar_init(&sh.drain[s], 1);
        }
        mbar_init(&sh.never, 1);
        for (int s = 0; s < 2; ++s)
            for (int w = 0; w < 4; ++w) mbar_init(&sh.turn[s][w], 1);
        for (int i = 0; i < C::NK; ++i) { mbar_init(&sh.k_full[i], 1); mbar_init(&sh.k_empty[i], 1); }
        for (int i = 0; i < C::NV; ++i) { mbar_init(&sh.v_full[i], 1); mbar_init(&sh.v_empty[i], 1); }
        for (int i = 0; i < C::NB; ++i) { mbar_init(&sh.b_full[i], 1); mbar_init(&sh.b_empty[i], 4); }
        mbar_fence_init();
    }
    if (warp == kLoadWarp && lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_v);
        if (C::HAS_BIAS) tma_prefetch_desc(&p.tm_bias);
    }
    // longest-first order of the BlockMask rows (the K ring is scratch until the
    // pipeline starts)
    if constexpr ((EXT & kExtRank) != 0) rank_rows(p, reinterpret_cast<uint32_t*>(smem + C::OFF_K));
    if (warp == kMmaWarp1) {
        // tiles of each stream: the lanes read 32 items' counts at a time
        bool bad_count = false;
        for (int s = 0; s < 2; ++s) {
            int total = 0;
            for (int k0 = 0; item_index(s, k0, gridDim.x, blockIdx.x) < p.num_items; k0 += 32) {
                int n = 0;
                ItemLoad L;
                item_issue<EXT>(p, item_index(s, k0 + lane, gridDim.x, blockIdx.x), L, false, false, -1);
                if (L.valid) n = item_finish<EXT>(p, L, bad_count).n;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xFFFFFFFFu, n, o);
                total += n;
            }
            if (lane == 0) sh.total[s] = total;
        }
        const bool any_bad = __any_sync(0xFFFFFFFFu, bad_count);
        if (lane == 0) sh.bad = any_bad ? 1 : 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const int T0 = sh.total[0], T1 = sh.total[1];

    Watchdog wd{p.watchdog_ns, false};
    bool bad = false;

    if (warp >= 8) {
        regs_dec<kOtherRegs>();
        // whole warps run these roles; one elected lane issues the copies and MMAs
        if (warp == kLoadWarp) producer_role<D, SCORE, EXT>(p, sh, smem, T0, T1, wd, bad);
        else if (warp == kMmaWarp0 || warp == kMmaWarp1)
            mma_role<D, SCORE, EXT>(p, sh, smem, tmem, warp == kMmaWarp0 ? 0 : 1, T0, T1, wd, bad);
        __syncwarp();
    } else {
        regs_inc<kSoftmaxRegs>();
        softmax_role<D, SCORE, EXT>(p, sh, smem, tmem, warp / 4, T0, T1, wd, bad);
    }

    if (bad || (threadIdx.x == 0 && sh.bad)) report(p, STATUS_BAD_BLOCKMASK);

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp0) tmem_dealloc(tmem, 512);
}

// Kernel attributes are per context: set them once for every context the
// variant is launched in (a second device, or the same device after
// cudaDeviceReset, gets its own set-up).
template <int D, int SCORE, int EXT>
cudaError_t configure_variant()
{
    static std::mutex mu;
    static std::vector<CtxKey> done;
    auto kern = flex_fwd_kernel<D, SCORE, EXT>;
    CtxKey key;
    std::lock_guard<std::mutex> lock(mu);
    if (current_ctx(&key))
        for (const CtxKey& k : done)
            if (k == key) return cudaSuccess;
    // The register split assumes the launch allocation; refuse anything else
    // rather than launch a kernel whose setmaxnreg.inc could never be served.
    cudaFuncAttributes fa_attr;
    cudaError_t e = cudaFuncGetAttributes(&fa_attr, kern);
    if (e != cudaSuccess) return e;
    if (fa_attr.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D, SCORE>::SMEM);
    if (e != cudaSuccess) return e;
    if (current_ctx(&key)) done.push_back(key);
    return cudaSuccess;
}

template <int D, int SCORE, int EXT>
cudaError_t launch_variant(const FwdParams& p, int grid, cudaStream_t stream)
{
    static_assert(Cfg<D, SCORE>::NK <= kMaxSlots && Cfg<D, SCORE>::NV <= kMaxSlots && Cfg<D, SCORE>::NB <= 3,
                  "ring deeper than its barriers");
    static_assert(Cfg<D, SCORE>::SMEM + sizeof(Shared) + sizeof(s_row_order) <= 232448,
                  "shared memory beyond 227 KB per CTA");
    cudaError_t e = configure_variant<D, SCORE, EXT>();
    if (e != cudaSuccess) return e;
    // (A programmatic dependent launch after the BlockMask kernel was measured:
    // it gained 3 us on the causal+ALiBi step and lost 78 us on the document
    // step, so the kernel is launched in plain stream order.)
    flex_fwd_kernel<D, SCORE, EXT><<<grid, kThreads, Cfg<D, SCORE>::SMEM, stream>>>(p);
    return cudaGetLastError();
}

// Every (D, score_kind) instance of the kernel with EXT = FWD_EXT.
cudaError_t launch_instances(const FwdParams& p, int D, int score_kind, int grid, cudaStream_t stream)
{
#define FA_LAUNCH_CASE(DD, SS) \
    if (D == DD && score_kind == SS) return launch_variant<DD, SS, FWD_EXT>(p, grid, stream);
    FA_LAUNCH_CASE(64, FA_SCORE_NONE) FA_LAUNCH_CASE(64, FA_SCORE_ALIBI) FA_LAUNCH_CASE(64, FA_SCORE_SOFTCAP)
    FA_LAUNCH_CASE(64, FA_SCORE_BIAS) FA_LAUNCH_CASE(128, FA_SCORE_NONE) FA_LAUNCH_CASE(128, FA_SCORE_ALIBI)
    FA_LAUNCH_CASE(128, FA_SCORE_SOFTCAP) FA_LAUNCH_CASE(128, FA_SCORE_BIAS)
    FA_LAUNCH_CASE(64, FA_SCORE_BIAS_SOFTCAP) FA_LAUNCH_CASE(128, FA_SCORE_BIAS_SOFTCAP)
#undef FA_LAUNCH_CASE
    return cudaErrorInvalidValue;
}

} // namespace

#if FWD_EXT == 3  // kExtRank | kExtPage
cudaError_t launch_flex_forward_ext(const FwdParams& p, int D, int score_kind, int grid, cudaStream_t stream)
{
    return launch_instances(p, D, score_kind, grid, stream);
}
#elif FWD_EXT == 2  // kExtPage
cudaError_t launch_flex_forward_paged(const FwdParams& p, int D, int score_kind, int grid, cudaStream_t stream)
{
    return launch_instances(p, D, score_kind, grid, stream);
}
#else
cudaError_t launch_flex_forward_base(const FwdParams& p, int D, int score_kind, int grid, cudaStream_t stream)
{
    return launch_instances(p, D, score_kind, grid, stream);
}

int flex_forward_smem_bytes(int D, int score_kind)
{
#define FA_SMEM_CASE(DD, SS) \
    if (D == DD && score_kind == SS) return Cfg<DD, SS>::SMEM;
    FA_SMEM_CASE(64, FA_SCORE_NONE) FA_SMEM_CASE(64, FA_SCORE_ALIBI) FA_SMEM_CASE(64, FA_SCORE_SOFTCAP)
    FA_SMEM_CASE(64, FA_SCORE_BIAS) FA_SMEM_CASE(128, FA_SCORE_NONE) FA_SMEM_CASE(128, FA_SCORE_ALIBI)
    FA_SMEM_CASE(128, FA_SCORE_SOFTCAP) FA_SMEM_CASE(128, FA_SCORE_BIAS) FA_SMEM_CASE(64, FA_SCORE_BIAS_SOFTCAP)
    FA_SMEM_CASE(128, FA_SCORE_BIAS_SOFTCAP)
#undef FA_SMEM_CASE
    return -1;
}

// Three sets of instances: masks with a DOCUMENT leaf run the ones with the
// longest-first ranking of BlockMask rows (and paged K / V) compiled in, other
// paged calls the ones with only the page-table read, every other call the base
// instances, whose code carries neither.
cudaError_t launch_flex_forward(const FwdParams& p, int D, int score_kind, int ext, int grid, cudaStream_t stream)
{
    if (ext & kExtRank) return launch_flex_forward_ext(p, D, score_kind, grid, stream);
    if (ext & kExtPage) return launch_flex_forward_paged(p, D, score_kind, grid, stream);
    return launch_flex_forward_base(p, D, score_kind, grid, stream);
}
#endif

} // namespace fa
