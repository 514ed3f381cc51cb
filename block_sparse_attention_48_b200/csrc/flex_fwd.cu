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
//   warp  8    MMA issue (one thread): S = Q K^T and O += P V with tcgen05.mma
//   warp  9    TMA producer (one thread): Q, K, V and bias tiles
//   warp  10   counts each stream's tiles at start-up, then idles
//   warp  11   idle (completes the third warpgroup for register reallocation)
// The softmax warpgroups take registers from the third warpgroup (setmaxnreg):
// launched at 168 per thread, they run at 200 and the third at 104.
//
// Each CTA runs two independent streams of work items (b, hq, query block), so
// that the tensor core computes one stream's MMAs while the other stream's
// softmax runs.  Accumulators live in tensor memory (TMEM):
//   S_s  columns [128 s, 128 s + 128)    fp32 scores of stream s
//   P_s  aliased on S_s columns [0, 64)  bf16 probabilities, A operand of P V
//   O_s  columns [256 + D s, 256 + D s + D)
// K and V tiles stream through shared-memory rings shared by both streams and
// filled in a fixed interleaved order (round r: stream 0's r-th tile, then
// stream 1's), so every role can compute which slot holds which tile.  The MMA
// warp may serve the two streams in either order; each stream's tiles are
// consumed in order.  Every role reads the BlockMask one step ahead of use.
//
// O is rescaled only when a row maximum grows by more than 2^8 (log2 domain):
// the final O / l and LSE are the same for any choice of the running maximum.
#include <cuda_runtime.h>

#include "flex_fwd.cuh"
#include "ptx.cuh"

namespace fa {

namespace {

constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
// registers per thread of the softmax warpgroups and of the third warpgroup
template <int D, int SCORE> struct RegSplit {
    static constexpr int softmax = 200;
    static constexpr int other = 104;
    static_assert(2 * 128 * softmax + 128 * other <= kThreads * kLaunchRegs,
                  "register split exceeds the launch allocation");
};
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kCountWarp = 10;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kBox = 16384;  // bytes of one 128-row x 64-column bf16 TMA box
// Of every three groups of four scores, the pairs marked here take the
// polynomial exponential in full tiles (the rest use MUFU ex2).
__device__ constexpr bool kPolyPair[3] = {true, true, false};

template <int D, int SCORE>
struct Cfg {
    static constexpr int TILE = 128 * D * 2;
    static constexpr int NK = D == 64 ? 3 : 2;
    static constexpr int NV = D == 64 ? 3 : 2;
    static constexpr int NB = SCORE == FA_SCORE_BIAS ? (D == 64 ? 2 : 1) : 0;
    static constexpr int BIAS_TILE = 128 * 128 * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 2 * TILE;
    static constexpr int OFF_V = OFF_K + NK * TILE;
    static constexpr int OFF_B = OFF_V + NV * TILE;
    static constexpr int SMEM = OFF_B + NB * BIAS_TILE + 1024;
    static constexpr uint32_t O_COL0 = 256;
};

struct __align__(16) Shared {
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[3], k_empty[3];
    uint64_t v_full[3], v_empty[3];
    uint64_t b_full[2], b_empty[2];
    uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int total[2];                      // tiles of each stream
    int bad;  // a count read by the counting warp was out of range
};

// A work item: query block qb of (b, hq), and its BlockMask row.
struct Item {
    int b, hq, qb;
    int nfull, n;  // tiles: [0, nfull) from the full list, [nfull, n) from the partial list
    const int32_t* full_list;
    const int32_t* part_list;
};

// Work item of stream s, k-th in that stream.  Items are numbered with the
// last query block first (most kv blocks under causal-like masks); rounds of
// 2 * grid items are dealt to CTAs in alternating (snake) order.
__device__ __forceinline__ long long item_index(int s, int k, int grid, int cta)
{
    int pos = (k & 1) ? 2 * (grid - 1 - cta) + s : 2 * cta + s;
    return (long long)k * 2 * grid + pos;
}

// BlockMask row of an item (b, hq, qb), broadcast over B / H extents of 1.
__device__ __forceinline__ int64_t item_row(const FwdParams& p, int b, int hq, int qb)
{
    const int mb = p.bm_B == 1 ? 0 : b;
    const int mh = p.bm_H == 1 ? 0 : hq;
    return ((int64_t)mb * p.bm_H + mh) * p.nq + qb;
}

// Coordinates and BlockMask lists of work item idx (counts left unset).
__device__ __forceinline__ Item item_at(const FwdParams& p, int idx)
{
    Item it;
    const int bh_count = p.B * p.Hq;
    const int qb_rank = idx / bh_count;
    const int bh = idx - qb_rank * bh_count;
    it.qb = p.nq - 1 - qb_rank;
    it.b = bh / p.Hq;
    it.hq = bh - it.b * p.Hq;
    const int64_t r = item_row(p, it.b, it.hq, it.qb);
    it.full_list = p.has_full ? p.full_idx + r * p.nkv : nullptr;
    it.part_list = p.kv_idx + r * p.nkv;
    it.nfull = it.n = 0;
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

__device__ __forceinline__ void item_issue(const FwdParams& p, long long idx, ItemLoad& L, bool want_first,
                                           bool want_slope, int row)
{
    L.valid = idx < p.num_items;
    L.f0_raw = L.p0_raw = 0;
    if (!L.valid) return;
    L.idx = (int)idx;
    const Item it = item_at(p, L.idx);
    const int64_t r = item_row(p, it.b, it.hq, it.qb);
    L.nf_raw = p.has_full ? __ldg(p.full_num + r) : 0;
    L.np_raw = __ldg(p.kv_num + r);
    if (want_first && p.nkv > 0) {
        L.f0_raw = p.has_full ? __ldg(it.full_list) : 0;
        L.p0_raw = __ldg(it.part_list);
    }
    if (want_slope) L.slope = __ldg(p.slopes + it.hq);
    if (row >= 0 && p.mask.has_doc) {
        const int64_t q = (int64_t)it.qb * 128 + row;
        L.qdoc = q < p.q_len ? __ldg(p.mask.doc_ids + (int64_t)it.b * p.mask.doc_stride + q) : INT32_MIN;
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

__device__ __forceinline__ Item item_finish(const FwdParams& p, const ItemLoad& L, bool& bad)
{
    Item it = item_at(p, L.idx);
    it.nfull = clamp_count(L.nf_raw, p.nkv, bad);
    it.n = it.nfull + clamp_count(L.np_raw, p.nkv, bad);
    return it;
}

// Raw (unvalidated) kv block of tile t of an item.
__device__ __forceinline__ int list_raw(const Item& it, int t)
{
    return t < it.nfull ? __ldg(it.full_list + t) : __ldg(it.part_list + (t - it.nfull));
}

// Position of stream s's r-th tile in the interleaved production order.
__device__ __forceinline__ uint32_t tile_seq(int s, int r, int T0, int T1)
{
    return (uint32_t)(min(r, T0) + min(r, T1) + ((s == 1 && r < T0) ? 1 : 0));
}

// Cursor over the tiles of one stream's non-empty items.  The next item's
// counts and the next tile's kv block are read one step ahead.
template <bool KB>
struct TileWalk {
    Item it;
    int t;
    int kb;           // kv block of tile t (KB)
    int kb_next_raw;  // kv block of tile t + 1, unvalidated (KB)
    int k;            // stream position of the next item to read
    ItemLoad nx;
    bool done;

    __device__ __forceinline__ void fetch(const FwdParams& p, int s)
    {
        item_issue(p, item_index(s, k++, gridDim.x, blockIdx.x), nx, KB, false, -1);
    }

    __device__ __forceinline__ void next_item(const FwdParams& p, int s, bool& bad)
    {
        for (;;) {
            if (!nx.valid) {
                done = true;
                return;
            }
            it = item_finish(p, nx, bad);
            if (it.n > 0) break;
            fetch(p, s);
        }
        t = 0;
        if (KB) kb = clamp_kb(it.nfull > 0 ? nx.f0_raw : nx.p0_raw, p.nkv, bad);
        fetch(p, s);
        if (KB) kb_next_raw = it.n > 1 ? list_raw(it, 1) : 0;
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
        if (KB) {
            kb = clamp_kb(kb_next_raw, p.nkv, bad);
            kb_next_raw = t + 1 < it.n ? list_raw(it, t + 1) : 0;
        }
    }
};

__device__ __forceinline__ void report(const FwdParams& p, int bits)
{
    atomicOr(p.status, bits);
}

// Odd polynomial for tanh on |y| <= 0.625 (least-squares fit of (tanh(y) - y) / y^3
// in u = y^2 on Chebyshev nodes, weighted by y^3; max abs error 4e-8 in fp32),
// evaluated on packed pairs; and 1 - 2 / (e^(2|y|) + 1) beyond.
__device__ __forceinline__ uint64_t tanh_poly2(uint64_t y)
{
    const uint64_t u = f2_mul(y, y);
    uint64_t p = f2_pack(-0.005561366677284241f, -0.005561366677284241f);
    p = f2_fma(p, u, f2_pack(0.020492956042289734f, 0.020492956042289734f));
    p = f2_fma(p, u, f2_pack(-0.05368727073073387f, -0.05368727073073387f));
    p = f2_fma(p, u, f2_pack(0.13330671191215515f, 0.13330671191215515f));
    p = f2_fma(p, u, f2_pack(-0.33333244919776917f, -0.33333244919776917f));
    return f2_fma(f2_mul(y, u), p, y);
}

// 2^x on packed pairs with FMA-pipe instructions only, for x <= 8 (arguments
// below -120 are raised to -120, whose 2^x is negligible against a row sum >= 1).
// Cody-Waite style split x = n + f, n = round(x) via the 1.5 * 2^23 shift, f in
// [-1/2, 1/2]; 2^f from a degree-4 polynomial (least-squares fit to 2^f on
// Chebyshev nodes with relative weights, refined toward equal ripple; max
// relative error 2.7e-6 in fp32); 2^n applied by adding n to the exponent field.
__device__ __forceinline__ void exp2_poly2(uint64_t x2, float& r0, float& r1)
{
    float x0, x1;
    f2_unpack(x2, x0, x1);
    x0 = fmaxf(x0, -120.0f);
    x1 = fmaxf(x1, -120.0f);
    const uint64_t xc = f2_pack(x0, x1);
    const uint64_t t = f2_add(xc, f2_pack(12582912.0f, 12582912.0f));
    const uint64_t fn = f2_add(t, f2_pack(-12582912.0f, -12582912.0f));
    const uint64_t f = f2_fma(fn, f2_pack(-1.0f, -1.0f), xc);
    uint64_t p = f2_pack(0.009570073336362839f, 0.009570073336362839f);
    p = f2_fma(p, f, f2_pack(0.05591785907745361f, 0.05591785907745361f));
    p = f2_fma(p, f, f2_pack(0.2402474582195282f, 0.2402474582195282f));
    p = f2_fma(p, f, f2_pack(0.6931217908859253f, 0.6931217908859253f));
    p = f2_fma(p, f, f2_pack(0.9999992847442627f, 0.9999992847442627f));
    float p0, p1, t0, t1;
    f2_unpack(p, p0, p1);
    f2_unpack(t, t0, t1);
    r0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
    r1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

__device__ __forceinline__ float tanh_far(float y)
{
    const float a = fabsf(y);
    const float e = ex2_approx(2.0f * kLog2e * a);
    const float t = 1.0f - __fdividef(2.0f, e + 1.0f);
    return copysignf(t, y);
}

// ---------------------------------------------------------------- MMA issue

// Shared-memory descriptors of every operand buffer, built once.  All K-major
// ones share one high word, the MN-major ones another; a K step of an MMA adds a
// small constant to the start-address field in the low word.
struct MmaDescs {
    uint32_t q[2];  // Q tile of stream 0 / 1 (K-major)
    uint32_t k[3];  // K ring slots (K-major)
    uint32_t v[3];  // V ring slots (MN-major, 64-column chunks 16 KB apart)
    uint32_t hi_k, hi_mn;
};

__device__ __forceinline__ uint64_t desc64(uint32_t hi, uint32_t lo)
{
    return ((uint64_t)hi << 32) | lo;
}

// The MMA warp needs only each item's tile count: a slim cursor with the next
// item's counts read one item ahead.
struct CountWalk {
    int n, t;       // tiles of the current item, tile within it
    int k;          // stream position of the next item to read
    int nf_raw, np_raw;
    bool nx_valid;

    __device__ __forceinline__ void fetch(const FwdParams& p, int s)
    {
        const long long idx = item_index(s, k++, gridDim.x, blockIdx.x);
        nx_valid = idx < p.num_items;
        if (!nx_valid) return;
        const int i = (int)idx;
        const int bh_count = p.B * p.Hq;
        const int qb_rank = i / bh_count;
        const int bh = i - qb_rank * bh_count;
        const int b = bh / p.Hq;
        const int64_t r = item_row(p, b, bh - b * p.Hq, p.nq - 1 - qb_rank);
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

struct MmaStream {
    CountWalk w;
    int r;         // tiles of this stream whose P V has been issued
    bool need_pv;  // S of tile r issued, its P V not yet
    uint32_t qcount, pcount, ocount;
    uint64_t* block_bar;  // barrier phase the stream waits for, when blocked
    uint32_t block_par;
};

// Issue the next MMA group of stream S if its operands are ready: S = Q K^T of
// tile r, or O (+)= P V of tile r.  Returns whether anything was issued.
template <int D, int SCORE, int S>
__device__ __forceinline__ bool mma_try(const FwdParams& p, Shared& sh, MmaStream& ms, int T, int T0, int T1,
                                        uint32_t tmem, const MmaDescs& dd, bool& bad)
{
    using C = Cfg<D, SCORE>;
    if (ms.r >= T) return false;
    const uint32_t seq = tile_seq(S, ms.r, T0, T1);
    const bool first = ms.w.t == 0;
    const bool last = ms.w.t == ms.w.n - 1;
    auto ready = [&](uint64_t* bar, uint32_t par) {
        if (mbar_test_wait(bar, par)) return true;
        ms.block_bar = bar;
        ms.block_par = par;
        return false;
    };
    if (!ms.need_pv) {
        const uint32_t slot = seq % C::NK;
        if (first && !ready(&sh.q_full[S], ms.qcount & 1)) return false;
        if (!ready(&sh.k_full[slot], (seq / C::NK) & 1)) return false;
        tc_fence_after();
        constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
        const uint32_t qd = dd.q[S];
        const uint32_t kd = slot == 0 ? dd.k[0] : (slot == 1 ? dd.k[1] : dd.k[2]);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
            // start address advances 32 bytes per K step inside a 128-byte row, 16 KB per 64 columns
            const uint32_t off = (uint32_t)(((k / 4) * kBox + (k % 4) * 32) >> 4);
            umma_ss(tmem + 128 * S, desc64(dd.hi_k, qd + off), desc64(dd.hi_k, kd + off), idesc_s, k > 0);
        }
        umma_commit(&sh.k_empty[slot]);
        umma_commit(&sh.s_full[S]);
        if (last) umma_commit(&sh.q_empty[S]);
        if (first) ms.qcount++;
        ms.need_pv = true;
        return true;
    }
    const uint32_t slot = seq % C::NV;
    if (!ready(&sh.p_full[S], ms.pcount & 1)) return false;
    if (!ready(&sh.v_full[slot], (seq / C::NV) & 1)) return false;
    if (first && !ready(&sh.o_empty[S], (ms.ocount & 1) ^ 1)) return false;
    tc_fence_after();
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
    const uint32_t vd = slot == 0 ? dd.v[0] : (slot == 1 ? dd.v[1] : dd.v[2]);
    const uint32_t o_col = tmem + C::O_COL0 + D * S;
#pragma unroll
    for (int k = 0; k < 8; ++k)  // 16 kv rows (2 KB) per K step
        umma_ts(o_col, tmem + 128 * S + 8 * k, desc64(dd.hi_mn, vd + (uint32_t)((k * 2048) >> 4)), idesc_o,
                (!first || k > 0) ? 1u : 0u);
    umma_commit(&sh.v_empty[slot]);
    if (last) umma_commit(&sh.o_full[S]);
    ms.pcount++;
    if (first) ms.ocount++;
    ms.need_pv = false;
    ms.r++;
    ms.w.advance(p, S, bad);
    return true;
}

// ---------------------------------------------------------------- producer

struct LoadState {
    uint32_t seq, qcount[2];
    uint32_t k_issued, v_issued, b_issued;
};

// Load the current tile of stream S (and its item's Q tile first, on the item's
// first tile).  Returns false if a wait for a free slot timed out.
template <int D, int SCORE, int S>
__device__ __forceinline__ bool produce_tile(const FwdParams& p, Shared& sh, uint8_t* smem, TileWalk<true>& w,
                                             LoadState& st, Watchdog& wd, bool& bad)
{
    using C = Cfg<D, SCORE>;
    const Item& I = w.it;
    if (w.t == 0) {
        if (!mbar_wait(&sh.q_empty[S], (st.qcount[S] & 1) ^ 1, wd)) return false;
        mbar_arrive_expect_tx(&sh.q_full[S], C::TILE);
        uint8_t* dst = smem + C::OFF_Q + S * C::TILE;
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
            tma_load_4d(dst + c * kBox, &p.tm_q, &sh.q_full[S], c * 64, I.qb * 128, I.hq, I.b);
        st.qcount[S]++;
    }
    const int kb = w.kb;
    const int hk = I.hq / p.G;
    const uint32_t seq = st.seq;
    {
        const uint32_t slot = seq % C::NK;
        if (!mbar_wait(&sh.k_empty[slot], ((seq / C::NK) & 1) ^ 1, wd)) return false;
        mbar_arrive_expect_tx(&sh.k_full[slot], C::TILE);
        uint8_t* dst = smem + C::OFF_K + slot * C::TILE;
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
            tma_load_4d(dst + c * kBox, &p.tm_k, &sh.k_full[slot], c * 64, kb * 128, hk, I.b);
        st.k_issued++;
    }
    if constexpr (SCORE == FA_SCORE_BIAS) {
        const uint32_t slot = seq % C::NB;
        if (!mbar_wait(&sh.b_empty[slot], ((seq / C::NB) & 1) ^ 1, wd)) return false;
        mbar_arrive_expect_tx(&sh.b_full[slot], C::BIAS_TILE);
        uint8_t* dst = smem + C::OFF_B + slot * C::BIAS_TILE;
#pragma unroll
        for (int c = 0; c < 2; ++c)
            tma_load_4d(dst + c * kBox, &p.tm_bias, &sh.b_full[slot], kb * 128 + c * 64, I.qb * 128, I.hq, I.b);
        st.b_issued++;
    }
    {
        const uint32_t slot = seq % C::NV;
        if (!mbar_wait(&sh.v_empty[slot], ((seq / C::NV) & 1) ^ 1, wd)) return false;
        mbar_arrive_expect_tx(&sh.v_full[slot], C::TILE);
        uint8_t* dst = smem + C::OFF_V + slot * C::TILE;
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
            tma_load_4d(dst + c * kBox, &p.tm_v, &sh.v_full[slot], c * 64, kb * 128, hk, I.b);
        st.v_issued++;
    }
    st.seq++;
    w.advance(p, S, bad);
    return true;
}

// ---------------------------------------------------------------- kernel

template <int D, int SCORE>
__global__ void __launch_bounds__(kThreads, 1) flex_fwd_kernel(const __grid_constant__ FwdParams p)
{
    using C = Cfg<D, SCORE>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ Shared sh;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (warp == kMmaWarp) {
        tmem_alloc(&sh.tmem_base, 512);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh.q_full[s], 1);
            mbar_init(&sh.q_empty[s], 1);
            mbar_init(&sh.s_full[s], 1);
            mbar_init(&sh.p_full[s], 128);
            mbar_init(&sh.o_full[s], 1);
            mbar_init(&sh.o_empty[s], 128);
        }
        for (int i = 0; i < C::NK; ++i) { mbar_init(&sh.k_full[i], 1); mbar_init(&sh.k_empty[i], 1); }
        for (int i = 0; i < C::NV; ++i) { mbar_init(&sh.v_full[i], 1); mbar_init(&sh.v_empty[i], 1); }
        for (int i = 0; i < C::NB; ++i) { mbar_init(&sh.b_full[i], 1); mbar_init(&sh.b_empty[i], 128); }
        mbar_init(&sh.drain, 1);
        mbar_fence_init();
    }
    if (warp == kLoadWarp && lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_v);
        if (SCORE == FA_SCORE_BIAS) tma_prefetch_desc(&p.tm_bias);
    }
    if (warp == kCountWarp) {
        // tiles of each stream: the lanes read 32 items' counts at a time
        bool bad_count = false;
        for (int s = 0; s < 2; ++s) {
            int total = 0;
            for (int k0 = 0; item_index(s, k0, gridDim.x, blockIdx.x) < p.num_items; k0 += 32) {
                int n = 0;
                ItemLoad L;
                item_issue(p, item_index(s, k0 + lane, gridDim.x, blockIdx.x), L, false, false, -1);
                if (L.valid) n = item_finish(p, L, bad_count).n;
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
        regs_dec<RegSplit<D, SCORE>::other>();
        if (warp == kLoadWarp) {
            // -------------------------------------------------------- producer
            if (lane == 0) {
                TileWalk<true> w0, w1;
                w0.init(p, 0, bad);
                w1.init(p, 1, bad);
                LoadState st;
                st.seq = 0;
                st.qcount[0] = st.qcount[1] = 0;
                st.k_issued = st.v_issued = st.b_issued = 0;
                const int rounds = max(T0, T1);
                for (int r = 0; r < rounds; ++r) {
                    if (r < T0 && !produce_tile<D, SCORE, 0>(p, sh, smem, w0, st, wd, bad)) break;
                    if (r < T1 && !produce_tile<D, SCORE, 1>(p, sh, smem, w1, st, wd, bad)) break;
                }
                if (wd.failed) {
                    report(p, STATUS_TIMEOUT);
                    // Let copies already in flight land before the CTA exits: wait
                    // (briefly, bounded) for the latest issued phase of every slot.
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
            __syncwarp();
        } else if (warp == kMmaWarp) {
            // -------------------------------------------------------- MMA issue
            if (lane == 0) {
                MmaStream m0, m1;
                m0.w.init(p, 0, bad);
                m1.w.init(p, 1, bad);
                m0.r = m1.r = 0;
                m0.need_pv = m1.need_pv = false;
                m0.qcount = m0.pcount = m0.ocount = m1.qcount = m1.pcount = m1.ocount = 0;
                m0.block_bar = m1.block_bar = nullptr;
                m0.block_par = m1.block_par = 0;
                MmaDescs dd;
                dd.hi_k = (uint32_t)(sdesc_sw128(0, 16, 1024) >> 32);
                dd.hi_mn = (uint32_t)(sdesc_sw128(0, kBox, 1024) >> 32);
                for (int i = 0; i < 2; ++i) dd.q[i] = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_Q + i * C::TILE), 16, 1024);
                for (int i = 0; i < 3; ++i) {
                    const int si = i < C::NK ? i : 0, vi = i < C::NV ? i : 0;
                    dd.k[i] = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_K + si * C::TILE), 16, 1024);
                    dd.v[i] = (uint32_t)sdesc_sw128(smem_u32(smem + C::OFF_V + vi * C::TILE), kBox, 1024);
                }
                uint64_t idle_since = 0;
                bool idle = false, flip = false;
                while (m0.r < T0 || m1.r < T1) {
                    bool progressed = mma_try<D, SCORE, 0>(p, sh, m0, T0, T0, T1, tmem, dd, bad);
                    progressed |= mma_try<D, SCORE, 1>(p, sh, m1, T1, T0, T1, tmem, dd, bad);
                    if (progressed) {
                        idle = false;
                        continue;
                    }
                    // nothing issuable: sleep briefly on a blocked stream's barrier
                    // (alternating), so the poll takes no issue slots from the softmax
                    flip = !flip;
                    const bool use1 = (flip && m1.r < T1) || m0.r >= T0;
                    uint64_t* bb = use1 ? m1.block_bar : m0.block_bar;
                    const uint32_t bp = use1 ? m1.block_par : m0.block_par;
                    if (bb) mbar_try_wait_hint(bb, bp, 20);
                    if (!idle) {
                        idle = true;
                        idle_since = globaltimer_ns();
                    } else if (globaltimer_ns() - idle_since > wd.limit_ns) {
                        wd.failed = true;
                        break;
                    }
                }
                // All issued MMAs complete before the CTA tears down TMEM.
                umma_commit(&sh.drain);
                Watchdog dw{wd.failed ? 1000000ull : wd.limit_ns, false};
                mbar_wait(&sh.drain, 0, dw);
                if (wd.failed || dw.failed) report(p, STATUS_TIMEOUT);
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ softmax
        regs_inc<RegSplit<D, SCORE>::softmax>();
        const int s = warp / 4;
        const int wq = warp % 4;
        const int row = wq * 32 + lane;
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        const uint32_t s_addr = tmem + lane_base + 128 * s;
        const uint32_t o_addr = tmem + lane_base + C::O_COL0 + D * s;

        // Frame of the modified scores x' (log2 units): the tile maximum is
        // max(x') * F + shift and p = exp2(x' * F + shift - m).
        float F;
        if constexpr (SCORE == FA_SCORE_NONE) F = p.scale_log2;
        else if constexpr (SCORE == FA_SCORE_BIAS) F = kLog2e;
        else if constexpr (SCORE == FA_SCORE_SOFTCAP) F = p.softcap_out;  // x' = tanh(s * scale / cap)
        else F = 1.0f;
        const uint64_t F2 = f2_pack(F, F);
        const float bias_scale = p.scale_log2 / kLog2e;  // x' = s * scale + bias (natural units)

        uint32_t scount = 0, ocount = 0;
        int r = 0;
        bool dead = false;
        ItemLoad nxt;
        item_issue(p, item_index(s, 0, gridDim.x, blockIdx.x), nxt, true, SCORE == FA_SCORE_ALIBI, row);
        for (int k = 0; !dead && nxt.valid; ++k) {
            const Item I = item_finish(p, nxt, bad);
            const int f0 = nxt.f0_raw, p0 = nxt.p0_raw;
            const float slope2 = SCORE == FA_SCORE_ALIBI ? nxt.slope * kLog2e : 0.f;
            const int32_t qdoc = nxt.qdoc;
            item_issue(p, item_index(s, k + 1, gridDim.x, blockIdx.x), nxt, true, SCORE == FA_SCORE_ALIBI, row);

            const int64_t q = (int64_t)I.qb * 128 + row;
            const bool q_in = q < p.q_len;
            if (I.n == 0) {
                uint16_t* orow = p.o + I.b * p.o_stride_b + I.hq * p.o_stride_h + q * p.o_stride_s;
                float* lse_ptr = p.lse ? p.lse + ((int64_t)I.b * p.Hq + I.hq) * p.q_len + q : nullptr;
                if (q_in) {
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(orow)[c] = make_uint4(0, 0, 0, 0);
                    if (lse_ptr) *lse_ptr = -INFINITY;
                }
                continue;
            }
            const int32_t* doc_row = p.mask.has_doc ? p.mask.doc_ids + (int64_t)I.b * p.mask.doc_stride : nullptr;

            float m_run = -INFINITY;
            uint64_t l2 = f2_pack(0.f, 0.f);
            int kb = clamp_kb(I.nfull > 0 ? f0 : p0, p.nkv, bad);
            int kb_next_raw = I.n > 1 ? list_raw(I, 1) : 0;
            for (int t = 0; t < I.n; ++t, ++r) {
                const int64_t k0 = (int64_t)kb * 128;
                const bool partial = t >= I.nfull;
                const bool ragged = (kb == p.nkv - 1) && (p.kv_len % 128 != 0);

                // per-row mask words (partial tiles and the ragged last kv tile)
                uint32_t mw[4] = {0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu};
                if (partial) {
                    uint32_t db[4] = {0u, 0u, 0u, 0u};
                    if (p.mask.has_doc) doc_bits(doc_row, k0, p.kv_len, qdoc, db);
                    row_mask_bits(p.mask, q, k0, p.kv_len, db, mw);
                } else if (ragged) {
                    const int64_t lastc = p.kv_len - 1 - k0;
#pragma unroll
                    for (int j = 0; j < 4; ++j) mw[j] = range_bits(0, lastc, 32 * j);
                }
                const bool masked = partial || ragged;
                float shift = 0.f;
                if constexpr (SCORE == FA_SCORE_ALIBI) shift = slope2 * (float)(k0 - q);

                bool ok = mbar_wait(&sh.s_full[s], scount & 1, wd);
                if (!__all_sync(0xFFFFFFFFu, ok)) { dead = true; break; }
                scount++;
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

                // score_mod: x' in the frame above
                if constexpr (SCORE == FA_SCORE_ALIBI) {
                    // x' = s * scale * log2(e) + slope * log2(e) * j: the column term as a
                    // running pair, recomputed exactly every 32 columns (accumulated
                    // rounding below 1e-4 in log2 units)
                    const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
                    const uint64_t step2 = f2_pack(2.0f * slope2, 2.0f * slope2);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint64_t cb = f2_pack(slope2 * (float)(32 * c), slope2 * (float)(32 * c + 1));
#pragma unroll
                        for (int j = 32 * c; j < 32 * c + 32; j += 2) {
                            f2_unpack(f2_fma(f2_pack(x[j], x[j + 1]), c2, cb), x[j], x[j + 1]);
                            cb = f2_add(cb, step2);
                        }
                    }
                } else if constexpr (SCORE == FA_SCORE_SOFTCAP) {
                    const uint64_t in2 = f2_pack(p.softcap_in, p.softcap_in);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        bool far = false;
#pragma unroll
                        for (int j = 32 * c; j < 32 * c + 32; j += 2) {
                            f2_unpack(f2_mul(f2_pack(x[j], x[j + 1]), in2), x[j], x[j + 1]);
                            far |= fabsf(x[j]) > 0.625f || fabsf(x[j + 1]) > 0.625f;
                        }
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
                } else if constexpr (SCORE == FA_SCORE_BIAS) {
                    const uint32_t seq = tile_seq(s, r, T0, T1);
                    const uint32_t slot = seq % C::NB;
                    bool okb = mbar_wait(&sh.b_full[slot], (seq / C::NB) & 1, wd);
                    if (!__all_sync(0xFFFFFFFFu, okb)) { dead = true; break; }
                    const uint8_t* brow = smem + C::OFF_B + slot * C::BIAS_TILE + row * 128;
                    const uint64_t sc2 = f2_pack(bias_scale, bias_scale);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const uint4 v4 = *reinterpret_cast<const uint4*>(brow + h * kBox + ((c ^ (row & 7)) * 16));
                            const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int j = h * 64 + c * 8 + 2 * e;
                                const uint64_t bb =
                                    f2_pack(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xFFFF0000u));
                                f2_unpack(f2_fma(f2_pack(x[j], x[j + 1]), sc2, bb), x[j], x[j + 1]);
                            }
                        }
                    }
                    mbar_arrive(&sh.b_empty[slot]);
                }

                if (masked) {
#pragma unroll
                    for (int j = 0; j < 128; ++j)
                        if (!((mw[j >> 5] >> (j & 31)) & 1u)) x[j] = -INFINITY;
                }

                float mx0 = max3(x[0], x[1], x[2]), mx1 = max3(x[3], x[4], x[5]);
                float mx2 = max3(x[6], x[7], x[8]), mx3 = max3(x[9], x[10], x[11]);
#pragma unroll
                for (int j = 12; j < 124; j += 8) {
                    mx0 = max3(mx0, x[j], x[j + 1]);
                    mx1 = max3(mx1, x[j + 2], x[j + 3]);
                    mx2 = max3(mx2, x[j + 4], x[j + 5]);
                    mx3 = max3(mx3, x[j + 6], x[j + 7]);
                }
                mx0 = max3(mx0, x[124], x[125]);
                mx1 = max3(mx1, x[126], x[127]);
                const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * F + shift;

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
                const float m_use = m_run == -INFINITY ? 0.f : m_run;
                const uint64_t b2 = f2_pack(shift - m_use, shift - m_use);
                uint64_t la = f2_pack(0.f, 0.f), lb = la;
                // In full tiles without a bias every argument is finite, so part of
                // the exponentials go to the FMA pipe (exp2_poly2) to unload MUFU.
                const bool split = (SCORE != FA_SCORE_BIAS) && !masked;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; j += 2) {
                        const int e = 32 * c + 2 * j;
                        const uint64_t a01 = f2_fma(f2_pack(x[e], x[e + 1]), F2, b2);
                        const uint64_t a23 = f2_fma(f2_pack(x[e + 2], x[e + 3]), F2, b2);
                        float e0, e1, e2, e3;
                        float a0, a1, a2, a3;
                        f2_unpack(a01, a0, a1);
                        e0 = ex2_approx(a0);
                        e1 = ex2_approx(a1);
                        if (split && kPolyPair[(e / 4) % 3]) {
                            exp2_poly2(a23, e2, e3);
                        } else {
                            f2_unpack(a23, a2, a3);
                            e2 = ex2_approx(a2);
                            e3 = ex2_approx(a3);
                        }
                        la = f2_add(la, f2_pack(e0, e1));
                        lb = f2_add(lb, f2_pack(e2, e3));
                        pk[j] = pack_bf16x2(e0, e1);
                        pk[j + 1] = pack_bf16x2(e2, e3);
                    }
                    tmem_st16(s_addr + 16 * c, pk);
                }
                l2 = f2_add(l2, f2_add(la, lb));
                // next tile's kv block (read one tile ahead)
                if (t + 1 < I.n) {
                    kb = clamp_kb(kb_next_raw, p.nkv, bad);
                    kb_next_raw = t + 2 < I.n ? list_raw(I, t + 2) : 0;
                }
                if (__any_sync(0xFFFFFFFFu, rescale)) {
                    // O is stable here: the commit that published S of this tile
                    // was issued after the previous tile's P V, and this tile's P V
                    // waits for the arrival below.
#pragma unroll
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
                mbar_arrive(&sh.p_full[s]);
            }
            if (dead) break;

            // epilogue: O / l -> bf16, LSE = ln(2) * (m + log2 l)
            float l_lo, l_hi;
            f2_unpack(l2, l_lo, l_hi);
            const float l_run = l_lo + l_hi;
            bool ok = mbar_wait(&sh.o_full[s], ocount & 1, wd);
            if (!__all_sync(0xFFFFFFFFu, ok)) { dead = true; break; }
            ocount++;
            tc_fence_after();
            const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
            uint16_t* orow = p.o + I.b * p.o_stride_b + I.hq * p.o_stride_h + q * p.o_stride_s;
            float* lse_ptr = p.lse ? p.lse + ((int64_t)I.b * p.Hq + I.hq) * p.q_len + q : nullptr;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t ov[32];
                tmem_ld32(o_addr + 32 * c, ov);
                tmem_ld_wait();
                if (c == D / 32 - 1) {
                    tc_fence_before();
                    mbar_arrive(&sh.o_empty[s]);
                }
                if (q_in) {
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        pk[j] = pack_bf16x2(__uint_as_float(ov[2 * j]) * inv_l, __uint_as_float(ov[2 * j + 1]) * inv_l);
                    uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
                    for (int j = 0; j < 4; ++j) dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                }
            }
            if (q_in && lse_ptr) *lse_ptr = l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
        }
        if (dead || wd.failed) {
            if (lane == 0) report(p, STATUS_TIMEOUT);
        }
    }

    if (bad || (threadIdx.x == 0 && sh.bad)) report(p, STATUS_BAD_BLOCKMASK);

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

template <int D, int SCORE>
cudaError_t launch_variant(const FwdParams& p, int grid, cudaStream_t stream)
{
    auto kern = flex_fwd_kernel<D, SCORE>;
    static bool configured = false;
    if (!configured) {
        // The register split assumes the launch allocation; refuse anything else
        // rather than launch a kernel whose setmaxnreg.inc could never be served.
        cudaFuncAttributes fa_attr;
        cudaError_t e = cudaFuncGetAttributes(&fa_attr, kern);
        if (e != cudaSuccess) return e;
        if (fa_attr.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D, SCORE>::SMEM);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    kern<<<grid, kThreads, Cfg<D, SCORE>::SMEM, stream>>>(p);
    return cudaGetLastError();
}

} // namespace

int flex_forward_smem_bytes(int D, int score_kind)
{
#define FA_SMEM_CASE(DD, SS) \
    if (D == DD && score_kind == SS) return Cfg<DD, SS>::SMEM;
    FA_SMEM_CASE(64, FA_SCORE_NONE) FA_SMEM_CASE(64, FA_SCORE_ALIBI) FA_SMEM_CASE(64, FA_SCORE_SOFTCAP)
    FA_SMEM_CASE(64, FA_SCORE_BIAS) FA_SMEM_CASE(128, FA_SCORE_NONE) FA_SMEM_CASE(128, FA_SCORE_ALIBI)
    FA_SMEM_CASE(128, FA_SCORE_SOFTCAP) FA_SMEM_CASE(128, FA_SCORE_BIAS)
#undef FA_SMEM_CASE
    return -1;
}

cudaError_t launch_flex_forward(const FwdParams& p, int D, int score_kind, int grid, cudaStream_t stream)
{
#define FA_LAUNCH_CASE(DD, SS) \
    if (D == DD && score_kind == SS) return launch_variant<DD, SS>(p, grid, stream);
    FA_LAUNCH_CASE(64, FA_SCORE_NONE) FA_LAUNCH_CASE(64, FA_SCORE_ALIBI) FA_LAUNCH_CASE(64, FA_SCORE_SOFTCAP)
    FA_LAUNCH_CASE(64, FA_SCORE_BIAS) FA_LAUNCH_CASE(128, FA_SCORE_NONE) FA_LAUNCH_CASE(128, FA_SCORE_ALIBI)
    FA_LAUNCH_CASE(128, FA_SCORE_SOFTCAP) FA_LAUNCH_CASE(128, FA_SCORE_BIAS)
#undef FA_LAUNCH_CASE
    return cudaErrorInvalidValue;
}

} // namespace fa
