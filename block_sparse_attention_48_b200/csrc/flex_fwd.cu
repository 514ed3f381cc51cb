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
//   warps 10-11 idle (they complete the third warpgroup for register reallocation)
// The softmax warpgroups take registers from the third warpgroup (setmaxnreg):
// launched at 168 per thread, they run at 232 and the third at 40.
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
// consumed in order.
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
constexpr int kSoftmaxRegs = 208;
constexpr int kOtherRegs = 88;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kBox = 16384;  // bytes of one 128-row x 64-column bf16 TMA box

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

struct __align__(8) Barriers {
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[3], k_empty[3];
    uint64_t v_full[3], v_empty[3];
    uint64_t b_full[2], b_empty[2];
    uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
};

struct Item {
    int b, hq, qb;
    int nfull, n;
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

__device__ __forceinline__ Item load_item(const FwdParams& p, int idx, bool& bad)
{
    Item it;
    const int bh_count = p.B * p.Hq;
    const int qb_rank = idx / bh_count;
    const int bh = idx - qb_rank * bh_count;
    it.qb = p.nq - 1 - qb_rank;
    it.b = bh / p.Hq;
    it.hq = bh - it.b * p.Hq;
    const int mb = p.bm_B == 1 ? 0 : it.b;
    const int mh = p.bm_H == 1 ? 0 : it.hq;
    const int64_t row = ((int64_t)mb * p.bm_H + mh) * p.nq + it.qb;
    int nf = p.has_full ? __ldg(p.full_num + row) : 0;
    int np = __ldg(p.kv_num + row);
    if (nf < 0 || nf > p.nkv) { bad = true; nf = nf < 0 ? 0 : p.nkv; }
    if (np < 0 || np > p.nkv) { bad = true; np = np < 0 ? 0 : p.nkv; }
    it.nfull = nf;
    it.n = nf + np;
    it.full_list = p.full_idx + row * p.nkv;
    it.part_list = p.kv_idx + row * p.nkv;
    return it;
}

__device__ __forceinline__ int tile_kb(const FwdParams& p, const Item& it, int t, bool& bad)
{
    int kb = t < it.nfull ? __ldg(it.full_list + t) : __ldg(it.part_list + (t - it.nfull));
    if (kb < 0 || kb >= p.nkv) {
        bad = true;
        kb = kb < 0 ? 0 : p.nkv - 1;
    }
    return kb;
}

__device__ __forceinline__ int stream_total(const FwdParams& p, int s, bool& bad)
{
    int T = 0;
    for (int k = 0;; ++k) {
        long long idx = item_index(s, k, gridDim.x, blockIdx.x);
        if (idx >= p.num_items) break;
        T += load_item(p, (int)idx, bad).n;
    }
    return T;
}

// Position of stream s's r-th tile in the interleaved production order.
__device__ __forceinline__ uint32_t tile_seq(int s, int r, int T0, int T1)
{
    return (uint32_t)(min(r, T0) + min(r, T1) + ((s == 1 && r < T0) ? 1 : 0));
}

// Iterator over the non-empty items of one stream.
struct Walk {
    int k;
    int idx;
    Item it;
    int t;
};

__device__ __forceinline__ void walk_next_item(const FwdParams& p, Walk& w, int s, bool& bad)
{
    for (;;) {
        long long idx = item_index(s, w.k, gridDim.x, blockIdx.x);
        if (idx >= p.num_items) {
            w.idx = p.num_items;
            return;
        }
        w.idx = (int)idx;
        w.it = load_item(p, w.idx, bad);
        w.k++;
        if (w.it.n > 0) {
            w.t = 0;
            return;
        }
    }
}

__device__ __forceinline__ void report(const FwdParams& p, int bits)
{
    atomicOr(p.status, bits);
}

// Odd minimax-style polynomial for tanh on |y| <= 0.625 (least-squares fit of
// (tanh(y) - y) / y^3 in u = y^2 on Chebyshev nodes, weighted by y^3; max abs
// error 4e-8 in fp32), and 1 - 2 / (e^(2|y|) + 1) beyond.
__device__ __forceinline__ float tanh_poly(float y)
{
    const float u = y * y;
    float p = -0.005561366677284241f;
    p = fmaf(p, u, 0.020492956042289734f);
    p = fmaf(p, u, -0.05368727073073387f);
    p = fmaf(p, u, 0.13330671191215515f);
    p = fmaf(p, u, -0.33333244919776917f);
    return fmaf(y * u, p, y);
}

__device__ __forceinline__ float tanh_far(float y)
{
    const float a = fabsf(y);
    const float e = ex2_approx(2.0f * kLog2e * a);
    const float t = 1.0f - __fdividef(2.0f, e + 1.0f);
    return copysignf(t, y);
}

template <int D, int SCORE>
__global__ void __launch_bounds__(kThreads, 1) flex_fwd_kernel(const __grid_constant__ FwdParams p)
{
    using C = Cfg<D, SCORE>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ Barriers bars;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (warp == kMmaWarp) {
        tmem_alloc(&bars.tmem_base, 512);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars.q_full[s], 1);
            mbar_init(&bars.q_empty[s], 1);
            mbar_init(&bars.s_full[s], 1);
            mbar_init(&bars.p_full[s], 128);
            mbar_init(&bars.o_full[s], 1);
            mbar_init(&bars.o_empty[s], 128);
        }
        for (int i = 0; i < C::NK; ++i) { mbar_init(&bars.k_full[i], 1); mbar_init(&bars.k_empty[i], 1); }
        for (int i = 0; i < C::NV; ++i) { mbar_init(&bars.v_full[i], 1); mbar_init(&bars.v_empty[i], 1); }
        for (int i = 0; i < C::NB; ++i) { mbar_init(&bars.b_full[i], 1); mbar_init(&bars.b_empty[i], 128); }
        mbar_init(&bars.drain, 1);
        mbar_fence_init();
    }
    if (warp == kLoadWarp && lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_v);
        if (SCORE == FA_SCORE_BIAS) tma_prefetch_desc(&p.tm_bias);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;

    Watchdog wd{p.watchdog_ns, false};
    bool bad = false;

    if (warp >= 8) {
      regs_dec<kOtherRegs>();
      if (warp == kLoadWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const int T0 = stream_total(p, 0, bad), T1 = stream_total(p, 1, bad);
            Walk w[2];
            w[0].k = 0;
            w[1].k = 0;
            walk_next_item(p, w[0], 0, bad);
            walk_next_item(p, w[1], 1, bad);
            uint32_t seq = 0, qcount[2] = {0, 0};
            uint32_t k_issued = 0, v_issued = 0, b_issued = 0;
            const int rounds = max(T0, T1);
            for (int r = 0; r < rounds && !wd.failed; ++r) {
                for (int s = 0; s < 2; ++s) {
                    if (r >= (s == 0 ? T0 : T1)) continue;
                    Walk& cw = w[s];
                    const Item& I = cw.it;
                    if (cw.t == 0) {
                        if (!mbar_wait(&bars.q_empty[s], (qcount[s] & 1) ^ 1, wd)) break;
                        mbar_arrive_expect_tx(&bars.q_full[s], C::TILE);
                        uint8_t* dst = smem + C::OFF_Q + s * C::TILE;
#pragma unroll
                        for (int c = 0; c < D / 64; ++c)
                            tma_load_4d(dst + c * kBox, &p.tm_q, &bars.q_full[s], c * 64, I.qb * 128, I.hq, I.b);
                        qcount[s]++;
                    }
                    const int kb = tile_kb(p, I, cw.t, bad);
                    const int hk = I.hq / p.G;
                    {
                        const uint32_t slot = seq % C::NK;
                        if (!mbar_wait(&bars.k_empty[slot], ((seq / C::NK) & 1) ^ 1, wd)) break;
                        mbar_arrive_expect_tx(&bars.k_full[slot], C::TILE);
                        uint8_t* dst = smem + C::OFF_K + slot * C::TILE;
#pragma unroll
                        for (int c = 0; c < D / 64; ++c)
                            tma_load_4d(dst + c * kBox, &p.tm_k, &bars.k_full[slot], c * 64, kb * 128, hk, I.b);
                        k_issued++;
                    }
                    if constexpr (SCORE == FA_SCORE_BIAS) {
                        const uint32_t slot = seq % C::NB;
                        if (!mbar_wait(&bars.b_empty[slot], ((seq / C::NB) & 1) ^ 1, wd)) break;
                        mbar_arrive_expect_tx(&bars.b_full[slot], C::BIAS_TILE);
                        uint8_t* dst = smem + C::OFF_B + slot * C::BIAS_TILE;
#pragma unroll
                        for (int c = 0; c < 2; ++c)
                            tma_load_4d(dst + c * kBox, &p.tm_bias, &bars.b_full[slot], kb * 128 + c * 64,
                                        I.qb * 128, I.hq, I.b);
                        b_issued++;
                    }
                    {
                        const uint32_t slot = seq % C::NV;
                        if (!mbar_wait(&bars.v_empty[slot], ((seq / C::NV) & 1) ^ 1, wd)) break;
                        mbar_arrive_expect_tx(&bars.v_full[slot], C::TILE);
                        uint8_t* dst = smem + C::OFF_V + slot * C::TILE;
#pragma unroll
                        for (int c = 0; c < D / 64; ++c)
                            tma_load_4d(dst + c * kBox, &p.tm_v, &bars.v_full[slot], c * 64, kb * 128, hk, I.b);
                        v_issued++;
                    }
                    seq++;
                    if (++cw.t == I.n) walk_next_item(p, cw, s, bad);
                }
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
                drain(bars.k_full, k_issued, C::NK);
                drain(bars.v_full, v_issued, C::NV);
                if (C::NB > 0) drain(bars.b_full, b_issued, C::NB > 0 ? C::NB : 1);
                for (int s = 0; s < 2; ++s)
                    if (qcount[s] > 0) {
                        dw.failed = false;
                        mbar_wait(&bars.q_full[s], (qcount[s] - 1) & 1, dw);
                    }
            }
        }
        __syncwarp();
      } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            const int T[2] = {stream_total(p, 0, bad), stream_total(p, 1, bad)};
            Walk w[2];
            int r[2] = {0, 0};
            bool need_pv[2] = {false, false};
            uint32_t qcount[2] = {0, 0}, pcount[2] = {0, 0}, ocount[2] = {0, 0};
            w[0].k = 0;
            w[1].k = 0;
            walk_next_item(p, w[0], 0, bad);
            walk_next_item(p, w[1], 1, bad);
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
            const uint32_t sq_base = smem_u32(smem + C::OFF_Q);
            const uint32_t sk_base = smem_u32(smem + C::OFF_K);
            const uint32_t sv_base = smem_u32(smem + C::OFF_V);
            uint64_t idle_since = 0;
            bool idle = false;
            while (r[0] < T[0] || r[1] < T[1]) {
                bool progressed = false;
#pragma unroll
                for (int s = 0; s < 2; ++s) {
                    if (r[s] >= T[s]) continue;
                    Walk& cw = w[s];
                    const uint32_t seq = tile_seq(s, r[s], T[0], T[1]);
                    const bool first = cw.t == 0;
                    const bool last = cw.t == cw.it.n - 1;
                    if (!need_pv[s]) {
                        const uint32_t slot = seq % C::NK;
                        if (first && !mbar_test_wait(&bars.q_full[s], qcount[s] & 1)) continue;
                        if (!mbar_test_wait(&bars.k_full[slot], (seq / C::NK) & 1)) continue;
                        tc_fence_after();
                        const uint32_t qa = sq_base + s * C::TILE;
                        const uint32_t kbase = sk_base + slot * C::TILE;
#pragma unroll
                        for (int k = 0; k < D / 16; ++k) {
                            const uint32_t off = (k / 4) * kBox + (k % 4) * 32;
                            umma_ss(tmem + 128 * s, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(kbase + off, 16, 1024),
                                    idesc_s, k > 0);
                        }
                        umma_commit(&bars.k_empty[slot]);
                        umma_commit(&bars.s_full[s]);
                        if (last) umma_commit(&bars.q_empty[s]);
                        if (first) qcount[s]++;
                        need_pv[s] = true;
                        progressed = true;
                    } else {
                        const uint32_t slot = seq % C::NV;
                        if (!mbar_test_wait(&bars.p_full[s], pcount[s] & 1)) continue;
                        if (!mbar_test_wait(&bars.v_full[slot], (seq / C::NV) & 1)) continue;
                        if (first && !mbar_test_wait(&bars.o_empty[s], (ocount[s] & 1) ^ 1)) continue;
                        tc_fence_after();
                        const uint32_t vbase = sv_base + slot * C::TILE;
                        const uint32_t o_col = tmem + C::O_COL0 + D * s;
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            umma_ts(o_col, tmem + 128 * s + 8 * k, sdesc_sw128(vbase + k * 2048, kBox, 1024), idesc_o,
                                    (!first || k > 0) ? 1u : 0u);
                        umma_commit(&bars.v_empty[slot]);
                        if (last) umma_commit(&bars.o_full[s]);
                        pcount[s]++;
                        if (first) ocount[s]++;
                        need_pv[s] = false;
                        r[s]++;
                        if (++cw.t == cw.it.n) walk_next_item(p, cw, s, bad);
                        progressed = true;
                    }
                }
                if (progressed) {
                    idle = false;
                } else if (!idle) {
                    idle = true;
                    idle_since = globaltimer_ns();
                } else if (globaltimer_ns() - idle_since > wd.limit_ns) {
                    wd.failed = true;
                    break;
                }
            }
            // All issued MMAs complete before the CTA tears down TMEM.
            umma_commit(&bars.drain);
            Watchdog dw{wd.failed ? 1000000ull : wd.limit_ns, false};
            mbar_wait(&bars.drain, 0, dw);
            if (wd.failed || dw.failed) report(p, STATUS_TIMEOUT);
        }
        __syncwarp();
      }
    } else {
        // ------------------------------------------------------------ softmax
        regs_inc<kSoftmaxRegs>();
        const int s = warp / 4;
        const int wq = warp % 4;
        const int row = wq * 32 + lane;
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        const uint32_t s_addr = tmem + lane_base + 128 * s;
        const uint32_t o_addr = tmem + lane_base + C::O_COL0 + D * s;
        int T0 = 0, T1 = 0;
        if constexpr (SCORE == FA_SCORE_BIAS) {
            T0 = stream_total(p, 0, bad);
            T1 = stream_total(p, 1, bad);
        }
        uint32_t scount = 0, ocount = 0;
        int r = 0;
        bool dead = false;
        const int32_t* doc_row = nullptr;
        for (int k = 0; !dead; ++k) {
            const long long idx64 = item_index(s, k, gridDim.x, blockIdx.x);
            if (idx64 >= p.num_items) break;
            const Item I = load_item(p, (int)idx64, bad);
            const int64_t q = (int64_t)I.qb * 128 + row;
            const bool q_in = q < p.q_len;
            uint16_t* orow = p.o + I.b * p.o_stride_b + I.hq * p.o_stride_h + q * p.o_stride_s;
            float* lse_ptr = p.lse ? p.lse + ((int64_t)I.b * p.Hq + I.hq) * p.q_len + q : nullptr;
            if (I.n == 0) {
                if (q_in) {
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(orow)[c] = make_uint4(0, 0, 0, 0);
                    if (lse_ptr) *lse_ptr = -INFINITY;
                }
                continue;
            }
            int32_t qdoc = 0;
            if (p.mask.has_doc) {
                doc_row = p.mask.doc_ids + (int64_t)I.b * p.mask.doc_stride;
                qdoc = q_in ? __ldg(doc_row + q) : INT32_MIN;
            }
            float slope2 = 0.f;
            if constexpr (SCORE == FA_SCORE_ALIBI) slope2 = __ldg(p.slopes + I.hq) * kLog2e;

            float m_run = -INFINITY, l_run = 0.f;
            for (int t = 0; t < I.n; ++t, ++r) {
                const int kb = tile_kb(p, I, t, bad);
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

                bool ok = mbar_wait(&bars.s_full[s], scount & 1, wd);
                if (!__all_sync(0xFFFFFFFFu, ok)) { dead = true; break; }
                scount++;
                tc_fence_after();

                float x[128];
                {
                    uint32_t raw[32];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        tmem_ld32(s_addr + 32 * c, raw);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) x[32 * c + j] = __uint_as_float(raw[j]);
                    }
                }

                // score_mod, in log2 units (factor applied later for NONE)
                float factor = 1.0f;
                if constexpr (SCORE == FA_SCORE_NONE) {
                    factor = p.scale_log2;
                } else if constexpr (SCORE == FA_SCORE_ALIBI) {
                    const float base = slope2 * (float)(k0 - q);
#pragma unroll
                    for (int j = 0; j < 128; ++j) x[j] = fmaf(x[j], p.scale_log2, fmaf(slope2, (float)j, base));
                } else if constexpr (SCORE == FA_SCORE_SOFTCAP) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        bool far = false;
#pragma unroll
                        for (int j = 32 * c; j < 32 * c + 32; ++j) {
                            x[j] *= p.softcap_in;
                            far |= fabsf(x[j]) > 0.625f;
                        }
                        if (__any_sync(0xFFFFFFFFu, far)) {
#pragma unroll
                            for (int j = 32 * c; j < 32 * c + 32; ++j)
                                x[j] = (fabsf(x[j]) > 0.625f ? tanh_far(x[j]) : tanh_poly(x[j])) * p.softcap_out;
                        } else {
#pragma unroll
                            for (int j = 32 * c; j < 32 * c + 32; ++j) x[j] = tanh_poly(x[j]) * p.softcap_out;
                        }
                    }
                } else if constexpr (SCORE == FA_SCORE_BIAS) {
                    const uint32_t seq = tile_seq(s, r, T0, T1);
                    const uint32_t slot = seq % C::NB;
                    bool okb = mbar_wait(&bars.b_full[slot], (seq / C::NB) & 1, wd);
                    if (!__all_sync(0xFFFFFFFFu, okb)) { dead = true; break; }
                    const uint8_t* brow = smem + C::OFF_B + slot * C::BIAS_TILE + row * 128;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const uint4 v4 = *reinterpret_cast<const uint4*>(brow + h * kBox + ((c ^ (row & 7)) * 16));
                            const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int j = h * 64 + c * 8 + 2 * e;
                                const float b0 = __uint_as_float(wv[e] << 16);
                                const float b1 = __uint_as_float(wv[e] & 0xFFFF0000u);
                                x[j] = fmaf(x[j], p.scale_log2, b0 * kLog2e);
                                x[j + 1] = fmaf(x[j + 1], p.scale_log2, b1 * kLog2e);
                            }
                        }
                    }
                    mbar_arrive(&bars.b_empty[slot]);
                }

                if (masked) {
#pragma unroll
                    for (int j = 0; j < 128; ++j)
                        if (!((mw[j >> 5] >> (j & 31)) & 1u)) x[j] = -INFINITY;
                }

                float mx0 = x[0], mx1 = x[1], mx2 = x[2], mx3 = x[3];
#pragma unroll
                for (int j = 4; j < 128; j += 4) {
                    mx0 = fmaxf(mx0, x[j]);
                    mx1 = fmaxf(mx1, x[j + 1]);
                    mx2 = fmaxf(mx2, x[j + 2]);
                    mx3 = fmaxf(mx3, x[j + 3]);
                }
                const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * factor;

                // running maximum: moved only when the tile maximum exceeds it by
                // more than the threshold (first tile: always set)
                float alpha = 1.0f;
                bool rescale = false;
                if (t == 0) {
                    m_run = m_tile;
                } else if (m_tile > m_run + kRescaleThreshold) {
                    alpha = ex2_approx(m_run - m_tile);
                    m_run = m_tile;
                    l_run *= alpha;
                    rescale = true;
                }
                const float m_use = m_run == -INFINITY ? 0.f : m_run;
                float l0 = 0.f, l1 = 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float e0 = ex2_approx(fmaf(x[32 * c + 2 * j], factor, -m_use));
                        const float e1 = ex2_approx(fmaf(x[32 * c + 2 * j + 1], factor, -m_use));
                        l0 += e0;
                        l1 += e1;
                        pk[j] = pack_bf16x2(e0, e1);
                    }
                    tmem_st16(s_addr + 16 * c, pk);
                }
                l_run += l0 + l1;
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
                mbar_arrive(&bars.p_full[s]);
            }
            if (dead) break;

            // epilogue: O / l -> bf16, LSE = ln(2) * (m + log2 l)
            bool ok = mbar_wait(&bars.o_full[s], ocount & 1, wd);
            if (!__all_sync(0xFFFFFFFFu, ok)) { dead = true; break; }
            ocount++;
            tc_fence_after();
            const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t ov[32];
                tmem_ld32(o_addr + 32 * c, ov);
                tmem_ld_wait();
                if (c == D / 32 - 1) {
                    tc_fence_before();
                    mbar_arrive(&bars.o_empty[s]);
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

    if (bad && (threadIdx.x == 0)) report(p, STATUS_BAD_BLOCKMASK);

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
