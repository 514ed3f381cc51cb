// Host build of the decode kernel's walk over the list of kv blocks
// (csrc/decode_walk.cuh), for CPU unit tests: the device qualifiers are defined
// away and __ldg becomes a plain load.
#include <cstdint>

#define __device__
#define __forceinline__ inline
template <typename T>
static inline T __ldg(const T* p)
{
    return *p;
}

#include "decode_walk.cuh"

namespace {

// The fields the walk reads, as in the kernel's parameter block.
struct HostDecParams {
    int32_t B, Hkv, nkv, bm_B, has_full;
    const int32_t* kv_num;
    const int32_t* full_num;
    const int32_t* kv_idx;
    const int32_t* full_idx;
};

HostDecParams params(int32_t B, int32_t Hkv, int32_t nkv, int32_t bm_B, int32_t has_full, const int32_t* kv_num,
                     const int32_t* full_num, const int32_t* kv_idx, const int32_t* full_idx)
{
    return HostDecParams{B, Hkv, nkv, bm_B, has_full, kv_num, full_num, kv_idx, full_idx};
}

void put(const fa::DecWalk& w, int32_t* out)
{
    out[0] = w.b;
    out[1] = w.hk;
    out[2] = w.t;
    out[3] = w.np;
    out[4] = w.n;
}

} // namespace

extern "C" long long fa_host_share_start(long long T, int c, int G)
{
    return fa::share_start(T, c, G);
}

// dec_find over rows [lo, hi) with `before` blocks in the rows before lo; out =
// (b, hk, t, np, n).  Returns 1 if found, and 2 more if a count was corrupt.
extern "C" int fa_host_dec_find(int32_t B, int32_t Hkv, int32_t nkv, int32_t bm_B, int32_t has_full,
                                const int32_t* kv_num, const int32_t* full_num, long long x, int lo, int hi,
                                long long before, int32_t* out)
{
    const HostDecParams p = params(B, Hkv, nkv, bm_B, has_full, kv_num, full_num, nullptr, nullptr);
    fa::DecWalk w{};
    bool bad = false;
    const bool found = fa::dec_find(p, x, lo, hi, before, w, bad);
    put(w, out);
    return (found ? 1 : 0) | (bad ? 2 : 0);
}

extern "C" void fa_host_dec_find_shared(int32_t B, int32_t Hkv, int32_t nkv, int32_t has_full, const int32_t* kv_num,
                                        const int32_t* full_num, long long x, long long n0, int32_t* out)
{
    const HostDecParams p = params(B, Hkv, nkv, 1, has_full, kv_num, full_num, nullptr, nullptr);
    bool bad = false;
    put(fa::dec_find_shared(p, x, n0, bad), out);
}

// `count` entries from position (b, hk, t) as the kernel walks them: out[5 i ..] =
// (b, hk, t, np, kb) of entry i.  Returns 1 if a count or index was corrupt.
extern "C" int fa_host_dec_walk(int32_t B, int32_t Hkv, int32_t nkv, int32_t bm_B, int32_t has_full,
                                const int32_t* kv_num, const int32_t* full_num, const int32_t* kv_idx,
                                const int32_t* full_idx, int b, int hk, int t, long long count, int32_t* out)
{
    const HostDecParams p = params(B, Hkv, nkv, bm_B, has_full, kv_num, full_num, kv_idx, full_idx);
    bool bad = false;
    fa::DecWalk w{b, hk, t, 0, 0};
    fa::dec_counts(p, fa::dec_row(p, w.b), w.np, w.n, bad);
    for (long long i = 0; i < count; ++i) {
        out[5 * i] = w.b;
        out[5 * i + 1] = w.hk;
        out[5 * i + 2] = w.t;
        out[5 * i + 3] = w.np;
        out[5 * i + 4] = fa::dec_block(p, w, bad);
        if (i + 1 < count) fa::dec_advance(p, w, bad);
    }
    return bad ? 1 : 0;
}
