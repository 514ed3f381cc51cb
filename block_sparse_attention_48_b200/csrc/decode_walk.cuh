// The decode kernel's walk over the list of kv blocks ("Flex Attention" paper
// review sec. 3.1, the decoding template: the work split along the KV
// dimension).  The list holds the kv blocks of every (batch, kv head) segment,
// segments in (batch, kv head) order, each its batch's BlockMask row (query
// block 0; partial blocks first, then full ones).  CTA c of G takes entries
// [share_start(c), share_start(c + 1)) and walks them with dec_advance.
//
// Device code, templated on the parameter block (fields B, Hkv, nkv, bm_B,
// has_full, kv_num, full_num, kv_idx, full_idx) so that the CPU tests build the
// same functions for the host.
#pragma once

#include <cstdint>

namespace fa {

// Position in the list: segment (b, hk), block t of the batch's row, which has
// np partial and n blocks in all.
struct DecWalk {
    int b, hk, t, np, n;
};

template <class P>
__device__ __forceinline__ int64_t dec_row(const P& p, int b)
{
    return p.bm_B == 1 ? 0 : b;
}

// Block counts of BlockMask row r: partial and partial + full, each clamped to
// [0, nkv] (a corrupt count sets `bad`).
template <class P>
__device__ __forceinline__ void dec_counts(const P& p, int64_t r, int& np, int& n, bool& bad)
{
    int a = __ldg(p.kv_num + r), f = p.has_full ? __ldg(p.full_num + r) : 0;
    if (a < 0 || a > p.nkv) { bad = true; a = a < 0 ? 0 : p.nkv; }
    if (f < 0 || f > p.nkv) { bad = true; f = f < 0 ? 0 : p.nkv; }
    np = a;
    n = a + f;
}

// kv block index of the position (clamped to [0, nkv), a bad entry sets `bad`).
template <class P>
__device__ __forceinline__ int dec_block(const P& p, const DecWalk& w, bool& bad)
{
    const int64_t r = dec_row(p, w.b) * p.nkv;
    int kb = w.t < w.np ? __ldg(p.kv_idx + r + w.t) : __ldg(p.full_idx + r + (w.t - w.np));
    if (kb < 0 || kb >= p.nkv) { bad = true; kb = kb < 0 ? 0 : p.nkv - 1; }
    return kb;
}

// The next position (called only while the share has entries left, so a
// non-empty segment follows; the batch index never passes B - 1).
template <class P>
__device__ __forceinline__ void dec_advance(const P& p, DecWalk& w, bool& bad)
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

// floor(c * T / G) without overflowing the product: where CTA c's share starts.
__device__ __forceinline__ long long share_start(long long T, int c, int G)
{
    return (T / G) * c + (T % G) * c / G;
}

// The position of list entry x, given that it lies in the segments of rows
// [lo, hi) and that the rows before lo hold `before` blocks (one row per
// batch).  Returns false if x is not in those rows.
template <class P>
__device__ __forceinline__ bool dec_find(const P& p, long long x, int lo, int hi, long long before, DecWalk& w,
                                         bool& bad)
{
    long long acc = before;
    for (int r = lo; r < hi; ++r) {
        int np, n;
        dec_counts(p, r, np, n, bad);
        if (x < (long long)p.Hkv * (acc + n)) {
            const long long off = x - (long long)p.Hkv * acc;
            w = DecWalk{r, (int)(off / n), (int)(off % n), np, n};
            return true;
        }
        acc += n;
    }
    return false;
}

// The position of list entry x when one BlockMask row of n0 > 0 blocks serves
// every batch.
template <class P>
__device__ __forceinline__ DecWalk dec_find_shared(const P& p, long long x, long long n0, bool& bad)
{
    const long long seg = x / n0;
    DecWalk w{(int)(seg / p.Hkv), (int)(seg % p.Hkv), (int)(x % n0), 0, 0};
    dec_counts(p, 0, w.np, w.n, bad);
    return w;
}

} // namespace fa
