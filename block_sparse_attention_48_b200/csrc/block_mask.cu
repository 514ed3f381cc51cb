// create_block_mask on the GPU ("Concepts", BlockMask Internals; paper review
// sec. 4.1-4.2): classify every 128 x 128 tile of the (q, kv) plane as full,
// partial or empty over its in-range positions and emit the ascending lists of
// partial (kv_indices) and full (full_kv_indices) kv blocks of each query block.
//
// One CTA per BlockMask row (b, h, qb).  Every tile is first summarised leaf by
// leaf, one thread per tile (interval leaves exactly, the document leaf from the
// id ranges of the two blocks, gathered first with independent loads); only the
// tiles the summaries leave undecided are counted position by position, one
// warp per tile, as 128-bit mask words per row.  Both routes give the same
// class, so the result is the exact classification.
#include <cuda_runtime.h>

#include "block_mask.cuh"
#include "mask_eval.cuh"

namespace fa {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

__device__ __forceinline__ int warp_min(int v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

__device__ __forceinline__ int warp_max(int v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Document-id range (min, max) of positions [k0, k1] by one warp: four ids per
// lane per 128 positions, 16-byte loads where the whole block is in range and
// starts on a 16-byte boundary (query positions with an offset need not).
__device__ __forceinline__ void doc_range(const int32_t* doc_row, int64_t k0, int64_t k1, int lane, int32_t& lo,
                                          int32_t& hi)
{
    int vmin = INT32_MAX, vmax = INT32_MIN;
    if (k1 - k0 + 1 == FA_BLOCK_SIZE && (k0 & 3) == 0) {
        const int4 v = __ldg(reinterpret_cast<const int4*>(doc_row + k0) + lane);
        vmin = min(min(v.x, v.y), min(v.z, v.w));
        vmax = max(max(v.x, v.y), max(v.z, v.w));
    } else {
        for (int64_t kv = k0 + lane; kv <= k1; kv += 32) {
            const int d = __ldg(doc_row + kv);
            vmin = min(vmin, d);
            vmax = max(vmax, d);
        }
    }
    lo = warp_min(vmin);
    hi = warp_max(vmax);
}

// kv blocks are classified in chunks, so the per-block scratch stays bounded
constexpr int kChunk = 2048;

__global__ void __launch_bounds__(kThreads) block_mask_kernel(BlockMaskLaunch p)
{
    extern __shared__ uint8_t cls[];  // [nkv]: 0 empty, 1 partial, 2 full
    __shared__ int s_qmin[kWarps], s_qmax[kWarps];
    __shared__ int32_t s_kmin[kChunk], s_kmax[kChunk];  // document-id range of each kv block of the chunk
    __shared__ int32_t s_mixed[kChunk];                 // kv blocks the summaries leave undecided
    __shared__ int s_nmixed;
    __shared__ __align__(16) int32_t s_kdoc[kWarps][FA_BLOCK_SIZE];  // a mixed tile's kv document ids, per warp

    const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const MaskParams& m = p.mask;
    const int32_t* doc_row = m.has_doc ? m.doc_ids + (int64_t)b * m.doc_stride : nullptr;

    // query positions of this block (rows plus the mask's offset)
    const int64_t q0 = (int64_t)qb * FA_BLOCK_SIZE + m.q_offset;
    const int64_t q1 = min((int64_t)qb * FA_BLOCK_SIZE + FA_BLOCK_SIZE, p.q_len) - 1 + m.q_offset;

    // document-id range of this query block
    int32_t qmin = 0, qmax = 0;
    if (m.has_doc) {
        if (warp == 0) {
            int32_t lo, hi;
            doc_range(doc_row, q0, q1, lane, lo, hi);
            if (lane == 0) { s_qmin[0] = lo; s_qmax[0] = hi; }
        }
        __syncthreads();
        qmin = s_qmin[0];
        qmax = s_qmax[0];
    }

    for (int c0 = 0; c0 < p.nkv; c0 += kChunk) {
        const int cn = min(kChunk, p.nkv - c0);
        if (threadIdx.x == 0) s_nmixed = 0;
        // 1. document-id ranges of the chunk's kv blocks: each warp issues the
        //    loads of four blocks before reducing any of them
        if (m.has_doc) {
            for (int i0 = warp; i0 < cn; i0 += 4 * kWarps) {
                int4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = i0 + u * kWarps;
                    const int64_t k0 = (int64_t)(c0 + i) * FA_BLOCK_SIZE;
                    v[u] = make_int4(0, 0, 0, 0);
                    if (i < cn && k0 + FA_BLOCK_SIZE <= p.kv_len)
                        v[u] = __ldg(reinterpret_cast<const int4*>(doc_row + k0) + lane);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = i0 + u * kWarps;
                    if (i >= cn) break;
                    const int64_t k0 = (int64_t)(c0 + i) * FA_BLOCK_SIZE;
                    int32_t lo, hi;
                    if (k0 + FA_BLOCK_SIZE <= p.kv_len) {
                        lo = warp_min(min(min(v[u].x, v[u].y), min(v[u].z, v[u].w)));
                        hi = warp_max(max(max(v[u].x, v[u].y), max(v[u].z, v[u].w)));
                    } else {
                        doc_range(doc_row, k0, p.kv_len - 1, lane, lo, hi);
                    }
                    if (lane == 0) { s_kmin[i] = lo; s_kmax[i] = hi; }
                }
            }
        }
        __syncthreads();
        // 2. one thread per kv block: the per-leaf summaries decide most tiles
        for (int i = threadIdx.x; i < cn; i += kThreads) {
            const int64_t k0 = (int64_t)(c0 + i) * FA_BLOCK_SIZE;
            const int64_t k1 = min(k0 + FA_BLOCK_SIZE, p.kv_len) - 1;
            const int32_t kmin = m.has_doc ? s_kmin[i] : 0, kmax = m.has_doc ? s_kmax[i] : 0;
            const int sm = mask_summary(m, q0, q1, k0, k1, qmin, qmax, kmin, kmax);
            if (sm == SUM_TRUE) cls[c0 + i] = 2;
            else if (sm == SUM_FALSE) cls[c0 + i] = 0;
            else s_mixed[atomicAdd(&s_nmixed, 1)] = c0 + i;
        }
        __syncthreads();
        // 3. undecided tiles, one warp per tile: each lane builds the 128-bit mask
        //    words of one row at a time and counts their bits; 32 rows at a time,
        //    the warp stops as soon as it has seen an admitted and a masked
        //    position (partial), else it has counted every position
        const int nmixed = s_nmixed;
        for (int i = warp; i < nmixed; i += kWarps) {
            const int kb = s_mixed[i];
            const int64_t k0 = (int64_t)kb * FA_BLOCK_SIZE;
            const int64_t k1 = min(k0 + FA_BLOCK_SIZE, p.kv_len) - 1;
            int32_t* kd = s_kdoc[warp];
            if (m.has_doc) {
                __syncwarp();
                for (int j = lane; j < FA_BLOCK_SIZE; j += 32) kd[j] = (k0 + j <= k1) ? doc_row[k0 + j] : INT32_MIN;
                __syncwarp();
            }
            const int ncols = (int)(k1 - k0 + 1);
            bool seen_in = false, seen_out = false;
            for (int64_t qr = q0; qr <= q1; qr += 32) {
                const int64_t q = qr + lane;
                if (q <= q1) {
                    uint32_t db[4] = {0u, 0u, 0u, 0u};
                    if (m.has_doc) {
                        const int32_t qd = doc_row[q];
                        const int4* kd4 = reinterpret_cast<const int4*>(kd);
#pragma unroll 8
                        for (int j4 = 0; j4 < FA_BLOCK_SIZE / 4; ++j4) {
                            const int4 d4 = kd4[j4];
                            const uint32_t bits = (uint32_t)(d4.x == qd) | ((uint32_t)(d4.y == qd) << 1) |
                                                  ((uint32_t)(d4.z == qd) << 2) | ((uint32_t)(d4.w == qd) << 3);
                            db[j4 >> 3] |= bits << ((4 * j4) & 31);
                        }
                    }
                    uint32_t w[4];
                    row_mask_words(m, q, k0, p.kv_len, db, w);
                    const int a = __popc(w[0]) + __popc(w[1]) + __popc(w[2]) + __popc(w[3]);
                    seen_in |= a > 0;
                    seen_out |= a < ncols;
                }
                seen_in = __any_sync(0xFFFFFFFFu, seen_in);
                seen_out = __any_sync(0xFFFFFFFFu, seen_out);
                if (seen_in && seen_out) break;
            }
            if (lane == 0) cls[kb] = !seen_in ? 0 : (seen_out ? 1 : 2);
        }
        __syncthreads();
    }

    // ordered compaction by warp 0: ballots over 32 kv blocks at a time
    if (warp == 0) {
        const int64_t row = ((int64_t)b * p.H + h) * p.nq + qb;
        int32_t* part_idx = p.kv_indices + row * p.nkv;
        int32_t* full_idx = p.full_kv_indices + row * p.nkv;
        int n_part = 0, n_full = 0;
        for (int base = 0; base < p.nkv; base += 32) {
            int kb = base + lane;
            uint8_t c = kb < p.nkv ? cls[kb] : 0;
            if (!p.split_full && c == 2) c = 1;  // no split: every non-empty tile is listed as partial
            uint32_t bp = __ballot_sync(0xFFFFFFFFu, c == 1);
            uint32_t bf = __ballot_sync(0xFFFFFFFFu, c == 2);
            uint32_t below = (1u << lane) - 1u;
            if (c == 1) part_idx[n_part + __popc(bp & below)] = kb;
            if (c == 2) full_idx[n_full + __popc(bf & below)] = kb;
            n_part += __popc(bp);
            n_full += __popc(bf);
        }
        // unused slots are 0
        for (int i = n_part + lane; i < p.nkv; i += 32) part_idx[i] = 0;
        for (int i = n_full + lane; i < p.nkv; i += 32) full_idx[i] = 0;
        if (lane == 0) {
            p.kv_num_blocks[row] = n_part;
            p.full_kv_num_blocks[row] = n_full;
        }
    }
}

// Does the ascending list `lst` of length n contain kb?  (Binary search.)
__device__ __forceinline__ bool list_has(const int32_t* lst, int n, int kb)
{
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int v = __ldg(lst + mid);
        if (v == kb) return true;
        if (v < kb) lo = mid + 1;
        else hi = mid;
    }
    return false;
}

// Transposed view of one kv block kb: lane i looks kb up in the partial and full
// lists of query block base + i; ballots compact the query blocks in ascending
// order.  Rows of the forward lists are read with clamped counts, so a corrupt
// count cannot move a read outside its row.
__global__ void __launch_bounds__(32) block_mask_transpose_kernel(TransposeLaunch p)
{
    const int kb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int lane = threadIdx.x;
    const int64_t bh = (int64_t)b * p.H + h;
    const int64_t out_row = bh * p.nkv + kb;
    int32_t* part_out = p.q_indices + out_row * p.nq;
    int32_t* full_out = p.full_q_indices + out_row * p.nq;
    int n_part = 0, n_full = 0;
    for (int base = 0; base < p.nq; base += 32) {
        const int qb = base + lane;
        int c = 0;  // 0 empty, 1 partial, 2 full
        if (qb < p.nq) {
            const int64_t row = bh * p.nq + qb;
            const int np = min(max(__ldg(p.kv_num_blocks + row), 0), p.nkv);
            if (list_has(p.kv_indices + row * p.nkv, np, kb)) c = 1;
            if (c == 0 && p.has_full) {
                const int nf = min(max(__ldg(p.full_kv_num_blocks + row), 0), p.nkv);
                if (list_has(p.full_kv_indices + row * p.nkv, nf, kb)) c = 2;
            }
        }
        const uint32_t bp = __ballot_sync(0xFFFFFFFFu, c == 1);
        const uint32_t bf = __ballot_sync(0xFFFFFFFFu, c == 2);
        const uint32_t below = (1u << lane) - 1u;
        if (c == 1) part_out[n_part + __popc(bp & below)] = qb;
        if (c == 2) full_out[n_full + __popc(bf & below)] = qb;
        n_part += __popc(bp);
        n_full += __popc(bf);
    }
    for (int i = n_part + lane; i < p.nq; i += 32) part_out[i] = 0;
    for (int i = n_full + lane; i < p.nq; i += 32) full_out[i] = 0;
    if (lane == 0) {
        p.q_num_blocks[out_row] = n_part;
        p.full_q_num_blocks[out_row] = n_full;
    }
}

} // namespace

cudaError_t launch_block_mask_transpose(const TransposeLaunch& p, int B, cudaStream_t stream)
{
    if (p.nkv == 0 || B == 0 || p.H == 0) return cudaSuccess;
    dim3 grid((unsigned)p.nkv, (unsigned)p.H, (unsigned)B);
    block_mask_transpose_kernel<<<grid, 32, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_block_mask(const BlockMaskLaunch& p, int B, cudaStream_t stream)
{
    if (p.nq == 0 || B == 0 || p.H == 0) return cudaSuccess;
    dim3 grid((unsigned)p.nq, (unsigned)p.H, (unsigned)B);
    size_t smem = (size_t)(p.nkv > 0 ? p.nkv : 1);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(block_mask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    block_mask_kernel<<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

} // namespace fa
