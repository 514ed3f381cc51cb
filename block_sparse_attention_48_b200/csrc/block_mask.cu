// create_block_mask on the GPU ("Concepts", BlockMask Internals; paper review
// sec. 4.1-4.2): classify every 128 x 128 tile of the (q, kv) plane as full,
// partial or empty over its in-range positions and emit the ascending lists of
// partial (kv_indices) and full (full_kv_indices) kv blocks of each query block.
//
// One CTA per BlockMask row (b, h, qb); one warp per kv tile at a time.  Each
// tile is first summarised leaf by leaf (interval leaves exactly, the document
// leaf from its id ranges); only tiles the summaries leave undecided are
// counted position by position, as 128-bit mask words per row.  Both routes
// give the same class, so the result is the exact classification.
#include <cuda_runtime.h>

#include "block_mask.cuh"
#include "mask_eval.cuh"
#include "ptx.cuh"

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

__device__ __forceinline__ long long warp_sum(long long v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

__global__ void __launch_bounds__(kThreads) block_mask_kernel(BlockMaskLaunch p)
{
    extern __shared__ uint8_t cls[];  // [nkv]: 0 empty, 1 partial, 2 full
    __shared__ int s_qmin[kWarps], s_qmax[kWarps];
    __shared__ int32_t s_kdoc[kWarps][FA_BLOCK_SIZE];  // a mixed tile's kv document ids, per warp

    // the forward kernel that usually follows may start its prologue now
    grid_launch_dependents();

    const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const MaskParams& m = p.mask;
    const int32_t* doc_row = m.has_doc ? m.doc_ids + (int64_t)b * m.doc_stride : nullptr;

    const int64_t q0 = (int64_t)qb * FA_BLOCK_SIZE;
    const int64_t q1 = min(q0 + FA_BLOCK_SIZE, p.q_len) - 1;

    // document-id range of this query block
    int32_t qmin = 0, qmax = 0;
    if (m.has_doc) {
        int vmin = INT32_MAX, vmax = INT32_MIN;
        for (int64_t q = q0 + threadIdx.x; q <= q1; q += kThreads) {
            int d = doc_row[q];
            vmin = min(vmin, d);
            vmax = max(vmax, d);
        }
        vmin = warp_min(vmin);
        vmax = warp_max(vmax);
        if (lane == 0) { s_qmin[warp] = vmin; s_qmax[warp] = vmax; }
        __syncthreads();
        qmin = s_qmin[0];
        qmax = s_qmax[0];
        for (int w = 1; w < kWarps; ++w) { qmin = min(qmin, s_qmin[w]); qmax = max(qmax, s_qmax[w]); }
    }

    for (int kb = warp; kb < p.nkv; kb += kWarps) {
        const int64_t k0 = (int64_t)kb * FA_BLOCK_SIZE;
        const int64_t k1 = min(k0 + FA_BLOCK_SIZE, p.kv_len) - 1;
        int32_t kmin = 0, kmax = 0;
        if (m.has_doc) {
            int vmin = INT32_MAX, vmax = INT32_MIN;
            for (int64_t kv = k0 + lane; kv <= k1; kv += 32) {
                int d = doc_row[kv];
                vmin = min(vmin, d);
                vmax = max(vmax, d);
            }
            kmin = warp_min(vmin);
            kmax = warp_max(vmax);
        }
        int s = mask_summary(m, q0, q1, k0, k1, qmin, qmax, kmin, kmax);
        uint8_t c;
        if (s == SUM_TRUE) c = 2;
        else if (s == SUM_FALSE) c = 0;
        else {
            // count every in-range position: each lane builds the 128-bit mask
            // words of four rows (kv >= kv_len already cleared) and counts bits
            int32_t* kd = s_kdoc[warp];
            if (m.has_doc) {
                __syncwarp();
                for (int j = lane; j < FA_BLOCK_SIZE; j += 32) kd[j] = (k0 + j <= k1) ? doc_row[k0 + j] : INT32_MIN;
                __syncwarp();
            }
            long long admitted = 0;
            for (int64_t q = q0 + lane; q <= q1; q += 32) {
                uint32_t db[4] = {0u, 0u, 0u, 0u};
                if (m.has_doc) {
                    const int32_t qd = doc_row[q];
                    for (int j = 0; j < FA_BLOCK_SIZE; ++j) db[j >> 5] |= (uint32_t)(kd[j] == qd) << (j & 31);
                }
                uint32_t w[4];
                row_mask_bits(m, q, k0, p.kv_len, db, w);
                admitted += __popc(w[0]) + __popc(w[1]) + __popc(w[2]) + __popc(w[3]);
            }
            admitted = warp_sum(admitted);
            long long total = (long long)(q1 - q0 + 1) * (long long)(k1 - k0 + 1);
            c = admitted == 0 ? 0 : (admitted == total ? 2 : 1);
        }
        if (lane == 0) cls[kb] = c;
    }
    __syncthreads();

    // ordered compaction by warp 0: ballots over 32 kv blocks at a time
    if (warp == 0) {
        const int64_t row = ((int64_t)b * p.H + h) * p.nq + qb;
        int32_t* part_idx = p.kv_indices + row * p.nkv;
        int32_t* full_idx = p.full_kv_indices + row * p.nkv;
        int n_part = 0, n_full = 0;
        for (int base = 0; base < p.nkv; base += 32) {
            int kb = base + lane;
            uint8_t c = kb < p.nkv ? cls[kb] : 0;
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

} // namespace

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
