// Host implementation of the C ABI in flexattn.h: argument validation, TMA
// descriptor encoding and kernel launches.  Nothing here allocates device memory
// or synchronises the host (except fa_get_device_status).
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include <cuda.h>
#include <cuda_runtime.h>

#include "block_mask.cuh"
#include "flex_bwd.cuh"
#include "flex_decode.cuh"
#include "flex_fwd.cuh"
#include "flexattn.h"
#include "tmap.cuh"

namespace {

constexpr int64_t kMaxLen = (int64_t(1) << 31) - 256;  // q_len / kv_len bound (int32 tile coordinates)
constexpr size_t kWorkspaceBytes = 256;
constexpr int kMaxNkv = 200000;                        // BlockMask build keeps one byte per kv block in smem

uint64_t g_watchdog_ns = 2000ull * 1000ull * 1000ull;
int g_selftest_stall = 0;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

int check_mask_desc(const fa_mask_desc* m, int64_t q_len, int64_t kv_len)
{
    if (!m) return FA_ERR_INVALID_ARG;
    if (m->n_leaves < 0 || m->n_leaves > FA_MAX_LEAVES) return FA_ERR_INVALID_ARG;
    if (m->op != FA_MASK_AND && m->op != FA_MASK_OR) return FA_ERR_INVALID_ARG;
    bool doc = false;
    for (int i = 0; i < m->n_leaves; ++i) {
        switch (m->kind[i]) {
        case FA_LEAF_CAUSAL:
        case FA_LEAF_SLIDING:
        case FA_LEAF_PREFIX:
            break;
        case FA_LEAF_DOCUMENT:
            doc = true;
            break;
        default:
            return FA_ERR_INVALID_ARG;
        }
    }
    if (m->q_offset < 0 || m->q_offset > kMaxLen - q_len) return FA_ERR_INVALID_ARG;
    if (doc) {
        const int64_t q_end = m->q_offset + q_len;
        if (!m->doc_ids || !aligned16(m->doc_ids)) return FA_ERR_INVALID_ARG;
        if (m->doc_stride < 0 || (m->doc_stride % 4) != 0) return FA_ERR_INVALID_ARG;
        if (m->doc_len < (q_end > kv_len ? q_end : kv_len)) return FA_ERR_INVALID_ARG;
    }
    return FA_OK;
}

fa::MaskParams to_params(const fa_mask_desc& m)
{
    fa::MaskParams p;
    std::memset(&p, 0, sizeof p);
    p.n_leaves = m.n_leaves;
    p.op = m.op;
    p.has_doc = 0;
    for (int i = 0; i < FA_MAX_LEAVES; ++i) {
        p.kind[i] = i < m.n_leaves ? m.kind[i] : -1;
        p.param[i] = i < m.n_leaves ? m.param[i] : 0;
        if (i < m.n_leaves && m.kind[i] == FA_LEAF_DOCUMENT) p.has_doc = 1;
    }
    p.doc_ids = p.has_doc ? m.doc_ids : nullptr;
    p.doc_stride = m.doc_stride;
    p.q_offset = m.q_offset;
    return p;
}

// A [B, H, S, D] bf16 tensor usable as a TMA source / 16-byte-vector target.  A
// stride of 0 (a broadcast, expanded dimension) is accepted only on a dimension of
// size 1: the tiles are addressed by coordinates, so an expanded dimension would
// read other data than the caller's.
int check_tensor(const fa_tensor* t)
{
    if (!t) return FA_ERR_INVALID_ARG;
    bool empty = false;
    for (int i = 0; i < 4; ++i) {
        if (t->dims[i] < 0) return FA_ERR_INVALID_ARG;
        empty |= t->dims[i] == 0;
    }
    if (empty) return FA_OK;  // never accessed
    if (!t->data) return FA_ERR_INVALID_ARG;
    if (t->strides[3] != 1) return FA_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i) {
        if (t->strides[i] < 0 || (t->strides[i] % 8) != 0) return FA_ERR_INVALID_ARG;
        if (t->strides[i] == 0 && t->dims[i] > 1) return FA_ERR_INVALID_ARG;
    }
    if (!aligned16(t->data)) return FA_ERR_INVALID_ARG;
    return FA_OK;
}

bool tmap_for(CUtensorMap* map, const fa_tensor* t)
{
    // dims innermost first: (D, S, H, B); strides of S, H, B in bytes
    uint64_t dims[4] = {(uint64_t)t->dims[3], (uint64_t)t->dims[2], (uint64_t)t->dims[1], (uint64_t)t->dims[0]};
    uint64_t st[3] = {(uint64_t)t->strides[2] * 2, (uint64_t)t->strides[1] * 2, (uint64_t)t->strides[0] * 2};
    // the CUDA driver wants every stride nonzero: give size-1 dimensions (the only
    // ones check_tensor lets have stride 0) a legal one
    for (int i = 0; i < 3; ++i)
        if (st[i] == 0) st[i] = 16;
    return fa::make_tmap_bf16_4d(map, t->data, dims, st, 128);
}

} // namespace

namespace {

int create_block_mask(const fa_mask_desc* m, int B, int H, int64_t q_len, int64_t kv_len, int block_size,
                      fa_block_mask* bm, void* stream, bool split_full)
{
    if (!bm || B < 1 || H < 1 || B > 65535 || H > 65535) return FA_ERR_INVALID_ARG;  // grid y / z extents
    int32_t nq = 0, nkv = 0;
    int rc = fa_block_mask_shape(q_len, kv_len, block_size, &nq, &nkv);
    if (rc != FA_OK) return rc;
    rc = check_mask_desc(m, q_len, kv_len);
    if (rc != FA_OK) return rc;
    if (nkv > kMaxNkv) return FA_ERR_UNSUPPORTED;
    if ((int64_t)B * H * nq > INT32_MAX / 2) return FA_ERR_UNSUPPORTED;
    if (nq > 0 && (!bm->kv_num_blocks || !bm->full_kv_num_blocks)) return FA_ERR_INVALID_ARG;
    if (nq > 0 && nkv > 0 && (!bm->kv_indices || !bm->full_kv_indices)) return FA_ERR_INVALID_ARG;
    // the transposed view is requested by setting its pointers; arrays of zero size may stay NULL
    const bool transposed = bm->q_num_blocks || bm->q_indices || bm->full_q_num_blocks || bm->full_q_indices;
    if (transposed && nkv > 0 && (!bm->q_num_blocks || !bm->full_q_num_blocks)) return FA_ERR_INVALID_ARG;
    if (transposed && nq > 0 && nkv > 0 && (!bm->q_indices || !bm->full_q_indices)) return FA_ERR_INVALID_ARG;
    if ((int64_t)B * H * nkv > INT32_MAX / 2) return FA_ERR_UNSUPPORTED;
    // a per-batch document layout needs one BlockMask row per batch
    bool doc = false;
    for (int i = 0; i < m->n_leaves; ++i) doc |= m->kind[i] == FA_LEAF_DOCUMENT;

    bm->B = B;
    bm->H = H;
    bm->nq = nq;
    bm->nkv = nkv;
    bm->block_size = block_size;
    bm->has_full = split_full ? 1 : 0;
    bm->q_len = q_len;
    bm->kv_len = kv_len;
    bm->mask = *m;
    if (!doc) {
        bm->mask.doc_ids = nullptr;
        bm->mask.doc_stride = 0;
        bm->mask.doc_len = 0;
    }

    fa::BlockMaskLaunch L;
    L.mask = to_params(*m);
    L.q_len = q_len;
    L.kv_len = kv_len;
    L.H = H;
    L.nq = nq;
    L.nkv = nkv;
    L.kv_num_blocks = bm->kv_num_blocks;
    L.kv_indices = bm->kv_indices;
    L.full_kv_num_blocks = bm->full_kv_num_blocks;
    L.full_kv_indices = bm->full_kv_indices;
    L.split_full = split_full ? 1 : 0;
    cudaError_t e = fa::launch_block_mask(L, B, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return FA_ERR_CUDA;
    if (transposed) {
        fa::TransposeLaunch T;
        T.H = H;
        T.nq = nq;
        T.nkv = nkv;
        T.has_full = bm->has_full;
        T.kv_num_blocks = bm->kv_num_blocks;
        T.kv_indices = bm->kv_indices;
        T.full_kv_num_blocks = bm->full_kv_num_blocks;
        T.full_kv_indices = bm->full_kv_indices;
        T.q_num_blocks = bm->q_num_blocks;
        T.q_indices = bm->q_indices;
        T.full_q_num_blocks = bm->full_q_num_blocks;
        T.full_q_indices = bm->full_q_indices;
        e = fa::launch_block_mask_transpose(T, B, static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return FA_ERR_CUDA;
    }
    return FA_OK;
}

} // namespace

namespace {

// fa_forward and fa_forward_paged.  With a page table, k and v are page pools
// [num_pages, Hkv, 128, D] and the logical kv length comes from the BlockMask.
int forward_impl(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const int32_t* page_table,
                 int64_t pt_stride, const fa_block_mask* bm, const fa_score_mod* sm, float scale, const fa_tensor* o,
                 float* lse, void* workspace, size_t workspace_bytes, void* stream)
{
    int rc;
    if ((rc = check_tensor(q)) || (rc = check_tensor(k)) || (rc = check_tensor(v)) || (rc = check_tensor(o))) return rc;
    if (!bm || !workspace || workspace_bytes < kWorkspaceBytes || !aligned16(workspace)) return FA_ERR_INVALID_ARG;

    const bool paged = page_table != nullptr;
    const int64_t B = q->dims[0], Hq = q->dims[1], q_len = q->dims[2], D = q->dims[3];
    const int64_t Hkv = k->dims[1], kv_len = paged ? bm->kv_len : k->dims[2];
    const int64_t num_pages = paged ? k->dims[0] : 0;
    if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
    for (int i = 0; i < 4; ++i)
        if (o->dims[i] != q->dims[i]) return FA_ERR_INVALID_ARG;
    for (int i = 0; i < 4; ++i)
        if (v->dims[i] != k->dims[i]) return FA_ERR_INVALID_ARG;
    if (k->dims[3] != D) return FA_ERR_INVALID_ARG;
    if (paged) {
        if (k->dims[2] != FA_BLOCK_SIZE || kv_len < 0 || (kv_len > 0 && num_pages < 1)) return FA_ERR_INVALID_ARG;
        if (pt_stride < (kv_len + FA_BLOCK_SIZE - 1) / FA_BLOCK_SIZE || num_pages > INT32_MAX) return FA_ERR_INVALID_ARG;
    } else if (k->dims[0] != B) {
        return FA_ERR_INVALID_ARG;
    }
    if (Hkv < 1 || Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
    if (q_len > kMaxLen || kv_len > kMaxLen || B > 65535 || Hq > 65535) return FA_ERR_INVALID_ARG;
    if (bm->block_size != FA_BLOCK_SIZE) return FA_ERR_UNSUPPORTED;
    if (bm->q_len != q_len || bm->kv_len != kv_len) return FA_ERR_INVALID_ARG;
    if ((bm->B != 1 && bm->B != B) || (bm->H != 1 && bm->H != Hq)) return FA_ERR_INVALID_ARG;
    int32_t nq = 0, nkv = 0;
    if ((rc = fa_block_mask_shape(q_len, kv_len, FA_BLOCK_SIZE, &nq, &nkv)) != FA_OK) return rc;
    if (bm->nq != nq || bm->nkv != nkv) return FA_ERR_INVALID_ARG;
    if ((rc = check_mask_desc(&bm->mask, q_len, kv_len)) != FA_OK) return rc;
    fa::MaskParams mp = to_params(bm->mask);
    if (mp.has_doc && bm->mask.doc_stride != 0 && bm->B != B && B > 1) return FA_ERR_INVALID_ARG;
    if (nq > 0 && (!bm->kv_num_blocks || (bm->has_full && !bm->full_kv_num_blocks))) return FA_ERR_INVALID_ARG;
    if (nq > 0 && nkv > 0 && (!bm->kv_indices || (bm->has_full && !bm->full_kv_indices))) return FA_ERR_INVALID_ARG;
    const int64_t items = B * Hq * nq;
    if (items > (int64_t(1) << 30)) return FA_ERR_UNSUPPORTED;

    const int kind = sm ? sm->kind : FA_SCORE_NONE;
    if (kind < FA_SCORE_NONE || kind > FA_SCORE_BIAS_SOFTCAP) return FA_ERR_INVALID_ARG;
    const bool has_bias = kind == FA_SCORE_BIAS || kind == FA_SCORE_BIAS_SOFTCAP;
    const bool has_cap = kind == FA_SCORE_SOFTCAP || kind == FA_SCORE_BIAS_SOFTCAP;
    if (kind == FA_SCORE_ALIBI && !sm->alibi_slopes) return FA_ERR_INVALID_ARG;
    if (has_cap && !(sm->softcap > 0.f)) return FA_ERR_INVALID_ARG;
    if (has_bias) {
        if (!sm->bias || !aligned16(sm->bias) || sm->bias_strides[3] != 1) return FA_ERR_INVALID_ARG;
        for (int i = 0; i < 3; ++i)
            if (sm->bias_strides[i] < 0 || sm->bias_strides[i] % 8 != 0) return FA_ERR_INVALID_ARG;
        // stride 0 broadcasts over the batch or the heads; not over the queries
        if (sm->bias_strides[2] == 0 && q_len > 1) return FA_ERR_INVALID_ARG;
    }
    if (items == 0) return FA_OK;  // nothing to compute (empty batch, heads or queries)

    fa::FwdParams P;
    std::memset(&P, 0, sizeof P);
    if (!tmap_for(&P.tm_q, q)) return FA_ERR_INVALID_ARG;
    if (kv_len > 0) {
        if (!tmap_for(&P.tm_k, k) || !tmap_for(&P.tm_v, v)) return FA_ERR_INVALID_ARG;
    } else {
        P.tm_k = P.tm_q;  // never read: every row has zero kv blocks
        P.tm_v = P.tm_q;
    }
    if (has_bias && kv_len > 0) {
        // a broadcast (stride 0) batch or head dimension is mapped as size 1 and
        // read at coordinate 0
        P.bias_b_bcast = sm->bias_strides[0] == 0 ? 1 : 0;
        P.bias_h_bcast = sm->bias_strides[1] == 0 ? 1 : 0;
        uint64_t dims[4] = {(uint64_t)kv_len, (uint64_t)q_len, P.bias_h_bcast ? 1u : (uint64_t)Hq,
                            P.bias_b_bcast ? 1u : (uint64_t)B};
        uint64_t st[3] = {(uint64_t)sm->bias_strides[2] * 2, (uint64_t)sm->bias_strides[1] * 2,
                          (uint64_t)sm->bias_strides[0] * 2};
        for (int i = 0; i < 3; ++i)
            if (st[i] == 0) st[i] = 16;
        if (!fa::make_tmap_bf16_4d(&P.tm_bias, sm->bias, dims, st, 128)) return FA_ERR_INVALID_ARG;
    } else {
        P.tm_bias = P.tm_q;
    }
    P.B = (int32_t)B;
    P.Hq = (int32_t)Hq;
    P.Hkv = (int32_t)Hkv;
    P.G = (int32_t)(Hq / Hkv);
    P.q_len = q_len;
    P.kv_len = kv_len;
    P.nq = nq;
    P.nkv = nkv;
    P.num_items = (int32_t)items;
    P.kv_num = bm->kv_num_blocks;
    P.kv_idx = bm->kv_indices;
    P.full_num = bm->full_kv_num_blocks;
    P.full_idx = bm->full_kv_indices;
    P.bm_B = bm->B;
    P.bm_H = bm->H;
    P.has_full = bm->has_full ? 1 : 0;
    // Rows are ranked by tile count in the kernel only for masks whose counts are
    // not already ordered by query block: a DOCUMENT leaf.  Interval leaves
    // (causal, window, prefix) give counts that grow with the query block, so the
    // query-block-descending order is already longest first, and the ranking's
    // start-up (a global read and two CTA barriers) measured 4 us on the causal
    // workload.  num_rows = 0 selects the query-block-descending order.
    P.num_rows = mp.has_doc ? bm->B * bm->H * nq : 0;
    P.mask = mp;
    const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)D);
    P.scale_log2 = sc * 1.4426950408889634f;
    if (has_cap) {
        P.softcap = sm->softcap;
        P.softcap_in = sc / sm->softcap;
        P.softcap_inv = 1.0f / sm->softcap;
        P.softcap_out = sm->softcap * 1.4426950408889634f;
    }
    P.slopes = kind == FA_SCORE_ALIBI ? sm->alibi_slopes : nullptr;
    P.o = static_cast<uint16_t*>(o->data);
    P.o_stride_b = o->strides[0];
    P.o_stride_h = o->strides[1];
    P.o_stride_s = o->strides[2];
    P.lse = lse;
    P.page_table = page_table;
    P.pt_stride = pt_stride;
    P.num_pages = (int32_t)num_pages;
    P.status = static_cast<int*>(workspace);
    P.watchdog_ns = g_watchdog_ns;
    P.selftest_stall = g_selftest_stall;

    const int sms = sm_count();
    if (sms <= 0) return FA_ERR_CUDA;
    const int64_t pairs = (items + 1) / 2;
    const int grid = (int)(pairs < sms ? pairs : sms);
    const int ext = (mp.has_doc ? fa::kExtRank | fa::kExtPage : 0) | (paged ? fa::kExtPage : 0);
    cudaError_t e = fa::launch_flex_forward(P, (int)D, kind, ext, grid, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

} // namespace

extern "C" {

const char* fa_status_string(int status)
{
    switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_BAD_BLOCKMASK: return "FA_ERR_BAD_BLOCKMASK";
    default: return "FA_ERR_UNKNOWN";
    }
}

int fa_set_watchdog_ms(int ms)
{
    if (ms < 0) return FA_ERR_INVALID_ARG;
    g_watchdog_ns = (ms == 0 ? 2000ull : (uint64_t)ms) * 1000ull * 1000ull;
    return FA_OK;
}

int fa_set_selftest_stall(int on)
{
    g_selftest_stall = on ? 1 : 0;
    return FA_OK;
}

int fa_block_mask_shape(int64_t q_len, int64_t kv_len, int block_size, int32_t* nq, int32_t* nkv)
{
    if (!nq || !nkv || q_len < 0 || kv_len < 0 || q_len > kMaxLen || kv_len > kMaxLen) return FA_ERR_INVALID_ARG;
    if (block_size != FA_BLOCK_SIZE) return FA_ERR_UNSUPPORTED;
    *nq = (int32_t)((q_len + FA_BLOCK_SIZE - 1) / FA_BLOCK_SIZE);
    *nkv = (int32_t)((kv_len + FA_BLOCK_SIZE - 1) / FA_BLOCK_SIZE);
    return FA_OK;
}

int fa_create_block_mask(const fa_mask_desc* m, int B, int H, int64_t q_len, int64_t kv_len, int block_size,
                         fa_block_mask* bm, void* stream)
{
    return create_block_mask(m, B, H, q_len, kv_len, block_size, bm, stream, true);
}

int fa_create_block_mask_unsplit(const fa_mask_desc* m, int B, int H, int64_t q_len, int64_t kv_len, int block_size,
                                 fa_block_mask* bm, void* stream)
{
    return create_block_mask(m, B, H, q_len, kv_len, block_size, bm, stream, false);
}

size_t fa_workspace_size(void) { return kWorkspaceBytes; }

int fa_forward(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const fa_block_mask* bm,
               const fa_score_mod* sm, float scale, const fa_tensor* o, float* lse, void* workspace,
               size_t workspace_bytes, void* stream)
{
    return forward_impl(q, k, v, nullptr, 0, bm, sm, scale, o, lse, workspace, workspace_bytes, stream);
}

int fa_forward_paged(const fa_tensor* q, const fa_tensor* k_pages, const fa_tensor* v_pages, const int32_t* page_table,
                     int64_t page_table_stride, const fa_block_mask* bm, const fa_score_mod* sm, float scale,
                     const fa_tensor* o, float* lse, void* workspace, size_t workspace_bytes, void* stream)
{
    if (!page_table) return FA_ERR_INVALID_ARG;
    return forward_impl(q, k_pages, v_pages, page_table, page_table_stride, bm, sm, scale, o, lse, workspace,
                        workspace_bytes, stream);
}

// Backward workspace: the status word, Delta [B, Hq, q_len] fp32 and the dQ
// accumulator [B, Hq, q_len, D] fp32, each 256-byte aligned relative to the base.
// Backward workspace: the status word, then per 128-row query block of every
// (batch, head) its LSE (log2 units) and Delta rows ([2][128] fp32), then the fp32
// dQ accumulator over the same padded rows.
static size_t bwd_ld_offset() { return kWorkspaceBytes; }

static size_t bwd_acc_offset(int64_t blocks) { return bwd_ld_offset() + (size_t)blocks * 256 * sizeof(float); }

size_t fa_backward_workspace_size(int64_t B, int64_t Hq, int64_t q_len, int64_t D)
{
    if (B < 0 || Hq < 0 || q_len < 0 || D < 0) return 0;
    const int64_t blocks = B * Hq * ((q_len + FA_BLOCK_SIZE - 1) / FA_BLOCK_SIZE);
    return bwd_acc_offset(blocks) + (size_t)blocks * FA_BLOCK_SIZE * (size_t)D * sizeof(float);
}

int fa_backward(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const fa_tensor* o,
                const fa_tensor* dout, const float* lse, const fa_block_mask* bm, const fa_score_mod* sm, float scale,
                const fa_tensor* dq, const fa_tensor* dk, const fa_tensor* dv, void* workspace,
                size_t workspace_bytes, void* stream)
{
    int rc;
    const fa_tensor* all[8] = {q, k, v, o, dout, dq, dk, dv};
    for (const fa_tensor* t : all)
        if ((rc = check_tensor(t)) != FA_OK) return rc;
    if (!bm || !workspace || !aligned16(workspace)) return FA_ERR_INVALID_ARG;
    const int64_t B = q->dims[0], Hq = q->dims[1], q_len = q->dims[2], D = q->dims[3];
    const int64_t Hkv = k->dims[1], kv_len = k->dims[2];
    if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
    for (int i = 0; i < 4; ++i) {
        if (o->dims[i] != q->dims[i] || dout->dims[i] != q->dims[i] || dq->dims[i] != q->dims[i])
            return FA_ERR_INVALID_ARG;
        if (v->dims[i] != k->dims[i] || dk->dims[i] != k->dims[i] || dv->dims[i] != k->dims[i])
            return FA_ERR_INVALID_ARG;
    }
    if (k->dims[0] != B || k->dims[3] != D) return FA_ERR_INVALID_ARG;
    if (Hkv < 1 || Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
    if (q_len > kMaxLen || kv_len > kMaxLen || B > 65535 || Hq > 65535) return FA_ERR_INVALID_ARG;
    if (workspace_bytes < fa_backward_workspace_size(B, Hq, q_len, D)) return FA_ERR_INVALID_ARG;
    if (bm->block_size != FA_BLOCK_SIZE) return FA_ERR_UNSUPPORTED;
    if (bm->q_len != q_len || bm->kv_len != kv_len) return FA_ERR_INVALID_ARG;
    if ((bm->B != 1 && bm->B != B) || (bm->H != 1 && bm->H != Hq)) return FA_ERR_INVALID_ARG;
    int32_t nq = 0, nkv = 0;
    if ((rc = fa_block_mask_shape(q_len, kv_len, FA_BLOCK_SIZE, &nq, &nkv)) != FA_OK) return rc;
    if (bm->nq != nq || bm->nkv != nkv) return FA_ERR_INVALID_ARG;
    if ((rc = check_mask_desc(&bm->mask, q_len, kv_len)) != FA_OK) return rc;
    fa::MaskParams mp = to_params(bm->mask);
    if (mp.has_doc && bm->mask.doc_stride != 0 && bm->B != B && B > 1) return FA_ERR_INVALID_ARG;
    // the transposed view ("used in backward")
    if (nkv > 0 && (!bm->q_num_blocks || (bm->has_full && !bm->full_q_num_blocks))) return FA_ERR_INVALID_ARG;
    if (nq > 0 && nkv > 0 && (!bm->q_indices || (bm->has_full && !bm->full_q_indices))) return FA_ERR_INVALID_ARG;
    const int64_t rows = B * Hq * q_len;
    if (rows > 0 && !lse) return FA_ERR_INVALID_ARG;
    const int64_t units = B * Hkv * nkv;
    const int64_t qblocks = B * Hq * nq, rows_pad = qblocks * FA_BLOCK_SIZE;
    // the dQ reductions address padded rows by a 32-bit TMA coordinate
    if (units > INT32_MAX || rows_pad > INT32_MAX) return FA_ERR_UNSUPPORTED;

    const int kind = sm ? sm->kind : FA_SCORE_NONE;
    if (kind < FA_SCORE_NONE || kind > FA_SCORE_BIAS_SOFTCAP) return FA_ERR_INVALID_ARG;
    const bool has_bias = kind == FA_SCORE_BIAS || kind == FA_SCORE_BIAS_SOFTCAP;
    const bool has_cap = kind == FA_SCORE_SOFTCAP || kind == FA_SCORE_BIAS_SOFTCAP;
    if (kind == FA_SCORE_ALIBI && !sm->alibi_slopes) return FA_ERR_INVALID_ARG;
    if (has_cap && !(sm->softcap > 0.f)) return FA_ERR_INVALID_ARG;
    if (has_bias) {
        if (!sm->bias || sm->bias_strides[3] != 1) return FA_ERR_INVALID_ARG;
        for (int i = 0; i < 3; ++i)
            if (sm->bias_strides[i] < 0) return FA_ERR_INVALID_ARG;
    }
    if (B == 0 || Hq == 0) return FA_OK;

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* ld = reinterpret_cast<float*>(ws + bwd_ld_offset());
    float* acc = reinterpret_cast<float*>(ws + bwd_acc_offset(qblocks));
    const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)D);
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    fa::BwdPrepParams pp;
    pp.o = static_cast<const uint16_t*>(o->data);
    pp.o_st0 = o->strides[0]; pp.o_st1 = o->strides[1]; pp.o_st2 = o->strides[2];
    pp.dout = static_cast<const uint16_t*>(dout->data);
    pp.do_st0 = dout->strides[0]; pp.do_st1 = dout->strides[1]; pp.do_st2 = dout->strides[2];
    pp.lse = lse;
    pp.slopes = kind == FA_SCORE_ALIBI ? sm->alibi_slopes : nullptr;
    pp.ld = ld;
    pp.dq_acc = acc;
    pp.Hq = (int32_t)Hq;
    pp.D = (int32_t)D;
    pp.nq = nq;
    pp.q_len = q_len;
    pp.rows_pad = rows_pad;
    if (fa::launch_bwd_prep(pp, st) != cudaSuccess) return FA_ERR_CUDA;

    if (units > 0) {
        fa::BwdParams P;
        std::memset(&P, 0, sizeof P);
        if (!tmap_for(&P.tm_k, k) || !tmap_for(&P.tm_v, v)) return FA_ERR_INVALID_ARG;
        if (q_len > 0) {
            if (!tmap_for(&P.tm_q, q) || !tmap_for(&P.tm_do, dout)) return FA_ERR_INVALID_ARG;
            if (!fa::make_tmap_f32_2d_box32(&P.tm_dq, acc, (uint64_t)D, (uint64_t)rows_pad)) return FA_ERR_CUDA;
        } else {
            P.tm_q = P.tm_k;  // never read: no query block attends
            P.tm_do = P.tm_k;
            P.tm_dq = P.tm_k;
        }
        P.B = (int32_t)B;
        P.Hq = (int32_t)Hq;
        P.Hkv = (int32_t)Hkv;
        P.G = (int32_t)(Hq / Hkv);
        P.q_len = q_len;
        P.kv_len = kv_len;
        P.nq = nq;
        P.nkv = nkv;
        P.num_units = (int32_t)units;
        P.num_sms = sm_count();
        P.q_num = bm->q_num_blocks;
        P.q_idx = bm->q_indices;
        P.full_q_num = bm->full_q_num_blocks;
        P.full_q_idx = bm->full_q_indices;
        P.bm_B = bm->B;
        P.bm_H = bm->H;
        P.has_full = bm->has_full ? 1 : 0;
        P.mask = mp;
        P.score_kind = kind;
        P.scale = sc;
        if (has_cap) {
            P.softcap = sm->softcap;
            P.softcap_in = sc / sm->softcap;
            P.softcap_inv = 1.0f / sm->softcap;
        }
        P.slopes = kind == FA_SCORE_ALIBI ? sm->alibi_slopes : nullptr;
        if (has_bias) {
            P.bias = static_cast<const uint16_t*>(sm->bias);
            P.bias_st0 = sm->bias_strides[0];
            P.bias_st1 = sm->bias_strides[1];
            P.bias_st2 = sm->bias_strides[2];
        }
        P.ld = ld;
        P.dk = static_cast<uint16_t*>(dk->data);
        P.dk_st0 = dk->strides[0]; P.dk_st1 = dk->strides[1]; P.dk_st2 = dk->strides[2];
        P.dv = static_cast<uint16_t*>(dv->data);
        P.dv_st0 = dv->strides[0]; P.dv_st1 = dv->strides[1]; P.dv_st2 = dv->strides[2];
        P.status = reinterpret_cast<int*>(ws);
        P.watchdog_ns = g_watchdog_ns;
        if (fa::launch_flex_backward(P, (int)D, st) != cudaSuccess) return FA_ERR_CUDA;
    }

    fa::BwdDqParams dp;
    dp.dq_acc = acc;
    dp.dq = static_cast<uint16_t*>(dq->data);
    dp.dq_st0 = dq->strides[0]; dp.dq_st1 = dq->strides[1]; dp.dq_st2 = dq->strides[2];
    dp.Hq = (int32_t)Hq;
    dp.D = (int32_t)D;
    dp.nq = nq;
    dp.q_len = q_len;
    dp.rows = rows;
    dp.scale = sc;
    if (fa::launch_bwd_dq(dp, st) != cudaSuccess) return FA_ERR_CUDA;
    return FA_OK;
}

// Decode workspace: the status word, the length of the work list, the first /
// last CTA of every (batch, kv head) segment, then per partial result (running max, sum) and the
// unnormalised O of every packed query row, each part 256-byte aligned.
struct DecLayout {
    int64_t grid, total, seg_first, seg_last, ml, o, end;
};

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

static DecLayout dec_layout(int64_t B, int64_t Hq, int64_t Hkv, int64_t q_len, int64_t kv_len, int64_t D)
{
    const int64_t nkv = (kv_len + FA_BLOCK_SIZE - 1) / FA_BLOCK_SIZE;
    const int sms = sm_count();
    // one CTA per SM, never more CTAs than kv blocks in all
    int64_t grid = sms > 0 ? sms : 1;
    const int64_t most = B * Hkv * nkv;
    if (most < grid) grid = most < 1 ? 1 : most;
    const int64_t segs = B * Hkv, rows = (Hq / Hkv) * q_len;
    const int64_t partials = (segs + grid) * fa::kDecodeWarps * rows;
    DecLayout L;
    L.grid = grid;
    L.total = kWorkspaceBytes;
    L.seg_first = L.total + 256;
    L.seg_last = L.seg_first + align256((size_t)segs * sizeof(int32_t));
    L.ml = L.seg_last + align256((size_t)segs * sizeof(int32_t));
    L.o = L.ml + align256((size_t)partials * 2 * sizeof(float));
    L.end = L.o + (size_t)partials * D * sizeof(float);
    return L;
}

size_t fa_decode_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t q_len, int64_t kv_len, int64_t D)
{
    if (B < 0 || Hq < 0 || Hkv < 1 || q_len < 0 || kv_len < 0 || D < 0) return 0;
    if (B * Hq * q_len == 0) return kWorkspaceBytes;
    return (size_t)dec_layout(B, Hq, Hkv, q_len, kv_len, D).end;
}

int fa_decode(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const fa_block_mask* bm,
              const fa_score_mod* sm, float scale, const fa_tensor* o, float* lse, void* workspace,
              size_t workspace_bytes, void* stream)
{
    int rc;
    if ((rc = check_tensor(q)) || (rc = check_tensor(k)) || (rc = check_tensor(v)) || (rc = check_tensor(o))) return rc;
    if (!bm || !workspace || !aligned16(workspace)) return FA_ERR_INVALID_ARG;
    const int64_t B = q->dims[0], Hq = q->dims[1], q_len = q->dims[2], D = q->dims[3];
    const int64_t Hkv = k->dims[1], kv_len = k->dims[2];
    if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
    for (int i = 0; i < 4; ++i) {
        if (o->dims[i] != q->dims[i] || v->dims[i] != k->dims[i]) return FA_ERR_INVALID_ARG;
    }
    if (k->dims[0] != B || k->dims[3] != D) return FA_ERR_INVALID_ARG;
    if (Hkv < 1 || Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
    if ((Hq / Hkv) * q_len > fa::kDecodeMaxRows) return FA_ERR_UNSUPPORTED;
    if (kv_len > kMaxLen || B > 65535 || Hkv > 65535) return FA_ERR_INVALID_ARG;
    if (workspace_bytes < fa_decode_workspace_size(B, Hq, Hkv, q_len, kv_len, D)) return FA_ERR_INVALID_ARG;
    if (bm->block_size != FA_BLOCK_SIZE) return FA_ERR_UNSUPPORTED;
    if (bm->q_len != q_len || bm->kv_len != kv_len) return FA_ERR_INVALID_ARG;
    if (bm->B != 1 && bm->B != B) return FA_ERR_INVALID_ARG;
    if (bm->H != 1) return FA_ERR_UNSUPPORTED;  // the packed query heads share one BlockMask row
    int32_t nq = 0, nkv = 0;
    if ((rc = fa_block_mask_shape(q_len, kv_len, FA_BLOCK_SIZE, &nq, &nkv)) != FA_OK) return rc;
    if (bm->nq != nq || bm->nkv != nkv) return FA_ERR_INVALID_ARG;
    if ((rc = check_mask_desc(&bm->mask, q_len, kv_len)) != FA_OK) return rc;
    fa::MaskParams mp = to_params(bm->mask);
    if (mp.has_doc && bm->mask.doc_stride != 0 && bm->B != B && B > 1) return FA_ERR_INVALID_ARG;
    if (nq > 0 && (!bm->kv_num_blocks || (bm->has_full && !bm->full_kv_num_blocks))) return FA_ERR_INVALID_ARG;
    if (nq > 0 && nkv > 0 && (!bm->kv_indices || (bm->has_full && !bm->full_kv_indices))) return FA_ERR_INVALID_ARG;
    const int kind = sm ? sm->kind : FA_SCORE_NONE;
    if (kind < FA_SCORE_NONE || kind > FA_SCORE_BIAS_SOFTCAP) return FA_ERR_INVALID_ARG;
    const bool has_bias = kind == FA_SCORE_BIAS || kind == FA_SCORE_BIAS_SOFTCAP;
    const bool has_cap = kind == FA_SCORE_SOFTCAP || kind == FA_SCORE_BIAS_SOFTCAP;
    if (kind == FA_SCORE_ALIBI && !sm->alibi_slopes) return FA_ERR_INVALID_ARG;
    if (has_cap && !(sm->softcap > 0.f)) return FA_ERR_INVALID_ARG;
    if (has_bias) {
        if (!sm->bias || sm->bias_strides[3] != 1) return FA_ERR_INVALID_ARG;
        for (int i = 0; i < 3; ++i)
            if (sm->bias_strides[i] < 0) return FA_ERR_INVALID_ARG;
    }
    const int64_t rows = B * Hq * q_len;
    if (rows == 0) return FA_OK;

    fa::DecParams P;
    std::memset(&P, 0, sizeof P);
    if (kv_len > 0) {
        if (!tmap_for(&P.tm_k, k) || !tmap_for(&P.tm_v, v)) return FA_ERR_INVALID_ARG;
    }
    const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)D);
    P.q = static_cast<const uint16_t*>(q->data);
    P.q_st0 = q->strides[0]; P.q_st1 = q->strides[1]; P.q_st2 = q->strides[2];
    P.o = static_cast<uint16_t*>(o->data);
    P.o_st0 = o->strides[0]; P.o_st1 = o->strides[1]; P.o_st2 = o->strides[2];
    P.lse = lse;
    P.B = (int32_t)B;
    P.Hq = (int32_t)Hq;
    P.Hkv = (int32_t)Hkv;
    P.G = (int32_t)(Hq / Hkv);
    P.q_len = (int32_t)q_len;
    P.kv_len = kv_len;
    P.nkv = nkv;
    P.rows = (int32_t)((Hq / Hkv) * q_len);
    P.kv_num = bm->kv_num_blocks;
    P.kv_idx = bm->kv_indices;
    P.full_num = bm->full_kv_num_blocks;
    P.full_idx = bm->full_kv_indices;
    P.bm_B = bm->B;
    P.has_full = bm->has_full ? 1 : 0;
    P.mask = mp;
    P.score_kind = kind;
    P.scale = sc;
    if (has_cap) {
        P.softcap = sm->softcap;
        P.softcap_in = sc / sm->softcap;
        P.softcap_inv = 1.0f / sm->softcap;
    }
    P.slopes = kind == FA_SCORE_ALIBI ? sm->alibi_slopes : nullptr;
    if (has_bias) {
        P.bias = static_cast<const uint16_t*>(sm->bias);
        P.bias_st0 = sm->bias_strides[0];
        P.bias_st1 = sm->bias_strides[1];
        P.bias_st2 = sm->bias_strides[2];
    }
    const DecLayout lay = dec_layout(B, Hq, Hkv, q_len, kv_len, D);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    P.grid = (int32_t)lay.grid;
    P.total = reinterpret_cast<long long*>(ws + lay.total);
    P.seg_first = reinterpret_cast<int32_t*>(ws + lay.seg_first);
    P.seg_last = reinterpret_cast<int32_t*>(ws + lay.seg_last);
    P.part_ml = reinterpret_cast<float*>(ws + lay.ml);
    P.part_o = reinterpret_cast<float*>(ws + lay.o);
    P.status = reinterpret_cast<int*>(ws);
    P.watchdog_ns = g_watchdog_ns;
    if (kv_len == 0) P.tm_k = P.tm_v = CUtensorMap{};  // never read: no kv block
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (fa::launch_flex_decode(P, (int)D, st) != cudaSuccess) return FA_ERR_CUDA;
    if (fa::launch_decode_merge(P, (int)D, st) != cudaSuccess) return FA_ERR_CUDA;
    return FA_OK;
}

int fa_get_device_status(void* workspace, void* stream)
{
    if (!workspace) return FA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int host = 0;
    if (cudaMemcpyAsync(&host, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return FA_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof(int), s) != cudaSuccess) return FA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_CUDA;
    if (host & fa::STATUS_TIMEOUT) return FA_ERR_TIMEOUT;
    if (host & fa::STATUS_BAD_BLOCKMASK) return FA_ERR_BAD_BLOCKMASK;
    return FA_OK;
}

} // extern "C"

// ---------------------------------------------------------------- allocation-free variant
//
// Some callers cannot allocate device memory when they call the forward pass:
// an engine that plans all memory up front and hands an operator only its input
// and output buffers, a serving loop that must not enter the allocator in the
// middle of a request, or code in a context where cudaMalloc would synchronise
// the device.  fa_forward_static_scratch serves them: its scratch (the device
// status word fa_forward keeps in the caller's workspace) lives in the array
// below, which every GPU that loads this library holds until the process exits.

#include <mutex>
#include <vector>

#include "context.cuh"

namespace {

constexpr size_t kStaticScratchBytes = 256;  // maximum scratch of the variant

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

struct ScratchAddr {
    fa::CtxKey ctx;
    void* ptr;
};
std::mutex g_static_scratch_mu;
std::vector<ScratchAddr> g_static_scratch_addr;

// Device address of the array in the current context.  In host code the array's
// name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress, with the device current, once per context: the first
// call on a device (and the first after a cudaDeviceReset of it, which rebuilds
// the context and the module) does the look-up, later calls reuse it.
int static_scratch_address(void** out)
{
    fa::CtxKey key;
    std::lock_guard<std::mutex> lock(g_static_scratch_mu);
    const bool keyed = fa::current_ctx(&key);
    if (keyed)
        for (const ScratchAddr& a : g_static_scratch_addr)
            if (a.ctx == key) {
                *out = a.ptr;
                return FA_OK;
            }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return FA_ERR_CUDA;
    // the look-up made the context current if none was; key it now
    if (fa::current_ctx(&key)) g_static_scratch_addr.push_back({key, p});
    *out = p;
    return FA_OK;
}

} // namespace

extern "C" int fa_forward_static_scratch(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v,
                                         const fa_block_mask* bm, const fa_score_mod* sm, float scale,
                                         const fa_tensor* o, float* lse, void* stream)
{
    if (fa_workspace_size() > kStaticScratchBytes) return FA_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    int rc = static_scratch_address(&scratch);
    if (rc != FA_OK) return rc;
    return fa_forward(q, k, v, bm, sm, scale, o, lse, scratch, kStaticScratchBytes, stream);
}
