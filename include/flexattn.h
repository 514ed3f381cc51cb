/*
 * flexattn.h — C ABI of the B200 (sm_100a) block-sparse FlexAttention forward and
 * backward passes.
 *
 *   out = softmax(mod(Q K^T / sqrt(d))) V
 *
 * ("Flex Attention: A Programming Model for Generating Optimized Attention
 * Kernels", paper review, sec. 2.1: every variant is a modification of the score
 * matrix before softmax.)  A mask_mod decides which (q_idx, kv_idx) positions
 * attend; a score_mod rewrites the scores that do.  This library replaces the
 * pages' JIT-compiled Python closures with enumerated variants:
 *
 *   mask_mod : causal, sliding window, document id, prefix, combined by one AND/OR
 *   score_mod: none, ALiBi, tanh soft-capping, a dynamic additive bias tensor, or
 *              the bias followed by soft-capping
 *
 * Conventions for every call:
 *   - All functions are host functions returning an fa_status (0 = FA_OK).
 *     Argument validation is synchronous; GPU work is enqueued asynchronously
 *     on the caller's stream (`stream` is a cudaStream_t; NULL = legacy default
 *     stream) and nothing synchronises the host, except fa_get_device_status.
 *   - The library allocates no device memory.  Every buffer (inputs, outputs,
 *     BlockMask arrays, workspace) is allocated and owned by the caller and must
 *     stay valid until the enqueued work has finished.
 *   - Device pointers must address memory of the current CUDA device.
 *   - Strides are in elements.  Sizes are int64_t.
 *   - On an error return nothing has been enqueued.
 */
#ifndef FLEXATTN_H
#define FLEXATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ status */

typedef enum fa_status {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, stride or alignment */
    FA_ERR_UNSUPPORTED = 2,   /* valid request outside what this library implements */
    FA_ERR_CUDA = 3,          /* a CUDA runtime call failed (launch, attribute, ...) */
    FA_ERR_TIMEOUT = 4,       /* a device-side pipeline wait ran out (watchdog) */
    FA_ERR_BAD_BLOCKMASK = 5  /* a BlockMask count or index was out of range */
} fa_status;

/* Human-readable name of a status code (static storage, never NULL). */
const char* fa_status_string(int status);

/* ------------------------------------------------------------------ mask_mod */

/* BLOCK_SIZE of the BlockMask: 128 x 128 ("Concepts", BlockMask Internals: the
 * attention matrix is divided into blocks of size BLOCK_SIZE, default 128x128). */
#define FA_BLOCK_SIZE 128
#define FA_MAX_LEAVES 4

typedef enum fa_leaf_kind {
    FA_LEAF_CAUSAL = 0,    /* q_idx >= kv_idx          ("Concepts", mask_mod)          */
    FA_LEAF_SLIDING = 1,   /* q_idx - kv_idx <= param  ("Concepts", Composing masks)   */
    FA_LEAF_DOCUMENT = 2,  /* doc[b][q_idx] == doc[b][kv_idx]  (paper review sec. 5.3) */
    FA_LEAF_PREFIX = 3     /* kv_idx < param  (prefix of a prefix-LM, paper review 4.4) */
} fa_leaf_kind;

typedef enum fa_mask_op {
    FA_MASK_AND = 0,       /* and_masks ("Concepts", Composing masks)     */
    FA_MASK_OR = 1         /* or_masks  (paper review sec. 4.4, logical fusion) */
} fa_mask_op;

/* An enumerated mask_mod: up to FA_MAX_LEAVES leaves combined by one operator.
 * n_leaves = 0 means every position attends.  No leaf depends on the head. */
typedef struct fa_mask_desc {
    int32_t n_leaves;
    int32_t op;                       /* fa_mask_op */
    int32_t kind[FA_MAX_LEAVES];      /* fa_leaf_kind per leaf */
    int64_t param[FA_MAX_LEAVES];     /* window W (SLIDING) or prefix length P (PREFIX) */
    /* DOCUMENT leaf only: device int32 ids, one per token position; row b starts at
     * doc_ids + b * doc_stride (doc_stride = 0 shares one row across the batch).
     * doc_len >= max(q_len, kv_len) positions per row. */
    const int32_t* doc_ids;
    int64_t doc_stride;
    int64_t doc_len;
    /* Position of query row 0: the leaves (and ALiBi) see query row i at position
     * q_offset + i.  0 for a prefill; the cache length before the new tokens for a
     * decoding step (the FlexDecoding masks of the pages evaluate the mask at the
     * step's position).  0 <= q_offset and q_offset + q_len < 2^31 - 128; a
     * DOCUMENT leaf then needs doc_len >= max(q_offset + q_len, kv_len). */
    int64_t q_offset;
} fa_mask_desc;

/* ------------------------------------------------------------------ BlockMask */

/* The block-sparse form of a mask ("Concepts", BlockMask Internals, key-attribute
 * table; paper review sec. 4.1-4.2).  Each 128x128 tile of the (q, kv) plane is
 *   full    — every in-range position attends: no per-element mask is evaluated;
 *   partial — some positions attend: the mask is evaluated per element;
 *   empty   — none attend: the tile is skipped.
 * Lists are disjoint: kv_indices holds the PARTIAL tiles of each query block and
 * full_kv_indices the FULL ones, each ascending by kv block index, unused slots 0.
 *
 *   kv_num_blocks      int32 [B, H, nq]        partial tiles per query block
 *   kv_indices         int32 [B, H, nq, nkv]   their kv block indices
 *   full_kv_num_blocks int32 [B, H, nq]        full tiles per query block
 *   full_kv_indices    int32 [B, H, nq, nkv]   their kv block indices
 *
 * All four are caller-allocated device buffers, contiguous row-major.  B = 1 or
 * H = 1 broadcasts over the batch / heads of the attention call.  The mask
 * descriptor is kept because partial tiles re-evaluate it per element; a
 * DOCUMENT leaf's doc_ids must therefore stay valid while the BlockMask is used.
 * Positions q >= q_len or kv >= kv_len never attend. */
typedef struct fa_block_mask {
    int32_t* kv_num_blocks;
    int32_t* kv_indices;
    int32_t* full_kv_num_blocks;
    int32_t* full_kv_indices;
    int32_t B, H;
    int32_t nq, nkv;
    int32_t block_size;               /* FA_BLOCK_SIZE */
    int32_t has_full;                 /* 0: full_* unused, every listed tile is masked per element */
    int64_t q_len, kv_len;
    fa_mask_desc mask;
    /* The transposed view, "used in backward" ("Concepts", BlockMask Internals):
     * for each kv block, its partial query blocks (q_*) and full ones (full_q_*),
     * ascending, unused slots 0.  Optional: all four NULL means it is not built;
     * fa_backward needs it.
     *   q_num_blocks      int32 [B, H, nkv]       q_indices      int32 [B, H, nkv, nq]
     *   full_q_num_blocks int32 [B, H, nkv]       full_q_indices int32 [B, H, nkv, nq] */
    int32_t* q_num_blocks;
    int32_t* q_indices;
    int32_t* full_q_num_blocks;
    int32_t* full_q_indices;
} fa_block_mask;

/* Sizes of the BlockMask arrays for a (q_len x kv_len) problem:
 * *nq = ceil(q_len / block_size), *nkv = ceil(kv_len / block_size).
 * block_size must be FA_BLOCK_SIZE (else FA_ERR_UNSUPPORTED). */
int fa_block_mask_shape(int64_t q_len, int64_t kv_len, int block_size, int32_t* nq, int32_t* nkv);

/* create_block_mask(mask_mod, B, H, Q_LEN, KV_LEN) ("Concepts", Inspecting a
 * BlockMask): evaluate the mask over every in-range position of every tile,
 * classify the tiles and write the four arrays of `bm`.
 *
 * In: m (copied into bm->mask), B >= 1, H >= 1, q_len >= 0, kv_len >= 0,
 *     block_size = FA_BLOCK_SIZE, and bm's four device pointers (arrays sized by
 *     fa_block_mask_shape; the count arrays may be NULL only when nq == 0, the
 *     index arrays only when nq * nkv == 0).
 *     When any of bm's q_* pointers is set, the transposed view is built as well
 *     (arrays sized [B, H, nkv] and [B, H, nkv, nq]; a pointer may be NULL only
 *     when its array has no element), by a second kernel on the same stream; when
 *     all four are NULL it is not.
 * Out: bm's arrays (asynchronously) and its descriptor fields (on return).
 * Errors: FA_ERR_INVALID_ARG for null/negative/over-long arguments (q_len and
 * kv_len must be < 2^31 - 128; B and H at most 65535), an unknown leaf or operator, a DOCUMENT leaf
 * without doc_ids or with doc_len < max(q_len, kv_len), a q_* array missing while
 * another is set; FA_ERR_UNSUPPORTED for block_size != 128; FA_ERR_CUDA if a launch fails. */
int fa_create_block_mask(const fa_mask_desc* m, int B, int H, int64_t q_len, int64_t kv_len, int block_size,
                         fa_block_mask* bm, void* stream);

/* The same BlockMask without the full / partial split: every non-empty tile is
 * listed in kv_num_blocks / kv_indices, so the forward pass evaluates the mask
 * per element in every tile it visits; full_kv_num_blocks is written 0 and
 * bm->has_full set to 0.  This is the baseline against which the paper review's
 * sec. 4.2 quotes the gain of the split (about 15% on causal-like masks); the
 * "Concepts" page likewise allows a BlockMask whose full_* lists are absent.
 * Arguments, ownership and errors as fa_create_block_mask. */
int fa_create_block_mask_unsplit(const fa_mask_desc* m, int B, int H, int64_t q_len, int64_t kv_len,
                                 int block_size, fa_block_mask* bm, void* stream);

/* ------------------------------------------------------------------ score_mod */

typedef enum fa_score_kind {
    FA_SCORE_NONE = 0,
    FA_SCORE_ALIBI = 1,    /* s + slopes[h] * (kv_idx - q_idx)    ("Concepts", score_mod) */
    FA_SCORE_SOFTCAP = 2,  /* cap * tanh(s / cap)                 (paper review sec. 2.1) */
    FA_SCORE_BIAS = 3,     /* s + bias[b, h, q_idx, kv_idx]       (attention-gym issue
                                                                   "Dynamic Bias Tensor") */
    FA_SCORE_BIAS_SOFTCAP = 4  /* cap * tanh((s + bias[b, h, q_idx, kv_idx]) / cap): the two
                                  score_mods composed, bias first (paper review sec. 2.1
                                  lists both; a score_mod is any function of the score) */
} fa_score_kind;

/* An enumerated score_mod, applied to the scaled score s = (Q K^T) * scale of
 * every position the mask admits (and to no other: "Concepts", When to use which).
 * Heads are query heads.  The bias pointer and values may change on every call;
 * nothing is rebuilt. */
typedef struct fa_score_mod {
    int32_t kind;                     /* fa_score_kind */
    float softcap;                    /* cap > 0 for SOFTCAP and BIAS_SOFTCAP */
    const float* alibi_slopes;        /* device fp32 [Hq] for ALIBI */
    const void* bias;                 /* device bf16 [B, Hq, q_len, kv_len] for BIAS and BIAS_SOFTCAP,
                                         16-byte aligned */
    int64_t bias_strides[4];          /* elements; innermost must be 1, others multiples of 8 (a
                                         bias whose kv_len is not a multiple of 8 needs padded rows).
                                         Stride 0 on the batch or head dimension broadcasts one
                                         [q_len, kv_len] plane over it (an expanded [1, 1, Sq, Skv]
                                         bias); stride 0 on the query dimension is rejected. */
} fa_score_mod;

/* ------------------------------------------------------------------ forward */

/* A 4-D bf16 device tensor [B, H, S, D]: innermost (D) stride must be 1, the
 * other strides multiples of 8 elements (16 bytes), base 16-byte aligned (the
 * tiles are fetched by TMA).  A stride may be 0 only on a dimension of size 1:
 * an expanded (broadcast) dimension of size > 1 is rejected with
 * FA_ERR_INVALID_ARG (materialise it first).  `data` may be NULL only when a
 * dimension is 0. */
typedef struct fa_tensor {
    void* data;
    int64_t dims[4];
    int64_t strides[4];
} fa_tensor;

/* Bytes of device workspace fa_forward needs: a device status word and the
 * per-launch scheduling counters.  Independent of the problem size.  Zero the
 * workspace once before its first use; fa_get_device_status clears the status
 * word after reading it. */
size_t fa_workspace_size(void);

/* flex_attention(q, k, v, block_mask, score_mod) -> (out, lse)
 * ("Concepts", score_mod vs mask_mod; paper review sec. 2.1, 4.2, 4.3).
 *
 * In:  q [B, Hq, q_len, D], k and v [B, Hkv, kv_len, D] (bf16; Hq % Hkv == 0,
 *      query head h reads kv head h / (Hq / Hkv)); D in {64, 128}.
 *      bm: a BlockMask from fa_create_block_mask with q_len / kv_len equal to the
 *      tensors' and B, H each 1 or equal to the tensors' B, Hq.
 *      sm: score_mod (NULL = none).  scale: multiplies Q K^T; <= 0 means 1/sqrt(D).
 *      workspace: caller-owned device buffer of >= fa_workspace_size() bytes,
 *      16-byte aligned; calls that overlap in time need distinct workspaces.
 * Out: o [B, Hq, q_len, D] bf16 (round to nearest even from fp32);
 *      lse: device fp32 [B, Hq, q_len] contiguous, the natural-log logsumexp of
 *      the modified, masked score row (NULL = not written).
 *      A row no position of which attends gets O = 0 and LSE = -inf.
 * Only the tiles that the BlockMask lists are computed; per-element masking runs
 * in partial tiles only (and in the ragged last kv tile).
 * Errors: FA_ERR_INVALID_ARG / FA_ERR_UNSUPPORTED as above (shapes, strides,
 * alignment, D, GQA ratio, BlockMask extents); FA_ERR_CUDA on a failed launch.
 * Device-side problems (pipeline watchdog, out-of-range BlockMask entries) are
 * recorded in the workspace and read with fa_get_device_status. */
int fa_forward(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const fa_block_mask* bm,
               const fa_score_mod* sm, float scale, const fa_tensor* o, float* lse, void* workspace,
               size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------ backward */

/* Bytes of device workspace fa_backward needs for B x Hq x q_len query rows of
 * head dimension D, with the rows of each (batch, head) padded to whole 128-row
 * blocks (nq = ceil(q_len / 128)): a device status word, then per block the LSE
 * (log2 units) and Delta = rowsum(dO * O) rows (fp32, 1 KB), then an fp32
 * accumulator for dQ (B * Hq * nq * 128 * D floats). */
size_t fa_backward_workspace_size(int64_t B, int64_t Hq, int64_t q_len, int64_t D);

/* The backward pass of flex_attention (paper review sec. 3.1, the backward
 * template; "Concepts", BlockMask Internals: q_num_blocks / q_indices are "used
 * in backward"): the gradients of out = softmax(mod(Q K^T * scale)) V with
 * respect to Q, K and V, given the upstream gradient dout.
 *
 * In:  q, k, v, bm, sm, scale exactly as passed to the fa_forward call that
 *      produced o and lse (o [B, Hq, q_len, D] bf16; lse device fp32 [B, Hq, q_len]
 *      contiguous); dout [B, Hq, q_len, D] bf16.  bm must carry the transposed view
 *      (built by fa_create_block_mask with its q_* arrays).  The score_mod is
 *      differentiated too (ALiBi and bias have derivative 1, soft-capping
 *      1 - tanh^2); no gradient is returned for the bias tensor or the slopes.
 *      workspace: >= fa_backward_workspace_size(B, Hq, q_len, D) bytes, 16-byte
 *      aligned, owned by the caller; calls that overlap in time need distinct
 *      workspaces.  Only its first 256 bytes (the status word) need to be zero
 *      before the first call; the call writes every other byte it reads.
 * Out: dq [B, Hq, q_len, D], dk and dv [B, Hkv, kv_len, D] (bf16, layouts as for
 *      fa_tensor).  Under GQA dk / dv sum over the query heads of each group.  A
 *      kv position no query attends to gets dK = dV = 0.
 * Only the tiles the BlockMask lists are computed; per-element masking runs in
 * partial tiles only (and at ragged edges).
 * Errors: as fa_forward, plus FA_ERR_INVALID_ARG when a shape differs from q / k,
 * lse is NULL, the workspace is too small or the transposed view is missing;
 * FA_ERR_UNSUPPORTED when B * Hq * nq * 128 exceeds 2^31 - 1.
 * Device-side problems are recorded in the workspace's first word and read with
 * fa_get_device_status. */
int fa_backward(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const fa_tensor* o,
                const fa_tensor* dout, const float* lse, const fa_block_mask* bm, const fa_score_mod* sm, float scale,
                const fa_tensor* dq, const fa_tensor* dk, const fa_tensor* dv, void* workspace,
                size_t workspace_bytes, void* stream);

/* flex_attention over a paged KV cache (paper review sec. 4.5: PagedAttention by
 * using the BlockMask's kv indices as a page table; the talk summary's "Page
 * Attention").  The BlockMask is built over LOGICAL positions (kv_len = the
 * logical sequence length); logical kv block kb of batch b lives in physical page
 * page_table[b * page_table_stride + kb] of the page pools.  A page holds one kv
 * block (FA_BLOCK_SIZE keys), so the tile the kernel fetches is exactly one page.
 *
 * In:  q, o, lse, bm, sm, scale, workspace as fa_forward.
 *      k_pages, v_pages: [num_pages, Hkv, FA_BLOCK_SIZE, D] bf16 page pools (same
 *      shape; fa_tensor layout rules).  Keys of the last logical block at or
 *      beyond bm->kv_len are ignored (masked), whatever the page holds.
 *      page_table: device int32, row b has page_table_stride >= nkv entries, entry
 *      kb in [0, num_pages) for kb < nkv.  Pages may be shared between rows.
 * Errors: as fa_forward; FA_ERR_INVALID_ARG for a NULL page table, a short
 * stride or pools of another shape.  An entry outside [0, num_pages) is clamped
 * in the kernel (no read outside the pools) and reported as FA_ERR_BAD_BLOCKMASK
 * by fa_get_device_status. */
int fa_forward_paged(const fa_tensor* q, const fa_tensor* k_pages, const fa_tensor* v_pages, const int32_t* page_table,
                     int64_t page_table_stride, const fa_block_mask* bm, const fa_score_mod* sm, float scale,
                     const fa_tensor* o, float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------ decoding */

/* Bytes of device workspace fa_decode needs: the status word, the list length
 * and each segment's first and last CTA, and the partial results (running max,
 * sum and unnormalised O per compute warp and piece of a segment) that the merge
 * kernel combines.  Depends on the SM count of the current device: query it on
 * the device of the call. */
size_t fa_decode_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t q_len, int64_t kv_len, int64_t D);

/* FlexDecoding (paper review sec. 3.1, the decoding template; rocketrecap talk
 * summary, "Flex Decoding": the work is split along the KV dimension and the
 * partial results are reduced at the end): the forward pass for a few query
 * tokens per sequence against a long KV cache.  Same result as fa_forward, by a
 * kernel built for this shape: the G = Hq / Hkv query heads of a kv head and
 * their q_len tokens are processed together (G * q_len <= 16), and the kv blocks
 * of the BlockMask row are spread over CTAs and merged by a second kernel.
 *
 * In:  as fa_forward, with G * q_len <= 16 and a head-independent BlockMask
 *      (bm->H == 1).  A decoding step at position t of a sequence uses a
 *      BlockMask built with mask q_offset = t (its queries' positions).
 *      workspace: >= fa_decode_workspace_size(...) bytes, 16-byte aligned.
 * Out: o, lse as fa_forward.
 * Errors: as fa_forward; FA_ERR_UNSUPPORTED for G * q_len > 16 or bm->H != 1. */
int fa_decode(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const fa_block_mask* bm,
              const fa_score_mod* sm, float scale, const fa_tensor* o, float* lse, void* workspace,
              size_t workspace_bytes, void* stream);

/* Synchronise `stream`, then return the device status recorded in `workspace`
 * by earlier fa_forward calls (FA_OK, FA_ERR_TIMEOUT or FA_ERR_BAD_BLOCKMASK) and
 * clear it.  FA_ERR_CUDA if the stream reports an error. */
int fa_get_device_status(void* workspace, void* stream);

/* Set the watchdog limit of device-side waits in milliseconds (default 2000;
 * process-wide; 0 restores the default). */
int fa_set_watchdog_ms(int ms);

/* Test facility for the device watchdog (off by default, process-wide).  While
 * `on` is nonzero, every fa_forward launch makes its TMA producer wait on a
 * barrier that nothing completes, so every pipeline wait of the kernel runs out
 * after the watchdog limit; the kernel then releases its resources and exits,
 * and fa_get_device_status reports FA_ERR_TIMEOUT.  No fault, trap or unbounded
 * wait is involved; O and LSE of such a launch are not written meaningfully.
 * Returns FA_OK. */
int fa_set_selftest_stall(int on);

/* fa_forward without a caller-provided workspace, for callers that cannot
 * allocate device memory: an engine that plans all memory up front and hands an
 * operator only its input and output buffers, a serving loop that must not enter
 * the allocator in the middle of a request, or code where cudaMalloc would
 * synchronise the device.  (The FlexAttention pages have no counterpart: this is
 * an interface choice of this library.)
 *
 * Same arguments, layouts, ownership and errors as fa_forward, minus the
 * workspace.  The scratch fa_forward keeps in the workspace (the device status
 * word) lives instead in a file-scope __device__ array of 256 bytes (the stated
 * maximum; every GPU that loads the library holds it until the process exits).
 * The call allocates nothing and calls no allocating routine; it returns
 * FA_ERR_UNSUPPORTED if the scratch the forward pass needs ever exceeds 256 bytes.
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it for that device's context; make that first call
 * before any stream capture (and again after a cudaDeviceReset, which rebuilds
 * the context).
 * Every call shares the array and it keeps the last call's contents; nothing in
 * it has to start at zero (the kernel only sets status bits), so the call clears
 * nothing.  Calls that overlap on the GPU race on the shared status word, and
 * that word is not readable through this ABI: device-side watchdog or BlockMask
 * errors of this variant are not reported. */
int fa_forward_static_scratch(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const fa_block_mask* bm,
                              const fa_score_mod* sm, float scale, const fa_tensor* o, float* lse, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FLEXATTN_H */
