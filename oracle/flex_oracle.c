/*
 * Plain fp64 CPU oracle for the block-sparse FlexAttention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file: only the tests, the package's smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or helper with the CUDA
 * library.
 *
 * What it computes, and where the pages define it:
 *
 *   out = softmax(mod(Q K^T / sqrt(d))) V
 *     "Flex Attention" paper review (xllm-io), sec. 2.1 "key insight":
 *     FlexAttention(Q,K,V) = softmax(mod(QK^T/sqrt(d_k))) V.
 *
 *   mask_mod(b, h, q_idx, kv_idx) -> bool, True = attend
 *     attention-gym "Concepts", section "mask_mod" (causal: q_idx >= kv_idx),
 *     section "Composing masks" (sliding window: q_idx - kv_idx <= window_size,
 *     and_masks / or_masks), paper review sec. 4.4 "logical fusion" (OR of masks),
 *     paper review sec. 5.3 (document mask from a B x N vector of document ids).
 *
 *   score_mod(score, b, h, q_idx, kv_idx) -> score, applied to unmasked scores only
 *     attention-gym "Concepts", section "score_mod" (ALiBi: score +
 *     alibi_slope[h] * (kv_idx - q_idx)) and "When to use which?" (the score mod
 *     is only applied to unmasked positions; a mask is a score mod returning -inf);
 *     paper review sec. 2.1 table (soft-capping); attention-gym issue "Dynamic Bias
 *     Tensor ... Without Recompilation" (an additive [B, H, S, S] bias).
 *
 *   BlockMask: kv_num_blocks / kv_indices / full_kv_num_blocks / full_kv_indices
 *     attention-gym "Concepts", section "BlockMask Internals" (block classes
 *     full / partial / empty; key-attribute table); paper review sec. 4.1, 4.2.
 *     The transposed lists q_num_blocks / q_indices (and full_q_*) of the same
 *     table ("used in backward"): for each kv block, its query blocks.
 *
 *   Backward pass (paper review sec. 3.1: the backward template; Hacker News
 *   thread: the backward runs at 85% of FlashAttention-2): the gradients of the
 *   forward pass above with respect to Q, K and V, given dO.  Written out from
 *   the chain rule of out = softmax(mod(QK^T * scale)) V:
 *     p = softmax row, dP = dO V^T, dS' = p * (dP - rowsum(p * dP)),
 *     dS = dS' * d mod / ds, dQ = scale dS K, dK = scale dS^T Q, dV = p^T dO.
 *
 * Everything is evaluated densely in fp64 from the exact bf16 input values: the
 * mask is materialised per element, every score row is formed in full, and the
 * softmax is taken over the whole row.  No blocking, fusion or reordering.
 *
 * Readings of points the pages leave open (each listed in the design notes):
 *   - kv_* lists hold the PARTIAL blocks only and full_* lists the FULL blocks;
 *     both ascending by block index, padded with 0; max_kv_blocks = nkv.
 *   - Blocks are classified over in-range positions only (q < q_len, kv < kv_len).
 *   - The sliding-window leaf is one-sided, q - kv <= W, inclusive.
 *   - Document leaf: doc[b][q] == doc[b][kv] (one id per token position).
 *   - Prefix leaf: kv < P (the bidirectional prefix of a prefix-LM).
 *   - score_mod receives the scaled score QK^T * scale.
 *   - Soft-capping: cap * tanh(s / cap).
 *   - GQA: query head hq reads kv head hq / (Hq / Hkv).
 *   - LSE is the natural-log logsumexp of the modified, masked scores.
 *   - A row with no admitted key has O = 0 and LSE = -inf.
 */

#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_LEAF_CAUSAL = 0, ORC_LEAF_SLIDING = 1, ORC_LEAF_DOCUMENT = 2, ORC_LEAF_PREFIX = 3 };
enum { ORC_OP_AND = 0, ORC_OP_OR = 1 };
enum { ORC_SCORE_NONE = 0, ORC_SCORE_ALIBI = 1, ORC_SCORE_SOFTCAP = 2, ORC_SCORE_BIAS = 3,
       ORC_SCORE_BIAS_SOFTCAP = 4 };
enum { ORC_EMPTY = 0, ORC_PARTIAL = 1, ORC_FULL = 2 };

#define ORC_MAX_LEAVES 4

typedef struct {
    int32_t n_leaves;
    int32_t op;                      /* ORC_OP_AND or ORC_OP_OR */
    int32_t kind[ORC_MAX_LEAVES];
    int64_t param[ORC_MAX_LEAVES];   /* window W for SLIDING, P for PREFIX */
    const int32_t* doc_ids;          /* [doc_B][doc_len], may be NULL without a DOCUMENT leaf */
    int64_t doc_len;
    int32_t doc_B;
    int32_t pad_;
    int64_t q_offset;                /* position of query row 0 (decoding: the cache length before it) */
} orc_mask;

typedef struct {
    /* Q [B,Hq,Sq,D], K/V [B,Hkv,Skv,D]: raw bf16 bit patterns with element strides */
    const uint16_t* q; int64_t q_stride[4];
    const uint16_t* k; int64_t k_stride[4];
    const uint16_t* v; int64_t v_stride[4];
    int32_t B, Hq, Hkv, D;
    int64_t q_len, kv_len;
    double scale;
    int32_t score_kind;
    int32_t pad_;
    const float* slopes;             /* [Hq] for ALIBI */
    double softcap;                  /* cap for SOFTCAP and BIAS_SOFTCAP */
    const uint16_t* bias;            /* [B,Hq,Sq,Skv] bf16 for BIAS and BIAS_SOFTCAP */
    int64_t bias_stride[4];
    int64_t q_offset;                /* position of query row 0 (ALiBi distances) */
} orc_problem;

/* bf16 is the upper half of an IEEE binary32: widening is exact. */
static double bf16_to_double(uint16_t h)
{
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* One mask leaf at one (b, q, kv) position; q is the query's position (its row
 * plus the mask's q_offset). */
static int leaf_value(const orc_mask* m, int i, int b, int64_t q, int64_t kv)
{
    switch (m->kind[i]) {
    case ORC_LEAF_CAUSAL:
        return q >= kv;
    case ORC_LEAF_SLIDING:
        return q - kv <= m->param[i];
    case ORC_LEAF_DOCUMENT: {
        int bb = (m->doc_B == 1) ? 0 : b;
        const int32_t* row = m->doc_ids + (int64_t)bb * m->doc_len;
        return row[q] == row[kv];
    }
    case ORC_LEAF_PREFIX:
        return kv < m->param[i];
    default:
        return 0;
    }
}

/* mask_mod(b, h, q_idx, kv_idx) for query row q: the leaves, evaluated at the
 * query position q + q_offset (a decoding step sees its position in the sequence,
 * as the pages' FlexDecoding masks do with an offset), combined by one AND or OR.
 * No leaf depends on h.  With no leaves every position attends. */
int orc_mask_value(const orc_mask* m, int b, int h, int64_t q, int64_t kv)
{
    (void)h;
    if (m->n_leaves == 0) return 1;
    const int64_t qp = q + m->q_offset;
    int acc = leaf_value(m, 0, b, qp, kv);
    for (int i = 1; i < m->n_leaves; ++i) {
        int x = leaf_value(m, i, b, qp, kv);
        acc = (m->op == ORC_OP_OR) ? (acc | x) : (acc & x);
    }
    return acc;
}

/* The dense boolean mask of one (b, h): out[q * kv_len + kv]. */
void orc_dense_mask(const orc_mask* m, int b, int h, int64_t q_len, int64_t kv_len, uint8_t* out)
{
    for (int64_t q = 0; q < q_len; ++q)
        for (int64_t kv = 0; kv < kv_len; ++kv)
            out[q * kv_len + kv] = (uint8_t)orc_mask_value(m, b, h, q, kv);
}

/* Class of one BLOCK_SIZE x BLOCK_SIZE tile: count admitted in-range positions. */
int orc_block_class(const orc_mask* m, int b, int h, int64_t q_len, int64_t kv_len, int bs,
                    int64_t qb, int64_t kb)
{
    int64_t q0 = qb * bs, q1 = q0 + bs < q_len ? q0 + bs : q_len;
    int64_t k0 = kb * bs, k1 = k0 + bs < kv_len ? k0 + bs : kv_len;
    int64_t total = 0, admitted = 0;
    for (int64_t q = q0; q < q1; ++q)
        for (int64_t kv = k0; kv < k1; ++kv) {
            total += 1;
            admitted += orc_mask_value(m, b, h, q, kv);
        }
    if (admitted == 0) return ORC_EMPTY;
    return admitted == total ? ORC_FULL : ORC_PARTIAL;
}

typedef struct {
    const orc_mask* m;
    int B, H, bs;
    int64_t q_len, kv_len, nq, nkv;
    int32_t *kv_num, *kv_idx, *full_num, *full_idx;
    int split_full;                  /* 0: full blocks are listed with the partial ones */
    int64_t next;                    /* next (b,h,qb) row to claim */
    pthread_mutex_t lock;
} bm_job;

static void block_mask_row(bm_job* J, int64_t r)
{
    int64_t qb = r % J->nq;
    int64_t bh = r / J->nq;
    int h = (int)(bh % J->H), b = (int)(bh / J->H);
    int32_t* pidx = J->kv_idx + r * J->nkv;
    int32_t* fidx = J->full_idx + r * J->nkv;
    int32_t np = 0, nf = 0;
    for (int64_t kb = 0; kb < J->nkv; ++kb) {
        pidx[kb] = 0;
        fidx[kb] = 0;
    }
    for (int64_t kb = 0; kb < J->nkv; ++kb) {
        int c = orc_block_class(J->m, b, h, J->q_len, J->kv_len, J->bs, qb, kb);
        if (c == ORC_PARTIAL || (c == ORC_FULL && !J->split_full)) pidx[np++] = (int32_t)kb;
        if (c == ORC_FULL && J->split_full) fidx[nf++] = (int32_t)kb;
    }
    J->kv_num[r] = np;
    J->full_num[r] = nf;
}

static void* block_mask_worker(void* arg)
{
    bm_job* J = (bm_job*)arg;
    int64_t rows = (int64_t)J->B * J->H * J->nq;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t r = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (r >= rows) break;
        block_mask_row(J, r);
    }
    return NULL;
}

static int run_threads(void* (*fn)(void*), void* job, int n_threads)
{
    if (n_threads <= 1) {
        fn(job);
        return 0;
    }
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!th) return -1;
    int started = 0;
    for (int i = 0; i < n_threads; ++i)
        if (pthread_create(&th[i], NULL, fn, job) == 0) started++;
        else break;
    if (started == 0) fn(job);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    return 0;
}

/* create_block_mask: classify every tile and emit the four int32 arrays,
 * kv_num/full_num [B,H,nq] and kv_idx/full_idx [B,H,nq,nkv], row-major.
 * With split_full = 0 there is no full / partial split (a BlockMask without its
 * optional full_* lists, "Concepts", BlockMask Internals): every non-empty block
 * is listed in kv_idx and the full lists stay empty. */
int orc_block_mask(const orc_mask* m, int B, int H, int64_t q_len, int64_t kv_len, int bs,
                   int32_t* kv_num, int32_t* kv_idx, int32_t* full_num, int32_t* full_idx,
                   int n_threads, int split_full)
{
    if (bs <= 0) return -1;
    bm_job J;
    memset(&J, 0, sizeof J);
    J.m = m; J.B = B; J.H = H; J.bs = bs; J.q_len = q_len; J.kv_len = kv_len;
    J.nq = (q_len + bs - 1) / bs;
    J.nkv = (kv_len + bs - 1) / bs;
    J.kv_num = kv_num; J.kv_idx = kv_idx; J.full_num = full_num; J.full_idx = full_idx;
    J.split_full = split_full;
    pthread_mutex_init(&J.lock, NULL);
    run_threads(block_mask_worker, &J, n_threads);
    pthread_mutex_destroy(&J.lock);
    return 0;
}

static double bias_at(const orc_problem* P, int b, int hq, int64_t q, int64_t kv)
{
    const int64_t* st = P->bias_stride;
    int64_t off = (int64_t)b * st[0] + (int64_t)hq * st[1] + q * st[2] + kv * st[3];
    return bf16_to_double(P->bias[off]);
}

/* score_mod applied to one scaled score.  BIAS_SOFTCAP composes two score_mods
 * (paper review sec. 2.1 lists both as variants; a score_mod is any function of
 * the score, so two compose): the bias is added first, then the sum is capped. */
static double score_mod(const orc_problem* P, double s, int b, int hq, int64_t q, int64_t kv)
{
    switch (P->score_kind) {
    case ORC_SCORE_ALIBI:
        return s + (double)P->slopes[hq] * (double)(kv - (q + P->q_offset));
    case ORC_SCORE_SOFTCAP:
        return P->softcap * tanh(s / P->softcap);
    case ORC_SCORE_BIAS:
        return s + bias_at(P, b, hq, q, kv);
    case ORC_SCORE_BIAS_SOFTCAP:
        return P->softcap * tanh((s + bias_at(P, b, hq, q, kv)) / P->softcap);
    default:
        return s;
    }
}

/* The full modified, masked score row of query (b, hq, q): s'[kv] for every kv. */
static void score_row(const orc_problem* P, const orc_mask* m, int b, int hq, int64_t q, double* s)
{
    int G = P->Hq / P->Hkv;
    int hk = hq / G;
    const uint16_t* qrow = P->q + b * P->q_stride[0] + hq * P->q_stride[1] + q * P->q_stride[2];
    for (int64_t kv = 0; kv < P->kv_len; ++kv) {
        const uint16_t* krow = P->k + b * P->k_stride[0] + hk * P->k_stride[1] + kv * P->k_stride[2];
        double dot = 0.0;
        for (int d = 0; d < P->D; ++d)
            dot += bf16_to_double(qrow[d * P->q_stride[3]]) * bf16_to_double(krow[d * P->k_stride[3]]);
        double sm = score_mod(P, dot * P->scale, b, hq, q, kv);
        s[kv] = orc_mask_value(m, b, hq, q, kv) ? sm : -INFINITY;
    }
}

/* Softmax probabilities of one row (for the row-sum property); returns LSE. */
double orc_prob_row(const orc_problem* P, const orc_mask* m, int b, int hq, int64_t q, double* p)
{
    score_row(P, m, b, hq, q, p);
    double mx = -INFINITY;
    for (int64_t kv = 0; kv < P->kv_len; ++kv) mx = p[kv] > mx ? p[kv] : mx;
    if (mx == -INFINITY) {
        for (int64_t kv = 0; kv < P->kv_len; ++kv) p[kv] = 0.0;
        return -INFINITY;
    }
    double l = 0.0;
    for (int64_t kv = 0; kv < P->kv_len; ++kv) {
        p[kv] = exp(p[kv] - mx);
        l += p[kv];
    }
    for (int64_t kv = 0; kv < P->kv_len; ++kv) p[kv] /= l;
    return mx + log(l);
}

/* O row and LSE of one query: O = sum_kv p[kv] V[kv,:] / l, LSE = m + ln l. */
static void forward_row(const orc_problem* P, const orc_mask* m, int b, int hq, int64_t q,
                        double* s, double* o, double* lse)
{
    int G = P->Hq / P->Hkv;
    int hk = hq / G;
    score_row(P, m, b, hq, q, s);
    double mx = -INFINITY;
    for (int64_t kv = 0; kv < P->kv_len; ++kv) mx = s[kv] > mx ? s[kv] : mx;
    for (int d = 0; d < P->D; ++d) o[d] = 0.0;
    if (mx == -INFINITY) {
        *lse = -INFINITY;
        return;
    }
    double l = 0.0;
    for (int64_t kv = 0; kv < P->kv_len; ++kv) {
        double p = exp(s[kv] - mx);
        l += p;
        const uint16_t* vrow = P->v + b * P->v_stride[0] + hk * P->v_stride[1] + kv * P->v_stride[2];
        for (int d = 0; d < P->D; ++d) o[d] += p * bf16_to_double(vrow[d * P->v_stride[3]]);
    }
    for (int d = 0; d < P->D; ++d) o[d] /= l;
    *lse = mx + log(l);
}

/* d mod / ds of one scaled score (the score_mod's derivative; 1 for the additive
 * mods, 1 - tanh^2 for soft-capping). */
static double score_mod_grad(const orc_problem* P, double s, int b, int hq, int64_t q, int64_t kv)
{
    switch (P->score_kind) {
    case ORC_SCORE_SOFTCAP: {
        double t = tanh(s / P->softcap);
        return 1.0 - t * t;
    }
    case ORC_SCORE_BIAS_SOFTCAP: {
        double t = tanh((s + bias_at(P, b, hq, q, kv)) / P->softcap);
        return 1.0 - t * t;
    }
    default:
        return 1.0;
    }
}

typedef struct {
    const orc_problem* P;
    const orc_mask* m;
    const uint16_t* dO; int64_t do_stride[4];   /* [B,Hq,Sq,D] bf16 */
    double* dq;                                  /* [B,Hq,Sq,D] */
    double* dk;                                  /* [B,Hkv,Skv,D] */
    double* dv;                                  /* [B,Hkv,Skv,D] */
    const int32_t* units;                        /* [n][2] = (b, hkv) */
    int64_t n;
    int64_t next;
    pthread_mutex_t lock;
} bw_job;

/* Gradients of one (b, hkv) unit: every query row of every query head that reads
 * kv head hkv contributes to dK and dV of that head; its own dQ row is complete
 * after its pass.  Each unit owns its outputs, so units run in parallel. */
static void backward_unit(bw_job* J, int b, int hk, double* s, double* p)
{
    const orc_problem* P = J->P;
    const int G = P->Hq / P->Hkv, D = P->D;
    const int64_t Sq = P->q_len, Skv = P->kv_len;
    double* dk = J->dk + (((int64_t)b * P->Hkv + hk) * Skv) * D;
    double* dv = J->dv + (((int64_t)b * P->Hkv + hk) * Skv) * D;
    for (int64_t i = 0; i < Skv * D; ++i) dk[i] = dv[i] = 0.0;
    for (int hq = hk * G; hq < hk * G + G; ++hq) {
        for (int64_t q = 0; q < Sq; ++q) {
            double* dq = J->dq + (((int64_t)b * P->Hq + hq) * Sq + q) * D;
            for (int d = 0; d < D; ++d) dq[d] = 0.0;
            /* the probability row p (softmax of the modified, masked scores) */
            score_row(P, J->m, b, hq, q, s);
            double mx = -INFINITY;
            for (int64_t kv = 0; kv < Skv; ++kv) mx = s[kv] > mx ? s[kv] : mx;
            if (mx == -INFINITY) continue;  /* no admitted key: every gradient term is 0 */
            double l = 0.0;
            for (int64_t kv = 0; kv < Skv; ++kv) {
                p[kv] = exp(s[kv] - mx);
                l += p[kv];
            }
            for (int64_t kv = 0; kv < Skv; ++kv) p[kv] /= l;
            const uint16_t* qrow = P->q + b * P->q_stride[0] + hq * P->q_stride[1] + q * P->q_stride[2];
            const uint16_t* dorow = J->dO + b * J->do_stride[0] + hq * J->do_stride[1] + q * J->do_stride[2];
            /* dP[kv] = dO . V[kv] (reuses s), and the row term sum_kv p dP */
            double delta = 0.0;
            for (int64_t kv = 0; kv < Skv; ++kv) {
                const uint16_t* vrow = P->v + b * P->v_stride[0] + hk * P->v_stride[1] + kv * P->v_stride[2];
                double dp = 0.0;
                for (int d = 0; d < D; ++d)
                    dp += bf16_to_double(dorow[d * J->do_stride[3]]) * bf16_to_double(vrow[d * P->v_stride[3]]);
                s[kv] = dp;
                delta += p[kv] * dp;
            }
            for (int64_t kv = 0; kv < Skv; ++kv) {
                if (p[kv] == 0.0) continue;
                const uint16_t* krow = P->k + b * P->k_stride[0] + hk * P->k_stride[1] + kv * P->k_stride[2];
                /* the raw scaled score, for the score_mod's derivative */
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += bf16_to_double(qrow[d * P->q_stride[3]]) * bf16_to_double(krow[d * P->k_stride[3]]);
                const double ds = p[kv] * (s[kv] - delta) * score_mod_grad(P, dot * P->scale, b, hq, q, kv);
                for (int d = 0; d < D; ++d) {
                    dq[d] += P->scale * ds * bf16_to_double(krow[d * P->k_stride[3]]);
                    dk[kv * D + d] += P->scale * ds * bf16_to_double(qrow[d * P->q_stride[3]]);
                    dv[kv * D + d] += p[kv] * bf16_to_double(dorow[d * J->do_stride[3]]);
                }
            }
        }
    }
}

static void* backward_worker(void* arg)
{
    bw_job* J = (bw_job*)arg;
    size_t n = (size_t)(J->P->kv_len > 0 ? J->P->kv_len : 1);
    double* s = (double*)malloc(sizeof(double) * n);
    double* p = (double*)malloc(sizeof(double) * n);
    if (s && p) {
        for (;;) {
            pthread_mutex_lock(&J->lock);
            int64_t i = J->next++;
            pthread_mutex_unlock(&J->lock);
            if (i >= J->n) break;
            backward_unit(J, J->units[2 * i], J->units[2 * i + 1], s, p);
        }
    }
    free(s);
    free(p);
    return NULL;
}

/* dQ [B,Hq,Sq,D], dK and dV [B,Hkv,Skv,D] (fp64, contiguous) of the forward pass
 * for upstream gradient dO, over the listed (b, hkv) units (other entries are
 * left untouched). */
int orc_backward(const orc_problem* P, const orc_mask* m, const uint16_t* dO, const int64_t* do_stride,
                 const int32_t* units, int64_t n_units, double* dq, double* dk, double* dv, int n_threads)
{
    if (P->Hkv <= 0 || P->Hq % P->Hkv != 0) return -1;
    bw_job J;
    memset(&J, 0, sizeof J);
    J.P = P; J.m = m; J.dO = dO;
    for (int i = 0; i < 4; ++i) J.do_stride[i] = do_stride[i];
    J.dq = dq; J.dk = dk; J.dv = dv; J.units = units; J.n = n_units;
    pthread_mutex_init(&J.lock, NULL);
    run_threads(backward_worker, &J, n_threads);
    pthread_mutex_destroy(&J.lock);
    return 0;
}

/* The transposed BlockMask ("Concepts", BlockMask Internals: q_num_blocks /
 * q_indices, full_q_num_blocks / full_q_indices): for each kv block, the query
 * blocks whose tile with it is partial (q_*) or full (full_q_*), ascending,
 * padded with 0; arrays [B,H,nkv] and [B,H,nkv,nq]. */
int orc_block_mask_transposed(const orc_mask* m, int B, int H, int64_t q_len, int64_t kv_len, int bs,
                              int32_t* q_num, int32_t* q_idx, int32_t* full_num, int32_t* full_idx)
{
    if (bs <= 0) return -1;
    const int64_t nq = (q_len + bs - 1) / bs, nkv = (kv_len + bs - 1) / bs;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int64_t kb = 0; kb < nkv; ++kb) {
                const int64_t r = ((int64_t)b * H + h) * nkv + kb;
                int32_t np = 0, nf = 0;
                for (int64_t qb = 0; qb < nq; ++qb) {
                    q_idx[r * nq + qb] = 0;
                    full_idx[r * nq + qb] = 0;
                }
                for (int64_t qb = 0; qb < nq; ++qb) {
                    int c = orc_block_class(m, b, h, q_len, kv_len, bs, qb, kb);
                    if (c == ORC_PARTIAL) q_idx[r * nq + np++] = (int32_t)qb;
                    if (c == ORC_FULL) full_idx[r * nq + nf++] = (int32_t)qb;
                }
                q_num[r] = np;
                full_num[r] = nf;
            }
    return 0;
}

typedef struct {
    const orc_problem* P;
    const orc_mask* m;
    const int64_t* rows;             /* [n][3] = (b, hq, q) */
    int64_t n;
    double* o;                       /* [n][D] */
    double* lse;                     /* [n] */
    int64_t next;
    pthread_mutex_t lock;
} fw_job;

static void* forward_worker(void* arg)
{
    fw_job* J = (fw_job*)arg;
    double* s = (double*)malloc(sizeof(double) * (size_t)(J->P->kv_len > 0 ? J->P->kv_len : 1));
    if (!s) return NULL;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t i = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (i >= J->n) break;
        const int64_t* r = J->rows + 3 * i;
        forward_row(J->P, J->m, (int)r[0], (int)r[1], r[2], s, J->o + i * J->P->D, J->lse + i);
    }
    free(s);
    return NULL;
}

/* The forward pass for a list of query rows (all rows of a problem, or a sample). */
int orc_forward_rows(const orc_problem* P, const orc_mask* m, const int64_t* rows, int64_t n,
                     double* o, double* lse, int n_threads)
{
    if (P->Hkv <= 0 || P->Hq % P->Hkv != 0) return -1;
    fw_job J;
    memset(&J, 0, sizeof J);
    J.P = P; J.m = m; J.rows = rows; J.n = n; J.o = o; J.lse = lse;
    pthread_mutex_init(&J.lock, NULL);
    run_threads(forward_worker, &J, n_threads);
    pthread_mutex_destroy(&J.lock);
    return 0;
}
