// Host build of the forward kernel's per-row mask-word evaluation (csrc/mask_eval.cuh),
// for CPU unit tests: the device qualifiers are defined away and the two CUDA
// intrinsics the header uses get plain host stand-ins.
#include <cstdint>

#define __device__
#define __forceinline__ inline
struct int4 {
    int x, y, z, w;
};
template <typename T>
static inline T __ldg(const T* p)
{
    return *p;
}

#include "mask_eval.cuh"

namespace {

fa::MaskParams params(int n_leaves, int op, const int32_t* kind, const int64_t* param)
{
    fa::MaskParams m{};
    m.n_leaves = n_leaves;
    m.op = op;
    for (int i = 0; i < FA_MAX_LEAVES; ++i) {
        m.kind[i] = i < n_leaves ? kind[i] : 0;
        m.param[i] = i < n_leaves ? param[i] : 0;
    }
    return m;
}

} // namespace

// words[4] for one row (row_mask_words: 32-bit tile-local intervals).
extern "C" void fa_host_row_mask(int n_leaves, int op, const int32_t* kind, const int64_t* param,
                                 int64_t q, int64_t k0, int64_t kv_len, const uint32_t* dbits, uint32_t* words)
{
    const fa::MaskParams m = params(n_leaves, op, kind, param);
    const uint32_t d[4] = {dbits[0], dbits[1], dbits[2], dbits[3]};
    uint32_t w[4];
    fa::row_mask_words(m, q, k0, kv_len, d, w);
    for (int j = 0; j < 4; ++j) words[j] = w[j];
}

// words[4] for one key row of the backward pass's transposed tile (col_mask_words).
extern "C" void fa_host_col_mask(int n_leaves, int op, const int32_t* kind, const int64_t* param, int64_t kv,
                                 int64_t q0, int64_t q_len, const uint32_t* dbits, uint32_t* words)
{
    const fa::MaskParams m = params(n_leaves, op, kind, param);
    const uint32_t d[4] = {dbits[0], dbits[1], dbits[2], dbits[3]};
    uint32_t w[4];
    fa::col_mask_words(m, kv, q0, q_len, d, w);
    for (int j = 0; j < 4; ++j) words[j] = w[j];
}

// Tile summary used by the BlockMask build: 0 all masked, 1 all admitted, 2 undecided.
extern "C" int fa_host_mask_summary(int n_leaves, int op, const int32_t* kind, const int64_t* param, int64_t q0,
                                    int64_t q1, int64_t k0, int64_t k1, int32_t qmin, int32_t qmax, int32_t kmin,
                                    int32_t kmax)
{
    const fa::MaskParams m = params(n_leaves, op, kind, param);
    return fa::mask_summary(m, q0, q1, k0, k1, qmin, qmax, kmin, kmax);
}
