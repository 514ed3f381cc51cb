// Score arithmetic shared by the forward and backward kernels: an accurate tanh
// for soft-capping (tanh.approx's ~2^-11 relative error, times a cap of 30, would
// move scores by ~1e-2).
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace fa {

constexpr float kTanhPolyMax = 0.625f;  // |y| up to which the polynomial is used

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

__device__ __forceinline__ float tanh_far(float y)
{
    const float a = fabsf(y);
    const float e = ex2_approx(2.0f * 1.4426950408889634f * a);
    const float t = 1.0f - __fdividef(2.0f, e + 1.0f);
    return copysignf(t, y);
}

// tanh(y) of one value: the polynomial for |y| <= 0.625, else the exponential form.
__device__ __forceinline__ float tanh_accurate(float y)
{
    if (fabsf(y) > kTanhPolyMax) return tanh_far(y);
    float t0, t1;
    f2_unpack(tanh_poly2(f2_pack(y, y)), t0, t1);
    return t0;
}

} // namespace fa
