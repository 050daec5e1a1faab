// Numeric building blocks shared by the scoring kernels (the two-phase
// score pass A / vote pass B and the fused one-kernel scoring): online
// softmax normalisers, the order-preserving float key of the integer warp
// max, the balanced chunk split of the persistent grids, and the exponential
// with an exactly formed argument that turns a logit and its head's
// log-normaliser into a soft-vote term.
#pragma once

#include <stdint.h>

namespace ts {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2eHi = 1.44269502162933349609375f;   // float nearest log2(e)
constexpr float kLog2eLo = 1.925963033500011e-08f;       // log2(e) - kLog2eHi
constexpr float kLn2 = 0.693147180559945309f;

// One logit x into a running (max m, sum z of exp(. - m)).
__device__ __forceinline__ void online_push(float &m, float &z, float x)
{
    if (x > m) {
        z = z * exp2f((m - x) * kLog2e) + 1.0f;
        m = x;
    } else {
        z += exp2f((x - m) * kLog2e);
    }
}

// Order-preserving map of a float to a signed integer (and back), for the
// integer warp max reduction.
__device__ __forceinline__ int32_t float_order_key(float x)
{
    const int32_t b = __float_as_int(x);
    return b >= 0 ? b : (b ^ 0x7fffffff);
}
__device__ __forceinline__ float float_from_order_key(int32_t k)
{
    return __int_as_float(k >= 0 ? k : (k ^ 0x7fffffff));
}

// floor(j * total / grid) for j <= grid <= 256 and total < 2^31: a double
// quotient is exact enough (a non-integer quotient is at least 1/grid away
// from an integer, far above the rounding error) and much cheaper than a
// 64-bit integer division.
__device__ __forceinline__ int32_t chunk_split(uint32_t j, int32_t total, uint32_t grid)
{
    return (int32_t)floor((double)j * (double)total / (double)grid);
}

// exp(s - L) for an fp32 logit s and a float64 log-normaliser L given as
// L = Lhi + Llo (Lhi = (float)L, Llo = (float)(L - Lhi)).
// s - L is formed exactly as t + d (two-sum of s and -Lhi, minus Llo), and
// the base-2 exponent u = (t + d) log2(e) is carried as an unevaluated pair:
// u_hi = fl(t * log2e_hi) and
//   u_lo = fma(t, log2e_hi, -u_hi) + t * log2e_lo + d * log2e_hi
// (the product error recovered with one fma, as in Dekker's exact product,
// with log2(e) split Cody-Waite style into a float head and tail), so that
// exp(s - L) = 2^u_hi * (1 + u_lo ln 2) up to second order in |u_lo| < 2^-17.
// The only rounding left is the hardware 2^x (a few 1e-8 relative); a plain
// fp32 s - L would lose up to half an ulp of |s - L| (~1e-6 relative for
// |s - L| ~ 20), the width of the selection band.
__device__ __forceinline__ float exp_exact_arg(float s, float Lhi, float Llo)
{
    const float t = s - Lhi;                       // two-sum: t + e == s - Lhi
    const float bp = t - s;
    const float e = (s - (t - bp)) + (-Lhi - bp);
    const float d = e - Llo;                       // s - L == t + d
    const float u = t * kLog2eHi;
    const float u_lo = fmaf(t, kLog2eHi, -u) + fmaf(t, kLog2eLo, d * kLog2eHi);
    const float p = exp2f(u);
    return fmaf(p, u_lo * kLn2, p);
}

}  // namespace ts
