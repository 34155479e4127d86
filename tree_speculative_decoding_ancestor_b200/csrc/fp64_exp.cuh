// Table-driven fp64 exponential for the bulk passes of the verifier.
//
// Method: P. T. P. Tang, "Table-driven implementation of the exponential
// function in IEEE floating-point arithmetic", ACM TOMS 15(2), 1989:
//   x = n * ln2/64 + r,  |r| <= ln2/128,
//   e^x = 2^(n >> 6) * 2^((n & 63)/64) * e^r,
// with 2^(j/64) from a 64-entry table (filled by the caller with CUDA's exp2)
// and e^r - 1 from its Taylor series to degree 5 (truncation below 4e-17).
// ln2/64 is split as C_HI + C_LO (C_HI has a 24-bit significand, so n*C_HI
// is exact for |n| < 2^29; C_LO is the remainder to ~1e-27, computed offline
// in 80-digit decimal arithmetic), which keeps the reduction error negligible
// over the whole range.  The relative error stays within a few ulp, far
// inside what the sums of probabilities need (the tokens are decided by the
// exact fp64 formula; these sums only set the normalisers and the CDF).
#pragma once

namespace tsd {

constexpr double kLn2Over64Hi = 0x1.62e43p-7;              // 0.010830424726009369
constexpr double kLn2Over64Lo = -0x1.05c610ca86c39p-35;     // -2.9760223436840126e-11
constexpr double kSixtyFourOverLn2 = 92.33248261689366;

// table[j] = 2^(j/64), j = 0..63.
__device__ __forceinline__ void fill_exp_table(double *table)
{
    for (int j = threadIdx.x; j < 64; j += blockDim.x)
        table[j] = exp2((double)j / 64.0);
}

__device__ __forceinline__ double table_exp(double x, const double *table)
{
    if (x < -708.0)
        return 0.0;
    const double n = rint(x * kSixtyFourOverLn2);
    const double r = fma(n, -kLn2Over64Lo, fma(n, -kLn2Over64Hi, x));
    const int ni = (int)n;
    double p = 1.0 / 120.0;
    p = fma(p, r, 1.0 / 24.0);
    p = fma(p, r, 1.0 / 6.0);
    p = fma(p, r, 0.5);
    p = fma(p, r, 1.0);
    p = p * r;                               // e^r - 1
    const double t = table[ni & 63];
    const double y = fma(t, p, t);           // 2^(j/64) * e^r, in [0.99, 2.02]
    const long long bits = __double_as_longlong(y) + ((long long)(ni >> 6) << 52);
    return __longlong_as_double(bits);
}

}  // namespace tsd
