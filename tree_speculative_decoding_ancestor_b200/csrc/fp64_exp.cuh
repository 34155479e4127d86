// Table-driven fp64 exponential for the bulk passes of the verifier.
//
// Method: P. T. P. Tang, "Table-driven implementation of the exponential
// function in IEEE floating-point arithmetic", ACM TOMS 15(2), 1989:
//   x = n * ln2/128 + r,  |r| <= ln2/256,
//   e^x = 2^(n >> 7) * 2^((n & 127)/128) * e^r,
// with 2^(j/128) from a 128-entry table (filled with CUDA's exp2 and
// pre-multiplied by a per-row factor, so a normalising 1/Z costs nothing)
// and e^r - 1 from its Taylor series to degree 4 (truncation below 1.3e-15).
// The reduction is Cody-Waite with ln2/128 split as C_HI + C_LO (C_HI has a
// 24-bit significand, so n*C_HI is exact for |n| < 2^29; C_LO is the
// remainder to ~1e-27, computed offline in 80-digit decimal arithmetic), so
// r is exact to rounding over the whole range.  The relative error stays
// within a few ulp -- far inside what the sums of probabilities need (tokens
// are decided by the exact fp64 formula; these sums only set the normalisers
// and the CDF).
#pragma once

namespace tsd {

constexpr int kExpTable = 128;
constexpr double kLn2Over128Hi = 0x1.62e43p-8;              // 0.0054152123630046844
constexpr double kLn2Over128Lo = -0x1.05c610ca86c39p-36;    // -1.4880111718420063e-11
constexpr double kOneTwentyEightOverLn2 = 184.66496523378731;

// table[j] = scale * 2^(j/128), j = 0..127 (all threads of the block help).
__device__ __forceinline__ void fill_exp_table(double *table, double scale)
{
    for (int j = threadIdx.x; j < kExpTable; j += blockDim.x)
        table[j] = scale * exp2((double)j / (double)kExpTable);
}

// scale * e^x for x <= 0; 0 for x < -708 (where e^x leaves the normal range).
// n = round(x * 128/ln2) by adding 1.5 * 2^52 (the sum's last significand
// bit is worth 1, so the addition rounds to nearest and leaves n in the low
// bits of the sum), which keeps the reduction on the FMA pipe instead of the
// conversion unit; n may differ by one from rounding the rounded product,
// which only moves r a rounding error past ln2/256.
__device__ __forceinline__ double table_exp(double x, const double *table)
{
    constexpr double kRound = 6755399441055744.0;   // 1.5 * 2^52
    const bool under = x < -708.0;
    x = under ? -708.0 : x;
    const double sum = fma(x, kOneTwentyEightOverLn2, kRound);
    const double n = sum - kRound;
    const double r = fma(n, -kLn2Over128Lo, fma(n, -kLn2Over128Hi, x));
    const int ni = __double2loint(sum);
    double p = 1.0 / 24.0;
    p = fma(p, r, 1.0 / 6.0);
    p = fma(p, r, 0.5);
    p = fma(p, r, 1.0);
    p = p * r;                               // e^r - 1
    const double t = table[ni & (kExpTable - 1)];
    const double y = fma(t, p, t);           // scale * 2^(j/128) * e^r
    const long long bits = __double_as_longlong(y) + ((long long)(ni >> 7) << 52);
    return under ? 0.0 : __longlong_as_double(bits);
}

}  // namespace tsd
