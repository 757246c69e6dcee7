// Exact arithmetic for the few candidates the fp32 filter cannot separate.
//
// A node score is x(k) = sum_n sum_d q[n][d] k[d] over the stored numbers
// (binary32, or bfloat16 widened exactly).  Every stored number is m * 2^e
// with an integer m < 2^24 and e >= -149, so x(k) is an integer multiple of
// 2^-298 and can be accumulated without rounding in fixed point (Kulisch's
// exact dot product): 20 digits of weight 2^(32 i - 298), each held in int64
// so carries are deferred to one final normalisation.
#pragma once

#include "common.cuh"

namespace akv {

constexpr int kScoreDigits = 20;  // |x| < 2^290 for N < 2^16, D <= 128

__device__ __forceinline__ int split_binary32(uint32_t bits, uint32_t &mant, int &lsb)
{
    const int neg = (int)(bits >> 31);
    const int biased = (int)((bits >> 23) & 0xffu);
    const uint32_t frac = bits & 0x7fffffu;
    if (biased == 0) {
        mant = frac;
        lsb = -149;
    } else {
        mant = frac | 0x800000u;
        lsb = biased - 150;
    }
    return neg;
}

// Carry-propagate int64 digits (radix 2^32) to canonical form: digits
// 0..n-2 in [0, 2^32), the top digit signed.
template <int NDIG>
__device__ __forceinline__ void normalize_digits(int64_t *dig)
{
#pragma unroll
    for (int i = 0; i < NDIG - 1; ++i) {
        const int64_t carry = dig[i] >> 32;  // arithmetic shift = floor division
        dig[i] -= carry * 4294967296LL;
        dig[i + 1] += carry;
    }
}

// Compare two canonical exact scores: -1, 0, +1.
__device__ __forceinline__ int exact_cmp(const uint32_t *a, const uint32_t *b)
{
    const int32_t ta = (int32_t)a[kScoreDigits - 1], tb = (int32_t)b[kScoreDigits - 1];
    if (ta != tb) return ta < tb ? -1 : 1;
    for (int i = kScoreDigits - 2; i >= 0; --i)
        if (a[i] != b[i]) return a[i] < b[i] ? -1 : 1;
    return 0;
}

// Strict total order used for selection: higher exact score first, then lower id.
__device__ __forceinline__ bool exact_better(const uint32_t *xa, int ida, const uint32_t *xb, int idb)
{
    const int c = exact_cmp(xa, xb);
    return c > 0 || (c == 0 && ida < idb);
}

}  // namespace akv
