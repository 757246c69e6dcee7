// Exact node scores for the few candidates the fp32 filter cannot separate.
//
// A node score is x(k) = sum_n sum_d q[n][d] k[d] over the stored numbers
// (binary32, or bfloat16 widened exactly).  Every stored number is m * 2^e
// with an integer m < 2^24 and e >= -149, so x(k) is an integer multiple of
// 2^-298 and can be accumulated without rounding in fixed point (Kulisch's
// exact dot product).  Here the token sums s[d] = sum_n q[n][d] are formed
// exactly first (10 signed 32-bit digits, weight of digit i = 2^(32 i - 149)),
// then x(k) = sum_d s[d] k[d] is accumulated in 20 digits of weight
// 2^(32 i - 298).  Digits live in int64 so carries are deferred to one final
// normalisation.
#pragma once

#include "common.cuh"

namespace akv {

constexpr int kSumDigits = 10;    // token-sum digits; |s| < 2^144 for N < 2^16
constexpr int kScoreDigits = 20;  // score digits; |x| < 2^290 for D <= 128

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

// Exact token sums of one traversal, one thread per column d (the calling
// block covers d = threadIdx.x, threadIdx.x + blockDim.x, ...).
// Output (shared): mag[i * D + d] digit i of |s[d]|, neg[d], lo[d]/hi[d] the
// first/last nonzero digit (lo > hi when s[d] = 0).  acc is int64 scratch of
// kSumDigits * D entries.
template <typename T, int D>
__device__ void exact_token_sums(const T *q, size_t q_row_stride, int N, int64_t *acc,
                                 uint32_t *mag, uint8_t *neg, int8_t *lo, int8_t *hi)
{
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
        int64_t a[kSumDigits];
#pragma unroll
        for (int i = 0; i < kSumDigits; ++i) a[i] = 0;
        for (int n = 0; n < N; ++n) {
            uint32_t m;
            int e;
            const int sgn = split_binary32(elem_bits(q[(size_t)n * q_row_stride + d]), m, e);
            if (m == 0) continue;
            const int p = e + 149;               // 0 .. 253
            const int di = p >> 5, sh = p & 31;
            const uint64_t v = ((uint64_t)m) << sh;   // < 2^55
            const int64_t c0 = (int64_t)(v & 0xffffffffull), c1 = (int64_t)(v >> 32);
            // di is dynamic: select into the register array without local memory
#pragma unroll
            for (int i = 0; i < kSumDigits - 1; ++i) {
                if (i == di) {
                    a[i] += sgn ? -c0 : c0;
                    a[i + 1] += sgn ? -c1 : c1;
                }
            }
        }
        normalize_digits<kSumDigits>(a);
        const bool negative = a[kSumDigits - 1] < 0;
        if (negative) {
#pragma unroll
            for (int i = 0; i < kSumDigits; ++i) a[i] = -a[i];
            normalize_digits<kSumDigits>(a);
        }
        int first = kSumDigits, last = -1;
#pragma unroll
        for (int i = 0; i < kSumDigits; ++i) {
            mag[i * D + d] = (uint32_t)a[i];
            if (a[i] != 0) {
                if (first == kSumDigits) first = i;
                last = i;
            }
        }
        neg[d] = negative ? 1 : 0;
        lo[d] = (int8_t)first;
        hi[d] = (int8_t)last;
        (void)acc;
    }
}

// Exact score of one key row, computed by one warp; lane 0 writes the 20
// canonical digits (uint32 each; the top one is a signed int32) to out.
template <typename T, int D>
__device__ void exact_row_score(const T *krow, const uint32_t *mag, const uint8_t *neg,
                                const int8_t *lo, const int8_t *hi, uint32_t *out)
{
    const int lane = threadIdx.x & 31;
    int64_t acc[kScoreDigits];
#pragma unroll
    for (int i = 0; i < kScoreDigits; ++i) acc[i] = 0;
    for (int d = lane; d < D; d += 32) {
        uint32_t mk;
        int ek;
        const int sk = split_binary32(elem_bits(krow[d]), mk, ek);
        if (mk == 0 || lo[d] > hi[d]) continue;
        const bool minus = (sk != 0) != (neg[d] != 0);
        for (int i = lo[d]; i <= hi[d]; ++i) {
            const uint32_t si = mag[i * D + d];
            if (si == 0) continue;
            const uint64_t prod = (uint64_t)si * (uint64_t)mk;  // < 2^56
            const int p = 32 * i + ek + 149;                     // >= 0
            const int di = p >> 5, sh = p & 31;
            const uint64_t lo64 = prod << sh;
            const uint64_t hi64 = sh ? (prod >> (64 - sh)) : 0ull;
            const int64_t c0 = (int64_t)(lo64 & 0xffffffffull);
            const int64_t c1 = (int64_t)(lo64 >> 32);
            const int64_t c2 = (int64_t)hi64;
#pragma unroll
            for (int j = 0; j < kScoreDigits - 2; ++j) {
                if (j == di) {
                    acc[j] += minus ? -c0 : c0;
                    acc[j + 1] += minus ? -c1 : c1;
                    acc[j + 2] += minus ? -c2 : c2;
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kScoreDigits; ++i) {
        int64_t v = acc[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        acc[i] = v;
    }
    if (lane == 0) {
        normalize_digits<kScoreDigits>(acc);
#pragma unroll
        for (int i = 0; i < kScoreDigits; ++i) out[i] = (uint32_t)acc[i];
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
