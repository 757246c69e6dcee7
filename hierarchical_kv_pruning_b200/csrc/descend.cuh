// Level-by-level HiKVP descent: one CTA per traversal (query b, head h).
//
// "AtlasKV: Augmenting LLMs with Billion-Scale Knowledge Graphs in 20GB VRAM",
// section "Quick read / How it works": score the query against the resident
// root keys, keep the top-K branches, bring in the children's keys, prune level
// by level down to the leaves.  Node score (reading of that section): mean over
// the query tokens of <q_n, k>/sqrt(D); ranking by x(k) = sum_d s[d] k[d] with
// s[d] = sum_n q[n][d] is equivalent.
//
// Ranking is exact.  Each candidate gets an fp32 score f (token sums and dot
// products in fp32) with the rigorous bound |f - x| <= E, where
//   E = (g_D (1 + g_N) + g_N) * ||a||_2 * max_k ||k||_2 + D 2^-148,
//   g_n = n u / (1 - n u), u = 2^-24, a[d] = sum_n |q[n][d]|
// (Higham's dot-product and summation bounds plus Cauchy-Schwarz; the last
// term covers underflow).  With t the K-th largest f, every candidate with
// f > t + 2E is certainly kept, every one with f < t - 2E certainly dropped;
// the rest (always containing t's candidate) are ranked by their exact score
// (exact.cuh) and then by lower row id.
#pragma once

#include <float.h>

#include "common.cuh"
#include "exact.cuh"

namespace akv {

constexpr int kDescendThreads = 256;
constexpr int kRefineChunk = 64;

struct DescendParams {
    const void *q_kg;            // [B][N][H][D]
    int B, N, H, H_kv, G;
    const void *keys[3];         // key base per level (level 2: device leaf keys or staged pool)
    long long rows[3];           // rows per KV head: b_R, b_R b_I, b_R b_I b_L
    int fanout[3];               // b_R, b_I, b_L
    const int32_t *child[2];     // root_child [H_kv][b_R][b_I], mid_child [H_kv][b_R b_I][b_L], or null
    const float *norm_bound;     // [3][H_kv] upper bounds of key row 2-norms
    int K[3];
    int32_t *kept[3];            // [B H][K_l] ascending row ids
    float *s_ws;                 // [B H][D] fp32 token sums (split launches)
    float *anorm_ws;             // [B H] upper bound of ||a||_2 (split launches)
    int first_level, last_level;
    int cap;                     // candidate capacity (power of two >= every level's C)
    int kcap;                    // kept capacity (power of two >= every K)
    // host-staged leaves: kept mid k of traversal bh has its leaf block at pool slot
    // leaf_slot[bh K_mid + k]; leaf candidate (k, j) is pool row slot * b_L + j.
    const int32_t *leaf_slot;
    int32_t *kept_leaf_row;      // [B H][K_leaf] pool row of each kept leaf (host path)
    int *status;
};

__device__ __forceinline__ double gamma_n(int n)
{
    const double nu = (double)n * 0x1p-24;
    return nu / (1.0 - nu);
}

// --------------------------------------------------------------------------
// Block-wide k-th largest (1-based) of n uint32 keys, MSB-first radix select.
template <typename KeyFn>
__device__ uint32_t block_kth_largest(int n, int k, KeyFn key_of, uint32_t *hist, int *misc)
{
    uint32_t prefix = 0, mask = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const uint32_t key = key_of(i);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            uint32_t cnt[8], tot = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                cnt[j] = hist[255 - 8 * lane - j];
                tot += cnt[j];
            }
            uint32_t incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const uint32_t excl = incl - tot;
            if (excl < (uint32_t)k && (uint32_t)k <= incl) {
                uint32_t run = excl;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (run + cnt[j] >= (uint32_t)k) {
                        misc[0] = 255 - 8 * lane - j;
                        misc[1] = k - (int)run;
                        break;
                    }
                    run += cnt[j];
                }
            }
        }
        __syncthreads();
        prefix |= ((uint32_t)misc[0]) << shift;
        mask |= 255u << shift;
        k = misc[1];
        __syncthreads();
    }
    return prefix;
}

// Ascending block bitonic sort of n (power of two) uint64 values.
__device__ void block_sort_u64(uint64_t *a, int n)
{
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncthreads();
            for (int i = threadIdx.x; i < n / 2; i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool asc = (lo & size) == 0;
                const uint64_t x = a[lo], y = a[hi];
                if ((x > y) == asc) {
                    a[lo] = y;
                    a[hi] = x;
                }
            }
        }
    }
    __syncthreads();
}

// --------------------------------------------------------------------------
// fp32 filter scores f[c] = sum_d s[d] * key[cand_row[c]][d].  Eight lanes per
// candidate, each holding the token sums of its slice of d; every 16-byte
// vector read is part of a 128-byte coalesced row segment.
template <typename T, int D>
__device__ void score_candidates(const T *__restrict__ base, const int32_t *cand_row, int C,
                                 const float *s, float *f)
{
    constexpr int EV = Vec16<T>::E;
    constexpr int VPR = D / EV;
    constexpr int LPG = 8;
    constexpr int VPL = VPR / LPG;
    constexpr int U = 4;
    static_assert(VPL >= 1 && VPR % LPG == 0, "row must split over 8 lanes");
    const int sub = threadIdx.x & 7;
    const int grp = threadIdx.x >> 3;
    const int ngrp = blockDim.x >> 3;
    float sreg[VPL * EV];
#pragma unroll
    for (int v = 0; v < VPL; ++v)
#pragma unroll
        for (int e = 0; e < EV; ++e) sreg[v * EV + e] = s[(sub + LPG * v) * EV + e];

    for (int base_c = 0; base_c < C; base_c += ngrp * U) {
        uint4 buf[U][VPL];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = base_c + u * ngrp + grp;
            const bool ok = c < C;
            const T *row = base + (size_t)(ok ? cand_row[c] : 0) * D;
#pragma unroll
            for (int v = 0; v < VPL; ++v)
                buf[u][v] = ok ? ldg16(row + (sub + LPG * v) * EV) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float acc = 0.f;
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                float x[EV];
                Vec16<T>::unpack(buf[u][v], x);
#pragma unroll
                for (int e = 0; e < EV; ++e) acc = fmaf(sreg[v * EV + e], x[e], acc);
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 4);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            const int c = base_c + u * ngrp + grp;
            if (sub == 0 && c < C) f[c] = acc;
        }
    }
}

// --------------------------------------------------------------------------
// Shared-memory layout of one descent CTA.
template <int D>
struct DescendSmem {
    float *s;          // [D] fp32 token sums
    float *absq;       // [D] fp32 sums of |q|
    int32_t *cand_id;  // [cap]
    int32_t *cand_row; // [cap]
    float *cand_f;     // [cap]   } contiguous: reused as the uint64 sort buffer
    int32_t *alist;    // [cap]   }
    int32_t *kept_pos; // [kcap]
    int32_t *kept_id;  // [kcap]  parents of the next level
    uint32_t *hist;    // [256]
    int *misc;         // [16]
    double *dmisc;     // [8]
    // refinement
    uint32_t *ex;      // [3 * kRefineChunk][kScoreDigits]
    int32_t *ex_id;    // [3 * kRefineChunk]
    int32_t *ex_pos;   // [3 * kRefineChunk]
    int32_t *ex_rank;  // [4 * kRefineChunk] ranks + validity flags
    uint32_t *smag;    // [kSumDigits * D]
    uint8_t *sneg;     // [D]
    int8_t *slo, *shi; // [D]

    __device__ DescendSmem(uint8_t *p, int cap, int kcap)
    {
        auto take = [&](size_t bytes) {
            uint8_t *r = p;
            p += (bytes + 15) & ~size_t(15);
            return r;
        };
        dmisc = (double *)take(8 * sizeof(double));
        s = (float *)take(D * sizeof(float));
        absq = (float *)take(D * sizeof(float));
        cand_id = (int32_t *)take(cap * 4);
        cand_row = (int32_t *)take(cap * 4);
        cand_f = (float *)take(cap * 4);
        alist = (int32_t *)take(cap * 4);
        kept_pos = (int32_t *)take(kcap * 4);
        kept_id = (int32_t *)take(kcap * 4);
        hist = (uint32_t *)take(256 * 4);
        misc = (int *)take(16 * 4);
        ex = (uint32_t *)take(3 * kRefineChunk * kScoreDigits * 4);
        ex_id = (int32_t *)take(3 * kRefineChunk * 4);
        ex_pos = (int32_t *)take(3 * kRefineChunk * 4);
        ex_rank = (int32_t *)take(4 * kRefineChunk * 4);
        smag = (uint32_t *)take(kSumDigits * D * 4);
        sneg = (uint8_t *)take(D);
        slo = (int8_t *)take(D);
        shi = (int8_t *)take(D);
    }

    static size_t bytes(int cap, int kcap)
    {
        auto r = [](size_t b) { return (b + 15) & ~size_t(15); };
        return r(64) + 2 * r(D * 4) + 4 * r((size_t)cap * 4) + 2 * r((size_t)kcap * 4) + r(1024) + r(64) +
               r(3 * kRefineChunk * kScoreDigits * 4) + 2 * r(3 * kRefineChunk * 4) + r(4 * kRefineChunk * 4) +
               r(kSumDigits * D * 4) + 3 * r(D);
    }
};

// Pick the r best of the ambiguous candidates alist[0..nA) by (exact score
// desc, row id asc) and append their positions to kept_pos[base_out..).
// The ambiguous set is processed in chunks with a bounded best-set; passes
// repeat (each excluding what earlier passes chose, i.e. everything not
// strictly worse than the last chosen "pivot") until r are chosen.
template <typename T, int D>
__device__ void refine_exact(DescendSmem<D> &sm, const T *qbase, size_t q_stride, int N,
                             const T *__restrict__ kbase, int nA, int r, int base_out)
{
    constexpr int RC = kRefineChunk;
    static_assert(kDescendThreads >= 2 * RC, "one pool element per thread");
    const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    exact_token_sums<T, D>(qbase, q_stride, N, nullptr, sm.smag, sm.sneg, sm.slo, sm.shi);
    __syncthreads();

    uint32_t *BEST = sm.ex;                        // [RC]
    uint32_t *CH = sm.ex + RC * kScoreDigits;      // [RC]
    uint32_t *TMP = sm.ex + 2 * RC * kScoreDigits; // [RC]
    int32_t *best_id = sm.ex_id, *ch_id = sm.ex_id + RC, *tmp_id = sm.ex_id + 2 * RC;
    int32_t *best_pos = sm.ex_pos, *ch_pos = sm.ex_pos + RC, *tmp_pos = sm.ex_pos + 2 * RC;
    int32_t *valid = sm.ex_rank + 2 * RC;          // [2 RC]
    int32_t *rank = sm.ex_rank;                    // [2 RC]

    int chosen = 0;
    bool have_pivot = false;
    uint32_t pivot[kScoreDigits];
    int pivot_id = 0;
    while (chosen < r) {
        const int want = min(r - chosen, RC);
        int nbest = 0;
        for (int b0 = 0; b0 < nA; b0 += RC) {
            const int len = min(RC, nA - b0);
            for (int i = warp; i < len; i += nwarps) {
                const int pos = sm.alist[b0 + i];
                exact_row_score<T, D>(kbase + (size_t)sm.cand_row[pos] * D, sm.smag, sm.sneg, sm.slo, sm.shi,
                                      CH + i * kScoreDigits);
                if ((threadIdx.x & 31) == 0) {
                    ch_id[i] = sm.cand_id[pos];
                    ch_pos[i] = pos;
                }
            }
            __syncthreads();
            // pool = BEST[0..nbest) + chunk members strictly worse than the pivot
            const int npool = nbest + len;
            const int e = threadIdx.x;
            const uint32_t *xe = nullptr;
            int ide = 0;
            if (e < npool) {
                xe = e < nbest ? BEST + e * kScoreDigits : CH + (e - nbest) * kScoreDigits;
                ide = e < nbest ? best_id[e] : ch_id[e - nbest];
                valid[e] = (e < nbest || !have_pivot || exact_better(pivot, pivot_id, xe, ide)) ? 1 : 0;
            }
            __syncthreads();
            int my_rank = 0x7fffffff;
            if (e < npool && valid[e]) {
                my_rank = 0;
                for (int f2 = 0; f2 < npool; ++f2) {
                    if (f2 == e || !valid[f2]) continue;
                    const uint32_t *xf = f2 < nbest ? BEST + f2 * kScoreDigits : CH + (f2 - nbest) * kScoreDigits;
                    const int idf = f2 < nbest ? best_id[f2] : ch_id[f2 - nbest];
                    if (exact_better(xf, idf, xe, ide)) ++my_rank;
                }
            }
            const int total_valid = __syncthreads_count(e < npool && valid[e]);
            if (my_rank < want) {
#pragma unroll
                for (int q = 0; q < kScoreDigits; ++q) TMP[my_rank * kScoreDigits + q] = xe[q];
                tmp_id[my_rank] = ide;
                tmp_pos[my_rank] = e < nbest ? best_pos[e] : ch_pos[e - nbest];
            }
            __syncthreads();
            nbest = min(want, total_valid);
            for (int i = threadIdx.x; i < nbest; i += blockDim.x) {
#pragma unroll
                for (int q = 0; q < kScoreDigits; ++q) BEST[i * kScoreDigits + q] = TMP[i * kScoreDigits + q];
                best_id[i] = tmp_id[i];
                best_pos[i] = tmp_pos[i];
            }
            __syncthreads();
        }
        for (int i = threadIdx.x; i < nbest; i += blockDim.x) sm.kept_pos[base_out + chosen + i] = best_pos[i];
        if (nbest == 0) break;  // only if r > nA, which the caller rules out
        chosen += nbest;
#pragma unroll
        for (int q = 0; q < kScoreDigits; ++q) pivot[q] = BEST[(nbest - 1) * kScoreDigits + q];
        pivot_id = best_id[nbest - 1];
        have_pivot = true;
        __syncthreads();
    }
    (void)rank;
}

// Select the K best candidates of cand_*[0..C) and leave their positions,
// sorted by ascending row id, in kept_pos[0..K); ids in kept_id.
template <typename T, int D>
__device__ void select_level(DescendSmem<D> &sm, int C, int K, double E, const T *qbase, size_t q_stride,
                             int N, const T *__restrict__ kbase, int cap)
{
    if (K >= C) {
        for (int c = threadIdx.x; c < C; c += blockDim.x) sm.kept_pos[c] = c;
        __syncthreads();
    } else {
        const float *f = sm.cand_f;
        const uint32_t tkey = block_kth_largest(C, K, [&](int i) { return float_key(f[i]); }, sm.hist, sm.misc);
        const double t = (double)key_float(tkey);
        // any non-finite filter score or bound: every candidate is ambiguous
        int bad = 0;
        for (int c = threadIdx.x; c < C; c += blockDim.x) bad |= !isfinite(f[c]);
        bad = __syncthreads_or(bad) || !isfinite(E) || !isfinite(t);
        const double two_e = 2.0 * E;
        const double hi = bad ? INFINITY : __dadd_ru(t, two_e);
        const double lo = bad ? -INFINITY : __dsub_rd(t, two_e);
        if (threadIdx.x == 0) {
            sm.misc[2] = 0;
            sm.misc[3] = 0;
        }
        __syncthreads();
        for (int c = threadIdx.x; c < C; c += blockDim.x) {
            const double fd = (double)f[c];
            if (!bad && fd > hi) {
                sm.kept_pos[atomicAdd(&sm.misc[2], 1)] = c;
            } else if (bad || fd >= lo) {
                sm.alist[atomicAdd(&sm.misc[3], 1)] = c;
            }
        }
        __syncthreads();
        const int n_in = sm.misc[2], nA = sm.misc[3];
        const int r = K - n_in;
        __syncthreads();
        if (nA == r) {
            for (int i = threadIdx.x; i < nA; i += blockDim.x) sm.kept_pos[n_in + i] = sm.alist[i];
            __syncthreads();
        } else {
            refine_exact<T, D>(sm, qbase, q_stride, N, kbase, nA, r, n_in);
            __syncthreads();
        }
    }
    // sort kept positions by row id: pack (id, pos) into uint64 in the cand_f/alist area
    int n2 = 1;
    while (n2 < K) n2 <<= 1;
    uint64_t *buf = reinterpret_cast<uint64_t *>(sm.cand_f);
    for (int i = threadIdx.x; i < n2; i += blockDim.x)
        buf[i] = i < K ? (((uint64_t)(uint32_t)sm.cand_id[sm.kept_pos[i]]) << 32) | (uint32_t)sm.kept_pos[i]
                       : ~0ull;
    block_sort_u64(buf, n2);
    for (int i = threadIdx.x; i < K; i += blockDim.x) {
        sm.kept_pos[i] = (int32_t)(uint32_t)(buf[i] & 0xffffffffull);
        sm.kept_id[i] = (int32_t)(buf[i] >> 32);
    }
    __syncthreads();
    (void)cap;
}

template <typename T, int D>
__global__ void __launch_bounds__(kDescendThreads) descend_kernel(const DescendParams p)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    DescendSmem<D> sm(smem_raw, p.cap, p.kcap);
    const int bh = blockIdx.x;
    const int b = bh / p.H, h = bh % p.H;
    const int hkv = h / p.G;
    const T *qbase = reinterpret_cast<const T *>(p.q_kg) + ((size_t)b * p.N * p.H + h) * D;
    const size_t q_stride = (size_t)p.H * D;

    // ---- token sums (a1) ----
    if (p.first_level == 0) {
        for (int d = threadIdx.x; d < D; d += blockDim.x) {
            float s = 0.f, a = 0.f;
            const T *q = qbase + d;
#pragma unroll 8
            for (int n = 0; n < p.N; ++n) {
                const float x = elem_f32(q[(size_t)n * q_stride]);
                s += x;
                a += fabsf(x);
            }
            sm.s[d] = s;
            sm.absq[d] = a;
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            double acc = 0.0;
            for (int d = threadIdx.x; d < D; d += 32) acc += (double)sm.absq[d] * (double)sm.absq[d];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (threadIdx.x == 0) {
                const double an = sqrt(acc) * (1.0 + 1e-12) / (1.0 - gamma_n(p.N));
                sm.dmisc[0] = an;
            }
        }
        __syncthreads();
        if (p.s_ws) {
            for (int d = threadIdx.x; d < D; d += blockDim.x) p.s_ws[(size_t)bh * D + d] = sm.s[d];
            if (threadIdx.x == 0) p.anorm_ws[bh] = (float)sm.dmisc[0] * (1.0f + 1e-6f);
        }
    } else {
        for (int d = threadIdx.x; d < D; d += blockDim.x) sm.s[d] = p.s_ws[(size_t)bh * D + d];
        if (threadIdx.x == 0) sm.dmisc[0] = (double)p.anorm_ws[bh];
        const int prev = p.first_level - 1;
        for (int i = threadIdx.x; i < p.K[prev]; i += blockDim.x)
            sm.kept_id[i] = p.kept[prev][(size_t)bh * p.K[prev] + i];
        __syncthreads();
    }
    const double anorm = sm.dmisc[0];
    const double cprime = gamma_n(D) * (1.0 + gamma_n(p.N)) + gamma_n(p.N);

    for (int L = p.first_level; L <= p.last_level; ++L) {
        const T *kbase = reinterpret_cast<const T *>(p.keys[L]);
        int C;
        if (L == 0) {
            C = p.fanout[0];
            for (int c = threadIdx.x; c < C; c += blockDim.x) {
                sm.cand_id[c] = c;
                sm.cand_row[c] = (int32_t)(hkv * p.rows[0] + c);
            }
        } else {
            const int fo = p.fanout[L];
            const int Kp = p.K[L - 1];
            C = Kp * fo;
            const long long prow = p.rows[L - 1];
            const int32_t *tab = p.child[L - 1];
            for (int c = threadIdx.x; c < C; c += blockDim.x) {
                const int k = c / fo, j = c - k * fo;
                const long long par = sm.kept_id[k];
                long long id = tab ? (long long)tab[((size_t)hkv * prow + par) * fo + j] : par * fo + j;
                if (id < 0 || id >= p.rows[L]) {
                    set_status(p.status, kDevBadChild);
                    id = 0;
                }
                sm.cand_id[c] = (int32_t)id;
                long long row;
                if (L == 2 && p.leaf_slot)
                    row = (long long)p.leaf_slot[(size_t)bh * Kp + k] * fo + j;
                else
                    row = hkv * p.rows[L] + id;
                sm.cand_row[c] = (int32_t)row;
            }
        }
        __syncthreads();
        score_candidates<T, D>(kbase, sm.cand_row, C, sm.s, sm.cand_f);
        __syncthreads();
        const double E = cprime * anorm * (double)p.norm_bound[L * p.H_kv + hkv] * (1.0 + 1e-6) + D * 0x1p-148;
        select_level<T, D>(sm, C, p.K[L], E, qbase, q_stride, p.N, kbase, p.cap);
        const int K = p.K[L];
        if (p.kept[L])
            for (int i = threadIdx.x; i < K; i += blockDim.x) p.kept[L][(size_t)bh * K + i] = sm.kept_id[i];
        if (L == 2 && p.kept_leaf_row)
            for (int i = threadIdx.x; i < K; i += blockDim.x)
                p.kept_leaf_row[(size_t)bh * K + i] = sm.cand_row[sm.kept_pos[i]];
        __syncthreads();
    }
}

// Per-level, per-KV-head maximum of key row 2-norms (for the filter bound),
// as float bits rounded up; grid.y = KV head, one warp per row.  atomicMax on
// the bit pattern is a max on non-negative floats.
template <typename T, int D>
__global__ void key_norm_kernel(const T *__restrict__ keys, long long rows_per_head, unsigned int *out_bits)
{
    const int lane = threadIdx.x & 31;
    const int hk = blockIdx.y;
    const long long nw = (long long)gridDim.x * (blockDim.x >> 5);
    const T *head = keys + (size_t)hk * rows_per_head * D;
    double best = 0.0;
    for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows_per_head; r += nw) {
        const T *row = head + (size_t)r * D;
        double acc = 0.0;
        for (int d = lane; d < D; d += 32) {
            const double x = (double)elem_f32(row[d]);
            acc = fma(x, x, acc);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        best = fmax(best, acc);
    }
    if (lane == 0 && best > 0.0) {
        const float nf = __double2float_ru(sqrt(best) * (1.0 + 1e-12));
        atomicMax(out_bits + hk, __float_as_uint(nf));
    }
}

// Child tables: every entry in range and every id hit exactly once per head.
__global__ void child_table_check_kernel(const int32_t *__restrict__ tab, long long entries_per_head, int H_kv,
                                         long long child_rows, unsigned int *hits, int *status)
{
    const long long total = entries_per_head * H_kv;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long hk = i / entries_per_head;
        const int32_t c = tab[i];
        if (c < 0 || c >= child_rows) {
            set_status(status, kDevBadChild);
            continue;
        }
        atomicAdd(hits + (size_t)hk * child_rows + c, 1u);
    }
}

__global__ void hits_check_kernel(const unsigned int *__restrict__ hits, long long n, int *status)
{
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        if (hits[i] != 1u) set_status(status, kDevBadChild);
}

}  // namespace akv
