// Level-by-level HiKVP descent.
//
// "AtlasKV: Augmenting LLMs with Billion-Scale Knowledge Graphs in 20GB VRAM",
// section "Quick read / How it works": score the query against the resident
// root keys, keep the top-K branches, bring in the children's keys, prune level
// by level down to the leaves.  Node score (reading of that section): mean over
// the query tokens of <q_n, k>/sqrt(D); ranking by x(k) = sum_d s[d] k[d] with
// s[d] = sum_n q[n][d] is equivalent.
//
// The descent runs level-synchronously over all traversals (query b, head h):
//   root_kernel    token sums s of GP heads per CTA, fp32 scores of all roots
//   select_kernel  one CTA (64 or 128 threads) per traversal: top-K of its
//                  candidates' fp32 scores, with a rigorous error band
//   exact_kernel   one warp per queued traversal: the band's candidates in
//                  fp64, then in exact arithmetic
//   score_kernel   one CTA per (query, KV head, chunk of GC <= 32 heads, chunk
//                  of the union of their kept parents): every child row is
//                  loaded once and scored against the GC token-sum vectors
// Scores live in a per-traversal buffer (workspace, L2-resident at the
// benchmark sizes); each phase is a wide, short kernel.
//
// Ranking is exact.  Each candidate gets an fp32 score f (token sums and dot
// products in fp32) with the rigorous bound |f - x| <= E, where
//   E = (g_D (1 + g_N) + g_N) * ||a||_2 * max_k ||k||_2 + D 2^-148,
//   g_n = n u / (1 - n u), u = 2^-24, a[d] = sum_n |q[n][d]|
// (Higham's dot-product and summation bounds, for any evaluation order, plus
// Cauchy-Schwarz; the last term covers underflow).  With t the K-th largest f,
// every candidate with f > t + 2E is certainly kept, every one with
// f < t - 2E certainly dropped; the rest (always containing t's candidate) are
// ranked by their exact score and then by lower row id.
#pragma once

#include <float.h>

#include "common.cuh"
#include "exact.cuh"

namespace akv {

constexpr int kScoreThreads = 256;
constexpr int kSelectWarps = 4;
constexpr int kRefineChunk = 16;   // exact scores per refinement chunk (a pool of two chunks fills a warp)

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
    float *s_ws;                 // [B H][D] fp32 token sums (rounded from s64)
    double *s64_ws;              // [B H][D] fp64 token sums
    double *a64_ws;              // [B H][D] fp64 sums of |q| over the tokens
    float *anorm_ws;             // [B H] upper bound of ||a||_2
    float *f_ws;                 // [B H][fstride] fp32 filter scores of the current level; for a traversal
                                 // left to the exact pass: its candidate list, then its decided entries
    int fstride;                 // floats per traversal in f_ws: cap + 2 kcap
    int cap;                     // per-traversal score capacity (>= every level's candidate count)
    int kcap;                    // kept capacity (power of two >= every K)
    int *queue;                  // [3][B H][4] (traversal, decided, listed, non-finite) left to the exact pass
    int *qcount;                 // [3] queue lengths (zeroed by the root kernel)
    // host-staged leaves: kept mid k of traversal bh has its leaf block at pool
    // slot leaf_slot[bh K_mid + k]; leaf candidate (k, j) is pool row slot * b_L + j.
    const int32_t *leaf_slot;
    int32_t *kept_leaf_row;      // [B H][K_leaf] pool row of each kept leaf (host path)
    unsigned long long *stats;   // [3][4] optional counters: selections, refined, ambiguous, exact scores
    int *status;
};

__device__ __forceinline__ double gamma_n(int n)
{
    const double nu = (double)n * 0x1p-24;
    return nu / (1.0 - nu);
}

__device__ __forceinline__ unsigned lanemask_lt() { return (1u << (threadIdx.x & 31)) - 1u; }

// ==========================================================================
// Scoring side (CTA-level)
// ==========================================================================

// Token sums of GP consecutive heads (a1), in float64: s64[g][d] =
// sum_n q[n][h0+g][d] and a64[g][d] = sum_n |q[n][h0+g][d]| (relative error
// below g_N in binary64).  The fp32 filter uses s = fl32(s64), whose error
// |s - sum_n q| <= (u32 + g64_N) a is well inside the g32_N a of the bound.
// Every thread issues 16-byte loads; partial sums over token slices meet in
// `part` ([SLICES][COMBOS][2][EV] doubles).
template <typename T, int D, int GP>
__device__ void token_sums(const T *qb, size_t q_stride, int N, float *s, double *s64, double *a64, double *part,
                           double *anorm)
{
    constexpr int EV = Vec16<T>::E;
    constexpr int VPH = D / EV;
    constexpr int COMBOS = GP * VPH;
    static_assert(kScoreThreads % COMBOS == 0, "columns must divide the block");
    constexpr int SLICES = kScoreThreads / COMBOS;
    const int combo = threadIdx.x % COMBOS, slice = threadIdx.x / COMBOS;
    const int g = combo / VPH, v = combo % VPH;
    double ps[EV], pa[EV];
#pragma unroll
    for (int e = 0; e < EV; ++e) ps[e] = pa[e] = 0.0;
    const T *col = qb + (size_t)g * D + v * EV;
    int n = slice;
    for (; n + 3 * SLICES < N; n += 4 * SLICES) {
        uint4 w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) w[u] = ldg16(col + (size_t)(n + u * SLICES) * q_stride);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float x[EV];
            Vec16<T>::unpack(w[u], x);
#pragma unroll
            for (int e = 0; e < EV; ++e) {
                ps[e] += (double)x[e];
                pa[e] += fabs((double)x[e]);
            }
        }
    }
    for (; n < N; n += SLICES) {
        float x[EV];
        Vec16<T>::unpack(ldg16(col + (size_t)n * q_stride), x);
#pragma unroll
        for (int e = 0; e < EV; ++e) {
            ps[e] += (double)x[e];
            pa[e] += fabs((double)x[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < EV; ++e) {
        part[((slice * COMBOS + combo) * 2 + 0) * EV + e] = ps[e];
        part[((slice * COMBOS + combo) * 2 + 1) * EV + e] = pa[e];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < GP * D; i += blockDim.x) {
        const int cb = i / EV, e = i % EV;   // i = (g * VPH + v) * EV + e
        double ss = 0.0, aa = 0.0;
        for (int sl = 0; sl < SLICES; ++sl) {
            ss += part[((sl * COMBOS + cb) * 2 + 0) * EV + e];
            aa += part[((sl * COMBOS + cb) * 2 + 1) * EV + e];
        }
        s64[i] = ss;
        a64[i] = aa;
        s[i] = (float)ss;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int gg = warp; gg < GP; gg += blockDim.x >> 5) {
        double acc = 0.0;
        for (int d = lane; d < D; d += 32) acc = fma(a64[gg * D + d], a64[gg * D + d], acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) anorm[gg] = sqrt(acc) * (1.0 + 1e-9);   // covers the binary64 rounding of a64
    }
    __syncthreads();
}

template <typename T, int D, int GP>
__host__ __device__ constexpr size_t root_kernel_smem()
{
    return (size_t)kScoreThreads * 2 * Vec16<T>::E * 8 + (size_t)2 * GP * D * 8;
}

// Score `nrows` rows against the GP token-sum vectors s (shared).  Eight lanes
// per row, each holding its slice of every s in registers; rows are fetched
// with 16-byte coalesced loads, four rows per lane group in flight.
// row_of(r) gives the row index (in units of D elements) of row r;
// store(g, r, value) stores head g's score of row r.
template <typename T, int D, int GP, typename RowFn, typename StoreFn>
__device__ void score_rows(const T *__restrict__ kbase, const float *s, int nrows, RowFn row_of, StoreFn store)
{
    constexpr int EV = Vec16<T>::E;
    constexpr int VPR = D / EV;
    constexpr int LPG = 8;
    constexpr int VPL = VPR / LPG;
    constexpr int U = 4;
    static_assert(VPL >= 1 && VPR % LPG == 0, "row must split over 8 lanes");
    static_assert(GP <= LPG, "one storing lane per head");
    const int sub = threadIdx.x & 7;
    const int grp = threadIdx.x >> 3;
    const int ngrp = blockDim.x >> 3;
    float sreg[GP][VPL * EV];
#pragma unroll
    for (int g = 0; g < GP; ++g)
#pragma unroll
        for (int v = 0; v < VPL; ++v)
#pragma unroll
            for (int e = 0; e < EV; ++e) sreg[g][v * EV + e] = s[g * D + (sub + LPG * v) * EV + e];

    for (int base_r = 0; base_r < nrows; base_r += ngrp * U) {
        uint4 buf[U][VPL];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int r = base_r + u * ngrp + grp;
            const T *rp = kbase + (size_t)(r < nrows ? row_of(r) : 0) * D;
#pragma unroll
            for (int v = 0; v < VPL; ++v)
                buf[u][v] = r < nrows ? ldg16(rp + (sub + LPG * v) * EV) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float acc[GP];
#pragma unroll
            for (int g = 0; g < GP; ++g) acc[g] = 0.f;
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                float x[EV];
                Vec16<T>::unpack(buf[u][v], x);
#pragma unroll
                for (int e = 0; e < EV; ++e)
#pragma unroll
                    for (int g = 0; g < GP; ++g) acc[g] = fmaf(sreg[g][v * EV + e], x[e], acc[g]);
            }
#pragma unroll
            for (int g = 0; g < GP; ++g) {
                acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], 4);
                acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], 2);
                acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], 1);
            }
            float val = acc[0];
#pragma unroll
            for (int g = 1; g < GP; ++g)
                if (g == sub) val = acc[g];
            const int r = base_r + u * ngrp + grp;
            if (sub < GP && r < nrows) store(sub, r, val);
        }
    }
}

// Root level (a1 + a2 scores): one CTA per GP heads of a (query, KV head).
template <typename T, int D, int GP>
__global__ void __launch_bounds__(kScoreThreads) root_kernel(const DescendParams p)
{
    constexpr int EV = Vec16<T>::E;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    double *part = reinterpret_cast<double *>(smem_raw);            // [256 * 2 * EV]
    double *s64 = part + kScoreThreads * 2 * EV;                     // [GP * D]
    double *a64 = s64 + GP * D;                                       // [GP * D]
    __shared__ float s[GP * D];
    __shared__ double anorm[GP];
    if (blockIdx.x == 0 && threadIdx.x < 3) p.qcount[threadIdx.x] = 0;
    const int chunks = p.G / GP;
    const int cid = blockIdx.x % chunks;
    const int grp_id = blockIdx.x / chunks;   // b * H_kv + hkv
    const int b = grp_id / p.H_kv, hkv = grp_id % p.H_kv;
    const int h0 = hkv * p.G + cid * GP;
    const long long bh0 = (long long)b * p.H + h0;
    const T *qb = reinterpret_cast<const T *>(p.q_kg) + ((size_t)b * p.N * p.H + h0) * D;
    token_sums<T, D, GP>(qb, (size_t)p.H * D, p.N, s, s64, a64, part, anorm);
    for (int i = threadIdx.x; i < GP * D; i += blockDim.x) {
        p.s_ws[(size_t)bh0 * D + i] = s[i];
        p.s64_ws[(size_t)bh0 * D + i] = s64[i];
        p.a64_ws[(size_t)bh0 * D + i] = a64[i];
    }
    if (threadIdx.x < GP) p.anorm_ws[bh0 + threadIdx.x] = (float)anorm[threadIdx.x] * (1.0f + 1e-6f);
    const T *kbase = reinterpret_cast<const T *>(p.keys[0]);
    const long long base_row = (long long)hkv * p.rows[0];
    float *f = p.f_ws;
    const int fstride = p.fstride;
    score_rows<T, D, GP>(
        kbase, s, p.fanout[0], [&](int r) -> long long { return base_row + r; },
        [&](int g, int r, float v) { f[(size_t)(bh0 + g) * fstride + r] = v; });
    (void)EV;
}

// --------------------------------------------------------------------------
// Children of the kept parents (levels 1 and 2).
//
// Grid: (query b, KV head, head chunk of GC <= 32 heads, parent chunk).  The
// CTA forms the union of its GC heads' kept parent lists (a shared-memory hash
// set: O(GC Kp) work) and scores every child row of the union parents
// [pc ppc, (pc + 1) ppc), [(pc + pchunks) ppc, ...) against all GC token-sum
// vectors, so each row crosses from L2/HBM once per head group.
//
// Rows reach the CTA in tiles of kScoreTile rows, copied by cp.async (LPG
// consecutive threads per row, kScoreStages - 1 tiles in flight ahead of the
// one being scored) into shared memory.  Each tile's row table (key row,
// union parent, child index) is built one tile ahead, one thread per row, so
// the copy and store loops do no index arithmetic.  For the dot products a
// row is split over LPG = D / EV lanes, one 16-byte vector each, so a warp's
// shared-memory read covers 32 / LPG whole rows without bank conflicts.  A
// warp serves HT heads and keeps their token-sum slices in registers; a lane
// group takes R = LPG / HT rows at a time, forms R x HT partial dot products
// per lane and reduces them over the group by recursive halving, after which
// lane `sub` of the group holds the full score of value index
// sub = (row k, head h) = (sub / HT, sub % HT).  Head g's score of child j of
// union parent P[i] lands at its own candidate slot kidx[g][i] fo + j.  The
// fp32 sum of D products, in whatever order, stays within the g_D bound of
// the filter.
constexpr int kScoreTile = 64;
constexpr int kScoreStages = 4;

__host__ __device__ constexpr int score_hash_size(int total)
{
    int hs = 64;
    while (hs < 2 * total) hs <<= 1;
    return hs;
}

struct ScoreRow {
    long long row;   // key row (units of D elements), -1: none
    int i, j;        // union parent, child index
};

// Region A holds the row tiles; before the first tile it holds the union's
// hash set (keys, inserting entry, union index: 3 hs ints) and each entry's
// slot (total ints).  Then the row tables, lists / P / owner (3 total ints)
// and kidx ([GC][total] int16).
template <int D, int E>
__host__ __device__ constexpr size_t score_region_a(int GC, int Kp)
{
    return (size_t)kScoreStages * kScoreTile * D * E > (size_t)(3 * score_hash_size(GC * Kp) + GC * Kp) * 4
               ? (size_t)kScoreStages * kScoreTile * D * E
               : ((size_t)(3 * score_hash_size(GC * Kp) + GC * Kp) * 4 + 15) / 16 * 16;
}

template <int D, int E>
__host__ __device__ constexpr size_t score_kernel_smem(int GC, int Kp)
{
    return score_region_a<D, E>(GC, Kp) + (size_t)(kScoreStages + 1) * kScoreTile * sizeof(ScoreRow) +
           (size_t)3 * GC * Kp * 4 + (size_t)GC * GC * Kp * 2 + 16;
}

template <typename T, int D, int HT>
__global__ void __launch_bounds__(kScoreThreads, 2) score_kernel(const DescendParams p, int L, int GC, int ppc,
                                                                  int pchunks)
{
    constexpr int EV = Vec16<T>::E;          // elements per 16-byte vector
    constexpr int LPG = D / EV;              // lanes per row = 16-byte vectors per row
    constexpr int GPW = 32 / LPG;            // rows per warp read
    constexpr int R = LPG / HT;              // rows per lane group per reduction
    static_assert(LPG >= 8 && LPG <= 32 && R >= 1 && R * HT == LPG, "one score per lane");
    constexpr int NW = kScoreThreads / 32;
    constexpr int ROWB = D * (int)sizeof(T);
    constexpr int TILEB = kScoreTile * ROWB;
    constexpr int NINFO = kScoreStages + 1;
    constexpr int CPR = kScoreThreads / LPG;               // rows one copy round of the CTA covers
    static_assert(kScoreTile % CPR == 0 && kScoreTile <= kScoreThreads, "tile shape");

    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int Kp = p.K[L - 1];
    const int fo = p.fanout[L];
    const int total = GC * Kp;
    const int hs = score_hash_size(total);
    uint8_t *tiles = smem_raw;                                // [stages][rows][D]
    int32_t *hkey = reinterpret_cast<int32_t *>(smem_raw);    // setup only: [hs] parent id or -1
    int32_t *hown = hkey + hs;                                // [hs] inserting entry
    int32_t *huid = hown + hs;                                // [hs] union index of the slot
    int32_t *eslot = huid + hs;                               // [total] hash slot of entry t
    ScoreRow *info = reinterpret_cast<ScoreRow *>(smem_raw + score_region_a<D, sizeof(T)>(GC, Kp));
    int32_t *lists = reinterpret_cast<int32_t *>(info + NINFO * kScoreTile);   // [GC][Kp] ascending
    int32_t *P = lists + total;                               // union parents
    int32_t *Pown = P + total;                                // an entry (g Kp + k) listing P[i]
    int16_t *kidx = reinterpret_cast<int16_t *>(Pown + total);   // [GC][total] slot of union parent i in g's list
    __shared__ int seg[kScoreThreads];
    __shared__ int nP_sh;

    const int pc = blockIdx.x % pchunks;
    const int rest = blockIdx.x / pchunks;
    const int hchunks = p.G / GC;
    const int hc = rest % hchunks;
    const int grp_id = rest / hchunks;
    const int b = grp_id / p.H_kv, hkv = grp_id % p.H_kv;
    const long long bh0 = (long long)b * p.H + (long long)hkv * p.G + (long long)hc * GC;

    for (int i = threadIdx.x; i < hs; i += blockDim.x) hkey[i] = -1;
    for (int i = threadIdx.x; i < GC * total; i += blockDim.x) kidx[i] = -1;
    for (int t = threadIdx.x; t < total; t += blockDim.x) {
        const int g = t / Kp, k = t - g * Kp;
        lists[t] = p.kept[L - 1][(bh0 + g) * Kp + k];
    }
    __syncthreads();
    // ---- union of the GC heads' kept parents: insert into the hash set ----
    for (int t = threadIdx.x; t < total; t += blockDim.x) {
        const int x = lists[t];
        unsigned h = ((unsigned)x * 2654435761u) & (unsigned)(hs - 1);
        for (int probe = 0; probe < hs; ++probe) {
            const int prev = atomicCAS(&hkey[h], -1, x);
            if (prev == -1) hown[h] = t;
            if (prev == -1 || prev == x) break;
            h = (h + 1) & (unsigned)(hs - 1);
        }
        eslot[t] = (int)h;
    }
    __syncthreads();
    // ---- number the occupied slots (table order): union index, P ----
    {
        const int per = (hs + (int)blockDim.x - 1) / (int)blockDim.x;
        const int t0 = min(hs, (int)threadIdx.x * per), t1 = min(hs, t0 + per);
        int cnt = 0;
        for (int t = t0; t < t1; ++t) cnt += (hkey[t] >= 0);
        seg[threadIdx.x] = cnt;
        __syncthreads();
        if (threadIdx.x < 32) {
            int run = 0;
            for (int base = 0; base < (int)blockDim.x; base += 32) {
                const int v = seg[base + threadIdx.x];
                int incl = v;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int w = __shfl_up_sync(0xffffffffu, incl, o);
                    if ((int)threadIdx.x >= o) incl += w;
                }
                seg[base + threadIdx.x] = run + incl - v;
                run += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (threadIdx.x == 0) nP_sh = run;
        }
        __syncthreads();
        int run = seg[threadIdx.x];
        for (int t = t0; t < t1; ++t)
            if (hkey[t] >= 0) {
                P[run] = hkey[t];
                Pown[run] = hown[t];
                huid[t] = run;
                ++run;
            }
    }
    __syncthreads();
    for (int t = threadIdx.x; t < total; t += blockDim.x) {
        const int g = t / Kp, k = t - g * Kp;
        kidx[g * total + huid[eslot[t]]] = (int16_t)k;
    }
    const int nP = nP_sh;
    if (pc * ppc >= nP) return;
    const int nchunks_mine = (nP - pc * ppc + pchunks * ppc - 1) / (pchunks * ppc);
    const int full_rows = ppc * fo;
    const int last_i0 = (pc + (nchunks_mine - 1) * pchunks) * ppc;
    const int nR = (nchunks_mine - 1) * full_rows + min(ppc, nP - last_i0) * fo;
    const int ntiles = (nR + kScoreTile - 1) / kScoreTile;

    const T *kbase = reinterpret_cast<const T *>(p.keys[L]);
    const int32_t *tab = p.child[L - 1];
    const long long prow = p.rows[L - 1], rows = p.rows[L];
    const int32_t *slot = (L == 2) ? p.leaf_slot : nullptr;
    float *f = p.f_ws;
    const int fstride = p.fstride;

    // row table of tile tl (threads 0 .. kScoreTile-1, one row each)
    auto build_info = [&](int tl) {
        if (threadIdx.x >= kScoreTile) return;
        ScoreRow sr;
        const int rho = tl * kScoreTile + (int)threadIdx.x;
        sr.row = -1;
        sr.i = 0;
        sr.j = 0;
        if (rho < nR) {
            const int cc = rho / full_rows, r = rho - cc * full_rows;
            const int i = (pc + cc * pchunks) * ppc + r / fo;
            const int j = r - (r / fo) * fo;
            long long row;
            if (slot) {
                const int own = Pown[i];
                row = (long long)slot[(bh0 + own / Kp) * Kp + own % Kp] * fo + j;
            } else {
                const long long par = P[i];
                long long id = tab ? (long long)tab[((size_t)hkv * prow + par) * fo + j] : par * fo + j;
                if (id < 0 || id >= rows) {
                    set_status(p.status, kDevBadChild);
                    id = 0;
                }
                row = (long long)hkv * rows + id;
            }
            sr.row = row;
            sr.i = i;
            sr.j = j;
        }
        info[(tl % NINFO) * kScoreTile + threadIdx.x] = sr;
    };
    // copy tile tl into stage tl % S: thread (row lr, vector lc), rows lr + CPR i
    const int lc = threadIdx.x % LPG, lr = threadIdx.x / LPG;
    auto load_tile = [&](int tl) {
        const ScoreRow *ti = info + (tl % NINFO) * kScoreTile;
        const uint32_t dst = (uint32_t)__cvta_generic_to_shared(tiles + (tl % kScoreStages) * TILEB) + lc * 16;
#pragma unroll
        for (int i = 0; i < kScoreTile / CPR; ++i) {
            const int r = lr + CPR * i;
            const long long row = ti[r].row;
            const T *src = row >= 0 ? kbase + (size_t)row * D + lc * EV : kbase;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst + r * ROWB), "l"(src),
                         "r"(row >= 0 ? 16 : 0));
        }
        asm volatile("cp.async.commit_group;\n" ::);
    };

    // warp -> (head group, row stream); lane -> (row group, vector of the row)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hgn = (GC + HT - 1) / HT;
    const int streams = NW / hgn;
    const bool computes = warp < streams * hgn;
    const int hg = warp % hgn, rs = warp / hgn;
    const int lg = lane / LPG, sub = lane % LPG;
    float sreg[HT][EV];
#pragma unroll
    for (int h = 0; h < HT; ++h) {
        const int g = hg * HT + h;
        const float *sp = p.s_ws + (size_t)(bh0 + (g < GC ? g : 0)) * D + sub * EV;
#pragma unroll
        for (int e = 0; e < EV; e += 4) {
            const float4 t4 = *reinterpret_cast<const float4 *>(sp + e);
            sreg[h][e] = g < GC ? t4.x : 0.f;
            sreg[h][e + 1] = g < GC ? t4.y : 0.f;
            sreg[h][e + 2] = g < GC ? t4.z : 0.f;
            sreg[h][e + 3] = g < GC ? t4.w : 0.f;
        }
    }
    const int k_mine = sub / HT, g_mine = hg * HT + (sub - (sub / HT) * HT);
    const bool stores = g_mine < GC;
    const int16_t *kid_mine = kidx + (stores ? g_mine : 0) * total;
    float *f_mine = f + (size_t)(bh0 + (stores ? g_mine : 0)) * fstride;

    for (int tl = 0; tl < kScoreStages; ++tl)
        if (tl < ntiles) build_info(tl);
    __syncthreads();   // kidx and the first row tables are complete
#pragma unroll
    for (int st = 0; st < kScoreStages - 1; ++st) {
        if (st < ntiles) load_tile(st);
        else asm volatile("cp.async.commit_group;\n" ::);
    }
    for (int tl = 0; tl < ntiles; ++tl) {
        asm volatile("cp.async.wait_group %0;\n" ::"n"(kScoreStages - 2));
        __syncthreads();   // tile tl landed for every warp; tile tl-1's stage and row table are free
        const int nx = tl + kScoreStages - 1;
        if (nx < ntiles) load_tile(nx);
        else asm volatile("cp.async.commit_group;\n" ::);
        if (nx + 1 < ntiles) build_info(nx + 1);
        if (!computes) continue;
        const uint8_t *tb = tiles + (tl % kScoreStages) * TILEB;
        const ScoreRow *ti = info + (tl % NINFO) * kScoreTile;
        const int tile_rows = min(kScoreTile, nR - tl * kScoreTile);
        for (int r0 = (rs * GPW + lg) * R; r0 < tile_rows; r0 += streams * GPW * R) {
            float v[LPG];
#pragma unroll
            for (int k = 0; k < R; ++k) {
                float xf[EV];
                Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(tb + (r0 + k) * ROWB + sub * 16), xf);
#pragma unroll
                for (int h = 0; h < HT; ++h) {
                    float acc = 0.f;
#pragma unroll
                    for (int e = 0; e < EV; ++e) acc = fmaf(sreg[h][e], xf[e], acc);
                    v[k * HT + h] = acc;
                }
            }
            // recursive halving over the LPG lanes of the group
#pragma unroll
            for (int m = LPG / 2; m >= 1; m >>= 1) {
                const bool upper = (sub & m) != 0;
#pragma unroll
                for (int q = 0; q < m; ++q) {
                    const float send = upper ? v[q] : v[q + m];
                    const float keep = upper ? v[q + m] : v[q];
                    v[q] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                }
            }
            const int rr = r0 + k_mine;
            if (stores && rr < tile_rows) {
                const ScoreRow sr = ti[rr];
                const int kk = kid_mine[sr.i];
                if (kk >= 0) f_mine[(size_t)kk * fo + sr.j] = v[0];
            }
        }
    }
    asm volatile("cp.async.wait_group 0;\n" ::);
}

// ==========================================================================
// Selection side (warp-level)
// ==========================================================================

// Ascending warp bitonic sort of n (power of two) uint64 in shared memory.
__device__ void warp_sort_u64(uint64_t *a, int n)
{
    const int lane = threadIdx.x & 31;
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncwarp();
            for (int i = lane; i < n / 2; i += 32) {
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
    __syncwarp();
}

// One traversal's candidates at one level: candidate c = (k, j) is child j of
// its k-th kept parent; at the root level c is the root itself.
struct LevelView {
    int L, C, fo;
    const int32_t *prev;      // kept parents (ascending ids), null at the root level
    const int32_t *tab;       // child table of the parent level, or null
    long long prow, rows;     // rows per KV head of the parent level / this level
    int hkv;
    const int32_t *slot;      // host pool slots of the kept parents (leaf level, host path), or null

    __device__ __forceinline__ int id(int c) const
    {
        if (L == 0) return c;
        const int k = c / fo, j = c - k * fo;
        const long long par = prev[k];
        long long v = tab ? (long long)tab[((size_t)hkv * prow + par) * fo + j] : par * fo + j;
        return (v < 0 || v >= rows) ? 0 : (int)v;
    }
    __device__ __forceinline__ long long row(int c) const
    {
        if (L == 0) return (long long)hkv * rows + c;
        if (slot) {
            const int k = c / fo, j = c - k * fo;
            return (long long)slot[k] * fo + j;
        }
        return (long long)hkv * rows + id(c);
    }
};

template <typename T>
__device__ LevelView level_view(const DescendParams &p, int L, long long bh, const int32_t *prev)
{
    const int h = (int)(bh % p.H);
    const int Kp = L == 0 ? 0 : p.K[L - 1];
    LevelView lv;
    lv.L = L;
    lv.fo = L == 0 ? 1 : p.fanout[L];
    lv.C = L == 0 ? p.fanout[0] : Kp * lv.fo;
    lv.tab = L == 0 ? nullptr : p.child[L - 1];
    lv.prow = L == 0 ? 0 : p.rows[L - 1];
    lv.rows = p.rows[L];
    lv.hkv = h / p.G;
    lv.slot = (L == 2 && p.leaf_slot) ? p.leaf_slot + bh * Kp : nullptr;
    lv.prev = prev;
    return lv;
}

// Shared scratch of one traversal's selection.
struct SelectScratch {
    float *f;          // [cap] scores
    int32_t *prev;     // [kcap] kept parents of the traversal
    uint32_t *hist;    // [256]
    uint64_t *sortb;   // [kcap] (id << 32 | position)
    uint64_t *tmp;     // [64]

    __host__ __device__ static size_t bytes(int cap, int kcap, int D)
    {
        (void)D;
        auto r = [](size_t b) { return (b + 15) & ~size_t(15); };
        return r((size_t)cap * 4) + r((size_t)kcap * 4) + r(1024) + r((size_t)kcap * 8) + r(512);
    }
    __device__ SelectScratch(uint8_t *p, int cap, int kcap, int D)
    {
        (void)D;
        auto take = [&](size_t b) {
            uint8_t *q = p;
            p += (b + 15) & ~size_t(15);
            return q;
        };
        f = (float *)take((size_t)cap * 4);
        prev = (int32_t *)take((size_t)kcap * 4);
        hist = (uint32_t *)take(1024);
        sortb = (uint64_t *)take((size_t)kcap * 8);
        tmp = (uint64_t *)take(512);
    }
};

// Write the final kept list of a traversal from sortb[0..K) (ascending after sorting).
__device__ void write_kept(const DescendParams &p, const LevelView &lv, int L, long long bh, uint64_t *sortb, int K)
{
    const int lane = threadIdx.x & 31;
    int n2 = 1;
    while (n2 < K) n2 <<= 1;
    for (int i = K + lane; i < n2; i += 32) sortb[i] = ~0ull;
    warp_sort_u64(sortb, n2);
    for (int i = lane; i < K; i += 32) p.kept[L][bh * K + i] = (int32_t)(sortb[i] >> 32);
    if (L == 2 && p.kept_leaf_row)
        for (int i = lane; i < K; i += 32)
            p.kept_leaf_row[bh * K + i] = (int32_t)lv.row((int)(sortb[i] & 0xffffffffu));
}

// Warp exclusive prefix sum.
__device__ __forceinline__ int warp_excl_scan(int v, int &total)
{
    const int lane = threadIdx.x & 31;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int w = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += w;
    }
    total = __shfl_sync(0xffffffffu, incl, 31);
    return incl - v;
}

// CTA-wide exclusive scan of one int per thread (NT threads): this thread's
// exclusive prefix; the total in `total`.  red: NT / 32 ints.
template <int NT>
__device__ __forceinline__ int cta_excl_scan(int v, int &total, int *red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int wt;
    const int ex = warp_excl_scan(v, wt);
    if (lane == 0) red[warp] = wt;
    __syncthreads();
    int base = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        const int x = red[w];
        base += w < warp ? x : 0;
        tot += x;
    }
    __syncthreads();
    total = tot;
    return base + ex;
}

// k-th largest (1-based) of the n floats f[0..n), by all NT threads of the CTA,
// given their min mn and max mx.  Values are bucketed linearly between min and
// max (a monotone map); the bucket holding the k-th largest is then searched
// exactly: sorted when it holds at most 64, else narrowed by MSB-first radix
// passes over the order-preserving bit image.  hist: 256 bins; tmp: 64 scratch
// uint64; sh: 8 ints of shared scratch.
template <int NT>
__device__ float cta_kth_largest(const float *f, int n, int k, float mn, float mx, uint32_t *hist, uint64_t *tmp,
                                 int *sh)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (mx == mn) return mx;   // all equal
    // warp 0: find the bin holding the k-th largest from the 256 counts
    auto pick = [&](int kk, int &bin, int &rem, int &bcount) {
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
        bin = rem = bcount = 0;
        const bool mine = excl < (uint32_t)kk && (uint32_t)kk <= incl;
        if (mine) {
            uint32_t run = excl;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (run + cnt[j] >= (uint32_t)kk) {
                    bin = 255 - 8 * lane - j;
                    rem = kk - (int)run;
                    bcount = (int)cnt[j];
                    break;
                }
                run += cnt[j];
            }
        }
        const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
        bin = __shfl_sync(0xffffffffu, bin, src);
        rem = __shfl_sync(0xffffffffu, rem, src);
        bcount = __shfl_sync(0xffffffffu, bcount, src);
    };
    if (mx > mn && isfinite(mx - mn)) {
        const float scale = 255.99f / (mx - mn);
        auto bucket = [&](float v) { return min(255, max(0, (int)((v - mn) * scale))); };
        for (int j = tid; j < 256; j += NT) hist[j] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += NT) atomicAdd(&hist[bucket(f[i])], 1u);
        __syncthreads();
        if (warp == 0) {
            int bk, rem, bcount;
            pick(k, bk, rem, bcount);
            if (lane == 0) {
                sh[0] = bk;
                sh[1] = rem;
                sh[2] = bcount;
                sh[3] = 0;
            }
        }
        __syncthreads();
        const int bk = sh[0], rem = sh[1], bcount = sh[2];
        if (bcount <= 64) {
            // the bucket's members (order is irrelevant: they are sorted next)
            for (int i = tid; i < n; i += NT)
                if (bucket(f[i]) == bk) tmp[atomicAdd(&sh[3], 1)] = ~(uint64_t)float_key(f[i]);
            __syncthreads();
            if (warp == 0) {
                for (int i = sh[3] + lane; i < 64; i += 32) tmp[i] = ~0ull;
                warp_sort_u64(tmp, 64);
                if (lane == 0) sh[4] = (int)(uint32_t)~tmp[rem - 1];
            }
            __syncthreads();
            const float t = key_float((uint32_t)sh[4]);
            __syncthreads();
            return t;
        }
        __syncthreads();
    }
    // general case: radix select on the bit image
    uint32_t prefix = 0, mask = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int j = tid; j < 256; j += NT) hist[j] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += NT) {
            const uint32_t key = float_key(f[i]);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            int digit, rem, unused;
            pick(k, digit, rem, unused);
            if (lane == 0) {
                sh[0] = digit;
                sh[1] = rem;
            }
        }
        __syncthreads();
        prefix |= ((uint32_t)sh[0]) << shift;
        mask |= 255u << shift;
        k = sh[1];
        __syncthreads();
    }
    return key_float(prefix);
}

// One CTA per traversal: top-K of level L's candidates, tier 1.  The fp32
// scores and their rigorous bound E settle every candidate outside the band
// [t - 2E, t + 2E] around the K-th largest score t.  When the band holds more
// candidates than places left, the traversal is queued for exact_kernel with
// its decided entries and the band's positions.  Every pass over the
// candidates is spread over the CTA's NT threads (64 or 128: the host picks
// the smaller when few traversals fill the GPU anyway); the small sorts run on
// warp 0.
template <typename T, int D, int NT>
__global__ void __launch_bounds__(NT) select_kernel(const DescendParams p, int L)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ int sh[8];
    __shared__ int red[NT / 32];
    __shared__ float redf[2][NT / 32];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long bh = blockIdx.x;
    if (bh >= (long long)p.B * p.H) return;
    SelectScratch sc(smem_raw, p.cap, p.kcap, D);
    const int Kp = L == 0 ? 0 : p.K[L - 1];
    for (int k = tid; k < Kp; k += NT) sc.prev[k] = p.kept[L - 1][bh * Kp + k];
    const LevelView lv = level_view<T>(p, L, bh, sc.prev);
    const int C = lv.C, K = p.K[L];
    float *fslot = p.f_ws + (size_t)bh * p.fstride;
    const int nv = (C + 3) >> 2;
    float mn = INFINITY, mx = -INFINITY;
    int bad = 0;
    {
        // 16-byte loads, several in flight per thread; min / max / finiteness on the way
        const float4 *src = reinterpret_cast<const float4 *>(fslot);
        float4 *dst = reinterpret_cast<float4 *>(sc.f);
        auto take = [&](float4 t, int v) {
            dst[v] = t;
            const float e[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (4 * v + q < C) {
                    mn = fminf(mn, e[q]);
                    mx = fmaxf(mx, e[q]);
                    bad |= !isfinite(e[q]);
                }
        };
        int v = tid;
        for (; v + 3 * NT < nv; v += 4 * NT) {
            float4 t[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) t[u] = __ldcg(src + v + u * NT);
#pragma unroll
            for (int u = 0; u < 4; ++u) take(t[u], v + u * NT);
        }
        for (; v < nv; v += NT) take(__ldcg(src + v), v);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        bad = __any_sync(0xffffffffu, bad);
        if (lane == 0) {
            redf[0][warp] = mn;
            redf[1][warp] = mx;
            red[warp] = bad;
        }
        __syncthreads();   // scores, kept parents and the partial reductions are visible
#pragma unroll
        for (int w = 0; w < NT / 32; ++w) {
            mn = fminf(mn, redf[0][w]);
            mx = fmaxf(mx, redf[1][w]);
            bad |= red[w];
        }
        __syncthreads();
    }
    if (p.stats && tid == 0) atomicAdd(p.stats + L * 4, 1ull);
    const float *f = sc.f;
    uint64_t *sortb = sc.sortb;
    if (K >= C) {
        for (int c = tid; c < C; c += NT) sortb[c] = ((uint64_t)(uint32_t)lv.id(c) << 32) | (uint32_t)c;
        __syncthreads();
        if (warp == 0) write_kept(p, lv, L, bh, sortb, K);
        return;
    }
    const double cprime = gamma_n(D) * (1.0 + gamma_n(p.N)) + gamma_n(p.N);
    const double E = cprime * (double)p.anorm_ws[bh] * (double)p.norm_bound[L * p.H_kv + lv.hkv] * (1.0 + 1e-6) +
                     D * 0x1p-148;
    const double t = bad ? 0.0 : (double)cta_kth_largest<NT>(f, C, K, mn, mx, sc.hist, sc.tmp, sh);
    const bool bad2 = bad || !isfinite(E) || !isfinite(t);
    // band edges rounded outward to fp32: the sure-kept and sure-dropped sets can
    // only shrink, so the classification stays rigorous
    const float hi32 = bad2 ? INFINITY : __double2float_ru(__dadd_ru(t, 2.0 * E));
    const float lo32 = bad2 ? -INFINITY : __double2float_rd(__dsub_rd(t, 2.0 * E));
    // class of candidate c: 1 kept for sure, 2 ambiguous, 0 dropped
    auto cls = [&](float fv) -> int {
        if (bad2) return 2;
        return fv > hi32 ? 1 : (fv >= lo32 ? 2 : 0);
    };
    const float4 *f4 = reinterpret_cast<const float4 *>(f);
    int my_in = 0, my_a = 0;
    for (int v = tid; v < nv; v += NT) {
        const float4 x = f4[v];
        const float e[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int k = 4 * v + q < C ? cls(e[q]) : 0;
            my_in += k == 1;
            my_a += k == 2;
        }
    }
    int n_in, nA;
    int off_in = cta_excl_scan<NT>(my_in, n_in, red);
    int off_a = cta_excl_scan<NT>(my_a, nA, red);
    const int r = K - n_in;
    const bool settle = nA == r;   // every ambiguous candidate is kept
    int *list = reinterpret_cast<int *>(fslot);
    if (settle) off_a += n_in;
    for (int v = tid; v < nv; v += NT) {
        const float4 x = f4[v];
        const float e[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int c = 4 * v + q;
            const int k = c < C ? cls(e[q]) : 0;
            if (k == 1) sortb[off_in++] = ((uint64_t)(uint32_t)lv.id(c) << 32) | (uint32_t)c;
            else if (k == 2) {
                if (settle) sortb[off_a++] = ((uint64_t)(uint32_t)lv.id(c) << 32) | (uint32_t)c;
                else list[off_a++] = c;
            }
        }
    }
    __syncthreads();
    if (settle) {
        if (warp == 0) write_kept(p, lv, L, bh, sortb, K);
        return;
    }
    if (p.stats && tid == 0) {
        atomicAdd(p.stats + L * 4 + 1, 1ull);
        atomicAdd(p.stats + L * 4 + 2, (unsigned long long)nA);
    }
    uint64_t *decided = reinterpret_cast<uint64_t *>(fslot + p.cap);
    for (int i = tid; i < n_in; i += NT) decided[i] = sortb[i];
    if (tid == 0) {
        const int qi = atomicAdd(p.qcount + L, 1);
        int *e = p.queue + ((size_t)L * p.B * p.H + qi) * 4;
        e[0] = (int)bh;
        e[1] = n_in;
        e[2] = nA;
        e[3] = bad2 ? 1 : 0;
    }
}

// Exact score of one key row: x = sum_n sum_d q[n][d] k[d] over the stored
// numbers (binary32, or bfloat16 widened exactly: every value is m 2^e with an
// integer m < 2^24 and e >= -149), accumulated without rounding in digits of
// weight 2^(32 i - 298) (Kulisch's exact dot product), one warp, lanes over d.
// Lane 0 writes the canonical digits to out.
template <typename T, int D>
__device__ void warp_exact_score(const T *q, size_t q_stride, int N, const T *krow, uint32_t *out)
{
    const int lane = threadIdx.x & 31;
    int64_t acc[kScoreDigits];
#pragma unroll
    for (int i = 0; i < kScoreDigits; ++i) acc[i] = 0;
    for (int d = lane; d < D; d += 32) {
        uint32_t mk;
        int ek;
        const int sk = split_binary32(elem_bits(krow[d]), mk, ek);
        if (mk == 0) continue;
        for (int n = 0; n < N; ++n) {
            uint32_t mq;
            int eq;
            const int sq = split_binary32(elem_bits(q[(size_t)n * q_stride + d]), mq, eq);
            if (mq == 0) continue;
            const uint64_t prod = (uint64_t)mq * (uint64_t)mk;   // < 2^48
            const int pos = eq + ek + 298;                         // >= 0
            const int di = pos >> 5, sh = pos & 31;
            const uint64_t lo64 = prod << sh;
            const uint64_t hi64 = sh ? (prod >> (64 - sh)) : 0ull;
            const int64_t c0 = (int64_t)(lo64 & 0xffffffffull), c1 = (int64_t)(lo64 >> 32), c2 = (int64_t)hi64;
            const bool minus = (sq != 0) != (sk != 0);
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
    __syncwarp();
}

struct ExactScratch {
    int32_t *prev;     // [kcap]
    uint64_t *sortb;   // [kcap]
    uint32_t *ex;      // [3 RC][kScoreDigits]
    int32_t *ids;      // [3 RC]
    int32_t *poss;     // [3 RC]
    int32_t *list2;    // [32] positions still ambiguous after tier 2
    double *s64;       // [D]
    double *a64;       // [D]
    __host__ __device__ static size_t bytes(int kcap, int D)
    {
        auto r = [](size_t b) { return (b + 15) & ~size_t(15); };
        return r((size_t)kcap * 4) + r((size_t)kcap * 8) + r(3 * kRefineChunk * kScoreDigits * 4) +
               2 * r(3 * kRefineChunk * 4) + r(128) + 2 * r((size_t)D * 8);
    }
    __device__ ExactScratch(uint8_t *p, int kcap, int D)
    {
        auto take = [&](size_t b) {
            uint8_t *q = p;
            p += (b + 15) & ~size_t(15);
            return q;
        };
        prev = (int32_t *)take((size_t)kcap * 4);
        sortb = (uint64_t *)take((size_t)kcap * 8);
        ex = (uint32_t *)take(3 * kRefineChunk * kScoreDigits * 4);
        ids = (int32_t *)take(3 * kRefineChunk * 4);
        poss = (int32_t *)take(3 * kRefineChunk * 4);
        list2 = (int32_t *)take(128);
        s64 = (double *)take((size_t)D * 8);
        a64 = (double *)take((size_t)D * 8);
    }
};

// Traversals tier 1 left open.  For each, with `decided` entries already kept
// and r = K - decided places left among the listed band candidates:
//   tier 2: when at most 32 are listed (and all scores were finite), each lane
//           scores one of them in float64 from the float64 token sums, with its
//           own rigorous bound  (g64_D (1 + g64_N) + g64_N) sum_d a64_d |k_d|,
//           and the band argument is repeated among them;
//   tier 3: whatever is still open is ranked by exact score, then row id: the
//           candidates are scanned in chunks of RC with a bounded best-set, and
//           passes repeat (each excluding everything not strictly worse than
//           the last one chosen) until r are chosen.
template <typename T, int D>
__global__ void __launch_bounds__(kSelectWarps * 32) exact_kernel(const DescendParams p, int L)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    constexpr int RC = kRefineChunk;
    constexpr int EV = Vec16<T>::E;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qn = p.qcount[L];
    ExactScratch sc(smem_raw + (size_t)warp * ExactScratch::bytes(p.kcap, D), p.kcap, D);
    uint32_t *BEST = sc.ex, *CH = sc.ex + RC * kScoreDigits, *TMP = sc.ex + 2 * RC * kScoreDigits;
    int32_t *best_id = sc.ids, *ch_id = sc.ids + RC, *tmp_id = sc.ids + 2 * RC;
    int32_t *best_pos = sc.poss, *ch_pos = sc.poss + RC, *tmp_pos = sc.poss + 2 * RC;
    for (int qi = blockIdx.x * kSelectWarps + warp; qi < qn; qi += gridDim.x * kSelectWarps) {
        const int *e = p.queue + ((size_t)L * p.B * p.H + qi) * 4;
        const long long bh = e[0];
        int nsel = e[1];
        int nlist = e[2];
        const bool bad = e[3] != 0;
        const int K = p.K[L];
        int r = K - nsel;
        const int Kp = L == 0 ? 0 : p.K[L - 1];
        // every load that depends only on the queue entry goes out together:
        // kept parents, decided entries, the fp64 token sums for tier 2 and
        // this lane's listed candidate
        const bool tier2 = !bad && nlist <= 32;
        const float *fslot = p.f_ws + (size_t)bh * p.fstride;
        const int *list = reinterpret_cast<const int *>(fslot);
        const uint64_t *decided = reinterpret_cast<const uint64_t *>(fslot + p.cap);
        for (int k = lane; k < Kp; k += 32) sc.prev[k] = p.kept[L - 1][bh * Kp + k];
        for (int i = lane; i < nsel; i += 32) sc.sortb[i] = decided[i];
        if (tier2)
            for (int d = lane; d < D; d += 32) {
                sc.s64[d] = p.s64_ws[(size_t)bh * D + d];
                sc.a64[d] = p.a64_ws[(size_t)bh * D + d];
            }
        const int my_pos = tier2 && lane < nlist ? list[lane] : -1;
        __syncwarp();
        const LevelView lv = level_view<T>(p, L, bh, sc.prev);
        const int b = (int)(bh / p.H), h = (int)(bh % p.H);
        const T *qh = reinterpret_cast<const T *>(p.q_kg) + ((size_t)b * p.N * p.H + h) * D;
        const size_t q_stride = (size_t)p.H * D;
        const T *kbase = reinterpret_cast<const T *>(p.keys[L]);

        if (tier2) {
            // ---- tier 2 ----
            double y = -INFINITY, e2 = 0.0;
            if (my_pos >= 0) {
                const T *krow = kbase + (size_t)lv.row(my_pos) * D;
                uint4 w[D / EV];
#pragma unroll
                for (int v = 0; v < D / EV; ++v) w[v] = ldg16(krow + v * EV);
                double acc = 0.0, mag = 0.0;
#pragma unroll
                for (int v = 0; v < D / EV; ++v) {
                    float x[EV];
                    Vec16<T>::unpack(w[v], x);
#pragma unroll
                    for (int q = 0; q < EV; ++q) {
                        acc = fma(sc.s64[v * EV + q], (double)x[q], acc);
                        mag = fma(sc.a64[v * EV + q], fabs((double)x[q]), mag);
                    }
                }
                const double g64d = (double)D * 0x1p-53 / (1.0 - (double)D * 0x1p-53);
                const double g64n = (double)p.N * 0x1p-53 / (1.0 - (double)p.N * 0x1p-53);
                y = acc;
                e2 = (g64d * (1.0 + g64n) + g64n) * mag * (1.0 + 1e-6) + 0x1p-1000;
            }
            double E2 = e2;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) E2 = fmax(E2, __shfl_xor_sync(0xffffffffu, E2, o));
            int rank = 0;
            for (int j = 0; j < nlist; ++j) {
                const double yj = __shfl_sync(0xffffffffu, y, j);
                rank += (yj > y) || (yj == y && j < lane);
            }
            const int tl = __ffs(__ballot_sync(0xffffffffu, my_pos >= 0 && rank == r - 1)) - 1;
            const double t2 = __shfl_sync(0xffffffffu, y, tl);
            const double hi2 = __dadd_ru(t2, 2.0 * E2), lo2 = __dsub_rd(t2, 2.0 * E2);
            const bool in2 = my_pos >= 0 && y > hi2;
            const bool amb2 = my_pos >= 0 && !in2 && y >= lo2;
            const unsigned min2 = __ballot_sync(0xffffffffu, in2);
            const unsigned ma2 = __ballot_sync(0xffffffffu, amb2);
            const int n_in2 = __popc(min2), nA2 = __popc(ma2);
            const bool settle = nA2 == r - n_in2;
            if (in2 || (settle && amb2)) {
                const unsigned m = settle ? (min2 | ma2) : min2;
                sc.sortb[nsel + __popc(m & lanemask_lt())] = ((uint64_t)(uint32_t)lv.id(my_pos) << 32) | (uint32_t)my_pos;
            }
            if (!settle && amb2) sc.list2[__popc(ma2 & lanemask_lt())] = my_pos;
            __syncwarp();
            if (settle) {
                write_kept(p, lv, L, bh, sc.sortb, K);
                __syncwarp();
                continue;
            }
            nsel += n_in2;
            r -= n_in2;
            nlist = nA2;
            list = sc.list2;
        }
        // ---- tier 3 ----
        int chosen = 0;
        bool have_pivot = false;
        uint32_t pivot[kScoreDigits];
        int pivot_id = 0;
        while (chosen < r) {
            const int want = min(r - chosen, RC);
            int nbest = 0;
            for (int b0 = 0; b0 < nlist; b0 += RC) {
                const int len = min(RC, nlist - b0);
                for (int i = 0; i < len; ++i) {
                    const int pos = list[b0 + i];
                    warp_exact_score<T, D>(qh, q_stride, p.N, kbase + (size_t)lv.row(pos) * D, CH + i * kScoreDigits);
                    if (lane == 0) {
                        ch_id[i] = lv.id(pos);
                        ch_pos[i] = pos;
                    }
                }
                if (p.stats && lane == 0) atomicAdd(p.stats + L * 4 + 3, (unsigned long long)len);
                __syncwarp();
                // merge the chunk into BEST: pool element ep = lane
                const int npool = nbest + len;
                const int ep = lane;
                const uint32_t *xe = ep < nbest ? BEST + ep * kScoreDigits : CH + (ep - nbest) * kScoreDigits;
                const int ide = ep < nbest ? best_id[ep] : (ep < npool ? ch_id[ep - nbest] : 0);
                const bool valid = ep < npool && (ep < nbest || !have_pivot || exact_better(pivot, pivot_id, xe, ide));
                const unsigned vmask = __ballot_sync(0xffffffffu, valid);
                int rk = 0x7fffffff;
                if (valid) {
                    rk = 0;
                    unsigned others = vmask & ~(1u << ep);
                    while (others) {
                        const int f2 = __ffs(others) - 1;
                        others &= others - 1;
                        const uint32_t *xf = f2 < nbest ? BEST + f2 * kScoreDigits : CH + (f2 - nbest) * kScoreDigits;
                        const int idf = f2 < nbest ? best_id[f2] : ch_id[f2 - nbest];
                        if (exact_better(xf, idf, xe, ide)) ++rk;
                    }
                }
                if (rk < want) {
#pragma unroll
                    for (int q = 0; q < kScoreDigits; ++q) TMP[rk * kScoreDigits + q] = xe[q];
                    tmp_id[rk] = ide;
                    tmp_pos[rk] = ep < nbest ? best_pos[ep] : ch_pos[ep - nbest];
                }
                __syncwarp();
                nbest = min(want, __popc(vmask));
                for (int i = lane; i < nbest * kScoreDigits; i += 32) BEST[i] = TMP[i];
                if (lane < nbest) {
                    best_id[lane] = tmp_id[lane];
                    best_pos[lane] = tmp_pos[lane];
                }
                __syncwarp();
            }
            if (nbest == 0) break;   // only if r exceeded the list, which cannot happen
            if (lane < nbest)
                sc.sortb[nsel + lane] = ((uint64_t)(uint32_t)best_id[lane] << 32) | (uint32_t)best_pos[lane];
            nsel += nbest;
            chosen += nbest;
#pragma unroll
            for (int q = 0; q < kScoreDigits; ++q) pivot[q] = BEST[(nbest - 1) * kScoreDigits + q];
            pivot_id = best_id[nbest - 1];
            have_pivot = true;
            __syncwarp();
        }
        write_kept(p, lv, L, bh, sc.sortb, K);
        __syncwarp();
    }
}

// ==========================================================================
// Tree set-up kernels
// ==========================================================================

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
