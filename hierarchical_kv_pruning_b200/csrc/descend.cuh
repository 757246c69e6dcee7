// Level-by-level HiKVP descent, one fused kernel.
//
// "AtlasKV: Augmenting LLMs with Billion-Scale Knowledge Graphs in 20GB VRAM",
// section "Quick read / How it works": score the query against the resident
// root keys, keep the top-K branches, bring in the children's keys, prune level
// by level down to the leaves.  Node score (reading of that section): mean over
// the query tokens of <q_n, k>/sqrt(D); ranking by x(k) = sum_d s[d] k[d] with
// s[d] = sum_n q[n][d] is equivalent.
//
// Every (query b, KV head) group descends independently of the others, so one
// CTA owns one group (or a chunk of GC <= 32 of its G query heads) for the
// whole descent and no step needs a grid-wide barrier:
//   token sums   s, and the float64 sums used by the refinement, of GC heads
//   per level    the union of the GC heads' kept parents (root level: the
//                b_R roots); every child row of the union is copied once into
//                a shared-memory ring by cp.async and scored against all GC
//                token-sum vectors with fp32 FMA; then one warp per head
//                selects that head's top-K with the certified band below,
//                refining in float64 and, if needed, in exact arithmetic.
// The per-traversal scores live in the workspace (L2-resident at the
// benchmark sizes); the row ring, the union tables and the selection scratch
// share one shared-memory region, used in turn.
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

#include <type_traits>

#include "common.cuh"
#include "exact.cuh"

namespace akv {

constexpr int kDescThreads = 256;
constexpr int kDescWarps = kDescThreads / 32;
constexpr int kRefineChunk = 16;   // exact scores per refinement chunk (a pool of two chunks fills a warp)
constexpr int kKbufSmem = 128;     // kept lists up to this size are built in shared memory
constexpr int kPassRows = 4096;    // rows of a level scored per pass (the pass's row table)
constexpr int kRingStages = 4;     // per row stream: three chunks in flight ahead of the one being scored
constexpr int kChunkBytes = 2048;  // a chunk: 32 / HT rows of D e bytes (HT >= 16 e / (4 ... ) keeps it at 2 KB)
constexpr int kMaxLevels = 4;      // levels of a tree (roots .. leaves)

struct DescendParams {
    const void *q_kg;            // [B][N][H][D]
    int B, N, H, H_kv, G;
    int GC;                      // query heads per CTA (divides G, <= 32)
    int n_levels;                // 3 for uniform trees; 2 .. kMaxLevels for CSR trees
    int Kpmax;                   // the largest K of a level that has children
    const void *keys[kMaxLevels];     // key base per level (a host-staged level: its pool)
    long long rows[kMaxLevels];       // rows per KV head of each level
    int fanout[kMaxLevels];           // uniform trees: children per node of level l - 1 (fanout[0] = roots)
    const int32_t *child[kMaxLevels - 1];   // uniform trees: [H_kv][rows_l][fanout_{l+1}] child rows, or null
    // CSR trees (variable numbers of children): per level l above the leaves,
    // coff[l] [H_kv][rows_l + 1] offsets into the child list and cid[l]
    // [H_kv][rows_{l+1}] the listed rows (null: the list positions are the rows)
    const int32_t *coff[kMaxLevels - 1];
    const int32_t *cid[kMaxLevels - 1];
    const float *norm_bound;     // [n_levels][H_kv] upper bounds of key row 2-norms
    int K[kMaxLevels];
    double cprime;               // g_D (1 + g_N) + g_N of the fp32 filter bound (computed on the host)
    int32_t *kept[kMaxLevels];   // [B H][K_l] ascending row ids
    float *s_ws;                 // [B H][D] fp32 token sums (rounded from s64)
    double *s64_ws;              // [B H][D] fp64 token sums
    double *a64_ws;              // [B H][D] fp64 sums of |q| over the tokens
    float *anorm_ws;             // [B H] upper bound of ||a||_2
    float *f_ws;                 // [B H][fstride]: cap fp32 scores of the current level (then the band
                                 // list), followed by kcap uint64 kept entries when kcap > kKbufSmem
    int fstride;                 // floats per traversal in f_ws: cap + 2 kcap
    int cap;                     // per-traversal score capacity (>= every level's candidate count)
    int kcap;                    // kept capacity (power of two >= every K)
    uint8_t *xs_ws;              // refinement scratch, [grid][min(GC, kDescWarps)][ExactScratch::bytes()]
    // host-staged levels L = 1, 2: kept parent k of traversal bh has its block
    // of children at pool slot slot[L][bh K[L-1] + k]; candidate (k, j) is pool
    // row slot * fanout[L] + j of keys[L] (the pool).  Null: keys[L] is the
    // level's own device array.
    const int32_t *slot[kMaxLevels];
    int32_t *kept_leaf_row;      // [B H][K_leaf] pool row of each kept leaf (host path)
    unsigned long long *stats;   // [kMaxLevels][4] optional counters: selections, refined, ambiguous, exact scores
    int *status;
};

__host__ __device__ __forceinline__ double gamma_n(int n)
{
    const double nu = (double)n * 0x1p-24;
    return nu / (1.0 - nu);
}

__device__ __forceinline__ unsigned lanemask_lt() { return (1u << (threadIdx.x & 31)) - 1u; }

// Warp exclusive prefix sum of one int per lane; the total in `total`.
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

// Two independent IEEE binary32 fused multiply-adds in one instruction: the
// low and high halves of the 64-bit operands are separate lanes (acc.lo +=
// a.lo * b.lo, acc.hi += a.hi * b.hi), each rounded to nearest.
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t acc)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(acc));
    return d;
}
__device__ __forceinline__ uint64_t pack2(float lo, float hi)
{
    return ((uint64_t)__float_as_uint(hi) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ float sum2(uint64_t v)
{
    return __uint_as_float((uint32_t)v) + __uint_as_float((uint32_t)(v >> 32));
}

// A 16-byte vector of key elements as EV / 2 packed pairs (element 2i low,
// 2i + 1 high).
template <typename T> struct Pairs16;
template <> struct Pairs16<__nv_bfloat16> {
    __device__ __forceinline__ static void get(const uint4 &v, uint64_t *o)
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] = ((uint64_t)(w[i] & 0xffff0000u) << 32) | (uint32_t)(w[i] << 16);
    }
};
template <> struct Pairs16<float> {
    __device__ __forceinline__ static void get(const uint4 &v, uint64_t *o)
    {
        o[0] = ((uint64_t)v.y << 32) | v.x;
        o[1] = ((uint64_t)v.w << 32) | v.z;
    }
};

// ==========================================================================
// Shared-memory plan of the descent CTA
// ==========================================================================

__host__ __device__ constexpr int desc_hash_size(int total)
{
    int hs = 64;
    while (hs < 2 * total) hs <<= 1;
    return hs;
}

// Per-warp selection scratch: a 256-bin histogram, 64 bucket members, the
// kept entries when they fit (kcap <= kKbufSmem), and a copy of the head's
// scores (cap floats): every pass of the selection reads shared memory.
__host__ __device__ constexpr size_t warp_sel_bytes(int kcap, int cap)
{
    return 1024 + 512 + (kcap <= kKbufSmem ? (size_t)kcap * 8 : 0) + (size_t)cap * 4;
}

// Warps that select (one head at a time each): at most GC and the CTA's
// warps, fewer when their score copies would take more than this much of
// shared memory (at least one).
constexpr size_t kSelBudget = 96 * 1024;
__host__ __device__ constexpr int selecting_warps(int GC, int kcap, int cap)
{
    int w = GC < kDescWarps ? GC : kDescWarps;
    while (w > 1 && (size_t)w * warp_sel_bytes(kcap, cap) > kSelBudget) --w;
    return w;
}

// Region A is used in turn by: the token sums' partial sums (level 0), the
// union hash set of a level, the warps' selection scratch.  Then the union
// lists, the per-head slot map and the CSR prefixes.
struct DescLayout {
    size_t regA, lists, P, Pown, kidx, rowpre, cpre, total_bytes;
    int total;   // capacity of the union: GC * max kept parents
    int hs;

    int nsel;    // selecting warps
    size_t ring, table;   // scoring: the row streams' rings and the pass's row table (both in region A)

    __host__ __device__ DescLayout(int GC, int Kpmax, int kcap, int cap, int D, int esz)
    {
        nsel = selecting_warps(GC, kcap, cap);
        auto r16 = [](size_t b) { return (b + 15) & ~size_t(15); };
        total = GC * Kpmax;
        hs = desc_hash_size(total);
        const int ev = 16 / esz;
        const int combos = GC * (D / ev);
        const int slices = combos <= kDescThreads ? kDescThreads / combos : 1;
        const size_t part = combos <= kDescThreads ? (size_t)slices * combos * 2 * ev * 8 : 0;
        const size_t setup = (size_t)(3 * hs + total) * 4;
        const size_t sel = (size_t)nsel * warp_sel_bytes(kcap, cap);
        // one ring per row stream (at most kDescWarps streams), then the table
        ring = 0;
        table = (size_t)kDescWarps * kRingStages * kChunkBytes;
        const size_t scoring = table + (size_t)kPassRows * 8;
        (void)D;
        size_t a = setup;
        if (scoring > a) a = scoring;
        if (part > a) a = part;
        if (sel > a) a = sel;
        regA = 0;
        lists = r16(a);
        P = lists + r16((size_t)total * 4);
        Pown = P + r16((size_t)total * 4);
        kidx = Pown + r16((size_t)total * 4);
        rowpre = kidx + r16((size_t)GC * total * 2);                  // CSR: [total + 1] union row prefix
        cpre = rowpre + r16((size_t)(total + 1) * 4);                 // CSR: [GC][Kpmax + 1] candidate prefix
        total_bytes = cpre + r16((size_t)GC * (Kpmax + 1) * 4);
    }
};

// ==========================================================================
// Token sums (a1)
// ==========================================================================

// Token sums of the GC consecutive heads starting at qb (token 0), in float64:
// s64[g][d] = sum_n q[n][h0+g][d] and a64[g][d] = sum_n |q[n][h0+g][d]|
// (relative error below g_N in binary64), written to the workspace rows of
// traversals bh0 .. bh0 + GC - 1 together with s = fl32(s64) and the bound of
// ||a||_2.  The fp32 filter uses s, whose error |s - sum_n q| <= (u32 + g64_N) a
// is well inside the g32_N a of the bound.  Each thread owns one 16-byte column
// vector of one head and a slice of the tokens; slices meet in `part`.
template <typename T, int D>
__device__ __noinline__ void token_sums(const DescendParams &p, const T *qb, long long bh0, int GC, double *part)
{
    constexpr int EV = Vec16<T>::E;
    constexpr int VPH = D / EV;
    const int combos = GC * VPH;
    const size_t q_stride = (size_t)p.H * D;
    const int N = p.N;
    float *s = p.s_ws + (size_t)bh0 * D;
    double *s64 = p.s64_ws + (size_t)bh0 * D;
    double *a64 = p.a64_ws + (size_t)bh0 * D;
    auto column = [&](int combo, int n0, int step, double *ps, double *pa) {
        const int g = combo / VPH, v = combo - g * VPH;
        const T *col = qb + (size_t)g * D + v * EV;
#pragma unroll
        for (int e = 0; e < EV; ++e) ps[e] = pa[e] = 0.0;
        int n = n0;
        for (; n + 7 * step < N; n += 8 * step) {   // eight tokens' loads in flight
            uint4 w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) w[u] = ldg16(col + (size_t)(n + u * step) * q_stride);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                float x[EV];
                Vec16<T>::unpack(w[u], x);
#pragma unroll
                for (int e = 0; e < EV; ++e) {
                    ps[e] += (double)x[e];
                    pa[e] += fabs((double)x[e]);
                }
            }
        }
        for (; n < N; n += step) {
            float x[EV];
            Vec16<T>::unpack(ldg16(col + (size_t)n * q_stride), x);
#pragma unroll
            for (int e = 0; e < EV; ++e) {
                ps[e] += (double)x[e];
                pa[e] += fabs((double)x[e]);
            }
        }
    };
    if (combos <= kDescThreads) {
        const int slices = kDescThreads / combos;
        const int combo = threadIdx.x % combos, slice = threadIdx.x / combos;
        if (slice < slices) {
            double ps[EV], pa[EV];
            column(combo, slice, slices, ps, pa);
#pragma unroll
            for (int e = 0; e < EV; ++e) {
                part[((slice * combos + combo) * 2 + 0) * EV + e] = ps[e];
                part[((slice * combos + combo) * 2 + 1) * EV + e] = pa[e];
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < GC * D; i += kDescThreads) {
            const int cb = i / EV, e = i % EV;   // i = (g VPH + v) EV + e
            double ss = 0.0, aa = 0.0;
            for (int sl = 0; sl < slices; ++sl) {
                ss += part[((sl * combos + cb) * 2 + 0) * EV + e];
                aa += part[((sl * combos + cb) * 2 + 1) * EV + e];
            }
            s64[i] = ss;
            a64[i] = aa;
            s[i] = (float)ss;
        }
    } else {
        for (int combo = threadIdx.x; combo < combos; combo += kDescThreads) {
            double ps[EV], pa[EV];
            column(combo, 0, 1, ps, pa);
#pragma unroll
            for (int e = 0; e < EV; ++e) {
                s64[combo * EV + e] = ps[e];
                a64[combo * EV + e] = pa[e];
                s[combo * EV + e] = (float)ps[e];
            }
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int g = warp; g < GC; g += kDescWarps) {
        double acc = 0.0;
        for (int d = lane; d < D; d += 32) acc = fma(a64[g * D + d], a64[g * D + d], acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        // sqrt(1 + 1e-9) covers the binary64 rounding of a64; (1 + 1e-6) the rounding to fp32
        if (lane == 0) p.anorm_ws[bh0 + g] = (float)(sqrt(acc) * (1.0 + 1e-9)) * (1.0f + 1e-6f);
    }
}

// ==========================================================================
// Selection helpers (one warp)
// ==========================================================================

// Ascending bitonic sort of the warp's 32 E values held in registers, lane l
// holding elements l E .. l E + E - 1 (E = 1, 2 or 4): partners within a lane
// are compared in place, the others exchanged by shuffles.  The stage loops
// stay rolled (small code: the selection runs beside many other warps).
__device__ __forceinline__ void cmp_swap(uint64_t &a, uint64_t &b, bool asc)
{
    const uint64_t lo = a < b ? a : b, hi = a < b ? b : a;
    a = asc ? lo : hi;
    b = asc ? hi : lo;
}

template <int S, int E>
__device__ __forceinline__ void lane_stage(uint64_t (&v)[E], int i0, int size)
{
#pragma unroll
    for (int e = 0; e < E; ++e)
        if ((e & S) == 0) cmp_swap(v[e], v[e + S], ((i0 + e) & size) == 0);
}

template <int E>
__device__ __forceinline__ void reg_bitonic(uint64_t (&v)[E])
{
    static_assert(E == 1 || E == 2 || E == 4 || E == 8, "E");
    const int lane = threadIdx.x & 31;
    constexpr int n = 32 * E;
#pragma unroll 1
    for (int size = 2; size <= n; size <<= 1) {
#pragma unroll 1
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            if (stride >= E) {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int i = lane * E + e;
                    const uint64_t o = __shfl_xor_sync(0xffffffffu, v[e], stride / E);
                    const bool lower = (i & stride) == 0, asc = (i & size) == 0;
                    v[e] = (lower == asc) ? (v[e] < o ? v[e] : o) : (v[e] > o ? v[e] : o);
                }
            } else if constexpr (E >= 2) {
                const int i0 = lane * E;
                if (stride == 1) {
                    lane_stage<1, E>(v, i0, size);
                } else if constexpr (E >= 4) {
                    if (stride == 2) lane_stage<2, E>(v, i0, size);
                    else if constexpr (E >= 8) lane_stage<4, E>(v, i0, size);
                }
            }
        }
    }
}

// Ascending warp bitonic sort of n (power of two) uint64 (shared or global).
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
    const int32_t *slot;      // pool slots of the kept parents (host-staged level), or null
    // CSR levels: cpre[k] = first candidate of kept parent k (cpre[Kp] = C),
    // off / ids the parent level's offsets and child rows of this KV head
    const int32_t *cpre, *off, *ids;
    int Kp;

    __device__ __forceinline__ int id(int c) const
    {
        if (L == 0) return c;
        if (cpre) {
            int lo = 0, hi = Kp - 1;   // the last k with cpre[k] <= c
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (cpre[mid] <= c) lo = mid;
                else hi = mid - 1;
            }
            const long long e = (long long)off[prev[lo]] + (c - cpre[lo]);
            const long long v = ids ? (long long)ids[e] : e;
            return (v < 0 || v >= rows) ? 0 : (int)v;
        }
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

// cpre: the traversal's candidate prefix of a CSR level (shared memory), else
// null; prev_sh: the traversal's kept parents in shared memory, or null (then
// they are read from the workspace).
__device__ __forceinline__ LevelView level_view(const DescendParams &p, int L, long long bh, const int32_t *cpre,
                                                const int32_t *prev_sh = nullptr)
{
    const int h = (int)(bh % p.H);
    const int Kp = L == 0 ? 0 : p.K[L - 1];
    LevelView lv;
    lv.L = L;
    lv.Kp = Kp;
    lv.fo = L == 0 ? 1 : p.fanout[L];
    lv.C = L == 0 ? (int)p.rows[0] : (cpre ? cpre[Kp] : Kp * lv.fo);
    lv.cpre = cpre;
    lv.off = nullptr;
    lv.ids = nullptr;
    if (cpre) {
        lv.off = p.coff[L - 1] + (size_t)(h / p.G) * (p.rows[L - 1] + 1);
        lv.ids = p.cid[L - 1] ? p.cid[L - 1] + (size_t)(h / p.G) * p.rows[L] : nullptr;
    }
    lv.tab = L == 0 ? nullptr : p.child[L - 1];
    lv.prow = L == 0 ? 0 : p.rows[L - 1];
    lv.rows = p.rows[L];
    lv.hkv = h / p.G;
    lv.slot = (L >= 1 && p.slot[L]) ? p.slot[L] + bh * Kp : nullptr;
    lv.prev = L == 0 ? nullptr : (prev_sh ? prev_sh : p.kept[L - 1] + bh * Kp);
    return lv;
}

// Exclusive prefix of count(i), i < n, into out[0..n) and the total into
// out[n], by one warp (n is small: a union of kept parents, a kept list).
template <typename CountFn>
__device__ __forceinline__ void warp_prefix_counts(int n, CountFn count, int32_t *out)
{
    const int lane = threadIdx.x & 31;
    int carry = 0;
    for (int b = 0; b < n; b += 32) {
        const int i = b + lane;
        const int v = i < n ? count(i) : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int w = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += w;
        }
        if (i < n) out[i] = carry + incl - v;
        carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) out[n] = carry;
    __syncwarp();
}

// Sort kbuf[0..K) (entries id << 32 | position) by id and write the ascending
// kept list of traversal bh (and the pool rows of kept leaves on the host path).
template <int E>
__device__ __forceinline__ void write_kept_reg(const DescendParams &p, const LevelView &lv, int L, long long bh,
                                               const uint64_t *kbuf, int K)
{
    const int lane = threadIdx.x & 31;
    uint64_t v[E];
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = lane * E + e < K ? kbuf[lane * E + e] : ~0ull;
    reg_bitonic<E>(v);
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int i = lane * E + e;
        if (i < K) {
            p.kept[L][bh * K + i] = (int32_t)(v[e] >> 32);
            if (L == 2 && p.kept_leaf_row) p.kept_leaf_row[bh * K + i] = (int32_t)lv.row((int)(v[e] & 0xffffffffu));
        }
    }
    __syncwarp();
}

__device__ __forceinline__ void write_kept(const DescendParams &p, const LevelView &lv, int L, long long bh,
                                           uint64_t *kbuf, int K)
{
    const int lane = threadIdx.x & 31;
    __syncwarp();
    if (K <= 32) return write_kept_reg<1>(p, lv, L, bh, kbuf, K);
    if (K <= 64) return write_kept_reg<2>(p, lv, L, bh, kbuf, K);
    if (K <= 128) return write_kept_reg<4>(p, lv, L, bh, kbuf, K);
    int n2 = 1;
    while (n2 < K) n2 <<= 1;
    for (int i = K + lane; i < n2; i += 32) kbuf[i] = ~0ull;
    warp_sort_u64(kbuf, n2);
    for (int i = lane; i < K; i += 32) p.kept[L][bh * K + i] = (int32_t)(kbuf[i] >> 32);
    if (L == 2 && p.kept_leaf_row)
        for (int i = lane; i < K; i += 32)
            p.kept_leaf_row[bh * K + i] = (int32_t)lv.row((int)(kbuf[i] & 0xffffffffu));
    __syncwarp();
}

// Pick the bin holding the kk-th largest value from a 256-bin histogram
// (bins ascending in value): its index, the rank inside it, and its count.
__device__ __forceinline__ void warp_pick_bin(const uint32_t *hist, int kk, int &bin, int &rem, int &bcount)
{
    const int lane = threadIdx.x & 31;
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
}

// k-th largest (1-based) of the n floats f[0..n) by one warp, given their min
// mn and max mx.  Values are bucketed linearly between min and max (a monotone
// map); the bucket holding the k-th largest is then searched exactly: sorted
// when it holds at most 64, else narrowed by MSB-first radix passes over the
// order-preserving bit image.  hist: 256 bins; tmp: 64 uint64.
__device__ __forceinline__ float warp_kth_largest(const float *f, int n, int k, float mn, float mx, uint32_t *hist,
                                                  uint64_t *tmp)
{
    const int lane = threadIdx.x & 31;
    if (mx == mn) return mx;   // all equal
    if (mx > mn && isfinite(mx - mn)) {
        const float scale = 255.99f / (mx - mn);
        auto bucket = [&](float v) { return min(255, max(0, (int)((v - mn) * scale))); };
        for (int j = lane; j < 256; j += 32) hist[j] = 0;
        __syncwarp();
        // four values per lane per step (f is 16-byte aligned, n rounded up to 4 is inside it)
        const float4 *f4 = reinterpret_cast<const float4 *>(f);
        const int nv = (n + 3) >> 2;
        for (int v4 = lane; v4 < nv; v4 += 32) {
            const float4 x = f4[v4];
            const float e[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (4 * v4 + q < n) atomicAdd(&hist[bucket(e[q])], 1u);
        }
        __syncwarp();
        int bk, rem, bcount;
        warp_pick_bin(hist, k, bk, rem, bcount);
        if (bcount <= 64) {
            // the bucket's members (order is irrelevant: they are sorted next)
            int base = 0;
            for (int b4 = 0; b4 < nv; b4 += 32) {
                const int v4 = b4 + lane;
                float e[4] = {0.f, 0.f, 0.f, 0.f};
                if (v4 < nv) {
                    const float4 x = f4[v4];
                    e[0] = x.x;
                    e[1] = x.y;
                    e[2] = x.z;
                    e[3] = x.w;
                }
                int cnt = 0;
                bool in[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    in[q] = v4 < nv && 4 * v4 + q < n && bucket(e[q]) == bk;
                    cnt += in[q];
                }
                int tot;
                int off = base + warp_excl_scan(cnt, tot);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (in[q]) tmp[off++] = ~(uint64_t)float_key(e[q]);
                base += tot;
            }
            __syncwarp();
            uint64_t r[2];
            r[0] = 2 * lane < base ? tmp[2 * lane] : ~0ull;
            r[1] = 2 * lane + 1 < base ? tmp[2 * lane + 1] : ~0ull;
            reg_bitonic<2>(r);
            const int idx = rem - 1;   // of the ascending ~key order: the rem-th largest value
            const uint64_t pick = __shfl_sync(0xffffffffu, (idx & 1) ? r[1] : r[0], idx >> 1);
            __syncwarp();
            return key_float((uint32_t)~pick);
        }
        __syncwarp();
    }
    // general case: radix select on the bit image
    uint32_t prefix = 0, mask = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int j = lane; j < 256; j += 32) hist[j] = 0;
        __syncwarp();
        for (int i = lane; i < n; i += 32) {
            const uint32_t key = float_key(f[i]);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncwarp();
        int digit, rem, unused;
        warp_pick_bin(hist, k, digit, rem, unused);
        prefix |= ((uint32_t)digit) << shift;
        mask |= 255u << shift;
        k = rem;
        __syncwarp();
    }
    return key_float(prefix);
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

// Per-warp scratch of the refinement (workspace memory: it is needed only for
// the few selections the fp32 band leaves open).
struct ExactScratch {
    uint32_t *ex;      // [3 RC][kScoreDigits]
    int32_t *ids;      // [3 RC]
    int32_t *poss;     // [3 RC]
    int32_t *list2;    // [32] positions still ambiguous after tier 2
    __host__ __device__ static constexpr size_t bytes()
    {
        return (size_t)3 * kRefineChunk * kScoreDigits * 4 + 2 * (size_t)3 * kRefineChunk * 4 + 128;
    }
    __device__ explicit ExactScratch(uint8_t *p)
    {
        ex = reinterpret_cast<uint32_t *>(p);
        ids = reinterpret_cast<int32_t *>(p + (size_t)3 * kRefineChunk * kScoreDigits * 4);
        poss = ids + 3 * kRefineChunk;
        list2 = poss + 3 * kRefineChunk;
    }
};

// Tier 2 of the refinement (see warp_refine): the listed candidates (at most
// 32, all scores finite) in float64 with their own bounds.  Returns true when
// that settles the selection (kbuf then holds K entries); otherwise the
// candidates kept for sure are appended (nsel, r updated) and list / nlist
// name the still-ambiguous ones (in sc.list2).
template <typename T, int D>
__device__ __forceinline__ bool refine_tier2(const DescendParams &p, const LevelView &lv, long long bh,
                                             uint64_t *kbuf, int &nsel, int &r, const int *&list, int &nlist,
                                             ExactScratch &sc)
{
    const int lane = threadIdx.x & 31;
    const T *kbase = reinterpret_cast<const T *>(p.keys[lv.L]);
    // lane d holds elements d, d + 32, ... of s64 and a64; every listed
    // candidate's fp64 dot product is split over the lanes and summed by
    // shuffles (binary64 in any order: the g64_D bound below holds), four
    // candidates' rows in flight at a time; lane j keeps candidate j's.
    constexpr int DL = D / 32;
    const double *s64 = p.s64_ws + (size_t)bh * D;
    const double *a64 = p.a64_ws + (size_t)bh * D;
    double sv[DL], av[DL];
#pragma unroll
    for (int j = 0; j < DL; ++j) {
        sv[j] = s64[lane + 32 * j];
        av[j] = a64[lane + 32 * j];
    }
    const int my_pos = lane < nlist ? list[lane] : -1;
    const long long my_row = my_pos >= 0 ? lv.row(my_pos) : 0;
    double y = -INFINITY, e2 = 0.0;
    const double g64d = (double)D * 0x1p-53 / (1.0 - (double)D * 0x1p-53);
    const double g64n = (double)p.N * 0x1p-53 / (1.0 - (double)p.N * 0x1p-53);
    for (int c0 = 0; c0 < nlist; c0 += 4) {
        float x[4][DL];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const long long rr = __shfl_sync(0xffffffffu, my_row, min(c0 + u, nlist - 1));
            const T *krow = kbase + (size_t)rr * D;
#pragma unroll
            for (int j = 0; j < DL; ++j) x[u][j] = elem_f32(krow[lane + 32 * j]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            double acc = 0.0, mag = 0.0;
#pragma unroll
            for (int j = 0; j < DL; ++j) {
                acc = fma(sv[j], (double)x[u][j], acc);
                mag = fma(av[j], fabs((double)x[u][j]), mag);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                acc += __shfl_xor_sync(0xffffffffu, acc, o);
                mag += __shfl_xor_sync(0xffffffffu, mag, o);
            }
            if (lane == c0 + u && lane < nlist) {
                y = acc;
                e2 = (g64d * (1.0 + g64n) + g64n) * mag * (1.0 + 1e-6) + 0x1p-1000;
            }
        }
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
        kbuf[nsel + __popc(m & lanemask_lt())] = ((uint64_t)(uint32_t)lv.id(my_pos) << 32) | (uint32_t)my_pos;
    }
    if (!settle && amb2) sc.list2[__popc(ma2 & lanemask_lt())] = my_pos;
    __syncwarp();
    if (settle) return true;
    nsel += n_in2;
    r -= n_in2;
    nlist = nA2;
    list = sc.list2;
    return false;
}

// A selection tier 1 left open: nsel entries are kept in kbuf already and
// r = K - nsel places remain among the nlist band candidates `list`.
//   tier 2: when at most 32 are listed (and all scores were finite), each lane
//           scores one of them in float64 from the float64 token sums, with its
//           own rigorous bound  (g64_D (1 + g64_N) + g64_N) sum_d a64_d |k_d|,
//           and the band argument is repeated among them;
//   tier 3: whatever is still open is ranked by exact score, then row id: the
//           candidates are scanned in chunks of RC with a bounded best-set, and
//           passes repeat (each excluding everything not strictly worse than
//           the last one chosen) until r are chosen.
// On return kbuf[0..K) holds the kept entries.
template <typename T, int D>
__device__ __noinline__ void warp_refine(const DescendParams &p, const LevelView &lv, int L, long long bh,
                                         uint64_t *kbuf, int nsel, const int *list, int nlist, bool bad,
                                         ExactScratch &sc)
{
    constexpr int RC = kRefineChunk;
    const int lane = threadIdx.x & 31;
    const int K = p.K[L];
    int r = K - nsel;
    const int b = (int)(bh / p.H), h = (int)(bh % p.H);
    const T *qh = reinterpret_cast<const T *>(p.q_kg) + ((size_t)b * p.N * p.H + h) * D;
    const size_t q_stride = (size_t)p.H * D;
    const T *kbase = reinterpret_cast<const T *>(p.keys[L]);
    uint32_t *BEST = sc.ex, *CH = sc.ex + RC * kScoreDigits, *TMP = sc.ex + 2 * RC * kScoreDigits;
    int32_t *best_id = sc.ids, *ch_id = sc.ids + RC, *tmp_id = sc.ids + 2 * RC;
    int32_t *best_pos = sc.poss, *ch_pos = sc.poss + RC, *tmp_pos = sc.poss + 2 * RC;

    if (!bad && nlist <= 32 && refine_tier2<T, D>(p, lv, bh, kbuf, nsel, r, list, nlist, sc)) return;
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
        if (lane < nbest) kbuf[nsel + lane] = ((uint64_t)(uint32_t)best_id[lane] << 32) | (uint32_t)best_pos[lane];
        nsel += nbest;
        chosen += nbest;
#pragma unroll
        for (int q = 0; q < kScoreDigits; ++q) pivot[q] = BEST[(nbest - 1) * kScoreDigits + q];
        pivot_id = best_id[nbest - 1];
        have_pivot = true;
        __syncwarp();
    }
}

// Top-K of traversal bh at level L by one warp, from its fp32 scores f[0..C)
// (tier 1): the scores and their rigorous bound E settle every candidate
// outside the band [t - 2E, t + 2E] around the K-th largest score t; when the
// band holds more candidates than places left, warp_refine decides them --
// here, or (kDefer) in a later kernel: the band list goes to the traversal's
// score row, the entries kept so far to its kept-entry area behind the scores,
// and (bh, kept so far, listed, bad) to the queue; then it returns false.
template <typename T, int D, bool kDefer = false>
__device__ __forceinline__ bool warp_select(const DescendParams &p, int L, long long bh, const int32_t *cpre,
                                            const int32_t *prev_sh, uint32_t *hist, uint64_t *tmp, uint64_t *kbuf,
                                            float *f, ExactScratch &xs, int4 *queue = nullptr,
                                            int *qcount = nullptr)
{
    const int lane = threadIdx.x & 31;
    const LevelView lv = level_view(p, L, bh, cpre, prev_sh);
    // kbuf entries are built as candidate positions and given their row ids
    // (id << 32 | position) in one pass of independent loads before sorting
    auto resolve_ids = [&](int n) {
        for (int i = lane; i < n; i += 32) {
            const int c = (int)(uint32_t)kbuf[i];
            kbuf[i] = ((uint64_t)(uint32_t)lv.id(c) << 32) | (uint32_t)c;
        }
        __syncwarp();
    };
    const int C = lv.C, K = p.K[L];
    // the bound's inputs are loaded first: their latency overlaps the copy
    const float anorm = p.anorm_ws[bh], knorm = p.norm_bound[L * p.H_kv + lv.hkv];
    float mn = INFINITY, mx = -INFINITY;
    int bad = 0;
    {
        // the head's scores into this warp's shared copy f: 16-byte loads,
        // several in flight per lane (the passes below then read shared
        // memory); min, max and finiteness on the way
        const float4 *src = reinterpret_cast<const float4 *>(p.f_ws + (size_t)bh * p.fstride);
        float4 *dst = reinterpret_cast<float4 *>(f);
        const int nv = (C + 3) >> 2;
        auto take = [&](const float4 &t4, int v4) {
            dst[v4] = t4;
            const float e[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (4 * v4 + q < C) {
                    mn = fminf(mn, e[q]);
                    mx = fmaxf(mx, e[q]);
                    bad |= !isfinite(e[q]);
                }
        };
        int v = lane;
        for (; v + 224 < nv; v += 256) {
            float4 t[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) t[u] = __ldcg(src + v + 32 * u);
#pragma unroll
            for (int u = 0; u < 8; ++u) take(t[u], v + 32 * u);
        }
        for (; v + 96 < nv; v += 128) {
            float4 t[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) t[u] = __ldcg(src + v + 32 * u);
#pragma unroll
            for (int u = 0; u < 4; ++u) take(t[u], v + 32 * u);
        }
        for (; v < nv; v += 32) take(__ldcg(src + v), v);
        __syncwarp();
    }
    if (p.stats && lane == 0) atomicAdd(p.stats + L * 4, 1ull);
    if (K >= C) {
        for (int c = lane; c < C; c += 32) kbuf[c] = (uint32_t)c;
        __syncwarp();
        resolve_ids(C);
        __syncwarp();
        write_kept(p, lv, L, bh, kbuf, K);
        return true;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    bad = __any_sync(0xffffffffu, bad);
    const double E = p.cprime * (double)anorm * (double)knorm * (1.0 + 1e-6) + D * 0x1p-148;
    const double t = bad ? 0.0 : (double)warp_kth_largest(f, C, K, mn, mx, hist, tmp);
    const bool bad2 = bad || !isfinite(E) || !isfinite(t);
    // band edges rounded outward to fp32: the sure-kept and sure-dropped sets can
    // only shrink, so the classification stays rigorous
    const float hi32 = bad2 ? INFINITY : __double2float_ru(__dadd_ru(t, 2.0 * E));
    const float lo32 = bad2 ? -INFINITY : __double2float_rd(__dsub_rd(t, 2.0 * E));
    // class of a candidate: 1 kept for sure, 2 ambiguous, 0 dropped.  The band
    // list is compacted in place over the scores: a list entry is stored at an
    // index below every score not yet read.
    // Four scores per lane per step; the step's reads all precede its writes
    // (the counts pass through the warp scan), and a step writes list entries
    // only below 4 (step + 1) 32.
    int *list = reinterpret_cast<int *>(f);
    int n_in = 0, nA = 0;
    {
        const float4 *f4 = reinterpret_cast<const float4 *>(f);
        const int nv = (C + 3) >> 2;
        for (int b4 = 0; b4 < nv; b4 += 32) {
            const int v4 = b4 + lane;
            float e[4] = {0.f, 0.f, 0.f, 0.f};
            if (v4 < nv) {
                const float4 x = f4[v4];
                e[0] = x.x;
                e[1] = x.y;
                e[2] = x.z;
                e[3] = x.w;
            }
            int k[4], c1 = 0, c2 = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const bool in = v4 < nv && 4 * v4 + q < C;
                k[q] = !in ? 0 : bad2 ? 2 : (e[q] > hi32 ? 1 : (e[q] >= lo32 ? 2 : 0));
                c1 += k[q] == 1;
                c2 += k[q] == 2;
            }
            int tot;
            const int pre = warp_excl_scan(c1 | (c2 << 16), tot);
            int o1 = n_in + (pre & 0xffff), o2 = nA + (pre >> 16);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (k[q] == 1) kbuf[o1++] = (uint32_t)(4 * v4 + q);
                if (k[q] == 2) list[o2++] = 4 * v4 + q;
            }
            n_in += tot & 0xffff;
            nA += tot >> 16;
        }
    }
    __syncwarp();
    const int r = K - n_in;
    if (nA == r) {   // every ambiguous candidate is kept
        for (int i = lane; i < nA; i += 32) {
            const int c = list[i];
            kbuf[n_in + i] = (uint32_t)c;
        }
        __syncwarp();
        resolve_ids(K);
        write_kept(p, lv, L, bh, kbuf, K);
        return true;
    }
    if (p.stats && lane == 0) {
        atomicAdd(p.stats + L * 4 + 1, 1ull);
        atomicAdd(p.stats + L * 4 + 2, (unsigned long long)nA);
    }
    resolve_ids(n_in);
    if constexpr (kDefer) {
        int *glist = reinterpret_cast<int *>(p.f_ws + (size_t)bh * p.fstride);
        uint64_t *gk = reinterpret_cast<uint64_t *>(p.f_ws + (size_t)bh * p.fstride + p.cap);
        for (int i = lane; i < nA; i += 32) glist[i] = list[i];
        if (gk != kbuf)
            for (int i = lane; i < n_in; i += 32) gk[i] = kbuf[i];
        __syncwarp();
        if (lane == 0) queue[atomicAdd(qcount, 1)] = make_int4((int)bh, n_in, nA, bad2 ? 1 : 0);
        (void)xs;
        return false;
    } else {
        warp_refine<T, D>(p, lv, L, bh, kbuf, n_in, list, nA, bad2, xs);
        __syncwarp();
        write_kept(p, lv, L, bh, kbuf, K);
        return true;
    }
}

// The same as a call: the fused kernel keeps the selection out of line (its
// registers go to the scoring loop).
template <typename T, int D>
__device__ __noinline__ void warp_select_call(const DescendParams &p, int L, long long bh, const int32_t *cpre,
                                              const int32_t *prev_sh, uint32_t *hist, uint64_t *tmp, uint64_t *kbuf,
                                              float *f, ExactScratch &xs)
{
    warp_select<T, D>(p, L, bh, cpre, prev_sh, hist, tmp, kbuf, f, xs);
}

// The same with the selection kept out of line and deferred refinement: the
// parent-major path's rare fallback.
template <typename T, int D>
__device__ __noinline__ bool warp_select_defer_call(const DescendParams &p, int L, long long bh, const int32_t *cpre,
                                                    const int32_t *prev_sh, uint32_t *hist, uint64_t *tmp,
                                                    uint64_t *kbuf, float *f, ExactScratch &xs, int4 *queue,
                                                    int *qcount)
{
    return warp_select<T, D, true>(p, L, bh, cpre, prev_sh, hist, tmp, kbuf, f, xs, queue, qcount);
}

// The k-th largest (1-based) of the warp's 32 E order-preserving float keys,
// k at most the number of real keys (padding keys are 0, below every real
// one): MSB-first, keep each bit while at least k keys are >= the prefix.
template <int E>
__device__ __forceinline__ uint32_t warp_kth_key(const uint32_t (&key)[E], int k)
{
    uint32_t t = 0;
#pragma unroll 1
    for (int b = 31; b >= 0; --b) {
        const uint32_t c = t | (1u << b);
        unsigned cnt = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) cnt += key[e] >= c;
        if (__reduce_add_sync(0xffffffffu, cnt) >= (unsigned)k) t = c;
    }
    return t;
}

// Tier 1 in one pass over the scores (read from the traversal's workspace
// row), for the parent-major path:
//   1. a sample of 128 scores (all of them when C <= 128) gives t0, the j-th
//      largest sample value (a radix select) with j = ceil(1.25 K 128 / C) + 2, so
//      that about 1.25 K scores are expected above it: t0 <= t (the K-th
//      largest score) unless fewer than K scores are >= t0, which the pass
//      counts;
//   2. the pass collects every candidate with f >= fl_down(t0 - 2E) and counts
//      those >= t0;
//   3. with at least K counted (so t >= t0), every candidate of the band
//      [t - 2E, t + 2E] and above was collected: t is the K-th largest of the
//      collected (a radix select over their order-preserving keys); those
//      above t + 2E are kept for sure, those down to t - 2E are the band.
//      (With C <= 128 the sample is every score: t comes from it directly.)
// Non-finite scores, too many collected (more than kCollectCap) or too few
// counted fall back to warp_select on the same row.  The certified band and
// the refinement are those of warp_select, so the kept sets are the same.
constexpr int kCollectCap = 512;

template <typename T, int D>
__device__ __forceinline__ bool warp_select_pm(const DescendParams &p, int L, long long bh, const int32_t *cpre,
                                               const int32_t *prev_sh, uint32_t *hist, uint64_t *tmp, uint64_t *kbuf,
                                               uint64_t *col, ExactScratch &xs, int4 *queue, int *qcount)
{
    const int lane = threadIdx.x & 31;
    const LevelView lv = level_view(p, L, bh, cpre, prev_sh);
    const int C = lv.C, K = p.K[L];
    float *f = p.f_ws + (size_t)bh * p.fstride;
    auto fallback = [&]() {
        return warp_select_defer_call<T, D>(p, L, bh, cpre, prev_sh, hist, tmp, kbuf, f, xs, queue, qcount);
    };
    auto resolve_ids = [&](int n) {
        for (int i = lane; i < n; i += 32) {
            const int c = (int)(uint32_t)kbuf[i];
            kbuf[i] = ((uint64_t)(uint32_t)lv.id(c) << 32) | (uint32_t)c;
        }
        __syncwarp();
    };
    if (K >= C) return fallback();
    const float anorm = p.anorm_ws[bh], knorm = p.norm_bound[L * p.H_kv + lv.hkv];
    const double E = p.cprime * (double)anorm * (double)knorm * (1.0 + 1e-6) + D * 0x1p-148;
    if (!isfinite(E)) return fallback();

    // ---- 1. the sample threshold (all scores when C <= 128) ----
    const bool all = C <= 128;
    uint32_t skey[4];
    float sval[4];
    int bad = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int i = lane * 4 + e;
        const int idx = all ? i : (int)(((long long)i * C) >> 7);
        sval[e] = (!all || i < C) ? __ldcg(f + idx) : -INFINITY;
        bad |= (!all || i < C) && !isfinite(sval[e]);
        skey[e] = float_key(sval[e]);
    }
    if (__any_sync(0xffffffffu, bad)) return fallback();
    float t;
    int ncol = 0;
    if (all) {   // every score is in the sample: t is exact
        t = key_float(warp_kth_key<4>(skey, K));
    } else {
        const int j = (5 * K * 128 + 4 * C - 1) / (4 * C) + 2;
        if (j > 127) return fallback();
        const float t0 = key_float(warp_kth_key<4>(skey, j + 1));
        const float c_lo = __double2float_rd(__dsub_rd((double)t0, 2.0 * E));

        // ---- 2. one pass: collect, count, check (four 16-byte loads in flight per lane) ----
        int cnt = 0;
        const float4 *f4 = reinterpret_cast<const float4 *>(f);
        const int nv = (C + 3) >> 2;
        for (int b4 = 0; b4 < nv; b4 += 128) {
            float4 x[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int v4 = b4 + 32 * u + lane;
                x[u] = v4 < nv ? __ldcg(f4 + v4) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int v4 = b4 + 32 * u + lane;
                const float e[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
                bool take[4];
                int c1 = 0;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const bool in = v4 < nv && 4 * v4 + q < C;
                    bad |= in && !isfinite(e[q]);
                    take[q] = in && e[q] >= c_lo;
                    cnt += in && e[q] >= t0;
                    c1 += take[q];
                }
                int tot;
                int off = ncol + warp_excl_scan(c1, tot);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (take[q]) {
                        if (off < kCollectCap) col[off] = ((uint64_t)float_key(e[q]) << 32) | (uint32_t)(4 * v4 + q);
                        ++off;
                    }
                ncol += tot;
            }
        }
        cnt = (int)__reduce_add_sync(0xffffffffu, (unsigned)cnt);
        bad = __any_sync(0xffffffffu, bad);
        if (bad || !isfinite(t0) || cnt < K || ncol > kCollectCap) return fallback();
        __syncwarp();

        // ---- 3. t: the K-th largest of the collected ----
        if (ncol <= 256) {
            uint32_t key[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) key[e] = lane * 8 + e < ncol ? (uint32_t)(col[lane * 8 + e] >> 32) : 0u;
            t = key_float(warp_kth_key<8>(key, K));
        } else {
            uint32_t key[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) key[e] = lane * 16 + e < ncol ? (uint32_t)(col[lane * 16 + e] >> 32) : 0u;
            t = key_float(warp_kth_key<16>(key, K));
        }
    }
    // the sure set above t + 2E (positions into kbuf) and the band down to
    // t - 2E (positions compacted to the front of col)
    const float hi32 = __double2float_ru(__dadd_ru((double)t, 2.0 * E));
    const float lo32 = __double2float_rd(__dsub_rd((double)t, 2.0 * E));
    int n_in = 0, nA = 0;
    if (all) {
        int c_in = 0, c_b = 0;
        bool sin[4], sb[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool valid = lane * 4 + e < C;
            sin[e] = valid && sval[e] > hi32;
            sb[e] = valid && !sin[e] && sval[e] >= lo32;
            c_in += sin[e];
            c_b += sb[e];
        }
        int tot;
        const int pre = warp_excl_scan(c_in | (c_b << 16), tot);
        int o1 = pre & 0xffff, o2 = pre >> 16;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (sin[e]) kbuf[o1++] = (uint32_t)(lane * 4 + e);
            if (sb[e]) col[o2++] = (uint32_t)(lane * 4 + e);
        }
        n_in = tot & 0xffff;
        nA = tot >> 16;
    } else {
        for (int i0 = 0; i0 < ncol; i0 += 32) {
            const int i = i0 + lane;
            const uint64_t ent = i < ncol ? col[i] : 0ull;
            const float v = key_float((uint32_t)(ent >> 32));
            const bool sin = i < ncol && v > hi32;
            const bool sb = i < ncol && !sin && v >= lo32;
            const unsigned mi = __ballot_sync(0xffffffffu, sin), mb = __ballot_sync(0xffffffffu, sb);
            if (sin) kbuf[n_in + __popc(mi & lanemask_lt())] = (uint32_t)ent;
            if (sb) col[nA + __popc(mb & lanemask_lt())] = (uint32_t)ent;   // at or below i: already read
            n_in += __popc(mi);
            nA += __popc(mb);
        }
    }
    __syncwarp();
    if (p.stats && lane == 0) atomicAdd(p.stats + L * 4, 1ull);
    const int r = K - n_in;
    if (nA == r) {   // every band candidate is kept
        for (int i = lane; i < nA; i += 32) kbuf[n_in + i] = (uint32_t)col[i];
        __syncwarp();
        resolve_ids(K);
        write_kept(p, lv, L, bh, kbuf, K);
        return true;
    }
    if (p.stats && lane == 0) {
        atomicAdd(p.stats + L * 4 + 1, 1ull);
        atomicAdd(p.stats + L * 4 + 2, (unsigned long long)nA);
    }
    resolve_ids(n_in);
    // tier 2 here when the band is short (the band's positions in hist)
    int nsel = n_in, rr = r, nl = nA;
    const int *lst = reinterpret_cast<const int *>(hist);
    if (nA <= 32) {
        if (lane < nA) hist[lane] = (uint32_t)col[lane];
        __syncwarp();
        if (refine_tier2<T, D>(p, lv, bh, kbuf, nsel, rr, lst, nl, xs)) {
            write_kept(p, lv, L, bh, kbuf, K);
            return true;
        }
    }
    // hand over to the refinement kernel: the open candidates' positions over
    // the scores (consumed), the entries kept so far behind them, a queue entry
    int *glist = reinterpret_cast<int *>(f);
    uint64_t *gk = reinterpret_cast<uint64_t *>(f + p.cap);
    __syncwarp();
    if (nA <= 32) {
        for (int i = lane; i < nl; i += 32) glist[i] = lst[i];
    } else {
        for (int i = lane; i < nA; i += 32) glist[i] = (int)(uint32_t)col[i];
    }
    if (gk != kbuf)
        for (int i = lane; i < nsel; i += 32) gk[i] = kbuf[i];
    __syncwarp();
    if (lane == 0) queue[atomicAdd(qcount, 1)] = make_int4((int)bh, nsel, nl, 0);
    (void)rr;
    return false;
}

// ==========================================================================
// The descent kernel
// ==========================================================================

// One CTA per (query b, KV head, chunk of GC heads); levels first..last.  When
// first > 0 the token sums and the kept lists of level first - 1 are read from
// the workspace (written by an earlier launch: the host-leaf path stages the
// leaf blocks between levels 1 and 2).
//
// Scoring a level: the CTA forms the union of its GC heads' kept parent lists
// (a shared-memory hash set: O(GC Kp) work; at the root level the b_R roots)
// and scores every child row of the union parents against all GC token-sum
// vectors, so each row crosses from L2/HBM once per head group.  The rows are
// cut into chunks of 32 / HT rows, which the warps of a row stream take in
// turn, with no CTA barrier until the level is scored: a row is split over
// LPG = D / EV lanes, each loading its 16-byte vector straight from global
// memory into registers, and a warp keeps the next chunk's loads in flight
// while it scores the current one (the other warps and CTAs of the SM hide
// the rest of the latency).  A warp serves HT heads and keeps their token-sum
// slices in registers; a lane group takes R = LPG / HT rows at a time, forms
// R x HT partial dot products per lane and reduces them over the group by
// recursive halving, after which lane `sub` of the group holds the full score
// of value index sub = (row k, head h) = (sub / HT, sub % HT).  Head g's score
// of child j of union parent P[i] lands at its own candidate slot
// kidx[g][i] fo + j (CSR levels: the head's candidate prefix of its kept
// parent, plus j).  The fp32 sum of D products, in whatever order, stays
// within the g_D bound of the filter.
template <typename T, int D, int HT>
__device__ __forceinline__ void descend_cta(const DescendParams &p, const unsigned bid, int first, int last)
{
    constexpr int EV = Vec16<T>::E;          // elements per 16-byte vector
    constexpr int LPG = D / EV;              // lanes per row = 16-byte vectors per row
    constexpr int GPW = 32 / LPG;            // rows per warp read
    constexpr int R = LPG / HT;              // rows per lane group per reduction
    static_assert(LPG >= 8 && LPG <= 32 && R >= 1 && R * HT == LPG, "one score per lane");
    constexpr int NW = kDescWarps;
    constexpr int RCH = GPW * R;             // rows a warp scores per step (a chunk)
    constexpr int ROWB = D * (int)sizeof(T);
    static_assert(R <= 4 && RCH * ROWB <= kChunkBytes, "a chunk fits its ring stage");

    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ int seg[kDescThreads];
    __shared__ int nP_sh;

    const int GC = p.GC;
    const int Kpmax = p.Kpmax;
    const DescLayout lay(GC, Kpmax, p.kcap, p.cap, D, (int)sizeof(T));
    const int hchunks = p.G / GC;
    const int hc = bid % hchunks;
    const int grp_id = bid / hchunks;
    const int b = grp_id / p.H_kv, hkv = grp_id % p.H_kv;
    const long long bh0 = (long long)b * p.H + (long long)hkv * p.G + (long long)hc * GC;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint8_t *regA = smem_raw;
    int32_t *lists = reinterpret_cast<int32_t *>(smem_raw + lay.lists);   // [GC][Kp] kept parents
    int32_t *P = reinterpret_cast<int32_t *>(smem_raw + lay.P);           // union parents
    int32_t *Pown = reinterpret_cast<int32_t *>(smem_raw + lay.Pown);     // an entry (g Kp + k) listing P[i]
    int16_t *kidx = reinterpret_cast<int16_t *>(smem_raw + lay.kidx);     // [GC][total] slot of P[i] in g's list

    if (first == 0) {
        const T *qb = reinterpret_cast<const T *>(p.q_kg) + ((size_t)b * p.N * p.H + (size_t)(bh0 - (long long)b * p.H)) * D;
        token_sums<T, D>(p, qb, bh0, GC, reinterpret_cast<double *>(regA));
    }

    // warp -> (head group, row stream); lane -> (row group, vector of the row)
    const int hgn = (GC + HT - 1) / HT;
    const int streams = NW / hgn;
    const bool computes = warp < streams * hgn;
    const int hg = warp % hgn, rs = warp / hgn;
    const int lg = lane / LPG, sub = lane % LPG;
    const int k_mine = sub / HT, g_mine = hg * HT + (sub - (sub / HT) * HT);
    const bool stores = g_mine < GC;

    for (int L = first; L <= last; ++L) {
        __syncthreads();   // token sums / previous level's kept lists are complete; region A is free
        const int fo = p.fanout[L];
        const int Kp = L == 0 ? 1 : p.K[L - 1];
        const int total = GC * Kp;
        const int hs = desc_hash_size(total);
        int nP;
        if (L == 0) {
            nP = 1;   // one virtual parent whose children are the b_R roots
        } else {
            int32_t *hkey = reinterpret_cast<int32_t *>(regA);   // [hs] parent id or -1
            int32_t *hown = hkey + hs;                           // [hs] inserting entry
            int32_t *huid = hown + hs;                           // [hs] union index of the slot
            int32_t *eslot = huid + hs;                          // [total] hash slot of entry t
            for (int i = threadIdx.x; i < hs; i += kDescThreads) hkey[i] = -1;
            for (int i = threadIdx.x; i < GC * total; i += kDescThreads) kidx[i] = -1;
            for (int t = threadIdx.x; t < total; t += kDescThreads) {
                const int g = t / Kp, k = t - g * Kp;
                lists[t] = p.kept[L - 1][(bh0 + g) * Kp + k];
            }
            __syncthreads();
            // ---- union of the GC heads' kept parents: insert into the hash set ----
            for (int t = threadIdx.x; t < total; t += kDescThreads) {
                const int x = lists[t];
                unsigned hh = ((unsigned)x * 2654435761u) & (unsigned)(hs - 1);
                for (int probe = 0; probe < hs; ++probe) {
                    const int prev = atomicCAS(&hkey[hh], -1, x);
                    if (prev == -1) hown[hh] = t;
                    if (prev == -1 || prev == x) break;
                    hh = (hh + 1) & (unsigned)(hs - 1);
                }
                eslot[t] = (int)hh;
            }
            __syncthreads();
            // ---- number the occupied slots (table order): union index, P ----
            {
                const int per = (hs + kDescThreads - 1) / kDescThreads;
                const int t0 = min(hs, (int)threadIdx.x * per), t1 = min(hs, t0 + per);
                int cnt = 0;
                for (int t = t0; t < t1; ++t) cnt += (hkey[t] >= 0);
                seg[threadIdx.x] = cnt;
                __syncthreads();
                if (threadIdx.x < 32) {
                    int run = 0;
                    for (int base = 0; base < kDescThreads; base += 32) {
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
            for (int t = threadIdx.x; t < total; t += kDescThreads) {
                const int g = t / Kp, k = t - g * Kp;
                kidx[g * total + huid[eslot[t]]] = (int16_t)k;
            }
            nP = nP_sh;
            // region A (the hash set) is reused by the ring after the barrier below
        }
        // CSR level: a variable number of children per parent.  rowpre[i] =
        // first row of union parent i among the level's rows (rowpre[nP] =
        // nR); cpre[g][k] = first candidate of head g's kept parent k.
        const int32_t *coff = L >= 1 ? p.coff[L - 1] : nullptr;
        const bool csr = coff != nullptr;
        int32_t *rowpre = reinterpret_cast<int32_t *>(smem_raw + lay.rowpre);
        int32_t *cpre = reinterpret_cast<int32_t *>(smem_raw + lay.cpre);
        const int32_t *off_h = csr ? coff + (size_t)hkv * (p.rows[L - 1] + 1) : nullptr;
        const int32_t *cid_h = (csr && p.cid[L - 1]) ? p.cid[L - 1] + (size_t)hkv * p.rows[L] : nullptr;
        if (csr) {
            __syncthreads();   // the union P and the lists are complete
            if (warp == 0)
                warp_prefix_counts(nP, [&](int i) { return off_h[P[i] + 1] - off_h[P[i]]; }, rowpre);
            for (int g = warp; g < GC; g += NW)
                warp_prefix_counts(
                    Kp, [&](int k) { return off_h[lists[g * Kp + k] + 1] - off_h[lists[g * Kp + k]]; },
                    cpre + g * (Kp + 1));
            __syncthreads();
        }
        const int nR = csr ? rowpre[nP] : nP * fo;
        const T *kbase = reinterpret_cast<const T *>(p.keys[L]);
        const int32_t *tab = L == 0 ? nullptr : p.child[L - 1];
        const long long prow = L == 0 ? 0 : p.rows[L - 1], rows = p.rows[L];
        const int32_t *slot = L >= 1 ? p.slot[L] : nullptr;
        const int fstride = p.fstride;

        // (union parent i, child j) of a level row: the key row to read
        auto row_of = [&](int i, int j) -> long long {
            if (L == 0) return (long long)hkv * rows + j;
            if (csr) {
                const long long e = (long long)off_h[P[i]] + j;
                long long id = cid_h ? (long long)cid_h[e] : e;
                if (id < 0 || id >= rows) {
                    set_status(p.status, kDevBadChild);
                    id = 0;
                }
                return (long long)hkv * rows + id;
            }
            if (slot) {
                const int own = Pown[i];
                return (long long)slot[(bh0 + own / Kp) * Kp + own % Kp] * fo + j;
            }
            const long long par = P[i];
            long long id = tab ? (long long)tab[((size_t)hkv * prow + par) * fo + j] : par * fo + j;
            if (id < 0 || id >= rows) {
                set_status(p.status, kDevBadChild);
                id = 0;
            }
            return (long long)hkv * rows + id;
        };

        // this lane's slice of every head's token sums, as packed pairs
        uint64_t sreg[HT][EV / 2];
#pragma unroll
        for (int h = 0; h < HT; ++h) {
            const int g = hg * HT + h;
            const float *sp = p.s_ws + (size_t)(bh0 + (g < GC ? g : 0)) * D + sub * EV;
#pragma unroll
            for (int e = 0; e < EV; e += 4) {
                float4 t4 = *reinterpret_cast<const float4 *>(sp + e);
                if (g >= GC) t4 = make_float4(0.f, 0.f, 0.f, 0.f);
                sreg[h][e / 2] = pack2(t4.x, t4.y);
                sreg[h][e / 2 + 1] = pack2(t4.z, t4.w);
            }
        }
        const int16_t *kid_mine = kidx + (stores ? g_mine : 0) * total;
        const int32_t *cpre_mine = cpre + (stores ? g_mine : 0) * (Kp + 1);
        float *f_mine = p.f_ws + (size_t)(bh0 + (stores ? g_mine : 0)) * fstride;
        int32_t *trow = reinterpret_cast<int32_t *>(regA + lay.table);     // [kPassRows] key row
        int32_t *tij = trow + kPassRows;                                    // [kPassRows] union parent << 16 | child
        uint8_t *ring = regA + lay.ring + (size_t)rs * kRingStages * kChunkBytes;
        const int tg = (int)threadIdx.x - rs * hgn * 32;                    // thread within the row stream
        auto stream_sync = [&]() {
            if (hgn == 1) __syncwarp();
            else asm volatile("bar.sync %0, %1;" ::"r"(1 + rs), "r"(hgn * 32) : "memory");
        };

        // Passes of up to kPassRows rows: the row table of a pass is built by
        // every thread; then each row stream (the hgn warps of its head groups)
        // scores chunks rs, rs + streams, ... of the pass through its own ring
        // (cp.async, kRingStages - 1 chunks ahead), synchronised within the
        // stream only.
        for (int p0 = 0; p0 < nR; p0 += kPassRows) {
            const int pr = min(kPassRows, nR - p0);
            for (int r = threadIdx.x; r < pr; r += kDescThreads) {
                const int rho = p0 + r;
                int i, j;
                if (csr) {   // the last union parent whose rows start at or before rho
                    int lo = 0, hi = nP - 1;
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (rowpre[mid] <= rho) lo = mid;
                        else hi = mid - 1;
                    }
                    i = lo;
                    j = rho - rowpre[lo];
                } else {
                    i = rho / fo;
                    j = rho - i * fo;
                }
                trow[r] = (int32_t)row_of(i, j);
                tij[r] = (i << 16) | j;
            }
            __syncthreads();   // the pass's row table is complete
            if (computes) {
                const int nck = (pr + RCH - 1) / RCH;
                // copy chunk c of the pass into stage st: RCH rows of LPG vectors
                auto issue = [&](int t) {
                    const int c = rs + t * streams;
                    if (c < nck) {
                        const uint32_t dst0 =
                            (uint32_t)__cvta_generic_to_shared(ring + (t % kRingStages) * kChunkBytes);
                        for (int q = tg; q < RCH * LPG; q += hgn * 32) {
                            const int r = q / LPG, v = q - (q / LPG) * LPG;
                            const int rr = c * RCH + r;
                            const bool ok = rr < pr;
                            const T *src = kbase + (size_t)(ok ? trow[rr] : 0) * D + v * EV;
                            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst0 + r * ROWB + v * 16),
                                         "l"(src), "r"(ok ? 16 : 0));
                        }
                    }
                    asm volatile("cp.async.commit_group;\n" ::);
                };
#pragma unroll
                for (int t = 0; t < kRingStages - 1; ++t) issue(t);
                for (int t = 0; rs + t * streams < nck; ++t) {   // the same bound for the whole stream
                    asm volatile("cp.async.wait_group %0;\n" ::"n"(kRingStages - 2));
                    stream_sync();   // chunk t landed for the stream; the stage of chunk t - 1 is free
                    issue(t + kRingStages - 1);
                    const int c = rs + t * streams;
                    const uint8_t *tb = ring + (t % kRingStages) * kChunkBytes;
                    float v[LPG];
#pragma unroll
                    for (int k = 0; k < R; ++k) {
                        uint64_t xp[EV / 2];
                        Pairs16<T>::get(*reinterpret_cast<const uint4 *>(tb + (lg * R + k) * ROWB + sub * 16), xp);
#pragma unroll
                        for (int h = 0; h < HT; ++h) {
                            uint64_t acc = 0;
#pragma unroll
                            for (int e = 0; e < EV / 2; ++e) acc = ffma2(sreg[h][e], xp[e], acc);
                            v[k * HT + h] = sum2(acc);
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
                    // lane `sub` now holds the score of its row k_mine, head g_mine
                    const int rr = c * RCH + lg * R + k_mine;
                    if (stores && rr < pr) {
                        const int ij = tij[rr];
                        const int mi = ij >> 16, mj = ij & 0xffff;
                        const int kk = L == 0 ? 0 : kid_mine[mi];
                        if (kk >= 0) f_mine[(csr ? (size_t)cpre_mine[kk] : (size_t)kk * fo) + mj] = v[0];
                    }
                }
                asm volatile("cp.async.wait_group 0;\n" ::);
            }
            __syncthreads();   // the rings and the table are free for the next pass
        }
        __syncthreads();   // every score of the level is stored; region A is free

        // ---- selection: one warp per head ----
        const int nsel = lay.nsel;
        uint8_t *ws = regA + (size_t)(warp < nsel ? warp : 0) * warp_sel_bytes(p.kcap, p.cap);
        uint32_t *hist = reinterpret_cast<uint32_t *>(ws);
        uint64_t *tmp = reinterpret_cast<uint64_t *>(ws + 1024);
        // refinement scratch: one slot per selecting warp (warps >= GC select nothing)
        ExactScratch xs(p.xs_ws + ((size_t)bid * nsel + (warp < nsel ? warp : 0)) * ExactScratch::bytes());
        for (int g = warp; g < GC && warp < nsel; g += nsel) {
            uint64_t *kbuf = p.kcap <= kKbufSmem ? reinterpret_cast<uint64_t *>(ws + 1536)
                                                 : reinterpret_cast<uint64_t *>(p.f_ws + (size_t)(bh0 + g) * fstride +
                                                                                p.cap);
            float *fs = reinterpret_cast<float *>(ws + warp_sel_bytes(p.kcap, 0));
            warp_select_call<T, D>(p, L, bh0 + g, csr ? cpre + g * (Kp + 1) : nullptr, L == 0 ? nullptr : lists + g * Kp,
                              hist, tmp, kbuf, fs, xs);
        }
    }
    (void)lane;
}

// One call: one CTA per (query, KV head, chunk of GC heads).
template <typename T, int D, int HT>
__global__ void __launch_bounds__(kDescThreads, 2)
    descend_kernel(const __grid_constant__ DescendParams p, int first, int last)
{
    __shared__ DescendParams ps;   // the parameters in shared memory: cheap, indexable by level
    if (threadIdx.x == 0) ps = p;
    __syncthreads();
    descend_cta<T, D, HT>(ps, blockIdx.x, first, last);
}

// Several layers' calls in one launch (each layer its own tree and inputs,
// the same shapes): layer l owns the CTAs [offs[l], offs[l + 1]).
constexpr int kMaxLayers = 32;
struct DescendBatch {
    int n;
    unsigned offs[kMaxLayers + 1];
    DescendParams p[kMaxLayers];
};

template <typename T, int D, int HT>
__global__ void __launch_bounds__(kDescThreads, 2)
    descend_layers_kernel(const __grid_constant__ DescendBatch b, int first, int last)
{
    int l = 0;
    while (l + 1 < b.n && blockIdx.x >= b.offs[l + 1]) ++l;
    __shared__ DescendParams ps;   // the layer's parameters in shared memory
    if (threadIdx.x == 0) ps = b.p[l];
    __syncthreads();
    descend_cta<T, D, HT>(ps, blockIdx.x - b.offs[l], first, last);
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
