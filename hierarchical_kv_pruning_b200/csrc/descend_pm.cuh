// Parent-major HiKVP descent.
//
// "AtlasKV: Augmenting LLMs with Billion-Scale Knowledge Graphs in 20GB VRAM",
// section "Quick read / How it works": every traversal (query b, head h)
// scores the children of its kept parents and keeps the top K.  Across a
// batch many traversals keep the same parents (a KV head's heads, and the
// queries of a batch, share the upper levels), so the child rows a level needs
// are far fewer than the traversals' candidates.  This path reads each needed
// child row about once per level:
//
//   token_sums_kernel  s, s64, a64 and ||a||_2 of every traversal
//   pm_score_kernel    one work item = one parent (level 0: a KV head's
//                      roots) and up to EC traversals that kept it: the
//                      parent's child rows pass through a cp.async ring once
//                      and are scored against the EC token-sum vectors; each
//                      score lands at the traversal's candidate slot
//   pm_select_kernel   one warp per traversal: top K of its candidates with
//                      the certified band (warp_select); then it counts its
//                      kept parents per (KV head, parent) for the next level
//   pm_scan_kernel     exclusive scan over all (KV head, parent) keys of the
//                      counts (decoupled look-back, one pass): each key's
//                      first list position and its work items
//   pm_fill_kernel     each kept entry into its key's segment of the list
//
// The scores, the band, the refinement and the kept lists are those of the
// fused kernel (the same device functions); only the order in which child rows
// are read changes, so the results are identical.
#pragma once

#include "descend.cuh"

namespace akv {

constexpr int kPmThreads = 128;                 // scoring CTA: 4 warps, one ring each
constexpr int kPmWarps = kPmThreads / 32;
constexpr int kPmPassRows = 1024;               // child rows whose table is built at a time
constexpr int kPmMaxEC = 32;                    // traversals per work item, at most
constexpr int kScanThreads = 256;
constexpr int kScanPerThread = 8;
constexpr int kScanTile = kScanThreads * kScanPerThread;
constexpr int kScanSpinLimit = 1 << 22;         // look-back wait bound (then an error status)
constexpr int kSelThreads = 256;

// The inversion of level L - 1's kept lists, read when level L is scored.
// Key of a kept entry e = bh Kp + k (traversal bh, its k-th kept parent):
// hkv rows[L - 1] + parent id.
struct PmLevel {
    int32_t *cnt;                 // [NK] entries per key (zero at the call's start)
    int32_t *eoff;                // [NK] first list position of the key's entries
    int32_t *rank;                // [E] rank of entry e among its key's entries
    int32_t *list;                // [E] entries grouped by key
    int4 *ctab;                   // [max_items] work items: (key, first list position, count, 0)
    unsigned long long *tval;     // [2 n_tiles] per scan tile: aggregate, inclusive prefix
    int32_t *tflag;               // [n_tiles] 0, 1 aggregate ready, 2 prefix ready (zero at the start)
    int32_t *ctr;                 // [4] tile ticket, number of work items (zero at the start)
    int32_t *cpre;                // CSR level: [BH][Kp + 1] first candidate of each kept parent, else null
    long long NK;
    int E, max_items, n_tiles;
};

__device__ __forceinline__ void copy_params(DescendParams &dst, const DescendParams &src)
{
    static_assert(sizeof(DescendParams) % 4 == 0, "word copy");
    const int *s = reinterpret_cast<const int *>(&src);
    int *d = reinterpret_cast<int *>(&dst);
    for (int i = threadIdx.x; i < (int)(sizeof(DescendParams) / 4); i += blockDim.x) d[i] = s[i];
}

__device__ __forceinline__ int ld_acquire(const int32_t *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(int32_t *p, int v)
{
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------------------
// Token sums: one CTA per (query, KV head, chunk of GC heads).
template <typename T, int D>
__global__ void __launch_bounds__(kDescThreads) token_sums_kernel(const __grid_constant__ DescendParams p, int GC)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int hchunks = p.G / GC;
    const int hc = (int)(blockIdx.x % hchunks);
    const int grp = (int)(blockIdx.x / hchunks);
    const int b = grp / p.H_kv, hkv = grp % p.H_kv;
    const long long bh0 = (long long)b * p.H + (long long)hkv * p.G + (long long)hc * GC;
    const T *qb = reinterpret_cast<const T *>(p.q_kg) + ((size_t)b * p.N * p.H + (size_t)(bh0 - (long long)b * p.H)) * D;
    token_sums<T, D>(p, qb, bh0, GC, reinterpret_cast<double *>(smem_raw));
}

// Shared-memory bytes of token_sums_kernel's partial sums for GC heads.
__host__ __device__ constexpr size_t token_sums_smem(int GC, int D, int esz)
{
    const int ev = 16 / esz;
    const int combos = GC * (D / ev);
    const int slices = combos <= kDescThreads ? kDescThreads / combos : 1;
    return combos <= kDescThreads ? (size_t)slices * combos * 2 * ev * 8 : 0;
}

// ---------------------------------------------------------------------------
// Scoring: work items in turn (blockIdx.x, + gridDim.x, ...).  A warp serves
// HT traversals of the item and holds their token-sum slices in registers; a
// key row spans LPG lanes (one 16-byte vector each) and a lane group takes R
// = LPG / HT rows at a time, reducing its R x HT partial dot products by
// recursive halving (as in the fused kernel).  The hgn = ceil(ne / HT) head
// groups of an item share the row stream; 4 / hgn streams split the rows.
template <typename T, int D, int HT>
__global__ void __launch_bounds__(kPmThreads, 4)
    pm_score_kernel(const __grid_constant__ DescendParams p0, const __grid_constant__ PmLevel pl, int L, int EC)
{
    constexpr int EV = Vec16<T>::E;
    constexpr int LPG = D / EV;
    constexpr int GPW = 32 / LPG;
    constexpr int R = LPG / HT;
    static_assert(LPG >= 8 && LPG <= 32 && R >= 1 && R * HT == LPG, "one score per lane");
    constexpr int RCH = GPW * R;
    constexpr int ROWB = D * (int)sizeof(T);
    static_assert(R <= 4 && RCH * ROWB <= kChunkBytes, "a chunk fits its ring stage");
    static_assert(kPmWarps * HT <= kPmMaxEC, "entries per item");

    __shared__ DescendParams p;
    __shared__ __align__(16) uint8_t ring_all[kPmWarps * kRingStages * kChunkBytes];
    __shared__ int32_t trow[kPmPassRows];
    __shared__ long long ent_bh[kPmMaxEC];
    __shared__ int ent_c0[kPmMaxEC];
    __shared__ long long item_base;
    __shared__ int item_i[5];
    copy_params(p, p0);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int lg = lane / LPG, sub = lane % LPG;
    const int k_mine = sub / HT, h_mine = sub - (sub / HT) * HT;
    const int BG = p.B * p.G;
    const int Kp = L == 0 ? 1 : p.K[L - 1];
    const int fo = p.fanout[L];
    const long long prow = L == 0 ? 1 : p.rows[L - 1], rows = p.rows[L];
    const T *kbase = reinterpret_cast<const T *>(p.keys[L]);
    const int32_t *coff = L >= 1 ? p.coff[L - 1] : nullptr;
    const int32_t *cid = L >= 1 ? p.cid[L - 1] : nullptr;
    const int32_t *tab = L >= 1 ? p.child[L - 1] : nullptr;
    const int32_t *slot = L >= 1 ? p.slot[L] : nullptr;
    const int per_hkv = (BG + EC - 1) / EC;
    const int n_items = L == 0 ? p.H_kv * per_hkv : min(pl.ctr[1], pl.max_items);

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        __syncthreads();   // the previous item's entries, row table and rings are free
        if (threadIdx.x == 0) {
            int hkv, par = 0, e0, ne, n_c;
            long long base = 0;   // CSR: the first child entry; slot: the pool row of child 0
            if (L == 0) {
                hkv = item / per_hkv;
                e0 = (item - hkv * per_hkv) * EC;
                ne = min(EC, BG - e0);
                n_c = (int)rows;
            } else {
                const int4 it = pl.ctab[item];
                hkv = (int)(it.x / prow);
                par = (int)(it.x - (long long)hkv * prow);
                e0 = it.y;
                ne = min(it.z, EC);
                if (coff) {
                    const int32_t *off_h = coff + (size_t)hkv * (prow + 1);
                    base = off_h[par];
                    n_c = off_h[par + 1] - (int)base;
                } else {
                    n_c = fo;
                    if (slot) base = (long long)slot[pl.list[e0]] * fo;   // any copy of the block will do
                }
            }
            item_i[0] = hkv;
            item_i[1] = par;
            item_i[2] = e0;
            item_i[3] = ne;
            item_i[4] = n_c;
            item_base = base;
        }
        __syncthreads();
        const int hkv = item_i[0], par = item_i[1], e0 = item_i[2], ne = item_i[3], n_c = item_i[4];
        const long long base = item_base;
        if ((int)threadIdx.x < ne) {
            long long bh;
            int c0;
            if (L == 0) {
                const int i = e0 + threadIdx.x;
                const int b = i / p.G;
                bh = (long long)b * p.H + (long long)hkv * p.G + (i - b * p.G);
                c0 = 0;
            } else {
                const int e = pl.list[e0 + threadIdx.x];
                bh = e / Kp;
                const int k = e - (int)bh * Kp;
                c0 = pl.cpre ? pl.cpre[bh * (Kp + 1) + k] : k * fo;
            }
            ent_bh[threadIdx.x] = bh;
            ent_c0[threadIdx.x] = c0;
        }
        __syncthreads();

        const int hgn = (ne + HT - 1) / HT;
        const int streams = kPmWarps / hgn;
        const bool computes = warp < streams * hgn;
        const int hg = warp % hgn, rs = warp / hgn;
        const int g_mine = hg * HT + h_mine;
        const bool stores = computes && g_mine < ne;

        // this lane's slice of the head group's token sums, as packed pairs
        uint64_t sreg[HT][EV / 2];
#pragma unroll
        for (int h = 0; h < HT; ++h) {
            const int g = hg * HT + h;
            const bool ok = computes && g < ne;
            const float *sp = p.s_ws + (size_t)(ok ? ent_bh[g] : 0) * D + sub * EV;
#pragma unroll
            for (int e = 0; e < EV; e += 4) {
                float4 t4 = *reinterpret_cast<const float4 *>(sp + e);
                if (!ok) t4 = make_float4(0.f, 0.f, 0.f, 0.f);
                sreg[h][e / 2] = pack2(t4.x, t4.y);
                sreg[h][e / 2 + 1] = pack2(t4.z, t4.w);
            }
        }
        float *f_mine = p.f_ws + (size_t)(stores ? ent_bh[g_mine] : 0) * p.fstride + (stores ? ent_c0[g_mine] : 0);
        uint8_t *ring = ring_all + (size_t)(rs < kPmWarps ? rs : 0) * kRingStages * kChunkBytes;
        const int tg = (int)threadIdx.x - rs * hgn * 32;
        auto stream_sync = [&]() {
            if (hgn == 1) __syncwarp();
            else asm volatile("bar.sync %0, %1;" ::"r"(1 + rs), "r"(hgn * 32) : "memory");
        };
        // key row of child j of the item's parent
        auto row_of = [&](int j) -> long long {
            if (L == 0) return (long long)hkv * rows + j;
            if (slot) return base + j;
            long long id;
            if (coff) {
                const long long e = base + j;
                id = cid ? (long long)cid[(size_t)hkv * rows + e] : e;
            } else {
                id = tab ? (long long)tab[((size_t)hkv * prow + par) * fo + j] : (long long)par * fo + j;
            }
            if (id < 0 || id >= rows) {
                set_status(p.status, kDevBadChild);
                id = 0;
            }
            return (long long)hkv * rows + id;
        };

        for (int q0 = 0; q0 < n_c; q0 += kPmPassRows) {
            const int pr = min(kPmPassRows, n_c - q0);
            for (int r = threadIdx.x; r < pr; r += kPmThreads) trow[r] = (int32_t)row_of(q0 + r);
            __syncthreads();   // the pass's row table is complete
            if (computes) {
                const int nck = (pr + RCH - 1) / RCH;
                auto issue = [&](int t) {
                    const int c = rs + t * streams;
                    if (c < nck) {
                        const uint32_t dst0 = (uint32_t)__cvta_generic_to_shared(ring + (t % kRingStages) * kChunkBytes);
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
                    const int rr = c * RCH + lg * R + k_mine;
                    if (stores && rr < pr) f_mine[q0 + rr] = v[0];
                }
                asm volatile("cp.async.wait_group 0;\n" ::);
            }
            __syncthreads();   // the rings and the table are free for the next pass
        }
    }
}

// ---------------------------------------------------------------------------
// Selection: one warp per traversal, nsel warps per CTA, each with pw bytes of
// shared memory: the selection scratch and score copy, the kept parents and
// (CSR) their candidate prefix.  With nx.cnt set, the warp then counts its
// kept entries per key for the next level (nx) and, on a CSR next level,
// writes their candidate prefix.
__host__ __device__ constexpr size_t pm_select_warp_bytes(int kcap, int cap, int Kpmax)
{
    return (warp_sel_bytes(kcap, cap) + (size_t)(2 * Kpmax + 2) * 4 + 15) & ~size_t(15);
}

template <typename T, int D>
__global__ void __launch_bounds__(kSelThreads, 2)
    pm_select_kernel(const __grid_constant__ DescendParams p0, const __grid_constant__ PmLevel nx, int L, int nsel, int pw)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ DescendParams p;
    copy_params(p, p0);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long BH = (long long)p.B * p.H;
    const long long bh = (long long)blockIdx.x * nsel + warp;
    if (warp >= nsel || bh >= BH) return;   // no CTA barrier below
    uint8_t *ws = smem_raw + (size_t)warp * pw;
    uint32_t *hist = reinterpret_cast<uint32_t *>(ws);
    uint64_t *tmp = reinterpret_cast<uint64_t *>(ws + 1024);
    uint64_t *kbuf = p.kcap <= kKbufSmem ? reinterpret_cast<uint64_t *>(ws + 1536)
                                         : reinterpret_cast<uint64_t *>(p.f_ws + (size_t)bh * p.fstride + p.cap);
    float *fs = reinterpret_cast<float *>(ws + warp_sel_bytes(p.kcap, 0));
    int32_t *prev = reinterpret_cast<int32_t *>(ws + warp_sel_bytes(p.kcap, p.cap));
    int32_t *cpre = prev + p.Kpmax;
    const int hkv = (int)(bh % p.H) / p.G;
    const int Kp = L == 0 ? 0 : p.K[L - 1];
    const bool csr = L >= 1 && p.coff[L - 1] != nullptr;
    if (L >= 1) {
        for (int k = lane; k < Kp; k += 32) prev[k] = p.kept[L - 1][bh * Kp + k];
        __syncwarp();
        if (csr) {
            const int32_t *off_h = p.coff[L - 1] + (size_t)hkv * (p.rows[L - 1] + 1);
            warp_prefix_counts(Kp, [&](int k) { return off_h[prev[k] + 1] - off_h[prev[k]]; }, cpre);
        }
    }
    ExactScratch xs(p.xs_ws + (size_t)bh * ExactScratch::bytes());
    warp_select<T, D>(p, L, bh, csr ? cpre : nullptr, L == 0 ? nullptr : prev, hist, tmp, kbuf, fs, xs);
    __syncwarp();
    if (nx.cnt) {
        const int K = p.K[L];
        const long long rws = p.rows[L];
        const int32_t *kl = p.kept[L] + bh * K;
        for (int k = lane; k < K; k += 32) {
            const int id = kl[k];
            if (id < 0 || id >= rws) {
                set_status(p.status, kDevBadChild);
                nx.rank[bh * K + k] = -1;
                continue;
            }
            nx.rank[bh * K + k] = atomicAdd(nx.cnt + (size_t)hkv * rws + id, 1);
        }
        if (nx.cpre) {
            const int32_t *off_h = p.coff[L] + (size_t)hkv * (rws + 1);
            warp_prefix_counts(
                K,
                [&](int k) {
                    const int id = kl[k];
                    return (id < 0 || id >= rws) ? 0 : off_h[id + 1] - off_h[id];
                },
                nx.cpre + bh * (K + 1));
        }
    }
}

// ---------------------------------------------------------------------------
// Inversion, part 1: exclusive scan over the keys of the packed pair (entries,
// work items) = (cnt, ceil(cnt / EC)), the entries in the low 32 bits.  Tiles
// take tickets in launch order and wait only on tiles with earlier tickets
// (running or finished), each wait bounded.  Per key with entries: its first
// list position and its work items (key, position, count).
__global__ void __launch_bounds__(kScanThreads) pm_scan_kernel(const __grid_constant__ PmLevel pl, int EC, int *status)
{
    __shared__ int tile_sh;
    __shared__ unsigned long long wsum[kScanThreads / 32];
    __shared__ unsigned long long pre_sh;
    if (threadIdx.x == 0) tile_sh = atomicAdd(pl.ctr, 1);
    __syncthreads();
    const int tile = tile_sh;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long k0 = (long long)tile * kScanTile + (long long)threadIdx.x * kScanPerThread;
    int c[kScanPerThread];
    unsigned long long loc = 0;
#pragma unroll
    for (int i = 0; i < kScanPerThread; ++i) {
        const long long key = k0 + i;
        c[i] = key < pl.NK ? pl.cnt[key] : 0;
        loc += (unsigned long long)(unsigned)c[i] | ((unsigned long long)(unsigned)((c[i] + EC - 1) / EC) << 32);
    }
    unsigned long long incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long w = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += w;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    unsigned long long wpre = 0, agg = 0;
    for (int w = 0; w < kScanThreads / 32; ++w) {
        if (w < warp) wpre += wsum[w];
        agg += wsum[w];
    }
    if (threadIdx.x == 0) {
        unsigned long long pre = 0;
        if (tile == 0) {
            pl.tval[1] = agg;
            st_release(pl.tflag, 2);
        } else {
            pl.tval[2 * tile] = agg;
            st_release(pl.tflag + tile, 1);
            int j = tile - 1, spins = 0;
            while (j >= 0) {
                const int f = ld_acquire(pl.tflag + j);
                if (f == 2) {
                    pre += pl.tval[2 * j + 1];
                    break;
                }
                if (f == 1) {
                    pre += pl.tval[2 * j];
                    --j;
                    continue;
                }
                if (++spins > kScanSpinLimit) {
                    set_status(status, kDevTimeout);
                    break;
                }
            }
            pl.tval[2 * tile + 1] = pre + agg;
            st_release(pl.tflag + tile, 2);
        }
        pre_sh = pre;
        if (tile == pl.n_tiles - 1) pl.ctr[1] = (int)((pre + agg) >> 32);
    }
    __syncthreads();
    unsigned long long run = pre_sh + wpre + incl - loc;
#pragma unroll
    for (int i = 0; i < kScanPerThread; ++i) {
        const long long key = k0 + i;
        if (c[i] > 0) {
            const int e0 = (int)(run & 0xffffffffu), i0 = (int)(run >> 32);
            pl.eoff[key] = e0;
            const int n = (c[i] + EC - 1) / EC;
            for (int j = 0; j < n; ++j)
                if (i0 + j < pl.max_items) pl.ctab[i0 + j] = make_int4((int)key, e0 + j * EC, min(EC, c[i] - j * EC), 0);
        }
        run += (unsigned long long)(unsigned)c[i] | ((unsigned long long)(unsigned)((c[i] + EC - 1) / EC) << 32);
    }
}

// Inversion, part 2: every kept entry of level L - 1 into its key's segment.
__global__ void pm_fill_kernel(const int32_t *__restrict__ kept_prev, int Kp, int H, int G, long long prow,
                               const __grid_constant__ PmLevel pl, int *status)
{
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < pl.E;
         e += (long long)gridDim.x * blockDim.x) {
        const long long bh = e / Kp;
        const int hkv = (int)(bh % H) / G;
        const int id = kept_prev[e];
        const int r = pl.rank[e];
        if (id < 0 || id >= prow || r < 0) {
            set_status(status, kDevBadChild);
            continue;
        }
        const long long pos = (long long)pl.eoff[(size_t)hkv * prow + id] + r;
        if (pos < 0 || pos >= pl.E) {
            set_status(status, kDevBadChild);
            continue;
        }
        pl.list[pos] = (int32_t)e;
    }
}

}  // namespace akv
