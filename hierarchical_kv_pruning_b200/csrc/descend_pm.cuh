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
    int4 *queue;                  // [BH] traversals of level L whose selection waits for refinement
    int32_t *qcount;              // queue length (zero at the start)
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
// Token sums: one CTA per (query, KV head, chunk of GC heads).  The grid also
// clears the call's zero-initialised inversion region (zero, zwords 16-byte
// words) once the previous grid on the stream is done.
template <typename T, int D>
__global__ void __launch_bounds__(kDescThreads)
    token_sums_kernel(const __grid_constant__ DescendParams p, int GC, uint4 *zero, long long zwords)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    griddep_launch();
    griddep_wait();
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < zwords; i += (long long)gridDim.x * blockDim.x)
        zero[i] = make_uint4(0u, 0u, 0u, 0u);
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
// Scoring: a small GEMM per work item.  Each warp takes items on its own
// (global warp gw: items gw, gw + all warps, ...; no CTA barrier), so an SM
// keeps many items in flight.  An item's child rows are taken kPmRP = 128 at
// a time (a pass); lane l owns rows l, l + 32, l + 64, l + 96 of the pass and
// holds a 4 x kPmEC register tile of partial scores (rows x traversals).  The
// contraction over D streams through two shared-memory stages of the warp:
// per stage a 64-byte slice of every row of the pass (cp.async, 16-byte
// pieces; piece c of row r at c ^ ((r >> 1) & 3), so a quarter-warp's eight
// rows sit in distinct banks) and the same slice of the item's token sums
// (read as broadcasts).  The next stage loads while this one is multiplied;
// the next item's table entry and traversals are loaded one item ahead.
// Scores go to the traversals' candidate slots, consecutive lanes to
// consecutive slots.  Products in fp32 pairs; the fp32 sum of D products, in
// whatever order, stays within the g_D bound of the filter.
constexpr int kPmEC = 8;        // traversals per work item
constexpr int kPmRP = 128;      // rows per pass (4 per lane)
constexpr int kPmSlice = 64;    // bytes of a row per stage

__host__ __device__ constexpr size_t pm_stage_bytes(int esz)
{
    return (size_t)kPmRP * kPmSlice + (size_t)kPmEC * (kPmSlice / esz) * 4;
}
__host__ __device__ constexpr size_t pm_score_smem(int esz)
{
    return (size_t)kPmWarps * 2 * pm_stage_bytes(esz);
}

// One item as a warp sees it: every lane holds the item's fields and, lane
// j < ne, traversal j's row index and first candidate slot.
struct PmItem {
    int hkv, par, ne, n_c;
    long long base;   // CSR: the first child entry; slot: the pool row of child 0
    long long bh;     // this lane's traversal
    int c0;           // its first candidate slot
};

template <typename T, int D>
__global__ void __launch_bounds__(kPmThreads, 3)
    pm_score_kernel(const __grid_constant__ DescendParams p0, const __grid_constant__ PmLevel pl, int L)
{
    constexpr int ESZ = (int)sizeof(T);
    constexpr int EV = Vec16<T>::E;             // elements per 16-byte piece
    constexpr int KE = kPmSlice / ESZ;          // elements of a row per stage
    constexpr int NKC = D / KE;                 // stages per pass
    constexpr int PPR = kPmSlice / 16;          // pieces per row slice (4)
    constexpr int EC = kPmEC, R = kPmRP / 32;
    constexpr int SB = (int)pm_stage_bytes(ESZ);
    static_assert(NKC >= 2 && PPR == 4 && R == 4, "layout");

    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ DescendParams p;
    griddep_launch();
    copy_params(p, p0);
    griddep_wait();
    __syncthreads();   // the only CTA barrier: the warps are independent from here on

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *wsm = smem_raw + (size_t)warp * 2 * SB;
    const uint32_t wsm_s = (uint32_t)__cvta_generic_to_shared(wsm);

    const int BG = p.B * p.G;
    const int Kp = L == 0 ? 1 : p.K[L - 1];
    const int fo = p.fanout[L];
    const long long prow = L == 0 ? 1 : p.rows[L - 1], rows = p.rows[L];
    const T *kbase = reinterpret_cast<const T *>(p.keys[L]);
    const float *s_ws = p.s_ws;
    float *f_ws = p.f_ws;
    const int fstride = p.fstride;
    const int32_t *coff = L >= 1 ? p.coff[L - 1] : nullptr;
    const int32_t *cid = L >= 1 ? p.cid[L - 1] : nullptr;
    const int32_t *tab = L >= 1 ? p.child[L - 1] : nullptr;
    const int32_t *slot = L >= 1 ? p.slot[L] : nullptr;
    const int per_hkv = (BG + EC - 1) / EC;
    const int n_items = L == 0 ? p.H_kv * per_hkv : min(pl.ctr[1], pl.max_items);
    const int gw = blockIdx.x * kPmWarps + warp, nw = gridDim.x * kPmWarps;
    if (gw >= n_items) return;

    auto load_item = [&](int item) {
        PmItem m;
        if (L == 0) {
            m.hkv = item / per_hkv;
            const int e0 = (item - m.hkv * per_hkv) * EC;
            m.par = 0;
            m.ne = min(EC, BG - e0);
            m.n_c = (int)rows;
            m.base = 0;
            const int i = e0 + (lane < m.ne ? lane : 0);
            const int b = i / p.G;
            m.bh = (long long)b * p.H + (long long)m.hkv * p.G + (i - b * p.G);
            m.c0 = 0;
        } else {
            const int4 it = pl.ctab[item];
            m.hkv = (int)(it.x / prow);
            m.par = (int)(it.x - (long long)m.hkv * prow);
            m.ne = min(it.z, EC);
            const int e = pl.list[it.y + (lane < m.ne ? lane : 0)];
            m.bh = e / Kp;
            const int k = e - (int)m.bh * Kp;
            m.c0 = pl.cpre ? pl.cpre[m.bh * (Kp + 1) + k] : k * fo;
            if (coff) {
                const int32_t *off_h = coff + (size_t)m.hkv * (prow + 1);
                m.base = off_h[m.par];
                m.n_c = off_h[m.par + 1] - (int)m.base;
            } else {
                m.n_c = fo;
                // any staged copy of the block will do: the first traversal's
                m.base = slot ? (long long)__shfl_sync(0xffffffffu, slot[e], 0) * fo : 0;
            }
        }
        return m;
    };
    // key row of child j of item m
    auto row_of = [&](const PmItem &m, int j) -> int {
        if (L == 0) return (int)((long long)m.hkv * rows + j);
        if (slot) return (int)(m.base + j);
        long long id;
        if (coff) {
            const long long e = m.base + j;
            id = cid ? (long long)cid[(size_t)m.hkv * rows + e] : e;
        } else {
            id = tab ? (long long)tab[((size_t)m.hkv * prow + m.par) * fo + j] : (long long)m.par * fo + j;
        }
        if (id < 0 || id >= rows) {
            set_status(p.status, kDevBadChild);
            id = 0;
        }
        return (int)((long long)m.hkv * rows + id);
    };
    // stage: slice kc of rows [q0, q0 + 128) of item m (row ids rid[j] of
    // rows q0 + lane + 32 j) and of its token sums, into buffer b
    auto issue = [&](const PmItem &m, int q0, int kc, const int (&rid)[R], int b) {
        const uint32_t dst = wsm_s + (uint32_t)(b * SB);
#pragma unroll
        for (int i = 0; i < 16; ++i) {   // 512 pieces: row (lane >> 2) + 8 i, piece lane & 3
            const int row = (lane >> 2) + 8 * i, pc = lane & 3;
            const int rr = __shfl_sync(0xffffffffu, rid[i >> 2], row & 31);
            const bool ok = q0 + row < m.n_c;
            const T *src = kbase + (size_t)(ok ? rr : 0) * D + kc * KE + pc * EV;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(
                             dst + (uint32_t)(row * kPmSlice + ((pc ^ ((row >> 1) & 3)) << 4))),
                         "l"(src), "r"(ok ? 16 : 0));
        }
        constexpr int SP = KE / 4;   // 16-byte pieces of a traversal's slice
        const uint32_t sdst = dst + kPmRP * kPmSlice;
#pragma unroll
        for (int i = 0; i < (EC * SP + 31) / 32; ++i) {
            const int q = lane + 32 * i;
            const int e = min(q / SP, m.ne - 1), v = q - (q / SP) * SP;
            const long long bhe = __shfl_sync(0xffffffffu, m.bh, e);
            if (q < m.ne * SP)
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sdst + (uint32_t)(e * KE + v * 4) * 4),
                             "l"(s_ws + (size_t)bhe * D + kc * KE + v * 4));
        }
    };
    auto row_ids = [&](const PmItem &m, int q0, int (&rid)[R]) {
#pragma unroll
        for (int j = 0; j < R; ++j) {
            const int row = q0 + lane + 32 * j;
            rid[j] = row < m.n_c ? row_of(m, row) : 0;
        }
    };

    // issue side (one stage ahead) and compute side
    int i_item = gw, i_q0 = 0, i_kc = 0;
    PmItem ii = load_item(gw);
    int pf_item = gw + nw;
    PmItem pf = ii;
    if (pf_item < n_items) pf = load_item(pf_item);
    int rid[R];
    row_ids(ii, 0, rid);
    issue(ii, 0, 0, rid, 0);
    asm volatile("cp.async.commit_group;\n" ::);
    bool i_done = false;
    PmItem ci = ii;
    int c_item = gw, c_q0 = 0, c_kc = 0;
    uint64_t acc[R][EC];
    for (int t = 0;; ++t) {
        // the issue side moves one stage on and loads it
        if (!i_done) {
            if (++i_kc == NKC) {
                i_kc = 0;
                i_q0 += kPmRP;
                if (i_q0 >= ii.n_c) {
                    i_q0 = 0;
                    i_item = pf_item;
                    if (i_item < n_items) {
                        ii = pf;
                        pf_item += nw;
                        if (pf_item < n_items) pf = load_item(pf_item);
                    } else {
                        i_done = true;
                    }
                }
                if (!i_done) row_ids(ii, i_q0, rid);
            }
            if (!i_done) issue(ii, i_q0, i_kc, rid, (t + 1) & 1);
        }
        asm volatile("cp.async.commit_group;\n" ::);
        asm volatile("cp.async.wait_group 1;\n" ::);
        __syncwarp();   // stage t landed for every lane
        if (c_kc == 0) {
#pragma unroll
            for (int j = 0; j < R; ++j)
#pragma unroll
                for (int h = 0; h < EC; ++h) acc[j][h] = 0;
        }
        {
            const uint8_t *st = wsm + (size_t)(t & 1) * SB;
            const float *ss = reinterpret_cast<const float *>(st + kPmRP * kPmSlice);
#pragma unroll
            for (int pc = 0; pc < PPR; ++pc) {
                uint64_t xp[R][EV / 2];
#pragma unroll
                for (int j = 0; j < R; ++j) {
                    const int row = lane + 32 * j;
                    Pairs16<T>::get(*reinterpret_cast<const uint4 *>(st + row * kPmSlice + ((pc ^ ((row >> 1) & 3)) << 4)),
                                    xp[j]);
                }
#pragma unroll
                for (int h = 0; h < EC; ++h) {
                    if (h < ci.ne) {
                        const uint64_t *sp = reinterpret_cast<const uint64_t *>(ss + h * KE + pc * EV);
                        uint64_t sv[EV / 2];
#pragma unroll
                        for (int e = 0; e < EV / 2; e += 2) {
                            const ulonglong2 w = *reinterpret_cast<const ulonglong2 *>(sp + e);
                            sv[e] = w.x;
                            sv[e + 1] = w.y;
                        }
#pragma unroll
                        for (int j = 0; j < R; ++j)
#pragma unroll
                            for (int e = 0; e < EV / 2; ++e) acc[j][h] = ffma2(sv[e], xp[j][e], acc[j][h]);
                    }
                }
            }
        }
        if (c_kc == NKC - 1) {
#pragma unroll
            for (int h = 0; h < EC; ++h) {
                const long long bhh = __shfl_sync(0xffffffffu, ci.bh, h);
                const int c0h = __shfl_sync(0xffffffffu, ci.c0, h);
                if (h < ci.ne) {
                    float *dst = f_ws + (size_t)bhh * fstride + c0h + c_q0;
#pragma unroll
                    for (int j = 0; j < R; ++j) {
                        const int row = lane + 32 * j;
                        if (c_q0 + row < ci.n_c) dst[row] = sum2(acc[j][h]);
                    }
                }
            }
        }
        __syncwarp();   // buffer t & 1 is free for stage t + 2
        // the compute side moves one stage on
        if (++c_kc == NKC) {
            c_kc = 0;
            c_q0 += kPmRP;
            if (c_q0 >= ci.n_c) {
                c_q0 = 0;
                c_item += nw;
                if (c_item >= n_items) break;
                ci = ii;   // the issue side is on this item's second stage (NKC >= 2)
            }
        }
    }
    asm volatile("cp.async.wait_group 0;\n" ::);
}

// ---------------------------------------------------------------------------
// Selection: one warp per traversal, nsel warps per CTA, each with pw bytes of
// shared memory: the selection scratch and score copy, the kept parents and
// (CSR) their candidate prefix.  With nx.cnt set, the warp then counts its
// kept entries per key for the next level (nx) and, on a CSR next level,
// writes their candidate prefix.
__host__ __device__ constexpr size_t pm_select_warp_bytes(int kcap, int Kpmax)
{
    return (warp_sel_bytes(kcap, 0) + (size_t)kCollectCap * 8 + (size_t)(2 * Kpmax + 2) * 4 + 15) & ~size_t(15);
}

// Counts traversal bh's kept entries of level L per key of the next level's
// inversion nx (and, on a CSR next level, their candidate prefix).  One warp.
__device__ __forceinline__ void pm_count_next(const DescendParams &p, const PmLevel &nx, int L, long long bh)
{
    const int lane = threadIdx.x & 31;
    const int hkv = (int)(bh % p.H) / p.G;
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

// Selections the fp32 band left open (queued by pm_select_kernel): one warp
// per queued traversal runs the refinement, writes the kept list and counts
// it for the next level.  Rare, and register-hungry (exact arithmetic), so it
// is kept out of the selection kernel.  Shared memory: per warp the kept
// parents' candidate prefix (CSR), Kpmax + 1 ints.
template <typename T, int D>
__global__ void __launch_bounds__(kSelThreads, 1)
    pm_refine_kernel(const __grid_constant__ DescendParams p0, const __grid_constant__ PmLevel self,
                     const __grid_constant__ PmLevel nx, int L)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ DescendParams p;
    griddep_launch();
    copy_params(p, p0);
    griddep_wait();
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    constexpr int NW = kSelThreads / 32;
    int32_t *cpre = reinterpret_cast<int32_t *>(smem_raw) + warp * (p.Kpmax + 1);
    const int nq = *self.qcount;
    const int K = p.K[L];
    const int Kp = L == 0 ? 0 : p.K[L - 1];
    const bool csr = L >= 1 && p.coff[L - 1] != nullptr;
    for (int i = blockIdx.x * NW + warp; i < nq; i += gridDim.x * NW) {
        const int4 q = self.queue[i];
        const long long bh = q.x;
        if (csr) {
            const int hkv = (int)(bh % p.H) / p.G;
            const int32_t *off_h = p.coff[L - 1] + (size_t)hkv * (p.rows[L - 1] + 1);
            const int32_t *prev = p.kept[L - 1] + bh * Kp;
            warp_prefix_counts(Kp, [&](int k) { return off_h[prev[k] + 1] - off_h[prev[k]]; }, cpre);
        }
        const LevelView lv = level_view(p, L, bh, csr ? cpre : nullptr);
        uint64_t *kbuf = reinterpret_cast<uint64_t *>(p.f_ws + (size_t)bh * p.fstride + p.cap);
        const int *list = reinterpret_cast<const int *>(p.f_ws + (size_t)bh * p.fstride);
        ExactScratch xs(p.xs_ws + (size_t)bh * ExactScratch::bytes());
        warp_refine<T, D>(p, lv, L, bh, kbuf, q.y, list, q.z, q.w != 0, xs);
        __syncwarp();
        write_kept(p, lv, L, bh, kbuf, K);
        if (nx.cnt) pm_count_next(p, nx, L, bh);
        __syncwarp();
    }
}

// MINB: CTAs per SM the registers are budgeted for (2: 128 registers, the
// fastest per warp; 3: 80, more warps resident when the traversals exceed one
// wave).
template <typename T, int D, int MINB>
__global__ void __launch_bounds__(kSelThreads, MINB)
    pm_select_kernel(const __grid_constant__ DescendParams p0, const __grid_constant__ PmLevel self,
                     const __grid_constant__ PmLevel nx, int L, int nsel, int pw)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ DescendParams p;
    griddep_launch();
    copy_params(p, p0);
    griddep_wait();
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
    uint64_t *col = reinterpret_cast<uint64_t *>(ws + warp_sel_bytes(p.kcap, 0));
    int32_t *prev = reinterpret_cast<int32_t *>(ws + warp_sel_bytes(p.kcap, 0) + (size_t)kCollectCap * 8);
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
    const bool done = warp_select_pm<T, D>(p, L, bh, csr ? cpre : nullptr, L == 0 ? nullptr : prev, hist, tmp, kbuf,
                                           col, xs, self.queue, self.qcount);
    __syncwarp();
    if (done && nx.cnt) pm_count_next(p, nx, L, bh);
    (void)lane;
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
    griddep_launch();
    griddep_wait();
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
    if (warp == 0) {
        // publish this tile's aggregate, then look back over the predecessors
        // 32 at a time: sum aggregates down to the nearest published prefix
        unsigned long long pre = 0;
        if (tile == 0) {
            if (lane == 0) {
                pl.tval[1] = agg;
                st_release(pl.tflag, 2);
            }
        } else {
            if (lane == 0) {
                pl.tval[2 * tile] = agg;
                st_release(pl.tflag + tile, 1);
            }
            int j = tile - 1, spins = 0;
            while (j >= 0) {
                const int idx = j - lane;
                const int f = idx >= 0 ? ld_acquire(pl.tflag + idx) : 2;
                if (__any_sync(0xffffffffu, f == 0)) {
                    if (++spins > kScanSpinLimit) {
                        if (lane == 0) set_status(status, kDevTimeout);
                        break;
                    }
                    continue;
                }
                const unsigned inc = __ballot_sync(0xffffffffu, f == 2);
                const int first = inc ? __ffs(inc) - 1 : 32;   // the nearest published prefix
                unsigned long long v = 0;
                if (idx >= 0 && lane < first) v = pl.tval[2 * idx];
                if (idx >= 0 && lane == first) v = pl.tval[2 * idx + 1];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                pre += v;
                if (inc) break;
                j -= 32;
            }
            if (lane == 0) {
                pl.tval[2 * tile + 1] = pre + agg;
                st_release(pl.tflag + tile, 2);
            }
        }
        if (lane == 0) {
            pre_sh = pre;
            if (tile == pl.n_tiles - 1) pl.ctr[1] = (int)((pre + agg) >> 32);
        }
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
    griddep_launch();
    griddep_wait();
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
