// Host staging: bring the key blocks of the kept parents (the mid blocks of the
// kept roots when the mid level lives in host memory, the leaf blocks of the
// kept mids), and later the kept leaves' value rows, from pinned host memory
// into HBM.
//
// "AtlasKV: Augmenting LLMs with Billion-Scale Knowledge Graphs in 20GB VRAM",
// section "Quick read / How it works": only the root keys need to stay on the
// GPU; after each level's pruning the next level's keys are loaded from CPU
// memory.  Section "Quick read / Results" names the cost: CPU-GPU movement
// between levels adds I/O latency.  So every block crosses the host link once
// per query: the G query heads of a query share one staged copy.
#pragma once

#include "common.cuh"

namespace akv {

constexpr int kDedupeThreads = 256;

// Per group q (one query and one KV head: the kept lists of its G query heads
// are contiguous): the n ids ids[q*n .. q*n+n) -> unique ids
// uniq[q*n .. q*n+count[q]) in ascending order, and slot[q*n + i] = q*n + rank
// of ids[q*n+i] among them.  Dynamic shared memory: n2 (power of two >= n)
// uint64 + n2 int32.
__global__ void __launch_bounds__(kDedupeThreads) dedupe_kernel(const int32_t *__restrict__ ids, int n, int n2,
                                                                 int32_t *uniq, int32_t *slot, int32_t *count)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint64_t *buf = reinterpret_cast<uint64_t *>(smem_raw);
    int32_t *flag = reinterpret_cast<int32_t *>(buf + n2);   // [n2] inclusive scan of "first of a run"
    const int b = blockIdx.x;   // group q
    const int32_t *src = ids + (size_t)b * n;
    for (int i = threadIdx.x; i < n2; i += blockDim.x)
        buf[i] = i < n ? ((uint64_t)(uint32_t)src[i] << 32) | (uint32_t)i : ~0ull;
    // bitonic sort ascending
    for (int size = 2; size <= n2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncthreads();
            for (int i = threadIdx.x; i < n2 / 2; i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool asc = (lo & size) == 0;
                const uint64_t x = buf[lo], y = buf[hi];
                if ((x > y) == asc) {
                    buf[lo] = y;
                    buf[hi] = x;
                }
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n2; i += blockDim.x)
        flag[i] = (i < n && (i == 0 || (buf[i] >> 32) != (buf[i - 1] >> 32))) ? 1 : 0;
    __syncthreads();
    // inclusive scan of flag: each thread scans a contiguous segment, then
    // the per-thread totals are scanned by warp 0
    __shared__ int seg_tot[kDedupeThreads];
    const int seg = (n2 + blockDim.x - 1) / blockDim.x;
    const int s0 = threadIdx.x * seg, s1 = min(n2, s0 + seg);
    int run = 0;
    for (int i = s0; i < s1; ++i) {
        run += flag[i];
        flag[i] = run;
    }
    seg_tot[threadIdx.x] = run;
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int t = 0; t < (int)blockDim.x; ++t) {
            const int v = seg_tot[t];
            seg_tot[t] = acc;
            acc += v;
        }
    }
    __syncthreads();
    for (int i = s0; i < s1; ++i) flag[i] += seg_tot[threadIdx.x];
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int u = flag[i] - 1;
        const int32_t id = (int32_t)(buf[i] >> 32);
        const int orig = (int)(buf[i] & 0xffffffffu);
        slot[(size_t)b * n + orig] = b * n + u;
        if (i == 0 || (buf[i] >> 32) != (buf[i - 1] >> 32)) uniq[(size_t)b * n + u] = id;
    }
    if (threadIdx.x == 0) count[b] = flag[n - 1];
}

// Copies from mapped host memory cross the host link with long latency, so
// every warp keeps kStageUnroll row groups in flight: a row is D e / 16
// lanes' 16-byte vectors and a warp instruction covers 32 / that rows; all
// loads of an iteration are issued before its stores.  A small grid (two CTAs
// per SM) then fills the link while leaving the SMs to the descent and the
// attention of the other query chunks running beside it.
constexpr int kStageUnroll = 4;
constexpr int kStageCtasPerSm = 2;

// Copy the b_c child-key rows of every unique kept parent of every group into
// the key pool: pool row (q*n + u) * b_c + j <- host child row child(parent, j)
// of KV head q % H_kv, with child() the level's table (or parent * b_c + j).
// Used for the leaf blocks of kept mids and the mid blocks of kept roots.
// With a leaf-block cache (cache non-null): block blk is read from cache slot
// csrc[blk] when that is >= 0 (HBM) instead of host memory, and also written
// to cache slot cfill[blk] when that is >= 0.
template <typename T, int D>
__global__ void __launch_bounds__(256) stage_blocks_kernel(
    const T *__restrict__ host_child_keys, const int32_t *__restrict__ child_tab, long long n_parent,
    long long n_child, int b_child, int H_kv, const int32_t *__restrict__ uniq, const int32_t *__restrict__ count,
    int n, int n_groups, T *pool, int *status, T *cache, const int32_t *__restrict__ csrc,
    const int32_t *__restrict__ cfill)
{
    constexpr int VPR = D * (int)sizeof(T) / 16;   // 16-byte vectors per row = lanes per row
    constexpr int RPI = 32 / VPR;                  // rows per warp instruction
    const int lane = threadIdx.x & 31, sub = lane % VPR, rsel = lane / VPR;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    const long long total = (long long)n_groups * n * b_child;
    for (long long r0 = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * (RPI * kStageUnroll);
         r0 < total; r0 += warps * RPI * kStageUnroll) {
        uint4 buf[kStageUnroll];
        uint4 *dst[kStageUnroll], *dst2[kStageUnroll];
#pragma unroll
        for (int k = 0; k < kStageUnroll; ++k) {
            const long long w = r0 + (long long)k * RPI + rsel;
            dst[k] = dst2[k] = nullptr;
            if (w < total) {
                const long long blk = w / b_child;
                const int j = (int)(w - blk * b_child);
                const int b = (int)(blk / n);
                const int u = (int)(blk - (long long)b * n);
                if (u < count[b]) {
                    const int hkv = b % H_kv;   // group b = query * H_kv + hkv
                    const int from = cache ? csrc[blk] : -1;
                    if (from >= 0) {   // a cached block: copied within HBM
                        buf[k] = reinterpret_cast<const uint4 *>(cache + ((size_t)from * b_child + j) * D)[sub];
                        dst[k] = reinterpret_cast<uint4 *>(pool + ((size_t)blk * b_child + j) * D) + sub;
                    } else {
                        const long long par = uniq[blk];
                        const long long ch = child_tab
                                                 ? (long long)child_tab[((size_t)hkv * n_parent + par) * b_child + j]
                                                 : par * b_child + j;
                        if (ch < 0 || ch >= n_child) {
                            set_status(status, kDevBadChild);
                        } else {
                            buf[k] =
                                reinterpret_cast<const uint4 *>(host_child_keys + ((size_t)hkv * n_child + ch) * D)[sub];
                            dst[k] = reinterpret_cast<uint4 *>(pool + ((size_t)blk * b_child + j) * D) + sub;
                            const int to = cache ? cfill[blk] : -1;
                            if (to >= 0) dst2[k] = reinterpret_cast<uint4 *>(cache + ((size_t)to * b_child + j) * D) + sub;
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int k = 0; k < kStageUnroll; ++k) {
            if (dst[k]) *dst[k] = buf[k];
            if (dst2[k]) *dst2[k] = buf[k];
        }
    }
}

// ---------------------------------------------------------------------------
// HBM cache of staged leaf blocks across calls, keyed by the kept mid
// ("Quick read / Results": the CPU-GPU movement between levels is the I/O
// cost; blocks of branches that recur need not cross the host link again).
// Set-associative: kCacheWays ways per set, least recently used way evicted.
// A way is one 64-bit word: call epoch (high 32 bits) | pending (bit 31) |
// key + 1 (bits 0..30, key = hkv rows_mid + mid; 0 = empty).  Claiming a
// victim and pinning a hit are single compare-and-swaps on that word, so a
// way cannot change owner between the check and the use.  A way claimed in
// this call stays pending until its block has been staged (cache_commit):
// other groups wanting the same block meanwhile read it from host memory.
// Ways stamped with the current epoch are never evicted in this call.
constexpr int kCacheWays = 8;
constexpr uint32_t kCachePending = 0x80000000u;
constexpr int kCacheAttempts = 16;

__device__ __forceinline__ uint32_t cache_hash(uint32_t key)
{
    uint32_t h = key * 0x9E3779B1u;
    return h ^ (h >> 15);
}

// One thread per unique block of the chunk: csrc[blk] = cache slot holding it
// (a hit), or -1; cfill[blk] = cache slot to fill while staging it (a miss
// that claimed a way), or -1.  stats: hits, fills, bypasses.
__global__ void cache_map_kernel(const int32_t *__restrict__ uniq, const int32_t *__restrict__ count, int n,
                                 int n_groups, int H_kv, long long rows_mid, unsigned long long *tag, long long n_sets,
                                 uint32_t epoch, int32_t *csrc, int32_t *cfill, unsigned long long *stats)
{
    const long long total = (long long)n_groups * n;
    for (long long blk = (long long)blockIdx.x * blockDim.x + threadIdx.x; blk < total;
         blk += (long long)gridDim.x * blockDim.x) {
        const int b = (int)(blk / n);
        const int u = (int)(blk - (long long)b * n);
        if (u >= count[b]) continue;
        const uint32_t key = (uint32_t)((long long)(b % H_kv) * rows_mid + uniq[blk]);
        const uint32_t kw = key + 1u;
        const long long set = (long long)(cache_hash(key) & (uint32_t)(n_sets - 1));
        unsigned long long *ways = tag + set * kCacheWays;
        int src = -1, fill = -1, kind = 2;   // 0 hit, 1 fill, 2 bypass
        for (int attempt = 0; attempt < kCacheAttempts; ++attempt) {
            unsigned long long w[kCacheWays];
#pragma unroll
            for (int i = 0; i < kCacheWays; ++i) w[i] = atomicAdd(ways + i, 0ull);
            int hit = -1, victim = -1;
            uint32_t oldest = 0xffffffffu;
#pragma unroll
            for (int i = 0; i < kCacheWays; ++i) {
                const uint32_t lo = (uint32_t)w[i], stamp = (uint32_t)(w[i] >> 32);
                if ((lo & ~kCachePending) == kw && hit < 0) hit = i;
                if (stamp != epoch && stamp < oldest) {
                    oldest = stamp;
                    victim = i;
                }
            }
            if (hit >= 0) {
                const uint32_t lo = (uint32_t)w[hit], stamp = (uint32_t)(w[hit] >> 32);
                if (lo & kCachePending) break;   // being filled in this call: bypass
                if (stamp == epoch) {            // pinned already
                    src = (int)(set * kCacheWays + hit);
                    kind = 0;
                    break;
                }
                const unsigned long long want = ((unsigned long long)epoch << 32) | kw;
                if (atomicCAS(ways + hit, w[hit], want) == w[hit]) {
                    src = (int)(set * kCacheWays + hit);
                    kind = 0;
                    break;
                }
                continue;   // the way changed: look again
            }
            if (victim < 0) break;   // every way holds a block of this call: bypass
            const unsigned long long want = ((unsigned long long)epoch << 32) | kCachePending | kw;
            if (atomicCAS(ways + victim, w[victim], want) == w[victim]) {
                fill = (int)(set * kCacheWays + victim);
                kind = 1;
                break;
            }
        }
        csrc[blk] = src;
        cfill[blk] = fill;
        if (stats) atomicAdd(stats + kind, 1ull);
    }
}

// After the chunk's staging: the ways it filled are no longer pending.
__global__ void cache_commit_kernel(const int32_t *__restrict__ count, int n, int n_groups,
                                    const int32_t *__restrict__ cfill, unsigned long long *tag)
{
    const long long total = (long long)n_groups * n;
    for (long long blk = (long long)blockIdx.x * blockDim.x + threadIdx.x; blk < total;
         blk += (long long)gridDim.x * blockDim.x) {
        const int b = (int)(blk / n);
        const int u = (int)(blk - (long long)b * n);
        if (u < count[b] && cfill[blk] >= 0) atomicAnd(tag + cfill[blk], ~(unsigned long long)kCachePending);
    }
}

// Copy value rows: vpool row (q*n + u) <- host leaf value row uniq[q*n + u]
// of KV head q % H_kv.
template <typename T, int D>
__global__ void __launch_bounds__(256) stage_value_rows_kernel(const T *__restrict__ host_leaf_values, long long n_leaf,
                                                               int H_kv, const int32_t *__restrict__ uniq,
                                                               const int32_t *__restrict__ count, int n, int n_groups,
                                                               T *vpool)
{
    constexpr int VPR = D * (int)sizeof(T) / 16;
    constexpr int RPI = 32 / VPR;
    const int lane = threadIdx.x & 31, sub = lane % VPR, rsel = lane / VPR;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    const long long total = (long long)n_groups * n;
    for (long long r0 = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * (RPI * kStageUnroll);
         r0 < total; r0 += warps * RPI * kStageUnroll) {
        uint4 buf[kStageUnroll];
        uint4 *dst[kStageUnroll];
#pragma unroll
        for (int k = 0; k < kStageUnroll; ++k) {
            const long long w = r0 + (long long)k * RPI + rsel;
            dst[k] = nullptr;
            if (w < total) {
                const int b = (int)(w / n);
                const int u = (int)(w - (long long)b * n);
                if (u < count[b]) {
                    const int hkv = b % H_kv;
                    const long long leaf = uniq[w];
                    buf[k] = reinterpret_cast<const uint4 *>(host_leaf_values + ((size_t)hkv * n_leaf + leaf) * D)[sub];
                    dst[k] = reinterpret_cast<uint4 *>(vpool + (size_t)w * D) + sub;
                }
            }
        }
#pragma unroll
        for (int k = 0; k < kStageUnroll; ++k)
            if (dst[k]) *dst[k] = buf[k];
    }
}

}  // namespace akv
