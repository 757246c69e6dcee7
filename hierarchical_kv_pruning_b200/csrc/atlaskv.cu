// C ABI of the HiKVP knowledge-graph attention library (see include/atlaskv.h).
//
// Host side: argument validation, workspace planning and kernel launches.  All
// device work of atlaskv_attend runs in the kernels of descend.cuh,
// staging.cuh and attend.cuh; nothing here computes on the host.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <string>
#include <utility>

#include "atlaskv.h"
#include "attend.cuh"
#include "attend_tc.cuh"
#include "descend.cuh"
#include "descend_pm.cuh"
#include "internal.h"
#include "staging.cuh"

namespace {

thread_local std::string g_last_error;

atlaskv_status fail(atlaskv_status st, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

#define AKV_CUDA(call)                                                                                 \
    do {                                                                                               \
        cudaError_t e_ = (call);                                                                       \
        if (e_ != cudaSuccess) return fail(ATLASKV_ECUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
    } while (0)

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Raise a kernel's dynamic shared-memory limit to `bytes` once per (kernel,
// device): later calls configure nothing, so an attend call can be captured
// into a CUDA graph after a first, uncaptured one.  (The default limit leaves
// 48 KB for static and dynamic shared memory together, so any dynamic size is
// set explicitly.)
atlaskv_status ensure_smem(const void *kernel, size_t bytes)
{
    if (bytes == 0) return ATLASKV_OK;
    int dev = 0;
    AKV_CUDA(cudaGetDevice(&dev));
    static std::mutex m;
    static std::map<std::pair<const void *, int>, size_t> done;
    std::lock_guard<std::mutex> lock(m);
    size_t &have = done[{kernel, dev}];
    if (have >= bytes) return ATLASKV_OK;
    AKV_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
    have = bytes;
    return ATLASKV_OK;
}
#define AKV_SMEM(kernel, bytes)                                                                   \
    do {                                                                                          \
        atlaskv_status e_ = ensure_smem(reinterpret_cast<const void *>(kernel), (size_t)(bytes)); \
        if (e_ != ATLASKV_OK) return e_;                                                          \
    } while (0)

int pow2_at_least(long long x, int floor_)
{
    int p = floor_;
    while (p < x) p <<= 1;
    return p;
}

constexpr int kMaxCandidates = 8192;   // per level and traversal (shared-memory bound of the descent CTA)
constexpr int kNumCounters = 4 * akv::kMaxLevels;   // descent counters: 4 per level
constexpr int kNumEvents = 6;   // descent begin / end, sequence part begin / end, leaf part begin / end
// Host-resident leaves: the batch is split into up to kMaxChunks query chunks
// so that staging one chunk's leaf blocks over the host link overlaps the
// scoring and attention of the others (a second stream owned by the tree).
constexpr int kMaxChunks = 4;
constexpr int kChunkEvents = 6;          // per chunk: one per pipeline phase that hands over to the other stream
int query_chunks(int B) { return B >= 2 * kMaxChunks ? kMaxChunks : 1; }
constexpr int kPhases = 7;               // per chunk at most: 3 descent ranges, 3 stagings, the knowledge part
constexpr int kTimingEvents = 2 * kPhases;   // per chunk: begin / end of each phase

enum : int { kPhaseDescend = 0, kPhaseStageKeys = 1, kPhaseStageValues = 2, kPhaseAttend = 3 };

// Kept counts of a call, one per level (roots first), and the logit scale.
struct Ks {
    int n;
    int K[akv::kMaxLevels];
    float scale;
};

Ks ks_of(const atlaskv_params *p)
{
    Ks k{};
    k.n = 3;
    k.K[0] = p->K_root;
    k.K[1] = p->K_mid;
    k.K[2] = p->K_leaf;
    k.scale = p->scale;
    return k;
}
struct Phase {
    int kind, first, last;   // kind; descent: level range; key staging: the level staged
};

}  // namespace

atlaskv_status akv_report(atlaskv_status st, const char *msg)
{
    g_last_error = msg;
    return st;
}

struct atlaskv_tree {
    atlaskv_tree_desc d;
    int n_levels;                  // 3 for a uniform tree, 2 .. 4 for a CSR tree
    long long rows[akv::kMaxLevels];
    const void *lkeys[akv::kMaxLevels];      // device-accessible keys of each level
    int min_ch[akv::kMaxLevels - 1], max_ch[akv::kMaxLevels - 1];   // children per node of level l
    bool csr;
    const int32_t *coff[akv::kMaxLevels - 1], *cid[akv::kMaxLevels - 1];   // CSR child lists
    const void *leaf_keys_dev;     // device-accessible leaf pointers (mapped for host leaves)
    const void *leaf_values_dev;
    const void *mid_keys_dev;      // device-accessible mid pointer (mapped for host mids)
    bool host_leaves, host_mids;
    float *norm_bound;             // device [3][H_kv]
    int *status;                   // device sticky status word
    unsigned long long *stats;     // device [kMaxLevels][4] descent counters (kept while counting)
    bool profiling;                // stage events recorded (ATLASKV_PROFILE_TIMES)
    bool counting;                 // descent counters kept (ATLASKV_PROFILE_COUNTERS)
    bool timed;                    // the last attend recorded events
    bool counted;                  // the last attend kept descent counters
    bool split;                    // bf16, D = 128: the sequence part runs on its own stream beside the descent
    bool host_mode_last;
    int chunks_last;
    int num_sms;                   // of the device the tree was created on (grid sizing only)
    cudaEvent_t ev[kNumEvents];
    cudaStream_t stage_stream;                        // host leaves: staging copies
    cudaStream_t seq_stream;                          // split: sequence part (lowest priority)
    cudaStream_t desc_stream;                         // split, HBM leaves: descent (highest priority)
    cudaEvent_t fev[3];                               // split: fork, descent done, sequence part done
    cudaEvent_t cev[kMaxChunks * kChunkEvents + 1];   // cross-stream ordering (+1: start)
    cudaEvent_t tev[kMaxChunks * kTimingEvents];      // segment timing while profiling
    Phase phase[kPhases];                             // host path: the per-chunk pipeline of the last call
    int nphases_last;
    int descent_mode;                                 // ATLASKV_DESCENT_*
    bool pm_last;                                     // the last attend ran the parent-major descent
    // HBM cache of staged leaf blocks (host leaves; atlaskv_set_leaf_cache)
    unsigned long long *cache_tag;                    // [sets * kCacheWays] way words
    void *cache_pool;                                 // [sets * kCacheWays][b_L][D]
    long long cache_sets;
    uint32_t cache_epoch;                             // calls that used the cache
    unsigned long long *cache_stats;                  // [3] hits, fills, bypasses (cumulative)
};

namespace {

size_t esize(int dtype) { return dtype == ATLASKV_F32 ? 4 : 2; }

// ---- descent launch -------------------------------------------------------
// One CTA per (query, KV head, chunk of GC heads) runs levels first..last of
// the descent.  GC: the largest divisor of G up to 32 whose shared-memory plan
// fits; a warp scores HT heads (GC rounded up to a power of two, at most 8).
struct DescPlan {
    int GC = 0, HT = 0, nsel = 0;
    size_t smem = 0;
};

// The largest kept count of a level that has children.
int kp_max(const Ks &k)
{
    int m = 1;
    for (int l = 0; l + 1 < k.n; ++l) m = std::max(m, k.K[l]);
    return m;
}

int k_max(const Ks &k)
{
    int m = 1;
    for (int l = 0; l < k.n; ++l) m = std::max(m, k.K[l]);
    return m;
}

DescPlan plan_descent(int G, const Ks &ks, int kcap, int cap, int D, int esz, long long groups, int num_sms)
{
    // the largest head chunk whose plan fits; smaller chunks (more CTAs, each
    // key row fetched once per chunk, the repeats from L2) while the grid
    // would leave SMs idle
    DescPlan dp;
    for (int c = std::min(G, 32); c >= 1; --c) {
        if (G % c) continue;
        const akv::DescLayout lay(c, kp_max(ks), kcap, cap, D, esz);
        if (lay.total_bytes > 200 * 1024) continue;
        dp.GC = c;
        // heads per warp: GC rounded up to a power of two, but at least a
        // quarter of the lanes a key row spans (so a lane group holds at
        // most 4 rows of a chunk), at most 8
        const int lpg = D * esz / 16;
        dp.HT = std::min(8, std::max(lpg / 4, c <= 1 ? 1 : c <= 2 ? 2 : c <= 4 ? 4 : 8));
        dp.smem = lay.total_bytes;
        dp.nsel = lay.nsel;
        if (groups * (G / c) >= num_sms) break;
    }
    return dp;
}

// ---- parent-major descent plan ---------------------------------------------
// Traversals with at least this many (B H) take the parent-major descent in
// ATLASKV_DESCENT_AUTO; fewer run the fused kernel (one launch).  Measured on
// B200: 512 traversals (47x47x47, B 16) run faster fused, 2048 (100x100x100,
// B 64) faster parent-major.
constexpr long long kPmAutoMinTraversals = 1024;
constexpr size_t kPmSelBudget = 56 * 1024;   // selection CTA's shared memory (several CTAs per SM)

struct PmPlan {
    bool ok = false;               // supported for this call
    int EC = 0;                    // traversals per scoring work item
    int nsel = 0, pw = 0;          // selection: warps per CTA, shared bytes per warp
    int ts_GC = 0;                 // token sums: heads per CTA
    size_t ts_smem = 0;
    long long BHc = 0;             // traversals of the largest query chunk
    long long NK[akv::kMaxLevels] = {}, E[akv::kMaxLevels] = {};
    int items[akv::kMaxLevels] = {}, tiles[akv::kMaxLevels] = {};
    bool cpre = false;
    size_t zero_bytes = 0, data_bytes = 0;   // per query chunk
};

size_t r16(size_t b) { return (b + 15) & ~size_t(15); }

PmPlan plan_pm(const atlaskv_tree *t, const Ks &ks, long long Bc, int H, int kcap)
{
    PmPlan pp;
    const int D = t->d.head_dim;
    const int esz = (int)(t->d.dtype == ATLASKV_F32 ? 4 : 2);
    const int G = H / t->d.n_kv_heads;
    pp.EC = akv::kPmEC;
    const size_t pw = akv::pm_select_warp_bytes(kcap, kp_max(ks));
    if (pw > 200 * 1024) return pp;
    pp.pw = (int)pw;
    pp.nsel = (int)std::max<size_t>(1, std::min<size_t>(8, kPmSelBudget / pw));
    const int ev = 16 / esz;
    for (int c = G; c >= 1; --c)
        if (G % c == 0 && c * (D / ev) <= akv::kDescThreads) {
            pp.ts_GC = c;
            break;
        }
    pp.ts_smem = akv::token_sums_smem(pp.ts_GC, D, esz);
    pp.BHc = Bc * H;
    pp.cpre = t->csr;
    // refinement queues: a length per level, one queue of BH entries reused by the levels
    pp.zero_bytes = 16 * akv::kMaxLevels;
    pp.data_bytes = r16((size_t)pp.BHc * 16);
    for (int l = 0; l < ks.n; ++l)   // key rows of a level are addressed with 32-bit row numbers
        if ((long long)t->d.n_kv_heads * t->rows[l] > (1LL << 31) - 1) return pp;
    for (int l = 1; l < ks.n; ++l) {
        pp.NK[l] = (long long)t->d.n_kv_heads * t->rows[l - 1];
        pp.E[l] = pp.BHc * ks.K[l - 1];
        if (pp.NK[l] > (1LL << 31) - 1 || pp.E[l] + pp.E[l] / pp.EC + 1 > (1LL << 31) - 1) return pp;
        pp.items[l] = (int)(pp.E[l] + pp.E[l] / pp.EC + 1);
        pp.tiles[l] = (int)((pp.NK[l] + akv::kScanTile - 1) / akv::kScanTile);
        pp.zero_bytes += r16(pp.NK[l] * 4) + r16((size_t)pp.tiles[l] * 4) + 16;
        pp.data_bytes += r16(pp.NK[l] * 4) + 2 * r16(pp.E[l] * 4) + (size_t)pp.items[l] * 16 +
                         (size_t)pp.tiles[l] * 16 + (pp.cpre ? r16((size_t)pp.BHc * (ks.K[l - 1] + 1) * 4) : 0);
    }
    pp.ok = true;
    return pp;
}

// The per-level inversion structures of one query chunk of BH traversals
// (at most pp.BHc: the regions are sized for the largest chunk).
void pm_bind(const PmPlan &pp, int n_levels, long long BH, uint8_t *zero, uint8_t *data, akv::PmLevel *lv)
{
    for (int l = 0; l < akv::kMaxLevels; ++l) lv[l] = akv::PmLevel{};
    for (int l = 0; l < n_levels; ++l) {
        lv[l].qcount = reinterpret_cast<int32_t *>(zero + 16 * l);
        lv[l].queue = reinterpret_cast<int4 *>(data);
    }
    zero += 16 * akv::kMaxLevels;
    data += r16((size_t)pp.BHc * 16);
    for (int l = 1; l < n_levels; ++l) {
        akv::PmLevel &v = lv[l];
        const long long Kp = pp.E[l] / pp.BHc;
        v.NK = pp.NK[l];
        v.E = (int)(BH * Kp);
        v.max_items = pp.items[l];
        v.n_tiles = pp.tiles[l];
        v.cnt = reinterpret_cast<int32_t *>(zero);
        zero += r16(pp.NK[l] * 4);
        v.tflag = reinterpret_cast<int32_t *>(zero);
        zero += r16((size_t)pp.tiles[l] * 4);
        v.ctr = reinterpret_cast<int32_t *>(zero);
        zero += 16;
        v.eoff = reinterpret_cast<int32_t *>(data);
        data += r16(pp.NK[l] * 4);
        v.rank = reinterpret_cast<int32_t *>(data);
        data += r16(pp.E[l] * 4);
        v.list = reinterpret_cast<int32_t *>(data);
        data += r16(pp.E[l] * 4);
        v.ctab = reinterpret_cast<int4 *>(data);
        data += (size_t)pp.items[l] * 16;
        v.tval = reinterpret_cast<unsigned long long *>(data);
        data += (size_t)pp.tiles[l] * 16;
        v.cpre = nullptr;
        if (pp.cpre) {
            v.cpre = reinterpret_cast<int32_t *>(data);
            data += r16((size_t)pp.BHc * (Kp + 1) * 4);
        }
    }
}

struct Layout {
    size_t s_ws, s64_ws, a64_ws, anorm_ws, f_ws, xs, kept[akv::kMaxLevels], leaf_slot, kept_leaf_row, vslot, umid, ucount_mid,
        csrc, cfill,
        uleaf, ucount_leaf, key_pool, val_pool, oseq, lse_seq, mid_slot, uroot, ucount_root, mid_pool, total;
    int cap, kcap, fstride;
    DescPlan desc;
    bool pm;                       // the parent-major descent runs
    PmPlan pmp;
    size_t pm_zero, pm_data;       // the chunks' zero-initialised parts, then their other parts
    int pm_chunks;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Scores per traversal a level can need: every root, or the children of the
// kept parents (at most K[l-1] times the most children of a node), rounded up
// to a multiple of four.
int score_cap(const atlaskv_tree *t, const Ks &ks)
{
    long long cmax = t->rows[0];
    for (int l = 1; l < ks.n; ++l) cmax = std::max(cmax, (long long)ks.K[l - 1] * t->max_ch[l - 1]);
    return (int)((cmax + 3) & ~3LL);
}

// Which descent a call takes (the tree's mode; the automatic choice by size).
bool use_pm(const atlaskv_tree *t, bool pm_ok, bool fused_ok, long long BH)
{
    if (t->descent_mode == ATLASKV_DESCENT_FUSED) return false;
    if (t->descent_mode == ATLASKV_DESCENT_PARENT_MAJOR) return pm_ok;
    return pm_ok && (!fused_ok || BH >= kPmAutoMinTraversals);
}

Layout plan(const atlaskv_tree *t, const Ks &ks, int B, int N, int H, int T, bool allow_pm = true)
{
    (void)N;
    (void)T;
    Layout L{};
    const size_t BH = (size_t)B * H;
    const int D = t->d.head_dim;
    const bool host = t->host_leaves;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    L.cap = score_cap(t, ks);
    L.kcap = pow2_at_least(k_max(ks), 32);
    L.fstride = L.cap + 2 * L.kcap;
    L.s_ws = take(BH * D * 4);
    L.s64_ws = take(BH * D * 8);
    L.a64_ws = take(BH * D * 8);
    L.anorm_ws = take(BH * 4);
    L.f_ws = take(BH * (size_t)L.fstride * 4);
    const int G = H / t->d.n_kv_heads;
    // host leaves: the descent runs per query chunk, so its grid is a chunk's
    const int chunk_b = host ? (B + query_chunks(B) - 1) / query_chunks(B) : B;
    L.desc = plan_descent(G, ks, L.kcap, L.cap, D, (int)esize(t->d.dtype), (long long)chunk_b * t->d.n_kv_heads,
                          t->num_sms);
    const int gc = L.desc.GC > 0 ? L.desc.GC : 1;
    L.pmp = plan_pm(t, ks, chunk_b, H, L.kcap);
    L.pm = allow_pm && use_pm(t, L.pmp.ok, L.desc.GC > 0, (long long)B * H);
    // refinement scratch: one slot per selecting warp of every descent CTA
    // (parent-major: one per traversal)
    L.xs = take(L.pm ? BH * akv::ExactScratch::bytes()
                     : (size_t)B * t->d.n_kv_heads * (G / gc) * std::max(1, L.desc.nsel) * akv::ExactScratch::bytes());
    for (int l = 0; l < ks.n; ++l) L.kept[l] = take(BH * (size_t)ks.K[l] * 4);
    if (t->split) {   // the sequence part's normalised output and log-sum-exp, fp32
        L.oseq = take(BH * (size_t)N * D * 4);
        L.lse_seq = take(BH * (size_t)N * 4);
    }
    if (host) {
        const size_t groups = (size_t)B * t->d.n_kv_heads;
        const size_t n_mid = (size_t)G * ks.K[1], n_leaf = (size_t)G * ks.K[2];
        L.leaf_slot = take(BH * ks.K[1] * 4);
        L.kept_leaf_row = take(BH * ks.K[2] * 4);
        L.vslot = take(BH * ks.K[2] * 4);
        L.umid = take(groups * n_mid * 4);
        L.ucount_mid = take(groups * 4);
        L.csrc = take(groups * n_mid * 4);    // leaf-block cache map (used when the tree has a cache)
        L.cfill = take(groups * n_mid * 4);
        L.uleaf = take(groups * n_leaf * 4);
        L.ucount_leaf = take(groups * 4);
        L.key_pool = take(groups * n_mid * (size_t)t->d.fanout[2] * D * esize(t->d.dtype));
        L.val_pool = take(groups * n_leaf * D * esize(t->d.dtype));
        if (t->host_mids) {   // the kept roots' mid blocks
            const size_t n_root = (size_t)G * ks.K[0];
            L.mid_slot = take(BH * ks.K[0] * 4);
            L.uroot = take(groups * n_root * 4);
            L.ucount_root = take(groups * 4);
            L.mid_pool = take(groups * n_root * (size_t)t->d.fanout[1] * D * esize(t->d.dtype));
        }
    }
    L.pm_chunks = host ? query_chunks(B) : 1;
    if (L.pm) {
        L.pm_zero = take(L.pm_chunks * L.pmp.zero_bytes);
        L.pm_data = take(L.pm_chunks * L.pmp.data_bytes);
    }
    L.total = off;
    return L;
}

atlaskv_status check_params(const atlaskv_tree *t, const Ks &ks, int B, int N, int H, int T)
{
    if (!t) return fail(ATLASKV_EINVAL, "null tree");
    if (ks.n != t->n_levels) return fail(ATLASKV_EINVAL, "%d kept counts for a tree of %d levels", ks.n, t->n_levels);
    if (B < 0) return fail(ATLASKV_EINVAL, "B = %d < 0", B);
    if (H < 1 || H % t->d.n_kv_heads != 0)
        return fail(ATLASKV_EINVAL, "H = %d is not a positive multiple of H_kv = %d", H, t->d.n_kv_heads);
    if (N < 1 || N > T) return fail(ATLASKV_EINVAL, "need 1 <= N <= T (N = %d, T = %d)", N, T);
    if (N > 65535) return fail(ATLASKV_EUNSUPPORTED, "N = %d above 65535", N);
    if (ks.K[0] < 1 || ks.K[0] > t->rows[0])
        return fail(ATLASKV_EINVAL, "K of level 0 = %d not in [1, %lld roots]", ks.K[0], t->rows[0]);
    if (t->rows[0] > kMaxCandidates)
        return fail(ATLASKV_EUNSUPPORTED, "more than %d roots", kMaxCandidates);
    for (int l = 1; l < ks.n; ++l) {
        // every traversal has at least K[l-1] * min_ch candidates at level l
        const long long lo = (long long)ks.K[l - 1] * t->min_ch[l - 1];
        if (ks.K[l] < 1 || ks.K[l] > lo)
            return fail(ATLASKV_EINVAL, "K of level %d = %d not in [1, K of level %d * fewest children = %lld]", l,
                        ks.K[l], l - 1, lo);
        if ((long long)ks.K[l - 1] * t->max_ch[l - 1] > kMaxCandidates)
            return fail(ATLASKV_EUNSUPPORTED, "level %d can have more than %d candidates per traversal", l,
                        kMaxCandidates);
    }
    if (!(ks.scale >= 0.f) || std::isinf(ks.scale)) return fail(ATLASKV_EINVAL, "scale must be finite and >= 0");
    if ((long long)B * H > (1LL << 31) - 1) return fail(ATLASKV_EUNSUPPORTED, "B * H too large");
    const int kcap = pow2_at_least(k_max(ks), 32);
    const bool fused_ok = plan_descent(H / t->d.n_kv_heads, ks, kcap, score_cap(t, ks), t->d.head_dim,
                                       (int)esize(t->d.dtype), (long long)B * t->d.n_kv_heads, t->num_sms)
                              .GC > 0;
    const int nc = t->host_leaves ? query_chunks(B) : 1;
    const bool pm_ok = plan_pm(t, ks, (B + nc - 1) / nc, H, kcap).ok;
    if (t->descent_mode == ATLASKV_DESCENT_FUSED && !fused_ok)
        return fail(ATLASKV_EUNSUPPORTED, "the fused descent's shared-memory plan does not fit for these K");
    if (t->descent_mode == ATLASKV_DESCENT_PARENT_MAJOR && !pm_ok)
        return fail(ATLASKV_EUNSUPPORTED, "the parent-major descent does not fit for these K and sizes");
    if (!fused_ok && !pm_ok) return fail(ATLASKV_EUNSUPPORTED, "no descent plan fits for these K and sizes");
    return ATLASKV_OK;
}

template <typename T, int D>
atlaskv_status launch_norms(const atlaskv_tree *t, const void *keys, long long rows, int level, cudaStream_t s)
{
    dim3 grid((unsigned)std::min<long long>((rows + 7) / 8, 4096), t->d.n_kv_heads);
    akv::key_norm_kernel<T, D><<<grid, 256, 0, s>>>(reinterpret_cast<const T *>(keys), rows,
                                                    reinterpret_cast<unsigned int *>(t->norm_bound) +
                                                        (size_t)level * t->d.n_kv_heads);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

template <typename T, int D>
atlaskv_status tree_norms(const atlaskv_tree *t, cudaStream_t s)
{
    for (int l = 0; l < t->n_levels; ++l) {
        atlaskv_status st = launch_norms<T, D>(t, t->lkeys[l], t->rows[l], l, s);
        if (st != ATLASKV_OK) return st;
    }
    return ATLASKV_OK;
}

atlaskv_status dispatch_norms(const atlaskv_tree *t, cudaStream_t s)
{
    const int D = t->d.head_dim;
    if (t->d.dtype == ATLASKV_F32) return D == 64 ? tree_norms<float, 64>(t, s) : tree_norms<float, 128>(t, s);
    return D == 64 ? tree_norms<__nv_bfloat16, 64>(t, s) : tree_norms<__nv_bfloat16, 128>(t, s);
}

atlaskv_status check_table(const int32_t *tab, long long entries_per_head, int H_kv, long long child_rows, int *status,
                           cudaStream_t s)
{
    unsigned int *hits = nullptr;
    const size_t n = (size_t)H_kv * child_rows;
    AKV_CUDA(cudaMallocAsync(&hits, n * sizeof(unsigned int), s));
    AKV_CUDA(cudaMemsetAsync(hits, 0, n * sizeof(unsigned int), s));
    akv::child_table_check_kernel<<<2048, 256, 0, s>>>(tab, entries_per_head, H_kv, child_rows, hits, status);
    akv::hits_check_kernel<<<2048, 256, 0, s>>>(hits, (long long)n, status);
    AKV_CUDA(cudaGetLastError());
    AKV_CUDA(cudaFreeAsync(hits, s));
    return ATLASKV_OK;
}

template <typename T, int D, int HT>
atlaskv_status launch_descend_ht(const akv::DescendParams &dp, size_t smem, int first, int last, cudaStream_t s)
{
    const long long grid = (long long)dp.B * dp.H_kv * (dp.G / dp.GC);
    if (grid > 0x7fffffffLL) return fail(ATLASKV_EUNSUPPORTED, "descent grid too large");
    if (grid == 0) return ATLASKV_OK;
    AKV_SMEM((akv::descend_kernel<T, D, HT>), smem);
    akv::descend_kernel<T, D, HT><<<(unsigned)grid, akv::kDescThreads, smem, s>>>(dp, first, last);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

// the smallest head count per warp a key row's lane group allows (see plan_descent)
template <typename T, int D>
constexpr int min_ht()
{
    return (D * (int)sizeof(T) / 16) / 4 < 1 ? 1 : (D * (int)sizeof(T) / 16) / 4;
}

template <typename T, int D>
atlaskv_status launch_descend(const akv::DescendParams &dp, int HT, size_t smem, int first, int last, cudaStream_t s)
{
    constexpr int lo = min_ht<T, D>();
    if constexpr (lo <= 2)
        if (HT <= 2) return launch_descend_ht<T, D, 2>(dp, smem, first, last, s);
    if constexpr (lo <= 4)
        if (HT <= 4) return launch_descend_ht<T, D, 4>(dp, smem, first, last, s);
    return launch_descend_ht<T, D, 8>(dp, smem, first, last, s);
}

atlaskv_status dispatch_descend(int dtype, int D, const akv::DescendParams &dp, int HT, size_t smem, int first,
                                int last, cudaStream_t s)
{
    if (dtype == ATLASKV_F32)
        return D == 64 ? launch_descend<float, 64>(dp, HT, smem, first, last, s)
                       : launch_descend<float, 128>(dp, HT, smem, first, last, s);
    return D == 64 ? launch_descend<__nv_bfloat16, 64>(dp, HT, smem, first, last, s)
                   : launch_descend<__nv_bfloat16, 128>(dp, HT, smem, first, last, s);
}

// Launch with programmatic stream serialization: the kernel may begin while
// the previous kernel on the stream drains; it waits (griddep_wait) before it
// reads anything that kernel wrote.
template <typename... KArgs, typename... Args>
atlaskv_status launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t s,
                          Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    AKV_CUDA(cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...));
    return ATLASKV_OK;
}

// ---- parent-major descent launches -------------------------------------------
// Levels first..last of one query chunk: token sums, root scores and root
// selection when first = 0; then per level the inversion of the kept parents
// (scan, fill), the scores by parent and the selection.  Each selection but
// the last level's counts its kept entries for the next level's inversion.
#define AKV_RET(x)                                 \
    do {                                           \
        const atlaskv_status st_ = (x);            \
        if (st_ != ATLASKV_OK) return st_;         \
    } while (0)

// zero / zero_bytes: the chunk's zero-initialised inversion region, cleared
// by the token-sum kernel (first = 0).
template <typename T, int D>
atlaskv_status run_pm(const atlaskv_tree *t, const PmPlan &pp, const akv::DescendParams &dp, const akv::PmLevel *lv,
                      uint8_t *zero, size_t zero_bytes, int first, int last, cudaStream_t s)
{
    const int nl = dp.n_levels;
    const long long BH = (long long)dp.B * dp.H;
    if (BH == 0) return ATLASKV_OK;
    const akv::PmLevel none{};
    const size_t sel_smem = (size_t)pp.nsel * pp.pw;
    AKV_SMEM((akv::pm_select_kernel<T, D, 2>), sel_smem);
    AKV_SMEM((akv::pm_select_kernel<T, D, 3>), sel_smem);
    const unsigned sel_grid = (unsigned)((BH + pp.nsel - 1) / pp.nsel);
    // more traversals than one wave of 2 CTAs per SM: the 3-CTA register budget
    const bool sel3 = (long long)sel_grid > 2LL * t->num_sms;
    const size_t score_smem = akv::pm_score_smem((int)sizeof(T));
    AKV_SMEM((akv::pm_score_kernel<T, D>), score_smem);
    // the scoring grid: as many CTAs as fit on the device at once (the warps loop over the items)
    static thread_local std::map<std::pair<const void *, int>, int> fit;
    int &per_sm = fit[{reinterpret_cast<const void *>(akv::pm_score_kernel<T, D>), t->num_sms}];
    if (per_sm == 0) {
        AKV_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, akv::pm_score_kernel<T, D>, akv::kPmThreads,
                                                               score_smem));
        per_sm = std::max(per_sm, 1);
    }
    const long long score_cap = (long long)t->num_sms * per_sm;
    const size_t ref_smem = (size_t)(akv::kSelThreads / 32) * (dp.Kpmax + 1) * 4;
    AKV_SMEM((akv::pm_refine_kernel<T, D>), ref_smem);
    const unsigned ref_grid = (unsigned)std::min<long long>((BH + 7) / 8, (long long)t->num_sms * 2);
    auto select = [&](int L) -> atlaskv_status {
        const akv::PmLevel &nx = L + 1 < nl ? lv[L + 1] : none;
        if (sel3)
            AKV_RET(launch_pdl(akv::pm_select_kernel<T, D, 3>, sel_grid, akv::kSelThreads, sel_smem, s, dp, lv[L], nx,
                               L, pp.nsel, pp.pw));
        else
            AKV_RET(launch_pdl(akv::pm_select_kernel<T, D, 2>, sel_grid, akv::kSelThreads, sel_smem, s, dp, lv[L], nx,
                               L, pp.nsel, pp.pw));
        AKV_RET(launch_pdl(akv::pm_refine_kernel<T, D>, ref_grid, akv::kSelThreads, ref_smem, s, dp, lv[L], nx, L));
        return ATLASKV_OK;
    };
    if (first == 0) {
        const long long tsg = (long long)dp.B * dp.H_kv * (dp.G / pp.ts_GC);
        AKV_RET(launch_pdl(akv::token_sums_kernel<T, D>, (unsigned)tsg, akv::kDescThreads, pp.ts_smem, s, dp, pp.ts_GC,
                           reinterpret_cast<uint4 *>(zero), (long long)(zero_bytes / 16)));
        const long long items = (long long)dp.H_kv * ((dp.B * dp.G + pp.EC - 1) / pp.EC);
        AKV_RET(launch_pdl(akv::pm_score_kernel<T, D>,
                           (unsigned)std::min((items + akv::kPmWarps - 1) / akv::kPmWarps, score_cap), akv::kPmThreads,
                           score_smem, s, dp, none, 0));
        AKV_RET(select(0));
    }
    for (int L = std::max(first, 1); L <= last; ++L) {
        const akv::PmLevel &v = lv[L];
        AKV_RET(launch_pdl(akv::pm_scan_kernel, (unsigned)v.n_tiles, akv::kScanThreads, 0, s, v, pp.EC, dp.status));
        const unsigned fg = (unsigned)std::min<long long>((v.E + 255) / 256, (long long)t->num_sms * 8);
        AKV_RET(launch_pdl(akv::pm_fill_kernel, std::max(1u, fg), 256, 0, s, (const int32_t *)dp.kept[L - 1],
                           dp.K[L - 1], dp.H, dp.G, (long long)dp.rows[L - 1], v, dp.status));
        AKV_RET(launch_pdl(akv::pm_score_kernel<T, D>,
                           (unsigned)std::min<long long>((v.max_items + akv::kPmWarps - 1) / akv::kPmWarps, score_cap),
                           akv::kPmThreads, score_smem, s, dp, v, L));
        AKV_RET(select(L));
    }
    return ATLASKV_OK;
}


atlaskv_status dispatch_pm(const atlaskv_tree *t, const PmPlan &pp, const akv::DescendParams &dp,
                           const akv::PmLevel *lv, uint8_t *zero, size_t zero_bytes, int first, int last,
                           cudaStream_t s)
{
    const int D = t->d.head_dim;
    if (t->d.dtype == ATLASKV_F32)
        return D == 64 ? run_pm<float, 64>(t, pp, dp, lv, zero, zero_bytes, first, last, s)
                       : run_pm<float, 128>(t, pp, dp, lv, zero, zero_bytes, first, last, s);
    return D == 64 ? run_pm<__nv_bfloat16, 64>(t, pp, dp, lv, zero, zero_bytes, first, last, s)
                   : run_pm<__nv_bfloat16, 128>(t, pp, dp, lv, zero, zero_bytes, first, last, s);
}

// ---- attention launch -----------------------------------------------------
template <int D>
atlaskv_status launch_attend_f32(const akv::AttnParams &ap, cudaStream_t s)
{
    const long long rows = (long long)ap.B * ap.N * ap.H;
    const long long grid = (rows + 3) / 4;
    if (grid > 0x7fffffffLL) return fail(ATLASKV_EUNSUPPORTED, "attention grid too large");
    akv::attend_f32_kernel<D><<<(unsigned)grid, 128, 0, s>>>(ap);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

// 4-D tensor map (bf16, 128-byte swizzle, zero fill outside) over a tensor
// [d3][d2][d1][D] (D = 64 or 128 innermost) with a (64, 1, rows, 1) box, for
// the attention kernel.  cuTensorMapEncodeTiled is a host-only call, reached
// through the runtime's driver entry point.
atlaskv_status encode_tc_map(CUtensorMap *map, const void *base, int D, long long d1, long long d2, long long d3,
                             int rows)
{
    // looked up once per process (thread-safe static initialisation)
    static const PFN_cuTensorMapEncodeTiled_v12000 encode = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        cudaDriverEntryPointQueryResult q;
        void *fn = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }();
    if (!encode) return fail(ATLASKV_ECUDA, "cuTensorMapEncodeTiled is not available from the driver");
    if (reinterpret_cast<uintptr_t>(base) & 15u) return fail(ATLASKV_EINVAL, "attention inputs must be 16-byte aligned");
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)d1, (cuuint64_t)d2, (cuuint64_t)d3};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)(d1 * D * 2), (cuuint64_t)(d2 * d1 * D * 2)};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(ATLASKV_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return ATLASKV_OK;
}

int num_sms();

// bf16, D = 64 or 128: tcgen05 tensor cores, units of 128 query rows of a
// (query, KV head) group on a persistent grid.  Sequence K / V [B][T][H_kv][D] by TMA
// (box of 64 keys); Q [B][N][H][D] by TMA too (box of min(N, 128) tokens of
// one head) when every head's rows start on a swizzle atom of the Q tile, i.e.
// N is a multiple of 8 that divides 128 or is divisible by it, else by
// cp.async.
template <int D>
atlaskv_status launch_attend_tc(const akv::AttnParams &ap, cudaStream_t s)
{
    const int rows = ap.G * ap.N;
    const int cpg = (rows + akv::tc::kCtaRows - 1) / akv::tc::kCtaRows;
    const long long units = (long long)ap.B * ap.H_kv * cpg;
    if (units > 0x7fffffffLL) return fail(ATLASKV_EUNSUPPORTED, "attention grid too large");
    if (units == 0) return ATLASKV_OK;
    if (ap.lk_rows >= (1LL << 31) || ap.lv_rows >= (1LL << 31))
        return fail(ATLASKV_EUNSUPPORTED, "more than 2^31 leaf rows");
    CUtensorMap mk, mv, mqs, mqk;
    atlaskv_status st = encode_tc_map(&mk, ap.k_seq, D, ap.H_kv, ap.T, ap.B, akv::tc::kKeys);
    if (st != ATLASKV_OK) return st;
    st = encode_tc_map(&mv, ap.v_seq, D, ap.H_kv, ap.T, ap.B, akv::tc::kKeys);
    if (st != ATLASKV_OK) return st;
    // a mode that reads only one of the two query tensors uses it for both maps
    const void *qs = ap.q_seq ? ap.q_seq : ap.q_kg, *qk = ap.q_kg ? ap.q_kg : ap.q_seq;
    const auto aligned = [](const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    const int q_maps = ap.N % 8 == 0 && (128 % ap.N == 0 || ap.N % 128 == 0) && aligned(qs) && aligned(qk);
    if (q_maps) {
        const int bn = ap.N < akv::tc::kRows ? ap.N : akv::tc::kRows;
        st = encode_tc_map(&mqs, qs, D, ap.H, ap.N, ap.B, bn);
        if (st != ATLASKV_OK) return st;
        st = encode_tc_map(&mqk, qk, D, ap.H, ap.N, ap.B, bn);
        if (st != ATLASKV_OK) return st;
    } else {
        mqs = mqk = mk;   // unused
    }
    constexpr int smem = akv::tc::TcSmem<D>::kBytes;
    AKV_SMEM(akv::attend_tc_kernel<D>, smem);
    // persistent grid: as many CTAs as are resident at once, each taking units
    // round-robin.  Two per SM by construction (112 KB of shared memory, 256
    // TMEM columns, the launch bounds); the occupancy query reports one here
    // (it assumes the default shared-memory carve-out), and a grid of one per SM
    // measured 1.4x slower.
    const long long resident = (long long)akv::tc::kMinCtasPerSm * num_sms();
    const unsigned grid = (unsigned)(units < resident ? units : resident);
    return launch_pdl(akv::attend_tc_kernel<D>, grid, akv::tc::kThreads, smem, s, ap, cpg,
                      (unsigned)units, mk, mv, mqs, mqk, q_maps);
}

atlaskv_status dispatch_attend(int dtype, int D, const akv::AttnParams &ap, cudaStream_t s)
{
    if (dtype == ATLASKV_F32) return D == 64 ? launch_attend_f32<64>(ap, s) : launch_attend_f32<128>(ap, s);
    return D == 64 ? launch_attend_tc<64>(ap, s) : launch_attend_tc<128>(ap, s);
}

// ---- staging launches -----------------------------------------------------
// SM count of the current device (a grid size, not a correctness matter).
int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        n <= 0)
        n = 148;
    return n;
}

atlaskv_status launch_dedupe(const int32_t *ids, int n, int groups, int32_t *uniq, int32_t *slot, int32_t *count,
                             cudaStream_t s)
{
    const int n2 = pow2_at_least(n, 2);
    const size_t smem = (size_t)n2 * 12;
    AKV_SMEM(akv::dedupe_kernel, smem);
    akv::dedupe_kernel<<<groups, akv::kDedupeThreads, smem, s>>>(ids, n, n2, uniq, slot, count);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

// Blocks of children of unique kept parents at level L (1: mids of kept
// roots, 2: leaves of kept mids) from host memory into the pool.
template <typename T, int D>
atlaskv_status stage_keys(const atlaskv_tree *t, int L, const int32_t *uniq, const int32_t *cnt, int n, int groups,
                          void *pool, const int32_t *csrc, const int32_t *cfill, cudaStream_t s)
{
    const void *src = L == 1 ? t->mid_keys_dev : t->leaf_keys_dev;
    const int32_t *tab = L == 1 ? t->d.root_child : t->d.mid_child;
    T *cache = csrc ? reinterpret_cast<T *>(t->cache_pool) : nullptr;
    akv::stage_blocks_kernel<T, D><<<akv::kStageCtasPerSm * t->num_sms, 256, 0, s>>>(
        reinterpret_cast<const T *>(src), tab, t->rows[L - 1], t->rows[L], t->d.fanout[L], t->d.n_kv_heads, uniq, cnt,
        n, groups, reinterpret_cast<T *>(pool), t->status, cache, csrc, cfill);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

template <typename T, int D>
atlaskv_status stage_values(const atlaskv_tree *t, const int32_t *uleaf, const int32_t *cnt, int n, int groups,
                            void *vpool, cudaStream_t s)
{
    akv::stage_value_rows_kernel<T, D><<<akv::kStageCtasPerSm * t->num_sms, 256, 0, s>>>(reinterpret_cast<const T *>(t->leaf_values_dev), t->rows[2],
                                                          t->d.n_kv_heads, uleaf, cnt, n, groups,
                                                          reinterpret_cast<T *>(vpool));
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

// csrc / cfill: the chunk's cache map (null without the leaf-block cache)
atlaskv_status dispatch_stage_keys(const atlaskv_tree *t, int L, const int32_t *uniq, const int32_t *cnt, int n,
                                   int groups, void *pool, cudaStream_t s, const int32_t *csrc = nullptr,
                                   const int32_t *cfill = nullptr)
{
    const int D = t->d.head_dim;
    if (t->d.dtype == ATLASKV_F32)
        return D == 64 ? stage_keys<float, 64>(t, L, uniq, cnt, n, groups, pool, csrc, cfill, s)
                       : stage_keys<float, 128>(t, L, uniq, cnt, n, groups, pool, csrc, cfill, s);
    return D == 64 ? stage_keys<__nv_bfloat16, 64>(t, L, uniq, cnt, n, groups, pool, csrc, cfill, s)
                   : stage_keys<__nv_bfloat16, 128>(t, L, uniq, cnt, n, groups, pool, csrc, cfill, s);
}

// The leaf-block cache's map and commit for one chunk's unique kept mids.
atlaskv_status cache_map(const atlaskv_tree *t, const int32_t *umid, const int32_t *cnt, int n, int groups,
                         int32_t *csrc, int32_t *cfill, cudaStream_t s)
{
    const unsigned g = (unsigned)std::max<long long>(1, std::min<long long>(((long long)groups * n + 255) / 256,
                                                                            (long long)t->num_sms * 4));
    akv::cache_map_kernel<<<g, 256, 0, s>>>(umid, cnt, n, groups, t->d.n_kv_heads, t->rows[1], t->cache_tag,
                                            t->cache_sets, t->cache_epoch, csrc, cfill, t->cache_stats);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

atlaskv_status cache_commit(const atlaskv_tree *t, const int32_t *cnt, int n, int groups, const int32_t *cfill,
                            cudaStream_t s)
{
    const unsigned g = (unsigned)std::max<long long>(1, std::min<long long>(((long long)groups * n + 255) / 256,
                                                                            (long long)t->num_sms * 4));
    akv::cache_commit_kernel<<<g, 256, 0, s>>>(cnt, n, groups, cfill, t->cache_tag);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

atlaskv_status dispatch_stage_values(const atlaskv_tree *t, const int32_t *uleaf, const int32_t *cnt, int n,
                                     int groups, void *vpool, cudaStream_t s)
{
    const int D = t->d.head_dim;
    if (t->d.dtype == ATLASKV_F32)
        return D == 64 ? stage_values<float, 64>(t, uleaf, cnt, n, groups, vpool, s)
                       : stage_values<float, 128>(t, uleaf, cnt, n, groups, vpool, s);
    return D == 64 ? stage_values<__nv_bfloat16, 64>(t, uleaf, cnt, n, groups, vpool, s)
                   : stage_values<__nv_bfloat16, 128>(t, uleaf, cnt, n, groups, vpool, s);
}

// ---- one call's parameters ---------------------------------------------------
atlaskv_status check_io(const atlaskv_io *io)
{
    if (!io->q_kg || !io->q_seq || !io->k_seq || !io->v_seq || !io->out)
        return fail(ATLASKV_EINVAL, "null q_kg/q_seq/k_seq/v_seq/out");
    const void *ptrs[] = {io->q_kg, io->q_seq, io->k_seq, io->v_seq, io->out, io->lse, io->kept_root, io->kept_mid,
                          io->kept_leaf};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return fail(ATLASKV_EINVAL, "io buffers must be 16-byte aligned");
    return ATLASKV_OK;
}

struct Call {
    Layout L;
    akv::DescendParams dp;
    akv::AttnParams ap;
    int32_t *kept[akv::kMaxLevels];
};

// Descent and attention parameters of one call on tree t with workspace ws;
// kept_out[l]: the caller's kept-id buffer of level l, or null.
void fill_call(const atlaskv_tree *t, const Ks &ks, const atlaskv_io *io, int32_t *const *kept_out, uint8_t *ws,
               Call &c)
{
    const Layout &L = c.L;
    const int D = t->d.head_dim;
    const int H_kv = t->d.n_kv_heads;
    const int G = io->H / H_kv;
    const int nl = t->n_levels;
    for (int l = 0; l < akv::kMaxLevels; ++l)
        c.kept[l] = l >= nl ? nullptr
                            : (kept_out && kept_out[l]) ? kept_out[l] : reinterpret_cast<int32_t *>(ws + L.kept[l]);
    akv::DescendParams &dp = c.dp;
    dp = akv::DescendParams{};
    dp.q_kg = io->q_kg;
    dp.B = io->B;
    dp.N = io->N;
    dp.H = io->H;
    dp.H_kv = H_kv;
    dp.G = G;
    dp.n_levels = nl;
    dp.Kpmax = kp_max(ks);
    for (int l = 0; l < nl; ++l) {
        dp.keys[l] = t->lkeys[l];
        dp.rows[l] = t->rows[l];
        dp.fanout[l] = l == 0 ? (int)t->rows[0] : t->max_ch[l - 1];
        dp.kept[l] = c.kept[l];
        dp.K[l] = ks.K[l];
    }
    for (int l = 0; l + 1 < nl; ++l) {
        dp.coff[l] = t->coff[l];
        dp.cid[l] = t->cid[l];
    }
    if (!t->csr) {
        dp.child[0] = t->d.root_child;
        dp.child[1] = t->d.mid_child;
    }
    dp.norm_bound = t->norm_bound;
    dp.cprime = akv::gamma_n(D) * (1.0 + akv::gamma_n(io->N)) + akv::gamma_n(io->N);
    dp.s_ws = reinterpret_cast<float *>(ws + L.s_ws);
    dp.anorm_ws = reinterpret_cast<float *>(ws + L.anorm_ws);
    dp.s64_ws = reinterpret_cast<double *>(ws + L.s64_ws);
    dp.a64_ws = reinterpret_cast<double *>(ws + L.a64_ws);
    dp.f_ws = reinterpret_cast<float *>(ws + L.f_ws);
    dp.fstride = L.fstride;
    dp.cap = L.cap;
    dp.kcap = L.kcap;
    dp.xs_ws = ws + L.xs;
    dp.GC = L.desc.GC;
    dp.status = t->status;
    dp.stats = t->counting ? t->stats : nullptr;

    const float scale = ks.scale > 0.f ? ks.scale : 1.0f / sqrtf((float)D);
    akv::AttnParams &ap = c.ap;
    ap = akv::AttnParams{};
    ap.q_kg = io->q_kg;
    ap.q_seq = io->q_seq;
    ap.k_seq = io->k_seq;
    ap.v_seq = io->v_seq;
    ap.out = io->out;
    ap.lse = io->lse;
    ap.B = io->B;
    ap.N = io->N;
    ap.H = io->H;
    ap.H_kv = H_kv;
    ap.G = G;
    ap.T = io->T;
    ap.K_L = ks.K[nl - 1];
    ap.scale_log2 = scale * 1.4426950408889634f;
    ap.status = t->status;
    if (t->split) {
        ap.oseq = reinterpret_cast<float *>(ws + L.oseq);
        ap.lse_seq = reinterpret_cast<float *>(ws + L.lse_seq);
    }
    if (!t->host_leaves) {   // leaves read in place; the host path sets its pools per query chunk
        ap.lk_base = t->lkeys[nl - 1];
        ap.lv_base = t->leaf_values_dev;
        ap.lk_idx = c.kept[nl - 1];
        ap.lv_idx = c.kept[nl - 1];
        ap.leaf_head_stride = t->rows[nl - 1];
        ap.lk_rows = ap.lv_rows = (long long)H_kv * t->rows[nl - 1];
    }
}

// ---- layer batches ---------------------------------------------------------
template <typename T, int D, int HT>
atlaskv_status launch_descend_layers_ht(const akv::DescendBatch &b, size_t smem, unsigned grid, cudaStream_t s)
{
    AKV_SMEM((akv::descend_layers_kernel<T, D, HT>), smem);
    akv::descend_layers_kernel<T, D, HT><<<grid, akv::kDescThreads, smem, s>>>(b, 0, 2);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

template <typename T, int D>
atlaskv_status launch_descend_layers(const akv::DescendBatch &b, int HT, size_t smem, unsigned grid, cudaStream_t s)
{
    constexpr int lo = min_ht<T, D>();
    if constexpr (lo <= 2)
        if (HT <= 2) return launch_descend_layers_ht<T, D, 2>(b, smem, grid, s);
    if constexpr (lo <= 4)
        if (HT <= 4) return launch_descend_layers_ht<T, D, 4>(b, smem, grid, s);
    return launch_descend_layers_ht<T, D, 8>(b, smem, grid, s);
}

atlaskv_status dispatch_descend_layers(int dtype, int D, const akv::DescendBatch &b, int HT, size_t smem,
                                       unsigned grid, cudaStream_t s)
{
    if (dtype == ATLASKV_F32)
        return D == 64 ? launch_descend_layers<float, 64>(b, HT, smem, grid, s)
                       : launch_descend_layers<float, 128>(b, HT, smem, grid, s);
    return D == 64 ? launch_descend_layers<__nv_bfloat16, 64>(b, HT, smem, grid, s)
                   : launch_descend_layers<__nv_bfloat16, 128>(b, HT, smem, grid, s);
}

// The tensor-core attention of every layer in one launch, in `mode`.
template <int D>
atlaskv_status launch_attend_tc_layers(const Call *calls, int n, int mode, cudaStream_t s)
{
    static akv::AttnBatch b;   // large: not on the stack; guarded below
    static std::mutex m;
    std::lock_guard<std::mutex> lock(m);
    const akv::AttnParams &a0 = calls[0].ap;
    const int rows = a0.G * a0.N;
    const int cpg = (rows + akv::tc::kCtaRows - 1) / akv::tc::kCtaRows;
    const long long per = (long long)a0.B * a0.H_kv * cpg;
    if (per * n > 0x7fffffffLL) return fail(ATLASKV_EUNSUPPORTED, "attention grid too large");
    b.n = n;
    b.ctas_per_group = cpg;
    for (int l = 0; l < n; ++l) {
        b.p[l] = calls[l].ap;
        b.p[l].mode = mode;
        b.offs[l] = (unsigned)(per * l);
        if (b.p[l].lk_rows >= (1LL << 31)) return fail(ATLASKV_EUNSUPPORTED, "more than 2^31 leaf rows");
        atlaskv_status st = encode_tc_map(&b.mk[l], b.p[l].k_seq, D, a0.H_kv, a0.T, a0.B, akv::tc::kKeys);
        if (st != ATLASKV_OK) return st;
        st = encode_tc_map(&b.mv[l], b.p[l].v_seq, D, a0.H_kv, a0.T, a0.B, akv::tc::kKeys);
        if (st != ATLASKV_OK) return st;
    }
    b.offs[n] = (unsigned)(per * n);
    constexpr int smem = akv::tc::TcSmem<D>::kBytes;
    AKV_SMEM(akv::attend_tc_layers_kernel<D>, smem);
    akv::attend_tc_layers_kernel<D><<<(unsigned)(per * n), akv::tc::kThreads, smem, s>>>(b);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

// Inflate the per-level key-norm bounds slightly (they were rounded up already).
atlaskv_status inflate_norms(atlaskv_tree *t)
{
    const int nb = t->n_levels * t->d.n_kv_heads;
    float *tmp = new (std::nothrow) float[nb];
    if (!tmp) return fail(ATLASKV_ENOMEM, "host allocation failed");
    cudaError_t e = cudaMemcpy(tmp, t->norm_bound, nb * sizeof(float), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) {
        for (int i = 0; i < nb; ++i) tmp[i] = nextafterf(tmp[i] * (1.0f + 0x1p-20f), INFINITY);
        e = cudaMemcpy(t->norm_bound, tmp, nb * sizeof(float), cudaMemcpyHostToDevice);
    }
    delete[] tmp;
    if (e != cudaSuccess) return fail(ATLASKV_ECUDA, "norm bounds: %s", cudaGetErrorString(e));
    return ATLASKV_OK;
}

// The tree's small device words and, for bf16 D = 128 with host-resident
// leaves, its two streams and events (shared by both create functions).  The
// sequence part runs as its own launch only there, where it overlaps the host
// link; with the leaves in HBM the descent keeps every SM busy and the
// attention is one launch after it.
atlaskv_status init_tree_device(atlaskv_tree *t)
{
    t->split = t->d.dtype == ATLASKV_BF16 && t->host_leaves;
    if (t->split) {
        // the sequence part runs beside the descent: lowest priority for it,
        // highest for the descent (the critical path); created once here so
        // attend creates nothing
        int lo_prio = 0, hi_prio = 0;
        if (cudaDeviceGetStreamPriorityRange(&lo_prio, &hi_prio) != cudaSuccess ||
            cudaStreamCreateWithPriority(&t->seq_stream, cudaStreamNonBlocking, lo_prio) != cudaSuccess ||
            cudaStreamCreateWithPriority(&t->desc_stream, cudaStreamNonBlocking, hi_prio) != cudaSuccess) {
            cudaGetLastError();
            return fail(ATLASKV_ECUDA, "creating the tree's streams failed");
        }
        for (cudaEvent_t &e : t->fev)
            if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
                cudaGetLastError();
                return fail(ATLASKV_ECUDA, "creating the tree's events failed");
            }
    }
    if (cudaMalloc(&t->norm_bound, akv::kMaxLevels * sizeof(float) * t->d.n_kv_heads) != cudaSuccess ||
        cudaMalloc(&t->status, sizeof(int)) != cudaSuccess ||
        cudaMalloc(&t->stats, kNumCounters * sizeof(unsigned long long)) != cudaSuccess) {
        cudaGetLastError();
        return fail(ATLASKV_ECUDA, "device allocation of the tree's bound/status words failed");
    }
    return ATLASKV_OK;
}

}  // namespace

extern "C" {

const char *atlaskv_last_error(void) { return g_last_error.c_str(); }

atlaskv_status atlaskv_create_tree(const atlaskv_tree_desc *d, void *stream, atlaskv_tree **out)
{
    if (!d || !out) return fail(ATLASKV_EINVAL, "null desc or out");
    if (d->dtype != ATLASKV_F32 && d->dtype != ATLASKV_BF16) return fail(ATLASKV_EINVAL, "unknown dtype %d", d->dtype);
    if (d->head_dim != 64 && d->head_dim != 128)
        return fail(ATLASKV_EUNSUPPORTED, "head_dim %d not supported (64 or 128)", d->head_dim);
    if (d->n_kv_heads < 1) return fail(ATLASKV_EINVAL, "n_kv_heads = %d", d->n_kv_heads);
    for (int i = 0; i < 3; ++i)
        if (d->fanout[i] < 1) return fail(ATLASKV_EINVAL, "fanout[%d] = %d", i, d->fanout[i]);
    const long long n_root = d->fanout[0], n_mid = n_root * d->fanout[1], n_leaf = n_mid * d->fanout[2];
    if (n_leaf > (1LL << 31) - 1 || n_leaf * d->n_kv_heads > (1LL << 31) - 1)
        return fail(ATLASKV_EUNSUPPORTED, "H_kv * M = %lld rows above 2^31 - 1", n_leaf * d->n_kv_heads);
    if (!d->root_keys || !d->mid_keys || !d->leaf_keys || !d->leaf_values)
        return fail(ATLASKV_EINVAL, "null key/value pointer");
    if (!aligned16(d->root_keys) || !aligned16(d->mid_keys) || !aligned16(d->leaf_keys) || !aligned16(d->leaf_values))
        return fail(ATLASKV_EINVAL, "key/value buffers must be 16-byte aligned");
    if (d->leaf_location != ATLASKV_LEAVES_DEVICE && d->leaf_location != ATLASKV_LEAVES_HOST_PINNED)
        return fail(ATLASKV_EINVAL, "unknown leaf_location %d", d->leaf_location);
    if (d->mid_location != ATLASKV_LEAVES_DEVICE && d->mid_location != ATLASKV_LEAVES_HOST_PINNED)
        return fail(ATLASKV_EINVAL, "unknown mid_location %d", d->mid_location);
    if (d->mid_location == ATLASKV_LEAVES_HOST_PINNED && d->leaf_location != ATLASKV_LEAVES_HOST_PINNED)
        return fail(ATLASKV_EINVAL, "mids in host memory need the leaves in host memory too");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    atlaskv_tree *t = new (std::nothrow) atlaskv_tree();
    if (!t) return fail(ATLASKV_ENOMEM, "host allocation failed");
    t->d = *d;
    t->rows[0] = n_root;
    t->rows[1] = n_mid;
    t->rows[2] = n_leaf;
    t->leaf_keys_dev = d->leaf_keys;
    t->leaf_values_dev = d->leaf_values;
    t->mid_keys_dev = d->mid_keys;
    t->host_leaves = d->leaf_location == ATLASKV_LEAVES_HOST_PINNED;
    t->host_mids = d->mid_location == ATLASKV_LEAVES_HOST_PINNED;
    t->num_sms = num_sms();
    t->n_levels = 3;
    t->csr = false;
    for (int l = 0; l < 2; ++l) t->min_ch[l] = t->max_ch[l] = d->fanout[l + 1];
    auto bail = [&](atlaskv_status st) {
        std::string msg = g_last_error;
        atlaskv_destroy(t);
        g_last_error = msg;
        return st;
    };
    if (d->leaf_location == ATLASKV_LEAVES_HOST_PINNED) {
        void *pk = nullptr, *pv = nullptr;
        if (cudaHostGetDevicePointer(&pk, const_cast<void *>(d->leaf_keys), 0) != cudaSuccess ||
            cudaHostGetDevicePointer(&pv, const_cast<void *>(d->leaf_values), 0) != cudaSuccess) {
            cudaGetLastError();
            return bail(fail(ATLASKV_EINVAL, "leaf buffers are not pinned (page-locked, mapped) host memory"));
        }
        t->leaf_keys_dev = pk;
        t->leaf_values_dev = pv;
        if (t->host_mids) {
            void *pm = nullptr;
            if (cudaHostGetDevicePointer(&pm, const_cast<void *>(d->mid_keys), 0) != cudaSuccess) {
                cudaGetLastError();
                return bail(fail(ATLASKV_EINVAL, "mid keys are not pinned (page-locked, mapped) host memory"));
            }
            t->mid_keys_dev = pm;
        }
        // the staging stream and its events exist from here on, so attend
        // creates nothing (and may be captured into a CUDA graph).  Highest
        // priority: the copies are bound by the host link, so the block
        // scheduler should keep them resident and let the compute fill in.
        int lo_prio = 0, hi_prio = 0;
        if (cudaDeviceGetStreamPriorityRange(&lo_prio, &hi_prio) != cudaSuccess ||
            cudaStreamCreateWithPriority(&t->stage_stream, cudaStreamNonBlocking, hi_prio) != cudaSuccess) {
            cudaGetLastError();
            return bail(fail(ATLASKV_ECUDA, "creating the staging stream failed"));
        }
        for (cudaEvent_t &e : t->cev)
            if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
                cudaGetLastError();
                return bail(fail(ATLASKV_ECUDA, "creating the staging events failed"));
            }
    }
    {
        const atlaskv_status st0 = init_tree_device(t);
        if (st0 != ATLASKV_OK) return bail(st0);
    }
    atlaskv_status st;
#define AKV_TRY(x)                             \
    do {                                       \
        st = (x);                              \
        if (st != ATLASKV_OK) return bail(st); \
    } while (0)
#define AKV_TRYC(x)                                                                              \
    do {                                                                                         \
        cudaError_t e_ = (x);                                                                    \
        if (e_ != cudaSuccess) return bail(fail(ATLASKV_ECUDA, "%s: %s", #x, cudaGetErrorString(e_))); \
    } while (0)
    AKV_TRYC(cudaMemsetAsync(t->norm_bound, 0, akv::kMaxLevels * sizeof(float) * d->n_kv_heads, s));
    AKV_TRYC(cudaMemsetAsync(t->status, 0, sizeof(int), s));
    t->lkeys[0] = d->root_keys;
    t->lkeys[1] = t->mid_keys_dev;
    t->lkeys[2] = t->leaf_keys_dev;
    AKV_TRY(dispatch_norms(t, s));
    if (d->root_child) AKV_TRY(check_table(d->root_child, n_mid, d->n_kv_heads, n_mid, t->status, s));
    // (tables are device arrays; the staging kernels read them from HBM)
    if (d->mid_child) AKV_TRY(check_table(d->mid_child, n_leaf, d->n_kv_heads, n_leaf, t->status, s));
    int dev_status = 0;
    AKV_TRYC(cudaMemcpyAsync(&dev_status, t->status, sizeof(int), cudaMemcpyDeviceToHost, s));
    AKV_TRYC(cudaStreamSynchronize(s));
    if (dev_status != akv::kDevOk)
        return bail(fail(ATLASKV_EINVAL, "child table has an out-of-range id or is not a permutation"));
    AKV_TRY(inflate_norms(t));
#undef AKV_TRY
#undef AKV_TRYC
    *out = t;
    return ATLASKV_OK;
}

atlaskv_status atlaskv_create_tree_csr(const atlaskv_csr_tree_desc *d, void *stream, atlaskv_tree **out)
{
    if (!d || !out) return fail(ATLASKV_EINVAL, "null desc or out");
    if (d->dtype != ATLASKV_F32 && d->dtype != ATLASKV_BF16) return fail(ATLASKV_EINVAL, "unknown dtype %d", d->dtype);
    if (d->head_dim != 64 && d->head_dim != 128)
        return fail(ATLASKV_EUNSUPPORTED, "head_dim %d not supported (64 or 128)", d->head_dim);
    if (d->n_kv_heads < 1) return fail(ATLASKV_EINVAL, "n_kv_heads = %d", d->n_kv_heads);
    const int nl = d->n_levels;
    if (nl < 2 || nl > ATLASKV_MAX_LEVELS) return fail(ATLASKV_EINVAL, "n_levels = %d not in [2, %d]", nl,
                                                        ATLASKV_MAX_LEVELS);
    for (int l = 0; l < nl; ++l) {
        if (d->rows[l] < 1) return fail(ATLASKV_EINVAL, "rows[%d] = %lld", l, (long long)d->rows[l]);
        if (d->rows[l] * d->n_kv_heads > (1LL << 31) - 1)
            return fail(ATLASKV_EUNSUPPORTED, "H_kv * rows[%d] above 2^31 - 1", l);
        if (!d->keys[l] || !aligned16(d->keys[l])) return fail(ATLASKV_EINVAL, "keys[%d] null or not 16-byte aligned", l);
        if (l + 1 < nl && !d->child_off[l]) return fail(ATLASKV_EINVAL, "child_off[%d] is null", l);
    }
    if (!d->leaf_values || !aligned16(d->leaf_values))
        return fail(ATLASKV_EINVAL, "leaf_values null or not 16-byte aligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    atlaskv_tree *t = new (std::nothrow) atlaskv_tree();
    if (!t) return fail(ATLASKV_ENOMEM, "host allocation failed");
    auto bail = [&](atlaskv_status st) {
        std::string msg = g_last_error;
        atlaskv_destroy(t);
        g_last_error = msg;
        return st;
    };
    t->d.dtype = d->dtype;
    t->d.n_kv_heads = d->n_kv_heads;
    t->d.head_dim = d->head_dim;
    t->d.fanout[0] = (int)d->rows[0];
    t->d.root_keys = d->keys[0];
    t->d.mid_keys = d->keys[nl > 2 ? 1 : 0];
    t->d.leaf_keys = d->keys[nl - 1];
    t->d.leaf_values = d->leaf_values;
    t->n_levels = nl;
    t->csr = true;
    for (int l = 0; l < nl; ++l) {
        t->rows[l] = d->rows[l];
        t->lkeys[l] = d->keys[l];
    }
    for (int l = 0; l + 1 < nl; ++l) {
        t->coff[l] = d->child_off[l];
        t->cid[l] = d->child_id[l];
    }
    t->leaf_keys_dev = d->keys[nl - 1];
    t->leaf_values_dev = d->leaf_values;
    t->mid_keys_dev = t->d.mid_keys;
    t->num_sms = num_sms();
    // the offsets, read once here: first 0, non-decreasing, last = rows of the
    // level below; and the fewest / most children of a node per level
    for (int l = 0; l + 1 < nl; ++l) {
        const size_t per = (size_t)d->rows[l] + 1, n = per * d->n_kv_heads;
        int32_t *h = new (std::nothrow) int32_t[n];
        if (!h) return bail(fail(ATLASKV_ENOMEM, "host allocation failed"));
        const cudaError_t e = cudaMemcpy(h, d->child_off[l], n * sizeof(int32_t), cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) {
            delete[] h;
            return bail(fail(ATLASKV_ECUDA, "reading child_off[%d]: %s", l, cudaGetErrorString(e)));
        }
        int mn = 0x7fffffff, mx = 0;
        bool ok = true;
        for (int hk = 0; hk < d->n_kv_heads && ok; ++hk) {
            const int32_t *o = h + (size_t)hk * per;
            ok = o[0] == 0 && o[per - 1] == d->rows[l + 1];
            for (size_t i = 0; i + 1 < per && ok; ++i) {
                const int c = o[i + 1] - o[i];
                ok = c >= 0;
                mn = std::min(mn, c);
                mx = std::max(mx, c);
            }
        }
        delete[] h;
        if (!ok) return bail(fail(ATLASKV_EINVAL, "child_off[%d] is not a valid offset list (first 0, non-decreasing, "
                                                  "last = rows[%d])", l, l + 1));
        t->min_ch[l] = mn;
        t->max_ch[l] = mx;
    }
    {
        const atlaskv_status st0 = init_tree_device(t);
        if (st0 != ATLASKV_OK) return bail(st0);
    }
    atlaskv_status st;
    cudaError_t e;
    if ((e = cudaMemsetAsync(t->norm_bound, 0, akv::kMaxLevels * sizeof(float) * d->n_kv_heads, s)) != cudaSuccess ||
        (e = cudaMemsetAsync(t->status, 0, sizeof(int), s)) != cudaSuccess)
        return bail(fail(ATLASKV_ECUDA, "%s", cudaGetErrorString(e)));
    if ((st = dispatch_norms(t, s)) != ATLASKV_OK) return bail(st);
    for (int l = 0; l + 1 < nl; ++l)
        if (d->child_id[l] &&
            (st = check_table(d->child_id[l], d->rows[l + 1], d->n_kv_heads, d->rows[l + 1], t->status, s)) != ATLASKV_OK)
            return bail(st);
    int dev_status = 0;
    if ((e = cudaMemcpyAsync(&dev_status, t->status, sizeof(int), cudaMemcpyDeviceToHost, s)) != cudaSuccess ||
        (e = cudaStreamSynchronize(s)) != cudaSuccess)
        return bail(fail(ATLASKV_ECUDA, "%s", cudaGetErrorString(e)));
    if (dev_status != akv::kDevOk)
        return bail(fail(ATLASKV_EINVAL, "a child list has an out-of-range id or is not a permutation"));
    if ((st = inflate_norms(t)) != ATLASKV_OK) return bail(st);
    *out = t;
    return ATLASKV_OK;
}

namespace {
atlaskv_status attend_impl(atlaskv_tree *t, const Ks &ks, const atlaskv_io *io, int32_t *const *kept_out,
                           void *workspace, size_t ws_bytes, void *stream);

Ks ks_of_levels(const atlaskv_tree *t, const atlaskv_level_params *p)
{
    Ks k{};
    k.n = t ? t->n_levels : 0;
    for (int l = 0; l < k.n; ++l) k.K[l] = p->K[l];
    k.scale = p->scale;
    return k;
}
}  // namespace

atlaskv_status atlaskv_workspace_size_csr(const atlaskv_tree *t, const atlaskv_level_params *p, int32_t B, int32_t N,
                                          int32_t H, int32_t T, size_t *bytes)
{
    if (!bytes || !p || !t) return fail(ATLASKV_EINVAL, "null tree, params or bytes");
    if (!t->csr) return fail(ATLASKV_EINVAL, "not a CSR tree (use atlaskv_workspace_size)");
    const Ks ks = ks_of_levels(t, p);
    atlaskv_status st = check_params(t, ks, B, N, H, T);
    if (st != ATLASKV_OK) return st;
    *bytes = plan(t, ks, B, N, H, T).total;
    return ATLASKV_OK;
}

atlaskv_status atlaskv_attend_csr(atlaskv_tree *t, const atlaskv_level_params *p, const atlaskv_io *io,
                                  int32_t *const *kept, void *workspace, size_t workspace_bytes, void *stream)
{
    if (!p || !io || !t) return fail(ATLASKV_EINVAL, "null tree, params or io");
    if (!t->csr) return fail(ATLASKV_EINVAL, "not a CSR tree (use atlaskv_attend)");
    if (kept)
        for (int l = 0; l < t->n_levels; ++l)
            if (kept[l] && !aligned16(kept[l])) return fail(ATLASKV_EINVAL, "kept buffers must be 16-byte aligned");
    return attend_impl(t, ks_of_levels(t, p), io, kept, workspace, workspace_bytes, stream);
}

atlaskv_status atlaskv_workspace_size(const atlaskv_tree *t, const atlaskv_params *p, int32_t B, int32_t N, int32_t H,
                                      int32_t T, size_t *bytes)
{
    if (!bytes || !p) return fail(ATLASKV_EINVAL, "null bytes or params");
    if (t && t->csr) return fail(ATLASKV_EINVAL, "a CSR tree is sized with atlaskv_workspace_size_csr");
    const Ks ks = ks_of(p);
    atlaskv_status st = check_params(t, ks, B, N, H, T);
    if (st != ATLASKV_OK) return st;
    *bytes = plan(t, ks, B, N, H, T).total;
    return ATLASKV_OK;
}

}  // extern "C"

namespace {

// The whole path for one call (uniform or CSR tree); kept_out[l] is the
// caller's kept-id buffer of level l, or null.
atlaskv_status attend_impl(atlaskv_tree *t, const Ks &ks, const atlaskv_io *io, int32_t *const *kept_out,
                           void *workspace, size_t ws_bytes, void *stream)
{
    if (!io) return fail(ATLASKV_EINVAL, "null io");
    atlaskv_status st = check_params(t, ks, io->B, io->N, io->H, io->T);
    if (st != ATLASKV_OK) return st;
    if (io->B == 0) return ATLASKV_OK;
    st = check_io(io);
    if (st != ATLASKV_OK) return st;
    Call call;
    call.L = plan(t, ks, io->B, io->N, io->H, io->T);
    const Layout &L = call.L;
    if (!workspace || ((uintptr_t)workspace & 255u)) return fail(ATLASKV_EINVAL, "workspace must be 256-byte aligned");
    if (ws_bytes < L.total)
        return fail(ATLASKV_ENOMEM, "workspace of %zu bytes, %zu needed", ws_bytes, L.total);

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
    const int D = t->d.head_dim;
    const int H_kv = t->d.n_kv_heads;
    const int G = io->H / H_kv;
    const bool host = t->host_leaves;
    fill_call(t, ks, io, kept_out, ws, call);
    akv::DescendParams &dp = call.dp;
    akv::AttnParams &ap = call.ap;
    int32_t *const *kept = call.kept;
    const atlaskv_params pk{ks.K[0], ks.K[1], ks.n > 2 ? ks.K[2] : 0, ks.scale};   // the host path's three levels
    const atlaskv_params *p = &pk;

    const bool prof = t->profiling;
#define AKV_STEP(x)                            \
    do {                                       \
        atlaskv_status st_ = (x);              \
        if (st_ != ATLASKV_OK) return st_;     \
    } while (0)

    if (t->counting) AKV_CUDA(cudaMemsetAsync(t->stats, 0, kNumCounters * sizeof(unsigned long long), s));
    auto tm = [&](int i, cudaStream_t st) -> atlaskv_status {
        if (prof) AKV_CUDA(cudaEventRecord(t->ev[i], st));
        return ATLASKV_OK;
    };
    // The sequence part depends only on the call's inputs: with the split it
    // starts at once on the tree's low-priority stream, beside the descent
    // (and the staging), and the leaf part merges with it afterwards.
    auto fork_sequence_part = [&]() -> atlaskv_status {
        AKV_CUDA(cudaStreamWaitEvent(t->seq_stream, t->fev[0], 0));
        akv::AttnParams a = ap;
        a.mode = akv::kAttnSeq;
        AKV_STEP(tm(2, t->seq_stream));
        AKV_STEP(D == 64 ? launch_attend_tc<64>(a, t->seq_stream) : launch_attend_tc<128>(a, t->seq_stream));
        AKV_STEP(tm(3, t->seq_stream));
        AKV_CUDA(cudaEventRecord(t->fev[2], t->seq_stream));
        return ATLASKV_OK;
    };
    // the whole descent of an HBM call on stream `st`
    auto descend_all = [&](cudaStream_t st) -> atlaskv_status {
        if (!L.pm) return dispatch_descend(t->d.dtype, D, dp, L.desc.HT, L.desc.smem, 0, t->n_levels - 1, st);
        akv::PmLevel lv[akv::kMaxLevels];
        pm_bind(L.pmp, t->n_levels, (long long)dp.B * dp.H, ws + L.pm_zero, ws + L.pm_data, lv);
        return dispatch_pm(t, L.pmp, dp, lv, ws + L.pm_zero, L.pmp.zero_bytes, 0, t->n_levels - 1, st);
    };
    t->pm_last = L.pm;
    if (!host) {
        if (t->split) {
            // fork: descent on the high-priority stream, sequence part on the
            // low-priority one; join both into the caller's stream for the leaf part
            AKV_CUDA(cudaEventRecord(t->fev[0], s));
            AKV_CUDA(cudaStreamWaitEvent(t->desc_stream, t->fev[0], 0));
            AKV_STEP(tm(0, t->desc_stream));
            AKV_STEP(descend_all(t->desc_stream));
            AKV_STEP(tm(1, t->desc_stream));
            AKV_CUDA(cudaEventRecord(t->fev[1], t->desc_stream));
            AKV_STEP(fork_sequence_part());
            AKV_CUDA(cudaStreamWaitEvent(s, t->fev[1], 0));
            AKV_CUDA(cudaStreamWaitEvent(s, t->fev[2], 0));
            ap.mode = akv::kAttnLeaf;
            AKV_STEP(tm(4, s));
            AKV_STEP(dispatch_attend(t->d.dtype, D, ap, s));
            AKV_STEP(tm(5, s));
        } else {
            AKV_STEP(tm(0, s));
            AKV_STEP(descend_all(s));
            AKV_STEP(tm(1, s));
            AKV_STEP(tm(4, s));
            AKV_STEP(dispatch_attend(t->d.dtype, D, ap, s));
            AKV_STEP(tm(5, s));
        }
    } else {
        // Query chunks: chunk c covers queries [b0, b0 + Bc).  The caller's
        // stream runs the descent and the knowledge part of each chunk; the
        // staging stream copies, for each host-resident level, the blocks of
        // children of the chunk's kept parents as soon as those are kept, and
        // at the end the kept leaves' value rows, so the host link works while
        // the other chunks compute.
        const int nc = query_chunks(io->B);
        cudaStream_t s1 = t->stage_stream;
        const int n_root = G * p->K_root, n_mid = G * p->K_mid, n_leaf = G * p->K_leaf;
        const size_t esz = esize(t->d.dtype);
        auto cev = [&](int c, int k) { return t->cev[c * kChunkEvents + k]; };
        auto tmark = [&](int c, int k, cudaStream_t st) -> atlaskv_status {
            if (prof) AKV_CUDA(cudaEventRecord(t->tev[c * kTimingEvents + k], st));
            return ATLASKV_OK;
        };
        struct Chunk {
            akv::DescendParams d;
            akv::AttnParams a;
            akv::PmLevel lv[akv::kMaxLevels];
            int groups;
            int32_t *uroot, *croot, *mid_slot, *umid, *cmid, *leaf_slot, *uleaf, *cleaf, *vslot, *csrc, *cfill;
        };
        Chunk ch[kMaxChunks];
        for (int c = 0; c < nc; ++c) {
            const int b0 = (int)((long long)io->B * c / nc), b1 = (int)((long long)io->B * (c + 1) / nc);
            const int Bc = b1 - b0;
            const size_t bh0 = (size_t)b0 * io->H, g0 = (size_t)b0 * H_kv;
            Chunk &k = ch[c];
            k.groups = Bc * H_kv;
            akv::DescendParams d = dp;
            d.B = Bc;
            d.q_kg = reinterpret_cast<const uint8_t *>(io->q_kg) + (size_t)b0 * io->N * io->H * D * esz;
            for (int l = 0; l < 3; ++l) d.kept[l] = kept[l] + bh0 * dp.K[l];
            d.s_ws = dp.s_ws + bh0 * D;
            d.s64_ws = dp.s64_ws + bh0 * D;
            d.a64_ws = dp.a64_ws + bh0 * D;
            d.anorm_ws = dp.anorm_ws + bh0;
            d.f_ws = dp.f_ws + bh0 * (size_t)L.fstride;
            d.xs_ws = L.pm ? dp.xs_ws + bh0 * akv::ExactScratch::bytes()
                           : dp.xs_ws + (size_t)b0 * H_kv * (G / L.desc.GC) * L.desc.nsel * akv::ExactScratch::bytes();
            if (L.pm)
                pm_bind(L.pmp, t->n_levels, (long long)Bc * io->H, ws + L.pm_zero + c * L.pmp.zero_bytes,
                        ws + L.pm_data + c * L.pmp.data_bytes, k.lv);
            k.leaf_slot = reinterpret_cast<int32_t *>(ws + L.leaf_slot) + bh0 * p->K_mid;
            k.vslot = reinterpret_cast<int32_t *>(ws + L.vslot) + bh0 * p->K_leaf;
            k.umid = reinterpret_cast<int32_t *>(ws + L.umid) + g0 * n_mid;
            k.cmid = reinterpret_cast<int32_t *>(ws + L.ucount_mid) + g0;
            k.csrc = reinterpret_cast<int32_t *>(ws + L.csrc) + g0 * n_mid;
            k.cfill = reinterpret_cast<int32_t *>(ws + L.cfill) + g0 * n_mid;
            k.uleaf = reinterpret_cast<int32_t *>(ws + L.uleaf) + g0 * n_leaf;
            k.cleaf = reinterpret_cast<int32_t *>(ws + L.ucount_leaf) + g0;
            uint8_t *pool = ws + L.key_pool + g0 * n_mid * (size_t)t->d.fanout[2] * D * esz;
            uint8_t *vpool = ws + L.val_pool + g0 * n_leaf * (size_t)D * esz;
            int32_t *kept_leaf_row = reinterpret_cast<int32_t *>(ws + L.kept_leaf_row) + bh0 * p->K_leaf;
            d.keys[2] = pool;
            d.slot[2] = k.leaf_slot;
            d.kept_leaf_row = kept_leaf_row;
            k.uroot = k.croot = k.mid_slot = nullptr;
            if (t->host_mids) {
                k.mid_slot = reinterpret_cast<int32_t *>(ws + L.mid_slot) + bh0 * p->K_root;
                k.uroot = reinterpret_cast<int32_t *>(ws + L.uroot) + g0 * n_root;
                k.croot = reinterpret_cast<int32_t *>(ws + L.ucount_root) + g0;
                d.keys[1] = ws + L.mid_pool + g0 * n_root * (size_t)t->d.fanout[1] * D * esz;
                d.slot[1] = k.mid_slot;
            }
            k.d = d;
            akv::AttnParams a = ap;
            a.B = Bc;
            const size_t qoff = (size_t)b0 * io->N * io->H * D * esz, kvoff = (size_t)b0 * io->T * H_kv * D * esz;
            a.q_kg = reinterpret_cast<const uint8_t *>(io->q_kg) + qoff;
            a.q_seq = reinterpret_cast<const uint8_t *>(io->q_seq) + qoff;
            a.out = reinterpret_cast<uint8_t *>(io->out) + qoff;
            a.lse = io->lse ? io->lse + (size_t)b0 * io->N * io->H : nullptr;
            a.oseq = ap.oseq ? ap.oseq + (size_t)b0 * io->N * io->H * D : nullptr;
            a.lse_seq = ap.lse_seq ? ap.lse_seq + (size_t)b0 * io->N * io->H : nullptr;
            a.k_seq = reinterpret_cast<const uint8_t *>(io->k_seq) + kvoff;
            a.v_seq = reinterpret_cast<const uint8_t *>(io->v_seq) + kvoff;
            a.lk_base = pool;
            a.lv_base = vpool;
            a.lk_idx = kept_leaf_row;
            a.lv_idx = k.vslot;
            a.leaf_head_stride = 0;
            a.lk_rows = (long long)k.groups * n_mid * t->d.fanout[2];
            a.lv_rows = (long long)k.groups * n_leaf;
            if (t->split) a.mode = akv::kAttnLeaf;
            k.a = a;
        }
        // The pipeline of one chunk: descent ranges on the caller's stream
        // alternate with stagings on the staging stream; each phase waits for
        // the chunk's previous one.  Mids in host memory:  levels 0 | stage the
        // kept roots' mid blocks | level 1 | stage the kept mids' leaf blocks |
        // level 2 | stage the kept leaves' values | knowledge part.  Only the
        // leaves:  levels 0-1 | leaf blocks | level 2 | values | knowledge part.
        int np = 0;
        auto add = [&](int kind, int first, int last) { t->phase[np++] = {kind, first, last}; };
        if (t->host_mids) {
            add(kPhaseDescend, 0, 0);
            add(kPhaseStageKeys, 1, 1);
            add(kPhaseDescend, 1, 1);
        } else {
            add(kPhaseDescend, 0, 1);
        }
        add(kPhaseStageKeys, 2, 2);
        add(kPhaseDescend, 2, 2);
        add(kPhaseStageValues, 0, 0);
        add(kPhaseAttend, 0, 0);
        t->nphases_last = np;
        // the staging stream starts after everything already queued on the caller's stream
        AKV_CUDA(cudaEventRecord(t->cev[kMaxChunks * kChunkEvents], s));
        AKV_CUDA(cudaStreamWaitEvent(s1, t->cev[kMaxChunks * kChunkEvents], 0));
        if (t->split) {
            AKV_CUDA(cudaEventRecord(t->fev[0], s));
            AKV_STEP(fork_sequence_part());
        }
        if (t->cache_pool) ++t->cache_epoch;   // this call's stamp (epoch 0 marks empty ways)
        for (int k = 0; k < np; ++k) {
            const Phase ph = t->phase[k];
            const bool on_stage = ph.kind == kPhaseStageKeys || ph.kind == kPhaseStageValues;
            cudaStream_t st = on_stage ? s1 : s;
            if (ph.kind == kPhaseAttend && t->split) AKV_CUDA(cudaStreamWaitEvent(s, t->fev[2], 0));
            for (int c = 0; c < nc; ++c) {
                Chunk &q = ch[c];
                if (k > 0) AKV_CUDA(cudaStreamWaitEvent(st, cev(c, k - 1), 0));
                AKV_STEP(tmark(c, 2 * k, st));
                switch (ph.kind) {
                case kPhaseDescend:
                    if (L.pm)
                        AKV_STEP(dispatch_pm(t, L.pmp, q.d, q.lv, ws + L.pm_zero + c * L.pmp.zero_bytes,
                                             L.pmp.zero_bytes, ph.first, ph.last, s));
                    else AKV_STEP(dispatch_descend(t->d.dtype, D, q.d, L.desc.HT, L.desc.smem, ph.first, ph.last, s));
                    break;
                case kPhaseStageKeys:
                    if (ph.first == 1) {
                        AKV_STEP(launch_dedupe(q.d.kept[0], n_root, q.groups, q.uroot, q.mid_slot, q.croot, s1));
                        AKV_STEP(dispatch_stage_keys(t, 1, q.uroot, q.croot, n_root, q.groups,
                                                     const_cast<void *>(q.d.keys[1]), s1));
                    } else {
                        AKV_STEP(launch_dedupe(q.d.kept[1], n_mid, q.groups, q.umid, q.leaf_slot, q.cmid, s1));
                        if (t->cache_pool) {
                            AKV_STEP(cache_map(t, q.umid, q.cmid, n_mid, q.groups, q.csrc, q.cfill, s1));
                            AKV_STEP(dispatch_stage_keys(t, 2, q.umid, q.cmid, n_mid, q.groups,
                                                         const_cast<void *>(q.d.keys[2]), s1, q.csrc, q.cfill));
                            AKV_STEP(cache_commit(t, q.cmid, n_mid, q.groups, q.cfill, s1));
                        } else {
                            AKV_STEP(dispatch_stage_keys(t, 2, q.umid, q.cmid, n_mid, q.groups,
                                                         const_cast<void *>(q.d.keys[2]), s1));
                        }
                    }
                    break;
                case kPhaseStageValues:
                    AKV_STEP(launch_dedupe(q.d.kept[2], n_leaf, q.groups, q.uleaf, q.vslot, q.cleaf, s1));
                    AKV_STEP(dispatch_stage_values(t, q.uleaf, q.cleaf, n_leaf, q.groups,
                                                   const_cast<void *>(q.a.lv_base), s1));
                    break;
                default:
                    AKV_STEP(dispatch_attend(t->d.dtype, D, q.a, s));
                    break;
                }
                AKV_STEP(tmark(c, 2 * k + 1, st));
                if (k + 1 < np) AKV_CUDA(cudaEventRecord(cev(c, k), st));
            }
        }
        t->chunks_last = nc;
    }
#undef AKV_STEP
    t->timed = prof;
    t->counted = t->counting;
    t->host_mode_last = host;
    return ATLASKV_OK;
}

}  // namespace

extern "C" {

atlaskv_status atlaskv_attend(atlaskv_tree *t, const atlaskv_params *p, const atlaskv_io *io, void *workspace,
                              size_t ws_bytes, void *stream)
{
    if (!p || !io) return fail(ATLASKV_EINVAL, "null params or io");
    if (t && t->csr) return fail(ATLASKV_EINVAL, "a CSR tree is attended with atlaskv_attend_csr");
    int32_t *kept[3] = {io->kept_root, io->kept_mid, io->kept_leaf};
    return attend_impl(t, ks_of(p), io, kept, workspace, ws_bytes, stream);
}

// ---- several layers in one call ----------------------------------------------
namespace {

// Checks shared by the two layer entry points; on OK, offs[l] is layer l's
// workspace offset and offs[n] the total.
atlaskv_status check_layers(int32_t n, atlaskv_tree *const *trees, const atlaskv_params *p, const atlaskv_io *ios,
                            size_t *offs)
{
    if (n < 1 || n > akv::kMaxLayers) return fail(ATLASKV_EINVAL, "n_layers = %d not in [1, %d]", n, akv::kMaxLayers);
    if (!trees || !p || !ios) return fail(ATLASKV_EINVAL, "null trees, params or ios");
    const atlaskv_tree *t0 = trees[0];
    size_t off = 0;
    for (int l = 0; l < n; ++l) {
        const atlaskv_tree *t = trees[l];
        if (!t) return fail(ATLASKV_EINVAL, "null tree of layer %d", l);
        if (t->host_leaves) return fail(ATLASKV_EUNSUPPORTED, "layer %d: host-resident levels are not batched", l);
        if (t->d.dtype != t0->d.dtype || t->d.head_dim != t0->d.head_dim || t->d.n_kv_heads != t0->d.n_kv_heads)
            return fail(ATLASKV_EINVAL, "layer %d: dtype, head_dim and n_kv_heads must match layer 0", l);
        const atlaskv_io &io = ios[l];
        if (io.B != ios[0].B || io.N != ios[0].N || io.H != ios[0].H || io.T != ios[0].T)
            return fail(ATLASKV_EINVAL, "layer %d: B, N, H and T must match layer 0", l);
        if (t->csr) return fail(ATLASKV_EUNSUPPORTED, "layer %d: CSR trees are not batched", l);
        atlaskv_status st = check_params(t, ks_of(p), io.B, io.N, io.H, io.T);
        if (st != ATLASKV_OK) return st;
        const Layout Lf = plan(t, ks_of(p), io.B, io.N, io.H, io.T, false);
        if (Lf.desc.GC == 0)
            return fail(ATLASKV_EUNSUPPORTED, "layer %d: the fused descent's plan does not fit for these K", l);
        offs[l] = off;
        off = align256(off + Lf.total);
    }
    offs[n] = off;
    return ATLASKV_OK;
}

}  // namespace

atlaskv_status atlaskv_workspace_size_layers(int32_t n_layers, atlaskv_tree *const *trees, const atlaskv_params *params,
                                             const atlaskv_io *ios, size_t *bytes)
{
    if (!bytes) return fail(ATLASKV_EINVAL, "null bytes");
    size_t offs[akv::kMaxLayers + 1];
    const atlaskv_status st = check_layers(n_layers, trees, params, ios, offs);
    if (st != ATLASKV_OK) return st;
    *bytes = offs[n_layers];
    return ATLASKV_OK;
}

atlaskv_status atlaskv_attend_layers(int32_t n_layers, atlaskv_tree *const *trees, const atlaskv_params *p,
                                     const atlaskv_io *ios, void *workspace, size_t ws_bytes, void *stream)
{
    size_t offs[akv::kMaxLayers + 1];
    atlaskv_status st = check_layers(n_layers, trees, p, ios, offs);
    if (st != ATLASKV_OK) return st;
    if (ios[0].B == 0) return ATLASKV_OK;
    for (int l = 0; l < n_layers; ++l) {
        st = check_io(&ios[l]);
        if (st != ATLASKV_OK) return st;
    }
    if (!workspace || ((uintptr_t)workspace & 255u)) return fail(ATLASKV_EINVAL, "workspace must be 256-byte aligned");
    if (ws_bytes < offs[n_layers])
        return fail(ATLASKV_ENOMEM, "workspace of %zu bytes, %zu needed", ws_bytes, offs[n_layers]);
    static Call calls[akv::kMaxLayers];   // large: not on the stack
    static akv::DescendBatch db;
    static std::mutex m;
    std::lock_guard<std::mutex> lock(m);
    uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
    for (int l = 0; l < n_layers; ++l) {
        const Ks ks = ks_of(p);
        int32_t *kept[3] = {ios[l].kept_root, ios[l].kept_mid, ios[l].kept_leaf};
        calls[l].L = plan(trees[l], ks, ios[l].B, ios[l].N, ios[l].H, ios[l].T, false);
        fill_call(trees[l], ks, &ios[l], kept, ws + offs[l], calls[l]);
    }
    // one descent launch: every layer's plan is the same (same shapes and K)
    const DescPlan &pl = calls[0].L.desc;
    for (int l = 1; l < n_layers; ++l)
        if (calls[l].L.desc.GC != pl.GC || calls[l].L.desc.smem != pl.smem)
            return fail(ATLASKV_EINVAL, "layer %d: descent plan differs from layer 0 (fan-outs must allow the same "
                                        "shared-memory plan)", l);
    const long long per = (long long)ios[0].B * trees[0]->d.n_kv_heads * (ios[0].H / trees[0]->d.n_kv_heads / pl.GC);
    if (per * n_layers > 0x7fffffffLL) return fail(ATLASKV_EUNSUPPORTED, "descent grid too large");
    db.n = n_layers;
    for (int l = 0; l < n_layers; ++l) {
        db.p[l] = calls[l].dp;
        db.offs[l] = (unsigned)(per * l);
    }
    db.offs[n_layers] = (unsigned)(per * n_layers);

    atlaskv_tree *t0 = trees[0];
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int D = t0->d.head_dim;
    const bool prof = t0->profiling;
    auto tm = [&](int i, cudaStream_t st2) -> atlaskv_status {
        if (prof) AKV_CUDA(cudaEventRecord(t0->ev[i], st2));
        return ATLASKV_OK;
    };
#define AKV_STEP(x)                            \
    do {                                       \
        atlaskv_status st_ = (x);              \
        if (st_ != ATLASKV_OK) return st_;     \
    } while (0)
    for (int l = 0; l < n_layers; ++l)
        if (trees[l]->counting) AKV_CUDA(cudaMemsetAsync(trees[l]->stats, 0, kNumCounters * sizeof(unsigned long long), s));
    const unsigned dgrid = (unsigned)(per * n_layers);
    if (t0->split) {
        // as one call: descent (all layers) on layer 0's high-priority stream,
        // sequence parts on its low-priority stream, knowledge parts on `stream`
        AKV_CUDA(cudaEventRecord(t0->fev[0], s));
        AKV_CUDA(cudaStreamWaitEvent(t0->desc_stream, t0->fev[0], 0));
        AKV_CUDA(cudaStreamWaitEvent(t0->seq_stream, t0->fev[0], 0));
        AKV_STEP(tm(0, t0->desc_stream));
        AKV_STEP(dispatch_descend_layers(t0->d.dtype, D, db, pl.HT, pl.smem, dgrid, t0->desc_stream));
        AKV_STEP(tm(1, t0->desc_stream));
        AKV_CUDA(cudaEventRecord(t0->fev[1], t0->desc_stream));
        AKV_STEP(tm(2, t0->seq_stream));
        AKV_STEP(D == 64 ? launch_attend_tc_layers<64>(calls, n_layers, akv::kAttnSeq, t0->seq_stream)
                         : launch_attend_tc_layers<128>(calls, n_layers, akv::kAttnSeq, t0->seq_stream));
        AKV_STEP(tm(3, t0->seq_stream));
        AKV_CUDA(cudaEventRecord(t0->fev[2], t0->seq_stream));
        AKV_CUDA(cudaStreamWaitEvent(s, t0->fev[1], 0));
        AKV_CUDA(cudaStreamWaitEvent(s, t0->fev[2], 0));
        AKV_STEP(tm(4, s));
        AKV_STEP(D == 64 ? launch_attend_tc_layers<64>(calls, n_layers, akv::kAttnLeaf, s)
                         : launch_attend_tc_layers<128>(calls, n_layers, akv::kAttnLeaf, s));
        AKV_STEP(tm(5, s));
    } else {
        AKV_STEP(tm(0, s));
        AKV_STEP(dispatch_descend_layers(t0->d.dtype, D, db, pl.HT, pl.smem, dgrid, s));
        AKV_STEP(tm(1, s));
        AKV_STEP(tm(4, s));
        if (t0->d.dtype == ATLASKV_BF16)   // every layer's attention in one launch
            AKV_STEP(D == 64 ? launch_attend_tc_layers<64>(calls, n_layers, akv::kAttnFused, s)
                             : launch_attend_tc_layers<128>(calls, n_layers, akv::kAttnFused, s));
        else
            for (int l = 0; l < n_layers; ++l) AKV_STEP(dispatch_attend(t0->d.dtype, D, calls[l].ap, s));
        AKV_STEP(tm(5, s));
    }
#undef AKV_STEP
    for (int l = 0; l < n_layers; ++l) {
        trees[l]->timed = l == 0 && prof;
        trees[l]->counted = trees[l]->counting;
        trees[l]->host_mode_last = false;
    }
    return ATLASKV_OK;
}

atlaskv_status atlaskv_sync_status(atlaskv_tree *t, void *stream)
{
    if (!t) return fail(ATLASKV_EINVAL, "null tree");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int v = 0;
    AKV_CUDA(cudaMemcpyAsync(&v, t->status, sizeof(int), cudaMemcpyDeviceToHost, s));
    AKV_CUDA(cudaStreamSynchronize(s));
    if (v == akv::kDevBadChild) return fail(ATLASKV_EDEVICE, "a child id was out of range on the device");
    if (v == akv::kDevTimeout) return fail(ATLASKV_ETIMEOUT, "a bounded device wait gave up");
    if (v == akv::kDevBadSmem) return fail(ATLASKV_EDEVICE, "the attention kernel's shared memory base was not 1024-byte aligned");
    if (v != akv::kDevOk) return fail(ATLASKV_EDEVICE, "device status %d", v);
    return ATLASKV_OK;
}

atlaskv_status atlaskv_set_profiling(atlaskv_tree *t, int32_t enable)
{
    if (!t) return fail(ATLASKV_EINVAL, "null tree");
    if ((enable & ATLASKV_PROFILE_TIMES) && !t->ev[0])
        for (int i = 0; i < kNumEvents; ++i) AKV_CUDA(cudaEventCreate(&t->ev[i]));
    if ((enable & ATLASKV_PROFILE_TIMES) && t->host_leaves && !t->tev[0])
        for (cudaEvent_t &e : t->tev) AKV_CUDA(cudaEventCreate(&e));
    t->profiling = (enable & ATLASKV_PROFILE_TIMES) != 0;
    t->counting = (enable & ATLASKV_PROFILE_COUNTERS) != 0;
    return ATLASKV_OK;
}

atlaskv_status atlaskv_set_leaf_cache(atlaskv_tree *t, int64_t blocks, void *stream)
{
    if (!t) return fail(ATLASKV_EINVAL, "null tree");
    if (blocks < 0) return fail(ATLASKV_EINVAL, "blocks = %lld < 0", (long long)blocks);
    if (blocks > 0 && (!t->host_leaves || t->csr))
        return fail(ATLASKV_EUNSUPPORTED, "the leaf-block cache is for three-level trees with host-resident leaves");
    if (blocks > 0 && (long long)t->d.n_kv_heads * t->rows[1] >= (1LL << 31) - 1)
        return fail(ATLASKV_EUNSUPPORTED, "too many mids for the cache's keys");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    AKV_CUDA(cudaStreamSynchronize(s));
    if (t->stage_stream) AKV_CUDA(cudaStreamSynchronize(t->stage_stream));
    if (t->cache_tag) AKV_CUDA(cudaFree(t->cache_tag));
    if (t->cache_pool) AKV_CUDA(cudaFree(t->cache_pool));
    if (t->cache_stats) AKV_CUDA(cudaFree(t->cache_stats));
    t->cache_tag = nullptr;
    t->cache_pool = nullptr;
    t->cache_stats = nullptr;
    t->cache_sets = 0;
    t->cache_epoch = 0;
    if (blocks == 0) return ATLASKV_OK;
    long long sets = 1;
    while (sets * akv::kCacheWays < blocks) sets <<= 1;
    const size_t slots = (size_t)sets * akv::kCacheWays;
    const size_t block_bytes = (size_t)t->d.fanout[2] * t->d.head_dim * esize(t->d.dtype);
    cudaError_t e = cudaMalloc(&t->cache_pool, slots * block_bytes);
    if (e == cudaSuccess) e = cudaMalloc(&t->cache_tag, slots * 8);
    if (e == cudaSuccess) e = cudaMalloc(&t->cache_stats, 3 * sizeof(unsigned long long));
    if (e == cudaSuccess) e = cudaMemsetAsync(t->cache_tag, 0, slots * 8, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(t->cache_stats, 0, 3 * sizeof(unsigned long long), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
        cudaGetLastError();
        if (t->cache_pool) cudaFree(t->cache_pool);
        if (t->cache_tag) cudaFree(t->cache_tag);
        if (t->cache_stats) cudaFree(t->cache_stats);
        t->cache_pool = nullptr;
        t->cache_tag = nullptr;
        t->cache_stats = nullptr;
        return fail(ATLASKV_ENOMEM, "leaf-block cache of %zu blocks: %s", slots, cudaGetErrorString(e));
    }
    t->cache_sets = sets;
    return ATLASKV_OK;
}

atlaskv_status atlaskv_leaf_cache_stats(atlaskv_tree *t, uint64_t *counts, int32_t n)
{
    if (!t || !counts || n < 0) return fail(ATLASKV_EINVAL, "null tree or counts");
    if (!t->cache_stats) return fail(ATLASKV_EINVAL, "the tree has no leaf-block cache");
    unsigned long long v[3];
    AKV_CUDA(cudaDeviceSynchronize());
    AKV_CUDA(cudaMemcpy(v, t->cache_stats, sizeof(v), cudaMemcpyDeviceToHost));
    for (int i = 0; i < n && i < 3; ++i) counts[i] = v[i];
    return ATLASKV_OK;
}

atlaskv_status atlaskv_set_descent(atlaskv_tree *t, int32_t mode)
{
    if (!t) return fail(ATLASKV_EINVAL, "null tree");
    if (mode != ATLASKV_DESCENT_AUTO && mode != ATLASKV_DESCENT_FUSED && mode != ATLASKV_DESCENT_PARENT_MAJOR)
        return fail(ATLASKV_EINVAL, "unknown descent mode %d", mode);
    t->descent_mode = mode;
    return ATLASKV_OK;
}

atlaskv_status atlaskv_stage_times(atlaskv_tree *t, float *ms, int32_t n)
{
    if (!t || !ms || n < 1) return fail(ATLASKV_EINVAL, "null tree/ms or n < 1");
    if (!t->timed) return fail(ATLASKV_EINVAL, "no attend call was timed (enable profiling first)");
    float v[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
    if (!t->host_mode_last) {
        AKV_CUDA(cudaEventSynchronize(t->ev[5]));   // the caller's stream joined every other stream before it
        AKV_CUDA(cudaEventElapsedTime(&v[0], t->ev[0], t->ev[1]));
        AKV_CUDA(cudaEventElapsedTime(&v[4], t->ev[4], t->ev[5]));
    } else {
        // busy time of each kind of segment, summed over the query chunks
        // (segments of different kinds overlap on the two streams)
        const int nc = t->chunks_last, np = t->nphases_last;
        AKV_CUDA(cudaEventSynchronize(t->tev[(nc - 1) * kTimingEvents + 2 * np - 1]));
        for (int c = 0; c < nc; ++c)
            for (int k = 0; k < np; ++k) {
                float seg = 0.f;
                AKV_CUDA(cudaEventElapsedTime(&seg, t->tev[c * kTimingEvents + 2 * k],
                                              t->tev[c * kTimingEvents + 2 * k + 1]));
                const int kind = t->phase[k].kind;
                v[kind == kPhaseDescend ? 0 : kind == kPhaseAttend ? 4 : 1] += seg;
            }
    }
    if (t->split) AKV_CUDA(cudaEventElapsedTime(&v[3], t->ev[2], t->ev[3]));
    v[2] = v[3] + v[4];
    for (int i = 0; i < n && i < 5; ++i) ms[i] = v[i];
    return ATLASKV_OK;
}

atlaskv_status atlaskv_refine_stats(atlaskv_tree *t, uint64_t *counts, int32_t n)
{
    if (!t || !counts || n < 1) return fail(ATLASKV_EINVAL, "null tree/counts or n < 1");
    if (!t->counted) return fail(ATLASKV_EINVAL, "no attend call kept counters (enable ATLASKV_PROFILE_COUNTERS first)");
    unsigned long long v[kNumCounters];
    AKV_CUDA(cudaMemcpy(v, t->stats, sizeof v, cudaMemcpyDeviceToHost));
    for (int i = 0; i < n && i < kNumCounters; ++i) counts[i] = v[i];
    return ATLASKV_OK;
}

atlaskv_status atlaskv_probe_wait_timeout(atlaskv_tree *t, void *stream)
{
    if (!t) return fail(ATLASKV_EINVAL, "null tree");
    akv::wait_timeout_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(t->status);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

atlaskv_status atlaskv_destroy(atlaskv_tree *t)
{
    if (!t) return ATLASKV_OK;
    if (t->norm_bound) cudaFree(t->norm_bound);
    if (t->status) cudaFree(t->status);
    if (t->stats) cudaFree(t->stats);
    if (t->cache_tag) cudaFree(t->cache_tag);
    if (t->cache_pool) cudaFree(t->cache_pool);
    if (t->cache_stats) cudaFree(t->cache_stats);
    for (int i = 0; i < kNumEvents; ++i)
        if (t->ev[i]) cudaEventDestroy(t->ev[i]);
    for (cudaEvent_t e : t->cev)
        if (e) cudaEventDestroy(e);
    for (cudaEvent_t e : t->tev)
        if (e) cudaEventDestroy(e);
    if (t->stage_stream) cudaStreamDestroy(t->stage_stream);
    if (t->seq_stream) cudaStreamDestroy(t->seq_stream);
    if (t->desc_stream) cudaStreamDestroy(t->desc_stream);
    for (cudaEvent_t e : t->fev)
        if (e) cudaEventDestroy(e);
    delete t;
    return ATLASKV_OK;
}

}  // extern "C"
