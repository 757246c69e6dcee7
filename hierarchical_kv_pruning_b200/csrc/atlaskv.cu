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
#include <new>
#include <string>

#include "atlaskv.h"
#include "attend.cuh"
#include "attend_tc.cuh"
#include "descend.cuh"
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

int pow2_at_least(long long x, int floor_)
{
    int p = floor_;
    while (p < x) p <<= 1;
    return p;
}

constexpr int kMaxCandidates = 8192;   // per level and traversal (shared-memory bound of the descent CTA)
constexpr int kNumEvents = 6;
// Host-resident leaves: the batch is split into up to kMaxChunks query chunks
// so that staging one chunk's leaf blocks over the host link overlaps the
// scoring and attention of the others (a second stream owned by the tree).
constexpr int kMaxChunks = 4;
constexpr int kChunkEvents = 4;          // per chunk: mids kept, keys staged, leaves kept, values staged
constexpr int kTimingEvents = 10;        // per chunk: begin / end of 5 segments

}  // namespace

atlaskv_status akv_report(atlaskv_status st, const char *msg)
{
    g_last_error = msg;
    return st;
}

struct atlaskv_tree {
    atlaskv_tree_desc d;
    long long rows[3];
    const void *leaf_keys_dev;     // device-accessible leaf pointers (mapped for host leaves)
    const void *leaf_values_dev;
    float *norm_bound;             // device [3][H_kv]
    int *status;                   // device sticky status word
    unsigned long long *stats;     // device [3][4] descent counters (filled while profiling)
    bool profiling;
    bool timed;                    // the last attend recorded events
    bool host_mode_last;
    int chunks_last;
    cudaEvent_t ev[kNumEvents];
    cudaStream_t stage_stream;                        // host leaves: staging copies
    cudaEvent_t cev[kMaxChunks * kChunkEvents + 1];   // cross-stream ordering (+1: start)
    cudaEvent_t tev[kMaxChunks * kTimingEvents];      // segment timing while profiling
};

namespace {

size_t esize(int dtype) { return dtype == ATLASKV_F32 ? 4 : 2; }

struct Layout {
    size_t s_ws, s64_ws, a64_ws, anorm_ws, f_ws, queue, qcount, kept[3], leaf_slot, kept_leaf_row, vslot, umid,
        ucount_mid, uleaf, ucount_leaf, key_pool, val_pool, total;
    int cap, kcap, fstride;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

Layout plan(const atlaskv_tree *t, const atlaskv_params *p, int B, int N, int H, int T)
{
    (void)N;
    (void)T;
    Layout L{};
    const size_t BH = (size_t)B * H;
    const int D = t->d.head_dim;
    const bool host = t->d.leaf_location == ATLASKV_LEAVES_HOST_PINNED;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    const long long cmax = std::max<long long>(t->d.fanout[0], std::max<long long>((long long)p->K_root * t->d.fanout[1],
                                                                                  (long long)p->K_mid * t->d.fanout[2]));
    L.cap = (int)((cmax + 3) & ~3LL);
    L.kcap = pow2_at_least(std::max(p->K_root, std::max(p->K_mid, p->K_leaf)), 32);
    L.fstride = L.cap + 2 * L.kcap;
    L.s_ws = take(BH * D * 4);
    L.s64_ws = take(BH * D * 8);
    L.a64_ws = take(BH * D * 8);
    L.anorm_ws = take(BH * 4);
    L.f_ws = take(BH * (size_t)L.fstride * 4);
    L.queue = take(3 * BH * 4 * 4);
    L.qcount = take(kMaxChunks * 4 * 4);   // per query chunk: [3] exact-pass queue lengths
    for (int l = 0; l < 3; ++l) L.kept[l] = take(BH * (size_t)(l == 0 ? p->K_root : l == 1 ? p->K_mid : p->K_leaf) * 4);
    if (host) {
        const int G = H / t->d.n_kv_heads;
        const size_t groups = (size_t)B * t->d.n_kv_heads;
        const size_t n_mid = (size_t)G * p->K_mid, n_leaf = (size_t)G * p->K_leaf;
        L.leaf_slot = take(BH * p->K_mid * 4);
        L.kept_leaf_row = take(BH * p->K_leaf * 4);
        L.vslot = take(BH * p->K_leaf * 4);
        L.umid = take(groups * n_mid * 4);
        L.ucount_mid = take(groups * 4);
        L.uleaf = take(groups * n_leaf * 4);
        L.ucount_leaf = take(groups * 4);
        L.key_pool = take(groups * n_mid * (size_t)t->d.fanout[2] * D * esize(t->d.dtype));
        L.val_pool = take(groups * n_leaf * D * esize(t->d.dtype));
    }
    L.total = off;
    return L;
}

atlaskv_status check_params(const atlaskv_tree *t, const atlaskv_params *p, int B, int N, int H, int T)
{
    if (!t || !p) return fail(ATLASKV_EINVAL, "null tree or params");
    const int *fo = t->d.fanout;
    if (B < 0) return fail(ATLASKV_EINVAL, "B = %d < 0", B);
    if (H < 1 || H % t->d.n_kv_heads != 0)
        return fail(ATLASKV_EINVAL, "H = %d is not a positive multiple of H_kv = %d", H, t->d.n_kv_heads);
    if (N < 1 || N > T) return fail(ATLASKV_EINVAL, "need 1 <= N <= T (N = %d, T = %d)", N, T);
    if (N > 65535) return fail(ATLASKV_EUNSUPPORTED, "N = %d above 65535", N);
    if (p->K_root < 1 || p->K_root > fo[0]) return fail(ATLASKV_EINVAL, "K_root = %d not in [1, b_R = %d]", p->K_root, fo[0]);
    if (p->K_mid < 1 || (long long)p->K_mid > (long long)p->K_root * fo[1])
        return fail(ATLASKV_EINVAL, "K_mid = %d not in [1, K_root * b_I = %lld]", p->K_mid, (long long)p->K_root * fo[1]);
    if (p->K_leaf < 1 || (long long)p->K_leaf > (long long)p->K_mid * fo[2])
        return fail(ATLASKV_EINVAL, "K_leaf = %d not in [1, K_mid * b_L = %lld]", p->K_leaf, (long long)p->K_mid * fo[2]);
    const long long c1 = (long long)p->K_root * fo[1], c2 = (long long)p->K_mid * fo[2];
    if (fo[0] > kMaxCandidates || c1 > kMaxCandidates || c2 > kMaxCandidates)
        return fail(ATLASKV_EUNSUPPORTED, "a level has more than %d candidates per traversal (%d, %lld, %lld)",
                    kMaxCandidates, fo[0], c1, c2);
    if (!(p->scale >= 0.f) || std::isinf(p->scale)) return fail(ATLASKV_EINVAL, "scale must be finite and >= 0");
    if ((long long)B * H > (1LL << 31) - 1) return fail(ATLASKV_EUNSUPPORTED, "B * H too large");
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
    const void *lv[3] = {t->d.root_keys, t->d.mid_keys, t->leaf_keys_dev};
    for (int l = 0; l < 3; ++l) {
        atlaskv_status st = launch_norms<T, D>(t, lv[l], t->rows[l], l, s);
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

// ---- descent launches -----------------------------------------------------
// Scoring CTAs serve GP query heads of a (query, KV head) group: the largest
// of 4, 2, 1 that divides G.  Selection runs one CTA per traversal.
int heads_per_cta(int G) { return G % 4 == 0 ? 4 : (G % 2 == 0 ? 2 : 1); }

template <typename T, int D, int GP>
atlaskv_status launch_root(const akv::DescendParams &dp, cudaStream_t s)
{
    const long long grid = (long long)dp.B * dp.H_kv * (dp.G / GP);
    const size_t smem = akv::root_kernel_smem<T, D, GP>();
    akv::root_kernel<T, D, GP><<<(unsigned)grid, akv::kScoreThreads, smem, s>>>(dp);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

// Children scoring: one CTA per (query, KV head, chunk of GC <= 32 heads,
// parent chunk); a warp serves HT heads (HT = GC rounded up to a power of two,
// at most 8).
template <typename T, int D, int HT>
atlaskv_status launch_score_ht(const akv::DescendParams &dp, int L, int GC, cudaStream_t s)
{
    const int Kp = dp.K[L - 1], fo = dp.fanout[L];
    const int ppc = std::max(1, 2048 / fo);           // parents per chunk: about 2048 rows per CTA
    const int pchunks = (Kp + ppc - 1) / ppc;         // covers a union of Kp parents; larger ones loop
    const long long grid = (long long)dp.B * dp.H_kv * (dp.G / GC) * pchunks;
    if (grid > 0x7fffffffLL) return fail(ATLASKV_EUNSUPPORTED, "scoring grid too large");
    const size_t smem = akv::score_kernel_smem<D, (int)sizeof(T)>(GC, Kp);
    if (smem > 227 * 1024) return fail(ATLASKV_EUNSUPPORTED, "scoring needs %zu bytes of shared memory", smem);
    // per device and cheap: set whenever the launch needs more than the default 48 KB
    if (smem > 48 * 1024) {
        AKV_CUDA(cudaFuncSetAttribute(akv::score_kernel<T, D, HT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem));
    }
    akv::score_kernel<T, D, HT><<<(unsigned)grid, akv::kScoreThreads, smem, s>>>(dp, L, GC, ppc, pchunks);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

template <typename T, int D>
atlaskv_status launch_score(const akv::DescendParams &dp, int L, cudaStream_t s)
{
    int GC = 1;
    for (int c = std::min(dp.G, 32); c >= 1; --c)
        if (dp.G % c == 0) {
            GC = c;
            break;
        }
    if (GC <= 1) return launch_score_ht<T, D, 1>(dp, L, GC, s);
    if (GC <= 2) return launch_score_ht<T, D, 2>(dp, L, GC, s);
    if (GC <= 4) return launch_score_ht<T, D, 4>(dp, L, GC, s);
    return launch_score_ht<T, D, 8>(dp, L, GC, s);
}

template <typename T, int D>
atlaskv_status launch_select(const akv::DescendParams &dp, int L, cudaStream_t s)
{
    const long long BH = (long long)dp.B * dp.H;
    const long long grid = BH;   // one CTA per traversal
    if (grid > 0x7fffffffLL) return fail(ATLASKV_EUNSUPPORTED, "selection grid too large");
    const size_t smem = akv::SelectScratch::bytes(dp.cap, dp.kcap, D);
    if (smem > 227 * 1024)
        return fail(ATLASKV_EUNSUPPORTED, "selection needs %zu bytes of shared memory per CTA", smem);
    // few traversals: 64 threads each (shorter barriers); many: 128 (shorter chains)
    auto run = [&](auto kern, int nt) -> atlaskv_status {
        if (smem > 48 * 1024)
            AKV_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        kern<<<(unsigned)grid, nt, smem, s>>>(dp, L);
        AKV_CUDA(cudaGetLastError());
        return ATLASKV_OK;
    };
    const atlaskv_status st =
        BH <= 4096 ? run(akv::select_kernel<T, D, 64>, 64) : run(akv::select_kernel<T, D, 128>, 128);
    if (st != ATLASKV_OK) return st;
    // tier 3 for whatever the bounds left undecided (usually nothing: the warps read an empty queue)
    const size_t esmem = (size_t)akv::kSelectWarps * akv::ExactScratch::bytes(dp.kcap, D);
    if (esmem > 48 * 1024) {
        AKV_CUDA(cudaFuncSetAttribute(akv::exact_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)esmem));
    }
    const long long egrid = std::min<long long>((BH + akv::kSelectWarps - 1) / akv::kSelectWarps, 2 * 148);
    akv::exact_kernel<T, D><<<(unsigned)egrid, akv::kSelectWarps * 32, esmem, s>>>(dp, L);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

// Run levels [first, last] of the descent (scores then selection per level).
template <typename T, int D>
atlaskv_status descend_levels(const akv::DescendParams &dp, int first, int last, cudaStream_t s)
{
    const int gp = heads_per_cta(dp.G);
    for (int L = first; L <= last; ++L) {
        atlaskv_status st;
        if (L == 0)
            st = gp == 4 ? launch_root<T, D, 4>(dp, s) : gp == 2 ? launch_root<T, D, 2>(dp, s) : launch_root<T, D, 1>(dp, s);
        else
            st = launch_score<T, D>(dp, L, s);
        if (st != ATLASKV_OK) return st;
        st = launch_select<T, D>(dp, L, s);
        if (st != ATLASKV_OK) return st;
    }
    return ATLASKV_OK;
}

atlaskv_status dispatch_descend(int dtype, int D, const akv::DescendParams &dp, int first, int last, cudaStream_t s)
{
    if (dtype == ATLASKV_F32)
        return D == 64 ? descend_levels<float, 64>(dp, first, last, s) : descend_levels<float, 128>(dp, first, last, s);
    return D == 64 ? descend_levels<__nv_bfloat16, 64>(dp, first, last, s)
                   : descend_levels<__nv_bfloat16, 128>(dp, first, last, s);
}

// ---- attention launch -----------------------------------------------------
template <int D>
atlaskv_status launch_attend_bf16(const akv::AttnParams &ap, cudaStream_t s)
{
    const int nchunks = (ap.N + 15) / 16;
    const int bpg = (ap.G * nchunks + akv::kAttnWarps - 1) / akv::kAttnWarps;
    const long long grid = (long long)ap.B * ap.H_kv * bpg;
    if (grid > 0x7fffffffLL) return fail(ATLASKV_EUNSUPPORTED, "attention grid too large");
    const int smem = akv::AttnSmem<D>::BYTES;
    // the attribute is per device: set it on every launch (a cheap host call)
    AKV_CUDA(cudaFuncSetAttribute(akv::attend_bf16_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    akv::attend_bf16_kernel<D><<<(unsigned)grid, akv::kAttnWarps * 32, smem, s>>>(ap, bpg);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

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

// Tensor map of a sequence K or V tensor [B][T][H_kv][D] (bf16, D = 128) for
// the attention kernel: dims (D, H_kv, T, B), box (64, 1, 64, 1), 128-byte
// swizzle, zero fill outside.  cuTensorMapEncodeTiled is a host-only call,
// reached through the runtime's driver entry point.
atlaskv_status encode_seq_map(CUtensorMap *map, const void *base, int B, int T, int H_kv)
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
    if (reinterpret_cast<uintptr_t>(base) & 15u) return fail(ATLASKV_EINVAL, "sequence K/V must be 16-byte aligned");
    const int D = akv::tc::kD;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H_kv, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H_kv * D * 2, (cuuint64_t)T * H_kv * D * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)akv::tc::kKeys, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(ATLASKV_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return ATLASKV_OK;
}

// bf16, D = 128: tcgen05 tensor cores, one CTA per kWG x 128 query rows of a
// (query, KV head) group, sequence tiles by TMA.
atlaskv_status launch_attend_tc(const akv::AttnParams &ap, cudaStream_t s)
{
    const int rows = ap.G * ap.N;
    const int cpg = (rows + akv::tc::kCtaRows - 1) / akv::tc::kCtaRows;
    const long long grid = (long long)ap.B * ap.H_kv * cpg;
    if (grid > 0x7fffffffLL) return fail(ATLASKV_EUNSUPPORTED, "attention grid too large");
    if (ap.lk_rows >= (1LL << 31) || ap.lv_rows >= (1LL << 31))
        return fail(ATLASKV_EUNSUPPORTED, "more than 2^31 leaf rows");
    CUtensorMap mk, mv;
    atlaskv_status st = encode_seq_map(&mk, ap.k_seq, ap.B, ap.T, ap.H_kv);
    if (st != ATLASKV_OK) return st;
    st = encode_seq_map(&mv, ap.v_seq, ap.B, ap.T, ap.H_kv);
    if (st != ATLASKV_OK) return st;
    // the attribute is per device: set it on every launch (a cheap host call)
    AKV_CUDA(cudaFuncSetAttribute(akv::attend_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  akv::tc::kSmemBytes));
    akv::attend_tc_kernel<<<(unsigned)grid, akv::tc::kThreads, akv::tc::kSmemBytes, s>>>(ap, cpg, mk, mv);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

atlaskv_status dispatch_attend(int dtype, int D, const akv::AttnParams &ap, cudaStream_t s)
{
    if (dtype == ATLASKV_F32) return D == 64 ? launch_attend_f32<64>(ap, s) : launch_attend_f32<128>(ap, s);
    return D == 64 ? launch_attend_bf16<64>(ap, s) : launch_attend_tc(ap, s);
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
    // per device and cheap: set whenever the launch needs more than the default 48 KB
    if (smem > 48 * 1024) {
        AKV_CUDA(cudaFuncSetAttribute(akv::dedupe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    }
    akv::dedupe_kernel<<<groups, akv::kDedupeThreads, smem, s>>>(ids, n, n2, uniq, slot, count);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

template <typename T, int D>
atlaskv_status stage_keys(const atlaskv_tree *t, const int32_t *umid, const int32_t *cnt, int n, int groups,
                          void *pool, cudaStream_t s)
{
    akv::stage_leaf_blocks_kernel<T, D><<<akv::kStageCtasPerSm * num_sms(), 256, 0, s>>>(
        reinterpret_cast<const T *>(t->leaf_keys_dev), t->d.mid_child, t->rows[1], t->rows[2], t->d.fanout[2],
        t->d.n_kv_heads, umid, cnt, n, groups, reinterpret_cast<T *>(pool), t->status);
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

template <typename T, int D>
atlaskv_status stage_values(const atlaskv_tree *t, const int32_t *uleaf, const int32_t *cnt, int n, int groups,
                            void *vpool, cudaStream_t s)
{
    akv::stage_value_rows_kernel<T, D><<<akv::kStageCtasPerSm * num_sms(), 256, 0, s>>>(reinterpret_cast<const T *>(t->leaf_values_dev), t->rows[2],
                                                          t->d.n_kv_heads, uleaf, cnt, n, groups,
                                                          reinterpret_cast<T *>(vpool));
    AKV_CUDA(cudaGetLastError());
    return ATLASKV_OK;
}

atlaskv_status dispatch_stage_keys(const atlaskv_tree *t, const int32_t *umid, const int32_t *cnt, int n, int groups,
                                   void *pool, cudaStream_t s)
{
    const int D = t->d.head_dim;
    if (t->d.dtype == ATLASKV_F32)
        return D == 64 ? stage_keys<float, 64>(t, umid, cnt, n, groups, pool, s)
                       : stage_keys<float, 128>(t, umid, cnt, n, groups, pool, s);
    return D == 64 ? stage_keys<__nv_bfloat16, 64>(t, umid, cnt, n, groups, pool, s)
                   : stage_keys<__nv_bfloat16, 128>(t, umid, cnt, n, groups, pool, s);
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
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    atlaskv_tree *t = new (std::nothrow) atlaskv_tree();
    if (!t) return fail(ATLASKV_ENOMEM, "host allocation failed");
    t->d = *d;
    t->rows[0] = n_root;
    t->rows[1] = n_mid;
    t->rows[2] = n_leaf;
    t->leaf_keys_dev = d->leaf_keys;
    t->leaf_values_dev = d->leaf_values;
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
    }
    if (cudaMalloc(&t->norm_bound, 3 * sizeof(float) * d->n_kv_heads) != cudaSuccess ||
        cudaMalloc(&t->status, sizeof(int)) != cudaSuccess ||
        cudaMalloc(&t->stats, 12 * sizeof(unsigned long long)) != cudaSuccess) {
        cudaGetLastError();
        return bail(fail(ATLASKV_ECUDA, "device allocation of the tree's bound/status words failed"));
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
    AKV_TRYC(cudaMemsetAsync(t->norm_bound, 0, 3 * sizeof(float) * d->n_kv_heads, s));
    AKV_TRYC(cudaMemsetAsync(t->status, 0, sizeof(int), s));
    AKV_TRY(dispatch_norms(t, s));
    if (d->root_child) AKV_TRY(check_table(d->root_child, n_mid, d->n_kv_heads, n_mid, t->status, s));
    if (d->mid_child) AKV_TRY(check_table(d->mid_child, n_leaf, d->n_kv_heads, n_leaf, t->status, s));
    int dev_status = 0;
    AKV_TRYC(cudaMemcpyAsync(&dev_status, t->status, sizeof(int), cudaMemcpyDeviceToHost, s));
    AKV_TRYC(cudaStreamSynchronize(s));
    if (dev_status != akv::kDevOk)
        return bail(fail(ATLASKV_EINVAL, "child table has an out-of-range id or is not a permutation"));
    // inflate the norm bounds slightly (they were rounded up already)
    {
        float hb[3 * 64];
        const int nb = 3 * d->n_kv_heads;
        float *tmp = nb <= 192 ? hb : new (std::nothrow) float[nb];
        if (!tmp) return bail(fail(ATLASKV_ENOMEM, "host allocation failed"));
        AKV_TRYC(cudaMemcpy(tmp, t->norm_bound, nb * sizeof(float), cudaMemcpyDeviceToHost));
        for (int i = 0; i < nb; ++i) tmp[i] = nextafterf(tmp[i] * (1.0f + 0x1p-20f), INFINITY);
        AKV_TRYC(cudaMemcpy(t->norm_bound, tmp, nb * sizeof(float), cudaMemcpyHostToDevice));
        if (tmp != hb) delete[] tmp;
    }
#undef AKV_TRY
#undef AKV_TRYC
    *out = t;
    return ATLASKV_OK;
}

atlaskv_status atlaskv_workspace_size(const atlaskv_tree *t, const atlaskv_params *p, int32_t B, int32_t N, int32_t H,
                                      int32_t T, size_t *bytes)
{
    if (!bytes) return fail(ATLASKV_EINVAL, "null bytes");
    atlaskv_status st = check_params(t, p, B, N, H, T);
    if (st != ATLASKV_OK) return st;
    *bytes = plan(t, p, B, N, H, T).total;
    return ATLASKV_OK;
}

atlaskv_status atlaskv_attend(atlaskv_tree *t, const atlaskv_params *p, const atlaskv_io *io, void *workspace,
                              size_t ws_bytes, void *stream)
{
    if (!io) return fail(ATLASKV_EINVAL, "null io");
    atlaskv_status st = check_params(t, p, io->B, io->N, io->H, io->T);
    if (st != ATLASKV_OK) return st;
    if (io->B == 0) return ATLASKV_OK;
    if (!io->q_kg || !io->q_seq || !io->k_seq || !io->v_seq || !io->out)
        return fail(ATLASKV_EINVAL, "null q_kg/q_seq/k_seq/v_seq/out");
    const void *ptrs[] = {io->q_kg, io->q_seq, io->k_seq, io->v_seq, io->out, io->lse, io->kept_root, io->kept_mid,
                          io->kept_leaf};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return fail(ATLASKV_EINVAL, "io buffers must be 16-byte aligned");
    const Layout L = plan(t, p, io->B, io->N, io->H, io->T);
    if (!workspace || ((uintptr_t)workspace & 255u)) return fail(ATLASKV_EINVAL, "workspace must be 256-byte aligned");
    if (ws_bytes < L.total)
        return fail(ATLASKV_ENOMEM, "workspace of %zu bytes, %zu needed", ws_bytes, L.total);

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
    const int D = t->d.head_dim;
    const int H_kv = t->d.n_kv_heads;
    const int G = io->H / H_kv;
    const bool host = t->d.leaf_location == ATLASKV_LEAVES_HOST_PINNED;
    const int BH = io->B * io->H;
    int32_t *kept[3] = {io->kept_root ? io->kept_root : reinterpret_cast<int32_t *>(ws + L.kept[0]),
                        io->kept_mid ? io->kept_mid : reinterpret_cast<int32_t *>(ws + L.kept[1]),
                        io->kept_leaf ? io->kept_leaf : reinterpret_cast<int32_t *>(ws + L.kept[2])};

    akv::DescendParams dp{};
    dp.q_kg = io->q_kg;
    dp.B = io->B;
    dp.N = io->N;
    dp.H = io->H;
    dp.H_kv = H_kv;
    dp.G = G;
    dp.keys[0] = t->d.root_keys;
    dp.keys[1] = t->d.mid_keys;
    dp.keys[2] = t->leaf_keys_dev;
    for (int l = 0; l < 3; ++l) {
        dp.rows[l] = t->rows[l];
        dp.fanout[l] = t->d.fanout[l];
        dp.kept[l] = kept[l];
    }
    dp.child[0] = t->d.root_child;
    dp.child[1] = t->d.mid_child;
    dp.norm_bound = t->norm_bound;
    dp.K[0] = p->K_root;
    dp.K[1] = p->K_mid;
    dp.K[2] = p->K_leaf;
    dp.s_ws = reinterpret_cast<float *>(ws + L.s_ws);
    dp.anorm_ws = reinterpret_cast<float *>(ws + L.anorm_ws);
    dp.s64_ws = reinterpret_cast<double *>(ws + L.s64_ws);
    dp.a64_ws = reinterpret_cast<double *>(ws + L.a64_ws);
    dp.f_ws = reinterpret_cast<float *>(ws + L.f_ws);
    dp.fstride = L.fstride;
    dp.cap = L.cap;
    dp.kcap = L.kcap;
    dp.queue = reinterpret_cast<int *>(ws + L.queue);
    dp.qcount = reinterpret_cast<int *>(ws + L.qcount);
    dp.status = t->status;
    dp.stats = t->profiling ? t->stats : nullptr;

    const float scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)D);
    akv::AttnParams ap{};
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
    ap.K_L = p->K_leaf;
    ap.scale_log2 = scale * 1.4426950408889634f;
    ap.status = t->status;

    const bool prof = t->profiling;
    auto mark = [&](int i) -> atlaskv_status {
        if (prof) AKV_CUDA(cudaEventRecord(t->ev[i], s));
        return ATLASKV_OK;
    };
#define AKV_STEP(x)                            \
    do {                                       \
        atlaskv_status st_ = (x);              \
        if (st_ != ATLASKV_OK) return st_;     \
    } while (0)

    if (prof) AKV_CUDA(cudaMemsetAsync(t->stats, 0, 12 * sizeof(unsigned long long), s));
    if (!host) {
        AKV_STEP(mark(0));
        AKV_STEP(dispatch_descend(t->d.dtype, D, dp, 0, 2, s));
        AKV_STEP(mark(1));
        ap.lk_base = t->d.leaf_keys;
        ap.lv_base = t->d.leaf_values;
        ap.lk_idx = kept[2];
        ap.lv_idx = kept[2];
        ap.leaf_head_stride = t->rows[2];
        ap.lk_rows = ap.lv_rows = (long long)H_kv * t->rows[2];
        AKV_STEP(dispatch_attend(t->d.dtype, D, ap, s));
        AKV_STEP(mark(2));
    } else {
        // Query chunks: chunk c covers queries [b0, b0 + Bc).  The caller's
        // stream runs the descent and the attention of each chunk; the staging
        // stream copies the chunk's leaf-key blocks once its mids are kept and
        // its value rows once its leaves are kept, so the host link works while
        // the other chunks compute.
        const int nc = io->B >= 2 * kMaxChunks ? kMaxChunks : 1;
        if (!t->stage_stream) {
            // highest priority: the copies are bound by the host link, so the
            // block scheduler should keep them resident and let the compute fill in
            int lo_prio = 0, hi_prio = 0;
            AKV_CUDA(cudaDeviceGetStreamPriorityRange(&lo_prio, &hi_prio));
            AKV_CUDA(cudaStreamCreateWithPriority(&t->stage_stream, cudaStreamNonBlocking, hi_prio));
            for (cudaEvent_t &e : t->cev) AKV_CUDA(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
        }
        if (prof && !t->tev[0])
            for (cudaEvent_t &e : t->tev) AKV_CUDA(cudaEventCreate(&e));
        cudaStream_t s1 = t->stage_stream;
        const int n_mid = G * p->K_mid, n_leaf = G * p->K_leaf;
        const size_t esz = esize(t->d.dtype);
        auto cev = [&](int c, int k) { return t->cev[c * kChunkEvents + k]; };
        auto tmark = [&](int c, int k, cudaStream_t st) -> atlaskv_status {
            if (prof) AKV_CUDA(cudaEventRecord(t->tev[c * kTimingEvents + k], st));
            return ATLASKV_OK;
        };
        akv::DescendParams dpc[kMaxChunks];
        akv::AttnParams apc[kMaxChunks];
        int32_t *umid[kMaxChunks], *cmid[kMaxChunks], *uleaf[kMaxChunks], *cleaf[kMaxChunks];
        int32_t *leaf_slot[kMaxChunks], *vslot[kMaxChunks];
        int groups[kMaxChunks];
        for (int c = 0; c < nc; ++c) {
            const int b0 = (int)((long long)io->B * c / nc), b1 = (int)((long long)io->B * (c + 1) / nc);
            const int Bc = b1 - b0;
            const size_t bh0 = (size_t)b0 * io->H, g0 = (size_t)b0 * H_kv;
            groups[c] = Bc * H_kv;
            akv::DescendParams d = dp;
            d.B = Bc;
            d.q_kg = reinterpret_cast<const uint8_t *>(io->q_kg) + (size_t)b0 * io->N * io->H * D * esz;
            for (int l = 0; l < 3; ++l) d.kept[l] = kept[l] + bh0 * dp.K[l];
            d.s_ws = dp.s_ws + bh0 * D;
            d.s64_ws = dp.s64_ws + bh0 * D;
            d.a64_ws = dp.a64_ws + bh0 * D;
            d.anorm_ws = dp.anorm_ws + bh0;
            d.f_ws = dp.f_ws + bh0 * (size_t)L.fstride;
            d.qcount = dp.qcount + 4 * c;
            leaf_slot[c] = reinterpret_cast<int32_t *>(ws + L.leaf_slot) + bh0 * p->K_mid;
            vslot[c] = reinterpret_cast<int32_t *>(ws + L.vslot) + bh0 * p->K_leaf;
            umid[c] = reinterpret_cast<int32_t *>(ws + L.umid) + g0 * n_mid;
            cmid[c] = reinterpret_cast<int32_t *>(ws + L.ucount_mid) + g0;
            uleaf[c] = reinterpret_cast<int32_t *>(ws + L.uleaf) + g0 * n_leaf;
            cleaf[c] = reinterpret_cast<int32_t *>(ws + L.ucount_leaf) + g0;
            uint8_t *pool = ws + L.key_pool + g0 * n_mid * (size_t)t->d.fanout[2] * D * esz;
            uint8_t *vpool = ws + L.val_pool + g0 * n_leaf * (size_t)D * esz;
            int32_t *kept_leaf_row = reinterpret_cast<int32_t *>(ws + L.kept_leaf_row) + bh0 * p->K_leaf;
            d.keys[2] = pool;
            d.leaf_slot = leaf_slot[c];
            d.kept_leaf_row = kept_leaf_row;
            dpc[c] = d;
            akv::AttnParams a = ap;
            a.B = Bc;
            const size_t qoff = (size_t)b0 * io->N * io->H * D * esz, kvoff = (size_t)b0 * io->T * H_kv * D * esz;
            a.q_kg = reinterpret_cast<const uint8_t *>(io->q_kg) + qoff;
            a.q_seq = reinterpret_cast<const uint8_t *>(io->q_seq) + qoff;
            a.out = reinterpret_cast<uint8_t *>(io->out) + qoff;
            a.lse = io->lse ? io->lse + (size_t)b0 * io->N * io->H : nullptr;
            a.k_seq = reinterpret_cast<const uint8_t *>(io->k_seq) + kvoff;
            a.v_seq = reinterpret_cast<const uint8_t *>(io->v_seq) + kvoff;
            a.lk_base = pool;
            a.lv_base = vpool;
            a.lk_idx = kept_leaf_row;
            a.lv_idx = vslot[c];
            a.leaf_head_stride = 0;
            a.lk_rows = (long long)groups[c] * n_mid * t->d.fanout[2];
            a.lv_rows = (long long)groups[c] * n_leaf;
            apc[c] = a;
        }
        // the staging stream starts after everything already queued on the caller's stream
        AKV_CUDA(cudaEventRecord(t->cev[kMaxChunks * kChunkEvents], s));
        AKV_CUDA(cudaStreamWaitEvent(s1, t->cev[kMaxChunks * kChunkEvents], 0));
        for (int c = 0; c < nc; ++c) {   // levels 0-1
            AKV_STEP(tmark(c, 0, s));
            AKV_STEP(dispatch_descend(t->d.dtype, D, dpc[c], 0, 1, s));
            AKV_STEP(tmark(c, 1, s));
            AKV_CUDA(cudaEventRecord(cev(c, 0), s));
        }
        for (int c = 0; c < nc; ++c) {   // leaf-key blocks of the kept mids
            AKV_CUDA(cudaStreamWaitEvent(s1, cev(c, 0), 0));
            AKV_STEP(tmark(c, 2, s1));
            AKV_STEP(launch_dedupe(dpc[c].kept[1], n_mid, groups[c], umid[c], leaf_slot[c], cmid[c], s1));
            AKV_STEP(dispatch_stage_keys(t, umid[c], cmid[c], n_mid, groups[c], const_cast<void *>(dpc[c].keys[2]), s1));
            AKV_STEP(tmark(c, 3, s1));
            AKV_CUDA(cudaEventRecord(cev(c, 1), s1));
        }
        for (int c = 0; c < nc; ++c) {   // level 2 on the staged blocks
            AKV_CUDA(cudaStreamWaitEvent(s, cev(c, 1), 0));
            AKV_STEP(tmark(c, 4, s));
            AKV_STEP(dispatch_descend(t->d.dtype, D, dpc[c], 2, 2, s));
            AKV_STEP(tmark(c, 5, s));
            AKV_CUDA(cudaEventRecord(cev(c, 2), s));
        }
        for (int c = 0; c < nc; ++c) {   // value rows of the kept leaves
            AKV_CUDA(cudaStreamWaitEvent(s1, cev(c, 2), 0));
            AKV_STEP(tmark(c, 6, s1));
            AKV_STEP(launch_dedupe(dpc[c].kept[2], n_leaf, groups[c], uleaf[c], vslot[c], cleaf[c], s1));
            AKV_STEP(dispatch_stage_values(t, uleaf[c], cleaf[c], n_leaf, groups[c], const_cast<void *>(apc[c].lv_base),
                                           s1));
            AKV_STEP(tmark(c, 7, s1));
            AKV_CUDA(cudaEventRecord(cev(c, 3), s1));
        }
        for (int c = 0; c < nc; ++c) {   // attention; the caller's stream joins the staging stream here
            AKV_CUDA(cudaStreamWaitEvent(s, cev(c, 3), 0));
            AKV_STEP(tmark(c, 8, s));
            AKV_STEP(dispatch_attend(t->d.dtype, D, apc[c], s));
            AKV_STEP(tmark(c, 9, s));
        }
        t->chunks_last = nc;
    }
#undef AKV_STEP
    t->timed = prof;
    t->host_mode_last = host;
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
    if (v != akv::kDevOk) return fail(ATLASKV_EDEVICE, "device status %d", v);
    return ATLASKV_OK;
}

atlaskv_status atlaskv_set_profiling(atlaskv_tree *t, int32_t enable)
{
    if (!t) return fail(ATLASKV_EINVAL, "null tree");
    if (enable && !t->ev[0])
        for (int i = 0; i < kNumEvents; ++i) AKV_CUDA(cudaEventCreate(&t->ev[i]));
    t->profiling = enable != 0;
    return ATLASKV_OK;
}

atlaskv_status atlaskv_stage_times(atlaskv_tree *t, float *ms, int32_t n)
{
    if (!t || !ms || n < 1) return fail(ATLASKV_EINVAL, "null tree/ms or n < 1");
    if (!t->timed) return fail(ATLASKV_EINVAL, "no attend call was timed (enable profiling first)");
    float v[3] = {0.f, 0.f, 0.f};
    if (!t->host_mode_last) {
        AKV_CUDA(cudaEventSynchronize(t->ev[2]));
        AKV_CUDA(cudaEventElapsedTime(&v[0], t->ev[0], t->ev[1]));
        AKV_CUDA(cudaEventElapsedTime(&v[2], t->ev[1], t->ev[2]));
    } else {
        // busy time of each kind of segment, summed over the query chunks
        // (segments of different kinds overlap on the two streams)
        const int nc = t->chunks_last;
        AKV_CUDA(cudaEventSynchronize(t->tev[(nc - 1) * kTimingEvents + 9]));
        for (int c = 0; c < nc; ++c) {
            float seg[5];
            for (int k = 0; k < 5; ++k)
                AKV_CUDA(cudaEventElapsedTime(&seg[k], t->tev[c * kTimingEvents + 2 * k],
                                              t->tev[c * kTimingEvents + 2 * k + 1]));
            v[0] += seg[0] + seg[2];
            v[1] += seg[1] + seg[3];
            v[2] += seg[4];
        }
    }
    for (int i = 0; i < n && i < 3; ++i) ms[i] = v[i];
    return ATLASKV_OK;
}

atlaskv_status atlaskv_refine_stats(atlaskv_tree *t, uint64_t *counts, int32_t n)
{
    if (!t || !counts || n < 1) return fail(ATLASKV_EINVAL, "null tree/counts or n < 1");
    if (!t->timed) return fail(ATLASKV_EINVAL, "no attend call was profiled (enable profiling first)");
    unsigned long long v[12];
    AKV_CUDA(cudaMemcpy(v, t->stats, sizeof v, cudaMemcpyDeviceToHost));
    for (int i = 0; i < n && i < 12; ++i) counts[i] = v[i];
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
    for (int i = 0; i < kNumEvents; ++i)
        if (t->ev[i]) cudaEventDestroy(t->ev[i]);
    for (cudaEvent_t e : t->cev)
        if (e) cudaEventDestroy(e);
    for (cudaEvent_t e : t->tev)
        if (e) cudaEventDestroy(e);
    if (t->stage_stream) cudaStreamDestroy(t->stage_stream);
    delete t;
    return ATLASKV_OK;
}

}  // extern "C"
