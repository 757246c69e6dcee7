// Knowledge + causal-sequence attention on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in Tensor Memory), bf16 inputs, D = 128.
//
// Same computation as attend.cuh ("AtlasKV: Augmenting LLMs with Billion-Scale
// Knowledge Graphs in 20GB VRAM": the lambda-weighted merge of the knowledge and
// sequence softmaxes equals one softmax over both key sets), organised for
// sm_100a:
//   * a CTA of 4 warps owns 128 query rows of one (query b, KV head): row
//     r = g N + n is token n of head g of the group, so the G heads of a KV head
//     share every sequence K/V tile;
//   * key tiles of 64 rows (first the CTA's heads' kept leaves, each visible
//     only to its own head's rows, then the causal sequence tiles) are copied by
//     cp.async into 128-byte-swizzled shared memory, double buffered;
//   * one thread issues S = Q K^T (M 128, N 64, K 128) into TMEM, every thread
//     reads back its own row of S (tcgen05.ld 32x32b), runs the online softmax
//     and writes its row of P (bf16, swizzled) to shared memory; then one
//     thread issues O_t = P V (M 128, N 128, K 64) into TMEM and every thread
//     folds its row of O_t into its register accumulator;
//   * tcgen05.commit arrives on an mbarrier when the issuing thread's MMAs are
//     done; every wait is bounded and reports ETIMEOUT through the tree status.
#pragma once

#include "attend.cuh"
#include "common.cuh"

namespace akv {
namespace tc {

constexpr int kRows = 128;       // query rows per CTA (UMMA M)
constexpr int kKeys = 64;        // keys per tile (UMMA N of QK^T, K of PV)
constexpr int kD = 128;          // head dim
constexpr int kThreads = 128;
constexpr long long kSpinLimit = 1ll << 22;   // bounded mbarrier waits (seconds at most)

// shared-memory layout (byte offsets; every operand region 1024-byte aligned).
// P (the bf16 probabilities of the current tile) is written over the K tile of
// the same stage once S = Q K^T has completed: that K tile is dead by then and
// the next copy into the stage starts only after P V has completed.
constexpr int kQBytes = kRows * kD * 2;            // 32 KB: 2 K-blocks of [128 rows][64]
constexpr int kKVBytes = kKeys * kD * 2;           // 16 KB: 2 blocks of [64 keys][64]
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;             // 2 stages (P aliases the current one)
constexpr int kOffV = kOffK + 2 * kKVBytes;        // 2 stages
constexpr int kOffMeta = kOffV + 2 * kKVBytes;     // mbarriers, TMEM base
constexpr int kMetaBytes = 1024;
constexpr int kSmemBytes = kOffMeta + kMetaBytes + 1024;   // + slack to align the base to 1024
constexpr int kTmemCols = 256;                     // S: columns [0, 64), O tile: [64, 192)

__device__ __forceinline__ uint32_t smem_addr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Byte offset of 16-byte chunk c (0..7) of row r inside a 128-byte-swizzled
// block of rows that are 128 bytes long (the canonical SWIZZLE_128B atom:
// chunk index XOR (row mod 8)).
__device__ __forceinline__ uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// UMMA shared-memory descriptor: SWIZZLE_128B, version 1 (sm_100).
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;            // version
    d |= (uint64_t)2 << 61;            // SWIZZLE_128B
    return d;
}

// UMMA instruction descriptor, kind::f16: bf16 x bf16 -> f32.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, int a_mn_major, int b_mn_major)
{
    return (1u << 4)                       // D format f32
           | (1u << 7)                     // A bf16
           | (1u << 10)                    // B bf16
           | ((uint32_t)a_mn_major << 15)  // A major
           | ((uint32_t)b_mn_major << 16)  // B major
           | ((uint32_t)(N >> 3) << 17)    // N
           | ((uint32_t)(M >> 4) << 24);   // M
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint32_t mbar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, int count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count));
}

// Bounded wait for the given phase parity; returns false on timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity)
{
    for (long long i = 0; i < kSpinLimit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v)
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void cp16(uint32_t dst, const void *src, bool valid)
{
    const int sz = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::); }
__device__ __forceinline__ void cp_wait_1() { asm volatile("cp.async.wait_group 1;\n" ::); }

}  // namespace tc

// One CTA per (query b, KV head, 128-row block of the group's G N rows).
__global__ void __launch_bounds__(tc::kThreads, 2) attend_tc_kernel(const AttnParams p, int blocks_per_group)
{
    using namespace tc;
    extern __shared__ __align__(1024) uint8_t tc_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_addr(smem);
    // meta: mbarriers at +0 (S done) and +8 (O tile done), TMEM base at +64
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMeta + 64);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int grp_id = blockIdx.x / blocks_per_group;
    const int blk = blockIdx.x - grp_id * blocks_per_group;
    const int b = grp_id / p.H_kv, hkv = grp_id - b * p.H_kv;
    const int GN = p.G * p.N;
    const int r0 = blk * kRows;
    const int row = r0 + tid;                 // this thread's query row in the group
    const bool row_ok = row < GN;
    const int g = row_ok ? row / p.N : 0;
    const int n = row_ok ? row - g * p.N : 0;
    const int h = hkv * p.G + g;
    const int last_key = p.T - p.N + n;       // causal limit of this row
    const int g_first = r0 / p.N;
    const int g_last = min(GN - 1, r0 + kRows - 1) / p.N;   // heads g_first..g_last own the rows
    const int nheads = g_last - g_first + 1;

    if (tid == 0) {
        mbar_init(sbase + kOffMeta, 1);
        mbar_init(sbase + kOffMeta + 8, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem;          // columns [0, 64): S
    const uint32_t tO = tmem + 64;     // columns [64, 192): O tile
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    // Loads are mapped so that 16 consecutive threads copy the 16 chunks of
    // one 256-byte row: a warp instruction reads two whole rows.
    const int lc = tid & 15, lr = tid >> 4;   // chunk, first row of this thread

    // ---- Q rows into the swizzled A tile ----
    auto load_q = [&](const void *qptr) {
        const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(qptr);
        const uint32_t dst0 = sbase + kOffQ + (lc >> 3) * (kRows * 128);
#pragma unroll 4
        for (int i = 0; i < kRows / 8; ++i) {
            const int r = lr + 8 * i, rr = r0 + r;
            const bool ok = rr < GN;
            const int gg = ok ? rr / p.N : 0, nn = ok ? rr - gg * p.N : 0;
            const __nv_bfloat16 *src = q + (((size_t)b * p.N + nn) * p.H + hkv * p.G + gg) * kD + lc * 8;
            cp16(dst0 + sw128(r, lc & 7), src, ok);
        }
        cp_commit();
    };

    // ---- key tile loaders (K and V rows into the swizzled tiles of a stage) ----
    const __nv_bfloat16 *kseq = reinterpret_cast<const __nv_bfloat16 *>(p.k_seq);
    const __nv_bfloat16 *vseq = reinterpret_cast<const __nv_bfloat16 *>(p.v_seq);
    // row_src(key) -> (K row, V row) pointers or nullptr for a zero row
    auto load_kv_rows = [&](int stage, auto row_src) {
        const uint32_t off0 = (lc >> 3) * (kKeys * 128);
        const uint32_t kb = sbase + kOffK + stage * kKVBytes + off0, vb = sbase + kOffV + stage * kKVBytes + off0;
#pragma unroll
        for (int i = 0; i < kKeys / 8; ++i) {
            const int key = lr + 8 * i;
            const __nv_bfloat16 *ks, *vs;
            row_src(key, ks, vs);
            const bool ok = ks != nullptr;
            const uint32_t off = sw128(key, lc & 7);
            cp16(kb + off, ok ? ks + lc * 8 : kseq, ok);
            cp16(vb + off, ok ? vs + lc * 8 : vseq, ok);
        }
        cp_commit();
    };

    // leaf keys of the CTA's heads: nheads * K_L of them, head-major
    const int n_leaf = nheads * p.K_L;
    const int n_leaf_tiles = (n_leaf + kKeys - 1) / kKeys;
    const __nv_bfloat16 *lkb = reinterpret_cast<const __nv_bfloat16 *>(p.lk_base);
    const __nv_bfloat16 *lvb = reinterpret_cast<const __nv_bfloat16 *>(p.lv_base);
    auto leaf_src = [&](int tile, int key, const __nv_bfloat16 *&ks, const __nv_bfloat16 *&vs) {
        const int j = tile * kKeys + key;
        if (j >= n_leaf) {
            ks = vs = nullptr;
            return;
        }
        const int gg = g_first + j / p.K_L, jj = j - (j / p.K_L) * p.K_L;
        const long long e = ((long long)b * p.H + hkv * p.G + gg) * p.K_L + jj;
        ks = lkb + (size_t)(p.leaf_head_stride * hkv + p.lk_idx[e]) * kD;
        vs = lvb + (size_t)(p.leaf_head_stride * hkv + p.lv_idx[e]) * kD;
    };
    // causal extent of the CTA's rows
    // causal extent of the CTA: its largest token index is N - 1 when its rows
    // span two heads, else that of its last row
    const int r_end = min(GN - 1, r0 + kRows - 1);
    const int cta_last = p.T - p.N + (r_end / p.N != r0 / p.N ? p.N - 1 : r_end % p.N);
    const int n_seq_tiles = (cta_last + kKeys) / kKeys;
    const size_t seq_stride = (size_t)p.H_kv * kD;
    const __nv_bfloat16 *kseq_b = kseq + ((size_t)b * p.T * p.H_kv + hkv) * kD;
    const __nv_bfloat16 *vseq_b = vseq + ((size_t)b * p.T * p.H_kv + hkv) * kD;
    auto issue_tile = [&](int t, int stage) {   // t < n_leaf_tiles: leaf tile; else sequence tile
        if (t < n_leaf_tiles) {
            load_kv_rows(stage, [&](int key, const __nv_bfloat16 *&ks, const __nv_bfloat16 *&vs) {
                leaf_src(t, key, ks, vs);
            });
        } else {
            const int t0 = (t - n_leaf_tiles) * kKeys;
            load_kv_rows(stage, [&](int key, const __nv_bfloat16 *&ks, const __nv_bfloat16 *&vs) {
                const bool ok = t0 + key < p.T;
                ks = ok ? kseq_b + (size_t)(t0 + key) * seq_stride : nullptr;
                vs = ok ? vseq_b + (size_t)(t0 + key) * seq_stride : nullptr;
            });
        }
    };

    const int n_tiles = n_leaf_tiles + n_seq_tiles;
    const uint32_t idesc_s = make_idesc(kRows, kKeys, 0, 0);   // Q (K-major) x K^T (K-major)
    const uint32_t idesc_o = make_idesc(kRows, kD, 0, 1);      // P (K-major) x V (MN-major)

    float o[kD];
#pragma unroll
    for (int i = 0; i < kD; ++i) o[i] = 0.f;
    float m = -INFINITY, l = 0.f;
    const float sl2 = p.scale_log2;
    bool failed = false;

    load_q(p.q_kg);
    issue_tile(0, 0);
    for (int t = 0; t < n_tiles && !failed; ++t) {
        const int stage = t & 1;
        const bool leaf = t < n_leaf_tiles;
        if (t == n_leaf_tiles) {
            // switch A to the sequence queries (the previous MMAs finished: O waited below)
            load_q(p.q_seq);
        }
        if (t + 1 < n_tiles) {
            issue_tile(t + 1, stage ^ 1);
            cp_wait_1();   // everything but the newest group: Q and tile t have landed
        } else {
            cp_wait_all();
        }
        fence_async_smem();   // make this thread's cp.async data visible to the tensor cores
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        // ---- S = Q K^T ----
        if (tid == 0) {
            const uint32_t qa = sbase + kOffQ, kbase = sbase + kOffK + stage * kKVBytes;
#pragma unroll
            for (int s = 0; s < kD / 16; ++s) {
                const uint64_t da = make_desc(qa + (s >> 2) * (kRows * 128) + (s & 3) * 32, 16, 1024);
                const uint64_t db = make_desc(kbase + (s >> 2) * (kKeys * 128) + (s & 3) * 32, 16, 1024);
                mma_bf16(tS, da, db, idesc_s, s > 0 ? 1u : 0u);
            }
            mma_commit(sbase + kOffMeta);
        }
        if (!mbar_wait(sbase + kOffMeta, (uint32_t)(t & 1))) failed = true;
        fence_after_sync();
        // ---- online softmax on this thread's row ----
        float sc[kKeys];
        tmem_ld32(tS + lane_off, sc);
        tmem_ld32(tS + lane_off + 32, sc + 32);
        tmem_wait_ld();
        float mx = m;
        // visible keys of this tile: [lo, hi) in tile-local index.  The leaves
        // are stored head by head, K_L per head, so a row sees one contiguous
        // run of them; a sequence tile is cut by the causal limit.
        int lo, hi;
        if (leaf) {
            lo = (g - g_first) * p.K_L - t * kKeys;
            hi = lo + p.K_L;
        } else {
            lo = 0;
            hi = last_key + 1 - (t - n_leaf_tiles) * kKeys;
        }
        if (!row_ok) hi = lo;
#pragma unroll
        for (int j = 0; j < kKeys; ++j) {
            sc[j] = (j >= lo && j < hi) ? sc[j] * sl2 : -INFINITY;
            mx = fmaxf(mx, sc[j]);
        }
        const float base = mx == -INFINITY ? 0.f : mx;
        const float alpha = exp2f(m - base);
        m = mx;
        float psum = 0.f;
        uint32_t pk[kKeys / 2];
#pragma unroll
        for (int j = 0; j < kKeys; j += 2) {
            const float e0 = exp2f(sc[j] - base), e1 = exp2f(sc[j + 1] - base);
            psum += e0 + e1;
            __nv_bfloat162 v2 = __floats2bfloat162_rn(e0, e1);
            pk[j / 2] = *reinterpret_cast<uint32_t *>(&v2);
        }
        l = l * alpha + psum;
        // row tid of P: 8 chunks of 16 bytes, swizzled
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            *reinterpret_cast<uint4 *>(smem + kOffK + stage * kKVBytes + sw128(tid, c)) = v;
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        // ---- O_t = P V ----
        if (tid == 0) {
            const uint32_t pa = sbase + kOffK + stage * kKVBytes, vbase = sbase + kOffV + stage * kKVBytes;
#pragma unroll
            for (int s = 0; s < kKeys / 16; ++s) {
                const uint64_t da = make_desc(pa + s * 32, 16, 1024);
                const uint64_t db = make_desc(vbase + s * 16 * 128, kKeys * 128, 1024);
                mma_bf16(tO, da, db, idesc_o, s > 0 ? 1u : 0u);
            }
            mma_commit(sbase + kOffMeta + 8);
        }
        if (!mbar_wait(sbase + kOffMeta + 8, (uint32_t)(t & 1))) failed = true;
        fence_after_sync();
#pragma unroll
        for (int c = 0; c < kD; c += 32) {
            float ot[32];
            tmem_ld32(tO + lane_off + c, ot);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[c + i] = fmaf(o[c + i], alpha, ot[i]);
        }
        fence_before_sync();
        failed = __syncthreads_or(failed);
    }
    if (failed && tid == 0) set_status(p.status, kDevTimeout);
    cp_wait_all();

    // ---- epilogue: this thread's row ----
    if (row_ok && !failed) {
        const float inv = 1.f / l;
        __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(p.out) + (((size_t)b * p.N + n) * p.H + h) * kD;
#pragma unroll
        for (int c = 0; c < kD; c += 8) {
            __nv_bfloat162 a0 = __floats2bfloat162_rn(o[c] * inv, o[c + 1] * inv);
            __nv_bfloat162 a1 = __floats2bfloat162_rn(o[c + 2] * inv, o[c + 3] * inv);
            __nv_bfloat162 a2 = __floats2bfloat162_rn(o[c + 4] * inv, o[c + 5] * inv);
            __nv_bfloat162 a3 = __floats2bfloat162_rn(o[c + 6] * inv, o[c + 7] * inv);
            uint4 v = make_uint4(*reinterpret_cast<uint32_t *>(&a0), *reinterpret_cast<uint32_t *>(&a1),
                                 *reinterpret_cast<uint32_t *>(&a2), *reinterpret_cast<uint32_t *>(&a3));
            *reinterpret_cast<uint4 *>(dst + c) = v;
        }
        if (p.lse) p.lse[((size_t)b * p.N + n) * p.H + h] = (m + log2f(l)) * 0.69314718055994530942f;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

}  // namespace akv
