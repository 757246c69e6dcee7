// Knowledge + causal-sequence attention on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in Tensor Memory), bf16 inputs, D = 64 or 128.
//
// Same computation as attend.cuh ("AtlasKV: Augmenting LLMs with Billion-Scale
// Knowledge Graphs in 20GB VRAM": the lambda-weighted merge of the knowledge and
// sequence softmaxes equals one softmax over both key sets), organised for
// sm_100a as a warp-specialised, persistent pipeline.  A unit of work is a
// 128-row block of one (query b, KV head) group (row r = g N + n is token n of
// head g) and its 64-key tiles: first the kept leaves of the block's heads
// (each visible only to its own head's rows), then the causal sequence; the
// online softmax is order-free.  A CTA (TMEM 256 columns, 112 KB of shared
// memory, two per SM, so one CTA's MMA, copy and softmax bubbles overlap the
// other's work) runs its units back to back through one pipeline, so a unit's
// start (leaf gathers, the Q load, the first S) overlaps the previous unit's
// last tiles and epilogue.
//
//   producer warp   sequence K/V tiles by TMA (4-D tensor maps, 128-byte
//                   swizzle) and gathered leaf rows by cp.async, into a K ring
//                   (a stage is released as soon as S has read it) and a
//                   three-stage V ring, each guarded by full / empty mbarriers;
//   MMA warp        one thread issues S(t) = Q K_t^T (M 128, N 64, K 128, both
//                   operands in shared memory) into a double-buffered S in
//                   TMEM, then O += P V_{t-1} (M 128, N 128, K 64) with P read
//                   from TMEM, so S(t) runs under softmax(t - 1); a unit's
//                   first P V starts O afresh once the previous unit's O has
//                   been read out; tcgen05.commit arrives on the mbarriers;
//   4 softmax warps one thread per query row: read its S row (tcgen05.ld),
//                   mask, online softmax with a lazily rescaled running max
//                   (O in TMEM is rescaled only when the row max grows by more
//                   than 2^8), P (bf16 pairs) written back over the first half
//                   of the same S buffer (tcgen05.st), so P never touches
//                   shared memory; the Q loads (q_kg, then q_seq, then the
//                   next unit's), each started as soon as the last S that
//                   reads the old Q has completed; finally O / l and the
//                   log-sum-exp.
// Shared-memory bandwidth is what the tensor core waits on here (the MMA
// operands plus the K/V copies); P in TMEM removes its store and its reread.
//
// Every mbarrier wait is bounded; a wait that gives up sets ETIMEOUT in the
// tree's status word and the roles drain without further waits.
#pragma once

#include <cuda.h>

#include "attend.cuh"
#include "common.cuh"

namespace akv {
namespace tc {

constexpr int kRows = 128;                 // query rows per warpgroup (UMMA M)
constexpr int kKeys = 64;                  // keys per tile
constexpr int kKStages = 2;                // K ring depth (a stage is freed when S = Q K^T completes)
constexpr int kVStages = 3;                // V ring depth (freed when P V completes; its wait bounds the K issue too)
constexpr int kMinCtasPerSm = 2;           // one softmax warpgroup per CTA, two CTAs per SM
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 32 * 6;
constexpr int kCtaRows = kRows;
constexpr long long kSpinLimit = 1ll << 18;   // bounded mbarrier waits: try_wait iterations, not a fixed time
constexpr float kRescaleLog2 = 8.f;            // rescale O only when the row max grows by more than this

// mbarriers (8 bytes each); the [2] arrays are indexed by the parity of the
// CTA's running tile count (tiles of all its units, in order)
constexpr int kBarFullK = 0;                        // [kKStages] K tile landed
constexpr int kBarEmptyK = kBarFullK + kKStages;    // [kKStages] S of the tile done
constexpr int kBarFullV = kBarEmptyK + kKStages;    // [kVStages] V tile landed
constexpr int kBarEmptyV = kBarFullV + kVStages;    // [kVStages] P V of the tile done
constexpr int kBarSFull = kBarEmptyV + kVStages;    // [2] S in TMEM buffer (tile & 1)
constexpr int kBarPReady = kBarSFull + 2;           // [2] P written over it, O rescaled (4 warps)
constexpr int kBarODone = kBarPReady + 2;           // [2] O += P V from that buffer done
constexpr int kBarQReady = kBarODone + 2;           // Q loaded (one phase per load; 4 warps with cp.async)
constexpr int kBarODrained = kBarQReady + 1;        // a unit's O read out of TMEM (4 warps)
constexpr int kBarDrain = kBarODrained + 1;         // every MMA the issuing thread committed has completed
constexpr int kNumBars = kBarDrain + 1;

// Shared memory for head dim D (64 or 128): byte offsets from a 1024-aligned
// base; operand tiles in the canonical 128-byte-swizzled UMMA layouts, made of
// D / 64 blocks of 64 columns (one 128-byte row per block).  No alignment
// slack: with no static shared memory the dynamic base is 1024-byte aligned
// (the kernel checks it and reports EDEVICE otherwise); 112 KB at D = 128
// keeps two CTAs per SM.
template <int D>
struct TcSmem {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kBlocks = D / 64;
    static constexpr int kQBytes = kRows * D * 2;       // 32 / 16 KB
    static constexpr int kKVBytes = kKeys * D * 2;      // 16 / 8 KB
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;                    // [kKStages]
    static constexpr int kOffV = kOffK + kKStages * kKVBytes;        // [kVStages]
    static constexpr int kOffBar = kOffV + kVStages * kKVBytes;
    static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
    static constexpr int kBytes = kOffTmemSlot + 16;
};
constexpr int kTmemCols = 256;                 // S / P buffers [0, 128), O [128, 128 + D)

__device__ __forceinline__ uint32_t smem_addr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Byte offset of 16-byte chunk c (0..7) of row r inside a 128-byte-swizzled
// block of 128-byte rows (the SWIZZLE_128B atom: chunk index XOR (row mod 8)).
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

// Same with the A operand (M x 16, K-major, 16-bit values packed in pairs
// per 32-bit column: 8 columns per K step) read from TMEM.
__device__ __forceinline__ void mma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc,
                                            uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(tmem_d),
        "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

__device__ __forceinline__ void mma_commit(uint32_t mbar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, int count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint32_t mbar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t mbar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
}

// Bounded wait for the phase with the given parity; false on timeout.
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

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float *v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

// 2^x with the MUFU approximation (ex2.approx.ftz: relative error about
// 2^-22, 2^-inf = 0); the probabilities are rounded to bf16 afterwards.
__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void cp16(uint32_t dst, const void *src, bool valid)
{
    const int sz = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }
__device__ __forceinline__ void cp_wait_1() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

// TMA tile load of a 4-D box into shared memory, completion counted in bytes
// on the mbarrier.  No multicast.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                            uint32_t mbar)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(mbar)
        : "memory");
}

}  // namespace tc

// A wait that cannot complete: one mbarrier with an expected arrival that
// never comes, waited on with the attention kernel's bounded wait, which gives
// up and reports ETIMEOUT through the status word.
__global__ void wait_timeout_probe_kernel(int *status)
{
    __shared__ __align__(8) uint64_t never;
    const uint32_t b = tc::smem_addr(&never);
    if (threadIdx.x == 0) {
        tc::mbar_init(b, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0 && !tc::mbar_wait(b, 0)) set_status(status, kDevTimeout);
}

// One unit of attention work: (query b, KV head, 128-row block of the group's
// G N rows; row r = g N + n is token n of head g).  Its tiles 0 ..
// n_leaf_tiles - 1 hold the kept leaves of the block's heads (stored head by
// head, K_L per head), the rest the causal sequence.
struct TcUnit {
    int b, hkv, grp, r0, rows, g_first, n_leaf, n_leaf_tiles, n_seq_tiles, n_tiles;
};

__device__ __forceinline__ TcUnit tc_unit(const AttnParams &p, unsigned u, int ctas_per_group)
{
    TcUnit U;
    U.grp = (int)(u / (unsigned)ctas_per_group);
    const int blk = (int)u - U.grp * ctas_per_group;
    U.b = U.grp / p.H_kv;
    U.hkv = U.grp - U.b * p.H_kv;
    const int GN = p.G * p.N;
    U.r0 = blk * tc::kRows;
    const int r_end = min(GN, U.r0 + tc::kRows) - 1;   // last valid row
    U.rows = r_end + 1 - U.r0;
    U.g_first = U.r0 / p.N;
    const int g_last = r_end / p.N;
    U.n_leaf = (g_last - U.g_first + 1) * p.K_L;
    U.n_leaf_tiles = p.mode == kAttnSeq ? 0 : (U.n_leaf + tc::kKeys - 1) / tc::kKeys;
    // causal extent: the largest token index of the block is N - 1 when its
    // rows span two heads, else that of its last row
    const int last = p.T - p.N + (g_last != U.g_first ? p.N - 1 : r_end % p.N);
    U.n_seq_tiles = p.mode == kAttnLeaf ? 0 : (last + tc::kKeys) / tc::kKeys;
    U.n_tiles = U.n_leaf_tiles + U.n_seq_tiles;
    return U;
}

// A CTA runs the units u0, u0 + ustride, ... below n_units back to back
// through one pipeline: the rings, the S / P buffers and every barrier phase
// run on over the units' tiles in order (T counts them), so the next unit's
// leaf gathers, Q load and first S overlap the last tiles and the epilogue of
// the current one.  Leaves come first in a unit: their gathers are its
// slowest copies, and the switch from q_kg to q_seq is then a load that runs
// under the softmax of the unit's last leaf tile.  Sequence K / V by TMA
// through tm_k / tm_v; Q by TMA through tm_qs / tm_qk when they are given and
// every head of a block starts on a swizzle atom of the Q tile (N a multiple
// of 8 that divides 128 or is divisible by it), else by cp.async.
template <int D>
__device__ __forceinline__ void attend_tc_run(const AttnParams &p, int ctas_per_group, unsigned u0, unsigned ustride,
                                              unsigned n_units, const CUtensorMap *tm_k, const CUtensorMap *tm_v,
                                              const CUtensorMap *tm_qs, const CUtensorMap *tm_qk)
{
    using namespace tc;
    using SM = TcSmem<D>;
    constexpr int kKVBytes = SM::kKVBytes, kOffQ = SM::kOffQ, kOffK = SM::kOffK, kOffV = SM::kOffV,
                  kOffBar = SM::kOffBar, kOffTmemSlot = SM::kOffTmemSlot, kBlocks = SM::kBlocks;
    extern __shared__ __align__(1024) uint8_t tc_smem_raw[];
    uint8_t *smem = tc_smem_raw;
    const uint32_t sb = smem_addr(smem);
    if (sb & 1023u) {   // the 128-byte swizzle atoms need a 1024-byte aligned base (CTA-uniform exit)
        if (threadIdx.x == 0) set_status(p.status, kDevBadSmem);
        return;
    }
    if (u0 >= n_units) return;   // CTA-uniform: no unit, nothing allocated yet
    auto bar = [&](int i) -> uint32_t { return sb + kOffBar + 8 * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffTmemSlot);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int GN = p.G * p.N;
    const bool q_tma = tm_qs != nullptr && p.N % 8 == 0 && (128 % p.N == 0 || p.N % 128 == 0);

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            const bool per_warp = i == kBarPReady || i == kBarPReady + 1 || i == kBarODrained ||
                                  (!q_tma && i == kBarQReady);
            mbar_init(bar(i), per_warp ? 4 : 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp < 4) {
        // ================= softmax warpgroup: one thread per query row =================
        const int lrow = tid;                                   // row of the Q tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint32_t tS = tmem, tO = tmem + 128;
        const uint32_t qa = sb + kOffQ;
        const float sl2 = p.scale_log2;
        bool failed = false;

        // Q rows of unit U into the swizzled A tile.  By TMA: one thread, one box
        // of min(N, 128) rows of one head per 64-column half, completion counted
        // in bytes on QReady; it returns at once.  Else cp.async, 16 consecutive
        // threads per 256-byte row; it returns once the rows have landed.
        auto load_q = [&](const TcUnit &U, bool seq) {
            if (q_tma) {
                if (tid != 0) return;
                const CUtensorMap *m = seq ? tm_qs : tm_qk;
                const int bn = min(p.N, kRows);
                mbar_arrive_expect_tx(bar(kBarQReady), (uint32_t)U.rows * D * 2);
                for (int rr = U.r0; rr < U.r0 + U.rows; rr += bn) {
                    const int gg = rr / p.N, tok = rr - gg * p.N;
#pragma unroll
                    for (int half = 0; half < kBlocks; ++half)
                        tma_load_4d(qa + half * (kRows * 128) + (rr - U.r0) * 128, m, half * 64, U.hkv * p.G + gg, tok,
                                    U.b, bar(kBarQReady));
                }
                return;
            }
            const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(seq ? p.q_seq : p.q_kg);
            constexpr int TPR = D / 8;   // threads per row: one 16-byte chunk each
            const int lc = lrow % TPR, lr = lrow / TPR;
            const uint32_t dst0 = qa + (lc >> 3) * (kRows * 128);
#pragma unroll 4
            for (int i = 0; i < kRows * TPR / 128; ++i) {
                const int rl = lr + (128 / TPR) * i;
                const bool ok = rl < U.rows;
                const int rr = U.r0 + (ok ? rl : 0);
                const int gg = rr / p.N, nn = rr - gg * p.N;
                const __nv_bfloat16 *src = q + (((size_t)U.b * p.N + nn) * p.H + U.hkv * p.G + gg) * D + lc * 8;
                cp16(dst0 + sw128(rl, lc & 7), src, ok);
            }
            cp_commit();
            cp_wait_all();
            fence_async_smem();   // visible to the tensor cores once the barrier is passed
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarQReady));
        };

        int T = 0;   // tiles of this CTA so far
        unsigned u = u0;
        TcUnit U = tc_unit(p, u, ctas_per_group);
        load_q(U, U.n_leaf_tiles == 0);
        for (int ui = 0; !failed; ++ui) {
            const unsigned un = u + ustride;
            const bool has_next = un < n_units;
            const int row = U.r0 + lrow;
            const bool row_ok = lrow < U.rows;
            const int g = row_ok ? row / p.N : U.g_first;
            const int n = row_ok ? row - g * p.N : 0;
            const int h = U.hkv * p.G + g;
            const int last_key = p.T - p.N + n;
            float m_used = -INFINITY, l = 0.f;
            for (int t = 0; t < U.n_tiles; ++t, ++T) {
                const int bs = T & 1;
                failed = __any_sync(0xffffffffu, !mbar_wait(bar(kBarSFull + bs), (T >> 1) & 1));
                if (failed) break;
                fence_after_sync();
                float sc[kKeys];
                tmem_ld32(tS + 64 * bs + lane_off, sc);
                tmem_ld32(tS + 64 * bs + 32 + lane_off, sc + 32);
                tmem_wait_ld();
                // the last S that reads this Q has completed: start the next Q
                if (t == U.n_leaf_tiles - 1 && U.n_seq_tiles > 0) load_q(U, true);
                else if (t == U.n_tiles - 1 && has_next) {
                    const TcUnit Un = tc_unit(p, un, ctas_per_group);
                    load_q(Un, Un.n_leaf_tiles == 0);
                }

                // visible keys of this tile, [lo, hi) in tile-local index: the
                // leaves are stored head by head, K_L per head; a sequence tile is
                // cut by the causal limit
                int lo, hi;
                if (t < U.n_leaf_tiles) {
                    lo = (g - U.g_first) * p.K_L - t * kKeys;
                    hi = lo + p.K_L;
                } else {
                    lo = 0;
                    hi = last_key + 1 - (t - U.n_leaf_tiles) * kKeys;
                }
                if (!row_ok) hi = lo;
                if (!(lo <= 0 && hi >= kKeys)) {
#pragma unroll
                    for (int j = 0; j < kKeys; ++j) sc[j] = (j >= lo && j < hi) ? sc[j] : -INFINITY;
                }
                // row max with 8 independent chains
                float mx8[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) mx8[k] = sc[k];
#pragma unroll
                for (int j = 8; j < kKeys; ++j) mx8[j & 7] = fmaxf(mx8[j & 7], sc[j]);
                const float tmax = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                         fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
                const float m_new = fmaxf(m_used, tmax * sl2);   // scores in log2 units (sl2 > 0)
                if (t == 0) {
                    m_used = m_new;   // O is initialised by the unit's first P V
                } else {
                    const bool need = m_new > m_used + kRescaleLog2;   // also when m_used is still -inf
                    if (__any_sync(0xffffffffu, need)) {
                        // O may be rescaled only once the previous P V has landed in it
                        failed = __any_sync(0xffffffffu,
                                            !mbar_wait(bar(kBarODone + ((T - 1) & 1)), ((T - 1) >> 1) & 1));
                        if (failed) break;
                        fence_after_sync();
                        const float f = need ? fast_exp2(m_used - m_new) : 1.f;
#pragma unroll
                        for (int c = 0; c < D; c += 32) {
                            float ov[32];
                            tmem_ld32(tO + lane_off + c, ov);
                            tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 32; ++i) ov[i] *= f;
                            tmem_st32(tO + lane_off + c, ov);
                        }
                        tmem_wait_st();
                        if (need) {
                            l *= f;
                            m_used = m_new;
                        }
                    }
                }
                float psum = 0.f;
                uint32_t pk[kKeys / 2];
                if (m_used != -INFINITY) {
                    const float neg = -m_used;
                    float ps8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int j = 0; j < kKeys; j += 2) {
                        const float e0 = fast_exp2(fmaf(sc[j], sl2, neg));
                        const float e1 = fast_exp2(fmaf(sc[j + 1], sl2, neg));
                        ps8[(j >> 1) & 7] += e0 + e1;
                        __nv_bfloat162 v2 = __floats2bfloat162_rn(e0, e1);
                        pk[j / 2] = *reinterpret_cast<uint32_t *>(&v2);
                    }
                    psum = ((ps8[0] + ps8[1]) + (ps8[2] + ps8[3])) + ((ps8[4] + ps8[5]) + (ps8[6] + ps8[7]));
                } else {
#pragma unroll
                    for (int j = 0; j < kKeys / 2; ++j) pk[j] = 0u;
                }
                l += psum;
                // P over the first 32 columns of S buffer bs (bf16 pairs: key 2c in
                // the low half of column c), the A operand of P V
                tmem_st32(tS + 64 * bs + lane_off, reinterpret_cast<const float *>(pk));
                tmem_wait_st();
                fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarPReady + bs));
            }
            if (failed) break;
            // the unit's last P V has landed in O
            failed = __any_sync(0xffffffffu, !mbar_wait(bar(kBarODone + ((T - 1) & 1)), ((T - 1) >> 1) & 1));
            if (failed) break;
            fence_after_sync();
            const float inv = 1.f / l;
            const size_t grow = (size_t)U.grp * GN + (row_ok ? row : 0);   // row of the group-row layout
            // lambda merge of the two blocks ("Quick read / How it works" merge
            // equation): lam_kg = e^{LSE_kg} / (e^{LSE_kg} + e^{LSE_seq}), in log2 units
            float lam_kg = 1.f, lam_seq = 0.f, lse2 = m_used + log2f(l);
            const float *os = nullptr;
            if (p.mode == kAttnLeaf && row_ok) {
                const float lse_kg2 = lse2;
                const float lse_seq2 = p.lse_seq[grow] * 1.44269504088896340736f;
                const float M = fmaxf(lse_kg2, lse_seq2);
                const float wk = exp2f(lse_kg2 - M), wq = exp2f(lse_seq2 - M);
                lam_kg = wk / (wk + wq);
                lam_seq = wq / (wk + wq);
                lse2 = M + log2f(wk + wq);
                os = p.oseq + grow * D;
            }
            __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(p.out) + (((size_t)U.b * p.N + n) * p.H + h) * D;
            float *odst = p.mode == kAttnSeq ? p.oseq + grow * D : nullptr;
            const float a = inv * lam_kg;
#pragma unroll
            for (int c = 0; c < D; c += 32) {
                float ov[32];
                tmem_ld32(tO + lane_off + c, ov);
                tmem_wait_ld();
                if (c == D - 32) {
                    // O has been read: the next unit's first P V may overwrite it
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(kBarODrained));
                }
                if (!row_ok) continue;
                if (odst) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4 *>(odst + c + i) =
                            make_float4(ov[i] * inv, ov[i + 1] * inv, ov[i + 2] * inv, ov[i + 3] * inv);
                    continue;
                }
                if (os) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const float4 q4 = *reinterpret_cast<const float4 *>(os + c + i);
                        ov[i] = fmaf(ov[i], a, lam_seq * q4.x);
                        ov[i + 1] = fmaf(ov[i + 1], a, lam_seq * q4.y);
                        ov[i + 2] = fmaf(ov[i + 2], a, lam_seq * q4.z);
                        ov[i + 3] = fmaf(ov[i + 3], a, lam_seq * q4.w);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] *= inv;
                }
#pragma unroll
                for (int i = 0; i < 32; i += 8) {
                    __nv_bfloat162 a0 = __floats2bfloat162_rn(ov[i], ov[i + 1]);
                    __nv_bfloat162 a1 = __floats2bfloat162_rn(ov[i + 2], ov[i + 3]);
                    __nv_bfloat162 a2 = __floats2bfloat162_rn(ov[i + 4], ov[i + 5]);
                    __nv_bfloat162 a3 = __floats2bfloat162_rn(ov[i + 6], ov[i + 7]);
                    *reinterpret_cast<uint4 *>(dst + c + i) =
                        make_uint4(*reinterpret_cast<uint32_t *>(&a0), *reinterpret_cast<uint32_t *>(&a1),
                                   *reinterpret_cast<uint32_t *>(&a2), *reinterpret_cast<uint32_t *>(&a3));
                }
            }
            if (row_ok) {
                const float lse_nat = lse2 * 0.69314718055994530942f;
                if (p.mode == kAttnSeq) p.lse_seq[grow] = lse_nat;
                else if (p.lse) p.lse[((size_t)U.b * p.N + n) * p.H + h] = lse_nat;
            }
            if (!has_next) break;
            u = un;
            U = tc_unit(p, u, ctas_per_group);
        }
        if (failed && lane == 0) set_status(p.status, kDevTimeout);
    } else if (warp == kProducerWarp) {
        // ================= producer: K and V tiles into their rings =================
        const __nv_bfloat16 *lkb = reinterpret_cast<const __nv_bfloat16 *>(p.lk_base);
        const __nv_bfloat16 *lvb = reinterpret_cast<const __nv_bfloat16 *>(p.lv_base);
        bool failed = false;
        int pending = -1;      // leaf tile (running count) whose cp.async copies are in flight, not yet announced
        uint32_t leafbits = 0; // bit (T mod 32): tile T was gathered (its full barrier is announced by this warp)
        // leaf rows of keys `lane` and `lane + 32` of leaf tile lt of unit U (-1: none)
        auto fetch_rows = [&](const TcUnit &U, int lt, int *rk, int *rv) {
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                const int j = lt * kKeys + lane + 32 * v;
                rk[v] = rv[v] = -1;
                if (j < U.n_leaf) {
                    const int gg = U.g_first + j / p.K_L, jj = j - (j / p.K_L) * p.K_L;
                    const long long e = ((long long)U.b * p.H + U.hkv * p.G + gg) * p.K_L + jj;
                    rk[v] = (int)(p.leaf_head_stride * U.hkv + p.lk_idx[e]);
                    rv[v] = (int)(p.leaf_head_stride * U.hkv + p.lv_idx[e]);
                }
            }
        };
        // cp.async of 64 gathered rows (D / 8 lanes per row, 256 / D rows per warp instruction)
        auto gather = [&](uint32_t dst, const __nv_bfloat16 *base, const int *rows2) {
            constexpr int CPR = D / 8, RPI = 32 / CPR;
            const int c = lane % CPR;
#pragma unroll 4
            for (int i = 0; i < kKeys / RPI; ++i) {
                const int r = RPI * i + lane / CPR;
                const int x = __shfl_sync(0xffffffffu, RPI * i < 32 ? rows2[0] : rows2[1], r & 31);
                cp16(dst + (c >> 3) * (kKeys * 128) + sw128(r, c & 7), x >= 0 ? base + (size_t)x * D + c * 8 : base,
                     x >= 0);
            }
            cp_commit();
        };
        // announce the pending leaf tile once its copies have landed (newer: groups committed after it)
        auto announce = [&](int newer) {
            if (newer) cp_wait_1();
            else cp_wait_all();
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(kBarFullK + pending % kKStages));
                mbar_arrive(bar(kBarFullV + pending % kVStages));
            }
            pending = -1;
        };
        int T = 0, k_issued = 0, v_issued = 0;   // tiles so far; tiles whose K / V copies have been issued
        for (unsigned u = u0; u < n_units && !failed; u += ustride) {
            const TcUnit U = tc_unit(p, u, ctas_per_group);
            int nk[2] = {-1, -1}, nv[2] = {-1, -1};
            if (U.n_leaf_tiles > 0) fetch_rows(U, 0, nk, nv);
            for (int t = 0; t < U.n_tiles; ++t, ++T) {
                const int sk = T % kKStages, sv = T % kVStages;
                const bool leaf = t < U.n_leaf_tiles;
                const int st = t - U.n_leaf_tiles;   // sequence tile index
                const uint32_t kd = sb + kOffK + sk * kKVBytes, vd = sb + kOffV + sv * kKVBytes;
                if (T >= kKStages) {
                    failed = __any_sync(0xffffffffu, !mbar_wait(bar(kBarEmptyK + sk), ((T / kKStages) + 1) & 1));
                    if (failed) break;
                }
                int rk[2] = {-1, -1}, rv[2] = {-1, -1};
                if (leaf) {
                    rk[0] = nk[0];
                    rk[1] = nk[1];
                    rv[0] = nv[0];
                    rv[1] = nv[1];
                    if (t + 1 < U.n_leaf_tiles) fetch_rows(U, t + 1, nk, nv);
                    gather(kd, lkb, rk);
                    leafbits |= 1u << (T & 31);
                } else {
                    leafbits &= ~(1u << (T & 31));
                    if (lane == 0) {
                        mbar_arrive_expect_tx(bar(kBarFullK + sk), kKVBytes);
#pragma unroll
                        for (int half = 0; half < kBlocks; ++half)
                            tma_load_4d(kd + half * (kKeys * 128), tm_k, half * 64, U.hkv, st * kKeys, U.b,
                                        bar(kBarFullK + sk));
                    }
                    __syncwarp();
                }
                k_issued = T + 1;
                // the previous leaf tile goes out before any wait on a V stage
                if (pending >= 0) announce(leaf ? 1 : 0);
                if (T >= kVStages) {
                    failed = __any_sync(0xffffffffu, !mbar_wait(bar(kBarEmptyV + sv), ((T / kVStages) + 1) & 1));
                    if (failed) break;
                }
                if (leaf) {
                    gather(vd, lvb, rv);
                    pending = T;
                } else {
                    if (lane == 0) {
                        mbar_arrive_expect_tx(bar(kBarFullV + sv), kKVBytes);
#pragma unroll
                        for (int half = 0; half < kBlocks; ++half)
                            tma_load_4d(vd + half * (kKeys * 128), tm_v, half * 64, U.hkv, st * kKeys, U.b,
                                        bar(kBarFullV + sv));
                    }
                    __syncwarp();
                }
                v_issued = T + 1;
            }
        }
        if (!failed && pending >= 0) announce(0);
        // The CTA must not exit with copies in flight, on the failure path too:
        // wait (bounded) until the last issued tile of each stage has landed.
        // Gathered tiles are drained by cp.async.wait_group; their full barrier
        // is only announced by this warp, so after a failure only the TMA
        // (sequence) tiles are waited for.
        bool drained = true;
        for (int t = max(0, k_issued - kKStages); t < k_issued; ++t)
            if (!failed || !((leafbits >> (t & 31)) & 1u))
                drained &= mbar_wait(bar(kBarFullK + t % kKStages), (t / kKStages) & 1);
        for (int t = max(0, v_issued - kVStages); t < v_issued; ++t)
            if (!failed || !((leafbits >> (t & 31)) & 1u))
                drained &= mbar_wait(bar(kBarFullV + t % kVStages), (t / kVStages) & 1);
        cp_wait_all();
        if ((failed || !drained) && lane == 0) set_status(p.status, kDevTimeout);
    } else {
        // ================= MMA issue: one thread =================
        if (lane == 0) {
            const uint32_t idesc_s = make_idesc(kRows, kKeys, 0, 0);   // Q (K-major) x K^T (K-major)
            const uint32_t idesc_o = make_idesc(kRows, D, 0, 1);      // P (K-major) x V (MN-major)
            // descriptors of the first tile of each operand region; a tile or
            // K-step offset is added to the start-address field (the low 14 bits,
            // in 16-byte units: shared addresses stay below 256 KB, so no carry)
            const uint64_t dq0 = make_desc(sb + kOffQ, 16, 1024);
            const uint64_t dk0 = make_desc(sb + kOffK, 16, 1024);
            const uint64_t dv0 = make_desc(sb + kOffV, kKeys * 128, 1024);
            int q_loads = 0;   // Q loads consumed so far (QReady phase)
            auto issue_s = [&](int T, bool new_q) -> bool {
                const int sk = T % kKStages, bs = T & 1;
                if (!mbar_wait(bar(kBarFullK + sk), (T / kKStages) & 1)) return false;
                if (new_q) {
                    if (!mbar_wait(bar(kBarQReady), q_loads & 1)) return false;
                    ++q_loads;
                }
                // buffer bs still holds the P of tile T - 2 until its P V has completed
                if (T >= 2 && !mbar_wait(bar(kBarODone + bs), ((T - 2) >> 1) & 1)) return false;
                fence_after_sync();
                const uint64_t kdsc = dk0 + (uint64_t)((sk * kKVBytes) >> 4);
                const uint32_t td = tmem + 64 * bs;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    mma_bf16(td, dq0 + (uint64_t)(((ks >> 2) * (kRows * 128) + (ks & 3) * 32) >> 4),
                             kdsc + (uint64_t)(((ks >> 2) * (kKeys * 128) + (ks & 3) * 32) >> 4), idesc_s,
                             ks > 0 ? 1u : 0u);
                mma_commit(bar(kBarSFull + bs));
                mma_commit(bar(kBarEmptyK + sk));
                return true;
            };
            // P V of tile T; first: the first tile of unit ui (O starts from zero
            // once the previous unit's O has been read out)
            auto issue_pv = [&](int T, bool first, int ui) -> bool {
                const int sv = T % kVStages, bs = T & 1;
                if (!mbar_wait(bar(kBarFullV + sv), (T / kVStages) & 1)) return false;
                if (!mbar_wait(bar(kBarPReady + bs), (T >> 1) & 1)) return false;
                if (first && ui > 0 && !mbar_wait(bar(kBarODrained), (ui - 1) & 1)) return false;
                fence_after_sync();
                const uint32_t ta = tmem + 64 * bs, td = tmem + 128;
                const uint64_t vdsc = dv0 + (uint64_t)((sv * kKVBytes) >> 4);
#pragma unroll
                for (int ks = 0; ks < kKeys / 16; ++ks)
                    mma_bf16_ts(td, ta + 8 * ks, vdsc + (uint64_t)((ks * 16 * 128) >> 4), idesc_o,
                                (!first || ks > 0) ? 1u : 0u);
                mma_commit(bar(kBarODone + bs));
                mma_commit(bar(kBarEmptyV + sv));
                return true;
            };
            bool ok = true;
            int T = 0, ui = 0, prev_ui = 0;
            bool prev_first = false;
            for (unsigned u = u0; u < n_units && ok; u += ustride, ++ui) {
                const TcUnit U = tc_unit(p, u, ctas_per_group);
                for (int t = 0; t < U.n_tiles && ok; ++t, ++T) {
                    // a new Q: the unit's first tile, and its first sequence tile after leaves
                    ok = issue_s(T, t == 0 || (t == U.n_leaf_tiles && t > 0));
                    if (ok && T > 0) ok = issue_pv(T - 1, prev_first, prev_ui);
                    prev_first = t == 0;
                    prev_ui = ui;
                }
            }
            if (ok && T > 0) ok = issue_pv(T - 1, prev_first, prev_ui);
            // before TMEM is released, every MMA this thread committed must have
            // completed, on the failure path too: one more commit tracks them all
            mma_commit(bar(kBarDrain));
            const bool drained = mbar_wait(bar(kBarDrain), 0);
            if (!ok || !drained) set_status(p.status, kDevTimeout);
        }
        __syncwarp();
    }

    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == kMmaWarp) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

// One call: n_units units of (query b, KV head, 128-row block of the group's
// G N rows), a persistent grid (at most as many CTAs as fit on the device)
// taking them round-robin.  tm_k / tm_v: the sequence keys / values
// [B][T][H_kv][D] as 4-D tensor maps (D, H_kv, T, B) with a (64, 1, 64, 1) box
// and 128-byte swizzle; with q_maps, tm_qs / tm_qk: q_seq / q_kg [B][N][H][D]
// as (D, H, N, B) with a (64, 1, min(N, 128), 1) box (else Q by cp.async).
template <int D>
__global__ void __launch_bounds__(tc::kThreads, tc::kMinCtasPerSm)
    attend_tc_kernel(const __grid_constant__ AttnParams p, int ctas_per_group, unsigned n_units,
                     const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_qs, const __grid_constant__ CUtensorMap tm_qk, int q_maps)
{
    griddep_launch();
    griddep_wait();   // the kept lists (and everything else) of the previous grid are visible
    attend_tc_run<D>(p, ctas_per_group, blockIdx.x, gridDim.x, n_units, &tm_k, &tm_v, q_maps ? &tm_qs : nullptr,
                  q_maps ? &tm_qk : nullptr);
}

// Several layers' calls in one launch (same shapes, each layer its own
// inputs and kept leaves): layer l owns the CTAs [offs[l], offs[l + 1]), one
// unit each.
constexpr int kMaxAttnLayers = 32;
struct AttnBatch {
    CUtensorMap mk[kMaxAttnLayers], mv[kMaxAttnLayers];
    AttnParams p[kMaxAttnLayers];
    unsigned offs[kMaxAttnLayers + 1];
    int n, ctas_per_group;
};

template <int D>
__global__ void __launch_bounds__(tc::kThreads, tc::kMinCtasPerSm)
    attend_tc_layers_kernel(const __grid_constant__ AttnBatch b)
{
    int l = 0;
    while (l + 1 < b.n && blockIdx.x >= b.offs[l + 1]) ++l;
    const unsigned u = blockIdx.x - b.offs[l];
    attend_tc_run<D>(b.p[l], b.ctas_per_group, u, 1u, u + 1, &b.mk[l], &b.mv[l], nullptr, nullptr);
}

}  // namespace akv
