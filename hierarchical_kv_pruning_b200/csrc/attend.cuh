// Knowledge + causal-sequence attention with the lambda merge, fused.
//
// "AtlasKV: Augmenting LLMs with Billion-Scale Knowledge Graphs in 20GB VRAM":
// the merge equation of "Quick read / How it works" weighs the softmax over the
// kept leaves and the softmax over the sequence by lambda_kg, lambda_seq; with
// lambda = normalised exp of the two log-sum-exps that is exactly one softmax
// over the union of both key sets ("Background / Rectangular attention in
// KBLaM").  Both kernels therefore run a single online softmax: first over the
// traversal's kept leaves (q_kg, no mask), then over the causal sequence (q_seq,
// token n sees positions 0..T-N+n, "Background / Self-attention").
#pragma once

#include "common.cuh"

namespace akv {

struct AttnParams {
    const void *q_kg, *q_seq;        // [B][N][H][D]
    const void *k_seq, *v_seq;       // [B][T][H_kv][D]
    const void *lk_base, *lv_base;   // leaf key / value row bases
    const int32_t *lk_idx, *lv_idx;  // [B H][K_L] row of each kept leaf
    long long leaf_head_stride;      // rows per KV head added to the index (0 when indices are absolute)
    long long lk_rows, lv_rows;      // rows in the leaf key / value arrays
    void *out;                       // [B][N][H][D]
    float *lse;                      // [B][N][H] or null
    int B, N, H, H_kv, G, T, K_L;
    float scale_log2;                // scale * log2(e)
    int *status;                     // sticky device status word (bounded waits report here)
    // tensor-core kernel only: which key sets one launch covers (kAttn*), and
    // the sequence part's results handed from the sequence launch to the leaf
    // launch, per (query, KV head) group and group row r = g N + n
    int mode;
    float *oseq;                     // [B H_kv][G N][D] normalised sequence-part output
    float *lse_seq;                  // [B H_kv][G N] its log-sum-exp (natural log)
};

// attend_tc_kernel modes: both key sets in one online softmax; the causal
// sequence alone (writes oseq / lse_seq); the kept leaves alone, merged with
// oseq / lse_seq by the lambda weights in the epilogue.
enum : int { kAttnFused = 0, kAttnSeq = 1, kAttnLeaf = 2 };

// ---------------------------------------------------------------------------
// fp32 path: one warp per (b, n, h) output row, CUDA-core FMA, expf.
template <int D>
__global__ void __launch_bounds__(128) attend_f32_kernel(const AttnParams p)
{
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= (long long)p.B * p.N * p.H) return;
    const int h = (int)(row % p.H);
    const int n = (int)((row / p.H) % p.N);
    const int b = (int)(row / ((long long)p.H * p.N));
    const int hkv = h / p.G;
    const long long bh = (long long)b * p.H + h;
    const float *qk = reinterpret_cast<const float *>(p.q_kg) + row * D;
    const float *qs = reinterpret_cast<const float *>(p.q_seq) + row * D;
    float a[PER], c[PER], acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        a[i] = qk[lane + 32 * i];
        c[i] = qs[lane + 32 * i];
        acc[i] = 0.f;
    }
    const float scale = p.scale_log2 * 0.69314718055994530942f;  // back to the natural-log scale
    float m = -INFINITY, l = 0.f;
    auto visit = [&](const float *krow, const float *vrow, const float *q) {
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) dot = fmaf(q[i], krow[lane + 32 * i], dot);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        const float s = dot * scale;
        const float mn = fmaxf(m, s);
        const float alpha = expf(m - mn);
        const float w = expf(s - mn);
        l = l * alpha + w;
#pragma unroll
        for (int i = 0; i < PER; ++i) acc[i] = fmaf(w, vrow[lane + 32 * i], acc[i] * alpha);
        m = mn;
    };
    const float *lk = reinterpret_cast<const float *>(p.lk_base);
    const float *lv = reinterpret_cast<const float *>(p.lv_base);
    for (int j = 0; j < p.K_L; ++j) {
        const long long rk = p.leaf_head_stride * hkv + p.lk_idx[bh * p.K_L + j];
        const long long rv = p.leaf_head_stride * hkv + p.lv_idx[bh * p.K_L + j];
        visit(lk + rk * D, lv + rv * D, a);
    }
    const float *ks = reinterpret_cast<const float *>(p.k_seq);
    const float *vs = reinterpret_cast<const float *>(p.v_seq);
    const int last = p.T - p.N + n;
    for (int i = 0; i <= last; ++i) {
        const long long r = ((long long)b * p.T + i) * p.H_kv + hkv;
        visit(ks + r * D, vs + r * D, c);
    }
    float *out = reinterpret_cast<float *>(p.out) + row * D;
    const float inv = 1.f / l;
#pragma unroll
    for (int i = 0; i < PER; ++i) out[lane + 32 * i] = acc[i] * inv;
    if (p.lse && lane == 0) p.lse[row] = m + logf(l);
}

// ---------------------------------------------------------------------------
// bf16 path: tensor cores (mma.sync m16n8k16 bf16 -> fp32).
//
// Work item = (b, hkv, g, 16-token chunk); a CTA of 4 warps takes 4 items of
// the same (b, hkv) so they share the sequence K/V tiles in shared memory.
// Sequence K/V tiles of 64 keys are double-buffered with cp.async; each warp's
// kept leaves go through a private 16-key staging area.  Rows are 16-byte
// chunks XOR-swizzled by (row & 7) so ldmatrix reads are conflict free.

namespace mma {

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool valid)
{
    const int sz = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src), "r"(sz));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float *c, const uint32_t *a, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

}  // namespace mma

constexpr int kAttnWarps = 4;
constexpr int kKeyTile = 64;

template <int D>
struct AttnSmem {
    static constexpr int CH = D / 8;                       // 16-byte chunks per row
    static constexpr int TILE_BYTES = kKeyTile * D * 2;    // one K or V tile
    static constexpr int LEAF_BYTES = 16 * D * 2;          // 16 leaf rows
    static constexpr int BYTES = 4 * TILE_BYTES + kAttnWarps * 2 * LEAF_BYTES;
    __device__ static uint32_t off(int row, int chunk) { return (uint32_t)(row * D * 2 + ((chunk ^ (row & 7)) << 4)); }
};

// Running state of one warp's 16 query rows: O accumulators (fp32), row max
// m (log2 domain) and partial row sums l for rows gq (0) and gq + 8 (1).
template <int D>
struct FlashRows {
    static constexpr int KSTEPS = D / 16;
    static constexpr int DT = D / 8;
    uint32_t qa[KSTEPS][4];
    float o[DT][4];
    float m0, m1, l0, l1;

    __device__ __forceinline__ void init()
    {
#pragma unroll
        for (int i = 0; i < DT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
    }

    // S = Q K^T for NT n8-tiles of keys held in `ksm` (swizzled rows 0..8 NT-1).
    template <int NT>
    __device__ __forceinline__ void qk(float (&sc)[NT][4], const uint8_t *ksm) const
    {
        const int lane = threadIdx.x & 31, mi = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
                const int key = np * 16 + (mi >> 1) * 8 + rr;
                const int c = kk * 2 + (mi & 1);
                uint32_t b0, b1, b2, b3;
                mma::ldsm_x4(mma::smem_u32(ksm + AttnSmem<D>::off(key, c)), b0, b1, b2, b3);
                mma::mma_bf16(sc[2 * np], qa[kk], b0, b1);
                mma::mma_bf16(sc[2 * np + 1], qa[kk], b2, b3);
            }
        }
    }

    // Online-softmax update with the (already scaled, masked) log2-domain
    // scores, then O += P V with V rows from `vsm`.
    template <int NT>
    __device__ __forceinline__ void softmax_pv(float (&sc)[NT][4], const uint8_t *vsm)
    {
        const int lane = threadIdx.x & 31, mi = lane >> 3, rr = lane & 7;
        float mx0 = m0, mx1 = m1;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
            mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        // a row that has not seen a valid key yet keeps m = -inf; use 0 as base
        const float base0 = mx0 == -INFINITY ? 0.f : mx0;
        const float base1 = mx1 == -INFINITY ? 0.f : mx1;
        const float al0 = exp2f(m0 - base0), al1 = exp2f(m1 - base1);
        m0 = mx0;
        m1 = mx1;
        l0 *= al0;
        l1 *= al1;
#pragma unroll
        for (int i = 0; i < DT; ++i) {
            o[i][0] *= al0;
            o[i][1] *= al0;
            o[i][2] *= al1;
            o[i][3] *= al1;
        }
#pragma unroll
        for (int kk = 0; kk < NT / 2; ++kk) {
            float e[8];
            e[0] = exp2f(sc[2 * kk][0] - base0);
            e[1] = exp2f(sc[2 * kk][1] - base0);
            e[2] = exp2f(sc[2 * kk][2] - base1);
            e[3] = exp2f(sc[2 * kk][3] - base1);
            e[4] = exp2f(sc[2 * kk + 1][0] - base0);
            e[5] = exp2f(sc[2 * kk + 1][1] - base0);
            e[6] = exp2f(sc[2 * kk + 1][2] - base1);
            e[7] = exp2f(sc[2 * kk + 1][3] - base1);
            l0 += e[0] + e[1] + e[4] + e[5];
            l1 += e[2] + e[3] + e[6] + e[7];
            uint32_t pa[4];
            pa[0] = mma::pack_bf16(e[0], e[1]);
            pa[1] = mma::pack_bf16(e[2], e[3]);
            pa[2] = mma::pack_bf16(e[4], e[5]);
            pa[3] = mma::pack_bf16(e[6], e[7]);
#pragma unroll
            for (int dp = 0; dp < DT / 2; ++dp) {
                const int key = kk * 16 + (mi & 1) * 8 + rr;
                const int c = dp * 2 + (mi >> 1);
                uint32_t b0, b1, b2, b3;
                mma::ldsm_x4_t(mma::smem_u32(vsm + AttnSmem<D>::off(key, c)), b0, b1, b2, b3);
                mma::mma_bf16(o[2 * dp], pa, b0, b1);
                mma::mma_bf16(o[2 * dp + 1], pa, b2, b3);
            }
        }
    }
};

template <int D>
__global__ void __launch_bounds__(kAttnWarps * 32, 2) attend_bf16_kernel(const AttnParams p, int blocks_per_group)
{
    using S = AttnSmem<D>;
    constexpr int CH = S::CH;
    constexpr int KSTEPS = D / 16;
    constexpr int DT = D / 8;
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *ktile[2] = {smem, smem + S::TILE_BYTES};
    uint8_t *vtile[2] = {smem + 2 * S::TILE_BYTES, smem + 3 * S::TILE_BYTES};

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;      // mma groupID / thread-in-group
    const int grp_id = blockIdx.x / blocks_per_group;
    const int blk = blockIdx.x - grp_id * blocks_per_group;
    const int b = grp_id / p.H_kv, hkv = grp_id - b * p.H_kv;
    const int nchunks = (p.N + 15) >> 4;
    const int item = blk * kAttnWarps + warp;
    const bool active = item < p.G * nchunks;
    const int g = active ? item / nchunks : 0;
    const int chunk = active ? item - g * nchunks : 0;
    const int h = hkv * p.G + g;
    const int n0 = chunk * 16;
    const long long bh = (long long)b * p.H + h;

    // causal extent of the CTA (max over its active warps) and of this warp
    int cta_last = -1;
    for (int w = 0; w < kAttnWarps; ++w) {
        const int it = blk * kAttnWarps + w;
        if (it < p.G * nchunks) {
            const int c = it % nchunks;
            cta_last = max(cta_last, p.T - p.N + min(c * 16 + 15, p.N - 1));
        }
    }
    const int warp_last = active ? p.T - p.N + min(n0 + 15, p.N - 1) : -1;
    const int ntiles = (cta_last + kKeyTile) / kKeyTile;   // tiles 0..ntiles-1 cover keys <= cta_last

    const __nv_bfloat16 *kseq = reinterpret_cast<const __nv_bfloat16 *>(p.k_seq);
    const __nv_bfloat16 *vseq = reinterpret_cast<const __nv_bfloat16 *>(p.v_seq);
    const size_t seq_row_stride = (size_t)p.H_kv * D;
    const __nv_bfloat16 *kseq_b = kseq + ((size_t)b * p.T * p.H_kv + hkv) * D;
    const __nv_bfloat16 *vseq_b = vseq + ((size_t)b * p.T * p.H_kv + hkv) * D;

    auto load_tile = [&](int t, int buf) {
        for (int i = threadIdx.x; i < kKeyTile * CH; i += blockDim.x) {
            const int r = i / CH, c = i - r * CH;
            const int key = t * kKeyTile + r;
            const bool ok = key < p.T;
            const size_t src = (size_t)(ok ? key : 0) * seq_row_stride + c * 8;
            mma::cp_async16(ktile[buf] + S::off(r, c), kseq_b + src, ok);
            mma::cp_async16(vtile[buf] + S::off(r, c), vseq_b + src, ok);
        }
        mma::cp_async_commit();
    };
    if (ntiles > 0) load_tile(0, 0);

    FlashRows<D> st;
    st.init();
    const int r0 = n0 + gq, r1 = n0 + gq + 8;
    auto load_q = [&](const void *qptr) {
        const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(qptr);
        const bool ok0 = active && r0 < p.N, ok1 = active && r1 < p.N;
        const __nv_bfloat16 *q0 = q + (((size_t)b * p.N + (ok0 ? r0 : 0)) * p.H + h) * D;
        const __nv_bfloat16 *q1 = q + (((size_t)b * p.N + (ok1 ? r1 : 0)) * p.H + h) * D;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            const int c = kk * 16 + 2 * tq;
            st.qa[kk][0] = ok0 ? *reinterpret_cast<const uint32_t *>(q0 + c) : 0u;
            st.qa[kk][1] = ok1 ? *reinterpret_cast<const uint32_t *>(q1 + c) : 0u;
            st.qa[kk][2] = ok0 ? *reinterpret_cast<const uint32_t *>(q0 + c + 8) : 0u;
            st.qa[kk][3] = ok1 ? *reinterpret_cast<const uint32_t *>(q1 + c + 8) : 0u;
        }
    };

    // ---- knowledge part: this warp's kept leaves, 16 at a time ----
    load_q(p.q_kg);
    uint8_t *lk_sm = smem + 4 * S::TILE_BYTES + warp * 2 * S::LEAF_BYTES;
    uint8_t *lv_sm = lk_sm + S::LEAF_BYTES;
    const __nv_bfloat16 *lkb = reinterpret_cast<const __nv_bfloat16 *>(p.lk_base);
    const __nv_bfloat16 *lvb = reinterpret_cast<const __nv_bfloat16 *>(p.lv_base);
    if (active) {
        for (int j0 = 0; j0 < p.K_L; j0 += 16) {
            for (int i = lane; i < 16 * CH; i += 32) {
                const int r = i / CH, c = i - r * CH;
                const int j = j0 + r;
                const bool ok = j < p.K_L;
                const long long rk = ok ? p.leaf_head_stride * hkv + p.lk_idx[bh * p.K_L + j] : 0;
                const long long rv = ok ? p.leaf_head_stride * hkv + p.lv_idx[bh * p.K_L + j] : 0;
                mma::cp_async16(lk_sm + S::off(r, c), lkb + (size_t)rk * D + c * 8, ok);
                mma::cp_async16(lv_sm + S::off(r, c), lvb + (size_t)rv * D + c * 8, ok);
            }
            mma::cp_async_commit();
            mma::cp_async_wait<0>();
            __syncwarp();
            float sc[2][4];
            st.template qk<2>(sc, lk_sm);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int j = j0 + nt * 8 + 2 * tq;
                sc[nt][0] = j < p.K_L ? sc[nt][0] * p.scale_log2 : -INFINITY;
                sc[nt][1] = j + 1 < p.K_L ? sc[nt][1] * p.scale_log2 : -INFINITY;
                sc[nt][2] = j < p.K_L ? sc[nt][2] * p.scale_log2 : -INFINITY;
                sc[nt][3] = j + 1 < p.K_L ? sc[nt][3] * p.scale_log2 : -INFINITY;
            }
            st.template softmax_pv<2>(sc, lv_sm);
            __syncwarp();
        }
    }

    // ---- sequence part: causal tiles shared by the CTA ----
    load_q(p.q_seq);
    const int lim0 = p.T - p.N + r0, lim1 = p.T - p.N + r1;   // last visible key per row
    for (int t = 0; t < ntiles; ++t) {
        if (t + 1 < ntiles) {
            load_tile(t + 1, (t + 1) & 1);
            mma::cp_async_wait<1>();
        } else {
            mma::cp_async_wait<0>();
        }
        __syncthreads();
        if (active && t * kKeyTile <= warp_last) {
            float sc[8][4];
            st.template qk<8>(sc, ktile[t & 1]);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int key = t * kKeyTile + nt * 8 + 2 * tq;
                sc[nt][0] = key <= lim0 && key < p.T ? sc[nt][0] * p.scale_log2 : -INFINITY;
                sc[nt][1] = key + 1 <= lim0 && key + 1 < p.T ? sc[nt][1] * p.scale_log2 : -INFINITY;
                sc[nt][2] = key <= lim1 && key < p.T ? sc[nt][2] * p.scale_log2 : -INFINITY;
                sc[nt][3] = key + 1 <= lim1 && key + 1 < p.T ? sc[nt][3] * p.scale_log2 : -INFINITY;
            }
            st.template softmax_pv<8>(sc, vtile[t & 1]);
        }
        __syncthreads();
    }

    // ---- epilogue ----
    if (!active) return;
    float l0 = st.l0, l1 = st.l1;
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float inv0 = 1.f / l0, inv1 = 1.f / l1;
    __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(p.out);
    __nv_bfloat16 *o0 = out + (((size_t)b * p.N + r0) * p.H + h) * D;
    __nv_bfloat16 *o1 = out + (((size_t)b * p.N + r1) * p.H + h) * D;
#pragma unroll
    for (int i = 0; i < DT; ++i) {
        const int c = i * 8 + 2 * tq;
        if (r0 < p.N) *reinterpret_cast<uint32_t *>(o0 + c) = mma::pack_bf16(st.o[i][0] * inv0, st.o[i][1] * inv0);
        if (r1 < p.N) *reinterpret_cast<uint32_t *>(o1 + c) = mma::pack_bf16(st.o[i][2] * inv1, st.o[i][3] * inv1);
    }
    if (p.lse && tq == 0) {
        const float ln2 = 0.69314718055994530942f;
        if (r0 < p.N) p.lse[((size_t)b * p.N + r0) * p.H + h] = (st.m0 + log2f(l0)) * ln2;
        if (r1 < p.N) p.lse[((size_t)b * p.N + r1) * p.H + h] = (st.m1 + log2f(l1)) * ln2;
    }
}

}  // namespace akv
