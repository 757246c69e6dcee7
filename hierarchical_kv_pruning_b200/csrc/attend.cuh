// Knowledge + causal-sequence attention with the lambda merge, fused.
//
// "AtlasKV: Augmenting LLMs with Billion-Scale Knowledge Graphs in 20GB VRAM":
// the merge equation of "Quick read / How it works" weighs the softmax over the
// kept leaves and the softmax over the sequence by lambda_kg, lambda_seq; with
// lambda = normalised exp of the two log-sum-exps that is exactly one softmax
// over the union of both key sets ("Background / Rectangular attention in
// KBLaM").  The kernels (attend_f32_kernel here for fp32 inputs, the tcgen05
// kernel of attend_tc.cuh for bf16) therefore run a single online softmax:
// over the traversal's kept leaves (q_kg, no mask) and over the causal
// sequence (q_seq, token n sees positions 0..T-N+n, "Background /
// Self-attention").
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

}  // namespace akv
