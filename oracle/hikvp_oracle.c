/*
 * HiKVP oracle: exact node ranking and the greedy level-by-level descent.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is a plain, slow CPU restatement of the
 * hierarchical key-value pruning (HiKVP) descent described in
 *   "AtlasKV: Augmenting LLMs with Billion-Scale Knowledge Graphs in 20GB VRAM",
 *   section "Quick read / How it works" (root keys resident, score the query
 *   against them, keep the top-K branches, load the next level, prune level by
 *   level down to the leaves) and section "Method details / Hierarchical
 *   clustering of KGKVs" (three levels: root, intermediate, leaf).
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg may load it.
 * It shares no code with the CUDA library and must never be used as a fallback.
 *
 * Node score.  The pages say only that the query is scored against the level's
 * keys.  The reading used here: one score per (query, head) and node, equal to
 * the mean over the query's N tokens of <q_n, k> / sqrt(D).  Since N*sqrt(D) > 0,
 * ranking by that mean is the same as ranking by
 *       x(k) = sum_n sum_d q[n][d] * k[d]
 * which is what this file computes, EXACTLY, as a real number: every input is a
 * binary32 value (bfloat16 inputs widen to binary32 without rounding), so every
 * product q*k is an integer times a power of two, and the sum of those products
 * is accumulated without any rounding in a long fixed-point accumulator
 * (Kulisch's exact dot product).  Ties in the exact value go to the lower
 * storage row id.  Kept sets are reported in ascending row-id order.
 *
 * Parity status: pinned.  tests/test_oracle_exact.py checks the exact values
 * against Python's fractions.Fraction; tests/test_oracle_descent.py checks the
 * per-level top-K property, nesting and the tie rule by brute force on tiny trees.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

/* ---------------------------------------------------------------------------
 * Exact accumulator.  Value = sum_i dig[i] * 2^(32*i - EX_ORIGIN).
 * A binary32 value is m * 2^e with integer m < 2^24 and e >= -149, so a product
 * of two is m * 2^e with m < 2^48 and e >= -298 = -EX_ORIGIN.  Digits are kept
 * in int64 so that up to 2^31 products can be added before normalising.
 * ------------------------------------------------------------------------- */
#define EX_DIGITS 20
#define EX_ORIGIN 298

typedef struct {
    int64_t dig[EX_DIGITS];
} exact_t;

/* Sign, integer significand and exponent of the least significant bit. */
static int split_binary32(uint32_t bits, uint64_t *mant, int *lsb_exp)
{
    int neg = (int)(bits >> 31);
    int biased = (int)((bits >> 23) & 0xffu);
    uint32_t frac = bits & 0x7fffffu;
    if (biased == 0) {            /* zero or subnormal */
        *mant = frac;
        *lsb_exp = -149;
    } else {                      /* normal (inputs are finite) */
        *mant = (uint64_t)(frac | 0x800000u);
        *lsb_exp = biased - 150;
    }
    return neg;
}

static uint32_t load_bits(const void *base, size_t idx, int is_bf16)
{
    if (is_bf16) {
        uint16_t h = ((const uint16_t *)base)[idx];
        return ((uint32_t)h) << 16;   /* bfloat16 -> binary32, exact */
    }
    uint32_t u;
    memcpy(&u, (const char *)base + 4 * idx, 4);
    return u;
}

static void exact_add_product(exact_t *acc, uint32_t a_bits, uint32_t b_bits)
{
    uint64_t ma, mb;
    int ea, eb;
    int neg = split_binary32(a_bits, &ma, &ea) ^ split_binary32(b_bits, &mb, &eb);
    uint64_t m = ma * mb;         /* < 2^48, exact */
    if (m == 0)
        return;
    int pos = ea + eb + EX_ORIGIN;            /* >= 0 */
    int di = pos >> 5, sh = pos & 31;
    unsigned __int128 v = ((unsigned __int128)m) << sh;   /* < 2^79 */
    int64_t c0 = (int64_t)(uint32_t)(v);
    int64_t c1 = (int64_t)(uint32_t)(v >> 32);
    int64_t c2 = (int64_t)(uint32_t)(v >> 64);
    if (neg) {
        acc->dig[di] -= c0;
        acc->dig[di + 1] -= c1;
        acc->dig[di + 2] -= c2;
    } else {
        acc->dig[di] += c0;
        acc->dig[di + 1] += c1;
        acc->dig[di + 2] += c2;
    }
}

/* Canonical form: digits 0..EX_DIGITS-2 in [0, 2^32), top digit signed. */
static void exact_normalize(exact_t *acc)
{
    for (int i = 0; i < EX_DIGITS - 1; ++i) {
        int64_t carry = acc->dig[i] >> 32;         /* floor division by 2^32 */
        acc->dig[i] -= carry * (int64_t)4294967296LL;
        acc->dig[i + 1] += carry;
    }
}

static int exact_cmp(const exact_t *a, const exact_t *b)
{
    for (int i = EX_DIGITS - 1; i >= 0; --i) {
        if (a->dig[i] != b->dig[i])
            return a->dig[i] < b->dig[i] ? -1 : 1;
    }
    return 0;
}

/* x(k) = sum_n sum_d q[n][d] * k[d] for one (query, head), exactly.
 * q points at token 0 of the head; consecutive tokens are q_row_stride
 * elements apart.  k is one key row of D elements. */
static void exact_node_score(const void *q, size_t q_off, size_t q_row_stride, int N,
                             const void *k, size_t k_off, int D, int is_bf16,
                             exact_t *out)
{
    memset(out, 0, sizeof(*out));
    for (int n = 0; n < N; ++n) {
        for (int d = 0; d < D; ++d) {
            uint32_t qb = load_bits(q, q_off + (size_t)n * q_row_stride + d, is_bf16);
            uint32_t kb = load_bits(k, k_off + d, is_bf16);
            exact_add_product(out, qb, kb);
        }
    }
    exact_normalize(out);
}

/* Exported for the pins: the normalized digits of x(k) for a q block [N][D]
 * (row stride D) and a key row k[D]. */
void oracle_exact_dot_digits(const void *q, int N, const void *k, int D, int is_bf16,
                             int64_t *digits_out)
{
    exact_t x;
    exact_node_score(q, 0, (size_t)D, N, k, 0, D, is_bf16, &x);
    memcpy(digits_out, x.dig, sizeof(x.dig));
}

int oracle_exact_digits(void) { return EX_DIGITS; }
int oracle_exact_origin(void) { return EX_ORIGIN; }

/* ---------------------------------------------------------------------------
 * Top-K of one candidate list: sort by (exact score descending, row id
 * ascending), keep the first K, report them in ascending row id.
 * ------------------------------------------------------------------------- */
typedef struct {
    exact_t score;
    int32_t row;
} cand_t;

static int cand_order(const void *pa, const void *pb)
{
    const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
    int c = exact_cmp(&a->score, &b->score);
    if (c != 0)
        return -c;                  /* higher score first */
    return (a->row > b->row) - (a->row < b->row);
}

static int int32_order(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* Tree description, matching the library's layout: keys row-major
 * [H_kv][rows][D]; child tables [H_kv][parents][fanout] of row ids or NULL for
 * the implicit layout child(p, j) = p * fanout + j. */
typedef struct {
    int is_bf16;
    int n_kv_heads, head_dim;
    int b_root, b_mid, b_leaf;       /* fan-outs: roots, mids per root, leaves per mid */
    const void *root_keys;
    const void *mid_keys;
    const void *leaf_keys;
    const int32_t *root_child;
    const int32_t *mid_child;
} oracle_tree;

static void select_level(const oracle_tree *t, const void *keys, size_t level_rows,
                         int hkv, const void *q, size_t q_off, size_t q_stride, int N,
                         const int32_t *cand_rows, int n_cand, int K,
                         cand_t *work, int32_t *kept)
{
    int D = t->head_dim;
    for (int c = 0; c < n_cand; ++c) {
        size_t k_off = ((size_t)hkv * level_rows + (size_t)cand_rows[c]) * (size_t)D;
        exact_node_score(q, q_off, q_stride, N, keys, k_off, D, t->is_bf16, &work[c].score);
        work[c].row = cand_rows[c];
    }
    qsort(work, (size_t)n_cand, sizeof(cand_t), cand_order);
    for (int i = 0; i < K; ++i)
        kept[i] = work[i].row;
    qsort(kept, (size_t)K, sizeof(int32_t), int32_order);
}

/*
 * The descent for a list of traversals (b, h), following the pages' order:
 * roots -> top K_R; children of the kept roots -> top K_I; children of the
 * kept mids -> top K_L.  Each query head h descends in the tree of its KV head
 * h / (H / H_kv).  q_kg is [B][N][H][D].  Outputs are [n_trav][K_*], ascending.
 * Returns 0, or -1 on a bad argument (K above the candidate count, bad table).
 */
int oracle_descend(const oracle_tree *t, const void *q_kg, int B, int N, int H,
                   int K_R, int K_I, int K_L,
                   int n_trav, const int32_t *trav_b, const int32_t *trav_h,
                   int32_t *kept_root, int32_t *kept_mid, int32_t *kept_leaf)
{
    const int D = t->head_dim;
    const int G = H / t->n_kv_heads;
    const size_t n_root = (size_t)t->b_root;
    const size_t n_mid = n_root * (size_t)t->b_mid;
    const size_t n_leaf = n_mid * (size_t)t->b_leaf;
    if (K_R < 1 || K_R > t->b_root || K_I < 1 || K_I > K_R * t->b_mid ||
        K_L < 1 || K_L > K_I * t->b_leaf || G < 1 || H % t->n_kv_heads != 0)
        return -1;
    int max_cand = t->b_root;
    if (K_R * t->b_mid > max_cand) max_cand = K_R * t->b_mid;
    if (K_I * t->b_leaf > max_cand) max_cand = K_I * t->b_leaf;
    int failed = 0;

#pragma omp parallel
    {
        cand_t *work = (cand_t *)malloc(sizeof(cand_t) * (size_t)max_cand);
        int32_t *rows = (int32_t *)malloc(sizeof(int32_t) * (size_t)max_cand);
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < n_trav; ++i) {
            int b = trav_b[i], h = trav_h[i];
            int hkv = h / G;
            size_t q_off = (((size_t)b * N) * H + h) * (size_t)D;
            size_t q_stride = (size_t)H * D;
            int32_t *kr = kept_root + (size_t)i * K_R;
            int32_t *km = kept_mid + (size_t)i * K_I;
            int32_t *kl = kept_leaf + (size_t)i * K_L;

            for (int r = 0; r < t->b_root; ++r)
                rows[r] = r;
            select_level(t, t->root_keys, n_root, hkv, q_kg, q_off, q_stride, N,
                         rows, t->b_root, K_R, work, kr);

            int nc = 0;
            for (int k = 0; k < K_R; ++k)
                for (int j = 0; j < t->b_mid; ++j) {
                    size_t p = (size_t)kr[k];
                    int32_t c = t->root_child
                        ? t->root_child[((size_t)hkv * n_root + p) * t->b_mid + j]
                        : (int32_t)(p * t->b_mid + j);
                    if (c < 0 || (size_t)c >= n_mid) { failed = 1; c = 0; }
                    rows[nc++] = c;
                }
            select_level(t, t->mid_keys, n_mid, hkv, q_kg, q_off, q_stride, N,
                         rows, nc, K_I, work, km);

            nc = 0;
            for (int k = 0; k < K_I; ++k)
                for (int j = 0; j < t->b_leaf; ++j) {
                    size_t p = (size_t)km[k];
                    int32_t c = t->mid_child
                        ? t->mid_child[((size_t)hkv * n_mid + p) * t->b_leaf + j]
                        : (int32_t)(p * t->b_leaf + j);
                    if (c < 0 || (size_t)c >= n_leaf) { failed = 1; c = 0; }
                    rows[nc++] = c;
                }
            select_level(t, t->leaf_keys, n_leaf, hkv, q_kg, q_off, q_stride, N,
                         rows, nc, K_L, work, kl);
        }
        free(work);
        free(rows);
    }
    return failed ? -1 : 0;
}

/* Exact x(k) for an arbitrary candidate list of one traversal, as normalized
 * digits [n_cand][EX_DIGITS]; used by the pins to check selections. */
void oracle_level_scores(const oracle_tree *t, int level, const void *q_kg, int N, int H,
                         int b, int h, const int32_t *rows, int n_cand, int64_t *digits_out)
{
    const int D = t->head_dim;
    const int G = H / t->n_kv_heads;
    const int hkv = h / G;
    const size_t n_root = (size_t)t->b_root;
    const size_t n_mid = n_root * (size_t)t->b_mid;
    const size_t n_leaf = n_mid * (size_t)t->b_leaf;
    const void *keys = level == 0 ? t->root_keys : (level == 1 ? t->mid_keys : t->leaf_keys);
    size_t level_rows = level == 0 ? n_root : (level == 1 ? n_mid : n_leaf);
    size_t q_off = (((size_t)b * N) * H + h) * (size_t)D;
    for (int c = 0; c < n_cand; ++c) {
        exact_t x;
        size_t k_off = ((size_t)hkv * level_rows + (size_t)rows[c]) * (size_t)D;
        exact_node_score(q_kg, q_off, (size_t)H * D, N, keys, k_off, D, t->is_bf16, &x);
        memcpy(digits_out + (size_t)c * EX_DIGITS, x.dig, sizeof(x.dig));
    }
}

/* ---------------------------------------------------------------------------
 * Trees of any depth with a variable number of children per node ("Method
 * details / Hierarchical clustering of KGKVs": the clustering gives clusters
 * of unequal size, and the depth can be set larger).  Level 0 holds the roots,
 * level n_levels - 1 the leaves.  The children of node p of level l (l <
 * n_levels - 1) are given in compressed-sparse-row form per KV head:
 * positions child_off[l][hkv * (rows[l] + 1) + p] .. (p + 1) - 1 of level l's
 * child list, whose entries are row ids of level l + 1 (child_id[l], laid out
 * [H_kv][rows[l + 1]]) or, when child_id[l] is NULL, the positions themselves.
 * The descent is the same greedy one: all roots are candidates; at each next
 * level the candidates are the children of the kept nodes of the level above,
 * ranked by exact score, ties to the lower row id; K[l] are kept per level.
 * ------------------------------------------------------------------------- */
#define ORACLE_MAX_LEVELS 8

typedef struct {
    int is_bf16;
    int n_kv_heads, head_dim, n_levels;
    const int64_t *rows;                       /* [n_levels] rows per KV head */
    const void *const *keys;                   /* [n_levels] keys [H_kv][rows[l]][D] */
    const int32_t *const *child_off;           /* [n_levels - 1] [H_kv][rows[l] + 1] */
    const int32_t *const *child_id;            /* [n_levels - 1] [H_kv][rows[l + 1]] or NULL entries */
} oracle_csr_tree;

/* kept: n_levels arrays, kept[l] is [n_trav][K[l]] (ascending row ids).
 * Returns 0, or -1 on a bad argument (a level with fewer candidates than K,
 * an id out of range). */
int oracle_descend_csr(const oracle_csr_tree *t, const void *q_kg, int N, int H, const int32_t *K,
                       int n_trav, const int32_t *trav_b, const int32_t *trav_h, int32_t *const *kept)
{
    const int D = t->head_dim;
    const int nl = t->n_levels;
    if (nl < 2 || nl > ORACLE_MAX_LEVELS || H % t->n_kv_heads != 0)
        return -1;
    const int G = H / t->n_kv_heads;
    /* the largest candidate list: all roots, or the children of K[l-1] parents */
    int64_t max_cand = t->rows[0];
    for (int l = 1; l < nl; ++l) {
        if (K[l - 1] < 1 || K[l - 1] > t->rows[l - 1])
            return -1;
        if ((int64_t)K[l - 1] * t->rows[l] > max_cand)   /* a safe upper bound */
            max_cand = (int64_t)K[l - 1] * t->rows[l];
    }
    if (K[nl - 1] < 1 || max_cand > (1 << 26))
        return -1;
    int failed = 0;

#pragma omp parallel
    {
        cand_t *work = (cand_t *)malloc(sizeof(cand_t) * (size_t)max_cand);
        int32_t *rows = (int32_t *)malloc(sizeof(int32_t) * (size_t)max_cand);
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < n_trav; ++i) {
            int b = trav_b[i], h = trav_h[i];
            int hkv = h / G;
            size_t q_off = (((size_t)b * N) * H + h) * (size_t)D;
            size_t q_stride = (size_t)H * D;
            const int32_t *prev = NULL;
            int n_prev = 0;
            for (int l = 0; l < nl && !failed; ++l) {
                int nc = 0;
                if (l == 0) {
                    for (int64_t r = 0; r < t->rows[0]; ++r)
                        rows[nc++] = (int32_t)r;
                } else {
                    const int32_t *off = t->child_off[l - 1] + (size_t)hkv * (size_t)(t->rows[l - 1] + 1);
                    const int32_t *ids = t->child_id[l - 1]
                        ? t->child_id[l - 1] + (size_t)hkv * (size_t)t->rows[l] : NULL;
                    for (int k = 0; k < n_prev; ++k) {
                        int32_t p = prev[k];
                        for (int32_t e = off[p]; e < off[p + 1]; ++e) {
                            int32_t c = ids ? ids[e] : e;
                            if (c < 0 || (int64_t)c >= t->rows[l]) { failed = 1; c = 0; }
                            rows[nc++] = c;
                        }
                    }
                }
                if (nc < K[l]) { failed = 1; break; }
                int32_t *out = kept[l] + (size_t)i * K[l];
                for (int c = 0; c < nc; ++c) {
                    size_t k_off = ((size_t)hkv * (size_t)t->rows[l] + (size_t)rows[c]) * (size_t)D;
                    exact_node_score(q_kg, q_off, q_stride, N, t->keys[l], k_off, D, t->is_bf16, &work[c].score);
                    work[c].row = rows[c];
                }
                qsort(work, (size_t)nc, sizeof(cand_t), cand_order);
                for (int k = 0; k < K[l]; ++k)
                    out[k] = work[k].row;
                qsort(out, (size_t)K[l], sizeof(int32_t), int32_order);
                prev = out;
                n_prev = K[l];
            }
        }
        free(work);
        free(rows);
    }
    return failed ? -1 : 0;
}
