/*
 * atlaskv.h -- C ABI of the B200 (sm_100a) HiKVP knowledge-graph attention library.
 *
 * HiKVP = hierarchical key-value pruning from "AtlasKV: Augmenting LLMs with
 * Billion-Scale Knowledge Graphs in 20GB VRAM" (ICLR 2026).  For every query b
 * and query head h (a "traversal"; KV head hkv = h / (H / H_kv)):
 *
 *   1. score the query against all root keys and keep the top K_root roots;
 *   2. score the children of the kept roots, keep the top K_mid mids;
 *   3. score the children of the kept mids (the leaves), keep the top K_leaf;
 *   4. attend over the kept leaves (knowledge part) and over the causal
 *      sequence, and merge the two with lambda weights;
 *   (section "Quick read / How it works" of the paper notes; leaves may live in
 *   pinned host memory and are then staged into HBM on demand.)
 *
 * Node score: the mean over the query's N tokens of <q_kg[n], k> / sqrt(D).
 * Ranking uses the EXACT real value of that score computed from the stored
 * numbers (the library filters in fp32 with a rigorous error bound and settles
 * the candidates the bound cannot separate with exact integer arithmetic), so
 * the kept sets depend on the inputs only.  Equal exact scores go to the lower
 * storage row id.  Kept ids are returned in ascending order.
 *
 * Merge ("Quick read / How it works" merge equation; "Method details /
 * Equivalent attention"):  y = lam_kg * Softmax(l_kg) V_kg + lam_seq *
 * Softmax(l_seq) V_seq with lam_kg = e^{LSE_kg} / (e^{LSE_kg} + e^{LSE_seq}),
 * lam_seq = 1 - lam_kg, which equals one softmax over the kept leaves and the
 * visible sequence keys ("Background / Rectangular attention in KBLaM").  The N
 * query tokens are the last N positions of the T-token sequence: token n sees
 * sequence positions 0..T-N+n ("Background / Self-attention" equation) and
 * every kept leaf.
 *
 * Layouts (all row-major, D contiguous, every base pointer 16-byte aligned):
 *   root_keys   [H_kv][b_R][D]            device
 *   mid_keys    [H_kv][b_R*b_I][D]        device, or pinned host memory (then the leaves too)
 *   leaf_keys   [H_kv][b_R*b_I*b_L][D]    device, or pinned host memory
 *   leaf_values [H_kv][b_R*b_I*b_L][D]    same location as leaf_keys
 *   root_child  [H_kv][b_R][b_I]    int32 mid row ids, or NULL: child(r,j) = r*b_I + j
 *   mid_child   [H_kv][b_R*b_I][b_L] int32 leaf row ids, or NULL: child(m,j) = m*b_L + j
 *   q_kg, q_seq [B][N][H][D]              device
 *   k_seq, v_seq [B][T][H_kv][D]          device
 *   out         [B][N][H][D]              device, tree dtype
 *   lse         [B][N][H] float32         device, optional (natural log, of the union)
 *   kept_root   [B][H][K_root] int32      device, optional (likewise kept_mid, kept_leaf)
 *
 * Ownership: the library borrows every buffer; the caller keeps them alive and
 * unmodified while a tree exists (tree buffers) or until the attend call's work
 * on its stream has finished (io buffers and workspace).  The library never
 * allocates device memory inside atlaskv_attend; the caller passes a workspace
 * of atlaskv_workspace_size() bytes (256-byte aligned).
 *
 * Errors: every call returns an atlaskv_status; on a non-OK return nothing was
 * enqueued and no output was written, and atlaskv_last_error() gives a
 * thread-local message.  atlaskv_attend is asynchronous: OK means validated and
 * enqueued on `stream`.  Errors found on the device (a child-table entry out of
 * range, a bounded wait that gave up) set a sticky status word in the tree,
 * read by atlaskv_sync_status().  No call aborts the process or traps the GPU.
 */
#ifndef ATLASKV_H
#define ATLASKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATLASKV_OK = 0,
    ATLASKV_EINVAL = 1,        /* bad argument: shape, K, pointer, alignment */
    ATLASKV_ENOMEM = 2,        /* workspace too small / host allocation failed */
    ATLASKV_ECUDA = 3,         /* a CUDA runtime call failed */
    ATLASKV_EUNSUPPORTED = 4,  /* valid but outside what this build supports */
    ATLASKV_ETIMEOUT = 5,      /* a bounded device wait gave up */
    ATLASKV_EDEVICE = 6        /* device-side check failed (child id out of range) */
} atlaskv_status;

typedef enum { ATLASKV_F32 = 0, ATLASKV_BF16 = 1 } atlaskv_dtype;

typedef enum {
    ATLASKV_LEAVES_DEVICE = 0,       /* leaf keys/values in HBM */
    ATLASKV_LEAVES_HOST_PINNED = 1   /* leaf keys/values in pinned (page-locked) host memory */
} atlaskv_leaf_location;

/* Tree description ("Method details / Hierarchical clustering of KGKVs": three
 * levels, root / intermediate / leaf; only leaves carry values).  Levels below
 * the roots may live in pinned host memory ("Quick read / How it works": only
 * the root keys stay in GPU memory, each next level is loaded from CPU memory
 * after the level above is pruned): the leaves (leaf_location), or the mids
 * and the leaves (mid_location as well).  Their blocks of children are then
 * staged into HBM pools in the workspace, per call, for the kept parents only. */
typedef struct {
    int32_t dtype;             /* atlaskv_dtype of every key/value/query buffer */
    int32_t n_kv_heads;        /* H_kv >= 1: one tree per KV head */
    int32_t head_dim;          /* D: 64 or 128 */
    int32_t fanout[3];         /* b_R roots, b_I mids per root, b_L leaves per mid; each >= 1 */
    const void *root_keys;
    const void *mid_keys;
    const void *leaf_keys;
    const void *leaf_values;
    int32_t leaf_location;     /* atlaskv_leaf_location */
    const int32_t *root_child; /* device, optional */
    const int32_t *mid_child;  /* device, optional */
    int32_t mid_location;      /* atlaskv_leaf_location of mid_keys; HOST_PINNED needs host-pinned leaves too */
} atlaskv_tree_desc;

typedef struct {
    int32_t K_root;            /* 1 <= K_root <= b_R */
    int32_t K_mid;             /* 1 <= K_mid  <= K_root * b_I */
    int32_t K_leaf;            /* 1 <= K_leaf <= K_mid * b_L */
    float scale;               /* logit scale; 0 means 1/sqrt(D) */
} atlaskv_params;

typedef struct {
    int32_t B;                 /* independent queries, >= 0 (0: nothing to do) */
    int32_t N;                 /* query tokens per query, 1 <= N <= T */
    int32_t H;                 /* query heads, a multiple of H_kv */
    int32_t T;                 /* causal sequence length */
    const void *q_kg;          /* KG query (knowledge part and node scores) */
    const void *q_seq;         /* sequence query */
    const void *k_seq;
    const void *v_seq;
    void *out;
    float *lse;                /* optional */
    int32_t *kept_root;        /* optional */
    int32_t *kept_mid;         /* optional */
    int32_t *kept_leaf;        /* optional */
} atlaskv_io;

typedef struct atlaskv_tree atlaskv_tree;

/* Validate a tree description and build the handle.  Checks child tables on
 * the device (every id in range, each level's table a permutation) and computes
 * per-level key-norm bounds used by the ranking filter; this reads every key
 * once (host-pinned leaves are read over the host link) and synchronises
 * `stream` (a cudaStream_t, or NULL for the legacy default stream).
 * Returns EINVAL for a bad description or table, EUNSUPPORTED for D not in
 * {64, 128}, ECUDA if a CUDA call fails.  *out is set only on OK. */
atlaskv_status atlaskv_create_tree(const atlaskv_tree_desc *desc, void *stream, atlaskv_tree **out);

/* ---- Trees of any depth with a variable number of children per node -------
 * "Method details / Hierarchical clustering of KGKVs": a clustering gives
 * clusters of unequal size, and the depth can be set larger than three.  Level
 * 0 holds the roots, level n_levels - 1 the leaves (the only level with
 * values).  The children of node p of level l are listed, per KV head, at
 * positions child_off[l][hkv][p] .. child_off[l][hkv][p + 1] - 1 of level l's
 * child list; child_id[l][hkv][e] is the row (of level l + 1) at position e,
 * or, with child_id[l] NULL, the position e is the row itself (children
 * stored contiguously).  Every row of level l + 1 must be listed exactly once.
 * The descent is the same: candidates of a level are the children of the
 * kept nodes above, K[l] are kept per level, ranked exactly, ties to the lower
 * row id.  All buffers on the device (no host-resident levels).  Calls:
 * atlaskv_create_tree_csr, atlaskv_workspace_size_csr, atlaskv_attend_csr;
 * sync_status, profiling and destroy are shared with the uniform trees. */
#define ATLASKV_MAX_LEVELS 4

typedef struct {
    int32_t dtype;                                 /* atlaskv_dtype */
    int32_t n_kv_heads;                            /* H_kv >= 1 */
    int32_t head_dim;                              /* D: 64 or 128 */
    int32_t n_levels;                              /* 2 .. ATLASKV_MAX_LEVELS */
    int64_t rows[ATLASKV_MAX_LEVELS];              /* nodes per KV head at each level, >= 1 */
    const void *keys[ATLASKV_MAX_LEVELS];          /* [H_kv][rows[l]][D] */
    const int32_t *child_off[ATLASKV_MAX_LEVELS - 1];   /* [H_kv][rows[l] + 1]: 0, non-decreasing, rows[l + 1] */
    const int32_t *child_id[ATLASKV_MAX_LEVELS - 1];    /* [H_kv][rows[l + 1]] rows, or NULL (positions are rows) */
    const void *leaf_values;                       /* [H_kv][rows[n_levels - 1]][D] */
} atlaskv_csr_tree_desc;

typedef struct {
    int32_t K[ATLASKV_MAX_LEVELS];   /* kept per level: 1 <= K[0] <= rows[0]; 1 <= K[l] <= K[l-1] * (fewest
                                        children of a node of level l-1), so every traversal has K[l] candidates */
    float scale;                     /* logit scale; 0 means 1/sqrt(D) */
} atlaskv_level_params;

/* Validate and build a CSR tree.  Reads the offsets to the host once (and
 * synchronises `stream`), checks the child lists on the device, computes the
 * key-norm bounds of every level.  EINVAL for a bad description or child
 * list, EUNSUPPORTED for D not in {64, 128}, ECUDA if a CUDA call fails. */
atlaskv_status atlaskv_create_tree_csr(const atlaskv_csr_tree_desc *desc, void *stream, atlaskv_tree **out);

/* Workspace bytes of atlaskv_attend_csr for these sizes. */
atlaskv_status atlaskv_workspace_size_csr(const atlaskv_tree *tree, const atlaskv_level_params *params,
                                          int32_t B, int32_t N, int32_t H, int32_t T, size_t *bytes);

/* atlaskv_attend for a CSR tree.  io is as for atlaskv_attend except that its
 * kept_root / kept_mid / kept_leaf are ignored: kept, when not NULL, holds
 * n_levels optional outputs, kept[l] [B][H][K[l]] int32 ascending row ids of
 * level l.  The attention uses the leaves kept at the last level. */
atlaskv_status atlaskv_attend_csr(atlaskv_tree *tree, const atlaskv_level_params *params, const atlaskv_io *io,
                                  int32_t *const *kept, void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace atlaskv_attend needs for these sizes (EINVAL on bad sizes). */
atlaskv_status atlaskv_workspace_size(const atlaskv_tree *tree, const atlaskv_params *params,
                                      int32_t B, int32_t N, int32_t H, int32_t T, size_t *bytes);

/* Enqueue the whole path on `stream`: descent (3 levels, staging of host
 * leaves when the tree's leaves are in host memory), knowledge + sequence
 * attention and merge.  `workspace` is device memory of at least
 * atlaskv_workspace_size() bytes, 256-byte aligned, not shared with a
 * concurrent call.
 * - bf16, D = 128: the sequence part depends only on the call's inputs, so it
 *   runs as its own launch on a low-priority stream owned by the tree, beside
 *   the descent (which runs on a high-priority stream owned by the tree); the
 *   knowledge part then merges with it by the lambda weights.
 * - Host-resident leaves: the batch is processed in query chunks (four when
 *   B >= 8, else one; each chunk launches the descent, the staging and the
 *   knowledge part) and the leaf blocks are staged on a third stream owned by
 *   the tree, so the host link works while other chunks compute.
 * Every stream the tree owns joins `stream` again before the call's last
 * kernel, so work enqueued on `stream` afterwards sees the complete results.
 * Because the tree's streams and events are shared by its calls, calls on one
 * tree must not overlap: serialise them, or create one tree per concurrent
 * caller (trees only borrow the key buffers).  The tree's streams and events
 * are created by atlaskv_create_tree; attend creates and allocates nothing.
 * Returns EINVAL / ENOMEM (workspace too small) / EUNSUPPORTED without
 * enqueuing anything. */
atlaskv_status atlaskv_attend(atlaskv_tree *tree, const atlaskv_params *params, const atlaskv_io *io,
                              void *workspace, size_t workspace_bytes, void *stream);

/* Several layers at once (multi-layer batching; per-layer knowledge keys as in
 * "Background / Rectangular attention in KBLaM", where every layer has its own
 * knowledge-key projections): layer l runs the whole path of atlaskv_attend on
 * trees[l] with ios[l], all with the same params.  The layers share one launch
 * per kernel (descent, sequence part, knowledge part), which is what makes a
 * decode step (N = 1, tiny per-layer work) cheap to launch.  Requirements:
 * 1 <= n_layers <= 32; every tree in HBM (no host-resident level), with the
 * same dtype, head_dim and n_kv_heads; every io with the same B, N, H and T;
 * fan-outs may differ as long as the descent's plan is the same (EINVAL
 * otherwise).  The workspace is atlaskv_workspace_size_layers() bytes,
 * 256-byte aligned.  Layer 0's tree lends its streams and events (and its
 * stage times, when its profiling is on): no call on trees[0] may overlap this
 * one.  Device errors of layer l are reported by trees[l]'s sync status. */
atlaskv_status atlaskv_workspace_size_layers(int32_t n_layers, atlaskv_tree *const *trees,
                                             const atlaskv_params *params, const atlaskv_io *ios, size_t *bytes);
atlaskv_status atlaskv_attend_layers(int32_t n_layers, atlaskv_tree *const *trees, const atlaskv_params *params,
                                     const atlaskv_io *ios, void *workspace, size_t workspace_bytes, void *stream);

/* Synchronise `stream` and return the tree's sticky device status (OK,
 * EDEVICE or ETIMEOUT), or ECUDA if the stream reports a CUDA error. */
atlaskv_status atlaskv_sync_status(atlaskv_tree *tree, void *stream);

/* Diagnostics; the paper has no counterpart.  atlaskv_set_profiling takes a
 * bit mask: ATLASKV_PROFILE_TIMES records CUDA events around each stage of
 * later attend calls (cheap, no extra device work); ATLASKV_PROFILE_COUNTERS
 * keeps the descent counters read by atlaskv_refine_stats (a memset and a few
 * atomics per call); 0 turns both off. */
#define ATLASKV_PROFILE_TIMES 1
#define ATLASKV_PROFILE_COUNTERS 2
atlaskv_status atlaskv_set_profiling(atlaskv_tree *tree, int32_t enable);

/* HBM cache of staged leaf blocks across calls (host-resident leaves of a
 * three-level tree).  "Quick read / Results" names the CPU-GPU movement
 * between levels as HiKVP's I/O cost; a branch that recurs over calls need
 * not cross the host link again.  The cache holds `blocks` leaf-key blocks
 * (rounded up to a power of two of 8-way sets; each block is the b_L child
 * key rows of one mid, b_L * head_dim elements) in device memory that the
 * tree allocates here and frees on destroy or on a later call with
 * blocks = 0.  Keyed by (KV head, mid row); least recently used way of a set
 * evicted; blocks of the current call are never evicted by it.  On a hit the
 * block is copied within HBM instead of over the host link; results are
 * identical with and without the cache.  Synchronises `stream` and the
 * tree's staging stream first.  EUNSUPPORTED for HBM-resident or CSR trees,
 * ENOMEM if the allocation fails (the tree then has no cache).  Not during a
 * stream capture. */
atlaskv_status atlaskv_set_leaf_cache(atlaskv_tree *tree, int64_t blocks, void *stream);

/* Cumulative leaf-block cache counters since atlaskv_set_leaf_cache:
 * counts[0] hits (block copied from the cache), [1] fills (read from host
 * memory and kept), [2] bypasses (read from host memory, not kept: its set
 * was full of this call's blocks, or another group of the call was filling
 * it).  Synchronises the device; n is the capacity of counts (at most 3
 * written).  EINVAL without a cache. */
atlaskv_status atlaskv_leaf_cache_stats(atlaskv_tree *tree, uint64_t *counts, int32_t n);

/* How the descent is run; the results are the same either way.
 * ATLASKV_DESCENT_FUSED: one kernel per call, one CTA per (query, KV head,
 *   chunk of heads), running every level; it reads the child rows of the
 *   union of its heads' kept parents (few launches: the choice for small
 *   calls).
 * ATLASKV_DESCENT_PARENT_MAJOR: a few kernels per level; the kept parents of
 *   the whole batch are grouped by (KV head, parent) and each parent's child
 *   rows are read once per group of up to 32 traversals that kept it, so the
 *   bytes read approach the unique rows a level needs (the choice for large
 *   batches).
 * ATLASKV_DESCENT_AUTO (the default): parent-major when B * H >= 1024, else
 *   fused (each where the other's plan does not fit).
 * The mode changes the workspace size: set it before atlaskv_workspace_size.
 * atlaskv_attend_layers always runs the fused kernel. */
#define ATLASKV_DESCENT_AUTO 0
#define ATLASKV_DESCENT_FUSED 1
#define ATLASKV_DESCENT_PARENT_MAJOR 2
atlaskv_status atlaskv_set_descent(atlaskv_tree *tree, int32_t mode);

/* Per-stage device times (ms) of the most recent attend call made with
 * ATLASKV_PROFILE_TIMES: [0] descent levels, [1] host-leaf staging (0 when
 * leaves are in HBM), [2] attention + merge ([3] + [4]), [3] the sequence
 * part when it runs as its own launch (bf16, D = 128; else 0), [4] the leaf
 * part (or the whole attention when it is one launch).  With host leaves
 * [0], [1] and [4] are busy times summed over the query chunks.  Synchronises
 * the stream of that call.  n is the capacity of ms (at most 5 written);
 * returns EINVAL if that call recorded no times. */
atlaskv_status atlaskv_stage_times(atlaskv_tree *tree, float *ms, int32_t n);

/* Descent counters of the most recent attend call made with
 * ATLASKV_PROFILE_COUNTERS, per level l = 0 (roots), 1 (mids), 2 (leaves) and,
 * for deeper CSR trees, 3: counts[4 l + 0] traversals selected, [4 l + 1]
 * selections the fp32 bound could not settle alone, [4 l + 2] ambiguous
 * candidates in those, [4 l + 3] exact scores computed.  Synchronises the
 * device; n is the capacity of counts (at most 16 written). */
atlaskv_status atlaskv_refine_stats(atlaskv_tree *tree, uint64_t *counts, int32_t n);

/* Size in bytes of the static device scratch used by atlaskv_attend_static. */
#define ATLASKV_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* Allocation-free variant of atlaskv_attend.  The paper has no counterpart:
 * this exists for callers that cannot give the library a device workspace --
 * a host program using only this C ABI with no device allocator of its own, a
 * process whose device memory is fully pre-partitioned by another runtime, or a
 * hot loop where a device allocation (which may synchronise the device and
 * take unbounded time) is not allowed.  Same inputs, outputs, validation and
 * results as atlaskv_attend; the scratch comes from a static device array of
 * ATLASKV_STATIC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits.
 * - Sizes whose atlaskv_workspace_size() exceeds ATLASKV_STATIC_SCRATCH_BYTES
 *   are rejected with ATLASKV_ENOMEM and nothing is enqueued (host-resident
 *   leaf trees of realistic size always are: their staging pools are large).
 * - The first call on a device looks up the array's device address (once per
 *   device, with that device current); make that first call before any stream
 *   capture.
 * - All calls share the one array, and it keeps the previous call's contents.
 *   Calls whose work overlaps on the GPU (different streams, or different host
 *   threads, without ordering between them) race on it: serialise them.
 * - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
atlaskv_status atlaskv_attend_static(atlaskv_tree *tree, const atlaskv_params *params, const atlaskv_io *io,
                                     void *stream);

/* Diagnostic; the paper has no counterpart.  Enqueues on `stream` one CTA
 * that waits, with the same bounded mbarrier wait the attention kernel uses,
 * on a barrier that nothing ever arrives on.  The wait gives up after its
 * iteration limit and sets ATLASKV_ETIMEOUT in the tree's sticky status word,
 * which the next atlaskv_sync_status returns; the CUDA context stays usable.
 * It shows that a stalled device wait is reported instead of hanging.  It
 * takes milliseconds or more (the hardware sets each try_wait's suspend
 * time), and it leaves the tree's status at ETIMEOUT, so run it on a tree
 * made for the purpose.  Returns ECUDA if the launch fails. */
atlaskv_status atlaskv_probe_wait_timeout(atlaskv_tree *tree, void *stream);

/* Release the handle and the small device buffers it owns; the caller's
 * buffers are untouched.  NULL is accepted. */
atlaskv_status atlaskv_destroy(atlaskv_tree *tree);

/* Message for the last non-OK status returned on this thread ("" if none). */
const char *atlaskv_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ATLASKV_H */
