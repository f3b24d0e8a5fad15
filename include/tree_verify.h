/*
 * tree_verify.h -- C ABI of the tree-verification library (libtreeverify.so).
 *
 * One speculative-decoding iteration verifies a whole draft token tree
 * against the target model in one pass (SpecExec: Massively Parallel
 * Speculative Decoding For Interactive LLM Inference on Consumer Devices,
 * "Approach").  This library implements the data-parallel hot path of that
 * step as three calls, each a set of hand-written CUDA kernels for sm_100a:
 *
 *   tree_verify_attn  -- tree-masked attention of every draft node over the
 *                        shared KV-cache prefix plus its own ancestors
 *                        (EasySpec page, "Experimental setup", the "+tree"
 *                        baseline; SpecExec page, "Approach"), optionally
 *                        restricted to the top-k prefix blocks chosen by a
 *                        cheap block-mean score ("Accelerate Speculative
 *                        Decoding with Sparse Computation in Verification",
 *                        "Methodology" 3, attention sparsity);
 *   tree_accept       -- the acceptance walk over the verified tree: greedy
 *                        longest match at temperature 0, multi-draft
 *                        speculative sampling with residual resampling
 *                        (SpecExec page, "Builds on": speculative sampling,
 *                        SpecInfer), or SpecExec's sample-and-descend rule
 *                        for deterministic trees (SpecExec page, "Approach");
 *   tree_expand_topb  -- one round of SpecExec's batched best-first
 *                        (Dijkstra-style) tree construction that keeps the
 *                        highest cumulative-probability continuations
 *                        (SpecExec page, "Approach"; "Builds on": Dijkstra's
 *                        algorithm);
 *   tree_commit_kv    -- the accepted path's K/V appended to the cache, so
 *                        that the accepted tokens are prefix for the next
 *                        iteration (SpecExec page, "Approach"; "Key
 *                        results": accepted tokens per target iteration).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every array pointer is DEVICE memory owned by the caller, unless the
 *   field says otherwise.  The argument structs themselves live in host
 *   memory and are read during the call only.
 * - Calls enqueue work on the caller's stream and never synchronise.  They
 *   return a tv_status after host-side argument checks and the launches
 *   (cudaGetLastError); a TV_OK return does not mean the kernels finished.
 * - The library keeps no state between calls and allocates nothing; scratch
 *   comes from a caller buffer `ws` of at least *_workspace_size() bytes
 *   (256-byte aligned).  The workspace must be zero-filled once before its
 *   first use; every call leaves it ready for the next one.  Two calls that
 *   may run concurrently must not share a workspace.
 * - Data-dependent faults are never trapped: the kernels OR bits into the
 *   caller's `dev_status` word (a device uint32, may be NULL) and write the
 *   documented defined output (NaN or -1) instead.
 * - A draft tree is a parent[] array: node 0 is the root (the last committed
 *   token), parent[0] = -1 and 0 <= parent[i] < i (topological order).  A
 *   node attends to itself; the root's row predicts the first new token.
 * - Tree node counts n_nodes[b] <= T may be given per sequence (device
 *   int32 array) or NULL (= T for every sequence).
 */
#ifndef TREE_VERIFY_H
#define TREE_VERIFY_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TV_API __attribute__((visibility("default")))
#else
#define TV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (cudaStream_t); NULL is the legacy default stream. */
typedef struct CUstream_st* tv_stream_t;

/* Host-side result of a call. */
typedef enum {
  TV_OK = 0,
  TV_ERR_INVALID_ARG = 1,   /* a host-checkable argument is out of range  */
  TV_ERR_UNSUPPORTED = 2,   /* valid, but outside what the kernels handle */
  TV_ERR_WORKSPACE = 3,     /* ws is NULL, misaligned or too small        */
  TV_ERR_CUDA = 4           /* a CUDA launch or API call failed           */
} tv_status;

/* Device status bits (ORed into *dev_status by the kernels). */
enum {
  TV_DEV_BAD_PARENT = 1,    /* parent[0] != -1 or parent[i] not in [0, i)  */
  TV_DEV_BAD_TOKEN = 2,     /* a draft token outside [0, V)                */
  TV_DEV_NONFINITE = 4,     /* NaN/Inf logits, or invalid probabilities    */
  TV_DEV_BAD_ROW = 8,       /* expansion row for a missing/expanded node,  */
                            /* or a malformed accepted path (commit)       */
  TV_DEV_BAD_LEN = 16,      /* n_nodes or prefix_len out of range          */
  TV_DEV_TIMEOUT = 32       /* a bounded in-kernel wait expired; the       */
                            /* affected outputs are NaN                    */
};

typedef enum { TV_FP32 = 0, TV_BF16 = 1 } tv_dtype;

/* ------------------------------------------------------------------------
 * tree_verify_attn
 *
 * For sequence b, draft node i < n_nodes[b] and query head h (kv head
 * g = h / (Hq / Hkv), contiguous GQA groups), with K(i) = prefix positions
 * 0 .. prefix_len[b]-1 of the cache plus the tree nodes on the path
 * root .. i (i included):
 *     out[b][i][h] = sum_{j in K(i)} softmax_j(scale * <q, k_j>) v_j
 *     lse[b][i][h] = log sum_{j in K(i)} exp(scale * <q, k_j>)   (natural log)
 * Queries and keys arrive post-RoPE; the caller positions node i at
 * prefix_len[b] + depth(i).  scale = 0 means 1/sqrt(d).
 *
 * Block top-k (sparse_topk > 0): the prefix is cut into blocks of
 * block_size positions; kbar[b][j][g] is the mean of block j's valid keys;
 * for each (b, i, g) the sparse_topk blocks with the largest
 * sum_{h in group g} <q_{i,h}, kbar_j> (ties: lower block index) are kept
 * and K(i) = their keys plus the tree path.  With at most sparse_topk
 * blocks every block is kept (identical to dense).
 *
 * Layouts (element strides; the innermost dimension d is contiguous):
 *   q        [B][T][Hq][d]      strides q_sb, q_st, q_sh
 *   k_cache, v_cache  [B][Lmax][Hkv][d]  strides kv_sb, kv_sl, kv_sh (shared)
 *   k_tree, v_tree    [B][T][Hkv][d]     strides kt_sb, kt_st, kt_sh (shared)
 *   out      [B][T][Hq][d]      strides o_sb, o_st, o_sh   (dtype of q)
 *   lse      [B][T][Hq] fp32 contiguous, or NULL
 *   parent   [B][T] int32, row stride parent_sb
 *   prefix_len [B] int32 (device), each in [0, Lmax]
 *   k_block_mean [B][ceil(Lmax/block_size)][Hkv][d] fp32 contiguous, or NULL
 *            (then computed inside the call)
 *   sel_blocks   [B][T][Hkv][sparse_topk] int32 or NULL: kept block ids,
 *            ascending, -1 padded
 * dtype: TV_FP32 (d in {32, 64, 128}) or TV_BF16 (d in {64, 128}); all of
 * q, caches, tree K/V and out share it.  B, T, Hq, Hkv >= 0; Hq % Hkv == 0.
 * Rows i >= n_nodes[b] are not written.  A node whose parent chain is
 * malformed gets NaN rows (TV_DEV_BAD_PARENT); a sequence whose prefix_len
 * is outside [0, Lmax] gets NaN rows and one whose n_nodes is outside
 * [0, T] gets none (TV_DEV_BAD_LEN).
 *
 * prefix_only = 1 computes a partial instead: each node attends to the
 * prefix keys alone (no tree keys; parent[] is not read), for splitting a
 * long prefix across GPUs (each rank passes its slice of the cache, e.g. a
 * view from row lo, with prefix_len = the slice's length per sequence; one
 * rank keeps prefix_only = 0 so the tree keys are counted once), then
 * tree_verify_attn_merge.  A row with no keys (an empty slice) gets O = 0
 * and lse = -inf.  Not with sparse_topk (TV_ERR_UNSUPPORTED).
 * ---------------------------------------------------------------------- */
typedef struct {
  int32_t dtype;
  int32_t B, T, Hq, Hkv, d, Lmax;
  const void* q;        int64_t q_sb, q_st, q_sh;
  const void* k_cache;
  const void* v_cache;  int64_t kv_sb, kv_sl, kv_sh;
  const int32_t* prefix_len;
  const void* k_tree;
  const void* v_tree;   int64_t kt_sb, kt_st, kt_sh;
  const int32_t* parent; int64_t parent_sb;
  const int32_t* n_nodes;
  float scale;
  int32_t sparse_topk;
  int32_t block_size;
  const float* k_block_mean;
  void* out;            int64_t o_sb, o_st, o_sh;
  float* lse;
  int32_t* sel_blocks;
  uint32_t* dev_status;
  int32_t prefix_only;
} tv_attn_args;

TV_API size_t tree_verify_attn_workspace_size(const tv_attn_args* a);
TV_API tv_status tree_verify_attn(const tv_attn_args* a, void* ws, size_t ws_bytes,
                           tv_stream_t stream);

/* ------------------------------------------------------------------------
 * tree_verify_attn_merge
 *
 * Combines N attention partials over disjoint key sets of the same rows
 * (the outputs and natural-log lse of tree_verify_attn calls on slices of a
 * split prefix, gathered from the ranks) by their log-sum-exp:
 *     M = max_r lse_r,  w_r = exp(lse_r - M),
 *     out = sum_r w_r o_r / sum_r w_r,  lse = M + log sum_r w_r
 * (the same algebra that merges a split prefix inside one GPU).  Layouts,
 * all contiguous device memory: o_parts [N][B][T][Hq][d] (dtype),
 * lse_parts [N][B][T][Hq] fp32, out [B][T][Hq][d] (dtype), lse [B][T][Hq]
 * fp32 or NULL.  A row whose partials are all -inf gets out = 0 and
 * lse = -inf; a NaN lse in any partial makes the row NaN.
 * 1 <= N <= 64, d in {32, 64, 128}; other values TV_ERR_INVALID_ARG /
 * TV_ERR_UNSUPPORTED.  No workspace; enqueues on `stream`.
 * ---------------------------------------------------------------------- */
typedef struct {
  int32_t dtype;
  int32_t N, B, T, Hq, d;
  const void* o_parts;
  const float* lse_parts;
  void* out;
  float* lse;
} tv_attn_merge_args;

TV_API tv_status tree_verify_attn_merge(const tv_attn_merge_args* a, tv_stream_t stream);

/* ------------------------------------------------------------------------
 * tree_accept
 *
 * Walks each sequence's tree from the root.  Row c of target_logits is the
 * target's logits after node c; row c of draft_probs is the draft
 * distribution node c's children were drawn from.  Children are tried in
 * ascending node index.
 *   GREEDY      a = argmax z_c (lowest index on ties); descend to the
 *               lowest-index child carrying a, else emit a and stop.
 *   SPECSAMPLE  p = softmax(z_c / temperature); child j (token x_j) is
 *               accepted when u_j < p(x_j) / q_c(x_j); on rejection p
 *               becomes (p - q_c)^+ / sum (p - q_c)^+ (unchanged when that
 *               sum is 0); with every child rejected (or at a leaf) emit
 *               the inverse-CDF sample of p (smallest t with
 *               sum_{s<=t} p_s > u * sum p) and stop.
 *   SPECEXEC    x = inverse-CDF sample of softmax(z_c / temperature);
 *               descend to the lowest-index child carrying x, else emit x.
 *   AUTO        GREEDY at temperature 0, else SPECSAMPLE.
 * temperature 0 means GREEDY in every mode.  Uniforms: Philox4x32-10
 * (Salmon et al., SC'11) with key (seed mod 2^32, seed >> 32) and counter
 * (node, b, (tag << 28) | draw, step mod 2^32); u = top 53 bits of
 * (w0 << 32 | w1) times 2^-53; tag 1 = test of the node's child number
 * `draw`, tag 2 = residual sample, tag 3 = deterministic-tree sample.
 *
 * Inputs:  target_logits [B][T][V] fp32 (row strides tl_sb, tl_st, rows
 *          contiguous); draft_probs [B][T][V] fp32 (dp_sb, dp_st), required
 *          for SPECSAMPLE at temperature > 0, else may be NULL;
 *          draft_tokens [B][T] int32 (tok_sb; entry 0 is ignored);
 *          parent [B][T] int32 (parent_sb); n_nodes [B] or NULL.
 * Outputs: n_accepted [B]; accepted_nodes [B][T] (the accepted path without
 *          the root, -1 padded); out_tokens [B][T+1] (accepted draft tokens
 *          then the bonus token, -1 padded); min_margin [B] fp64 or NULL
 *          (smallest |u - ratio| or relative inverse-CDF margin met on the
 *          path; +inf when none) -- all contiguous.
 * Faults: children with tokens outside [0, V) are skipped (TV_DEV_BAD_TOKEN);
 *          nodes with a malformed parent are nobody's child
 *          (TV_DEV_BAD_PARENT); a visited non-finite row stops the walk with
 *          bonus -1 (TV_DEV_NONFINITE); n_nodes outside [0, T] accepts
 *          nothing (TV_DEV_BAD_LEN).
 * ---------------------------------------------------------------------- */
typedef enum {
  TV_ACCEPT_AUTO = 0,
  TV_ACCEPT_GREEDY = 1,
  TV_ACCEPT_SPECSAMPLE = 2,
  TV_ACCEPT_SPECEXEC = 3
} tv_accept_mode;

typedef struct {
  int32_t B, T, V;
  const float* target_logits;  int64_t tl_sb, tl_st;
  const float* draft_probs;    int64_t dp_sb, dp_st;
  const int32_t* draft_tokens; int64_t tok_sb;
  const int32_t* parent;       int64_t parent_sb;
  const int32_t* n_nodes;
  int32_t mode;
  float temperature;
  uint64_t seed;
  uint64_t step;
  int32_t* n_accepted;
  int32_t* accepted_nodes;
  int32_t* out_tokens;
  double* min_margin;
  uint32_t* dev_status;
} tv_accept_args;

TV_API size_t tree_accept_workspace_size(const tv_accept_args* a);
TV_API tv_status tree_accept(const tv_accept_args* a, void* ws, size_t ws_bytes,
                      tv_stream_t stream);

/* tree_accept without a caller workspace (an interface addition of this
 * library, not a step of the method).  For callers that cannot allocate
 * device memory: code whose device memory is owned by another runtime that
 * reserved it up front (an inference server's pool), or code on a path
 * where cudaMalloc's implicit device-wide synchronisation is not allowed.
 * It computes exactly what tree_accept computes, with the same arguments.
 * Scratch lives in a file-scope device array of the library, about 576 KB,
 * held on every GPU that loads the library until the process exits; it is
 * sized for B * T <= 32768 node rows and B <= 16384, and larger calls return
 * TV_ERR_UNSUPPORTED.  The call allocates nothing (no cudaMalloc/cudaFree);
 * it clears the counters it needs with cudaMemsetAsync on `stream`.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls share the one array and it keeps
 * the last call's contents: calls that may overlap on the GPU (different
 * streams, different host threads) race and must be serialised by the
 * caller. */
TV_API tv_status tree_accept_noalloc(const tv_accept_args* a, tv_stream_t stream);

/* ------------------------------------------------------------------------
 * tree_expand_topb
 *
 * One round of batched best-first expansion.  Tree state (caller-owned
 * device memory, persistent across rounds, set up by tree_expand_init):
 *   n_nodes [1] int32, parent/token [budget] int32, logp [budget] fp64
 *   (cumulative draft log-probability; root 0), and an opaque candidate
 *   pool of tree_expand_pool_bytes(budget, V) bytes.
 * Per call: R rows of draft logits draft_logits [R][V] fp32 (row stride
 * ld_logits elements), row r holding the draft logits after tree node
 * row_node[r] (-1 = no row).  Every (node, token) becomes a candidate with
 *     score = (logp[node] + z[token] / draft_temperature) - lse(node)
 * (lse = logsumexp of z / draft_temperature over the row, fp64); the call
 * appends the sel = min(Bsel, budget - n_nodes) best candidates of the pool
 * plus the new rows under the total order (score desc, parent asc, token
 * asc) as nodes n_nodes, n_nodes+1, ... in that order, writes them to
 * frontier [Bsel] (-1 padded) and *n_appended, and keeps the rest of the
 * candidates that can still be taken in the pool.  A row for a node that
 * is not yet in the tree or was expanded before is skipped
 * (TV_DEV_BAD_ROW); a row with a non-finite logit is skipped
 * (TV_DEV_NONFINITE).
 * mode TV_EXPAND_BEAM (the SpecExec page's ablation, "Replace parallel SSSP
 * tree search with standard beam search") instead ranks only the children of
 * this call's rows: the sel best of them are appended, in the same order,
 * and no candidate is carried to later calls (the rows of one call are one
 * depth of the beam).  Mixing the modes between calls of one tree is not
 * supported.
 * Limits: 1 <= budget <= 8192, 1 <= V <= 262144, 1 <= Bsel,
 * draft_temperature > 0.
 * ---------------------------------------------------------------------- */
typedef enum { TV_EXPAND_BESTFIRST = 0, TV_EXPAND_BEAM = 1 } tv_expand_mode;

typedef struct {
  int32_t V, R, Bsel, budget;
  float draft_temperature;
  const float* draft_logits;  int64_t ld_logits;
  const int32_t* row_node;
  int32_t* n_nodes;
  int32_t* parent;
  int32_t* token;
  double* logp;
  void* pool;                 size_t pool_bytes;
  int32_t* frontier;
  int32_t* n_appended;
  uint32_t* dev_status;
  int32_t mode;               /* tv_expand_mode */
} tv_expand_args;

TV_API size_t tree_expand_pool_bytes(int32_t budget, int32_t V);
TV_API size_t tree_expand_workspace_size(const tv_expand_args* a);
/* Resets the tree to the root alone (token root_token, logp 0) and empties
 * the pool.  The pool needs no other initialisation. */
TV_API tv_status tree_expand_init(const tv_expand_args* a, int32_t root_token,
                           tv_stream_t stream);
TV_API tv_status tree_expand_topb(const tv_expand_args* a, void* ws, size_t ws_bytes,
                           tv_stream_t stream);

/* ------------------------------------------------------------------------
 * tree_commit_kv
 *
 * Makes the accepted tokens prefix for the next iteration (SpecExec page,
 * "Approach"; "Key results" count accepted tokens per target iteration;
 * the pages do not spell out the cache update and this is its plain
 * reading).  For sequence b with L = prefix_len[b], n = n_accepted[b] and
 * the path rows = (0, accepted_nodes[b][0], ..., accepted_nodes[b][n-1]) --
 * the root, then the nodes tree_accept accepted, in path order --
 *     k_cache[b][L + r][g][:] = k_tree[b][rows[r]][g][:]   (V likewise)
 * for r = 0 .. n and every kv head g, then prefix_len[b] = L + n + 1.  The
 * walk's bonus token has no K/V yet: it is the next tree's root.
 * Every row is read before any row is written, so the tree K/V may be rows
 * of the cache itself at or after row L of the same sequence (k_tree =
 * k_cache + L * kv_sl with kt_st = kv_sl, and so on): the accepted rows
 * are then compacted to the front.  No other overlap between the tree and
 * the cache, and none between sequences, is allowed.
 * Layouts (element strides, d contiguous): k_cache, v_cache
 * [B][Lmax][Hkv][d] (kv_sb, kv_sl, kv_sh) and k_tree, v_tree [B][T][Hkv][d]
 * (kt_sb, kt_st, kt_sh) as in tree_verify_attn; n_accepted [B] and
 * accepted_nodes [B][T] (row stride acc_sb) as tree_accept writes them;
 * prefix_len [B] int32, read and then advanced.  dtype TV_FP32 or TV_BF16,
 * 1 <= d <= 1024, base pointers aligned to the element size.  No workspace.
 * Faults: n outside [0, T-1], L outside [0, Lmax] or L + n + 1 > Lmax ->
 * TV_DEV_BAD_LEN; a path node outside [1, T), or a path that does not
 * increase -> TV_DEV_BAD_ROW; such a sequence is left as it was (cache and
 * prefix_len).
 * ---------------------------------------------------------------------- */
typedef struct {
  int32_t dtype;
  int32_t B, T, Hkv, d, Lmax;
  void* k_cache;
  void* v_cache;        int64_t kv_sb, kv_sl, kv_sh;
  int32_t* prefix_len;
  const void* k_tree;
  const void* v_tree;   int64_t kt_sb, kt_st, kt_sh;
  const int32_t* n_accepted;
  const int32_t* accepted_nodes; int64_t acc_sb;
  uint32_t* dev_status;
} tv_commit_args;

TV_API tv_status tree_commit_kv(const tv_commit_args* a, tv_stream_t stream);

/* ------------------------------------------------------------------------
 * Utilities
 * ---------------------------------------------------------------------- */
/* Which kernels tree_verify_attn would run for these arguments:
 * 0 = CUDA-core split-KV, 1 = tcgen05 tensor-core prefix kernel,
 * 2 = block top-k sparse path on CUDA cores, 3 = block top-k sparse path on
 * the tensor-core kernel (bf16, d = 128, blocks of 64, G >= 4),
 * 4 = the tcgen05 kernel in its two-query-tile form (each CTA takes two
 * 128-row tiles of packed (node, head) rows that share every K/V tile;
 * chosen by the same cost model as 1, for long prefixes; the prefix chunks
 * of a tile pair form a thread-block cluster and merge on chip),
 * 5 = the same two-query-tile kernel with up to 16 prefix chunks per tile
 * pair merged through the workspace (no cluster: the planner's choice when
 * more chunks than a cluster fills the GPU better; the workspace holds the
 * chunks' fp32 rows),
 * -1 = the arguments are rejected. */
TV_API int32_t tv_attn_path(const tv_attn_args* a);
/* How many kernels tree_verify_attn launches for these arguments (0 when
 * B or T is 0, -1 when the arguments are rejected): 1 for the tensor-core
 * kernels (paths 1 and 4: prefix chunks are merged inside the launch), 3 on the
 * CUDA-core path (prefix, tree paths, merge), 5 or 6 on
 * the block top-k CUDA-core path (block means unless the caller passes
 * them, block scores, block selection, sparse prefix, tree paths, merge),
 * 3 or 4 on the block top-k tensor-core path (block means, scores,
 * selection, the tensor-core kernel).  Host only; nothing runs. */
TV_API int32_t tv_attn_launches(const tv_attn_args* a);
/* Library version, e.g. "treeverify 0.1.0 sm_100a". */
TV_API const char* tree_verify_version(void);
/* Static text for a tv_status value. */
TV_API const char* tv_status_string(tv_status s);
/* The acceptance uniforms of n draws, computed by the device Philox used in
 * tree_accept: out[k] = u(seed, step, b[k], node[k], draw[k], tag[k]).
 * All arrays are device memory of n entries. */
TV_API tv_status tv_philox_uniforms(uint64_t seed, uint64_t step, const int32_t* b,
                             const int32_t* node, const int32_t* draw,
                             const int32_t* tag, double* out, int32_t n,
                             tv_stream_t stream);
/* The exponential behind tree_expand_topb's fp64 log-sum-exp of a row (a
 * table-driven method: Tang, ACM TOMS 15(2), 1989), for checking it:
 * out[k] = e^(t[k]) for -700 <= t[k] <= 0, 0 for t[k] < -700 (such terms
 * are below 1e-300 of a row's largest, which contributes 1).  t and out
 * are device memory of n entries; t[k] > 0 is not supported (out[k] is
 * then unspecified). */
TV_API tv_status tv_expand_exp(const double* t, double* out, int32_t n, tv_stream_t stream);
/* Test hook for the bounded waits of tree_expand_topb.  With polls > 0,
 * every row staged in shared memory (rows 16-byte aligned with a row stride
 * of a multiple of 4 elements, V*4 bytes small enough) waits for its first
 * chunk as if that copy were lost: `polls` non-blocking tests of a barrier
 * phase that nothing completes.  The wait expires, the row's real copies
 * are drained (bounded wait), the row is dropped (its node counts as
 * expanded, with no children) and TV_DEV_TIMEOUT is set in dev_status.
 * polls = 0 restores normal waits.  Applies to the current device,
 * synchronously; not for use while expansion calls are in flight. */
TV_API tv_status tv_expand_set_wait_limit(uint32_t polls);

#ifdef __cplusplus
}
#endif
#endif /* TREE_VERIFY_H */
