/*
 * medusa.h -- C ABI of libmedusa.so: one Medusa speculative decode step on an
 * NVIDIA B200 (sm_100a).
 *
 * The step has four calls (tree_attention reads none of medusa_heads'
 * outputs, so the two may run concurrently on two streams; tree_verify needs
 * the node tokens and the target's output; kv_commit needs tree_verify's):
 *   medusa_heads    Medusa heads, top-s per head, candidate-tree tokens
 *                   (medusa_heads_shard / medusa_heads_merge: the same over
 *                   vocabulary shards, one per GPU)
 *   tree_attention  attention of every tree node over the prefix KV cache and
 *                   its tree ancestors (one attention layer)
 *   tree_verify     greedy or stochastic verification: longest accepted
 *                   root-to-node path plus one bonus token
 *                   (tree_verify_logits: the stochastic walk reading the
 *                   target's logits at a temperature; tree_verify_greedy_rows
 *                   and tree_verify_greedy_walk: greedy verification's two
 *                   launches on their own)
 *   kv_commit       append the accepted path's K/V to the cache
 * tree_attention_incache and kv_compact are the pair for a cache that already
 * holds the tree's K/V after each prefix (compaction of every layer at once).
 * tree_attention_paged and kv_commit_paged are the two cache calls over a
 * paged KV cache (a page pool and a block table).
 *
 * Sources of the operations (public web pages on Medusa):
 *   [SPEC]  "Speculative Decoding & Medusa Tree Attention: Accelerating LLM
 *           Inference by 3x Without Accuracy Loss", section 2 "The
 *           Mathematical Foundation of Speculative Sampling".
 *   [GUIDE] "Medusa Explained: Multi-Head Speculative Decoding Guide",
 *           sections "The Architectural Blueprint", "1. Combinatorial Tree
 *           Construction", "2. Single-Pass Tree Attention Verification".
 *   [MTP]   "Multi-Token Prediction & Draft-Model-Free Speculative Decoding",
 *           sections "2. EAGLE & EAGLE-2: Feature-Level Autoregression", "The
 *           2D Tree Attention Mask" and "Production Deployment Guidelines".
 *
 * Conventions shared by every call
 *   - Every function returns MEDUSA_OK (0) or a negative MEDUSA_ERR_* code;
 *     medusa_last_error() then gives a message (thread-local).
 *   - Tensor pointers are caller-owned DEVICE memory on the current device,
 *     row-major and contiguous in the layout stated, 16-byte aligned.  The
 *     library never frees or retains them.
 *   - Compute calls are asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  They do not synchronise and do not allocate:
 *     scratch memory is the caller's `workspace` of at least the size the
 *     matching *_workspace_size() query returns.
 *   - Host-side argument errors (null pointer, bad shape, misalignment, too
 *     small a workspace) are reported by the return code before anything is
 *     launched.  Errors that only the data shows (a token id >= V, a cache
 *     overflow, a prefix length out of range, a distribution with no mass)
 *     are OR-ed as MEDUSA_STATUS_* bits into the caller's device int32
 *     `status` (nullable; never cleared by the library) and never trap.
 *   - dtype MEDUSA_F32 computes in fp32 throughout; MEDUSA_BF16 takes bf16
 *     inputs, accumulates in fp32 and stores bf16 activations.
 */
#ifndef MEDUSA_H
#define MEDUSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* medusa_stream_t; /* same type as cudaStream_t */

enum {
    MEDUSA_OK = 0,
    MEDUSA_ERR_INVALID_ARG = -1, /* null pointer, bad size, misaligned pointer, bad tree */
    MEDUSA_ERR_UNSUPPORTED = -2, /* T > 128, head_dim not 64/128, unsupported dtype */
    MEDUSA_ERR_WORKSPACE = -3,   /* workspace smaller than the query says */
    MEDUSA_ERR_CUDA = -4         /* a CUDA launch or runtime call failed */
};

/* device-side status bits (OR-ed into *status) */
enum {
    MEDUSA_STATUS_BAD_TOKEN = 1,      /* a token / node id outside its range */
    MEDUSA_STATUS_CACHE_OVERFLOW = 2, /* kv_commit: prefix_len + len > S_max */
    MEDUSA_STATUS_BAD_PREFIX = 4,     /* prefix_len outside [0, max_prefix] */
    MEDUSA_STATUS_NO_MASS = 8,        /* stochastic bonus drawn from an all-zero distribution */
    MEDUSA_STATUS_TIMEOUT = 16,       /* an internal pipeline wait gave up after ~2 s (a library bug), or after
                                         the limit set by medusa_debug_set_wait_limit */
    MEDUSA_STATUS_BAD_PAGE = 32,      /* a needed block-table entry outside [0, num_pages) */
    MEDUSA_STATUS_BAD_LAYER = 64      /* kv_compact: a layer's cache pointer is NULL or not 16-byte aligned */
};

typedef enum { MEDUSA_F32 = 0, MEDUSA_BF16 = 1 } medusa_dtype;
typedef enum { MEDUSA_VERIFY_GREEDY = 0, MEDUSA_VERIFY_STOCHASTIC = 1 } medusa_verify_mode;

/* largest top-s list per head and largest tree */
#define MEDUSA_TOPK 8
#define MEDUSA_MAX_TREE 128

/* Message of the last failed call on this thread ("" if none). */
const char* medusa_last_error(void);

/* ABI version (major * 100 + minor). */
int medusa_version(void);

/*
 * Error-path testing aid (not part of the method).  Every pipeline wait in
 * the bf16 heads and tree attention kernels (a stage's copy, an MMA, a
 * hand-over flag, a grid barrier) gives up after a limit, sets
 * MEDUSA_STATUS_TIMEOUT in the call's status word and lets the kernel finish
 * without hanging the GPU.  This sets that limit for calls launched
 * afterwards, process-wide: ns = 0 restores the default (about two seconds);
 * ns = 1 makes a wait give up at once unless already satisfied, so those
 * calls end with MEDUSA_STATUS_TIMEOUT and meaningless outputs.  Waits for
 * copies and MMAs a kernel has already issued always keep the default limit,
 * so no kernel exits with work of its own in flight.
 */
void medusa_debug_set_wait_limit(uint64_t ns);

/*
 * Launch shape of the calls the calling host thread makes afterwards (a
 * library convenience for running calls concurrently on separate streams;
 * not part of the method).  heads_ctas > 0: the bf16 tensor-core heads
 * kernel (one cooperative CTA per SM by default) uses at most that many
 * CTAs, leaving the other SMs to kernels on other streams.
 * attention_splits > 0: the bf16 tensor-core tree attention kernel uses at
 * most that many key splits per 128-row tile (1: no thread-block cluster,
 * so its CTAs can run on any free SM).  0 restores the default.  Results
 * stay within the float tolerances; the launch shape may change the last
 * bits of floating-point outputs (rounding order of partial sums), never
 * which work is done.  Returns MEDUSA_ERR_INVALID_ARG for negative values.
 */
int medusa_set_launch_shape(int heads_ctas, int attention_splits);

/* ------------------------------------------------------------------------ */
/* Candidate tree                                                            */
/* ------------------------------------------------------------------------ */

/*
 * Opaque, immutable description of a candidate tree ([GUIDE] "1. Combinatorial
 * Tree Construction": the tree is flattened into one packed sequence of T
 * nodes; [MTP] "The 2D Tree Attention Mask": node i may attend to node j when
 * j is an ancestor of i or j = i).
 *
 * parent_host: HOST array of T int32.  Node 0 is the single root
 *   (parent -1); for i > 0, 0 <= parent[i] < i.  Siblings are ordered by
 *   index.  A node's depth counts the root as 1; a node at depth k >= 2 with
 *   sibling rank r (number of earlier siblings) holds entry r of Medusa head
 *   k-1's top-s list.
 * T: 1 <= T <= MEDUSA_MAX_TREE.
 * out: receives the handle.  The call allocates a few KB of device memory on
 *   the current device (set-up time, not on the step) and synchronises; the
 *   handle is valid on that device only.
 * Errors: MEDUSA_ERR_INVALID_ARG (bad parent array), MEDUSA_ERR_UNSUPPORTED
 *   (T > 128), MEDUSA_ERR_CUDA.
 */
typedef struct medusa_tree medusa_tree;
int medusa_tree_create(const int32_t* parent_host, int T, medusa_tree** out);

/*
 * One tree per sequence ([MTP] "2. EAGLE & EAGLE-2: Feature-Level
 * Autoregression": dynamic trees shaped per sequence; "Production
 * Deployment Guidelines": tree depth tuned to the workload).  Tree i's parent
 * array is parents_host[offsets_host[i] .. offsets_host[i+1]) (HOST arrays;
 * offsets_host has ntrees + 1 entries, offsets_host[0] = 0), each obeying the
 * rules above.  A handle with ntrees > 1 is used by calls with B = ntrees:
 * sequence b uses tree b.  Such calls keep the [B, T, ...] layouts of the
 * single-tree calls with T = the largest tree's node count (medusa_tree_info);
 * sequence b uses the first T_b rows of its block.  Rows past T_b are
 * ignored on input; on output node_tokens holds -1 and node_q 0 there, and
 * tree_attention writes zeros (lse -inf).  q_row of tree_verify is then
 * [B, T] (row b * T + u for node u of sequence b).
 * Errors: as medusa_tree_create, naming the offending tree.
 */
int medusa_tree_create_ragged(const int32_t* parents_host, const int32_t* offsets_host, int ntrees,
                              medusa_tree** out);

/* Frees the handle (synchronises the device first).  NULL is a no-op. */
int medusa_tree_destroy(medusa_tree* tree);

/* Node count, maximum depth (root = 1) and the largest child count; over all
 * trees of the handle (T: the largest tree's node count). */
int medusa_tree_info(const medusa_tree* tree, int* T, int* max_depth, int* max_children);

/* Number of trees in the handle (1 for medusa_tree_create) and, if T_each is
 * not NULL, each tree's node count (HOST array of ntrees int32). */
int medusa_tree_ntrees(const medusa_tree* tree, int* ntrees, int32_t* T_each);

/* ------------------------------------------------------------------------ */
/* Medusa heads                                                              */
/* ------------------------------------------------------------------------ */

/*
 * [GUIDE] "The Architectural Blueprint": for every sequence b and Medusa head
 * k = 1..K (array index k-1),
 *     h^(k) = SiLU(W_res^(k) h) + h,    p^(k) = softmax(W_head^(k) h^(k)),
 * no bias.  Then ([GUIDE] "1. Combinatorial Tree Construction") each head's
 * top-MEDUSA_TOPK tokens (logit descending, lower token id first among equal
 * logits) with their probabilities, and, if `tree` is given, the tree's node
 * tokens: node 0 gets root_token[b] (w_{t+1}, the base model's own next
 * token); a node at depth k+1 with sibling rank r gets topk_idx[b,k-1,r].
 *
 * h        [B, d]         dtype dt
 * W_res    [K, d, d]      dtype dt, row = output feature, column = input
 * W_head   [K, V, d]      dtype dt
 * root_token [B] int32    (read only when tree != NULL)
 * topk_idx [B, K, 8] int32 out   (-1 where V < 8)
 * topk_prob [B, K, 8] f32 out    softmax probability of each entry
 * node_tokens [B, T] int32 out  (tree != NULL)
 * node_q   [B, T] f32 out, nullable: probability of each node's token under
 *          the head that proposed it (1 at the root)
 * h_res_out [B, K, d] dtype dt, nullable: h^(k) (bf16-rounded for BF16)
 * logits_out [B, K, V] f32, nullable;  probs_out [B, K, V] f32, nullable
 * Limits: d % 8 == 0 (BF16) or d % 4 == 0 (F32); d <= 16384; 1 <= V;
 *   1 <= K <= 16; tree max depth <= K + 1 and every sibling rank < 8.
 * Workspace: medusa_heads_workspace_size(B, d, V, K, dt) bytes.
 */
size_t medusa_heads_workspace_size(int B, int d, int V, int K, medusa_dtype dt);
int medusa_heads(const void* h, const void* W_res, const void* W_head, int B, int d, int V, int K,
                 medusa_dtype dt, const medusa_tree* tree, const int32_t* root_token, int32_t* topk_idx,
                 float* topk_prob, int32_t* node_tokens, float* node_q, void* h_res_out, float* logits_out,
                 float* probs_out, void* workspace, size_t workspace_bytes, int32_t* status,
                 medusa_stream_t stream);

/*
 * medusa_heads without a workspace argument (the pages have no counterpart:
 * this is a library convenience, not part of the method).  For callers that
 * cannot allocate device memory -- a plug-in inside a framework that owns all
 * of the GPU's memory and offers it no allocator, or a loop that must never
 * call cudaMalloc/cudaFree because they synchronise the device.  Same
 * arguments and results as medusa_heads, minus workspace/workspace_bytes.
 *   - Scratch is a fixed 32 MiB array inside the library's device code; every
 *     GPU that loads the library holds it until the process exits.  Sizes
 *     whose medusa_heads_workspace_size exceeds 32 MiB are rejected with
 *     MEDUSA_ERR_UNSUPPORTED and a message; nothing is launched.
 *   - Every call looks up the array's device address on the current device
 *     (a host-side lookup, repeated per call so that a reset and re-created
 *     context never leaves a stale address behind).  The first call on a
 *     device may also load the library's device code there; make that first
 *     call before any stream capture begins.
 *   - The call itself allocates nothing (no cudaMalloc/cudaFree).
 *   - Every call on a device shares the one array: calls whose work overlaps
 *     on the GPU (different streams, or different host threads) race and
 *     corrupt each other's results; serialise them.  No part of the scratch
 *     needs to start at zero: each call writes every byte it later reads.
 */
int medusa_heads_noalloc(const void* h, const void* W_res, const void* W_head, int B, int d, int V, int K,
                         medusa_dtype dt, const medusa_tree* tree, const int32_t* root_token, int32_t* topk_idx,
                         float* topk_prob, int32_t* node_tokens, float* node_q, void* h_res_out, float* logits_out,
                         float* probs_out, int32_t* status, medusa_stream_t stream);

/*
 * Vocabulary-sharded heads (one GPU per shard of W_head's rows; the pages
 * describe no sharding, so this is a library layout, not a step of the
 * method): the softmax over the full vocabulary and its top-8 are recovered
 * exactly from each shard's (m, l, top-8), because
 *     M = max_r m_r,   L = sum_r l_r * exp(m_r - M),   p(x) = exp(z(x) - M) / L
 * and the global top-8 is the top-8 of the shards' top-8 lists.  Each rank
 * runs medusa_heads_shard on its rows, the ranks exchange the B*K partials
 * (72 bytes each; an all-gather in rank order), and every rank (or one) runs
 * medusa_heads_merge, whose outputs are those of medusa_heads.
 *
 * medusa_head_partial: softmax statistics (m = max logit, l = sum of
 * exp(logit - m)) of one (sequence, head) over a set of vocabulary rows, and
 * its 8 best (logit, token id) pairs, best first (larger logit, lower id
 * among equal ones); missing entries are (-inf, INT32_MAX).
 */
typedef struct {
    float m, l;
    float val[MEDUSA_TOPK];
    int32_t idx[MEDUSA_TOPK];
} medusa_head_partial;

/*
 * medusa_heads over vocabulary rows [v_offset, v_offset + V_shard):
 * W_head_shard [K, V_shard, d] (those rows of W_head); h, W_res, B, d, K,
 * dt as medusa_heads (the residual block is computed in full on every
 * shard).  partial_out [B, K] device: the shard's partial per (sequence,
 * head), token ids in the full vocabulary.  No tree is filled.
 * Errors as medusa_heads; v_offset >= 0 and v_offset + V_shard <= INT32_MAX.
 * Workspace: medusa_heads_shard_workspace_size(B, d, V_shard, K, dt) bytes.
 */
size_t medusa_heads_shard_workspace_size(int B, int d, int V_shard, int K, medusa_dtype dt);
int medusa_heads_shard(const void* h, const void* W_res, const void* W_head_shard, int B, int d, int V_shard,
                       int v_offset, int K, medusa_dtype dt, medusa_head_partial* partial_out, void* workspace,
                       size_t workspace_bytes, int32_t* status, medusa_stream_t stream);

/*
 * Merges n_shards partial sets partials [n_shards, B, K] (device; shard r's
 * block in rank order, each from medusa_heads_shard) into medusa_heads'
 * outputs: topk_idx, topk_prob [B, K, 8] and, if tree is given, node_tokens
 * and node_q [B, T] from root_token [B] (same rules and errors as
 * medusa_heads).  V is the full vocabulary size (token ids must lie below
 * it).  The shards' statistics are merged in shard order, so the result does
 * not depend on which rank merges.  No workspace.
 */
int medusa_heads_merge(const medusa_head_partial* partials, int n_shards, int B, int K, int V,
                       const medusa_tree* tree, const int32_t* root_token, int32_t* topk_idx, float* topk_prob,
                       int32_t* node_tokens, float* node_q, int32_t* status, medusa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Tree attention                                                            */
/* ------------------------------------------------------------------------ */

/*
 * [GUIDE] "2. Single-Pass Tree Attention Verification" and [MTP] "The 2D Tree
 * Attention Mask": every tree node i attends to the whole cached prefix and
 * to the tree nodes j that are its ancestors or itself.  For query head h
 * (kv-head g = h / (Hq/Hkv)):
 *     O[b,i,h,:] = sum_j softmax_j(scale * <q[b,i,h,:], k_j>) v_j
 * over j in cache positions [0, prefix_len[b]) of kv-head g and the visible
 * tree nodes.  RoPE and all projections are the caller's (Q/K/V arrive ready).
 *
 * q        [B, T, Hq, D]       dtype dt
 * k_tree, v_tree [B, T, Hkv, D] dtype dt (this step's tree K/V)
 * k_cache, v_cache [B, Hkv, S_max, D] dtype dt (only [0, prefix_len[b]) read)
 * prefix_len [B] int32, device; each in [0, max_prefix]
 * max_prefix: upper bound of prefix_len the grid is sized for (0 = S_max)
 * scale: softmax scale; <= 0 means 1/sqrt(D)
 * out      [B, T, Hq, D]       dtype dt
 * lse      [B, T, Hq] f32, nullable: natural-log sum of exp of the scaled scores
 * Limits: D in {64, 128}; Hq % Hkv == 0; T = tree node count (<= 128; with
 * one tree per sequence, the largest tree's).
 * A prefix_len outside [0, max_prefix] sets MEDUSA_STATUS_BAD_PREFIX and the
 * sequence's rows are computed over the clamped prefix.
 * Workspace: tree_attention_workspace_size(...) bytes.
 */
size_t tree_attention_workspace_size(int B, int Hq, int Hkv, int D, int S_max, int max_prefix,
                                     const medusa_tree* tree, medusa_dtype dt);
int tree_attention(const void* q, const void* k_tree, const void* v_tree, const void* k_cache,
                   const void* v_cache, const int32_t* prefix_len, int B, int Hq, int Hkv, int D, int S_max,
                   int max_prefix, float scale, medusa_dtype dt, const medusa_tree* tree, void* out, float* lse,
                   void* workspace, size_t workspace_bytes, int32_t* status, medusa_stream_t stream);

/*
 * tree_attention with this step's tree K/V already written into the cache
 * right after each prefix (the layout an engine has when the target model's
 * layers append the tree's K/V to the cache before attention; the commit is
 * then an in-place compaction, kv_compact):
 *     k_tree[b, j, g, :] is k_cache[b, g, prefix_len[b] + j, :]  (j < T_b)
 * and likewise for V.  Every other argument, output and error as
 * tree_attention; no k_tree / v_tree.  Rows of the cache at or past
 * prefix_len[b] + T_b are never used (they may hold anything).
 * Limits: contiguous caches only; max_prefix + T <= S_max (max_prefix 0
 * means S_max - T), else MEDUSA_ERR_INVALID_ARG.
 * Workspace: tree_attention_incache_workspace_size(...) bytes.
 */
size_t tree_attention_incache_workspace_size(int B, int Hq, int Hkv, int D, int S_max, int max_prefix,
                                             const medusa_tree* tree, medusa_dtype dt);
int tree_attention_incache(const void* q, const void* k_cache, const void* v_cache, const int32_t* prefix_len,
                           int B, int Hq, int Hkv, int D, int S_max, int max_prefix, float scale, medusa_dtype dt,
                           const medusa_tree* tree, void* out, float* lse, void* workspace, size_t workspace_bytes,
                           int32_t* status, medusa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Verification                                                              */
/* ------------------------------------------------------------------------ */

/*
 * GREEDY ([GUIDE] "2. Single-Pass Tree Attention Verification", steps 2-4;
 * [MTP] "The 2D Tree Attention Mask": the longest accepted path plus one
 * bonus token from the target): the target's prediction after node u is
 * argmax(target[b,u,:]) (largest logit, lowest id among equal ones, NaN never
 * wins).  The root is accepted; node c is accepted when its parent is and
 * node_tokens[b,c] equals the parent's prediction.  The path ends at the
 * deepest accepted node (lowest index among equally deep ones); the bonus is
 * that node's prediction.
 *   target: logits [B, T, V], dtype target_dt (F32 or BF16).
 *
 * STOCHASTIC ([SPEC] section 2: accept x with probability
 * min(1, P_target(x)/P_draft(x)); on rejection resample from
 * normalize(max(0, P_target - P_draft))), walked over the tree: at the
 * current node u, with current distribution P (first p[b,u,:]) and draft
 * Q = q[b, q_row[u], :], children are tried in index order.  Child c with
 * token x is accepted iff u_c * Q(x) < P(x); the walk then moves to c with
 * P = p[b,c,:].  On rejection P becomes the residual W/S with
 * W(y) = floor(max(0, P(y) - Q(y)) * 2^32), S = sum W (P kept when S = 0).
 * When no child is left the bonus is the smallest y whose inclusive prefix
 * sum of floor(P(y) * 2^32) exceeds floor(U * S / 2^32).  Uniforms come from
 * Philox4x32-10 (Salmon et al., SC'11) with key (seed low word, seed high
 * word) and counter (b, node, step, 0): u_c = (word0 >> 8) * 2^-24 of child
 * c's block, U = word1 of the block of the node where the walk ends.  All
 * arithmetic is integer or correctly rounded fp64, so results are exact.
 *   target: p [B, T, V] f32 (target_dt must be MEDUSA_F32);
 *   q [B, q_rows, V] f32; q_row [T] int32 device ([B, T] with one tree per
 *   sequence), nullable (identity, then q_rows must equal T).  Medusa heads' probs_out [B, K, V] serves as q with
 *   q_row[u] = depth(u) - 1.
 *
 * node_tokens [B, T] int32; accept_path [B, max_path] int32 out (node ids,
 * root first, -1 padded); accept_len [B] int32 out (>= 1, counts the root);
 * bonus [B] int32 out.  max_path >= the tree's max depth.
 * Workspace: tree_verify_workspace_size(...) bytes, 16-byte aligned, device
 * memory owned by the caller (greedy: row-argmax partials; stochastic: two
 * 8-byte integer weights per sequence and vocabulary entry, 16 * B * V bytes
 * plus alignment).  Its contents need no initialisation; concurrent calls
 * need separate workspaces.  Too small a workspace fails with
 * MEDUSA_ERR_WORKSPACE before anything is launched.
 */
size_t tree_verify_workspace_size(medusa_verify_mode mode, int B, int V, const medusa_tree* tree);
int tree_verify(medusa_verify_mode mode, const void* target, medusa_dtype target_dt, const float* q, int q_rows,
                const int32_t* q_row, const int32_t* node_tokens, int B, int V, const medusa_tree* tree,
                uint64_t seed, uint32_t step, int32_t* accept_path, int max_path, int32_t* accept_len,
                int32_t* bonus, void* workspace, size_t workspace_bytes, int32_t* status,
                medusa_stream_t stream);

/*
 * GREEDY verification in its two launches, for callers that run the scan of
 * the target's rows while other work is still producing the node tokens
 * (the row scan reads only the target logits; the walk reads the node
 * tokens).  tree_verify_greedy_rows followed by tree_verify_greedy_walk on
 * the same workspace gives exactly tree_verify(MEDUSA_VERIFY_GREEDY, ...).
 * The caller orders the two (same stream, or an event) and must not reuse
 * the workspace in between.  Arguments as tree_verify; workspace:
 * tree_verify_workspace_size(MEDUSA_VERIFY_GREEDY, ...).  The walk writes
 * no status bits (greedy verification has no data-dependent errors).
 */
int tree_verify_greedy_rows(const void* target, medusa_dtype target_dt, int B, int V, const medusa_tree* tree,
                            void* workspace, size_t workspace_bytes, medusa_stream_t stream);
int tree_verify_greedy_walk(const int32_t* node_tokens, int B, int V, const medusa_tree* tree, int32_t* accept_path,
                            int max_path, int32_t* accept_len, int32_t* bonus, const void* workspace,
                            size_t workspace_bytes, medusa_stream_t stream);

/*
 * tree_verify_greedy_walk followed, in the same launch, by the commit of the
 * path it finds ("Multi-Token Prediction & Draft-Model-Free Speculative
 * Decoding", section "The 2D Tree Attention Mask": the longest accepted path
 * is committed; "Medusa Explained", "2. Single-Pass Tree Attention
 * Verification", step 4).  Gives exactly tree_verify_greedy_walk then
 * kv_commit (block_table NULL: contiguous cache [B, Hkv, S_max, D]) or
 * kv_commit_paged (block_table non-NULL: page pools [num_pages, Hkv,
 * page_size, D]; S_max ignored) with T = the tree's node count, in one
 * kernel per step instead of two dependent ones.  Walk arguments as
 * tree_verify_greedy_walk (after tree_verify_greedy_rows on the same
 * workspace); cache arguments as kv_commit / kv_commit_paged, including
 * their checks, status bits (CACHE_OVERFLOW, BAD_TOKEN) and in-place
 * new_prefix_len == prefix_len.  dt is the K/V dtype.
 */
int tree_verify_greedy_walk_commit(const int32_t* node_tokens, int B, int V, const medusa_tree* tree,
                                   int32_t* accept_path, int max_path, int32_t* accept_len, int32_t* bonus,
                                   const void* workspace, size_t workspace_bytes, void* k_cache, void* v_cache,
                                   const void* k_tree, const void* v_tree, const int32_t* prefix_len,
                                   int32_t* new_prefix_len, int Hkv, int D, int S_max, const int32_t* block_table,
                                   int max_pages, int page_size, int num_pages, medusa_dtype dt, int32_t* status,
                                   medusa_stream_t stream);

/*
 * STOCHASTIC verification reading the target's logits instead of its
 * probabilities: the walk of tree_verify (STOCHASTIC) with P, wherever the
 * walk reads the target's own row of node u, taken as
 *     m = max_y z(y),   e(y) = exp((z(y) - m) * (1/tau)),   Z = sum_y e(y),
 *     P(y) = e(y) * (1/Z)
 * in fp64 (z = logits[b,u,:] widened exactly; each product, difference and
 * quotient rounded once; 1/tau computed on the host).  The pages write
 * P_target without saying how it comes from the model's logits; tau = 1 is
 * the plain softmax, other tau the usual sampling temperature.  No
 * probability row is materialised: the maximum and Z of each visited row are
 * reduced over the sequence's thread-block cluster on entry.  The
 * exponentials and Z's summation order may differ from a sequential fp64
 * evaluation in the last bits of P; integer decisions differ only when a
 * value falls within that rounding of a boundary.
 *   logits [B, T, V], dtype logits_dt (MEDUSA_F32 or MEDUSA_BF16); NaN
 *   entries are skipped by the maximum and make the row's mass NaN (no
 *   acceptance; MEDUSA_STATUS_NO_MASS if the walk ends there), as does a row
 *   without a finite maximum.
 *   temperature: > 0 and finite, with 1/temperature finite, else
 *   MEDUSA_ERR_INVALID_ARG.
 * Every other argument, output and error as tree_verify in STOCHASTIC mode;
 * workspace: tree_verify_workspace_size(MEDUSA_VERIFY_STOCHASTIC, ...).
 */
int tree_verify_logits(const void* logits, medusa_dtype logits_dt, double temperature, const float* q, int q_rows,
                       const int32_t* q_row, const int32_t* node_tokens, int B, int V, const medusa_tree* tree,
                       uint64_t seed, uint32_t step, int32_t* accept_path, int max_path, int32_t* accept_len,
                       int32_t* bonus, void* workspace, size_t workspace_bytes, int32_t* status,
                       medusa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* KV commit                                                                 */
/* ------------------------------------------------------------------------ */

/*
 * [MTP] "The 2D Tree Attention Mask" (the engine commits the longest accepted
 * path) and "Production Deployment Guidelines" (unselected branches are
 * culled): for t < accept_len[b],
 *     cache[b, g, prefix_len[b] + t, :] = tree[b, accept_path[b,t], g, :]
 * for K and V and every kv-head g, bit for bit; then
 *     new_prefix_len[b] = prefix_len[b] + accept_len[b].
 * k_cache, v_cache [B, Hkv, S_max, D] (in place); k_tree, v_tree
 * [B, T, Hkv, D]; accept_path [B, max_path]; accept_len [B];
 * prefix_len [B] in; new_prefix_len [B] out (may alias prefix_len).
 * A sequence whose commit would pass S_max, or whose path holds an id
 * outside [0, T), is left untouched (new_prefix_len = prefix_len) and sets
 * MEDUSA_STATUS_CACHE_OVERFLOW or MEDUSA_STATUS_BAD_TOKEN.
 */
int kv_commit(void* k_cache, void* v_cache, const void* k_tree, const void* v_tree, const int32_t* accept_path,
              int max_path, const int32_t* accept_len, const int32_t* prefix_len, int32_t* new_prefix_len, int B,
              int T, int Hkv, int D, int S_max, medusa_dtype dt, int32_t* status, medusa_stream_t stream);

/*
 * The commit when the tree's K/V were appended to the cache before attention
 * (tree_attention_incache): the accepted path's rows are moved down to just
 * after the prefix, in place, in every layer's cache in one launch
 * ([MTP] "The 2D Tree Attention Mask": the longest accepted path is kept;
 * "Production Deployment Guidelines": the other branches are culled):
 *     cache_l[b, g, prefix_len[b] + t, :] = old cache_l[b, g, prefix_len[b] + accept_path[b,t], :]
 * for t < accept_len[b], every layer l < n_layers, K and V, every kv-head g,
 * bit for bit; then new_prefix_len[b] = prefix_len[b] + accept_len[b].
 * Rows past the new prefix keep whatever they held.
 * k_caches, v_caches: DEVICE arrays of n_layers pointers (16-byte aligned
 *   arrays), each a cache [B, Hkv, S_max, D] of dtype dt, 16-byte aligned,
 *   updated in place.
 * accept_path [B, max_path] int32 (strictly increasing node ids < T; the
 *   output of tree_verify); accept_len [B]; prefix_len [B];
 *   new_prefix_len [B] out, must not be prefix_len itself (other layers'
 *   CTAs still read prefix_len), else MEDUSA_ERR_INVALID_ARG.
 * A sequence whose path is not strictly increasing, holds a node id outside
 * [0, T) or has accept_len outside [0, max_path] is left untouched
 * (MEDUSA_STATUS_BAD_TOKEN); one whose rows would reach S_max
 * (prefix_len + accept_path[L-1] >= S_max) too (MEDUSA_STATUS_CACHE_OVERFLOW);
 * new_prefix_len = prefix_len for both.  A layer whose pointer is NULL or not
 * 16-byte aligned is skipped (MEDUSA_STATUS_BAD_LAYER).
 * Limits: 1 <= n_layers <= 65535; D * element size a multiple of 16 bytes;
 * T, max_path <= 128.
 */
int kv_compact(void* const* k_caches, void* const* v_caches, int n_layers, const int32_t* accept_path, int max_path,
               const int32_t* accept_len, const int32_t* prefix_len, int32_t* new_prefix_len, int B, int T, int Hkv,
               int D, int S_max, medusa_dtype dt, int32_t* status, medusa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Paged KV cache                                                            */
/* ------------------------------------------------------------------------ */

/*
 * [MTP] "Production Deployment Guidelines": tree attention runs inside
 * PagedAttention, the KV cache held in non-contiguous physical blocks.  The
 * caches of all sequences live in one pool of pages
 *     k_pages, v_pages [num_pages, Hkv, page_size, D]   dtype dt
 * and position s of sequence b is slot s % page_size of page
 *     block_table[b * max_pages + s / page_size]        int32, device
 * A call reads only the entries it needs: tree_attention_paged those of the
 * positions below prefix_len[b], kv_commit_paged those of the positions it
 * writes; the rest of the table may hold anything (-1, say).
 */

/*
 * tree_attention with the prefix read through the block table.  Arguments,
 * layouts, limits, tree handles and the workspace are those of
 * tree_attention (with tree_attention_paged_workspace_size); max_prefix = 0
 * means max_pages * page_size, and max_prefix may not exceed it.
 * page_size >= 1.  bf16 with page_size a multiple of 64 or one of 8, 16, 32
 * runs on the tensor-core kernel, other page sizes on the fallback kernel.
 * Slots at or past prefix_len[b] in the sequence's last page may hold
 * anything, NaN included: they are masked and never reach the output.
 * A needed table entry outside [0, num_pages) sets MEDUSA_STATUS_BAD_PAGE;
 * that page's keys are then skipped and the sequence's output is not
 * meaningful.
 */
size_t tree_attention_paged_workspace_size(int B, int Hq, int Hkv, int D, int max_prefix, int max_pages,
                                           int page_size, const medusa_tree* tree, medusa_dtype dt);
int tree_attention_paged(const void* q, const void* k_tree, const void* v_tree, const void* k_pages,
                         const void* v_pages, const int32_t* block_table, int max_pages, int page_size, int num_pages,
                         const int32_t* prefix_len, int B, int Hq, int Hkv, int D, int max_prefix, float scale,
                         medusa_dtype dt, const medusa_tree* tree, void* out, float* lse, void* workspace,
                         size_t workspace_bytes, int32_t* status, medusa_stream_t stream);

/*
 * kv_commit into the page pool: for t < accept_len[b], position
 * prefix_len[b] + t of sequence b receives tree[b, accept_path[b,t], g, :]
 * (K and V, every kv-head g, bit for bit); new_prefix_len[b] =
 * prefix_len[b] + accept_len[b].  A sequence whose new positions need a
 * block index >= max_pages or a table entry outside [0, num_pages) is left
 * untouched (new_prefix_len = prefix_len) and sets
 * MEDUSA_STATUS_CACHE_OVERFLOW; a path id outside [0, T) sets
 * MEDUSA_STATUS_BAD_TOKEN.  Other arguments as kv_commit.
 */
int kv_commit_paged(void* k_pages, void* v_pages, const void* k_tree, const void* v_tree, const int32_t* block_table,
                    int max_pages, int page_size, int num_pages, const int32_t* accept_path, int max_path,
                    const int32_t* accept_len, const int32_t* prefix_len, int32_t* new_prefix_len, int B, int T,
                    int Hkv, int D, medusa_dtype dt, int32_t* status, medusa_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MEDUSA_H */
