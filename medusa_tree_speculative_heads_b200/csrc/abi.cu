// C ABI of libmedusa: argument validation, the candidate-tree handle,
// workspace queries and launches.  See include/medusa.h for the contract of
// every entry point.
#include <atomic>
#include <cmath>
#include <limits.h>
#include <stdarg.h>
#include <stddef.h>
#include <stdio.h>
#include <string.h>

#include <string>
#include <vector>

#include "kernels.h"

// One tree shared by every sequence, or one tree per sequence.  `host` holds
// the union's extremes (T = the largest tree's node count, the deepest depth,
// the most children); `trees` every tree as the kernels read it.
struct medusa_tree {
    medusa::TreeDev host;
    std::vector<medusa::TreeDev> trees;
    medusa::TreeDev* dev;
    int device;
    int ntrees() const { return (int)trees.size(); }
    medusa::TreeRef ref() const { return medusa::TreeRef{dev, ntrees() > 1 ? 1 : 0, host.T}; }
};

namespace medusa {

namespace {
thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int ok() {
    g_err.clear();
    return MEDUSA_OK;
}

bool al16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int cuda_fail(cudaError_t e, const char* what) {
    return fail(MEDUSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int check_tree(const medusa_tree* t, int B) {
    if (!t) return fail(MEDUSA_ERR_INVALID_ARG, "tree is NULL");
    int dev = -1;
    cudaGetDevice(&dev);
    if (dev != t->device)
        return fail(MEDUSA_ERR_INVALID_ARG, "tree was created on device %d, current device is %d", t->device, dev);
    if (t->ntrees() > 1 && t->ntrees() != B)
        return fail(MEDUSA_ERR_INVALID_ARG, "the handle holds %d per-sequence trees, the call has B=%d sequences",
                    t->ntrees(), B);
    return MEDUSA_OK;
}

// Validates one parent array and fills its device description.
int build_tree(const int32_t* parent, int T, TreeDev& h, const char* who) {
    if (T < 1) return fail(MEDUSA_ERR_INVALID_ARG, "%s: T = %d < 1", who, T);
    if (T > kMaxTree) return fail(MEDUSA_ERR_UNSUPPORTED, "%s: T = %d > %d", who, T, kMaxTree);
    if (parent[0] != -1) return fail(MEDUSA_ERR_INVALID_ARG, "%s: node 0 must be the root (parent -1)", who);
    for (int i = 1; i < T; ++i)
        if (parent[i] < 0 || parent[i] >= i)
            return fail(MEDUSA_ERR_INVALID_ARG,
                        "%s: parent[%d] = %d; need 0 <= parent[i] < i (one root, topological order)", who, i,
                        parent[i]);
    memset(&h, 0, sizeof h);
    h.T = T;
    int cnt[kMaxTree] = {0};
    h.parent[0] = -1;
    h.depth[0] = 1;
    h.anc[0][0] = 1u;
    h.max_depth = 1;
    for (int i = 1; i < T; ++i) {
        const int p = parent[i];
        h.parent[i] = (int16_t)p;
        h.depth[i] = (uint8_t)(h.depth[p] + 1);
        h.rank[i] = (uint8_t)cnt[p]++;
        for (int w = 0; w < 4; ++w) h.anc[i][w] = h.anc[p][w];
        h.anc[i][i >> 5] |= 1u << (i & 31);
        if (h.depth[i] > h.max_depth) h.max_depth = h.depth[i];
    }
    int off = 0;
    for (int u = 0; u < T; ++u) {
        h.child_off[u] = (uint8_t)off;
        off += cnt[u];
        if (cnt[u] > h.max_children) h.max_children = cnt[u];
    }
    h.child_off[T] = (uint8_t)off;
    int fill[kMaxTree] = {0};
    for (int c = 1; c < T; ++c) {
        const int p = parent[c];
        h.child_idx[h.child_off[p] + fill[p]++] = (uint8_t)c;
    }
    return MEDUSA_OK;
}

// Uploads the trees of a new handle.
int finish_tree(medusa_tree* t, medusa_tree** out, const char* who) {
    TreeDev& x = t->host;
    memset(&x, 0, sizeof x);
    for (const TreeDev& h : t->trees) {
        if (h.T > x.T) x.T = h.T;
        if (h.max_depth > x.max_depth) x.max_depth = h.max_depth;
        if (h.max_children > x.max_children) x.max_children = h.max_children;
    }
    cudaGetDevice(&t->device);
    t->dev = nullptr;
    const size_t bytes = sizeof(TreeDev) * t->trees.size();
    cudaError_t e = cudaMalloc((void**)&t->dev, bytes);
    if (e == cudaSuccess) e = cudaMemcpy(t->dev, t->trees.data(), bytes, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        if (t->dev) cudaFree(t->dev);
        delete t;
        return cuda_fail(e, who);
    }
    *out = t;
    return MEDUSA_OK;
}
}  // namespace

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// lets other translation units set this thread's last-error message
int report_error(int code, const char* msg) { return fail(code, "%s", msg); }

namespace {
std::atomic<uint64_t> g_wait_limit{0};  // 0: kWaitLimitNs
}  // namespace

namespace {
thread_local int g_heads_ctas = 0;        // 0: one CTA per SM
thread_local int g_attention_splits = 0;  // 0: chosen per call
}  // namespace

int launch_heads_ctas() { return g_heads_ctas; }
int launch_attention_splits() { return g_attention_splits; }

uint64_t wait_limit_ns() {
    const uint64_t v = g_wait_limit.load(std::memory_order_relaxed);
    return v ? v : kWaitLimitNs;
}

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!cache[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cache[dev] = n > 0 ? n : 1;
    }
    return cache[dev];
}

}  // namespace medusa

using namespace medusa;

extern "C" const char* medusa_last_error(void) { return g_err.c_str(); }

extern "C" int medusa_version(void) { return 100; }

extern "C" void medusa_debug_set_wait_limit(uint64_t ns) { g_wait_limit.store(ns, std::memory_order_relaxed); }

extern "C" int medusa_set_launch_shape(int heads_ctas, int attention_splits) {
    if (heads_ctas < 0 || attention_splits < 0)
        return fail(MEDUSA_ERR_INVALID_ARG, "medusa_set_launch_shape: negative value (%d, %d)", heads_ctas,
                    attention_splits);
    g_heads_ctas = heads_ctas;
    g_attention_splits = attention_splits;
    return ok();
}

// ---------------------------------------------------------------------------
// tree handle
// ---------------------------------------------------------------------------

extern "C" int medusa_tree_create(const int32_t* parent, int T, medusa_tree** out) {
    if (!parent || !out) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_tree_create: NULL argument");
    medusa_tree* t = new medusa_tree();
    t->trees.resize(1);
    int rc = build_tree(parent, T, t->trees[0], "medusa_tree_create");
    if (rc) {
        delete t;
        return rc;
    }
    rc = finish_tree(t, out, "medusa_tree_create");
    return rc ? rc : ok();
}

extern "C" int medusa_tree_create_ragged(const int32_t* parents, const int32_t* offsets, int ntrees,
                                         medusa_tree** out) {
    if (!parents || !offsets || !out) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_tree_create_ragged: NULL argument");
    if (ntrees < 1) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_tree_create_ragged: ntrees = %d < 1", ntrees);
    if (offsets[0] != 0) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_tree_create_ragged: offsets[0] must be 0");
    medusa_tree* t = new medusa_tree();
    t->trees.resize(ntrees);
    for (int i = 0; i < ntrees; ++i) {
        char who[64];
        snprintf(who, sizeof who, "medusa_tree_create_ragged (tree %d)", i);
        const int rc = build_tree(parents + offsets[i], offsets[i + 1] - offsets[i], t->trees[i], who);
        if (rc) {
            delete t;
            return rc;
        }
    }
    const int rc = finish_tree(t, out, "medusa_tree_create_ragged");
    return rc ? rc : ok();
}

extern "C" int medusa_tree_destroy(medusa_tree* t) {
    if (!t) return ok();
    cudaDeviceSynchronize();
    cudaError_t e = cudaFree(t->dev);
    delete t;
    if (e != cudaSuccess) return cuda_fail(e, "medusa_tree_destroy");
    return ok();
}

extern "C" int medusa_tree_info(const medusa_tree* t, int* T, int* max_depth, int* max_children) {
    if (!t) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_tree_info: tree is NULL");
    if (T) *T = t->host.T;
    if (max_depth) *max_depth = t->host.max_depth;
    if (max_children) *max_children = t->host.max_children;
    return ok();
}

extern "C" int medusa_tree_ntrees(const medusa_tree* t, int* ntrees, int32_t* T_each) {
    if (!t || !ntrees) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_tree_ntrees: NULL argument");
    *ntrees = t->ntrees();
    if (T_each)
        for (int i = 0; i < t->ntrees(); ++i) T_each[i] = t->trees[i].T;
    return ok();
}

// ---------------------------------------------------------------------------
// medusa_heads
// ---------------------------------------------------------------------------

extern "C" size_t medusa_heads_workspace_size(int B, int d, int V, int K, medusa_dtype dt) {
    if (B < 1 || d < 1 || V < 1 || K < 1) return 0;
    return heads_workspace_size(B, d, V, K, dt);
}

// the tree a heads call fills: depth <= K + 1, every sibling rank below
// min(V, 8), with root tokens and a node-token output
static int check_heads_tree(const char* fn, const medusa_tree* tree, int B, int V, int K, const int32_t* root_token,
                            const int32_t* node_tokens) {
    int rc = check_tree(tree, B);
    if (rc) return rc;
    if (!node_tokens || !root_token)
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: a tree needs root_token and node_tokens", fn);
    if (tree->host.max_depth > K + 1)
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: tree depth %d needs more than K=%d heads", fn, tree->host.max_depth,
                    K);
    const int smax = V < kTopK ? V : kTopK;
    for (int n = 0; n < tree->ntrees(); ++n) {
        const TreeDev& th = tree->trees[n];
        for (int i = 1; i < th.T; ++i)
            if (th.rank[i] >= smax)
                return fail(MEDUSA_ERR_UNSUPPORTED, "%s: node %d of tree %d has sibling rank %d >= %d", fn, i, n,
                            th.rank[i], smax);
    }
    return MEDUSA_OK;
}

extern "C" int medusa_heads(const void* h, const void* W_res, const void* W_head, int B, int d, int V, int K,
                            medusa_dtype dt, const medusa_tree* tree, const int32_t* root_token, int32_t* topk_idx,
                            float* topk_prob, int32_t* node_tokens, float* node_q, void* h_res_out,
                            float* logits_out, float* probs_out, void* workspace, size_t workspace_bytes,
                            int32_t* status, medusa_stream_t stream) {
    if (dt != MEDUSA_F32 && dt != MEDUSA_BF16) return fail(MEDUSA_ERR_UNSUPPORTED, "medusa_heads: unknown dtype");
    if (!h || !W_res || !W_head || !topk_idx || !topk_prob || !workspace)
        return fail(MEDUSA_ERR_INVALID_ARG, "medusa_heads: NULL tensor argument");
    if (B < 1 || d < 1 || V < 1 || K < 1 || K > 16 || d > 16384)
        return fail(MEDUSA_ERR_INVALID_ARG, "medusa_heads: bad sizes B=%d d=%d V=%d K=%d", B, d, V, K);
    const int vec = dt == MEDUSA_BF16 ? 8 : 4;
    if (d % vec) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_heads: d=%d must be a multiple of %d", d, vec);
    if (!al16(h) || !al16(W_res) || !al16(W_head) || !al16(h_res_out))
        return fail(MEDUSA_ERR_INVALID_ARG, "medusa_heads: h, W_res, W_head, h_res_out must be 16-byte aligned");
    if (workspace_bytes < heads_workspace_size(B, d, V, K, dt) || !al16(workspace))
        return fail(MEDUSA_ERR_WORKSPACE, "medusa_heads: workspace of %zu bytes, need %zu (16-byte aligned)",
                    workspace_bytes, heads_workspace_size(B, d, V, K, dt));
    int T = 0;
    if (tree) {
        int rc = check_heads_tree("medusa_heads", tree, B, V, K, root_token, node_tokens);
        if (rc) return rc;
        T = tree->host.T;
    }
    HeadsArgs a;
    a.h = h;
    a.W_res = W_res;
    a.W_head = W_head;
    a.B = B;
    a.d = d;
    a.V = V;
    a.K = K;
    a.dt = dt;
    a.tree = tree ? tree->ref() : TreeRef{nullptr, 0, 0};
    a.T = T;
    a.root_token = root_token;
    a.topk_idx = topk_idx;
    a.topk_prob = topk_prob;
    a.node_tokens = node_tokens;
    a.node_q = node_q;
    a.h_res_out = h_res_out;
    a.logits_out = logits_out;
    a.probs_out = probs_out;
    a.ws = workspace;
    a.ws_bytes = workspace_bytes;
    a.status = status;
    cudaError_t e = heads_launch(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "medusa_heads launch");
    return ok();
}

static_assert(sizeof(medusa_head_partial) == 72 && offsetof(medusa_head_partial, val) == 8 &&
                  offsetof(medusa_head_partial, idx) == 40,
              "medusa_head_partial must match the kernels' per-(sequence, head) partial");

extern "C" size_t medusa_heads_shard_workspace_size(int B, int d, int V_shard, int K, medusa_dtype dt) {
    if (B < 1 || d < 1 || V_shard < 1 || K < 1 || K > 16) return 0;
    return heads_shard_workspace_size(B, d, V_shard, K, dt);
}

extern "C" int medusa_heads_shard(const void* h, const void* W_res, const void* W_head_shard, int B, int d,
                                  int V_shard, int v_offset, int K, medusa_dtype dt, medusa_head_partial* partial_out,
                                  void* workspace, size_t workspace_bytes, int32_t* status, medusa_stream_t stream) {
    if (dt != MEDUSA_F32 && dt != MEDUSA_BF16) return fail(MEDUSA_ERR_UNSUPPORTED, "medusa_heads_shard: unknown dtype");
    if (!h || !W_res || !W_head_shard || !partial_out || !workspace)
        return fail(MEDUSA_ERR_INVALID_ARG, "medusa_heads_shard: NULL argument");
    if (B < 1 || d < 1 || V_shard < 1 || K < 1 || K > 16 || d > 16384 || v_offset < 0 ||
        (long long)v_offset + V_shard > INT_MAX)
        return fail(MEDUSA_ERR_INVALID_ARG, "medusa_heads_shard: bad sizes B=%d d=%d V_shard=%d v_offset=%d K=%d", B,
                    d, V_shard, v_offset, K);
    const int vec = dt == MEDUSA_BF16 ? 8 : 4;
    if (d % vec) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_heads_shard: d=%d must be a multiple of %d", d, vec);
    if (!al16(h) || !al16(W_res) || !al16(W_head_shard) || !al16(partial_out))
        return fail(MEDUSA_ERR_INVALID_ARG, "medusa_heads_shard: tensors must be 16-byte aligned");
    const size_t need = heads_shard_workspace_size(B, d, V_shard, K, dt);
    if (workspace_bytes < need || !al16(workspace))
        return fail(MEDUSA_ERR_WORKSPACE, "medusa_heads_shard: workspace of %zu bytes, need %zu (16-byte aligned)",
                    workspace_bytes, need);
    HeadsArgs a;
    memset(&a, 0, sizeof a);
    a.h = h;
    a.W_res = W_res;
    a.W_head = W_head_shard;
    a.B = B;
    a.d = d;
    a.V = V_shard;
    a.K = K;
    a.dt = dt;
    a.tree = TreeRef{nullptr, 0, 0};
    a.ws = workspace;
    a.ws_bytes = workspace_bytes;
    a.status = status;
    cudaError_t e = heads_shard_launch(a, v_offset, partial_out, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "medusa_heads_shard launch");
    return ok();
}

extern "C" int medusa_heads_merge(const medusa_head_partial* partials, int n_shards, int B, int K, int V,
                                  const medusa_tree* tree, const int32_t* root_token, int32_t* topk_idx,
                                  float* topk_prob, int32_t* node_tokens, float* node_q, int32_t* status,
                                  medusa_stream_t stream) {
    if (!partials || !topk_idx || !topk_prob) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_heads_merge: NULL argument");
    if (n_shards < 1 || B < 1 || K < 1 || K > 16 || V < 1 || (long long)B * K > 2147483647LL)
        return fail(MEDUSA_ERR_INVALID_ARG, "medusa_heads_merge: bad sizes n_shards=%d B=%d K=%d V=%d", n_shards, B, K,
                    V);
    if (!al16(partials)) return fail(MEDUSA_ERR_INVALID_ARG, "medusa_heads_merge: partials must be 16-byte aligned");
    if (tree) {
        int rc = check_heads_tree("medusa_heads_merge", tree, B, V, K, root_token, node_tokens);
        if (rc) return rc;
    }
    cudaError_t e = heads_merge_shards_launch(partials, n_shards, B, K, V, tree ? tree->ref() : TreeRef{nullptr, 0, 0},
                                              root_token, topk_idx, topk_prob, node_tokens, node_q, status,
                                              (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "medusa_heads_merge launch");
    return ok();
}

// ---------------------------------------------------------------------------
// tree_attention
// ---------------------------------------------------------------------------

extern "C" size_t tree_attention_workspace_size(int B, int Hq, int Hkv, int D, int S_max, int max_prefix,
                                                const medusa_tree* tree, medusa_dtype dt) {
    if (!tree || B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || (D != 64 && D != 128)) return 0;
    if (max_prefix <= 0) max_prefix = S_max;
    return attn_workspace_size(B, tree->host.T, Hq, Hkv, D, max_prefix, dt);
}

extern "C" size_t tree_attention_incache_workspace_size(int B, int Hq, int Hkv, int D, int S_max, int max_prefix,
                                                        const medusa_tree* tree, medusa_dtype dt) {
    if (!tree || B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || (D != 64 && D != 128)) return 0;
    if (max_prefix <= 0) max_prefix = S_max - tree->host.T;
    if (max_prefix < 0) return 0;
    return attn_workspace_size(B, tree->host.T, Hq, Hkv, D, max_prefix, dt);
}

// shared by tree_attention and tree_attention_incache (k_tree = v_tree = NULL:
// the tree's K/V are the cache rows that follow each prefix)
static int attention_common(const char* fn, const void* q, const void* k_tree, const void* v_tree,
                            const void* k_cache, const void* v_cache, const int32_t* prefix_len, int B, int Hq,
                            int Hkv, int D, int S_max, int max_prefix, float scale, medusa_dtype dt,
                            const medusa_tree* tree, void* out, float* lse, void* workspace, size_t workspace_bytes,
                            int32_t* status, medusa_stream_t stream) {
    const bool in_cache = k_tree == nullptr && v_tree == nullptr;
    if (dt != MEDUSA_F32 && dt != MEDUSA_BF16) return fail(MEDUSA_ERR_UNSUPPORTED, "%s: unknown dtype", fn);
    if (!q || (!in_cache && (!k_tree || !v_tree)) || !k_cache || !v_cache || !prefix_len || !out)
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: NULL tensor argument", fn);
    int rc = check_tree(tree, B);
    if (rc) return rc;
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || S_max < 0)
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: bad sizes B=%d Hq=%d Hkv=%d S_max=%d", fn, B, Hq, Hkv, S_max);
    if (D != 64 && D != 128) return fail(MEDUSA_ERR_UNSUPPORTED, "%s: head_dim %d (64 or 128)", fn, D);
    const int T = tree->host.T;
    if (max_prefix <= 0) max_prefix = in_cache ? S_max - T : S_max;
    if (max_prefix > S_max || (in_cache && max_prefix + T > S_max))
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: max_prefix %d%s > S_max %d", fn, max_prefix,
                    in_cache ? " + T" : "", S_max);
    if (max_prefix < 0) return fail(MEDUSA_ERR_INVALID_ARG, "%s: S_max %d below the tree's T %d", fn, S_max, T);
    if (!al16(q) || !al16(k_tree) || !al16(v_tree) || !al16(k_cache) || !al16(v_cache) || !al16(out))
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", fn);
    const size_t need = attn_workspace_size(B, T, Hq, Hkv, D, max_prefix, dt);
    if (need && (!workspace || workspace_bytes < need || !al16(workspace)))
        return fail(MEDUSA_ERR_WORKSPACE, "%s: workspace of %zu bytes, need %zu (16-byte aligned)", fn,
                    workspace_bytes, need);
    AttnArgs a;
    a.q = q;
    a.k_tree = k_tree;
    a.v_tree = v_tree;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.prefix_len = prefix_len;
    a.B = B;
    a.T = T;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.D = D;
    a.S_max = S_max;
    a.max_prefix = max_prefix;
    a.scale = scale;
    a.dt = dt;
    a.tree = tree->ref();
    a.block_table = nullptr;
    a.max_pages = a.page_size = a.num_pages = 0;
    a.out = out;
    a.lse = lse;
    a.ws = workspace;
    a.ws_bytes = workspace_bytes;
    a.status = status;
    cudaError_t e = attn_launch(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return ok();
}

extern "C" int tree_attention(const void* q, const void* k_tree, const void* v_tree, const void* k_cache,
                              const void* v_cache, const int32_t* prefix_len, int B, int Hq, int Hkv, int D,
                              int S_max, int max_prefix, float scale, medusa_dtype dt, const medusa_tree* tree,
                              void* out, float* lse, void* workspace, size_t workspace_bytes, int32_t* status,
                              medusa_stream_t stream) {
    if (!k_tree || !v_tree) return fail(MEDUSA_ERR_INVALID_ARG, "tree_attention: NULL tensor argument");
    return attention_common("tree_attention", q, k_tree, v_tree, k_cache, v_cache, prefix_len, B, Hq, Hkv, D, S_max,
                            max_prefix, scale, dt, tree, out, lse, workspace, workspace_bytes, status, stream);
}

extern "C" int tree_attention_incache(const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* prefix_len, int B, int Hq, int Hkv, int D, int S_max,
                                      int max_prefix, float scale, medusa_dtype dt, const medusa_tree* tree, void* out,
                                      float* lse, void* workspace, size_t workspace_bytes, int32_t* status,
                                      medusa_stream_t stream) {
    return attention_common("tree_attention_incache", q, nullptr, nullptr, k_cache, v_cache, prefix_len, B, Hq, Hkv,
                            D, S_max, max_prefix, scale, dt, tree, out, lse, workspace, workspace_bytes, status,
                            stream);
}

// ---------------------------------------------------------------------------
// tree_verify
// ---------------------------------------------------------------------------

extern "C" size_t tree_verify_workspace_size(medusa_verify_mode mode, int B, int V, const medusa_tree* tree) {
    if (!tree || B < 1 || V < 1) return 0;
    return verify_workspace_size(mode, B, V, tree->host.T);
}

// shared by tree_verify and tree_verify_logits: `fn` names the call in
// messages; logits selects the logits form of the stochastic walk
static int verify_common(const char* fn, medusa_verify_mode mode, const void* target, medusa_dtype target_dt,
                         bool logits, double temperature, const float* q, int q_rows, const int32_t* q_row,
                         const int32_t* node_tokens, int B, int V, const medusa_tree* tree, uint64_t seed,
                         uint32_t step, int32_t* accept_path, int max_path, int32_t* accept_len, int32_t* bonus,
                         void* workspace, size_t workspace_bytes, int32_t* status, medusa_stream_t stream) {
    if (mode != MEDUSA_VERIFY_GREEDY && mode != MEDUSA_VERIFY_STOCHASTIC)
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: unknown mode", fn);
    if (!target || !node_tokens || !accept_path || !accept_len || !bonus)
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: NULL tensor argument", fn);
    int rc = check_tree(tree, B);
    if (rc) return rc;
    const int T = tree->host.T;
    if (B < 1 || V < 1) return fail(MEDUSA_ERR_INVALID_ARG, "%s: bad sizes B=%d V=%d", fn, B, V);
    if (max_path < tree->host.max_depth || max_path > kMaxTree)
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: max_path %d outside [tree depth %d, %d]", fn, max_path,
                    tree->host.max_depth, kMaxTree);
    if (mode == MEDUSA_VERIFY_GREEDY || logits) {
        if (target_dt != MEDUSA_F32 && target_dt != MEDUSA_BF16)
            return fail(MEDUSA_ERR_UNSUPPORTED, "%s: logits dtype must be MEDUSA_F32 or MEDUSA_BF16", fn);
    } else if (target_dt != MEDUSA_F32) {
        return fail(MEDUSA_ERR_UNSUPPORTED, "%s: stochastic target p must be MEDUSA_F32", fn);
    }
    if (logits && !(temperature > 0.0 && std::isfinite(temperature) && std::isfinite(1.0 / temperature)))
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: temperature %g must be positive and finite", fn, temperature);
    if (mode == MEDUSA_VERIFY_STOCHASTIC) {
        if (!q) return fail(MEDUSA_ERR_INVALID_ARG, "%s: stochastic mode needs q", fn);
        if (q_rows < 1 || (!q_row && q_rows != T))
            return fail(MEDUSA_ERR_INVALID_ARG, "%s: q_rows=%d (must equal T=%d without q_row)", fn, q_rows, T);
    }
    const size_t need = verify_workspace_size(mode, B, V, T);
    if (need > 0 && (!workspace || workspace_bytes < need || !al16(workspace)))
        return fail(MEDUSA_ERR_WORKSPACE, "%s: workspace of %zu bytes, need %zu", fn, workspace_bytes, need);
    VerifyArgs a;
    a.mode = mode;
    a.target = target;
    a.target_dt = target_dt;
    a.q = q;
    a.q_rows = q_rows;
    a.q_row = q_row;
    a.node_tokens = node_tokens;
    a.B = B;
    a.V = V;
    a.T = T;
    a.tree = tree->ref();
    a.seed = seed;
    a.step = step;
    a.accept_path = accept_path;
    a.max_path = max_path;
    a.accept_len = accept_len;
    a.bonus = bonus;
    a.ws = workspace;
    a.ws_bytes = workspace_bytes;
    a.status = status;
    a.logits = logits;
    a.inv_tau = logits ? 1.0 / temperature : 1.0;
    cudaError_t e = verify_launch(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return ok();
}

extern "C" int tree_verify(medusa_verify_mode mode, const void* target, medusa_dtype target_dt, const float* q,
                           int q_rows, const int32_t* q_row, const int32_t* node_tokens, int B, int V,
                           const medusa_tree* tree, uint64_t seed, uint32_t step, int32_t* accept_path, int max_path,
                           int32_t* accept_len, int32_t* bonus, void* workspace, size_t workspace_bytes,
                           int32_t* status, medusa_stream_t stream) {
    return verify_common("tree_verify", mode, target, target_dt, false, 1.0, q, q_rows, q_row, node_tokens, B, V,
                         tree, seed, step, accept_path, max_path, accept_len, bonus, workspace, workspace_bytes,
                         status, stream);
}

extern "C" int tree_verify_greedy_rows(const void* target, medusa_dtype target_dt, int B, int V,
                                       const medusa_tree* tree, void* workspace, size_t workspace_bytes,
                                       medusa_stream_t stream) {
    if (!target) return fail(MEDUSA_ERR_INVALID_ARG, "tree_verify_greedy_rows: NULL target");
    if (target_dt != MEDUSA_F32 && target_dt != MEDUSA_BF16)
        return fail(MEDUSA_ERR_UNSUPPORTED, "tree_verify_greedy_rows: logits dtype must be MEDUSA_F32 or MEDUSA_BF16");
    int rc = check_tree(tree, B);
    if (rc) return rc;
    if (B < 1 || V < 1) return fail(MEDUSA_ERR_INVALID_ARG, "tree_verify_greedy_rows: bad sizes B=%d V=%d", B, V);
    const size_t need = verify_workspace_size(MEDUSA_VERIFY_GREEDY, B, V, tree->host.T);
    if (!workspace || workspace_bytes < need || !al16(workspace))
        return fail(MEDUSA_ERR_WORKSPACE, "tree_verify_greedy_rows: workspace of %zu bytes, need %zu",
                    workspace_bytes, need);
    VerifyArgs a;
    memset(&a, 0, sizeof a);
    a.mode = MEDUSA_VERIFY_GREEDY;
    a.target = target;
    a.target_dt = target_dt;
    a.B = B;
    a.V = V;
    a.T = tree->host.T;
    a.tree = tree->ref();
    a.ws = workspace;
    a.ws_bytes = workspace_bytes;
    cudaError_t e = verify_greedy_rows_launch(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "tree_verify_greedy_rows");
    return ok();
}

extern "C" int tree_verify_greedy_walk(const int32_t* node_tokens, int B, int V, const medusa_tree* tree,
                                       int32_t* accept_path, int max_path, int32_t* accept_len, int32_t* bonus,
                                       const void* workspace, size_t workspace_bytes, medusa_stream_t stream) {
    if (!node_tokens || !accept_path || !accept_len || !bonus)
        return fail(MEDUSA_ERR_INVALID_ARG, "tree_verify_greedy_walk: NULL tensor argument");
    int rc = check_tree(tree, B);
    if (rc) return rc;
    if (B < 1 || V < 1) return fail(MEDUSA_ERR_INVALID_ARG, "tree_verify_greedy_walk: bad sizes B=%d V=%d", B, V);
    if (max_path < tree->host.max_depth || max_path > kMaxTree)
        return fail(MEDUSA_ERR_INVALID_ARG, "tree_verify_greedy_walk: max_path %d outside [tree depth %d, %d]",
                    max_path, tree->host.max_depth, kMaxTree);
    const size_t need = verify_workspace_size(MEDUSA_VERIFY_GREEDY, B, V, tree->host.T);
    if (!workspace || workspace_bytes < need || !al16(workspace))
        return fail(MEDUSA_ERR_WORKSPACE, "tree_verify_greedy_walk: workspace of %zu bytes, need %zu",
                    workspace_bytes, need);
    VerifyArgs a;
    memset(&a, 0, sizeof a);
    a.mode = MEDUSA_VERIFY_GREEDY;
    a.node_tokens = node_tokens;
    a.B = B;
    a.V = V;
    a.T = tree->host.T;
    a.tree = tree->ref();
    a.accept_path = accept_path;
    a.max_path = max_path;
    a.accept_len = accept_len;
    a.bonus = bonus;
    a.ws = const_cast<void*>(workspace);
    a.ws_bytes = workspace_bytes;
    cudaError_t e = verify_greedy_walk_launch(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "tree_verify_greedy_walk");
    return ok();
}

extern "C" int tree_verify_greedy_walk_commit(const int32_t* node_tokens, int B, int V, const medusa_tree* tree,
                                              int32_t* accept_path, int max_path, int32_t* accept_len,
                                              int32_t* bonus, const void* workspace, size_t workspace_bytes,
                                              void* k_cache, void* v_cache, const void* k_tree, const void* v_tree,
                                              const int32_t* prefix_len, int32_t* new_prefix_len, int Hkv, int D,
                                              int S_max, const int32_t* block_table, int max_pages, int page_size,
                                              int num_pages, medusa_dtype dt, int32_t* status,
                                              medusa_stream_t stream) {
    const char* fn = "tree_verify_greedy_walk_commit";
    if (!node_tokens || !accept_path || !accept_len || !bonus)
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: NULL verification argument", fn);
    if (!k_cache || !v_cache || !k_tree || !v_tree || !prefix_len || !new_prefix_len)
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: NULL cache argument", fn);
    if (dt != MEDUSA_F32 && dt != MEDUSA_BF16) return fail(MEDUSA_ERR_UNSUPPORTED, "%s: unknown dtype", fn);
    int rc = check_tree(tree, B);
    if (rc) return rc;
    const int T = tree->host.T;
    if (B < 1 || V < 1 || Hkv < 1 || D < 1)
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: bad sizes B=%d V=%d Hkv=%d D=%d", fn, B, V, Hkv, D);
    if (max_path < tree->host.max_depth || max_path > kMaxTree)
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: max_path %d outside [tree depth %d, %d]", fn, max_path,
                    tree->host.max_depth, kMaxTree);
    if (block_table ? (max_pages < 1 || page_size < 1 || num_pages < 1) : S_max < 0)
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: bad cache sizes S_max=%d max_pages=%d page_size=%d num_pages=%d", fn,
                    S_max, max_pages, page_size, num_pages);
    const int esize = dt == MEDUSA_BF16 ? 2 : 4;
    if ((D * esize) % 16)
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: a K/V row (%d bytes) must be a multiple of 16 bytes", fn, D * esize);
    if (!al16(k_cache) || !al16(v_cache) || !al16(k_tree) || !al16(v_tree))
        return fail(MEDUSA_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", fn);
    const size_t need = verify_workspace_size(MEDUSA_VERIFY_GREEDY, B, V, T);
    if (!workspace || workspace_bytes < need || !al16(workspace))
        return fail(MEDUSA_ERR_WORKSPACE, "%s: workspace of %zu bytes, need %zu", fn, workspace_bytes, need);
    VerifyArgs a;
    memset(&a, 0, sizeof a);
    a.mode = MEDUSA_VERIFY_GREEDY;
    a.node_tokens = node_tokens;
    a.B = B;
    a.V = V;
    a.T = T;
    a.tree = tree->ref();
    a.accept_path = accept_path;
    a.max_path = max_path;
    a.accept_len = accept_len;
    a.bonus = bonus;
    a.ws = const_cast<void*>(workspace);
    a.ws_bytes = workspace_bytes;
    CommitArgs c;
    memset(&c, 0, sizeof c);
    c.k_cache = k_cache;
    c.v_cache = v_cache;
    c.k_tree = k_tree;
    c.v_tree = v_tree;
    c.accept_path = accept_path;
    c.max_path = max_path;
    c.accept_len = accept_len;
    c.prefix_len = prefix_len;
    c.new_prefix_len = new_prefix_len;
    c.B = B;
    c.T = T;
    c.Hkv = Hkv;
    c.D = D;
    c.S_max = block_table ? 0 : S_max;
    c.esize = esize;
    c.block_table = block_table;
    c.max_pages = block_table ? max_pages : 0;
    c.page_size = block_table ? page_size : 0;
    c.num_pages = block_table ? num_pages : 0;
    c.status = status;
    cudaError_t e = verify_greedy_walk_commit_launch(a, c, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return ok();
}

extern "C" int tree_verify_logits(const void* logits, medusa_dtype logits_dt, double temperature, const float* q,
                                  int q_rows, const int32_t* q_row, const int32_t* node_tokens, int B, int V,
                                  const medusa_tree* tree, uint64_t seed, uint32_t step, int32_t* accept_path,
                                  int max_path, int32_t* accept_len, int32_t* bonus, void* workspace,
                                  size_t workspace_bytes, int32_t* status, medusa_stream_t stream) {
    return verify_common("tree_verify_logits", MEDUSA_VERIFY_STOCHASTIC, logits, logits_dt, true, temperature, q,
                         q_rows, q_row, node_tokens, B, V, tree, seed, step, accept_path, max_path, accept_len, bonus,
                         workspace, workspace_bytes, status, stream);
}

// ---------------------------------------------------------------------------
// kv_commit
// ---------------------------------------------------------------------------

extern "C" int kv_commit(void* k_cache, void* v_cache, const void* k_tree, const void* v_tree,
                         const int32_t* accept_path, int max_path, const int32_t* accept_len,
                         const int32_t* prefix_len, int32_t* new_prefix_len, int B, int T, int Hkv, int D, int S_max,
                         medusa_dtype dt, int32_t* status, medusa_stream_t stream) {
    if (dt != MEDUSA_F32 && dt != MEDUSA_BF16) return fail(MEDUSA_ERR_UNSUPPORTED, "kv_commit: unknown dtype");
    if (!k_cache || !v_cache || !k_tree || !v_tree || !accept_path || !accept_len || !prefix_len || !new_prefix_len)
        return fail(MEDUSA_ERR_INVALID_ARG, "kv_commit: NULL tensor argument");
    const int esize = dt == MEDUSA_BF16 ? 2 : 4;
    if (B < 1 || T < 1 || T > kMaxTree || Hkv < 1 || D < 1 || S_max < 0 || max_path < 1 || max_path > kMaxTree)
        return fail(MEDUSA_ERR_INVALID_ARG, "kv_commit: bad sizes B=%d T=%d Hkv=%d D=%d S_max=%d max_path=%d", B, T,
                    Hkv, D, S_max, max_path);
    if ((D * esize) % 16)
        return fail(MEDUSA_ERR_INVALID_ARG, "kv_commit: a K/V row (%d bytes) must be a multiple of 16 bytes",
                    D * esize);
    if (!al16(k_cache) || !al16(v_cache) || !al16(k_tree) || !al16(v_tree))
        return fail(MEDUSA_ERR_INVALID_ARG, "kv_commit: tensors must be 16-byte aligned");
    CommitArgs a;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.k_tree = k_tree;
    a.v_tree = v_tree;
    a.accept_path = accept_path;
    a.max_path = max_path;
    a.accept_len = accept_len;
    a.prefix_len = prefix_len;
    a.new_prefix_len = new_prefix_len;
    a.B = B;
    a.T = T;
    a.Hkv = Hkv;
    a.D = D;
    a.S_max = S_max;
    a.esize = esize;
    a.block_table = nullptr;
    a.max_pages = a.page_size = a.num_pages = 0;
    a.status = status;
    cudaError_t e = commit_launch(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "kv_commit launch");
    return ok();
}

extern "C" int kv_compact(void* const* k_caches, void* const* v_caches, int n_layers, const int32_t* accept_path,
                          int max_path, const int32_t* accept_len, const int32_t* prefix_len, int32_t* new_prefix_len,
                          int B, int T, int Hkv, int D, int S_max, medusa_dtype dt, int32_t* status,
                          medusa_stream_t stream) {
    if (dt != MEDUSA_F32 && dt != MEDUSA_BF16) return fail(MEDUSA_ERR_UNSUPPORTED, "kv_compact: unknown dtype");
    if (!k_caches || !v_caches || !accept_path || !accept_len || !prefix_len || !new_prefix_len)
        return fail(MEDUSA_ERR_INVALID_ARG, "kv_compact: NULL argument");
    if (new_prefix_len == prefix_len)
        return fail(MEDUSA_ERR_INVALID_ARG, "kv_compact: new_prefix_len must not alias prefix_len");
    const int esize = dt == MEDUSA_BF16 ? 2 : 4;
    if (n_layers < 1 || n_layers > 65535 || B < 1 || T < 1 || T > kMaxTree || Hkv < 1 || D < 1 || S_max < 0 ||
        max_path < 1 || max_path > kMaxTree)
        return fail(MEDUSA_ERR_INVALID_ARG,
                    "kv_compact: bad sizes n_layers=%d B=%d T=%d Hkv=%d D=%d S_max=%d max_path=%d", n_layers, B, T,
                    Hkv, D, S_max, max_path);
    if ((D * esize) % 16)
        return fail(MEDUSA_ERR_INVALID_ARG, "kv_compact: a K/V row (%d bytes) must be a multiple of 16 bytes",
                    D * esize);
    if (!al16(k_caches) || !al16(v_caches))
        return fail(MEDUSA_ERR_INVALID_ARG, "kv_compact: the pointer arrays must be 16-byte aligned");
    CompactArgs a;
    a.k_caches = k_caches;
    a.v_caches = v_caches;
    a.n_layers = n_layers;
    a.accept_path = accept_path;
    a.max_path = max_path;
    a.accept_len = accept_len;
    a.prefix_len = prefix_len;
    a.new_prefix_len = new_prefix_len;
    a.B = B;
    a.T = T;
    a.Hkv = Hkv;
    a.D = D;
    a.S_max = S_max;
    a.esize = esize;
    a.status = status;
    cudaError_t e = compact_launch(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "kv_compact launch");
    return ok();
}

// ---------------------------------------------------------------------------
// paged KV cache
// ---------------------------------------------------------------------------

extern "C" size_t tree_attention_paged_workspace_size(int B, int Hq, int Hkv, int D, int max_prefix, int max_pages,
                                                      int page_size, const medusa_tree* tree, medusa_dtype dt) {
    if (!tree || B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || (D != 64 && D != 128) || max_pages < 1 || page_size < 1)
        return 0;
    if (max_prefix <= 0) max_prefix = max_pages * page_size;
    return attn_workspace_size(B, tree->host.T, Hq, Hkv, D, max_prefix, dt);
}

extern "C" int tree_attention_paged(const void* q, const void* k_tree, const void* v_tree, const void* k_pages,
                                    const void* v_pages, const int32_t* block_table, int max_pages, int page_size,
                                    int num_pages, const int32_t* prefix_len, int B, int Hq, int Hkv, int D,
                                    int max_prefix, float scale, medusa_dtype dt, const medusa_tree* tree, void* out,
                                    float* lse, void* workspace, size_t workspace_bytes, int32_t* status,
                                    medusa_stream_t stream) {
    if (dt != MEDUSA_F32 && dt != MEDUSA_BF16)
        return fail(MEDUSA_ERR_UNSUPPORTED, "tree_attention_paged: unknown dtype");
    if (!q || !k_tree || !v_tree || !k_pages || !v_pages || !block_table || !prefix_len || !out)
        return fail(MEDUSA_ERR_INVALID_ARG, "tree_attention_paged: NULL tensor argument");
    int rc = check_tree(tree, B);
    if (rc) return rc;
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || max_pages < 1 || page_size < 1 || num_pages < 1 ||
        (long)max_pages * page_size > (1L << 30))
        return fail(MEDUSA_ERR_INVALID_ARG,
                    "tree_attention_paged: bad sizes B=%d Hq=%d Hkv=%d max_pages=%d page_size=%d num_pages=%d", B, Hq,
                    Hkv, max_pages, page_size, num_pages);
    if (D != 64 && D != 128) return fail(MEDUSA_ERR_UNSUPPORTED, "tree_attention_paged: head_dim %d (64 or 128)", D);
    const int cap = max_pages * page_size;
    if (max_prefix <= 0) max_prefix = cap;
    if (max_prefix > cap)
        return fail(MEDUSA_ERR_INVALID_ARG, "tree_attention_paged: max_prefix %d > max_pages * page_size = %d",
                    max_prefix, cap);
    if (!al16(q) || !al16(k_tree) || !al16(v_tree) || !al16(k_pages) || !al16(v_pages) || !al16(out))
        return fail(MEDUSA_ERR_INVALID_ARG, "tree_attention_paged: tensors must be 16-byte aligned");
    const size_t need = attn_workspace_size(B, tree->host.T, Hq, Hkv, D, max_prefix, dt);
    if (need && (!workspace || workspace_bytes < need || !al16(workspace)))
        return fail(MEDUSA_ERR_WORKSPACE, "tree_attention_paged: workspace of %zu bytes, need %zu (16-byte aligned)",
                    workspace_bytes, need);
    AttnArgs a;
    a.q = q;
    a.k_tree = k_tree;
    a.v_tree = v_tree;
    a.k_cache = k_pages;
    a.v_cache = v_pages;
    a.prefix_len = prefix_len;
    a.B = B;
    a.T = tree->host.T;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.D = D;
    a.S_max = cap;
    a.max_prefix = max_prefix;
    a.scale = scale;
    a.dt = dt;
    a.tree = tree->ref();
    a.block_table = block_table;
    a.max_pages = max_pages;
    a.page_size = page_size;
    a.num_pages = num_pages;
    a.out = out;
    a.lse = lse;
    a.ws = workspace;
    a.ws_bytes = workspace_bytes;
    a.status = status;
    cudaError_t e = attn_launch(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "tree_attention_paged launch");
    return ok();
}

extern "C" int kv_commit_paged(void* k_pages, void* v_pages, const void* k_tree, const void* v_tree,
                               const int32_t* block_table, int max_pages, int page_size, int num_pages,
                               const int32_t* accept_path, int max_path, const int32_t* accept_len,
                               const int32_t* prefix_len, int32_t* new_prefix_len, int B, int T, int Hkv, int D,
                               medusa_dtype dt, int32_t* status, medusa_stream_t stream) {
    if (dt != MEDUSA_F32 && dt != MEDUSA_BF16) return fail(MEDUSA_ERR_UNSUPPORTED, "kv_commit_paged: unknown dtype");
    if (!k_pages || !v_pages || !k_tree || !v_tree || !block_table || !accept_path || !accept_len || !prefix_len ||
        !new_prefix_len)
        return fail(MEDUSA_ERR_INVALID_ARG, "kv_commit_paged: NULL tensor argument");
    const int esize = dt == MEDUSA_BF16 ? 2 : 4;
    if (B < 1 || T < 1 || T > kMaxTree || Hkv < 1 || D < 1 || max_path < 1 || max_path > kMaxTree ||
        max_pages < 1 || page_size < 1 || num_pages < 1)
        return fail(MEDUSA_ERR_INVALID_ARG,
                    "kv_commit_paged: bad sizes B=%d T=%d Hkv=%d D=%d max_path=%d max_pages=%d page_size=%d "
                    "num_pages=%d", B, T, Hkv, D, max_path, max_pages, page_size, num_pages);
    if ((D * esize) % 16)
        return fail(MEDUSA_ERR_INVALID_ARG, "kv_commit_paged: a K/V row (%d bytes) must be a multiple of 16 bytes",
                    D * esize);
    if (!al16(k_pages) || !al16(v_pages) || !al16(k_tree) || !al16(v_tree))
        return fail(MEDUSA_ERR_INVALID_ARG, "kv_commit_paged: tensors must be 16-byte aligned");
    CommitArgs a;
    a.k_cache = k_pages;
    a.v_cache = v_pages;
    a.k_tree = k_tree;
    a.v_tree = v_tree;
    a.accept_path = accept_path;
    a.max_path = max_path;
    a.accept_len = accept_len;
    a.prefix_len = prefix_len;
    a.new_prefix_len = new_prefix_len;
    a.B = B;
    a.T = T;
    a.Hkv = Hkv;
    a.D = D;
    a.S_max = 0;
    a.esize = esize;
    a.block_table = block_table;
    a.max_pages = max_pages;
    a.page_size = page_size;
    a.num_pages = num_pages;
    a.status = status;
    cudaError_t e = commit_launch(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "kv_commit_paged launch");
    return ok();
}
