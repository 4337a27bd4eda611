// Internal launch interface between the C ABI (abi.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace medusa {

// ------------------------------- heads -------------------------------------
struct HeadsArgs {
    const void* h;
    const void* W_res;
    const void* W_head;
    int B, d, V, K;
    medusa_dtype dt;
    TreeRef tree;  // base NULL: no tree
    int T;
    const int32_t* root_token;
    int32_t* topk_idx;
    float* topk_prob;
    int32_t* node_tokens;
    float* node_q;
    void* h_res_out;
    float* logits_out;
    float* probs_out;
    void* ws;
    size_t ws_bytes;
    int32_t* status;
};
size_t heads_workspace_size(int B, int d, int V, int K, medusa_dtype dt);
cudaError_t heads_launch(const HeadsArgs& a, cudaStream_t st);
// vocabulary shard: the heads over rows [v_offset, v_offset + V) of the full
// vocabulary, reduced to one partial (m, l, top-8 logits, global ids) per
// (sequence, head) in partial_out [B*K] (layout of medusa_head_partial)
size_t heads_shard_workspace_size(int B, int d, int V_shard, int K, medusa_dtype dt);
cudaError_t heads_shard_launch(const HeadsArgs& a, int v_offset, void* partial_out, cudaStream_t st);
// merge of n_shards partial sets [n_shards][B][K] into the heads' outputs
cudaError_t heads_merge_shards_launch(const void* parts, int n_shards, int B, int K, int V_total, TreeRef tree,
                                      const int32_t* root_token, int32_t* topk_idx, float* topk_prob,
                                      int32_t* node_tokens, float* node_q, int32_t* status, cudaStream_t st);
// tensor-core path (bf16, 1 <= B <= 64, d % 8 == 0)
bool heads_tc_supported(int B, int d, medusa_dtype dt);
// ctr: 2 + 2 * num_sms() + K counters (zeroed here); slots: 2 * num_sms() * B * 128 floats
cudaError_t heads_tc_launch(const HeadsArgs& a, void* hk, void* part, unsigned int* ctr, float* slots, float2* stats,
                            float* logits, cudaStream_t st);

// ------------------------------ attention ----------------------------------
struct AttnArgs {
    const void* q;
    const void* k_tree;
    const void* v_tree;
    const void* k_cache;
    const void* v_cache;
    const int32_t* prefix_len;
    int B, T, Hq, Hkv, D, S_max, max_prefix;
    float scale;
    medusa_dtype dt;
    TreeRef tree;  // T is tree.T
    const int32_t* block_table;  // NULL: contiguous caches [B, Hkv, S_max, D]; else page pools
    int max_pages, page_size, num_pages;
    void* out;
    float* lse;
    void* ws;
    size_t ws_bytes;
    int32_t* status;
};
size_t attn_workspace_size(int B, int T, int Hq, int Hkv, int D, int max_prefix, medusa_dtype dt);
cudaError_t attn_launch(const AttnArgs& a, cudaStream_t st);
// tensor-core split kernel (bf16, D in {64,128}, power-of-two group size <= 16)
bool attn_tc_supported(int Hq, int Hkv, int D, int T, medusa_dtype dt);
int attn_tc_ctas_per_sm();
// page sizes the tensor-core kernel reads (multiples of 64, or 8, 16, 32)
bool attn_tc_page_ok(int page_size);
// key splits per 128-row tile (the CTAs of one cluster, at most 8)
int attn_tc_splits(int B, int T, int Hq, int Hkv, int max_prefix);
// writes the output (and lse) itself: the splits merge inside their cluster
cudaError_t attn_tc_launch(const AttnArgs& a, int m_tiles, int n_splits, float scale_log2, cudaStream_t st);

// ------------------------------- verify ------------------------------------
struct VerifyArgs {
    medusa_verify_mode mode;
    const void* target;
    medusa_dtype target_dt;
    const float* q;
    int q_rows;
    const int32_t* q_row;
    const int32_t* node_tokens;
    int B, V, T;
    TreeRef tree;
    uint64_t seed;
    uint32_t step;
    int32_t* accept_path;
    int max_path;
    int32_t* accept_len;
    int32_t* bonus;
    void* ws;
    size_t ws_bytes;
    int32_t* status;
    bool logits;     // stochastic: target holds logits (target_dt f32/bf16), P = softmax((z - max z) * inv_tau)
    double inv_tau;  // 1 / temperature
};
size_t verify_workspace_size(medusa_verify_mode mode, int B, int V, int T);
cudaError_t verify_launch(const VerifyArgs& a, cudaStream_t st);
// greedy mode's two launches on their own (verify_launch = rows then walk)
cudaError_t verify_greedy_rows_launch(const VerifyArgs& a, cudaStream_t st);
cudaError_t verify_greedy_walk_launch(const VerifyArgs& a, cudaStream_t st);

// ------------------------------- commit ------------------------------------
struct CommitArgs {
    void* k_cache;
    void* v_cache;
    const void* k_tree;
    const void* v_tree;
    const int32_t* accept_path;
    int max_path;
    const int32_t* accept_len;
    const int32_t* prefix_len;
    int32_t* new_prefix_len;
    int B, T, Hkv, D, S_max, esize;
    const int32_t* block_table;  // NULL: contiguous cache [B, Hkv, S_max, D]
    int max_pages, page_size, num_pages;
    int32_t* status;
};
cudaError_t commit_launch(const CommitArgs& a, cudaStream_t st);
// greedy verification's walk (VerifyArgs as for verify_greedy_walk_launch)
// followed, in the same block per sequence, by the commit of the path it found
// (CommitArgs as for commit_launch; its path, length and T come from the walk)
cudaError_t verify_greedy_walk_commit_launch(const VerifyArgs& a, const CommitArgs& c, cudaStream_t st);

// in-place compaction of the tree rows after each prefix, every layer at once
struct CompactArgs {
    void* const* k_caches;  // device array [n_layers] of caches [B, Hkv, S_max, D]
    void* const* v_caches;
    int n_layers;
    const int32_t* accept_path;
    int max_path;
    const int32_t* accept_len;
    const int32_t* prefix_len;
    int32_t* new_prefix_len;
    int B, T, Hkv, D, S_max, esize;
    int32_t* status;
};
cudaError_t compact_launch(const CompactArgs& a, cudaStream_t st);

// limit of the pipeline waits (hand-overs, phases, grid barriers) that the
// heads and tree attention kernels are given: kWaitLimitNs unless changed by
// medusa_debug_set_wait_limit; drains of issued copies and MMAs always wait
// the full kWaitLimitNs
uint64_t wait_limit_ns();

// launch shape set by medusa_set_launch_shape on the calling thread: the
// heads kernel's largest CTA count (0: one per SM) and the attention
// kernel's largest number of key splits (0: chosen per call)
int launch_heads_ctas();
int launch_attention_splits();

// device properties, cached per device
int num_sms();
size_t align256(size_t x);

}  // namespace medusa
