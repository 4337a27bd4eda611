// KV commit on B200 ("Multi-Token Prediction & Draft-Model-Free Speculative
// Decoding", sections "The 2D Tree Attention Mask" -- the longest accepted
// path is committed -- and "Production Deployment Guidelines" -- unselected
// branches are culled): the accepted path's K/V rows are appended to each
// sequence's cache after its prefix, either a contiguous cache or a page pool
// read through a block table ("Production Deployment Guidelines": tree
// attention inside PagedAttention).  One CTA per sequence; 16-byte copies.
// With the tree's K/V already in the cache after the prefix (appended before
// attention), the commit of every layer is one in-place compaction launch.
#include "commit_common.cuh"
#include "kernels.h"

namespace medusa {

namespace {

__global__ void __launch_bounds__(256) kv_commit_kernel(uint8_t* __restrict__ kc, uint8_t* __restrict__ vc,
                                                        const uint8_t* __restrict__ kt, const uint8_t* __restrict__ vt,
                                                        const int32_t* __restrict__ path, int max_path,
                                                        const int32_t* __restrict__ len, const int32_t* prefix_len,
                                                        int32_t* new_prefix_len, int T, int Hkv, int S_max,
                                                        int row_bytes, const int32_t* __restrict__ table,
                                                        int max_pages, int page_size, int num_pages, int32_t* status) {
    commit_sequence(blockIdx.x, kc, vc, kt, vt, path, max_path, len, prefix_len, new_prefix_len, T, Hkv, S_max,
                    row_bytes, table, max_pages, page_size, num_pages, status);
}

// In-place compaction of the tree rows that follow each prefix, in every
// layer's cache at once: row S + t <- row S + path[t] for t < L.  A path is
// strictly increasing, so path[t] >= t, and a row is only overwritten after
// every read of it: the rows a batch of steps reads lie at or past its first
// destination row and past every earlier destination.  Each thread owns one
// 16-byte column of one (layer, sequence, kv-head) block and moves it in
// batches of kBatch rows, all loads of a batch before its stores.
constexpr int kBatch = 8;
__global__ void __launch_bounds__(128) kv_compact_kernel(uint8_t* const* __restrict__ kcs, uint8_t* const* __restrict__ vcs,
                                                         const int32_t* __restrict__ path, int max_path,
                                                         const int32_t* __restrict__ len,
                                                         const int32_t* __restrict__ prefix_len,
                                                         int32_t* __restrict__ new_prefix_len, int T, int Hkv,
                                                         int S_max, int row_bytes, int32_t* status) {
    __shared__ int s_node[MEDUSA_MAX_TREE];
    __shared__ int s_ok;
    const int b = blockIdx.x, layer = blockIdx.y, tid = threadIdx.x;
    const int S = prefix_len[b], L = len[b];
    const bool len_ok = L >= 0 && L <= max_path && L <= MEDUSA_MAX_TREE && S >= 0;
    bool node_ok = true;
    if (len_ok)
        for (int t = tid; t < L; t += blockDim.x) {
            const int n = path[(long)b * max_path + t];
            const int prev = t > 0 ? path[(long)b * max_path + t - 1] : -1;
            node_ok &= n > prev && n < T;  // strictly increasing node ids below T
            s_node[t] = n;
        }
    const bool all_ok = __syncthreads_and(node_ok);
    if (tid == 0) {
        int ok = 1;
        if (!len_ok || !all_ok) {
            ok = 0;
            if (layer == 0) set_status(status, MEDUSA_STATUS_BAD_TOKEN);
        } else if (L > 0 && (long)S + s_node[L - 1] >= S_max) {
            ok = 0;
            if (layer == 0) set_status(status, MEDUSA_STATUS_CACHE_OVERFLOW);
        }
        s_ok = ok;
    }
    __syncthreads();
    uint8_t* kc = kcs[layer];
    uint8_t* vc = vcs[layer];
    const bool layer_ok = kc && vc && ((((uintptr_t)kc) | ((uintptr_t)vc)) & 15u) == 0;
    if (!layer_ok && tid == 0 && b == 0) set_status(status, MEDUSA_STATUS_BAD_LAYER);
    if (s_ok && layer_ok) {
        const int vecs = row_bytes / 16;
        for (int col = tid; col < Hkv * vecs; col += blockDim.x) {
            const int g = col / vecs, c = col % vecs;
            const long base = (((long)b * Hkv + g) * S_max + S) * row_bytes + c * 16;
            for (int t0 = 0; t0 < L; t0 += kBatch) {
                uint4 kr[kBatch], vr[kBatch];
#pragma unroll
                for (int i = 0; i < kBatch; ++i)
                    if (t0 + i < L) {
                        const long src = base + (long)s_node[t0 + i] * row_bytes;
                        kr[i] = *reinterpret_cast<const uint4*>(kc + src);
                        vr[i] = *reinterpret_cast<const uint4*>(vc + src);
                    }
#pragma unroll
                for (int i = 0; i < kBatch; ++i)
                    if (t0 + i < L) {
                        const long dst = base + (long)(t0 + i) * row_bytes;
                        *reinterpret_cast<uint4*>(kc + dst) = kr[i];
                        *reinterpret_cast<uint4*>(vc + dst) = vr[i];
                    }
            }
        }
    }
    if (tid == 0 && layer == 0) new_prefix_len[b] = s_ok ? S + L : S;
}

}  // namespace

cudaError_t compact_launch(const CompactArgs& a, cudaStream_t st) {
    const dim3 grid(a.B, a.n_layers);
    prefer_max_smem(kv_compact_kernel);
    kv_compact_kernel<<<grid, 128, 0, st>>>((uint8_t* const*)a.k_caches, (uint8_t* const*)a.v_caches, a.accept_path,
                                            a.max_path, a.accept_len, a.prefix_len, a.new_prefix_len, a.T, a.Hkv,
                                            a.S_max, a.D * a.esize, a.status);
    return cudaGetLastError();
}

cudaError_t commit_launch(const CommitArgs& a, cudaStream_t st) {
    prefer_max_smem(kv_commit_kernel);
    kv_commit_kernel<<<a.B, 256, 0, st>>>((uint8_t*)a.k_cache, (uint8_t*)a.v_cache, (const uint8_t*)a.k_tree,
                                          (const uint8_t*)a.v_tree, a.accept_path, a.max_path, a.accept_len,
                                          a.prefix_len, a.new_prefix_len, a.T, a.Hkv, a.S_max, a.D * a.esize,
                                          a.block_table, a.max_pages, a.page_size, a.num_pages, a.status);
    return cudaGetLastError();
}

}  // namespace medusa
