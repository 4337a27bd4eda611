// The commit of one sequence's accepted path, shared by the commit kernel
// and the greedy walk that commits as soon as it has found the path
// ("Multi-Token Prediction & Draft-Model-Free Speculative Decoding", sections
// "The 2D Tree Attention Mask" -- the longest accepted path is committed --
// and "Production Deployment Guidelines" -- unselected branches are culled,
// the cache may be paged).
#pragma once

#include "common.cuh"

namespace medusa {

// The commit of a path already in shared memory: cache row t (t < L) gets
// the K/V of tree node s_node[t] at position S + t of every kv-head, in a
// contiguous cache [B, Hkv, S_max, row] or, with a block table, a page pool
// [num_pages, Hkv, page_size, row].  Every check (path length, node ids,
// cache room or owned pages) is made before anything is written; a failed
// check sets a status bit and writes nothing but new_prefix_len = S.  S is
// the sequence's prefix length, read before anything is written (so
// new_prefix_len may alias prefix_len).  Whole block (blockDim.x >=
// MEDUSA_MAX_TREE threads), 16-byte copies.
static __device__ __noinline__ void commit_path(int b, const int* s_node, int L, int S, bool len_ok,
                                                uint8_t* __restrict__ kc, uint8_t* __restrict__ vc,
                                                const uint8_t* __restrict__ kt, const uint8_t* __restrict__ vt,
                                                int32_t* new_prefix_len, int T, int Hkv, int S_max, int row_bytes,
                                                const int32_t* __restrict__ table, int max_pages, int page_size,
                                                int num_pages, int32_t* status) {
    __shared__ int s_ok;
    __shared__ int s_page[MEDUSA_MAX_TREE];  // paged: the page of position S + t
    const int tid = threadIdx.x;
    len_ok = len_ok && L >= 0 && L <= MEDUSA_MAX_TREE && S >= 0;
    bool node_ok = true, page_ok = true;
    if (len_ok && tid < L) {  // every node id (and page) checked at once
        const int n = s_node[tid];
        node_ok = n >= 0 && n < T;
        if (table) {
            const int blk = (S + tid) / page_size;
            const int page = blk < max_pages ? table[(long)b * max_pages + blk] : -1;
            page_ok = page >= 0 && page < num_pages;
            s_page[tid] = page;
        }
    }
    const bool all_nodes_ok = __syncthreads_and(node_ok);
    const bool all_pages_ok = __syncthreads_and(page_ok);
    if (tid == 0) {
        int ok = 1;
        if (!len_ok || !all_nodes_ok) {
            ok = 0;
            set_status(status, MEDUSA_STATUS_BAD_TOKEN);
        } else if (table ? !all_pages_ok : S + L > S_max) {
            ok = 0;
            set_status(status, MEDUSA_STATUS_CACHE_OVERFLOW);
        }
        s_ok = ok;
    }
    __syncthreads();
    const bool ok = s_ok;
    if (ok) {
        // four rows' K and V loads in flight per thread before any store
        constexpr int kBatch = 4;
        const int vecs = row_bytes / 16;
        const int per_t = Hkv * vecs;
        const int total = L * per_t;
        for (int e0 = tid; e0 < total; e0 += kBatch * blockDim.x) {
            uint4 kr[kBatch], vr[kBatch];
            long dst[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int e = e0 + j * blockDim.x;
                if (e < total) {
                    const int t = e / per_t, rem = e % per_t;
                    const int g = rem / vecs, c = rem % vecs;
                    const long src = (((long)b * T + s_node[t]) * Hkv + g) * row_bytes + c * 16;
                    dst[j] = table ? (((long)s_page[t] * Hkv + g) * page_size + (S + t) % page_size) * row_bytes + c * 16
                                   : (((long)b * Hkv + g) * S_max + S + t) * row_bytes + c * 16;
                    kr[j] = *reinterpret_cast<const uint4*>(kt + src);
                    vr[j] = *reinterpret_cast<const uint4*>(vt + src);
                }
            }
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                if (e0 + j * blockDim.x < total) {
                    *reinterpret_cast<uint4*>(kc + dst[j]) = kr[j];
                    *reinterpret_cast<uint4*>(vc + dst[j]) = vr[j];
                }
            }
        }
    }
    if (tid == 0) new_prefix_len[b] = ok ? S + L : S;
}

// The commit of sequence b's path as kv_commit receives it: path [B,
// max_path] and len [B] in global memory (see commit_path).
static __device__ __noinline__ void commit_sequence(int b, uint8_t* __restrict__ kc, uint8_t* __restrict__ vc,
                                                    const uint8_t* __restrict__ kt, const uint8_t* __restrict__ vt,
                                                    const int32_t* path, int max_path, const int32_t* len,
                                                    const int32_t* prefix_len, int32_t* new_prefix_len, int T,
                                                    int Hkv, int S_max, int row_bytes,
                                                    const int32_t* __restrict__ table, int max_pages, int page_size,
                                                    int num_pages, int32_t* status) {
    __shared__ int s_node[MEDUSA_MAX_TREE];
    const int tid = threadIdx.x;
    const int S = prefix_len[b], L = len[b];
    const bool len_ok = L >= 0 && L <= max_path && L <= MEDUSA_MAX_TREE;
    if (len_ok && tid < L) s_node[tid] = path[(long)b * max_path + tid];
    __syncthreads();
    commit_path(b, s_node, L, S, len_ok, kc, vc, kt, vt, new_prefix_len, T, Hkv, S_max, row_bytes, table, max_pages,
                page_size, num_pages, status);
}

}  // namespace medusa
