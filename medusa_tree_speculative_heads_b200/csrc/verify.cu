// Tree verification on B200.
//
// Greedy ("Medusa Explained: Multi-Head Speculative Decoding Guide", section
// "2. Single-Pass Tree Attention Verification", steps 2-4; "Multi-Token
// Prediction & Draft-Model-Free Speculative Decoding", section "The 2D Tree
// Attention Mask": longest accepted path plus a bonus token): every node's
// target prediction is a row argmax over the vocabulary; the row scans are
// spread over many CTAs (the HBM-bound part), then one warp per sequence
// walks the tree.
//
// Stochastic ("Speculative Decoding & Medusa Tree Attention", section 2:
// accept with probability min(1, P_target/P_draft), else resample from
// normalize(max(0, P_target - P_draft))): one CTA per sequence walks the tree;
// every vocabulary pass is a block-wide exact integer reduction, and the
// current distribution after j rejections is recomputed element-wise from the
// j residual sums, so no V-sized scratch is needed.  All decisions use
// integer or correctly rounded fp64 operations (explicit _rn intrinsics, no
// contraction), so results are bit-reproducible.
#include <limits.h>

#include "kernels.h"

namespace medusa {

namespace {

constexpr int kArgmaxThreads = 256;
constexpr int kStochThreads = 512;

// ------------------------------- greedy ------------------------------------

__device__ __forceinline__ void argmax_merge(float& bv, int& bi, float v, int i) {
    if (beats(v, i, bv, bi)) {
        bv = v;
        bi = i;
    }
}

// Row argmax partials over vocabulary chunks, one block per (row, chunk),
// 8 independent 16-byte loads in flight per thread.
template <typename E>
__global__ void __launch_bounds__(kArgmaxThreads, 4) row_argmax_kernel(const E* __restrict__ x, int V, int splits,
                                                                    int chunk, float* __restrict__ pval,
                                                                    int* __restrict__ pidx) {
    constexpr int VEC = Elt<E>::kVec;
    constexpr int NW = kArgmaxThreads / 32;
    constexpr int U = 8;
    const long row = blockIdx.x;
    const int s = blockIdx.y;
    const int v0 = s * chunk;
    const int v1 = min(V, v0 + chunk);
    const E* rp = x + row * (long)V;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float bv = -INFINITY;
    int bi = v0;  // lowest index of the chunk: the answer when nothing beats -inf
    if (v0 < v1) {
        int va = v0;
        if ((((uintptr_t)(rp + v0)) & 15) == 0) {
            const int nvec = (v1 - v0) / VEC;
            for (int c0 = threadIdx.x; c0 < nvec; c0 += U * kArgmaxThreads) {
                uint4 raw[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + u * kArgmaxThreads;
                    raw[u] = c < nvec ? ld_stream(rp + v0 + (long)c * VEC) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + u * kArgmaxThreads;
                    if (c < nvec) {
                        float f[VEC];
                        Elt<E>::unpack(raw[u], f);
#pragma unroll
                        for (int e = 0; e < VEC; ++e) argmax_merge(bv, bi, f[e], v0 + c * VEC + e);
                    }
                }
            }
            va = v0 + nvec * VEC;
        }
        for (int v = va + threadIdx.x; v < v1; v += kArgmaxThreads) argmax_merge(bv, bi, Elt<E>::to_float(rp[v]), v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(kFull, bv, o);
        const int oi = __shfl_xor_sync(kFull, bi, o);
        argmax_merge(bv, bi, ov, oi);
    }
    __shared__ float sv[NW];
    __shared__ int si[NW];
    if (lane == 0) {
        sv[warp] = bv;
        si[warp] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < NW; ++w) argmax_merge(bv, bi, sv[w], si[w]);
        pval[row * splits + s] = bv;
        pidx[row * splits + s] = bi;
    }
}

// One block of 128 threads per sequence, one thread per node: node u's
// prediction is the merge of its partials (split order); node c "matches"
// when its token equals its parent's prediction (the root always does).  A
// node is accepted iff every node on its root path matches, i.e. iff its
// ancestor bitmask has no bit outside the match mask.  The deepest accepted
// node (lowest index among equally deep ones) ends the path, whose nodes are
// the set bits of its ancestor mask in increasing index order (a parent's
// index is below its child's).
constexpr int kWalkThreads = kMaxTree;
constexpr int kMaxSplits = 16;
__global__ void __launch_bounds__(kWalkThreads) greedy_walk_kernel(const float* __restrict__ pval,
                                                                   const int* __restrict__ pidx, int splits,
                                                                   const int32_t* __restrict__ node_tokens,
                                                                   const TreeDev* __restrict__ tree,
                                                                   int32_t* accept_path, int max_path,
                                                                   int32_t* accept_len, int32_t* bonus) {
    __shared__ int pred[kMaxTree];
    __shared__ uint32_t match[kMaxTree / 32];
    __shared__ int best_key[kMaxTree / 32];
    const int b = blockIdx.x, u = threadIdx.x, lane = u & 31, w = u >> 5;
    const int T = tree->T;
    float bv = -INFINITY;
    int bi = INT_MAX;
    int tok = 0, par = -1, dep = 0;
    if (u < T) {
        const long base = ((long)b * T + u) * splits;
        float lv[kMaxSplits];
        int li[kMaxSplits];
#pragma unroll
        for (int s = 0; s < kMaxSplits; ++s) {  // every load issued before any is used
            lv[s] = s < splits ? pval[base + s] : -INFINITY;
            li[s] = s < splits ? pidx[base + s] : INT_MAX;
        }
        tok = node_tokens[(long)b * T + u];
        par = tree->parent[u];
        dep = tree->depth[u];
#pragma unroll
        for (int s = 0; s < kMaxSplits; ++s) argmax_merge(bv, bi, lv[s], li[s]);
        pred[u] = bi;
    }
    __syncthreads();
    const bool m = u < T && (u == 0 || tok == pred[par]);
    const uint32_t mb = __ballot_sync(kFull, m);
    if (lane == 0) match[w] = mb;
    __syncthreads();
    bool accepted = false;
    if (u < T) {
        accepted = true;
#pragma unroll
        for (int k = 0; k < kMaxTree / 32; ++k) accepted &= (tree->anc[u][k] & ~match[k]) == 0u;
    }
    // deepest accepted node, lowest index among equally deep: maximise depth*256 + (255 - index)
    int key = accepted ? dep * 256 + (255 - u) : -1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) key = max(key, __shfl_xor_sync(kFull, key, o));
    if (lane == 0) best_key[w] = key;
    __syncthreads();
    if (u == 0) {
        int k = best_key[0];
        for (int i = 1; i < kMaxTree / 32; ++i) k = max(k, best_key[i]);
        const int best = 255 - (k & 255);
        const int L = k >> 8;
        int t = 0;
        for (int j = 0; j <= best; ++j)
            if ((tree->anc[best][j >> 5] >> (j & 31)) & 1u) accept_path[(long)b * max_path + t++] = j;
        for (int j = L; j < max_path; ++j) accept_path[(long)b * max_path + j] = -1;
        accept_len[b] = L;
        bonus[b] = pred[best];
    }
}

// ----------------------------- stochastic ----------------------------------

// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): ten rounds of the
// two-multiplier S-box with the Weyl key schedule.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
        const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c;
}

// P after n rejections at the current node, for one vocabulary entry: each
// step is W = floor(max(0, P - Q) * 2^32), P = W / S_j (P kept when S_j = 0).
__device__ __forceinline__ double residual_chain(double P, double Q, const unsigned long long* S_hist, int n) {
    for (int j = 0; j < n; ++j) {
        const double diff = __dsub_rn(P, Q);
        const unsigned long long W = diff > 0.0 ? (unsigned long long)floor(__dmul_rn(diff, 4294967296.0)) : 0ull;
        const unsigned long long S = S_hist[j];
        if (S > 0) P = __ddiv_rn((double)W, (double)S);
    }
    return P;
}

__device__ __forceinline__ unsigned long long block_sum_u64(unsigned long long x, unsigned long long* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = x;
    __syncthreads();
    unsigned long long t = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    return t;
}

__global__ void __launch_bounds__(kStochThreads) verify_stochastic_kernel(
    const float* __restrict__ p, const float* __restrict__ q, int q_rows, const int32_t* __restrict__ q_row,
    const int32_t* __restrict__ node_tokens, int V, const TreeDev* __restrict__ tree, uint32_t key0, uint32_t key1,
    uint32_t step, int32_t* accept_path, int max_path, int32_t* accept_len, int32_t* bonus, int32_t* status) {
    __shared__ unsigned long long S_hist[kMaxTree];
    __shared__ unsigned long long red[kStochThreads / 32];
    __shared__ int s_flag, s_found;
    const int b = blockIdx.x, tid = threadIdx.x;
    const int T = tree->T;
    const float* Pb = p + (long)b * T * V;
    int u = 0, L = 1;
    if (tid == 0) {
        accept_path[(long)b * max_path] = 0;
        for (int t = 1; t < max_path; ++t) accept_path[(long)b * max_path + t] = -1;
    }
    int nrej = 0;
    const float* Qrow = nullptr;
    for (;;) {
        const int c_begin = tree->child_off[u], c_end = tree->child_off[u + 1];
        nrej = 0;
        if (c_begin == c_end) break;  // a leaf: no drafted children
        const int qr = q_row ? q_row[u] : u;
        if (qr < 0 || qr >= q_rows) {
            if (tid == 0) set_status(status, MEDUSA_STATUS_BAD_TOKEN);
            break;
        }
        Qrow = q + ((long)b * q_rows + qr) * V;
        const float* Prow = Pb + (long)u * V;
        bool moved = false;
        for (int ci = c_begin; ci < c_end; ++ci) {
            const int c = tree->child_idx[ci];
            const int x = node_tokens[(long)b * T + c];
            if (x < 0 || x >= V) {
                if (tid == 0) set_status(status, MEDUSA_STATUS_BAD_TOKEN);
                continue;
            }
            if (tid == 0) {
                const uint4 r = philox4x32_10(make_uint4((uint32_t)b, (uint32_t)c, step, 0u), key0, key1);
                const double uc = (double)(r.x >> 8) * (1.0 / 16777216.0);
                const double Qx = (double)Qrow[x];
                const double Px = residual_chain((double)Prow[x], Qx, S_hist, nrej);
                s_flag = __dmul_rn(uc, Qx) < Px;
            }
            __syncthreads();
            const bool acc = s_flag;
            __syncthreads();
            if (acc) {
                u = c;
                if (tid == 0) accept_path[(long)b * max_path + L] = c;
                ++L;
                moved = true;
                break;
            }
            // rejected: residual sum at this node
            unsigned long long part = 0;
            for (int y = tid; y < V; y += kStochThreads) {
                const double Qy = (double)Qrow[y];
                const double P = residual_chain((double)Prow[y], Qy, S_hist, nrej);
                const double diff = __dsub_rn(P, Qy);
                part += diff > 0.0 ? (unsigned long long)floor(__dmul_rn(diff, 4294967296.0)) : 0ull;
            }
            const unsigned long long S = block_sum_u64(part, red);
            if (tid == 0) S_hist[nrej] = S;
            __syncthreads();
            ++nrej;
        }
        if (!moved) break;
    }
    // bonus from the current distribution P (p[b,u,:] after nrej residual steps)
    const float* Prow = Pb + (long)u * V;
    unsigned long long part = 0;
    for (int y = tid; y < V; y += kStochThreads) {
        const double P = nrej ? residual_chain((double)Prow[y], (double)Qrow[y], S_hist, nrej) : (double)Prow[y];
        part += P > 0.0 ? (unsigned long long)floor(__dmul_rn(P, 4294967296.0)) : 0ull;
    }
    const unsigned long long S = block_sum_u64(part, red);
    const uint4 r = philox4x32_10(make_uint4((uint32_t)b, (uint32_t)u, step, 0u), key0, key1);
    // t = floor(U * S / 2^32) from the exact 128-bit product
    const unsigned long long lo = (unsigned long long)r.y * (S & 0xffffffffull);
    const unsigned long long hi = (unsigned long long)r.y * (S >> 32);
    const unsigned long long t = (lo >> 32) + hi;
    if (tid == 0) s_found = -1;
    __syncthreads();
    int tok = 0;
    if (S == 0) {
        if (tid == 0) set_status(status, MEDUSA_STATUS_NO_MASS);
    } else {
        // inverse CDF: smallest y with inclusive prefix sum > t, block by block
        unsigned long long run = 0;
        const int warp = tid >> 5, lane = tid & 31;
        __shared__ unsigned long long wsum[kStochThreads / 32];
        for (int y0 = 0; y0 < V; y0 += kStochThreads) {
            const int y = y0 + tid;
            unsigned long long w = 0;
            if (y < V) {
                const double P =
                    nrej ? residual_chain((double)Prow[y], (double)Qrow[y], S_hist, nrej) : (double)Prow[y];
                w = P > 0.0 ? (unsigned long long)floor(__dmul_rn(P, 4294967296.0)) : 0ull;
            }
            unsigned long long inc = w;  // inclusive scan within the warp
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                unsigned long long n = __shfl_up_sync(kFull, inc, o);
                if (lane >= o) inc += n;
            }
            if (lane == 31) wsum[warp] = inc;
            __syncthreads();
            unsigned long long before = run;
            for (int w2 = 0; w2 < warp; ++w2) before += wsum[w2];
            unsigned long long total = run;
            for (int w2 = 0; w2 < kStochThreads / 32; ++w2) total += wsum[w2];
            const unsigned long long incl = before + inc;
            if (y < V && w > 0 && incl > t && incl - w <= t) s_found = y;  // exactly one such y
            __syncthreads();
            if (s_found >= 0) break;
            run = total;
        }
        tok = s_found >= 0 ? s_found : 0;
    }
    if (tid == 0) {
        accept_len[b] = L;
        bonus[b] = tok;
    }
}

int argmax_splits(int rows, int V) {
    int target = 4 * num_sms();  // four 256-thread blocks per SM: one balanced wave
    int s = (target + rows / 2) / rows;
    int max_s = (V + 2047) / 2048;
    if (s > max_s) s = max_s;
    if (s > kMaxSplits) s = kMaxSplits;
    if (s < 1) s = 1;
    return s;
}

}  // namespace

size_t verify_workspace_size(medusa_verify_mode mode, int B, int V, int T) {
    if (mode != MEDUSA_VERIFY_GREEDY) return 0;
    int s = argmax_splits(B * T, V);
    return align256((size_t)B * T * s * sizeof(float)) + align256((size_t)B * T * s * sizeof(int));
}

cudaError_t verify_launch(const VerifyArgs& a, cudaStream_t st) {
    if (a.mode == MEDUSA_VERIFY_GREEDY) {
        const int rows = a.B * a.T;
        const int splits = argmax_splits(rows, a.V);
        int chunk = (a.V + splits - 1) / splits;
        chunk = (chunk + 7) / 8 * 8;
        float* pval = (float*)a.ws;
        int* pidx = (int*)((char*)a.ws + align256((size_t)rows * splits * sizeof(float)));
        dim3 grid(rows, splits);
        if (a.target_dt == MEDUSA_BF16)
            row_argmax_kernel<__nv_bfloat16>
                <<<grid, kArgmaxThreads, 0, st>>>((const __nv_bfloat16*)a.target, a.V, splits, chunk, pval, pidx);
        else
            row_argmax_kernel<float><<<grid, kArgmaxThreads, 0, st>>>((const float*)a.target, a.V, splits, chunk,
                                                                      pval, pidx);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        greedy_walk_kernel<<<a.B, kWalkThreads, 0, st>>>(pval, pidx, splits, a.node_tokens, a.tree, a.accept_path,
                                                         a.max_path, a.accept_len, a.bonus);
        return cudaGetLastError();
    }
    verify_stochastic_kernel<<<a.B, kStochThreads, 0, st>>>(
        (const float*)a.target, a.q, a.q_rows, a.q_row, a.node_tokens, a.V, a.tree, (uint32_t)a.seed,
        (uint32_t)(a.seed >> 32), a.step, a.accept_path, a.max_path, a.accept_len, a.bonus, a.status);
    return cudaGetLastError();
}

}  // namespace medusa
