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
// normalize(max(0, P_target - P_draft))): one thread-block cluster per
// sequence walks the tree, each CTA of the cluster owning a contiguous share
// of the vocabulary and each warp a contiguous segment of that share (its
// lanes read consecutive entries).  The
// current distribution is kept in workspace as the last effective residual's
// integer weights W and their sum S (P = W / S), so a rejection costs one
// pass over the vocabulary whatever the number of earlier rejections; sums
// are exact 64-bit integer reductions over the cluster (shared memory of the
// peer CTAs).  All decisions use integer or correctly rounded fp64
// operations (explicit _rn intrinsics, no contraction), so results are
// bit-reproducible and independent of the cluster size.
//
// The stochastic walk can also read the target's logits z instead of its
// probabilities: on entering a node the cluster takes the row maximum m and
// Z = sum exp((z - m) / tau) (fp64, fixed reduction order: lanes, warps,
// CTAs in rank order), and P(y) = exp((z(y) - m) / tau) / Z is evaluated
// wherever the walk reads P, so no probability row is ever materialised.
// The fp64 exponentials and Z's summation order (which follows the cluster
// size) differ from a sequential evaluation only in the last bits of P.
#include <cooperative_groups.h>
#include <limits.h>
#include <string.h>

#include "commit_common.cuh"
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
// 8 independent 16-byte loads in flight per thread.  A thread visits its
// vectors in increasing index order and keeps the first vector whose maximum
// beats everything before it (the vector maximum is a paired max, a few
// instructions per eight logits instead of a compare-and-select per logit);
// the winning element is the vector's first one equal to that maximum, so
// ties go to the lowest index and NaN never wins, as in `beats`.
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
            int bc = -1;      // the thread's winning vector
            uint4 braw = make_uint4(0, 0, 0, 0);
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
                    const float mv = Elt<E>::vmax(raw[u]);
                    if (c < nvec && mv > bv) {
                        bv = mv;
                        bc = c;
                        braw = raw[u];
                    }
                }
            }
            if (bc >= 0) {
                float f[VEC];
                Elt<E>::unpack(braw, f);
                int e = 0;
#pragma unroll
                for (int i = VEC - 1; i >= 0; --i)
                    if (f[i] == bv) e = i;
                bi = v0 + bc * VEC + e;
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

// The same scan with the chunk staged in shared memory by the bulk-copy
// engine: one thread issues the chunk's copies (four pieces, each completing
// on its own mbarrier) as soon as the block starts, so the whole chunk is in
// flight at once; the threads reduce each piece as it lands.  With four
// blocks per SM the staged chunks (up to kStageBytes each) hold a whole
// wave's share of the rows: one DRAM round trip instead of two.
constexpr int kStageBytes = 52 * 1024;
constexpr int kStagePieces = 4;
template <typename E>
__global__ void __launch_bounds__(kArgmaxThreads, 4) row_argmax_staged_kernel(const E* __restrict__ x, int V, int splits,
                                                                           int chunk, float* __restrict__ pval,
                                                                           int* __restrict__ pidx, int32_t* status) {
    constexpr int VEC = Elt<E>::kVec;
    constexpr int NW = kArgmaxThreads / 32;
    extern __shared__ __align__(16) uint8_t sbuf[];
    __shared__ uint64_t bars[kStagePieces];
    const long row = blockIdx.x;
    const int s = blockIdx.y;
    const int v0 = s * chunk;
    const int v1 = min(V, v0 + chunk);
    const E* rp = x + row * (long)V;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nvec = v1 > v0 ? (v1 - v0) / VEC : 0;  // the row starts on a 16-byte boundary (checked by the host)
    if (threadIdx.x == 0) {
        for (int p = 0; p < kStagePieces; ++p) mbar_init(&bars[p], 1);
        mbar_fence_init();
        for (int p = 0; p < kStagePieces; ++p) {
            const int vb = nvec * p / kStagePieces, ve = nvec * (p + 1) / kStagePieces;
            const uint32_t bytes = (uint32_t)(ve - vb) * 16u;
            mbar_arrive_expect_tx(&bars[p], bytes);
            if (bytes) bulk_g2s(sbuf + (size_t)vb * 16, rp + v0 + (long)vb * VEC, bytes, &bars[p]);
        }
    }
    __syncthreads();  // the barriers are initialised before anyone waits on them
    float bv = -INFINITY;
    int bi = v0;  // lowest index of the chunk: the answer when nothing beats -inf
    int bc = -1;  // the thread's winning vector
    uint4 braw = make_uint4(0, 0, 0, 0);
    bool ok = true;
    for (int p = 0; p < kStagePieces; ++p) {
        const int vb = nvec * p / kStagePieces, ve = nvec * (p + 1) / kStagePieces;
        if (ok && !mbar_wait(&bars[p], 0)) {
            ok = false;
            set_status(status, MEDUSA_STATUS_TIMEOUT);
        }
        if (!ok) continue;
        // this thread's vectors of the piece, in increasing index order
        int c = vb + (int)(((unsigned)(threadIdx.x - vb)) % kArgmaxThreads);
        for (; c < ve; c += kArgmaxThreads) {
            const uint4 raw = *reinterpret_cast<const uint4*>(sbuf + (size_t)c * 16);
            const float mv = Elt<E>::vmax(raw);
            if (mv > bv) {
                bv = mv;
                bc = c;
                braw = raw;
            }
        }
    }
    if (!ok)  // the copies still in flight land before the block exits
        for (int p = 0; p < kStagePieces; ++p) mbar_wait(&bars[p], 0);
    if (bc >= 0) {
        float f[VEC];
        Elt<E>::unpack(braw, f);
        int e = 0;
#pragma unroll
        for (int i = VEC - 1; i >= 0; --i)
            if (f[i] == bv) e = i;
        bi = v0 + bc * VEC + e;
    }
    for (int v = v0 + nvec * VEC + threadIdx.x; v < v1; v += kArgmaxThreads) argmax_merge(bv, bi, Elt<E>::to_float(rp[v]), v);
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
// With a commit (kc != NULL) the same block then appends the accepted path's
// K/V to the sequence's cache, as kv_commit does.
struct WalkCommit {
    uint8_t* kc;  // NULL: no commit
    uint8_t* vc;
    const uint8_t* kt;
    const uint8_t* vt;
    const int32_t* prefix_len;
    int32_t* new_prefix_len;
    int Hkv, S_max, row_bytes;
    const int32_t* table;  // NULL: contiguous cache
    int max_pages, page_size, num_pages;
    int32_t* status;
};
constexpr int kWalkThreads = kMaxTree;
constexpr int kMaxSplits = 16;
__global__ void __launch_bounds__(kWalkThreads) greedy_walk_kernel(const float* __restrict__ pval,
                                                                   const int* __restrict__ pidx, int splits,
                                                                   const int32_t* __restrict__ node_tokens,
                                                                   TreeRef trees, int32_t* accept_path, int max_path,
                                                                   int32_t* accept_len, int32_t* bonus,
                                                                   const WalkCommit cm) {
    __shared__ int pred[kMaxTree];
    __shared__ uint32_t match[kMaxTree / 32];
    __shared__ int best_key[kMaxTree / 32];
    __shared__ uint32_t s_anc_best[kMaxTree / 32];
    __shared__ int s_path[kMaxTree];
    const int b = blockIdx.x, u = threadIdx.x, lane = u & 31, w = u >> 5;
    const TreeDev* tree = trees.at(b);
    const int T = tree->T, Tn = trees.T;  // this sequence's nodes; node stride of the arrays
    // every input is loaded up front, the commit's prefix length included
    const int S_commit = cm.kc ? cm.prefix_len[b] : 0;
    float bv = -INFINITY;
    int bi = INT_MAX;
    int tok = 0, par = -1, dep = 0;
    uint32_t anc[kMaxTree / 32] = {0u, 0u, 0u, 0u};
    if (u < T) {
        const long base = ((long)b * Tn + u) * splits;
        float lv[kMaxSplits];
        int li[kMaxSplits];
#pragma unroll
        for (int s = 0; s < kMaxSplits; ++s) {  // every load issued before any is used
            lv[s] = s < splits ? pval[base + s] : -INFINITY;
            li[s] = s < splits ? pidx[base + s] : INT_MAX;
        }
        tok = node_tokens[(long)b * Tn + u];
        par = tree->parent[u];
        dep = tree->depth[u];
#pragma unroll
        for (int k = 0; k < kMaxTree / 32; ++k) anc[k] = tree->anc[u][k];
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
        for (int k = 0; k < kMaxTree / 32; ++k) accepted &= (anc[k] & ~match[k]) == 0u;
    }
    // deepest accepted node, lowest index among equally deep: maximise depth*256 + (255 - index)
    int key = accepted ? dep * 256 + (255 - u) : -1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) key = max(key, __shfl_xor_sync(kFull, key, o));
    if (lane == 0) best_key[w] = key;
    __syncthreads();
    int k = best_key[0];
#pragma unroll
    for (int i = 1; i < kMaxTree / 32; ++i) k = max(k, best_key[i]);
    const int best = 255 - (k & 255);
    const int L = k >> 8;
    if (u == best) {
#pragma unroll
        for (int i = 0; i < kMaxTree / 32; ++i) s_anc_best[i] = anc[i];
    }
    __syncthreads();
    // the path: the best node's ancestors and itself in increasing index order
    // (a parent's index is below its child's); node j goes to position
    // popcount(ancestor bits below j)
    {
        const uint32_t word = s_anc_best[u >> 5];
        if ((word >> (u & 31)) & 1u) {
            int t = __popc(word & ((1u << (u & 31)) - 1u));
            for (int i = 0; i < (u >> 5); ++i) t += __popc(s_anc_best[i]);
            s_path[t] = u;
            accept_path[(long)b * max_path + t] = u;
        }
        if (u >= L && u < max_path) accept_path[(long)b * max_path + u] = -1;
        if (u == 0) {
            accept_len[b] = L;
            bonus[b] = pred[best];
        }
    }
    if (cm.kc) {
        __syncthreads();  // s_path is complete
        commit_path(b, s_path, L, S_commit, L <= max_path, cm.kc, cm.vc, cm.kt, cm.vt, cm.new_prefix_len, Tn, cm.Hkv,
                    cm.S_max, cm.row_bytes, cm.table, cm.max_pages, cm.page_size, cm.num_pages, cm.status);
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

constexpr double kTwo32 = 4294967296.0;

// floor(max(0, x) * 2^32) as an integer weight
__device__ __forceinline__ unsigned long long weight_2p32(double x) {
    return x > 0.0 ? (unsigned long long)floor(__dmul_rn(x, kTwo32)) : 0ull;
}

// Exact sums over the cluster.  Every thread passes its partial; returns the
// cluster total, and in *before the sum of the partials of lower-ranked CTAs
// and of lower-indexed warps of this CTA (the exclusive prefix of this warp's
// segment in vocabulary order: shares and segments are contiguous and
// rank-ordered).
struct ClusterSum {
    unsigned long long warp_tot[kStochThreads / 32];
    unsigned long long cta_tot;
    double warp_d[kStochThreads / 32];
    double cta_d;
};
__device__ unsigned long long cluster_sum(unsigned long long x, ClusterSum* sh, unsigned long long* before) {
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    unsigned long long wt = x;  // warp total
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wt += __shfl_xor_sync(kFull, wt, o);
    if (lane == 0) sh->warp_tot[warp] = wt;
    __syncthreads();
    unsigned long long wbefore = 0, cta = 0;
    for (int w = 0; w < kStochThreads / 32; ++w) {
        const unsigned long long t = sh->warp_tot[w];
        if (w < warp) wbefore += t;
        cta += t;
    }
    if (tid == 0) sh->cta_tot = cta;
    __syncwarp();  // the cluster barrier is an aligned one: whole warps
    cl.sync();     // every CTA's total (and its earlier global writes) visible
    const int rank = (int)cl.block_rank(), C = (int)cl.num_blocks();
    unsigned long long tot = 0, rbefore = 0;
    for (int r = 0; r < C; ++r) {
        const unsigned long long t = cl.map_shared_rank(sh, r)->cta_tot;
        if (r < rank) rbefore += t;
        tot += t;
    }
    cl.sync();  // nobody reuses sh before every CTA has read it
    if (before) *before = rbefore + wbefore;
    return tot;
}

// fp64 maximum (kMax; NaN skipped) or sum over the cluster, in a fixed
// order (lane butterfly, warps 0.., CTAs 0..): every thread of the cluster
// gets the same bits.
template <bool kMax>
__device__ double cluster_reduce_f64(double x, ClusterSum* sh) {
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double y = __shfl_xor_sync(kFull, x, o);
        x = kMax ? fmax(x, y) : __dadd_rn(x, y);
    }
    if (lane == 0) sh->warp_d[warp] = x;
    __syncthreads();
    if (tid == 0) {
        double c = sh->warp_d[0];
        for (int w = 1; w < kStochThreads / 32; ++w) c = kMax ? fmax(c, sh->warp_d[w]) : __dadd_rn(c, sh->warp_d[w]);
        sh->cta_d = c;
    }
    __syncwarp();
    cl.sync();
    const int C = (int)cl.num_blocks();
    double t = cl.map_shared_rank(sh, 0)->cta_d;
    for (int r = 1; r < C; ++r) {
        const double v = cl.map_shared_rank(sh, r)->cta_d;
        t = kMax ? fmax(t, v) : __dadd_rn(t, v);
    }
    cl.sync();
    return t;
}

// target rows: kSrc 0 = probabilities p (f32), 1 = f32 logits, 2 = bf16 logits
template <int kSrc>
__device__ __forceinline__ double target_at(const void* row, int y) {
    if constexpr (kSrc == 2) return (double)__bfloat162float(((const __nv_bfloat16*)row)[y]);
    else return (double)((const float*)row)[y];
}

template <int kSrc>
__global__ void __launch_bounds__(kStochThreads, 2) verify_stochastic_kernel(
    const void* __restrict__ target, double inv_tau, const float* __restrict__ q, int q_rows, const int32_t* __restrict__ q_row,
    const int32_t* __restrict__ node_tokens, int V, TreeRef trees, uint32_t key0, uint32_t key1,
    uint32_t step, int32_t* accept_path, int max_path, int32_t* accept_len, int32_t* bonus,
    unsigned long long* ws_w, int32_t* status) {
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    __shared__ ClusterSum sh;
    const int C = (int)cl.num_blocks(), rank = (int)cl.block_rank();
    const int b = blockIdx.x / C, tid = threadIdx.x;
    const bool lead = rank == 0 && tid == 0;
    const TreeDev* tree = trees.at(b);
    const int T = trees.T;  // node stride of target, node_tokens (and of q_row with one tree per sequence)
    constexpr int kEsz = kSrc == 2 ? 2 : 4;
    const char* Pb = (const char*)target + (long)b * T * V * kEsz;
    // Two weight buffers.  `valid` holds the last effective residual (S > 0)
    // of the current node, -1 while P is still p[b,u,:].  `keep` is the
    // buffer the latest accept decision may have read (threads of the
    // cluster may still be reading it, also after the walk moved on); a pass
    // writes the other one, which becomes valid if its sum is positive (a
    // residual with S = 0 keeps P).  The cluster-wide sum that ends a pass
    // orders every later reuse.
    const long BV = (long)gridDim.x / C * V;
    // this warp's vocabulary segment [y0, y1); lane l takes y0 + l + 32 i
    const int warp = tid >> 5, lane = tid & 31;
    const int share = (V + C - 1) / C;
    const int v0 = min(V, rank * share), v1 = min(V, v0 + share);
    const int seg = (v1 - v0 + kStochThreads / 32 - 1) / (kStochThreads / 32);
    const int y0 = min(v1, v0 + warp * seg), y1 = min(v1, y0 + seg);
    constexpr int U = 8;  // entries in flight per lane

    int u = 0, L = 1, valid = -1, keep = -1;
    unsigned long long S_valid = 0;
    const void* Prow = Pb;
    double row_m = 0.0, row_r = 1.0;  // logits: the row's maximum and 1 / Z
    auto Wbuf = [&](int i) { return ws_w + (i & 1) * BV + (long)b * V; };
    // the target's own distribution at y of the current node's row
    auto target_p = [&](int y) -> double {
        const double z = target_at<kSrc>(Prow, y);
        if constexpr (kSrc == 0) return z;
        else return __dmul_rn(exp(__dmul_rn(__dsub_rn(z, row_m), inv_tau)), row_r);
    };
    // current target distribution at y
    auto cur = [&](int y) -> double {
        if (valid < 0) return target_p(y);
        return __ddiv_rn((double)Wbuf(valid)[y], (double)S_valid);
    };
    // move to node n's row; with logits, the row's maximum and normaliser
    // (every thread of the cluster, in step)
    auto enter_row = [&](int n) {
        Prow = Pb + (long)n * V * kEsz;
        if constexpr (kSrc != 0) {
            double m = -INFINITY;
            for (int y = y0 + lane; y < y1; y += 32 * U) {
                double z[U];
#pragma unroll
                for (int i = 0; i < U; ++i) z[i] = y + 32 * i < y1 ? target_at<kSrc>(Prow, y + 32 * i) : -INFINITY;
#pragma unroll
                for (int i = 0; i < U; ++i) m = fmax(m, z[i]);
            }
            m = cluster_reduce_f64<true>(m, &sh);
            double Z = 0.0;
            for (int y = y0 + lane; y < y1; y += 32 * U) {
                double z[U];
#pragma unroll
                for (int i = 0; i < U; ++i) z[i] = y + 32 * i < y1 ? target_at<kSrc>(Prow, y + 32 * i) : 0.0;
#pragma unroll
                for (int i = 0; i < U; ++i)
                    if (y + 32 * i < y1) Z = __dadd_rn(Z, exp(__dmul_rn(__dsub_rn(z[i], m), inv_tau)));
            }
            Z = cluster_reduce_f64<false>(Z, &sh);
            row_m = m;
            row_r = __ddiv_rn(1.0, Z);
        }
    };
    if (lead) {
        accept_path[(long)b * max_path] = 0;
        for (int t = 1; t < max_path; ++t) accept_path[(long)b * max_path + t] = -1;
    }
    const float* Qrow = nullptr;
    for (;;) {
        const int c_begin = tree->child_off[u], c_end = tree->child_off[u + 1];
        if (valid >= 0) keep = valid;
        valid = -1;
        enter_row(u);
        if (c_begin == c_end) break;  // a leaf: no drafted children
        const int qr = q_row ? q_row[(trees.stride ? (long)b * T : 0) + u] : u;
        if (qr < 0 || qr >= q_rows) {
            if (lead) set_status(status, MEDUSA_STATUS_BAD_TOKEN);
            break;
        }
        Qrow = q + ((long)b * q_rows + qr) * V;
        bool moved = false;
        for (int ci = c_begin; ci < c_end; ++ci) {
            const int c = tree->child_idx[ci];
            const int x = node_tokens[(long)b * T + c];
            if (x < 0 || x >= V) {
                if (lead) set_status(status, MEDUSA_STATUS_BAD_TOKEN);
                continue;
            }
            // every thread takes the same decision from the same values
            const uint4 r = philox4x32_10(make_uint4((uint32_t)b, (uint32_t)c, step, 0u), key0, key1);
            const double uc = (double)(r.x >> 8) * (1.0 / 16777216.0);
            const double Qx = (double)Qrow[x];
            if (__dmul_rn(uc, Qx) < cur(x)) {
                u = c;
                if (lead) accept_path[(long)b * max_path + L] = c;
                ++L;
                moved = true;
                break;
            }
            // rejected: W(y) = floor(max(0, P(y) - Q(y)) * 2^32), S = sum W
            unsigned long long part = 0;
            const int nb = keep < 0 ? 0 : keep ^ 1;
            unsigned long long* Wn = Wbuf(nb);
            for (int y = y0 + lane; y < y1; y += 32 * U) {
                double P[U], Q[U];
#pragma unroll
                for (int i = 0; i < U; ++i) {
                    const int yy = y + 32 * i;
                    P[i] = yy < y1 ? cur(yy) : 0.0;
                    Q[i] = yy < y1 ? (double)Qrow[yy] : 0.0;
                }
#pragma unroll
                for (int i = 0; i < U; ++i) {
                    const int yy = y + 32 * i;
                    if (yy < y1) {
                        const unsigned long long w = weight_2p32(__dsub_rn(P[i], Q[i]));
                        Wn[yy] = w;
                        part += w;
                    }
                }
            }
            const unsigned long long S = cluster_sum(part, &sh, nullptr);
            if (S > 0) {
                valid = keep = nb;
                S_valid = S;
            }
        }
        if (!moved) break;
    }
    // bonus from the current distribution: weights floor(P(y) * 2^32), kept
    // in the next buffer for the scan below
    unsigned long long* Wb = Wbuf(keep < 0 ? 0 : keep ^ 1);
    unsigned long long part = 0;
    for (int y = y0 + lane; y < y1; y += 32 * U) {
        double P[U];
#pragma unroll
        for (int i = 0; i < U; ++i) P[i] = y + 32 * i < y1 ? cur(y + 32 * i) : 0.0;
#pragma unroll
        for (int i = 0; i < U; ++i)
            if (y + 32 * i < y1) {
                const unsigned long long w = weight_2p32(P[i]);
                Wb[y + 32 * i] = w;
                part += w;
            }
    }
    unsigned long long start;
    const unsigned long long S = cluster_sum(part, &sh, &start);
    if (lead) accept_len[b] = L;
    if (S == 0) {
        if (lead) {
            set_status(status, MEDUSA_STATUS_NO_MASS);
            bonus[b] = 0;
        }
        return;
    }
    const uint4 r = philox4x32_10(make_uint4((uint32_t)b, (uint32_t)u, step, 0u), key0, key1);
    // t = floor(U * S / 2^32) from the exact 128-bit product
    const unsigned long long lo = (unsigned long long)r.y * (S & 0xffffffffull);
    const unsigned long long hi = (unsigned long long)r.y * (S >> 32);
    const unsigned long long t = (lo >> 32) + hi;
    // the smallest y whose inclusive prefix sum exceeds t lies in the one
    // warp segment with start <= t < start + (segment total)
    unsigned long long wtot = part;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wtot += __shfl_xor_sync(kFull, wtot, o);
    if (start <= t && t < start + wtot) {
        unsigned long long run = start;
        for (int y = y0; y < y1; y += 32) {
            const unsigned long long w = y + lane < y1 ? Wb[y + lane] : 0ull;
            unsigned long long inc = w;  // inclusive scan of 32 consecutive entries
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long n = __shfl_up_sync(kFull, inc, o);
                if (lane >= o) inc += n;
            }
            const unsigned long long total = __shfl_sync(kFull, inc, 31);
            if (run + total > t) {
                const unsigned m = __ballot_sync(kFull, run + inc > t);
                if (lane == 0) bonus[b] = y + __ffs(m) - 1;
                break;
            }
            run += total;
        }
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

// cluster size of the stochastic kernel: up to 8 CTAs per sequence while the
// grid fits in one wave
int stoch_cluster(int B) {
    int c = 1;
    while (c < 8 && (long)B * c * 2 <= 2L * num_sms()) c *= 2;  // two 512-thread CTAs per SM
    return c;
}

size_t verify_workspace_size(medusa_verify_mode mode, int B, int V, int T) {
    if (mode != MEDUSA_VERIFY_GREEDY)  // two buffers of W (u64) per sequence and vocabulary entry
        return align256(2 * (size_t)B * V * sizeof(unsigned long long));
    int s = argmax_splits(B * T, V);
    return align256((size_t)B * T * s * sizeof(float)) + align256((size_t)B * T * s * sizeof(int));
}

// greedy: the row-argmax partials of every node's target row, in workspace
cudaError_t verify_greedy_rows_launch(const VerifyArgs& a, cudaStream_t st) {
    const int rows = a.B * a.T;
    const int splits = argmax_splits(rows, a.V);
    int chunk = (a.V + splits - 1) / splits;
    chunk = (chunk + 7) / 8 * 8;
    float* pval = (float*)a.ws;
    int* pidx = (int*)((char*)a.ws + align256((size_t)rows * splits * sizeof(float)));
    dim3 grid(rows, splits);
    const size_t elt = a.target_dt == MEDUSA_BF16 ? 2 : 4;
    const size_t stage = (size_t)chunk * elt;
    // staged when every row starts on a 16-byte boundary and a chunk fits the
    // stage (contiguous chunks of whole vectors; the row's tail is read directly)
    if (((uintptr_t)a.target & 15) == 0 && ((size_t)a.V * elt) % 16 == 0 && stage <= (size_t)kStageBytes) {
        if (a.target_dt == MEDUSA_BF16) {
            auto k = row_argmax_staged_kernel<__nv_bfloat16>;
            cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kStageBytes);
            prefer_max_smem(k);
            k<<<grid, kArgmaxThreads, stage, st>>>((const __nv_bfloat16*)a.target, a.V, splits, chunk, pval, pidx,
                                                  a.status);
        } else {
            auto k = row_argmax_staged_kernel<float>;
            cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kStageBytes);
            prefer_max_smem(k);
            k<<<grid, kArgmaxThreads, stage, st>>>((const float*)a.target, a.V, splits, chunk, pval, pidx, a.status);
        }
        return cudaGetLastError();
    }
    if (a.target_dt == MEDUSA_BF16) prefer_max_smem(row_argmax_kernel<__nv_bfloat16>);
    else prefer_max_smem(row_argmax_kernel<float>);
    if (a.target_dt == MEDUSA_BF16)
        row_argmax_kernel<__nv_bfloat16>
            <<<grid, kArgmaxThreads, 0, st>>>((const __nv_bfloat16*)a.target, a.V, splits, chunk, pval, pidx);
    else
        row_argmax_kernel<float><<<grid, kArgmaxThreads, 0, st>>>((const float*)a.target, a.V, splits, chunk, pval,
                                                                  pidx);
    return cudaGetLastError();
}

// greedy: the tree walk over those partials, optionally followed by the commit
static cudaError_t walk_launch(const VerifyArgs& a, const WalkCommit& cm, cudaStream_t st) {
    const int rows = a.B * a.T;
    const int splits = argmax_splits(rows, a.V);
    const float* pval = (const float*)a.ws;
    const int* pidx = (const int*)((const char*)a.ws + align256((size_t)rows * splits * sizeof(float)));
    prefer_max_smem(greedy_walk_kernel);
    greedy_walk_kernel<<<a.B, kWalkThreads, 0, st>>>(pval, pidx, splits, a.node_tokens, a.tree, a.accept_path,
                                                     a.max_path, a.accept_len, a.bonus, cm);
    return cudaGetLastError();
}

cudaError_t verify_greedy_walk_launch(const VerifyArgs& a, cudaStream_t st) {
    WalkCommit cm;
    memset(&cm, 0, sizeof cm);
    return walk_launch(a, cm, st);
}

cudaError_t verify_greedy_walk_commit_launch(const VerifyArgs& a, const CommitArgs& c, cudaStream_t st) {
    WalkCommit cm;
    cm.kc = (uint8_t*)c.k_cache;
    cm.vc = (uint8_t*)c.v_cache;
    cm.kt = (const uint8_t*)c.k_tree;
    cm.vt = (const uint8_t*)c.v_tree;
    cm.prefix_len = c.prefix_len;
    cm.new_prefix_len = c.new_prefix_len;
    cm.Hkv = c.Hkv;
    cm.S_max = c.S_max;
    cm.row_bytes = c.D * c.esize;
    cm.table = c.block_table;
    cm.max_pages = c.max_pages;
    cm.page_size = c.page_size;
    cm.num_pages = c.num_pages;
    cm.status = c.status;
    return walk_launch(a, cm, st);
}

cudaError_t verify_launch(const VerifyArgs& a, cudaStream_t st) {
    if (a.mode == MEDUSA_VERIFY_GREEDY) {
        cudaError_t e = verify_greedy_rows_launch(a, st);
        if (e != cudaSuccess) return e;
        return verify_greedy_walk_launch(a, st);
    }
    const int C = stoch_cluster(a.B);
    unsigned long long* ws_w = (unsigned long long*)a.ws;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.B * C);
    cfg.blockDim = dim3(kStochThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    auto kernel = !a.logits ? verify_stochastic_kernel<0>
                  : a.target_dt == MEDUSA_BF16 ? verify_stochastic_kernel<2> : verify_stochastic_kernel<1>;
    const double inv_tau = a.logits ? a.inv_tau : 1.0;
    prefer_max_smem(kernel);
    return cudaLaunchKernelEx(&cfg, kernel, a.target, inv_tau, a.q, a.q_rows, a.q_row, a.node_tokens, a.V, a.tree,
                              (uint32_t)a.seed, (uint32_t)(a.seed >> 32), a.step, a.accept_path, a.max_path,
                              a.accept_len, a.bonus, ws_w, a.status);
}

}  // namespace medusa
