// Device helpers shared by the heads kernels: running softmax statistics and
// top-8 lists per (sequence, head), their merges, and the final per-head
// merge that writes top-8 entries and fills the candidate tree.
#pragma once

#include <limits.h>

#include "common.cuh"

namespace medusa {

// Running softmax statistics and top-8 list of one (sequence, head) over a
// set of vocabulary rows: m = max logit, l = sum exp(logit - m).
struct HeadState {
    float m, l;
    float val[kTopK];
    int idx[kTopK];
};

__device__ __forceinline__ HeadState empty_state() {
    HeadState s;
    s.m = -INFINITY;
    s.l = 0.f;
#pragma unroll
    for (int j = 0; j < kTopK; ++j) {
        s.val[j] = -INFINITY;
        s.idx[j] = INT_MAX;
    }
    return s;
}

// merge softmax statistics (m2, l2) into (m, l); every product and the sum
// rounded once (no fused multiply-add), so merge(a, b) == merge(b, a) bit for
// bit and the lanes of a butterfly reduction all end with the same (m, l)
__device__ __forceinline__ void merge_ml(float& m, float& l, float m2, float l2) {
    if (m2 == -INFINITY) return;
    if (m == -INFINITY) {
        m = m2;
        l = l2;
        return;
    }
    float mn = fmaxf(m, m2);
    l = __fadd_rn(__fmul_rn(l, expf(m - mn)), __fmul_rn(l2, expf(m2 - mn)));
    m = mn;
}

// Insert (v, i) into a register-resident list sorted best-first.
__device__ __forceinline__ void list_insert(float (&lv)[kTopK], int (&li)[kTopK], float v, int i) {
    if (!beats(v, i, lv[kTopK - 1], li[kTopK - 1])) return;
    lv[kTopK - 1] = v;
    li[kTopK - 1] = i;
#pragma unroll
    for (int j = kTopK - 1; j > 0; --j) {
        if (beats(lv[j], li[j], lv[j - 1], li[j - 1])) {
            float tv = lv[j];
            lv[j] = lv[j - 1];
            lv[j - 1] = tv;
            int ti = li[j];
            li[j] = li[j - 1];
            li[j - 1] = ti;
        }
    }
}

// Warp-wide selection of the best kTopK candidates from per-lane sorted
// lists.  Lane j < kTopK receives the j-th best in (out_v, out_i).
__device__ __forceinline__ void warp_select(float (&lv)[kTopK], int (&li)[kTopK], float& out_v, int& out_i) {
    const int lane = threadIdx.x & 31;
    out_v = -INFINITY;
    out_i = INT_MAX;
#pragma unroll 1
    for (int r = 0; r < kTopK; ++r) {
        float wv = lv[0];
        int wi = li[0];
        int wl = lane;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float ov = __shfl_xor_sync(kFull, wv, o);
            int oi = __shfl_xor_sync(kFull, wi, o);
            int ol = __shfl_xor_sync(kFull, wl, o);
            if (beats(ov, oi, wv, wi) || (ov == wv && oi == wi && ol < wl)) {
                wv = ov;
                wi = oi;
                wl = ol;
            }
        }
        if (lane == r) {
            out_v = wv;
            out_i = wi;
        }
        if (lane == wl) {  // pop the head of the winning lane's list
#pragma unroll
            for (int j = 0; j < kTopK - 1; ++j) {
                lv[j] = lv[j + 1];
                li[j] = li[j + 1];
            }
            lv[kTopK - 1] = -INFINITY;
            li[kTopK - 1] = INT_MAX;
        }
    }
}

// ---------------------------------------------------------------------------
// Which CTAs hold a partial of head k.  The K*uph tiles (head k owning tiles
// [k*uph, (k+1)*uph)) are cut into upt units each; nparts CTAs split the
// K*uph*upt units evenly and CTA c owns the tiles whose first unit falls in
// its share.  The CTAs owning head k's tiles lie in [c_lo, c_hi], the owners
// of its first and last tiles (unit u lies in the share of CTA
// ceil((u+1) nparts / R) - 1); when every share holds a tile start, every
// CTA of that range owns one of head k's tiles.
// ---------------------------------------------------------------------------
struct HeadCover {
    long R;
    int nparts, upt, c_lo, c_hi;
    bool dense;
    __device__ HeadCover(int nparts_, long uph, int upt_, int K, int k) : nparts(nparts_), upt(upt_) {
        R = (long)K * uph * upt;
        c_lo = owner((long)k * uph * upt);
        c_hi = owner(((long)(k + 1) * uph - 1) * upt);
        dense = R / nparts >= upt;
    }
    __device__ int owner(long u) const { return (int)(((u + 1) * nparts + R - 1) / R - 1); }
    __device__ bool covers(int c) const {
        if (c < c_lo || c > c_hi) return false;
        if (dense) return true;
        const long r0 = R * c / nparts, r1 = R * (c + 1) / nparts;
        return (r1 + upt - 1) / upt > (r0 + upt - 1) / upt;  // owns a tile (in head k, by the range)
    }
    __device__ int count() const {
        if (dense) return c_hi - c_lo + 1;
        int n = 0;
        for (int c = c_lo; c <= c_hi; ++c) n += covers(c);
        return n;
    }
};

// ---------------------------------------------------------------------------
// Merge of one (sequence, head): the partials of the CTAs that covered the
// head, in CTA order, so the result does not depend on which CTA runs the
// merge.  The K*uph tiles (head k owning tiles [k*uph, (k+1)*uph)) are cut
// into upt units each; the CTAs split the K*uph*upt units evenly and CTA c
// owns the tiles whose first unit falls in its share; partial (c, k, b) sits
// at part[(c*K + k)*bstride + b].  Writes the top-8 entries with their
// probabilities, the head's softmax statistics, and fills the nodes of
// sequence b's tree that this head proposes (node_tokens and node_q have Tn
// nodes per sequence; head 0 also writes the root and sets the rows past
// that tree to -1 and 0).  One warp.
// Partials are read through L2 (they may have been written by other CTAs of
// the same kernel).  dry: everything but the writes (the reads stay inside
// the workspace and the tree), to bring the code into the instruction cache
// ahead of a merge on the critical path.
// ---------------------------------------------------------------------------
static __device__ __noinline__ void merge_head(const HeadState* __restrict__ part, int nparts, long uph, int upt,
                                               int bstride, int bb,
                                       int b, int V, int K, int k,
                           const TreeDev* __restrict__ tree, int Tn, const int32_t* __restrict__ root_token,
                           int32_t* __restrict__ topk_idx, float* __restrict__ topk_prob,
                           int32_t* __restrict__ node_tokens, float* __restrict__ node_q, float2* __restrict__ stats,
                           int32_t* status, bool dry = false) {
    const int lane = threadIdx.x & 31;
    // the tree's shape and the root token are needed at the end: load them
    // first, so their latency overlaps the partials'
    constexpr int kTreeChunks = kMaxTree / 32;
    int rk[kTreeChunks], dp[kTreeChunks];
    const int T = tree ? tree->T : 0;
#pragma unroll
    for (int j = 0; j < kTreeChunks; ++j) {
        const int i = lane + 32 * j;
        rk[j] = i < T ? tree->rank[i] : 0;
        dp[j] = i < T ? tree->depth[i] : 0;
    }
    const int rt = (tree && k == 0) ? root_token[b] : 0;
    float mm = -INFINITY, ll = 0.f;
    float lv[kTopK];
    int li[kTopK];
#pragma unroll
    for (int j = 0; j < kTopK; ++j) {
        lv[j] = -INFINITY;
        li[j] = INT_MAX;
    }
    const HeadCover hc(nparts, uph, upt, K, k);
    const int c_lo = hc.c_lo, c_hi = hc.c_hi;
    auto covers = [&](int c) -> bool { return hc.covers(c); };
    // lane l takes CTAs c_lo + l, c_lo + l + 32, ...; two of them per round,
    // all loads of a round issued before any is used
    for (int j0 = 0; c_lo + 32 * j0 <= c_hi; j0 += 2) {
        const int cc[2] = {c_lo + lane + 32 * j0, c_lo + lane + 32 * (j0 + 1)};
        const bool cv[2] = {covers(cc[0]), covers(cc[1])};
        float pv[2][kTopK], sm[2], sl[2];
        int pi[2][kTopK];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (!cv[u]) continue;
            const HeadState* s = &part[((long)cc[u] * K + k) * bstride + bb];
#pragma unroll
            for (int j = 0; j < kTopK; ++j) {
                pv[u][j] = __ldcg(&s->val[j]);
                pi[u][j] = __ldcg(&s->idx[j]);
            }
            sm[u] = __ldcg(&s->m);
            sl[u] = __ldcg(&s->l);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (!cv[u]) continue;
            merge_ml(mm, ll, sm[u], sl[u]);
            if (li[0] == INT_MAX) {
                // the lane's list is empty: a partial's list is sorted, copy it
#pragma unroll
                for (int j = 0; j < kTopK; ++j) {
                    lv[j] = pv[u][j];
                    li[j] = pi[u][j];
                }
            } else {
                // insert in order, up to the first entry that does not make it
                for (int j = 0; j < kTopK; ++j) {
                    if (!beats(pv[u][j], pi[u][j], lv[kTopK - 1], li[kTopK - 1])) break;
                    list_insert(lv, li, pv[u][j], pi[u][j]);
                }
            }
        }
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float m2 = __shfl_xor_sync(kFull, mm, o);
        const float l2 = __shfl_xor_sync(kFull, ll, o);
        merge_ml(mm, ll, m2, l2);
    }
    float ov;
    int oi;
    warp_select(lv, li, ov, oi);
    const bool valid = oi != INT_MAX;
    const float prob = valid ? expf(ov - mm) / ll : 0.f;
    if (dry) return;
    if (lane < kTopK) {
        topk_idx[((long)b * K + k) * kTopK + lane] = valid ? oi : -1;
        topk_prob[((long)b * K + k) * kTopK + lane] = prob;
    }
    if (lane == 0 && stats) stats[(long)b * K + k] = make_float2(mm, ll);
    if (tree) {
#pragma unroll
        for (int j = 0; j < kTreeChunks; ++j) {
            const int i = lane + 32 * j;
            const int tok = __shfl_sync(kFull, valid ? oi : -1, rk[j] & (kTopK - 1));
            const float pq = __shfl_sync(kFull, prob, rk[j] & (kTopK - 1));
            if (i < T && i > 0 && dp[j] == k + 2) {
                node_tokens[(long)b * Tn + i] = tok;
                if (node_q) node_q[(long)b * Tn + i] = pq;
                if (tok < 0) set_status(status, MEDUSA_STATUS_BAD_TOKEN);
            }
            if (k == 0 && i >= T && i < Tn) {  // rows past this sequence's own tree
                node_tokens[(long)b * Tn + i] = -1;
                if (node_q) node_q[(long)b * Tn + i] = 0.f;
            }
        }
        if (k == 0 && lane == 0) {
            node_tokens[(long)b * Tn] = rt;
            if (node_q) node_q[(long)b * Tn] = 1.f;
            if (rt < 0 || rt >= V) set_status(status, MEDUSA_STATUS_BAD_TOKEN);
        }
    }
}

}  // namespace medusa
