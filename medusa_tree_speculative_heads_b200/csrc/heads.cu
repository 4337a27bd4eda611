// Medusa heads on B200: residual block, LM projection with fused online
// softmax statistics and top-8 selection, merge and candidate-tree fill.
//
// Operation ("Medusa Explained: Multi-Head Speculative Decoding Guide",
// section "The Architectural Blueprint"):
//     h^(k) = SiLU(W_res^(k) h) + h,   p^(k) = softmax(W_head^(k) h^(k)),
// then the top-s_k tokens of each head fill the candidate tree (section
// "1. Combinatorial Tree Construction").
//
// At decode batch sizes both products are matrix-vector products that read
// every weight exactly once, so the kernels are HBM streams: 16-byte
// coalesced loads that bypass L1, many independent loads in flight per warp,
// fp32 accumulation, and all per-row epilogue work (softmax statistics, top-8)
// fused so the logits never make a round trip through HBM.
#include <float.h>
#include <limits.h>

#include "kernels.h"

namespace medusa {

namespace {

constexpr int kResWarps = 8;   // warps per block of the residual kernel
constexpr int kLmWarps = 8;    // warps per block of the LM-head kernel
constexpr int kBG = 8;         // sequences handled per LM-head launch
constexpr int kUnroll = 8;     // 16-byte loads issued back to back per lane

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

// merge softmax statistics (m2, l2) into (m, l)
__device__ __forceinline__ void merge_ml(float& m, float& l, float m2, float l2) {
    if (m2 == -INFINITY) return;
    if (m == -INFINITY) {
        m = m2;
        l = l2;
        return;
    }
    float mn = fmaxf(m, m2);
    l = l * expf(m - mn) + l2 * expf(m2 - mn);
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
// K1: residual block.  One warp per output feature (k, o); the W_res row is
// streamed once and dotted with every sequence's h.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kResWarps * 32) heads_res_kernel(const T* __restrict__ h,
                                                                   const T* __restrict__ W_res, int B, int d, int K,
                                                                   T* __restrict__ hk, T* __restrict__ hk_out) {
    constexpr int VEC = Elt<T>::kVec;
    const int lane = threadIdx.x & 31;
    const long row = (long)blockIdx.x * kResWarps + (threadIdx.x >> 5);  // k * d + o
    if (row >= (long)K * d) return;
    const int k = (int)(row / d), o = (int)(row % d);
    const int nvec = d / VEC;
    const T* wrow = W_res + row * (long)d;
    for (int b0 = 0; b0 < B; b0 += kBG) {
        float acc[kBG];
#pragma unroll
        for (int bb = 0; bb < kBG; ++bb) acc[bb] = 0.f;
        for (int c0 = 0; c0 < nvec; c0 += 32 * kUnroll) {
            uint4 wv[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                int c = c0 + u * 32 + lane;
                wv[u] = c < nvec ? ld_stream(wrow + (long)c * VEC) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                int c = c0 + u * 32 + lane;
                if (c >= nvec) break;
                float wf[VEC];
                Elt<T>::unpack(wv[u], wf);
#pragma unroll
                for (int bb = 0; bb < kBG; ++bb) {
                    if (b0 + bb < B) {
                        float hf[VEC];
                        Elt<T>::unpack(ld_nc(h + (long)(b0 + bb) * d + (long)c * VEC), hf);
#pragma unroll
                        for (int e = 0; e < VEC; ++e) acc[bb] = fmaf(wf[e], hf[e], acc[bb]);
                    }
                }
            }
        }
#pragma unroll
        for (int bb = 0; bb < kBG; ++bb) acc[bb] = warp_sum(acc[bb]);
        if (lane == 0) {
#pragma unroll
            for (int bb = 0; bb < kBG; ++bb) {
                int b = b0 + bb;
                if (b < B) {
                    float z = acc[bb];
                    float y = z / (1.f + expf(-z)) + Elt<T>::to_float(h[(long)b * d + o]);
                    T yt = Elt<T>::from_float(y);
                    long off = ((long)b * K + k) * d + o;
                    hk[off] = yt;
                    if (hk_out) hk_out[off] = yt;
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// K2: LM-head projection.  The K*V weight rows are split into one contiguous
// range per CTA (grid = a full wave of CTAs); warps take rows round-robin.
// Each row's logits (for up to kBG sequences) update the warp's running
// softmax statistics and top-8 list; the CTA merges its warps and writes one
// partial per (head, sequence) it covered.  HREG: a single sequence whose
// h^(k) fits in registers (d/VEC <= 32*kUnroll*2).
// ---------------------------------------------------------------------------
template <typename T, bool HREG>
__global__ void __launch_bounds__(kLmWarps * 32) heads_lm_kernel(const T* __restrict__ W_head,
                                                                 const T* __restrict__ hk, int B, int d, int V,
                                                                 int K, float* __restrict__ logits,
                                                                 HeadState* __restrict__ part) {
    constexpr int VEC = Elt<T>::kVec;
    constexpr int NREG = 2 * kUnroll;  // register-held chunks of h per lane (HREG)
    extern __shared__ HeadState sstate[];  // [kLmWarps][K][kBG]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long R = (long)K * V;
    const long r0 = R * blockIdx.x / gridDim.x, r1 = R * (blockIdx.x + 1) / gridDim.x;
    const int nvec = d / VEC;
    const int nb = min(B, kBG);

    for (int t = threadIdx.x; t < kLmWarps * K * kBG; t += blockDim.x) sstate[t] = empty_state();
    __syncthreads();

    float m[kBG], l[kBG], tv[kBG];
    int ti[kBG];
#pragma unroll
    for (int bb = 0; bb < kBG; ++bb) {
        m[bb] = -INFINITY;
        l[bb] = 0.f;
        tv[bb] = -INFINITY;
        ti[bb] = INT_MAX;
    }
    uint4 hr[HREG ? NREG : 1];
    int cur_k = -1;

    auto flush = [&](int kk) {
#pragma unroll
        for (int bb = 0; bb < kBG; ++bb) {
            HeadState* s = &sstate[(warp * K + kk) * kBG + bb];
            if (lane < kTopK) {
                s->val[lane] = tv[bb];
                s->idx[lane] = ti[bb];
            }
            if (lane == 0) {
                s->m = m[bb];
                s->l = l[bb];
            }
            m[bb] = -INFINITY;
            l[bb] = 0.f;
            tv[bb] = -INFINITY;
            ti[bb] = INT_MAX;
        }
    };

    for (long r = r0 + warp; r < r1; r += kLmWarps) {
        const int k = (int)(r / V);
        const int v = (int)(r - (long)k * V);
        if (k != cur_k) {
            if (cur_k >= 0) flush(cur_k);
            cur_k = k;
            if constexpr (HREG) {
#pragma unroll
                for (int j = 0; j < NREG; ++j) {
                    int c = j * 32 + lane;
                    hr[j] = c < nvec ? ld_nc(hk + (long)k * d + (long)c * VEC) : make_uint4(0, 0, 0, 0);
                }
            }
        }
        const T* wrow = W_head + r * (long)d;
        float acc[kBG];
#pragma unroll
        for (int bb = 0; bb < kBG; ++bb) acc[bb] = 0.f;
        if constexpr (HREG) {
            uint4 wv[NREG];
#pragma unroll
            for (int j = 0; j < NREG; ++j) {
                int c = j * 32 + lane;
                wv[j] = c < nvec ? ld_stream(wrow + (long)c * VEC) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int j = 0; j < NREG; ++j) {
                float wf[VEC], hf[VEC];
                Elt<T>::unpack(wv[j], wf);
                Elt<T>::unpack(hr[j], hf);
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[0] = fmaf(wf[e], hf[e], acc[0]);
            }
        } else {
            for (int c0 = 0; c0 < nvec; c0 += 32 * kUnroll) {
                uint4 wv[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    int c = c0 + u * 32 + lane;
                    wv[u] = c < nvec ? ld_stream(wrow + (long)c * VEC) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    int c = c0 + u * 32 + lane;
                    if (c >= nvec) break;
                    float wf[VEC];
                    Elt<T>::unpack(wv[u], wf);
#pragma unroll
                    for (int bb = 0; bb < kBG; ++bb) {
                        if (bb < nb) {
                            float hf[VEC];
                            Elt<T>::unpack(ld_nc(hk + ((long)bb * K + k) * d + (long)c * VEC), hf);
#pragma unroll
                            for (int e = 0; e < VEC; ++e) acc[bb] = fmaf(wf[e], hf[e], acc[bb]);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int bb = 0; bb < kBG; ++bb) {
            if (bb >= nb) break;
            const float x = warp_sum(acc[bb]);
            if (logits && lane == 0) logits[((long)bb * K + k) * V + v] = x;
            // online softmax statistics (NaN logits poison l, as in exact arithmetic)
            if (x > -INFINITY || x != x) {
                float mn = fmaxf(m[bb], x);
                l[bb] = (m[bb] == -INFINITY ? 0.f : l[bb] * expf(m[bb] - mn)) + expf(x - mn);
                m[bb] = mn;
            }
            // top-8: lane j < 8 holds entry j, best first
            unsigned mask = __ballot_sync(kFull, lane < kTopK && beats(x, v, tv[bb], ti[bb]));
            if (mask) {
                int pos = __ffs(mask) - 1;
                float pv = __shfl_up_sync(kFull, tv[bb], 1);
                int pi = __shfl_up_sync(kFull, ti[bb], 1);
                if (lane == pos) {
                    tv[bb] = x;
                    ti[bb] = v;
                } else if (lane > pos && lane < kTopK) {
                    tv[bb] = pv;
                    ti[bb] = pi;
                }
            }
        }
    }
    if (cur_k >= 0) flush(cur_k);
    __syncthreads();

    // merge the warps' states of each (head, sequence) this CTA covered
    if (r1 <= r0) return;
    const int k_lo = (int)(r0 / V), k_hi = (int)((r1 - 1) / V);
    const int npairs = (k_hi - k_lo + 1) * nb;
    for (int pr = warp; pr < npairs; pr += kLmWarps) {
        const int k = k_lo + pr / nb, bb = pr % nb;
        float mm = -INFINITY, ll = 0.f;
        if (lane < kLmWarps) {
            const HeadState* s = &sstate[(lane * K + k) * kBG + bb];
            mm = s->m;
            ll = s->l;
        }
        // fixed-order tree merge of the 8 warps' statistics
#pragma unroll
        for (int o = 1; o < kLmWarps; o <<= 1) {
            float m2 = __shfl_xor_sync(kFull, mm, o);
            float l2 = __shfl_xor_sync(kFull, ll, o);
            merge_ml(mm, ll, m2, l2);
        }
        // candidates: lane j takes list entries 2(j%4), 2(j%4)+1 of warp j/4
        float lv[kTopK];
        int li[kTopK];
#pragma unroll
        for (int j = 0; j < kTopK; ++j) {
            lv[j] = -INFINITY;
            li[j] = INT_MAX;
        }
        {
            const HeadState* s = &sstate[((lane >> 2) * K + k) * kBG + bb];
            int e = (lane & 3) * 2;
            list_insert(lv, li, s->val[e], s->idx[e]);
            list_insert(lv, li, s->val[e + 1], s->idx[e + 1]);
        }
        float ov;
        int oi;
        warp_select(lv, li, ov, oi);
        HeadState* dst = &part[((long)blockIdx.x * K + k) * kBG + bb];
        if (lane < kTopK) {
            dst->val[lane] = ov;
            dst->idx[lane] = oi;
        }
        if (lane == 0) {
            dst->m = mm;
            dst->l = ll;
        }
    }
}

// ---------------------------------------------------------------------------
// K3: merge the CTAs' partials of one (sequence, head) in a fixed order,
// write the top-8 entries with their probabilities and the head's softmax
// statistics, and fill the tree nodes this head proposes.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32) heads_merge_kernel(const HeadState* __restrict__ part, int nparts, int b0,
                                                         int nb, int V, int K, const TreeDev* __restrict__ tree,
                                                         const int32_t* __restrict__ root_token,
                                                         int32_t* __restrict__ topk_idx,
                                                         float* __restrict__ topk_prob,
                                                         int32_t* __restrict__ node_tokens,
                                                         float* __restrict__ node_q, float2* __restrict__ stats,
                                                         int32_t* status) {
    const int lane = threadIdx.x;
    const int bb = blockIdx.x % nb, k = blockIdx.x / nb;
    const int b = b0 + bb;
    const long R = (long)K * V;
    float mm = -INFINITY, ll = 0.f;
    float lv[kTopK];
    int li[kTopK];
#pragma unroll
    for (int j = 0; j < kTopK; ++j) {
        lv[j] = -INFINITY;
        li[j] = INT_MAX;
    }
    for (int c = lane; c < nparts; c += 32) {
        const long r0 = R * c / nparts, r1 = R * (c + 1) / nparts;
        if (r1 <= r0 || (long)(k + 1) * V <= r0 || r1 <= (long)k * V) continue;  // CTA c did not cover head k
        const HeadState* s = &part[((long)c * K + k) * kBG + bb];
        merge_ml(mm, ll, s->m, s->l);
#pragma unroll
        for (int j = 0; j < kTopK; ++j) list_insert(lv, li, s->val[j], s->idx[j]);
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        float m2 = __shfl_xor_sync(kFull, mm, o);
        float l2 = __shfl_xor_sync(kFull, ll, o);
        merge_ml(mm, ll, m2, l2);
    }
    float ov;
    int oi;
    warp_select(lv, li, ov, oi);
    const bool valid = oi != INT_MAX;
    const float prob = valid ? expf(ov - mm) / ll : 0.f;
    if (lane < kTopK) {
        topk_idx[((long)b * K + k) * kTopK + lane] = valid ? oi : -1;
        topk_prob[((long)b * K + k) * kTopK + lane] = prob;
    }
    if (lane == 0 && stats) stats[(long)b * K + k] = make_float2(mm, ll);
    if (tree) {
        const int T = tree->T;
        for (int i0 = 0; i0 < T; i0 += 32) {
            int i = i0 + lane;
            int rk = i < T ? tree->rank[i] : 0;
            int tok = __shfl_sync(kFull, valid ? oi : -1, rk & (kTopK - 1));
            float pq = __shfl_sync(kFull, prob, rk & (kTopK - 1));
            if (i < T && i > 0 && tree->depth[i] == k + 2) {
                node_tokens[(long)b * T + i] = tok;
                if (node_q) node_q[(long)b * T + i] = pq;
                if (tok < 0) set_status(status, MEDUSA_STATUS_BAD_TOKEN);
            }
        }
        if (k == 0 && lane == 0) {
            int rt = root_token[b];
            node_tokens[(long)b * T] = rt;
            if (node_q) node_q[(long)b * T] = 1.f;
            if (rt < 0 || rt >= V) set_status(status, MEDUSA_STATUS_BAD_TOKEN);
        }
    }
}

// probs[b,k,v] = exp(logit - m) / l
__global__ void heads_probs_kernel(const float* __restrict__ logits, const float2* __restrict__ stats, int B,
                                   int K, int V, float* __restrict__ probs) {
    const long n = (long)B * K * V;
    for (long t = (long)blockIdx.x * blockDim.x + threadIdx.x; t < n; t += (long)gridDim.x * blockDim.x) {
        float2 s = stats[t / V];
        probs[t] = expf(logits[t] - s.x) / s.y;
    }
}

// --------------------------- launch helpers --------------------------------

struct LmConfig {
    int grid;
    size_t smem;
};

template <typename T, bool HREG>
LmConfig lm_config(int K) {
    LmConfig c;
    c.smem = sizeof(HeadState) * kLmWarps * K * kBG;
    int occ = 0;
    auto kern = heads_lm_kernel<T, HREG>;
    if (c.smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)c.smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kLmWarps * 32, c.smem);
    c.grid = num_sms() * (occ > 0 ? occ : 1);
    return c;
}

// largest grid any configuration uses (workspace sizing)
int lm_grid_bound() { return num_sms() * (2048 / (kLmWarps * 32)); }

struct HeadsWs {
    size_t hk, part, stats, logits, total;
};

HeadsWs heads_ws_layout(int B, int d, int V, int K, medusa_dtype dt) {
    HeadsWs w;
    size_t esz = dt == MEDUSA_BF16 ? 2 : 4;
    w.hk = 0;
    w.part = w.hk + align256((size_t)B * K * d * esz);
    w.stats = w.part + align256((size_t)lm_grid_bound() * K * kBG * sizeof(HeadState));
    w.logits = w.stats + align256((size_t)B * K * sizeof(float2));
    w.total = w.logits + align256((size_t)B * K * V * sizeof(float));
    return w;
}

template <typename T>
cudaError_t heads_launch_t(const HeadsArgs& a, cudaStream_t st) {
    constexpr int VEC = Elt<T>::kVec;
    HeadsWs w = heads_ws_layout(a.B, a.d, a.V, a.K, a.dt);
    char* ws = (char*)a.ws;
    T* hk = (T*)(ws + w.hk);
    HeadState* part = (HeadState*)(ws + w.part);
    float2* stats = (float2*)(ws + w.stats);
    float* logits = a.logits_out ? a.logits_out : (a.probs_out ? (float*)(ws + w.logits) : nullptr);

    const long rows = (long)a.K * a.d;
    heads_res_kernel<T><<<(unsigned)((rows + kResWarps - 1) / kResWarps), kResWarps * 32, 0, st>>>(
        (const T*)a.h, (const T*)a.W_res, a.B, a.d, a.K, hk, (T*)a.h_res_out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    const bool hreg = a.B == 1 && a.d / VEC <= 32 * 2 * kUnroll;
    for (int b0 = 0; b0 < a.B; b0 += kBG) {
        const int nb = a.B - b0 < kBG ? a.B - b0 : kBG;
        LmConfig c = hreg ? lm_config<T, true>(a.K) : lm_config<T, false>(a.K);
        const T* hk_g = hk + (long)b0 * a.K * a.d;
        float* lg = logits ? logits + (long)b0 * a.K * a.V : nullptr;
        if (hreg)
            heads_lm_kernel<T, true><<<c.grid, kLmWarps * 32, c.smem, st>>>((const T*)a.W_head, hk_g, nb, a.d, a.V,
                                                                          a.K, lg, part);
        else
            heads_lm_kernel<T, false><<<c.grid, kLmWarps * 32, c.smem, st>>>((const T*)a.W_head, hk_g, nb, a.d,
                                                                           a.V, a.K, lg, part);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        heads_merge_kernel<<<nb * a.K, 32, 0, st>>>(part, c.grid, b0, nb, a.V, a.K, a.tree, a.root_token,
                                                    a.topk_idx, a.topk_prob, a.node_tokens, a.node_q, stats,
                                                    a.status);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.probs_out) {
        long n = (long)a.B * a.K * a.V;
        int grid = (int)((n + 255) / 256);
        if (grid > num_sms() * 8) grid = num_sms() * 8;
        heads_probs_kernel<<<grid, 256, 0, st>>>(logits, stats, a.B, a.K, a.V, a.probs_out);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace

size_t heads_workspace_size(int B, int d, int V, int K, medusa_dtype dt) {
    return heads_ws_layout(B, d, V, K, dt).total;
}

cudaError_t heads_launch(const HeadsArgs& a, cudaStream_t st) {
    if (a.dt == MEDUSA_BF16) return heads_launch_t<__nv_bfloat16>(a, st);
    return heads_launch_t<float>(a, st);
}

}  // namespace medusa
