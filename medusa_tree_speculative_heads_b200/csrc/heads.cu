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

#include "heads_common.cuh"
#include "kernels.h"

namespace medusa {

namespace {

constexpr int kResWarps = 8;   // warps per block of the residual kernel
constexpr int kLmWarps = 8;    // warps per block of the LM-head kernel
constexpr int kBG = 8;         // sequences handled per LM-head launch
constexpr int kUnroll = 8;     // 16-byte loads issued back to back per lane

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
// Fused heads for one sequence (rows of <= 8 KB): a persistent cooperative
// kernel, one CTA per SM, that runs the whole medusa_heads call.
//   - A producer thread streams contiguous chunks of weight rows into a ring
//     of kFStages shared-memory stages with bulk asynchronous copies (192 KB
//     in flight per SM, independent of register pressure): first the CTA's
//     slice of W_res rows, then, without a break, its slice of W_head rows.
//   - kFC consumer warps dot each row with the vector held in registers:
//     phase 1 writes h^(k) = SiLU(W_res h) + h; after a grid-wide barrier
//     (all of h^(k) written; the producer keeps prefetching W_head meanwhile)
//     phase 2 computes logits and keeps running softmax statistics and a
//     top-8 list per head.
//   - Each CTA merges its warps into one partial per head; the last CTA to
//     finish merges all partials (in CTA order) and fills the tree.
// Every wait -- ring barriers and the grid barrier -- gives up after ~2 s and
// sets MEDUSA_STATUS_TIMEOUT instead of hanging.
// ---------------------------------------------------------------------------
#ifndef MEDUSA_FC
#define MEDUSA_FC 6
#endif
#ifndef MEDUSA_FSTAGES
#define MEDUSA_FSTAGES 4
#endif
constexpr int kFC = MEDUSA_FC;           // consumer warps (+1 producer warp)
constexpr int kFStages = MEDUSA_FSTAGES; // ring depth
constexpr int kRowCap = 8192;    // largest weight row (bytes) the fused kernel takes

struct FusedArgs {
    const void* h;
    const void* W_res;
    const void* W_head;
    int d, V, K;
    void* hk;
    void* hk_out;
    float* logits;
    HeadState* part;     // [grid][K][kBG]
    unsigned int* ctr;   // [2], zero at launch: grid-barrier arrivals, CTAs done
    TreeRef tree;
    const int32_t* root_token;
    int32_t* topk_idx;
    float* topk_prob;
    int32_t* node_tokens;
    float* node_q;
    float2* stats;
    int32_t* status;
};

size_t fused_smem_bytes(int row_bytes, int K) {
    const int rpw = kRowCap / row_bytes;
    return (size_t)kFStages * kFC * rpw * row_bytes + 2 * kFStages * sizeof(uint64_t) +
           (size_t)kFC * K * sizeof(HeadState) + 16;
}

__device__ __forceinline__ uint4 ld_cg(const void* p) {
    uint4 r;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"r"(kFC * 32) : "memory"); }

template <typename T>
__global__ void __launch_bounds__((kFC + 1) * 32, 1) heads_fused_kernel(const __grid_constant__ FusedArgs a) {
    constexpr int VEC = Elt<T>::kVec;
    constexpr int NXV = kRowCap / 16 / 32;  // 16-byte pieces of a row per lane
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_flag;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int row_bytes = a.d * (int)sizeof(T);
    const int nvec = a.d / VEC;
    const int rpw = kRowCap / row_bytes;
    const int srows = kFC * rpw;
    const int stage_bytes = srows * row_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kFStages * stage_bytes);
    uint64_t* empty = full + kFStages;
    HeadState* sstate = reinterpret_cast<HeadState*>(empty + kFStages);  // [kFC][K]
    const long R1 = (long)a.K * a.d, R2 = (long)a.K * a.V;
    const long a0 = R1 * blockIdx.x / gridDim.x, a1 = R1 * (blockIdx.x + 1) / gridDim.x;
    const long b0 = R2 * blockIdx.x / gridDim.x, b1 = R2 * (blockIdx.x + 1) / gridDim.x;
    const int n1 = (int)((a1 - a0 + srows - 1) / srows);
    const int n2 = (int)((b1 - b0 + srows - 1) / srows);

    if (threadIdx.x == 0) {
        for (int st = 0; st < kFStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], kFC);
        }
        mbar_fence_init();
        s_flag = 0;
    }
    for (int t = threadIdx.x; t < kFC * a.K; t += blockDim.x) sstate[t] = empty_state();
    sync_block();

    if (warp == kFC) {
        // ---------------- producer ----------------
        if (lane == 0) {
            int issued = 0;
            for (int it = 0; it < n1 + n2; ++it) {
                const int st = it % kFStages;
                if (it >= kFStages && !mbar_wait(&empty[st], ((it / kFStages) - 1) & 1)) {
                    set_status(a.status, MEDUSA_STATUS_TIMEOUT);
                    break;
                }
                long row0, nr;
                const uint8_t* src;
                if (it < n1) {
                    row0 = a0 + (long)it * srows;
                    nr = min((long)srows, a1 - row0);
                    src = (const uint8_t*)a.W_res;
                } else {
                    row0 = b0 + (long)(it - n1) * srows;
                    nr = min((long)srows, b1 - row0);
                    src = (const uint8_t*)a.W_head;
                }
                const uint32_t bytes = (uint32_t)(nr * row_bytes);
                mbar_arrive_expect_tx(&full[st], bytes);
                bulk_g2s(smem + st * stage_bytes, src + row0 * row_bytes, bytes, &full[st]);
                ++issued;
            }
            for (int st = 0; st < kFStages && st < issued; ++st) {  // drain before exit
                const int last = st + ((issued - 1 - st) / kFStages) * kFStages;
                mbar_wait(&full[st], (last / kFStages) & 1);
            }
        }
    } else {
        // ---------------- consumers ----------------
        uint4 xr[NXV];
        auto load_x = [&](const T* src, bool written_here) {
#pragma unroll
            for (int j = 0; j < NXV; ++j) {
                const int c = j * 32 + lane;
                xr[j] = c >= nvec ? make_uint4(0, 0, 0, 0) : written_here ? ld_cg(src + (long)c * VEC)
                                                                           : ld_nc(src + (long)c * VEC);
            }
        };
        auto dot = [&](const uint8_t* rowp) {
            const uint4* row = reinterpret_cast<const uint4*>(rowp);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < NXV; ++j) {
                const int c = j * 32 + lane;
                if (c < nvec) {
                    float wf[VEC], xf[VEC];
                    Elt<T>::unpack(row[c], wf);
                    Elt<T>::unpack(xr[j], xf);
#pragma unroll
                    for (int e = 0; e < VEC; ++e) acc[j & 3] = fmaf(wf[e], xf[e], acc[j & 3]);
                }
            }
            return warp_sum((acc[0] + acc[1]) + (acc[2] + acc[3]));
        };
        // ok: results are valid so far; dead: a ring wait expired, so this warp
        // stops consuming (and releasing) stages -- the producer's own bounded
        // wait then ends the stream and it drains its copies.
        bool ok = true, dead = false;
        // phase 1: h^(k) rows
        load_x((const T*)a.h, false);
        int it = 0;
        for (; it < n1 && !dead; ++it) {
            const int st = it % kFStages;
            if (!mbar_wait(&full[st], (it / kFStages) & 1)) {
                if (lane == 0) set_status(a.status, MEDUSA_STATUS_TIMEOUT);
                ok = false;
                dead = true;
                break;
            }
            {
                const uint8_t* stage = smem + st * stage_bytes;
                for (int j = 0; j < rpw; ++j) {
                    const int lr = j * kFC + warp;
                    const long r = a0 + (long)it * srows + lr;
                    if (r >= a1) break;
                    const int o = (int)(r % a.d);
                    const float hres = Elt<T>::to_float(((const T*)a.h)[o]);
                    const float z = dot(stage + lr * row_bytes);
                    if (lane == 0) {
                        const T y = Elt<T>::from_float(z / (1.f + expf(-z)) + hres);
                        ((T*)a.hk)[r] = y;
                        if (a.hk_out) ((T*)a.hk_out)[r] = y;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        // grid barrier: every CTA's h^(k) rows are written before any is read
        consumers_sync();
        if (warp == 0 && lane == 0) {
            __threadfence();
            atomicAdd(&a.ctr[0], 1u);
            const uint64_t t0 = global_ns();
            while (ld_acquire_u32(&a.ctr[0]) < gridDim.x) {
                if (global_ns() - t0 > 2000000000ull) {
                    set_status(a.status, MEDUSA_STATUS_TIMEOUT);
                    s_flag = 1;
                    break;
                }
                __nanosleep(64);
            }
            __threadfence();
        }
        consumers_sync();
        if (s_flag) ok = false;
        // phase 2: logits, softmax statistics and top-8 per head
        float m = -INFINITY, l = 0.f, tv = -INFINITY;
        int ti = INT_MAX, cur_k = -1;
        auto flush = [&](int kk) {
            HeadState* sp = &sstate[warp * a.K + kk];
            if (lane < kTopK) {
                sp->val[lane] = tv;
                sp->idx[lane] = ti;
            }
            if (lane == 0) {
                sp->m = m;
                sp->l = l;
            }
            m = -INFINITY;
            l = 0.f;
            tv = -INFINITY;
            ti = INT_MAX;
        };
        for (it = n1; it < n1 + n2 && !dead; ++it) {
            const int st = it % kFStages;
            if (!mbar_wait(&full[st], (it / kFStages) & 1)) {
                if (lane == 0) set_status(a.status, MEDUSA_STATUS_TIMEOUT);
                ok = false;
                dead = true;
                break;
            }
            if (ok) {
                const uint8_t* stage = smem + st * stage_bytes;
                for (int j = 0; j < rpw; ++j) {
                    const int lr = j * kFC + warp;
                    const long r = b0 + (long)(it - n1) * srows + lr;
                    if (r >= b1) break;
                    const int k = (int)(r / a.V);
                    const int v = (int)(r - (long)k * a.V);
                    if (k != cur_k) {
                        if (cur_k >= 0) flush(cur_k);
                        cur_k = k;
                        load_x((const T*)a.hk + (long)k * a.d, true);
                    }
                    const float z = dot(stage + lr * row_bytes);
                    if (a.logits && lane == 0) a.logits[r] = z;
                    if (z > -INFINITY || z != z) {
                        const float mn = fmaxf(m, z);
                        l = (m == -INFINITY ? 0.f : l * expf(m - mn)) + expf(z - mn);
                        m = mn;
                    }
                    const unsigned mask = __ballot_sync(kFull, lane < kTopK && beats(z, v, tv, ti));
                    if (mask) {
                        const int pos = __ffs(mask) - 1;
                        const float pv = __shfl_up_sync(kFull, tv, 1);
                        const int pi = __shfl_up_sync(kFull, ti, 1);
                        if (lane == pos) {
                            tv = z;
                            ti = v;
                        } else if (lane > pos && lane < kTopK) {
                            tv = pv;
                            ti = pi;
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        if (cur_k >= 0) flush(cur_k);
    }
    sync_block();

    // this CTA's partial per head it covered
    if (warp < kFC && b1 > b0) {
        const int k_lo = (int)(b0 / a.V), k_hi = (int)((b1 - 1) / a.V);
        for (int k = k_lo + warp; k <= k_hi; k += kFC) {
            float mm = -INFINITY, ll = 0.f;
            if (lane < kFC) {
                mm = sstate[lane * a.K + k].m;
                ll = sstate[lane * a.K + k].l;
            }
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                const float m2 = __shfl_xor_sync(kFull, mm, o);
                const float l2 = __shfl_xor_sync(kFull, ll, o);
                merge_ml(mm, ll, m2, l2);
            }
            float lv[kTopK];
            int li[kTopK];
#pragma unroll
            for (int j = 0; j < kTopK; ++j) {
                lv[j] = -INFINITY;
                li[j] = INT_MAX;
            }
            if ((lane >> 2) < kFC) {  // lane j takes entries 2(j%4), 2(j%4)+1 of warp j/4
                const HeadState* sp = &sstate[(lane >> 2) * a.K + k];
                const int e = (lane & 3) * 2;
                list_insert(lv, li, sp->val[e], sp->idx[e]);
                list_insert(lv, li, sp->val[e + 1], sp->idx[e + 1]);
            }
            float ov;
            int oi;
            warp_select(lv, li, ov, oi);
            HeadState* dst = &a.part[((long)blockIdx.x * a.K + k) * kBG];
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
    // the last CTA to finish merges every head
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_flag = atomicAdd(&a.ctr[1], 1u) == gridDim.x - 1;
    sync_block();
    if (!s_flag) return;
    __threadfence();
    for (int k = warp; k < a.K; k += kFC + 1)
        merge_head(a.part, gridDim.x, a.V, 1, kBG, 0, 0, a.V, a.K, k, a.tree.base ? a.tree.at(0) : nullptr, a.tree.T,
                   a.root_token, a.topk_idx, a.topk_prob,
                   a.node_tokens, a.node_q, a.stats, a.status);
}

// K3 of the general path: one warp per (sequence, head).
__global__ void __launch_bounds__(32) heads_merge_kernel(const HeadState* __restrict__ part, int nparts, int b0,
                                                         int nb, int V, int K, TreeRef tree,
                                                         const int32_t* __restrict__ root_token,
                                                         int32_t* __restrict__ topk_idx,
                                                         float* __restrict__ topk_prob,
                                                         int32_t* __restrict__ node_tokens,
                                                         float* __restrict__ node_q, float2* __restrict__ stats,
                                                         int32_t* status) {
    const int bb = blockIdx.x % nb, k = blockIdx.x / nb;
    merge_head(part, nparts, V, 1, kBG, bb, b0 + bb, V, K, k, tree.base ? tree.at(b0 + bb) : nullptr, tree.T,
               root_token, topk_idx, topk_prob, node_tokens, node_q,
               stats, status);
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
    size_t hk, part, stats, ctr, slots, logits, total;
};

HeadsWs heads_ws_layout(int B, int d, int V, int K, medusa_dtype dt) {
    HeadsWs w;
    size_t esz = dt == MEDUSA_BF16 ? 2 : 4;
    w.hk = 0;
    w.part = w.hk + align256((size_t)B * K * d * esz);
    const int bstride = B > kBG ? (B < 64 ? B : 64) : kBG;  // tensor-core path keeps one partial per sequence
    w.stats = w.part + align256((size_t)lm_grid_bound() * K * bstride * sizeof(HeadState));
    w.ctr = w.stats + align256((size_t)B * K * sizeof(float2));
    // counters, and on the tensor-core path one hand-over flag per CTA and
    // phase plus the handed-over partial tiles ([2][grid][B][128] fp32)
    w.slots = w.ctr + align256((size_t)(2 + 2 * num_sms() + K) * sizeof(unsigned int));
    const size_t slots = heads_tc_supported(B, d, dt) ? (size_t)2 * num_sms() * B * 128 * sizeof(float) : 0;
    w.logits = w.slots + align256(slots);
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

    const int row_bytes = a.d * (int)sizeof(T);
    cudaError_t e;
    if (heads_tc_supported(a.B, a.d, a.dt)) {
        // bf16: weight streaming on the tensor cores (one cooperative kernel)
        e = heads_tc_launch(a, hk, part, (unsigned int*)(ws + w.ctr), (float*)(ws + w.slots), stats, logits, st);
        if (e != cudaSuccess) return e;
        if (a.probs_out) {
            const long n = (long)a.B * a.K * a.V;
            int pg = (int)((n + 255) / 256);
            if (pg > num_sms() * 8) pg = num_sms() * 8;
            heads_probs_kernel<<<pg, 256, 0, st>>>(logits, stats, a.B, a.K, a.V, a.probs_out);
            e = cudaGetLastError();
        }
        return e;
    }
    if (a.B == 1 && row_bytes <= kRowCap && row_bytes % 16 == 0) {
        // one sequence: the whole call is one cooperative persistent kernel
        const size_t smem = fused_smem_bytes(row_bytes, a.K);
        auto kern = heads_fused_kernel<T>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        int occ = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, (kFC + 1) * 32, smem);
        if (occ >= 1) {
            unsigned int* ctr = (unsigned int*)(ws + w.ctr);
            if ((e = cudaMemsetAsync(ctr, 0, 2 * sizeof(unsigned int), st)) != cudaSuccess) return e;
            FusedArgs fa;
            fa.h = a.h;
            fa.W_res = a.W_res;
            fa.W_head = a.W_head;
            fa.d = a.d;
            fa.V = a.V;
            fa.K = a.K;
            fa.hk = hk;
            fa.hk_out = a.h_res_out;
            fa.logits = logits;
            fa.part = part;
            fa.ctr = ctr;
            fa.tree = a.tree;
            fa.root_token = a.root_token;
            fa.topk_idx = a.topk_idx;
            fa.topk_prob = a.topk_prob;
            fa.node_tokens = a.node_tokens;
            fa.node_q = a.node_q;
            fa.stats = stats;
            fa.status = a.status;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(num_sms());  // one CTA per SM, all resident (cooperative)
            cfg.blockDim = dim3((kFC + 1) * 32);
            cfg.dynamicSmemBytes = smem;
            cfg.stream = st;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeCooperative;
            attr[0].val.cooperative = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if ((e = cudaLaunchKernelEx(&cfg, kern, fa)) != cudaSuccess) return e;
            if (a.probs_out) {
                const long n = (long)a.K * a.V;
                int pg = (int)((n + 255) / 256);
                if (pg > num_sms() * 8) pg = num_sms() * 8;
                heads_probs_kernel<<<pg, 256, 0, st>>>(logits, stats, 1, a.K, a.V, a.probs_out);
                e = cudaGetLastError();
            }
            return e;
        }
    }

    const long rows = (long)a.K * a.d;
    heads_res_kernel<T><<<(unsigned)((rows + kResWarps - 1) / kResWarps), kResWarps * 32, 0, st>>>(
        (const T*)a.h, (const T*)a.W_res, a.B, a.d, a.K, hk, (T*)a.h_res_out);
    e = cudaGetLastError();
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

// ---------------------------------------------------------------------------
// Vocabulary-sharded heads: each shard's (m, l, top-8) per (sequence, head)
// with global token ids, and the merge of the shards' partials.
// ---------------------------------------------------------------------------

// one warp per (sequence, head): the shard's statistics and its top-8 logits
// (read back from the shard's logits at the top-8 ids), ids offset to the
// full vocabulary
__global__ void __launch_bounds__(32) heads_pack_shard_kernel(const float2* __restrict__ stats,
                                                              const int32_t* __restrict__ topk_idx,
                                                              const float* __restrict__ logits, int BK, int V,
                                                              int v_offset, HeadState* __restrict__ out) {
    const int p = blockIdx.x, lane = threadIdx.x;
    if (p >= BK) return;
    if (lane < kTopK) {
        const int i = topk_idx[(long)p * kTopK + lane];
        out[p].val[lane] = i >= 0 ? logits[(long)p * V + i] : -INFINITY;
        out[p].idx[lane] = i >= 0 ? i + v_offset : INT_MAX;
    }
    if (lane == 0) {
        const float2 s = stats[p];
        out[p].m = s.x;
        out[p].l = s.y;
    }
}

// one warp per (sequence, head): the shards' partials merged in shard order
// (lane r takes shards r, r + 32, ...; the lanes' statistics are then merged
// by a butterfly and their lists by a warp selection), then the head's
// top-8 entries, their probabilities exp(logit - M) / L, and the tree nodes
// this head proposes, as in the unsharded merge
__global__ void __launch_bounds__(32) heads_merge_shards_kernel(const HeadState* __restrict__ parts, int n_shards,
                                                                int B, int K, int V_total, TreeRef trees,
                                                                const int32_t* __restrict__ root_token,
                                                                int32_t* __restrict__ topk_idx,
                                                                float* __restrict__ topk_prob,
                                                                int32_t* __restrict__ node_tokens,
                                                                float* __restrict__ node_q, int32_t* status) {
    const int b = blockIdx.x % B, k = blockIdx.x / B, lane = threadIdx.x;
    float mm = -INFINITY, ll = 0.f;
    float lv[kTopK];
    int li[kTopK];
#pragma unroll
    for (int j = 0; j < kTopK; ++j) {
        lv[j] = -INFINITY;
        li[j] = INT_MAX;
    }
    for (int r = lane; r < n_shards; r += 32) {
        const HeadState* s = &parts[((long)r * B + b) * K + k];
        merge_ml(mm, ll, s->m, s->l);
#pragma unroll
        for (int j = 0; j < kTopK; ++j) list_insert(lv, li, s->val[j], s->idx[j]);
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
    if (lane < kTopK) {
        topk_idx[((long)b * K + k) * kTopK + lane] = valid ? oi : -1;
        topk_prob[((long)b * K + k) * kTopK + lane] = prob;
    }
    if (!trees.base) return;
    const TreeDev* tree = trees.at(b);
    const int T = tree->T, Tn = trees.T;
    // every lane takes the (token, prob) of each rank from the lane holding it
    int tok_r[kTopK];
    float q_r[kTopK];
#pragma unroll
    for (int j = 0; j < kTopK; ++j) {
        tok_r[j] = __shfl_sync(kFull, valid ? oi : -1, j);
        q_r[j] = __shfl_sync(kFull, prob, j);
    }
    for (int i = lane; i < Tn; i += 32) {
        if (i > 0 && i < T && tree->depth[i] == k + 2) {
            int tok = -1;
            float pq = 0.f;
#pragma unroll
            for (int j = 0; j < kTopK; ++j)
                if (j == tree->rank[i]) {
                    tok = tok_r[j];
                    pq = q_r[j];
                }
            node_tokens[(long)b * Tn + i] = tok;
            if (node_q) node_q[(long)b * Tn + i] = pq;
            if (tok < 0) set_status(status, MEDUSA_STATUS_BAD_TOKEN);
        }
        if (k == 0 && i >= T) {  // rows past this sequence's own tree
            node_tokens[(long)b * Tn + i] = -1;
            if (node_q) node_q[(long)b * Tn + i] = 0.f;
        }
    }
    if (k == 0 && lane == 0) {
        const int rt = root_token[b];
        node_tokens[(long)b * Tn] = rt;
        if (node_q) node_q[(long)b * Tn] = 1.f;
        if (rt < 0 || rt >= V_total) set_status(status, MEDUSA_STATUS_BAD_TOKEN);
    }
}

}  // namespace

size_t heads_workspace_size(int B, int d, int V, int K, medusa_dtype dt) {
    return heads_ws_layout(B, d, V, K, dt).total;
}

cudaError_t heads_launch(const HeadsArgs& a, cudaStream_t st) {
    if (a.dt == MEDUSA_BF16) return heads_launch_t<__nv_bfloat16>(a, st);
    return heads_launch_t<float>(a, st);
}

size_t heads_shard_workspace_size(int B, int d, int V_shard, int K, medusa_dtype dt) {
    return heads_ws_layout(B, d, V_shard, K, dt).total + align256((size_t)B * K * kTopK * 8);
}

cudaError_t heads_shard_launch(const HeadsArgs& x, int v_offset, void* partial_out, cudaStream_t st) {
    const HeadsWs w = heads_ws_layout(x.B, x.d, x.V, x.K, x.dt);
    char* ws = (char*)x.ws;
    HeadsArgs a = x;
    a.tree = TreeRef{nullptr, 0, 0};
    a.T = 0;
    a.root_token = nullptr;
    a.node_tokens = nullptr;
    a.node_q = nullptr;
    a.h_res_out = nullptr;
    a.probs_out = nullptr;
    a.logits_out = (float*)(ws + w.logits);  // the shard's logits, for the top-8 values
    a.topk_idx = (int32_t*)(ws + w.total);
    a.topk_prob = (float*)(ws + w.total + (size_t)x.B * x.K * kTopK * 4);
    cudaError_t e = heads_launch(a, st);
    if (e != cudaSuccess) return e;
    const int BK = x.B * x.K;
    heads_pack_shard_kernel<<<BK, 32, 0, st>>>((const float2*)(ws + w.stats), a.topk_idx, a.logits_out, BK, x.V,
                                               v_offset, (HeadState*)partial_out);
    return cudaGetLastError();
}

cudaError_t heads_merge_shards_launch(const void* parts, int n_shards, int B, int K, int V_total, TreeRef tree,
                                      const int32_t* root_token, int32_t* topk_idx, float* topk_prob,
                                      int32_t* node_tokens, float* node_q, int32_t* status, cudaStream_t st) {
    heads_merge_shards_kernel<<<B * K, 32, 0, st>>>((const HeadState*)parts, n_shards, B, K, V_total, tree,
                                                    root_token, topk_idx, topk_prob, node_tokens, node_q, status);
    return cudaGetLastError();
}

}  // namespace medusa
