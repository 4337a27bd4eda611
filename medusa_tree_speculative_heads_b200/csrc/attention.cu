// Tree attention on B200.
//
// Operation ("Medusa Explained: Multi-Head Speculative Decoding Guide",
// section "2. Single-Pass Tree Attention Verification"; "Multi-Token
// Prediction & Draft-Model-Free Speculative Decoding", section "The 2D Tree
// Attention Mask"): every tree node attends to the cached prefix and to the
// tree nodes that are its ancestors or itself.
//
// bf16 path: grouped-query, split-KV attention.  For one (sequence, kv-head)
// the T*G query rows (node-major: row = node * G + q-head-in-group) share
// every K/V element, so a CTA takes a 64-row tile of them and streams K/V
// chunks of 64 keys through shared memory (cp.async double buffering, XOR
// swizzled rows), with QK^T and PV on the tensor cores and an fp32 online
// softmax in registers.  The key range is split across CTAs: prefix splits
// see every key (up to the sequence's prefix length); the last split holds
// the tree's own keys and applies each row's ancestor bitmask.  A combine
// kernel merges the splits by their log-sum-exp.
//
// fp32 path: one warp per query row on the CUDA cores (fp32 end to end).
#include <limits.h>

#include "kernels.h"

namespace medusa {

namespace {

constexpr int kBM = 64;   // query rows per CTA (4 warps x 16)
constexpr int kBN = 64;   // keys per chunk
constexpr int kThreads = 128;

struct AttnParams {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k_tree;  // NULL: the tree's K/V sit in the cache at rows prefix_len .. prefix_len + T_b
    const __nv_bfloat16* v_tree;
    const __nv_bfloat16* k_cache;
    const __nv_bfloat16* v_cache;
    const int32_t* prefix_len;
    int B, T, Hq, Hkv, G, S_max, max_prefix;
    float scale_log2;
    int R;          // query-row stride per (sequence, kv-head) = T * G (T: the largest tree)
    int n_splits;   // prefix splits + 1 (tree split last)
    int split_len;  // prefix keys per split, a multiple of kBN
    TreeRef tree;
    const int32_t* block_table;  // NULL: contiguous caches; else page pools [num_pages, Hkv, page_size, D]
    int max_pages, page_size, num_pages;
    float* part_o;    // [n_splits][B*Hkv][R][D], normalised
    float* part_lse;  // [n_splits][B*Hkv][R], log2 units
    int32_t* status;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D (16x8 f32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// byte offset of 16-byte chunk `ch` of row `row` in a [rows][D] bf16 tile
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int ch) {
    return (uint32_t)(row * D * 2 + ((ch ^ (row & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kThreads) tree_attn_mma_kernel(const __grid_constant__ AttnParams p) {
    constexpr int CH = D / 8;  // 16-byte chunks per row
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* sQ = smem;                                 // [kBM][D]
    uint8_t* sK = sQ + kBM * D * 2;                     // [2][kBN][D]
    uint8_t* sV = sK + 2 * kBN * D * 2;                 // [2][kBN][D]
    uint32_t* sAnc = (uint32_t*)(sV + 2 * kBN * D * 2);  // [kBM][4]

    const int mt = blockIdx.x, bg = blockIdx.y, split = blockIdx.z;
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool tree_split = split == p.n_splits - 1;
    const TreeDev* tree = p.tree.at(b);
    const int Rb = tree->T * p.G;  // this sequence's query rows

    int S = p.prefix_len[b];
    if (S < 0 || S > p.max_prefix) {
        if (tid == 0 && split == 0 && mt == 0 && g == 0) set_status(p.status, MEDUSA_STATUS_BAD_PREFIX);
        S = S < 0 ? 0 : p.max_prefix;
    }
    int k_begin, k_end;
    if (tree_split) {
        k_begin = 0;
        k_end = tree->T;
    } else {
        k_begin = split * p.split_len;
        k_end = min(S, k_begin + p.split_len);
    }
    const int n_keys = max(0, k_end - k_begin);
    const int n_chunks = (n_keys + kBN - 1) / kBN;

    // ---- Q tile and (tree split) ancestor masks ----
    for (int c = tid; c < kBM * CH; c += kThreads) {
        const int row = c / CH, ch = c % CH;
        const int r = mt * kBM + row;
        const bool valid = r < Rb;
        const int node = valid ? r / p.G : 0, hh = valid ? r % p.G : 0;
        const __nv_bfloat16* src = p.q + (((long)b * p.T + node) * p.Hq + g * p.G + hh) * D + ch * 8;
        cp_async16(smem_u32(sQ) + swz<D>(row, ch), src, valid);
    }
    if (tree_split) {
        for (int t = tid; t < kBM * 4; t += kThreads) {
            const int row = t >> 2, w = t & 3;
            const int r = mt * kBM + row;
            sAnc[t] = r < Rb ? tree->anc[r / p.G][w] : 0u;
        }
    }
    auto load_chunk = [&](int chunk, int buf) {
        const int key0 = k_begin + chunk * kBN;
        for (int c = tid; c < kBN * CH; c += kThreads) {
            const int row = c / CH, ch = c % CH;
            const int key = key0 + row;
            bool valid = key < k_end;
            long off;
            const __nv_bfloat16 *ks, *vs;
            if (tree_split && !p.k_tree) {  // the tree's rows follow the prefix in the cache
                off = (((long)b * p.Hkv + g) * p.S_max + S + (valid ? key : 0)) * D + ch * 8;
                ks = p.k_cache + off;
                vs = p.v_cache + off;
            } else if (tree_split) {
                off = (((long)b * p.T + (valid ? key : 0)) * p.Hkv + g) * D + ch * 8;
                ks = p.k_tree + off;
                vs = p.v_tree + off;
            } else if (p.block_table) {
                int page = valid ? __ldg(&p.block_table[(long)b * p.max_pages + key / p.page_size]) : 0;
                if (valid && (page < 0 || page >= p.num_pages)) {
                    if (ch == 0) set_status(p.status, MEDUSA_STATUS_BAD_PAGE);
                    valid = false;
                    page = 0;
                }
                off = (((long)page * p.Hkv + g) * p.page_size + (valid ? key % p.page_size : 0)) * D + ch * 8;
                ks = p.k_cache + off;
                vs = p.v_cache + off;
            } else {
                off = (((long)b * p.Hkv + g) * p.S_max + (valid ? key : 0)) * D + ch * 8;
                ks = p.k_cache + off;
                vs = p.v_cache + off;
            }
            const uint32_t o = swz<D>(row, ch) + buf * kBN * D * 2;
            cp_async16(smem_u32(sK) + o, ks, valid);
            cp_async16(smem_u32(sV) + o, vs, valid);
        }
    };
    if (n_chunks > 0) load_chunk(0, 0);
    cp_async_commit();

    float o_acc[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) o_acc[i][e] = 0.f;
    float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
    uint32_t qf[D / 16][4];

    for (int chunk = 0; chunk < n_chunks; ++chunk) {
        const int buf = chunk & 1;
        if (chunk + 1 < n_chunks) load_chunk(chunk + 1, buf ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (chunk == 0) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int row = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int ch = 2 * kk + (lane >> 4);
                ldmatrix_x4(smem_u32(sQ) + swz<D>(row, ch), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
            }
        }
        // ---- S = Q K^T (16 rows x 64 keys per warp) ----
        float s[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[n][e] = 0.f;
        const uint32_t kbase = smem_u32(sK) + buf * kBN * D * 2;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                const int key = 16 * np + (lane & 7) + (lane >> 4) * 8;
                const int ch = 2 * kk + ((lane >> 3) & 1);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(kbase + swz<D>(key, ch), b0, b1, b2, b3);
                mma_bf16(s[2 * np], qf[kk], b0, b1);
                mma_bf16(s[2 * np + 1], qf[kk], b2, b3);
            }
        }
        // ---- mask, online softmax (log2 domain) ----
        const int key0 = k_begin + chunk * kBN;
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = key0 + n * 8 + (lane & 3) * 2 + (e & 1);
                const int lrow = warp * 16 + (lane >> 2) + (e >> 1) * 8;
                bool ok = key < k_end;
                if (tree_split && ok) ok = (sAnc[lrow * 4 + (key >> 5)] >> (key & 31)) & 1u;
                const float v = ok ? s[n][e] * p.scale_log2 : -INFINITY;
                s[n][e] = v;
                mx[e >> 1] = fmaxf(mx[e >> 1], v);
            }
        float alpha[2], mu[2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            mx[h2] = fmaxf(mx[h2], __shfl_xor_sync(kFull, mx[h2], 1));
            mx[h2] = fmaxf(mx[h2], __shfl_xor_sync(kFull, mx[h2], 2));
            const float mn = fmaxf(m_r[h2], mx[h2]);
            mu[h2] = mn == -INFINITY ? 0.f : mn;
            alpha[h2] = exp2f(m_r[h2] - mu[h2]);
            m_r[h2] = mn;
        }
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float pv = exp2f(s[n][e] - mu[e >> 1]);
                s[n][e] = pv;
                rs[e >> 1] += pv;
            }
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) l_r[h2] = l_r[h2] * alpha[h2] + rs[h2];
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            o_acc[i][0] *= alpha[0];
            o_acc[i][1] *= alpha[0];
            o_acc[i][2] *= alpha[1];
            o_acc[i][3] *= alpha[1];
        }
        // ---- O += P V ----
        const uint32_t vbase = smem_u32(sV) + buf * kBN * D * 2;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
            uint32_t pa[4];
            pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
            pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
            pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
            pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                const int key = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int ch = 2 * dp + (lane >> 4);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(vbase + swz<D>(key, ch), b0, b1, b2, b3);
                mma_bf16(o_acc[2 * dp], pa, b0, b1);
                mma_bf16(o_acc[2 * dp + 1], pa, b2, b3);
            }
        }
        __syncthreads();  // the buffer is refilled by the next prefetch
    }
    cp_async_wait<0>();

    // ---- finalize: normalise and write this split's partial ----
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
        l_r[h2] += __shfl_xor_sync(kFull, l_r[h2], 1);
        l_r[h2] += __shfl_xor_sync(kFull, l_r[h2], 2);
    }
    const long BH = (long)p.B * p.Hkv;
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
        const int r = mt * kBM + warp * 16 + (lane >> 2) + h2 * 8;
        if (r >= Rb) continue;
        const float inv = l_r[h2] > 0.f ? 1.f / l_r[h2] : 0.f;
        float* dst = p.part_o + (((long)split * BH + bg) * p.R + r) * D;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            const int dcol = i * 8 + (lane & 3) * 2;
            *reinterpret_cast<float2*>(dst + dcol) = make_float2(o_acc[i][2 * h2] * inv, o_acc[i][2 * h2 + 1] * inv);
        }
        if ((lane & 3) == 0)
            p.part_lse[((long)split * BH + bg) * p.R + r] = l_r[h2] > 0.f ? m_r[h2] + log2f(l_r[h2]) : -INFINITY;
    }
}

// One warp per output row (b, node, q-head): log-sum-exp merge of the splits.
// Lane s holds split s's log-sum-exp (32 splits at a time), so the row's
// loads are independent of each other.
template <int D>
__global__ void __launch_bounds__(256) attn_combine_kernel(const float* __restrict__ part_o,
                                                           const float* __restrict__ part_lse, int B, int T, int Hq,
                                                           int Hkv, int n_splits, TreeRef tree,
                                                           __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
    const long row = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= (long)B * T * Hq) return;
    const int h = (int)(row % Hq);
    const int i = (int)((row / Hq) % T);
    const int b = (int)(row / ((long)Hq * T));
    const int G = Hq / Hkv, g = h / G, hh = h % G;
    const int R = T * G, r = i * G + hh;
    if (i >= tree.at(b)->T) {  // past this sequence's tree: no partials, zero output
        __nv_bfloat16* dst = out + row * D + lane * (D / 32);
#pragma unroll
        for (int e = 0; e < D / 32; ++e) dst[e] = __float2bfloat16_rn(0.f);
        if (lse && lane == 0) lse[row] = -INFINITY;
        return;
    }
    const long BH = (long)B * Hkv, bg = (long)b * Hkv + g;
    constexpr int PL = D / 32;
    float acc[PL];
#pragma unroll
    for (int e = 0; e < PL; ++e) acc[e] = 0.f;
    float M = -INFINITY, wsum = 0.f;
    for (int s0 = 0; s0 < n_splits; s0 += 32) {
        const int s = s0 + lane;
        const float ls = s < n_splits ? __ldg(&part_lse[((long)s * BH + bg) * R + r]) : -INFINITY;
        float m2 = ls;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m2 = fmaxf(m2, __shfl_xor_sync(kFull, m2, o));
        if (m2 == -INFINITY) continue;
        const float Mn = fmaxf(M, m2);
        const float rescale = M == -INFINITY ? 0.f : exp2f(M - Mn);
        wsum *= rescale;
#pragma unroll
        for (int e = 0; e < PL; ++e) acc[e] *= rescale;
        M = Mn;
        const float w = ls == -INFINITY ? 0.f : exp2f(ls - M);
        const int cnt = min(32, n_splits - s0);
        for (int t0 = 0; t0 < cnt; t0 += 8) {  // 8 splits' loads in flight at once
            float vals[8][PL];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float* src = part_o + (((long)(s0 + t0 + u) * BH + bg) * R + r) * D + lane * PL;
#pragma unroll
                for (int e = 0; e < PL; ++e) vals[u][e] = t0 + u < cnt ? __ldg(&src[e]) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float wt = __shfl_sync(kFull, w, (t0 + u) & 31);
                if (t0 + u < cnt) {
                    wsum += wt;
#pragma unroll
                    for (int e = 0; e < PL; ++e) acc[e] += wt * vals[u][e];
                }
            }
        }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    __nv_bfloat16* dst = out + row * D + lane * PL;
#pragma unroll
    for (int e = 0; e < PL; ++e) dst[e] = __float2bfloat16_rn(acc[e] * inv);
    if (lse && lane == 0) lse[row] = wsum > 0.f ? (M + log2f(wsum)) * 0.69314718055994531f : -INFINITY;
}

// fp32 path: one warp per query row, keys in order (prefix, then the visible
// tree nodes), online softmax with expf.
template <int D>
__global__ void __launch_bounds__(256) tree_attn_f32_kernel(const float* __restrict__ q, const float* __restrict__ k_tree,
                                                            const float* __restrict__ v_tree,
                                                            const float* __restrict__ k_cache,
                                                            const float* __restrict__ v_cache,
                                                            const int32_t* __restrict__ prefix_len, int B, int T,
                                                            int Hq, int Hkv, int S_max, int max_prefix, float scale,
                                                            const int32_t* __restrict__ table, int max_pages,
                                                            int page_size, int num_pages, TreeRef trees,
                                                            float* __restrict__ out,
                                                            float* __restrict__ lse, int32_t* status) {
    constexpr int PL = D / 32;
    const long row = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= (long)B * T * Hq) return;
    const int h = (int)(row % Hq);
    const int i = (int)((row / Hq) % T);
    const int b = (int)(row / ((long)Hq * T));
    const int g = h / (Hq / Hkv);
    const TreeDev* tree = trees.at(b);
    if (i >= tree->T) {  // past this sequence's tree: zero output
#pragma unroll
        for (int e = 0; e < PL; ++e) out[row * D + lane * PL + e] = 0.f;
        if (lse && lane == 0) lse[row] = -INFINITY;
        return;
    }
    int S = prefix_len[b];
    if (S < 0 || S > max_prefix) {
        if (lane == 0 && i == 0 && h == 0) set_status(status, MEDUSA_STATUS_BAD_PREFIX);
        S = S < 0 ? 0 : max_prefix;
    }
    float qv[PL], o[PL];
#pragma unroll
    for (int e = 0; e < PL; ++e) {
        qv[e] = q[row * D + lane * PL + e];
        o[e] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    auto visit = [&](const float* kp, const float* vp) {
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < PL; ++e) d = fmaf(qv[e], kp[lane * PL + e], d);
        const float sc = warp_sum(d) * scale;
        const float mn = fmaxf(m, sc);
        const float a = m == -INFINITY ? 0.f : expf(m - mn);
        const float w = expf(sc - mn);
        l = l * a + w;
#pragma unroll
        for (int e = 0; e < PL; ++e) o[e] = o[e] * a + w * vp[lane * PL + e];
        m = mn;
    };
    // prefix keys in order, their K/V rows loaded 8 at a time ahead of use
    // (the same per-key arithmetic as visit(), so the same result)
    constexpr int kU = 8;
    const long cbase = ((long)b * Hkv + g) * S_max;
    for (int j0 = 0; j0 < S; j0 += kU) {
        float kr[kU][PL], vr[kU][PL];
        bool have[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int j = j0 + u;
            long row = -1;
            if (j < S) {
                if (table) {
                    const int page = table[(long)b * max_pages + j / page_size];
                    if (page >= 0 && page < num_pages) row = ((long)page * Hkv + g) * page_size + j % page_size;
                    else if (lane == 0) set_status(status, MEDUSA_STATUS_BAD_PAGE);
                } else {
                    row = cbase + j;
                }
            }
            have[u] = row >= 0;
#pragma unroll
            for (int e = 0; e < PL; ++e) {
                kr[u][e] = have[u] ? k_cache[row * D + lane * PL + e] : 0.f;
                vr[u][e] = have[u] ? v_cache[row * D + lane * PL + e] : 0.f;
            }
        }
        float sc[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            float d = 0.f;
#pragma unroll
            for (int e = 0; e < PL; ++e) d = fmaf(qv[e], kr[u][e], d);
            sc[u] = warp_sum(d) * scale;
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            if (!have[u]) continue;
            const float mn = fmaxf(m, sc[u]);
            const float a = m == -INFINITY ? 0.f : expf(m - mn);
            const float w = expf(sc[u] - mn);
            l = l * a + w;
#pragma unroll
            for (int e = 0; e < PL; ++e) o[e] = o[e] * a + w * vr[u][e];
            m = mn;
        }
    }
    for (int j = 0; j < tree->T; ++j) {
        if (!((tree->anc[i][j >> 5] >> (j & 31)) & 1u)) continue;
        if (k_tree) {
            visit(k_tree + (((long)b * T + j) * Hkv + g) * D, v_tree + (((long)b * T + j) * Hkv + g) * D);
        } else {  // the tree's rows follow the prefix in the (contiguous) cache
            const long r = ((long)b * Hkv + g) * S_max + S + j;
            visit(k_cache + r * D, v_cache + r * D);
        }
    }
#pragma unroll
    for (int e = 0; e < PL; ++e) out[row * D + lane * PL + e] = o[e] / l;
    if (lse && lane == 0) lse[row] = m + logf(l);
}

struct SplitPlan {
    int m_tiles, n_splits, split_len;
};

// Key splits so that the grid fills the GPU: tile_rows query rows per CTA,
// `waves` CTAs per SM targeted.
SplitPlan plan_splits(int B, int T, int Hq, int Hkv, int max_prefix, int tile_rows = kBM, int waves = 2) {
    SplitPlan sp;
    const int R = T * (Hq / Hkv);
    sp.m_tiles = (R + tile_rows - 1) / tile_rows;
    const long per_split = (long)sp.m_tiles * B * Hkv;
    const long target = (long)waves * num_sms();
    int nps = 0;
    sp.split_len = kBN;
    if (max_prefix > 0) {
        long want = (target + per_split - 1) / per_split - 1;
        const int max_nps = (max_prefix + kBN - 1) / kBN;
        if (want < 1) want = 1;
        if (want > max_nps) want = max_nps;
        int len = (int)((max_prefix + want - 1) / want);
        len = (len + kBN - 1) / kBN * kBN;
        sp.split_len = len;
        nps = (max_prefix + len - 1) / len;
    }
    sp.n_splits = nps + 1;
    return sp;
}

// the tensor-core kernel runs these shapes (and page sizes, when paged)
bool use_tc(const AttnArgs& a, int D) {
    return attn_tc_supported(a.Hq, a.Hkv, D, a.T, a.dt) && (!a.block_table || attn_tc_page_ok(a.page_size));
}

SplitPlan plan_bf16(int B, int T, int Hq, int Hkv, int max_prefix) {
    return plan_splits(B, T, Hq, Hkv, max_prefix);
}

template <int D>
cudaError_t attn_launch_bf16(const AttnArgs& a, cudaStream_t st) {
    const bool tc = use_tc(a, D);
    SplitPlan sp = plan_bf16(a.B, a.T, a.Hq, a.Hkv, a.max_prefix);
    AttnParams p;
    p.q = (const __nv_bfloat16*)a.q;
    p.k_tree = (const __nv_bfloat16*)a.k_tree;
    p.v_tree = (const __nv_bfloat16*)a.v_tree;
    p.k_cache = (const __nv_bfloat16*)a.k_cache;
    p.v_cache = (const __nv_bfloat16*)a.v_cache;
    p.prefix_len = a.prefix_len;
    p.B = a.B;
    p.T = a.T;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.G = a.Hq / a.Hkv;
    p.S_max = a.S_max;
    p.max_prefix = a.max_prefix;
    const float scale = a.scale > 0.f ? a.scale : 1.f / sqrtf((float)D);
    p.scale_log2 = scale * 1.4426950408889634f;
    p.R = a.T * p.G;
    p.n_splits = sp.n_splits;
    p.split_len = sp.split_len;
    p.tree = a.tree;
    p.block_table = a.block_table;
    p.max_pages = a.max_pages;
    p.page_size = a.page_size;
    p.num_pages = a.num_pages;
    const long BH = (long)a.B * a.Hkv;
    p.part_o = (float*)a.ws;
    p.part_lse = (float*)((char*)a.ws + align256((size_t)sp.n_splits * BH * p.R * D * sizeof(float)));
    p.status = a.status;
    if (tc) {
        // 128-row tiles; the key splits of a tile merge inside their cluster
        const int m_tiles = (a.T * p.G + 127) / 128;
        return attn_tc_launch(a, m_tiles, attn_tc_splits(a.B, a.T, a.Hq, a.Hkv, a.max_prefix), p.scale_log2, st);
    }
    {
        const size_t smem = (size_t)kBM * D * 2 + 4 * (size_t)kBN * D * 2 + kBM * 4 * sizeof(uint32_t);
        cudaFuncSetAttribute(tree_attn_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        dim3 grid(sp.m_tiles, (unsigned)BH, sp.n_splits);
        tree_attn_mma_kernel<D><<<grid, kThreads, smem, st>>>(p);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const long rows = (long)a.B * a.T * a.Hq;
    prefer_max_smem(attn_combine_kernel<D>);
    attn_combine_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(p.part_o, p.part_lse, a.B, a.T, a.Hq, a.Hkv,
                                                                     sp.n_splits, a.tree, (__nv_bfloat16*)a.out, a.lse);
    return cudaGetLastError();
}

template <int D>
cudaError_t attn_launch_f32(const AttnArgs& a, cudaStream_t st) {
    const long rows = (long)a.B * a.T * a.Hq;
    const float scale = a.scale > 0.f ? a.scale : 1.f / sqrtf((float)D);
    tree_attn_f32_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
        (const float*)a.q, (const float*)a.k_tree, (const float*)a.v_tree, (const float*)a.k_cache,
        (const float*)a.v_cache, a.prefix_len, a.B, a.T, a.Hq, a.Hkv, a.S_max, a.max_prefix, scale, a.block_table,
        a.max_pages, a.page_size, a.num_pages, a.tree,
        (float*)a.out, a.lse, a.status);
    return cudaGetLastError();
}

}  // namespace

size_t attn_workspace_size(int B, int T, int Hq, int Hkv, int D, int max_prefix, medusa_dtype dt) {
    if (dt != MEDUSA_BF16) return 0;
    // the mma.sync kernel's split partials (the tensor-core kernel needs none,
    // but a paged call may run either kernel, by page size)
    const SplitPlan a = plan_bf16(B, T, Hq, Hkv, max_prefix);
    const size_t splits = a.n_splits;
    const size_t R = (size_t)T * (Hq / Hkv);
    const size_t BH = (size_t)B * Hkv;
    return align256(splits * BH * R * D * sizeof(float)) + align256(splits * BH * R * sizeof(float));
}

cudaError_t attn_launch(const AttnArgs& a, cudaStream_t st) {
    if (a.dt == MEDUSA_BF16) return a.D == 128 ? attn_launch_bf16<128>(a, st) : attn_launch_bf16<64>(a, st);
    return a.D == 128 ? attn_launch_f32<128>(a, st) : attn_launch_f32<64>(a, st);
}

}  // namespace medusa
