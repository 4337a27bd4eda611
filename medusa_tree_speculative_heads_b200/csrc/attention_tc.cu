// Tree attention on the 5th-generation tensor cores (bf16, head_dim 64/128,
// a power-of-two number of q-heads per kv-head).
//
// Operation ("Medusa Explained: Multi-Head Speculative Decoding Guide",
// section "2. Single-Pass Tree Attention Verification"; "Multi-Token
// Prediction & Draft-Model-Free Speculative Decoding", section "The 2D Tree
// Attention Mask"): every tree node attends to the cached prefix and to its
// ancestors and itself.
//
// One CTA takes 128 query rows of one (sequence, kv-head) -- rows are
// node-major, row = node * G + (q-head within the group), so the G q-heads
// of a node share every K/V element -- and a run of 64-key chunks.  A
// sequence's chunks are its prefix chunks followed by its tree's one or two
// chunks; the C CTAs of a thread-block cluster (cluster dims (1, 1, C), C <=
// 8) take equal runs of that list.  Per chunk:
//   S   = Q K^T      tcgen05.mma M=128, N=64,  K=D   (both operands K-major)
//   P   = exp2(S * scale * log2 e - m), masked; bf16, written back into TMEM
//         over S's own columns
//   O  += P V        tcgen05.mma M=128, N=D,   K=64  (A = P from TMEM, V read
//                    MN-major from shared memory)
// with fp32 accumulators in TMEM (S/P double-buffered, O accumulated across
// chunks).  The reference max m of a row is raised only when a chunk's max
// exceeds it by more than 8 (log2 units), so P <= 2^8; when it is raised the
// softmax thread rescales its row of O in TMEM by exp2(m_old - m_new) after
// the previous PV completed.  The result is the same after the final 1/l.
// Warps: 0 TMA producer (Q once, K and V chunks in separate rings), 1 TMEM
// allocation + MMA issue (QK of chunk j+1 overlaps the softmax of chunk j),
// 2-5 softmax / output.  Contiguous prefix chunks are laid backwards from the
// sequence's prefix end, so no cache slot at or past prefix_len is ever read
// (the first chunk may start before position 0: TMA zero-fills those rows,
// and they are masked); paged prefix chunks are page-aligned from position 0.
// Tree keys are masked with each row's ancestor bitmask.
// With C = 1 the softmax threads write the bf16 output rows directly.  With
// C > 1, after a cluster barrier (every CTA's K/V rings drained), each softmax
// thread stores its normalised partial row and log-sum-exp through
// distributed shared memory into the receive buffer of the CTA that merges
// that row (row r: CTA r % C); after a second barrier every CTA merges its
// rows from local shared memory in split order (so the result does not
// depend on which CTA merges).  Every pipeline wait is
// bounded (~2 s) and sets MEDUSA_STATUS_TIMEOUT on expiry.
#include <cooperative_groups.h>
#include <limits.h>

#include "kernels.h"
#include "tc.cuh"
#include "tma.h"

namespace medusa {

namespace {

constexpr int kAW = 6;       // 0 producer, 1 MMA, 2-5 softmax
constexpr int kAM = 128;     // query rows per CTA (MMA M)
constexpr int kCh = 64;      // keys per chunk
constexpr int kCtasPerSm = 2;
// K and V rings: a K stage is free once its QK product is done, a V stage
// once its PV product is; at head_dim 128 three K and two V stages keep a CTA
// within half of an SM's shared memory
template <int D> constexpr int k_stages() { return D == 128 ? 3 : 4; }
template <int D> constexpr int v_stages() { return D == 128 ? 2 : 4; }
template <int D> constexpr int n_bars() { return 1 + 2 * k_stages<D>() + 2 * v_stages<D>() + 6; }
constexpr int kPageRing = 8 * 8 * 4;  // bytes of the page-id ring (8 chunks x 8 boxes)
constexpr int kMaxCluster = 8;        // key splits per tile: at most a portable cluster of 8
// floats per row of a parked partial (D + 4: 16-byte row accesses of
// consecutive rows fall on distinct banks)
template <int D> constexpr int o_stride() { return D + 4; }

struct TcAttnArgs {
    CUtensorMap mq;    // q as (D, Hq, B*T), box (64, G, 128/G)
    CUtensorMap mkc;   // k_cache as (D, S_max, B*Hkv), box (64, 64, 1); paged: k_pages as
    CUtensorMap mvc;   //   (D, page_size, num_pages*Hkv), box (64, page_rows, 1)
    CUtensorMap mkt;   // k_tree as (D, Hkv, B*T), box (64, 1, 64); unused when the tree is in the cache
    CUtensorMap mvt;
    const int32_t* prefix_len;
    TreeRef tree;
    const int32_t* block_table;  // NULL: contiguous caches
    int max_pages, page_size, num_pages, page_rows;  // page_rows = min(page_size, 64) rows per TMA box
    __nv_bfloat16* out;  // [B, T, Hq, D]
    float* lse;          // [B, T, Hq], natural log; nullable
    int32_t* status;
    int B, T, Hq, Hkv, G, S_max, max_prefix;
    int tree_in_cache;  // the tree's K/V are cache rows prefix_len .. prefix_len + T_b (contiguous caches)
    float scale_log2;
    uint64_t wait_ns;   // limit of the pipeline waits (drains of issued work: kWaitLimitNs)
};

// 4-byte asynchronous global -> shared copy (cp.async group semantics)
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// 2^x with the SFU's approximate exponential (relative error ~2^-22, far
// below the bf16 rounding P goes through; 2^-inf = 0)
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// descriptor of an MN-major operand stored as TMA writes a (64 MN x rows K)
// box with a 128-byte swizzle: 8 K-rows of 128 bytes per 1024-byte group;
// `lbo` = byte distance to the next 64-element MN block
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t smem_byte_addr, uint32_t lbo) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_byte_addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// kTestWaits: the protocol waits take their limit from the arguments (a
// shortened limit set to test the error paths); otherwise it is the constant
template <int D, bool kTestWaits>
__global__ void __launch_bounds__(kAW * 32, kCtasPerSm) tree_attn_tc_kernel(const __grid_constant__ TcAttnArgs a) {
    const uint64_t wait_ns = kTestWaits ? a.wait_ns : kWaitLimitNs;
    constexpr int NSUB = D / 64;              // 64-element blocks along D
    constexpr int kQBytes = kAM * D * 2;
    constexpr int kSub = kCh * 128;           // [64 keys x 64 D] block = 8 KB
    constexpr int kKVBytes = kCh * D * 2;     // one chunk of K (or of V)
    constexpr int KS = k_stages<D>(), VS = v_stages<D>();
    constexpr uint32_t kIdescQK = idesc_bf16_f32(kAM, kCh);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(kAM, D) | (1u << 16);  // A (P) from TMEM, B (V) MN-major
    constexpr uint32_t kTmemCols = 256;       // S: 2 x 64 columns, O: D columns at 128
    // Dynamic shared memory starts on a 1024-byte boundary when the kernel has
    // no static shared memory; the tiles below rely on it (checked at entry,
    // so two CTAs fit per SM without alignment padding).
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sQ = smem;
    uint8_t* sK = sQ + kQBytes;
    uint8_t* sV = sK + KS * kKVBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sV + VS * kKVBytes);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + KS;
    uint64_t* v_full = k_empty + KS;
    uint64_t* v_empty = v_full + VS;
    uint64_t* s_full = v_empty + VS;
    uint64_t* p_full = s_full + 2;
    uint64_t* o_full = p_full + 2;  // one phase per PV product
    // a single phase, completed with the last PV product: a parity wait on
    // o_full cannot tell "the last PV done" from "two PVs done" once both of
    // the last two have completed
    uint64_t* o_last = o_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_last + 1);
    // paged: the page of each box of the last 8 K chunks, for their V loads
    int* pg_ring = reinterpret_cast<int*>(tmem_slot + 4);  // [8][8]

    namespace cg = cooperative_groups;
    const int mt = blockIdx.x, bg = blockIdx.y;
    const int C = (int)gridDim.z, split = blockIdx.z;  // the key splits of a tile form one cluster
    const int b = bg / a.Hkv, g = bg % a.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const TreeDev* tree = a.tree.at(b);
    const int Tb = tree->T;  // this sequence's tree (a.T: the row stride of q, out and the tree K/V)
    if (smem_addr(smem) & 1023u) {  // never expected (uniform over the grid); refuse rather than misread tiles
        if (threadIdx.x == 0) set_status(a.status, MEDUSA_STATUS_TIMEOUT);
        return;
    }
    const int NB = kAM / a.G;  // nodes per tile

    int S = a.prefix_len[b];
    if (S < 0 || S > a.max_prefix) {
        if (threadIdx.x == 0 && split == 0 && mt == 0 && g == 0) set_status(a.status, MEDUSA_STATUS_BAD_PREFIX);
        S = S < 0 ? 0 : a.max_prefix;
    }
    const bool paged = a.block_table != nullptr;
    // the sequence's chunks: nP prefix chunks, then nT tree chunks; this split
    // takes chunks [c0, c0 + nc) of them
    const int nP = (S + kCh - 1) / kCh, nT = (Tb + kCh - 1) / kCh, N = nP + nT;
    const int c0 = (int)((long)N * split / C);
    const int nc = (int)((long)N * (split + 1) / C) - c0;
    auto is_tree = [&](int j) { return c0 + j >= nP; };
    // first key of chunk j: a prefix position (contiguous chunks end exactly at
    // S, the first one may start below 0; paged ones start at multiples of 64)
    // or, for a tree chunk, a node index
    auto chunk_key0 = [&](int j) {
        const int c = c0 + j;
        return c >= nP ? (c - nP) * kCh : paged ? c * kCh : S - (nP - c) * kCh;
    };

    if (threadIdx.x == 32) {  // the descriptors' first use is the producer's first copy
        tma_prefetch_desc(&a.mq);
        tma_prefetch_desc(&a.mkc);
        tma_prefetch_desc(&a.mvc);
        if (!a.tree_in_cache) {
            tma_prefetch_desc(&a.mkt);
            tma_prefetch_desc(&a.mvt);
        }
    }
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < KS; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < VS; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
        }
        mbar_init(o_full, 1);
        mbar_init(o_last, 1);
        mbar_fence_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    sync_block();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // the softmax threads' row: its final (unnormalised) O, max m and sum l
    const int lr = (warp & 3) * 32 + lane;   // TMEM lane = tile row of a softmax thread
    const int rrow = mt * kAM + lr;          // row within the (sequence, kv-head)
    const bool row_ok = warp >= 2 && rrow < Tb * a.G;
    float o[D];
    float m = -INFINITY, l = 0.f;

    if (warp == 0) {
        // ---------------- producer ----------------
        // K chunks run ahead of V chunks; each is loaded as soon as its ring
        // stage is free (polled without blocking, so a late V stage never
        // holds back the next K)
        if (lane == 0 && nc > 0) {
            mbar_arrive_expect_tx(q_full, kQBytes);
#pragma unroll
            for (int sub = 0; sub < NSUB; ++sub)
                tma_load_3d(sQ + sub * (kAM * 128), &a.mq, sub * 64, g * a.G, b * a.T + mt * NB, q_full);
            // Paged: the page of every box (page_rows keys) of a prefix chunk,
            // copied asynchronously into the chunk's pg_ring slot one chunk
            // ahead (a K chunk waits only for its own ids; its V chunk reuses
            // them).  Boxes at or past S are not loaded (their rows are masked,
            // and cleared in V); an out-of-range page is skipped and reported.
            const int pr = paged ? a.page_rows : kCh, nbox = kCh / pr;
            auto fetch_pages = [&](int j) {
                if (j >= nc || is_tree(j)) return;
                int* ring = pg_ring + (j & 7) * 8;
                const int cs = chunk_key0(j);
                for (int i = 0; i < nbox; ++i) {
                    const int pos = cs + i * pr;
                    if (pos < S)
                        cp_async4(smem_addr(ring + i), &a.block_table[(long)b * a.max_pages + pos / a.page_size]);
                    else
                        ring[i] = -1;
                }
                cp_async_commit();
            };
            auto issue_chunk = [&](uint8_t* base, const CUtensorMap* mc, const CUtensorMap* mtr, uint64_t* bar,
                                   int j, bool is_k) {
                const int cs = chunk_key0(j);
                const bool tr = is_tree(j);
                if (tr || !paged) {
                    mbar_arrive_expect_tx(bar, kKVBytes);
#pragma unroll
                    for (int sub = 0; sub < NSUB; ++sub) {
                        if (tr && a.tree_in_cache)  // rows S + cs .. of this (sequence, kv-head)
                            tma_load_3d(base + sub * kSub, mc, sub * 64, S + cs, bg, bar);
                        else if (tr) tma_load_3d(base + sub * kSub, mtr, sub * 64, g, b * a.T + cs, bar);
                        else tma_load_3d(base + sub * kSub, mc, sub * 64, cs, bg, bar);
                    }
                    return;
                }
                int* ring = pg_ring + (j & 7) * 8;
                if (is_k) {
                    cp_async_wait_all();  // this chunk's ids (the only group in flight)
                    for (int i = 0; i < nbox; ++i) {
                        const int page = ring[i];
                        if (page >= a.num_pages || (page < 0 && cs + i * pr < S)) {
                            set_status(a.status, MEDUSA_STATUS_BAD_PAGE);
                            ring[i] = -1;
                        }
                    }
                    fetch_pages(j + 1);  // the next chunk's ids, in flight meanwhile
                }
                int nload = 0;
                for (int i = 0; i < nbox; ++i) nload += ring[i] >= 0;
                mbar_arrive_expect_tx(bar, (uint32_t)(nload * pr * 128 * NSUB));
                for (int i = 0; i < nbox; ++i) {
                    const int page = ring[i];
                    if (page < 0) continue;
                    const int pos = cs + i * pr;
#pragma unroll
                    for (int sub = 0; sub < NSUB; ++sub)
                        tma_load_3d(base + sub * kSub + i * pr * 128, mc, sub * 64, pos % a.page_size,
                                    page * a.Hkv + g, bar);
                }
            };
            if (paged) fetch_pages(0);
            int jk = 0, jv = 0;
            uint64_t t0 = global_ns();
            uint32_t idle = 0;
            while (jk < nc || jv < nc) {
                bool prog = false;
                if (jk < nc && (jk < KS || mbar_test(&k_empty[jk % KS], ((jk / KS) - 1) & 1))) {
                    const int s = jk % KS;
                    issue_chunk(sK + s * kKVBytes, &a.mkc, &a.mkt, &k_full[s], jk, true);
                    ++jk;
                    prog = true;
                }
                if (jv < jk && (jv < VS || mbar_test(&v_empty[jv % VS], ((jv / VS) - 1) & 1))) {
                    const int s = jv % VS;
                    issue_chunk(sV + s * kKVBytes, &a.mvc, &a.mvt, &v_full[s], jv, false);
                    ++jv;
                    prog = true;
                }
                if (prog) {
                    idle = 0;
                    t0 = global_ns();
                } else if ((++idle & 255u) == 0 && global_ns() - t0 > wait_ns) {
                    set_status(a.status, MEDUSA_STATUS_TIMEOUT);
                    break;
                }
            }
            // drain: no copy may still be landing when the CTA exits
            cp_async_wait_all();
            mbar_wait(q_full, 0);
            for (int s = 0; s < KS && s < jk; ++s) {
                const int last = s + ((jk - 1 - s) / KS) * KS;
                mbar_wait(&k_full[s], (last / KS) & 1);
            }
            for (int s = 0; s < VS && s < jv; ++s) {
                const int last = s + ((jv - 1 - s) / VS) * VS;
                mbar_wait(&v_full[s], (last / VS) & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0 && nc > 0) {
            bool ok = mbar_wait(q_full, 0, wait_ns);
            // S_j goes to TMEM columns (j&1)*64; P_j is written over it, so the
            // buffer is free for S_{j+2} once PV_j has completed (o_full phase j)
            auto issue_qk = [&](int j) -> bool {
                const int s = j % KS, sb = j & 1;
                if (!mbar_wait(&k_full[s], (j / KS) & 1, wait_ns)) return false;
                if (j >= 2 && !mbar_wait(o_full, (j - 2) & 1, wait_ns)) return false;
                tc_fence_after();
#pragma unroll
                for (int sub = 0; sub < NSUB; ++sub) {
                    const uint64_t ad = sw128_kmajor_desc(smem_addr(sQ + sub * (kAM * 128)));
                    const uint64_t bd = sw128_kmajor_desc(smem_addr(sK + s * kKVBytes + sub * kSub));
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        tc_mma_bf16(tmem + sb * kCh, ad + 2 * ks, bd + 2 * ks, kIdescQK, (sub | ks) != 0);
                }
                tc_commit(&s_full[sb]);
                tc_commit(&k_empty[s]);
                return true;
            };
            if (ok) ok = issue_qk(0);
            for (int j = 0; j < nc && ok; ++j) {
                if (j + 1 < nc && !(ok = issue_qk(j + 1))) break;
                if (!mbar_wait(&p_full[j & 1], (j >> 1) & 1, wait_ns)) {
                    ok = false;
                    break;
                }
                const int s = j % VS;
                if (!mbar_wait(&v_full[s], (j / VS) & 1, wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t bd = sw128_mnmajor_desc(smem_addr(sV + s * kKVBytes), kSub);
#pragma unroll
                for (int ks = 0; ks < kCh / 16; ++ks)  // 16 keys: 8 P columns, +2 K-groups (2048 B) in V
                    tc_mma_bf16_ts(tmem + 128, tmem + (j & 1) * kCh + ks * 8, bd + (uint64_t)(2048 >> 4) * ks,
                                   kIdescPV, (j | ks) != 0);
                tc_commit(o_full);
                tc_commit(&v_empty[s]);
                if (j == nc - 1) tc_commit(o_last);
            }
            if (!ok) {
                // o_last was not committed (the loop left before the last
                // chunk): commit it now, so that it completes once every MMA
                // this thread did issue has finished writing TMEM
                set_status(a.status, MEDUSA_STATUS_TIMEOUT);
                tc_commit(o_last);
            }
            mbar_wait(o_last, 0);  // every MMA done before TMEM is released (bounded)
        }
    } else {
        // ---------------- softmax ----------------
        const int q = warp & 3;
        const int node = row_ok ? rrow / a.G : 0;
        uint32_t anc[4] = {0u, 0u, 0u, 0u};
        if (row_ok && nc > 0 && is_tree(nc - 1))
#pragma unroll
            for (int w = 0; w < 4; ++w) anc[w] = tree->anc[node][w];
        bool ok = true;
        const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
        for (int j = 0; j < nc && ok; ++j) {
            // every wait before a warp-collective tcgen05 operation is decided
            // for the whole warp (its lanes test the barrier independently)
            if (!__all_sync(kFull, mbar_wait(&s_full[j & 1], (j >> 1) & 1, wait_ns))) {
                ok = false;
                break;
            }
            tc_fence_after();
            float sv[kCh];
            {
                uint32_t raw[kCh / 16][16];
#pragma unroll
                for (int c = 0; c < kCh / 16; ++c) tmem_ld16_async(lane_base + (j & 1) * kCh + c * 16, raw[c]);
                tmem_wait_ld(raw);
#pragma unroll
                for (int c = 0; c < kCh / 16; ++c)
#pragma unroll
                    for (int e = 0; e < 16; ++e) sv[c * 16 + e] = __uint_as_float(raw[c][e]);
            }
            // visible keys of this chunk for this row, bit c = key key0 + c
            const int key0 = chunk_key0(j);
            const bool tr = is_tree(j);
            uint64_t vis;
            if (tr) {
                // ancestor bits (keys >= T have none); key0 is 0 or 64
                vis = key0 == 0 ? ((uint64_t)anc[1] << 32 | anc[0]) : ((uint64_t)anc[3] << 32 | anc[2]);
            } else {
                // prefix keys [0, S): a contiguous first chunk may start below
                // 0, a paged last chunk may reach past S
                const int lo = key0 >= 0 ? 0 : -key0, hi = S - key0;
                vis = lo > 0 ? ~0ull << lo : ~0ull;
                if (hi < kCh) vis &= (1ull << hi) - 1ull;
            }
            // online softmax in the log2 domain: p = 2^(s * scale * log2 e - mu)
            float mx;
            if (vis == ~0ull) {
                float m4[4] = {sv[0], sv[1], sv[2], sv[3]};
#pragma unroll
                for (int c = 4; c < kCh; ++c) m4[c & 3] = fmaxf(m4[c & 3], sv[c]);
                mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            } else {
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int c = 0; c < kCh; ++c) {
                    sv[c] = (vis >> c) & 1ull ? sv[c] : -INFINITY;
                    m4[c & 3] = fmaxf(m4[c & 3], sv[c]);
                }
                mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            }
            mx *= a.scale_log2;  // the scale is positive: the max commutes with it
            // lazy reference max: raised only when the chunk's max exceeds it by > 8
            const bool raise = mx > m + 8.f;
            const float mn = raise ? mx : m;
            const float mu = mn == -INFINITY ? 0.f : mn;
            const float alpha = raise ? fast_exp2(m - mu) : 1.f;
            float rs;
            {
                uint32_t pk[2][16];  // P row: 64 keys as 32 bf16 pairs
                float r4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < kCh / 2; ++c) {
                    const float p0 = fast_exp2(fmaf(sv[2 * c], a.scale_log2, -mu));
                    const float p1 = fast_exp2(fmaf(sv[2 * c + 1], a.scale_log2, -mu));
                    __nv_bfloat162 v2 = __floats2bfloat162_rn(p0, p1);
                    // the row sum uses the same bf16 weights PV multiplies by
                    r4[c & 3] += __low2float(v2) + __high2float(v2);
                    pk[c >> 4][c & 15] = *reinterpret_cast<uint32_t*>(&v2);
                }
                rs = (r4[0] + r4[1]) + (r4[2] + r4[3]);
                tmem_st16(lane_base + (j & 1) * kCh, pk[0]);
                tmem_st16(lane_base + (j & 1) * kCh + 16, pk[1]);
            }
            l = l * alpha + rs;
            // rescale this warp's rows of O when some row's reference max rose
            // (after the previous PV has completed)
            if (j >= 1 && __any_sync(kFull, raise)) {
                if (!__all_sync(kFull, mbar_wait(o_full, (j - 1) & 1, wait_ns))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float f = alpha;
#pragma unroll
                for (int c0 = 0; c0 < D / 16; c0 += 4) {
                    uint32_t raw[4][16];
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        if (c0 + c < D / 16) tmem_ld16_async(lane_base + 128 + (c0 + c) * 16, raw[c]);
                    tmem_wait_ld(raw);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        if (c0 + c < D / 16) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) raw[c][e] = __float_as_uint(__uint_as_float(raw[c][e]) * f);
                            tmem_st16(lane_base + 128 + (c0 + c) * 16, raw[c]);
                        }
                }
                tmem_wait_st();
            }
            m = mn;
            const int key_end = tr ? Tb : S;
            if (key0 + kCh > key_end) {
                // the chunk's rows past this sequence's keys (tree padding,
                // another sequence's rows, page slots past the prefix, boxes
                // not loaded) have P = 0, but a NaN in V would still reach O
                // (0 * NaN), so those V rows are cleared before PV may start
                const int s = j % VS;
                if (!__all_sync(kFull, mbar_wait(&v_full[s], (j / VS) & 1, wait_ns))) {
                    ok = false;
                    break;
                }
                const int r0 = key_end - key0, lt = (warp - 2) * 32 + lane;
                uint8_t* vs = sV + s * kKVBytes;
                for (int idx = lt; idx < (kCh - r0) * NSUB * 8; idx += 128) {
                    const int row = r0 + idx / (NSUB * 8), rem = idx % (NSUB * 8);
                    *reinterpret_cast<uint4*>(vs + (rem >> 3) * kSub + row * 128 + (rem & 7) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_shared();
            }
            tmem_wait_st();  // P (and any rescaled O) in TMEM before the MMA reads it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[j & 1]);
        }
        // final O (after the last PV) for this row
        if (ok && nc > 0) ok = __all_sync(kFull, mbar_wait(o_last, 0, wait_ns));
        if (ok && nc > 0) {
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < D / 16; c0 += 4) {
                uint32_t raw[4][16];
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (c0 + c < D / 16) tmem_ld16_async(lane_base + 128 + (c0 + c) * 16, raw[c]);
                tmem_wait_ld(raw);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (c0 + c < D / 16)
#pragma unroll
                        for (int e = 0; e < 16; ++e) o[(c0 + c) * 16 + e] = __uint_as_float(raw[c][e]);
            }
        } else {
#pragma unroll
            for (int e = 0; e < D; ++e) o[e] = 0.f;
            l = 0.f;
        }
        if (!ok && lane == 0) set_status(a.status, MEDUSA_STATUS_TIMEOUT);
        if (!row_ok) {  // a row past this sequence's tree (or the tile): zero
#pragma unroll
            for (int e = 0; e < D; ++e) o[e] = 0.f;
            l = 0.f;
        }
    }
    // every role is done: no MMA in flight, no copy landing
    tc_fence_before();
    sync_block();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    const int rows_T = a.T * a.G;   // rows of the (sequence, kv-head) in the output (past Tb * G: zeros)
    // output row r of this (sequence, kv-head): (node, q-head) = (r / G, g * G + r % G)
    auto out_row = [&](int r) -> long { return ((long)b * a.T + r / a.G) * a.Hq + g * a.G + r % a.G; };
    if (C == 1) {
        // a single split: this CTA's rows are final
        if (warp >= 2 && rrow < rows_T) {
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const long orow = out_row(rrow);
            uint4* dst = reinterpret_cast<uint4*>(a.out + orow * D);
#pragma unroll
            for (int e = 0; e < D; e += 8) {
                uint4 v;
                v.x = pack2_bf16(o[e] * inv, o[e + 1] * inv);
                v.y = pack2_bf16(o[e + 2] * inv, o[e + 3] * inv);
                v.z = pack2_bf16(o[e + 4] * inv, o[e + 5] * inv);
                v.w = pack2_bf16(o[e + 6] * inv, o[e + 7] * inv);
                dst[e / 8] = v;
            }
            if (a.lse) a.lse[orow] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
        }
        return;
    }
    // ---- several splits: each row's partial goes to the CTA that merges it ----
    // Row r of the tile is merged by the cluster's CTA r % C, as its row
    // r / C.  After a first cluster barrier (every CTA's K/V rings are drained
    // and free), each softmax thread stores its normalised partial row and its
    // log-sum-exp (in the row's padding) into that CTA's receive buffer
    // [C][RPC][OS], at [split][r / C]; after a second barrier each CTA merges
    // its rows from local shared memory, in split order.
    constexpr int OS = o_stride<D>();
    const int RPC = (kAM + C - 1) / C;           // rows merged per CTA
    float* recv = reinterpret_cast<float*>(sK);  // [C][RPC][OS] over the drained K/V rings
    const int nrows = min(kAM, rows_T - mt * kAM);
    cg::cluster_group cl = cg::this_cluster();
    __syncwarp();  // the cluster barrier is an aligned one: whole warps
    cl.sync();     // every CTA of the cluster is past its main loop
    if (warp >= 2 && lr < nrows) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        float* dst = cl.map_shared_rank(recv, lr % C) + ((long)split * RPC + lr / C) * OS;
#pragma unroll
        for (int e = 0; e < D; e += 4)
            *reinterpret_cast<float4*>(dst + e) = make_float4(o[e] * inv, o[e + 1] * inv, o[e + 2] * inv, o[e + 3] * inv);
        *reinterpret_cast<float4*>(dst + D) = make_float4(l > 0.f ? m + log2f(l) : -INFINITY, 0.f, 0.f, 0.f);
    }
    __syncwarp();
    cl.sync();  // every partial row has arrived (the stores are released by the barrier)
    constexpr int PL = D / 32;  // elements of a row per lane
    for (int i = warp; i * C + split < nrows; i += kAW) {
        const int r = i * C + split;
        const long orow = out_row(mt * kAM + r);
        __nv_bfloat16* dst = a.out + orow * D + lane * PL;
        if (mt * kAM + r >= Tb * a.G) {  // past this sequence's tree: zero output
#pragma unroll
            for (int e = 0; e < PL; ++e) dst[e] = __float2bfloat16_rn(0.f);
            if (a.lse && lane == 0) a.lse[orow] = -INFINITY;
            continue;
        }
        const float ls = lane < C ? recv[((long)lane * RPC + i) * OS + D] : -INFINITY;
        float M = ls;
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o2));
        const float wl = ls == -INFINITY ? 0.f : exp2f(ls - M);
        float acc[PL], wsum = 0.f;
#pragma unroll
        for (int e = 0; e < PL; ++e) acc[e] = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < kMaxCluster; ++s2) {  // in split order
            if (s2 >= C) break;
            const float ws = __shfl_sync(kFull, wl, s2);
            if (ws > 0.f) {
                const float* src = recv + ((long)s2 * RPC + i) * OS + lane * PL;
                wsum += ws;
#pragma unroll
                for (int e = 0; e < PL; ++e) acc[e] = fmaf(ws, src[e], acc[e]);
            }
        }
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
        for (int e = 0; e < PL; e += 2)
            *reinterpret_cast<uint32_t*>(dst + e) = pack2_bf16(acc[e] * inv, acc[e + 1] * inv);
        if (a.lse && lane == 0) a.lse[orow] = wsum > 0.f ? (M + log2f(wsum)) * 0.69314718055994531f : -INFINITY;
    }
}

template <int D>
size_t tc_attn_smem() {
    // Q, the K and V rings, the mbarriers, the TMEM address slot and the page-id ring
    return (size_t)kAM * D * 2 + (size_t)(k_stages<D>() + v_stages<D>()) * kCh * D * 2 + n_bars<D>() * 8 + 16 +
           kPageRing;
}
// the receive buffer ([C][ceil(128 / C)][OS] floats, at most 135 rows for
// C <= 8) fits over the K/V rings
static_assert((kAM + kMaxCluster - 1) * o_stride<128>() * 4 <= (k_stages<128>() + v_stages<128>()) * kCh * 128 * 2,
              "receive buffer (D=128)");
static_assert((kAM + kMaxCluster - 1) * o_stride<64>() * 4 <= (k_stages<64>() + v_stages<64>()) * kCh * 64 * 2,
              "receive buffer (D=64)");

cudaError_t launch_attn(void (*kern)(TcAttnArgs), cudaLaunchConfig_t& cfg, const TcAttnArgs& a) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cfg.dynamicSmemBytes);
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace

int attn_tc_ctas_per_sm() { return kCtasPerSm; }

bool attn_tc_page_ok(int page_size) {
    return page_size > 0 && (page_size % 64 == 0 || page_size == 8 || page_size == 16 || page_size == 32);
}

bool attn_tc_supported(int Hq, int Hkv, int D, int T, medusa_dtype dt) {
    const int G = Hkv > 0 ? Hq / Hkv : 0;
    return dt == MEDUSA_BF16 && (D == 64 || D == 128) && G >= 1 && G <= 16 && (G & (G - 1)) == 0 && T <= kMaxTree;
}

// Key splits per 128-row tile: enough CTAs for two per SM, at most a portable
// cluster of 8 (a cluster of 9 CTAs at two per SM does not pack into the GPCs:
// measured, the 288 CTAs of llama8b ran in two waves) and at most the chunks
// of the longest sequence.
int attn_tc_splits(int B, int T, int Hq, int Hkv, int max_prefix) {
    const int G = Hq / Hkv;
    const long m_tiles = ((long)T * G + kAM - 1) / kAM;
    const long per_split = m_tiles * B * Hkv;
    const long target = (long)kCtasPerSm * num_sms();
    long c = (target + per_split - 1) / per_split;
    const long chunks = (max_prefix + kCh - 1) / kCh + (T + kCh - 1) / kCh;
    if (c > kMaxCluster) c = kMaxCluster;
    if (c > chunks) c = chunks;
    // With few chunks per split (a short prefix) one CTA per SM does better:
    // a whole SM per CTA and fewer partials to merge (2048 keys at llama8b
    // shapes: 4 splits of 128 CTAs 25.4 us, 8 splits of 256 CTAs 28.7 us;
    // at 32k keys 8 splits stay best)
    if (chunks < 8 * c) {
        const long c1 = num_sms() / per_split;
        if (c1 >= 1 && c1 < c) c = c1;
    }
    const int cap = launch_attention_splits();
    if (cap > 0 && c > cap) c = cap;
    return c < 1 ? 1 : (int)c;
}

// launch the tensor-core kernel: m_tiles 128-row tiles per (sequence, kv-head),
// n_splits key splits per tile (one cluster); writes the output (and lse)
cudaError_t attn_tc_launch(const AttnArgs& x, int m_tiles, int n_splits, float scale_log2, cudaStream_t st) {
    TcAttnArgs a;
    const uint64_t D = x.D, Hq = x.Hq, Hkv = x.Hkv, BT = (uint64_t)x.B * x.T, Smax = x.S_max, BH = (uint64_t)x.B * x.Hkv;
    const int G = x.Hq / x.Hkv;
    if (n_splits < 1 || n_splits > kMaxCluster) return cudaErrorInvalidValue;
    {
        const uint64_t dims[3] = {D, Hq, BT}, strides[2] = {D * 2, Hq * D * 2};
        const uint32_t box[3] = {64, (uint32_t)G, (uint32_t)(kAM / G)};
        if (!make_tmap_bf16(&a.mq, x.q, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    if (x.block_table) {
        const uint64_t ps = x.page_size, NP = (uint64_t)x.num_pages * Hkv;
        const uint64_t dims[3] = {D, ps, NP}, strides[2] = {D * 2, ps * D * 2};
        const uint32_t box[3] = {64, (uint32_t)(x.page_size < kCh ? x.page_size : kCh), 1};
        if (!make_tmap_bf16(&a.mkc, x.k_cache, 3, dims, strides, box)) return cudaErrorInvalidValue;
        if (!make_tmap_bf16(&a.mvc, x.v_cache, 3, dims, strides, box)) return cudaErrorInvalidValue;
    } else {
        const uint64_t dims[3] = {D, Smax, BH}, strides[2] = {D * 2, Smax * D * 2};
        const uint32_t box[3] = {64, (uint32_t)kCh, 1};
        if (!make_tmap_bf16(&a.mkc, x.k_cache, 3, dims, strides, box)) return cudaErrorInvalidValue;
        if (!make_tmap_bf16(&a.mvc, x.v_cache, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    a.block_table = x.block_table;
    a.max_pages = x.max_pages;
    a.page_size = x.page_size;
    a.num_pages = x.num_pages;
    a.page_rows = x.page_size < kCh ? x.page_size : kCh;
    a.tree_in_cache = x.k_tree == nullptr;
    if (!a.tree_in_cache) {
        const uint64_t dims[3] = {D, Hkv, BT}, strides[2] = {D * 2, Hkv * D * 2};
        const uint32_t box[3] = {64, 1, (uint32_t)kCh};
        if (!make_tmap_bf16(&a.mkt, x.k_tree, 3, dims, strides, box)) return cudaErrorInvalidValue;
        if (!make_tmap_bf16(&a.mvt, x.v_tree, 3, dims, strides, box)) return cudaErrorInvalidValue;
    } else {
        a.mkt = a.mkc;  // never read
        a.mvt = a.mvc;
    }
    a.prefix_len = x.prefix_len;
    a.tree = x.tree;
    a.out = (__nv_bfloat16*)x.out;
    a.lse = x.lse;
    a.status = x.status;
    a.B = x.B;
    a.T = x.T;
    a.Hq = x.Hq;
    a.Hkv = x.Hkv;
    a.G = G;
    a.S_max = x.S_max;
    a.max_prefix = x.max_prefix;
    a.scale_log2 = scale_log2;
    a.wait_ns = wait_limit_ns();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(m_tiles, (unsigned)BH, n_splits);
    cfg.blockDim = dim3(kAW * 32);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = n_splits;
    cfg.attrs = attr;
    cfg.numAttrs = n_splits > 1 ? 1 : 0;
    const bool test_waits = a.wait_ns != kWaitLimitNs;
    if (x.D == 128) {
        cfg.dynamicSmemBytes = tc_attn_smem<128>();
        return launch_attn(test_waits ? tree_attn_tc_kernel<128, true> : tree_attn_tc_kernel<128, false>, cfg, a);
    }
    cfg.dynamicSmemBytes = tc_attn_smem<64>();
    return launch_attn(test_waits ? tree_attn_tc_kernel<64, true> : tree_attn_tc_kernel<64, false>, cfg, a);
}

}  // namespace medusa
