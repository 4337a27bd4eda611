// Medusa heads on the 5th-generation tensor cores (bf16, batch <= 64).
//
// Operation ("Medusa Explained: Multi-Head Speculative Decoding Guide",
// section "The Architectural Blueprint"): h^(k) = SiLU(W_res^(k) h) + h,
// p^(k) = softmax(W_head^(k) h^(k)), then each head's top-8 fills the
// candidate tree ("1. Combinatorial Tree Construction").
//
// Both products read every weight once, with only B (1..64) columns on the
// other side: weight streaming is the cost, so the kernel is built around
// keeping HBM busy and the SMs' ALUs idle.  Each weight tile of 128 rows x 64
// k-elements (16 KB) is a tcgen05 MMA A operand (M = 128), the batch vectors
// are the B operand (N = batch rounded up to 16; TMA zero-fills the padding
// rows), and the fp32 accumulator lives in TMEM.  One cooperative persistent
// kernel per call, one CTA per SM, 7 warps:
//   warp 0   TMA producer of weight tiles (a ring of shared-memory stages)
//   warp 1   TMEM allocation; one thread issues the MMAs (double-buffered
//            accumulator, commits release ring stages and hand tiles over)
//   warp 2   TMA producer of the batch-vector tiles; before the first
//            vocabulary tile it waits at the grid barrier (all of h^(k) must
//            be written by every CTA)
//   warps 3-6 epilogue, one TMEM lane (= weight row) per thread, reading
//            the accumulator 16 columns at a time: residual tiles write
//            h^(k) = SiLU(z) + h (bf16); vocabulary tiles are transposed
//            through shared memory, then each column's (sequence's) running
//            softmax statistics and top-8 list are updated (by warp units up
//            to 32 sequences, by thread segments above: see row_blocks and
//            units_epilogue); at a head change they become the CTA's
//            partial for (head, sequence).
// Work split ("stream-K"): in the vocabulary phase (and in the residual phase
// when it has more tiles than there are CTAs; otherwise each CTA takes one
// whole residual tile) the tiles' 64-element k-blocks are laid end to end and
// every CTA takes an equal contiguous run of them, so all SMs stream the same
// number of bytes.  A tile cut by a run boundary is summed by the CTA holding
// its first k-block (its owner, which reaches it last in its run); the CTAs
// holding the rest reach their part first in theirs, and hand it over as an
// fp32 partial in global memory with a release flag.  The weight producer
// keeps prefetching across the grid barrier.  A head's (sequence, head)
// partials are merged, each in CTA order, and its tree nodes filled, by the
// last CTA to publish its partial of that head (a per-head arrival counter,
// no waiting); only the merges of the heads whose last tiles end the stream
// are left at the end of the kernel.  With more than 4 sequences one CTA would take too long over a
// head's merges, so there a grid barrier is followed by the merges of all
// heads spread over every warp of the grid.
// Every wait is bounded (~2 s) and sets MEDUSA_STATUS_TIMEOUT on expiry.
#include <limits.h>

#include "heads_common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tma.h"

namespace medusa {

namespace {

constexpr int kTcWarps = 7;
constexpr int kTM = 128;                 // weight rows per tile (MMA M)
constexpr int kTK = 64;                  // k-elements per stage (128 bytes, one swizzle row)
constexpr int kABytes = kTM * kTK * 2;   // 16 KB
constexpr int kEpiWarp0 = 3;             // first epilogue warp
constexpr int kSmemBudget = 227 * 1024;
constexpr int kTS = kTM + 1;             // transposed tile: column stride in floats (odd: no bank conflicts)
// Up to this many sequences a head is merged by its last CTA as soon as the
// head is done; above it (one CTA would hold up the end with the merges of
// many sequences) after a grid barrier, spread over every warp of the grid
constexpr int kMergePerHeadMaxB = 4;

// The vocabulary epilogue splits a tile's B columns (sequences) x 128 rows
// into units of one column and 128 / R rows (R = row blocks per column); unit
// u is column u / R, row block u % R, taken by warp u % 4.  R = 1: with fewer
// than four sequences some epilogue warps idle, but a column's state then
// needs no merge of row blocks at a head change (splitting one sequence's
// column over the four warps cost 4 us at llama8b, in the final merge's
// serial path).
__host__ __device__ constexpr int row_blocks(int) { return 1; }
// Above 32 sequences each warp would take 9..16 units, and a unit's top-8
// list starts empty in every CTA and head (about 30 insertions per column,
// each a warp-wide step), so there each thread takes one column segment of
// 128 / seg_per_col(B) rows instead: its running statistics and top-8 list
// stay in registers, and every row goes through a branch-free insertion
// (no divergence between the lanes' columns).
template <int N> constexpr bool units_epilogue() { return N <= 32; }
__host__ __device__ constexpr int seg_per_col(int B) { return 128 / B < 16 ? 128 / B : 16; }
__host__ __device__ constexpr int epi_blocks(int B, bool units) { return units ? row_blocks(B) : seg_per_col(B); }

struct TopEntry {
    float v;
    int i;
};

// Insert (v, i) into a top-kTopK list held across a warp, lane j < kTopK
// holding the j-th best (lanes past kTopK hold -inf and never change).  The
// entries the new item beats are a suffix of the sorted list; it takes the
// first of them and the rest move down one lane.
__device__ __forceinline__ void warp_list_insert(float& lv, int& li, float v, int i) {
    const int lane = threadIdx.x & 31;
    const unsigned worse = __ballot_sync(kFull, beats(v, i, lv, li)) & ((1u << kTopK) - 1u);
    const float uv = __shfl_up_sync(kFull, lv, 1);
    const int ui = __shfl_up_sync(kFull, li, 1);
    if (worse) {
        const int p = __ffs(worse) - 1;
        if (lane == p) {
            lv = v;
            li = i;
        } else if (lane > p && lane < kTopK) {
            lv = uv;
            li = ui;
        }
    }
}

struct TcHeadsArgs {
    CUtensorMap mW_res;   // W_res  as (d_in, d_out, K), box (64, 128, 1)
    CUtensorMap mW_head;  // W_head as (d, V, K),        box (64, 128, 1)
    CUtensorMap mh;       // h      as (d, B),           box (64, N)
    CUtensorMap mhk;      // h^(k)  as (d, K, B),        box (64, 1, N)
    const __nv_bfloat16* h;
    __nv_bfloat16* hk;      // [B][K][d] (workspace)
    __nv_bfloat16* hk_out;  // nullable copy for the caller
    float* logits;          // [B][K][V], nullable
    HeadState* part;        // [grid][K][B]
    float* slots;           // [2 phases][grid][B][128] handed-over partial tiles
    unsigned int* ctr;      // [2 + 2 * grid], zero at launch: grid-barrier arrivals, then the slots' flags
    TreeRef tree;
    const int32_t* root_token;
    int32_t* topk_idx;
    float* topk_prob;
    int32_t* node_tokens;
    float* node_q;
    float2* stats;
    int32_t* status;
    int B, d, V, K;
    int stages;
    int merge_per_head;  // B <= kMergePerHeadMaxB: each head merged by its last CTA; else after a grid barrier
    uint64_t wait_ns;    // limit of the pipeline waits when it differs from kWaitLimitNs (drains: kWaitLimitNs)
};

// A CTA's run of one phase: k-block units [u0, u1) of the phase's tiles laid
// end to end (tile t holds units [t nkb, (t+1) nkb)), the runs contiguous
// and in CTA order.  Piece i of the run is the part of one tile it covers.
struct Run {
    long u0, u1;
    int nkb;
    __device__ Run(long U, int c, int G, int nkb_) : u0(U * c / G), u1(U * (c + 1) / G), nkb(nkb_) {}
    // whole tiles: CTA c takes tile c of T, none when c >= T
    __device__ static Run whole(long T, int c, int nkb_) {
        Run r(0, 0, 1, nkb_);
        r.u0 = (c < T ? c : T) * (long)nkb_;
        r.u1 = (c < T ? c + 1 : T) * (long)nkb_;
        return r;
    }
    __device__ int count() const { return u1 > u0 ? (int)((u1 - 1) / nkb - u0 / nkb + 1) : 0; }
    __device__ void piece(int i, long& t, int& kb0, int& kb1) const {
        t = u0 / nkb + i;
        const long lo = u0 > t * nkb ? u0 : t * nkb;
        const long hi = u1 < (t + 1) * nkb ? u1 : (t + 1) * nkb;
        kb0 = (int)(lo - t * nkb);
        kb1 = (int)(hi - t * nkb);
    }
};

__device__ __forceinline__ void st_release_u32(unsigned int* p, unsigned int v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// bounded wait for a hand-over flag; false after limit_ns
__device__ __forceinline__ bool wait_flag(const unsigned int* f, uint64_t limit_ns) {
    if (ld_acquire_u32(f)) return true;
    const uint64_t t0 = global_ns();
    while (!ld_acquire_u32(f)) {
        if (global_ns() - t0 > limit_ns) return false;
        __nanosleep(32);
    }
    return true;
}

// the four epilogue warps' barrier (aligned: each warp reconverges first)
__device__ __forceinline__ void epi_sync() {
    __syncwarp();
    asm volatile("bar.sync 2, 128;" ::: "memory");
}

// kTestWaits: the waits take their limit from the arguments (a shortened limit
// set to test the error paths); otherwise the limit is the constant one, which
// keeps the pipeline loops free of the run-time choice (a measurable cost in
// the weight stream)
template <int N, bool kTestWaits>
__global__ void __launch_bounds__(kTcWarps * 32, 1) heads_tc_kernel(const __grid_constant__ TcHeadsArgs a) {
    const uint64_t wait_ns = kTestWaits ? a.wait_ns : kWaitLimitNs;
    constexpr int kBBytes = N * kTK * 2;  // batch tile per stage (multiple of 1024)
    constexpr int kTmemCols = N * 2 <= 32 ? 32 : N * 2 <= 64 ? 64 : 128;
    constexpr uint32_t kIdesc = idesc_bf16_f32(kTM, N);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    // One ring of stages, each a weight tile (from HBM) and a batch-vector
    // tile (from L2; issued as early as its weight tile: under a full HBM
    // stream its latency is as long).  A stage is full when both producers'
    // copies landed (one barrier, two arrivals with their byte counts: a
    // single wait per k-block for the MMA thread).
    const int S = a.stages;
    uint8_t* sA = smem;
    uint8_t* sB = sA + (size_t)S * kABytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + (size_t)S * kBBytes);
    uint64_t* empty = full + S;
    uint64_t* acc_full = empty + S;    // [2]
    uint64_t* acc_empty = acc_full + 2;  // [2]
    uint64_t* mma_done = acc_empty + 2;  // every MMA issued has completed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    int* last_flag = reinterpret_cast<int*>(tmem_slot + 1);  // this CTA merges the head it just flushed
    float* sT = reinterpret_cast<float*>(tmem_slot + 4);  // [B][kTS] transposed tile
    HeadState* stS = reinterpret_cast<HeadState*>(sT + ((a.B * kTS + 3) & ~3));  // [row block][B] flush states
    constexpr bool kUnits = units_epilogue<N>();
    const int nunits = a.B * epi_blocks(a.B, kUnits);  // units, or column segments
    float2* sU = reinterpret_cast<float2*>(stS + nunits);       // [unit][lane] running (max, sum)
    TopEntry* sL = reinterpret_cast<TopEntry*>(sU + nunits * 32);  // [unit][kTopK] top list, best first

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int K = a.K, B = a.B;
    const int G = gridDim.x, cta = blockIdx.x;
    const int tph_r = (a.d + kTM - 1) / kTM;   // residual tiles per head
    const int tph_l = (a.V + kTM - 1) / kTM;   // vocabulary tiles per head
    const int nkb = (a.d + kTK - 1) / kTK;     // k-blocks per tile
    const long U1 = (long)K * tph_r * nkb, U2 = (long)K * tph_l * nkb;
    // The residual phase takes whole tiles when there are no more of them than
    // CTAs: a tile split over several CTAs has its owner wait for the others'
    // partial sums before its epilogue, and at these sizes the waits and the
    // reads of the partials cost more than the streaming time an even split
    // saves (llama8b: 128 tiles on 148 CTAs, 1 MB each).
    const long T1 = (long)K * tph_r;
    const Run run1 = T1 <= G ? Run::whole(T1, cta, nkb) : Run(U1, cta, G, nkb), run2(U2, cta, G, nkb);
    const int n1 = run1.count(), n2 = run2.count();
    const int ntiles = n1 + n2;  // pieces, residual phase first
    auto piece = [&](int li, long& t, int& kb0, int& kb1) {
        if (li < n1) run1.piece(li, t, kb0, kb1);
        else run2.piece(li - n1, t, kb0, kb1);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 2);  // the weight and the batch producer each arrive with their bytes
            mbar_init(&empty[s], 1);
        }
        for (int j = 0; j < 2; ++j) {
            mbar_init(&acc_full[j], 1);
            mbar_init(&acc_empty[j], 4);
        }
        mbar_init(mma_done, 1);
        mbar_fence_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&a.mW_res);
        tma_prefetch_desc(&a.mW_head);
        tma_prefetch_desc(&a.mh);
        tma_prefetch_desc(&a.mhk);
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    sync_block();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 || warp == 2) {
        // ---------------- producers ----------------
        if (lane == 0) {
            const bool weights = warp == 0;
            const uint32_t bytes = weights ? kABytes : kBBytes;
            int it = 0;  // k-blocks issued (ring position)
            bool ok = true;
            for (int li = 0; li < ntiles && ok; ++li) {
                const bool res = li < n1;
                long t;
                int kb0, kb1;
                piece(li, t, kb0, kb1);
                const int k = (int)(res ? t / tph_r : t / tph_l);
                const int row0 = (int)(res ? t % tph_r : t % tph_l) * kTM;
                if (!weights && li == n1) {
                    // vocabulary tiles read h^(k): wait until every CTA wrote its rows
                    const uint64_t t0 = global_ns();
                    while (ld_acquire_u32(&a.ctr[0]) < gridDim.x) {
                        if (global_ns() - t0 > wait_ns) {
                            set_status(a.status, MEDUSA_STATUS_TIMEOUT);
                            ok = false;
                            break;
                        }
                        __nanosleep(100);
                    }
                    fence_proxy_async_global();
                    if (!ok) break;
                }
                for (int kb = kb0; kb < kb1; ++kb) {
                    const int s = it % S;
                    if (it >= S && !mbar_wait<true>(&empty[s], ((it / S) - 1) & 1, wait_ns)) {
                        set_status(a.status, MEDUSA_STATUS_TIMEOUT);
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], bytes);
                    if (weights)
                        tma_load_3d(sA + (size_t)s * kABytes, res ? &a.mW_res : &a.mW_head, kb * kTK, row0, k,
                                    &full[s]);
                    else if (res)
                        tma_load_2d(sB + (size_t)s * kBBytes, &a.mh, kb * kTK, 0, &full[s]);
                    else
                        tma_load_3d(sB + (size_t)s * kBBytes, &a.mhk, kb * kTK, k, 0, &full[s]);
                    ++it;
                }
            }
            // drain: no copy may still be landing when the CTA exits.  A stage's
            // phase also needs the other producer's arrival; if that producer
            // stopped early (a timed-out wait) the phase never completes, so the
            // whole drain has one deadline rather than one per stage (the copies
            // themselves land within microseconds).
            const uint64_t t_end = global_ns() + kWaitLimitNs;
            for (int s = 0; s < S && s < it; ++s) {
                const int last = s + ((it - 1 - s) / S) * S;
                const uint64_t now = global_ns();
                if (now >= t_end) break;
                mbar_wait<true>(&full[s], (last / S) & 1, t_end - now);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            bool ok = true;
            int it = 0;
            for (int li = 0; li < ntiles && ok; ++li) {
                const int buf = li & 1;
                if (li >= 2 && !mbar_wait<true>(&acc_empty[buf], ((li >> 1) - 1) & 1, wait_ns)) {
                    set_status(a.status, MEDUSA_STATUS_TIMEOUT);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + buf * N;
                long t;
                int kb0, kb1;
                piece(li, t, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb) {
                    const int s = it % S;
                    if (!mbar_wait<true>(&full[s], (it / S) & 1, wait_ns)) {
                        set_status(a.status, MEDUSA_STATUS_TIMEOUT);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = sw128_kmajor_desc(smem_addr(sA + (size_t)s * kABytes));
                    const uint64_t bdesc = sw128_kmajor_desc(smem_addr(sB + (size_t)s * kBBytes));
#pragma unroll
                    for (int ks = 0; ks < kTK / 16; ++ks)  // 16 k-elements = 32 bytes per MMA
                        tc_mma_bf16(d_tmem, adesc + 2 * ks, bdesc + 2 * ks, kIdesc, (kb != kb0 || ks != 0) ? 1u : 0u);
                    tc_commit(&empty[s]);
                    ++it;
                }
                tc_commit(&acc_full[buf]);
            }
            // every MMA this thread issued completes before TMEM is released
            tc_commit(mma_done);
            mbar_wait<true>(mma_done, 0);
        }
    } else {
        // ---------------- epilogue ----------------
        const int et = threadIdx.x - kEpiWarp0 * 32;  // 0..127
        const int ew = warp - kEpiWarp0;               // 0..3
        const int q = warp & 3;                        // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;                 // weight row of the tile held by this thread
        // transposed phase: this warp's units (see row_blocks), state in
        // shared memory that only the owning warp touches: per unit a lane
        // keeps the running max and sum of exp(x - max) of its rows (sU), and
        // the unit's top-8 list (sL) is read into lanes 0..7 when it changes
        const int R = epi_blocks(B, kUnits);      // row blocks (units) or segments per column
        const int rpu = (kTM + R - 1) / R;        // rows per unit or segment (units: R divides kTM)
        // segments: thread et takes column et % B, rows [r_lo, r_hi)
        const bool col_thread = et < B * R;
        const int col = et % B, seg = et / B;
        const int r_lo = col_thread ? seg * rpu : 0, r_hi = col_thread ? min(kTM, r_lo + rpu) : 0;
        float cm = -INFINITY, cl = 0.f;  // running max and sum of exp(x - cm)
        float lv[kTopK];
        int lx[kTopK];
        auto reset_units = [&]() {
            if constexpr (kUnits) {
                for (int u = ew; u < nunits; u += 4) {
                    sU[u * 32 + lane] = make_float2(-INFINITY, 0.f);
                    if (lane < kTopK) sL[u * kTopK + lane] = TopEntry{-INFINITY, INT_MAX};
                }
                __syncwarp();
            } else {
                cm = -INFINITY;
                cl = 0.f;
#pragma unroll
                for (int j = 0; j < kTopK; ++j) {
                    lv[j] = -INFINITY;
                    lx[j] = INT_MAX;
                }
            }
        };
        reset_units();
        int cur_k = -1;
        bool ok = true;
        auto flush = [&](int kk) {
            // each unit's state, its lanes' statistics merged by a butterfly,
            // (or each segment's) goes to stS[row block][column]
            if constexpr (!kUnits) {
                if (col_thread) {
                    HeadState* o = &stS[et];  // = [seg][col]
                    o->m = cm;
                    o->l = cl;
#pragma unroll
                    for (int j = 0; j < kTopK; ++j) {
                        o->val[j] = lv[j];
                        o->idx[j] = lx[j];
                    }
                }
            }
            for (int u = ew; kUnits && u < nunits; u += 4) {
                const float2 ml = sU[u * 32 + lane];
                float mm = ml.x, ll = ml.y;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float m2 = __shfl_xor_sync(kFull, mm, o);
                    const float l2 = __shfl_xor_sync(kFull, ll, o);
                    merge_ml(mm, ll, m2, l2);
                }
                HeadState* o = &stS[(u % R) * B + u / R];
                if (lane == 0) {
                    o->m = mm;
                    o->l = ll;
                }
                if (lane < kTopK) {
                    const TopEntry te = sL[u * kTopK + lane];
                    o->val[lane] = te.v;
                    o->idx[lane] = te.i;
                }
            }
            const int nseg = R;
            epi_sync();
            if (et < B) {
                // merge the column's row blocks in order
                float mm = -INFINITY, ll = 0.f;
                float mv[kTopK];
                int mi[kTopK];
#pragma unroll
                for (int j = 0; j < kTopK; ++j) {
                    mv[j] = -INFINITY;
                    mi[j] = INT_MAX;
                }
                for (int sg = 0; sg < nseg; ++sg) {
                    const HeadState* o = &stS[sg * B + et];
                    merge_ml(mm, ll, o->m, o->l);
                    for (int j = 0; j < kTopK; ++j) {  // each list is sorted: stop at the first that fails
                        const float v = o->val[j];
                        const int i = o->idx[j];
                        if (!beats(v, i, mv[kTopK - 1], mi[kTopK - 1])) break;
                        list_insert(mv, mi, v, i);
                    }
                }
                HeadState* dst = &a.part[((long)blockIdx.x * K + kk) * B + et];
                dst->m = mm;
                dst->l = ll;
#pragma unroll
                for (int j = 0; j < kTopK; ++j) {
                    dst->val[j] = mv[j];
                    dst->idx[j] = mi[j];
                }
            }
            if (a.merge_per_head) {
                // the last CTA to publish its partial of head kk merges the
                // head (every sequence), while its producers and MMA go on
                // streaming
                __threadfence();
                epi_sync();  // stS is free again; every partial of this CTA is written
                if (et == 0)
                    *last_flag = atomicAdd(&a.ctr[2 + 2 * G + kk], 1u) + 1u ==
                                 (unsigned)HeadCover(G, tph_l, nkb, K, kk).count();
                epi_sync();
                if (*last_flag) {
                    __threadfence();
                    for (int b = ew; b < B; b += 4)
                        merge_head(a.part, G, tph_l, nkb, B, b, b, a.V, K, kk,
                                   a.tree.base ? a.tree.at(b) : nullptr, a.tree.T, a.root_token, a.topk_idx,
                                   a.topk_prob, a.node_tokens, a.node_q, a.stats, a.status);
                }
            }
            epi_sync();  // stS is free again (and last_flag read) before the next flush
            reset_units();
        };
        auto arrive_grid = [&]() {
            // this CTA's h^(k) rows are written: publish them (also to the TMA proxy)
            fence_proxy_async_global();
            __threadfence();
            epi_sync();
            if (ew == 0 && lane == 0) atomicAdd(&a.ctr[0], 1u);
        };
        if (n1 == 0) arrive_grid();
        // A whole residual tile: its h rows are read into sT (free until the
        // first vocabulary tile) while the MMA streams the tile, so the
        // epilogue does not wait on them afterwards.
        const bool h_staged = T1 <= G && n1 == 1;
        if (h_staged) {
            const int o = (int)(cta % tph_r) * kTM + row;
            if (o < a.d) {
                for (int e0 = 0; e0 < B; e0 += 16) {
                    float hv[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        hv[e] = e0 + e < B ? __bfloat162float(a.h[(long)(e0 + e) * a.d + o]) : 0.f;
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        if (e0 + e < B) sT[(e0 + e) * kTS + row] = hv[e];
                }
            }
        }
        for (int li = 0; li < ntiles; ++li) {
            const int buf = li & 1;
            const int ph = li < n1 ? 0 : 1;
            const long U = ph == 0 ? U1 : U2;
            long t;
            int kb0, kb1;
            piece(li, t, kb0, kb1);
            // kb0 > 0: the later k-blocks of a tile owned by an earlier CTA (the
            // first piece of this CTA's run), handed over as a partial sum
            const bool handover = kb0 > 0;
            const bool res = li < n1;
            const int k = (int)(res ? t / tph_r : t / tph_l);
            const int row0 = (int)(res ? t % tph_r : t % tph_l) * kTM;
            if (!handover && !res) {
                if (k != cur_k) {
                    if (cur_k >= 0) flush(cur_k);
                    cur_k = k;
                }
                epi_sync();  // the previous tile's readers are done with sT
            }
            if (li == (ntiles >= 2 ? ntiles - 2 : 0)) {
                // the merges at the end of the kernel run from a cold
                // instruction cache: a dry merge while the last tiles stream
                // brings their code in on each epilogue warp's scheduler (the
                // last piece can be short, so this goes one piece earlier)
                merge_head(a.part, G, tph_l, nkb, B, 0, 0, a.V, K, cur_k >= 0 ? cur_k : 0,
                           a.tree.base ? a.tree.at(0) : nullptr, a.tree.T, a.root_token, a.topk_idx, a.topk_prob,
                           a.node_tokens, a.node_q, a.stats, a.status, true);
            }
            if (ok && !mbar_wait<true>(&acc_full[buf], (li >> 1) & 1, wait_ns)) {
                if (lane == 0) set_status(a.status, MEDUSA_STATUS_TIMEOUT);
                ok = false;
            }
            // an owned tile cut by a run boundary: its rest is the first pieces
            // of the next CTAs' runs, [cta + 1, c2_end), handed over by flags
            int c2_end = cta + 1;
            if (!handover && kb1 < nkb && ok) {
                const long tend = (t + 1) * nkb;
                for (int c2 = cta + 1; c2 < G && U * c2 / G < tend; ++c2) {
                    c2_end = c2 + 1;
                    if (U * (c2 + 1) / G == U * c2 / G) continue;  // an empty run
                    if (!wait_flag(&a.ctr[2 + ph * G + c2], wait_ns)) {
                        if (lane == 0) set_status(a.status, MEDUSA_STATUS_TIMEOUT);
                        ok = false;
                        break;
                    }
                }
            }
            // decided for the whole warp before its collective TMEM loads (the
            // lanes test barriers and flags independently)
            ok = __all_sync(kFull, ok);
            if (ok) tc_fence_after();
            const int o = row0 + row;  // residual: output element; vocabulary: token id
            // 16 columns (sequences) at a time from TMEM: few registers live.
            // Not unrolled: the residual tile's epilogue runs once per CTA, from
            // a cold instruction cache, and its four unrolled copies at N = 64
            // took 6 us each to fetch (22 against 10 us for the residual
            // epilogue, measured with per-CTA timestamps).
#pragma unroll 1
            for (int c = 0; c < N / 16; ++c) {
                float v[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = 0.f;
                if (ok) tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + buf * N + c * 16, v);
                if (handover) {
                    float* dst = a.slots + (long)(ph * G + cta) * B * kTM;
                    if (ok) {
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            if (c * 16 + e < B) dst[(c * 16 + e) * kTM + row] = v[e];
                    }
                    continue;
                }
                if (ok) {
                    for (int c2 = cta + 1; c2 < c2_end; ++c2) {
                        if (U * (c2 + 1) / G == U * c2 / G) continue;
                        const float* src = a.slots + (long)(ph * G + c2) * B * kTM;
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            if (c * 16 + e < B) v[e] += __ldcg(&src[(c * 16 + e) * kTM + row]);
                    }
                }
                if (res) {
                    // residual tile: h^(k)[b, o] = SiLU(z) + h[b, o]
                    if (ok && o < a.d) {
                        float hv[16];  // every load before the first store
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            hv[e] = c * 16 + e >= B ? 0.f
                                    : h_staged      ? sT[(c * 16 + e) * kTS + row]
                                                    : __bfloat162float(a.h[(long)(c * 16 + e) * a.d + o]);
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int bq = c * 16 + e;
                            if (bq < B) {
                                const float z = v[e];
                                // SiLU with the fast exponential and divide: their
                                // error is far below the bf16 rounding of h^(k), and
                                // the accurate divide's slow path (a denominator of
                                // inf when z < -88) made this loop 1/3 slower
                                const __nv_bfloat16 yb = __float2bfloat16_rn(__fdividef(z, 1.f + __expf(-z)) + hv[e]);
                                a.hk[((long)bq * K + k) * a.d + o] = yb;
                                if (a.hk_out) a.hk_out[((long)bq * K + k) * a.d + o] = yb;
                            }
                        }
                    }
                    continue;
                }
                // vocabulary tile
                if (a.logits && ok && o < a.V) {
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        if (c * 16 + e < B) a.logits[((long)(c * 16 + e) * K + k) * a.V + o] = v[e];
                }
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    if (c * 16 + e < B) sT[(c * 16 + e) * kTS + row] = v[e];
            }
            if (ok) tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
            if (handover) {
                __threadfence();
                epi_sync();
                if (et == 0) st_release_u32(&a.ctr[2 + ph * G + cta], 1u);
                if (li == n1 - 1) arrive_grid();
                continue;
            }
            if (res) {
                if (li == n1 - 1) arrive_grid();
                continue;
            }
            epi_sync();
            if (!kUnits && ok && col_thread) {
                const float* src = sT + col * kTS;
                const int hi = min(r_hi, a.V - row0);  // rows past V are zero-filled weights
                float tm = -INFINITY;
                for (int r = r_lo; r < hi; ++r) tm = fmaxf(tm, src[r]);
                if (tm > -INFINITY) {
                    const float mn = fmaxf(cm, tm);
                    float sum = 0.f;
                    for (int r = r_lo; r < hi; ++r) sum += expf(src[r] - mn);
                    cl = (cm == -INFINITY ? 0.f : cl * expf(cm - mn)) + sum;
                    cm = mn;
                }
                // top-8: every row goes through a branch-free insertion (kept
                // if it beats the last entry, then bubbled up).  Most rows of a
                // CTA's first tiles of a head are kept, so filtering first (and
                // inserting the survivors from a queue) cost more: 30 us on a
                // first tile against 8-12 us here, measured per CTA at B=64.
                for (int r = r_lo; r < hi; ++r) {
                    const float v = src[r];
                    const int i = row0 + r;
                    const bool in = beats(v, i, lv[kTopK - 1], lx[kTopK - 1]);
                    lv[kTopK - 1] = in ? v : lv[kTopK - 1];
                    lx[kTopK - 1] = in ? i : lx[kTopK - 1];
#pragma unroll
                    for (int j = kTopK - 1; j > 0; --j) {
                        const bool sw = beats(lv[j], lx[j], lv[j - 1], lx[j - 1]);
                        const float a0 = lv[j], b0 = lv[j - 1];
                        const int ai = lx[j], bi = lx[j - 1];
                        lv[j - 1] = sw ? a0 : b0;
                        lv[j] = sw ? b0 : a0;
                        lx[j - 1] = sw ? ai : bi;
                        lx[j] = sw ? bi : ai;
                    }
                }
            }
            if (kUnits && ok) {
                for (int u = ew; u < nunits; u += 4) {
                    const int rb = u % R;
                    const float* src = sT + (u / R) * kTS + rb * rpu;
                    const int base = row0 + rb * rpu;
                    // lane-row j of the unit is row base + 32 j + lane (rows
                    // past V are zero-filled weights and take no part)
                    float x[4];
                    bool in[4];
                    float tm = -INFINITY;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        in[j] = 32 * j < rpu && base + 32 * j + lane < a.V;
                        x[j] = in[j] ? src[32 * j + lane] : -INFINITY;
                        tm = fmaxf(tm, x[j]);
                    }
                    if (tm > -INFINITY) {
                        float2 ml = sU[u * 32 + lane];
                        const float mn = fmaxf(ml.x, tm);
                        float sum = 0.f;
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            if (in[j]) sum += expf(x[j] - mn);
                        ml.y = (ml.x == -INFINITY ? 0.f : ml.y * expf(ml.x - mn)) + sum;
                        ml.x = mn;
                        sU[u * 32 + lane] = ml;
                    }
                    // top-8: the rows beating the list's last entry are the
                    // candidates; the best remaining one is inserted while it
                    // still beats the last entry (at most kTopK rounds, fewer
                    // once the list holds the head's large values)
                    const TopEntry last = sL[u * kTopK + kTopK - 1];
                    unsigned mine = 0u;  // bit j: lane-row j is a remaining candidate
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (in[j] && beats(x[j], base + 32 * j + lane, last.v, last.i)) mine |= 1u << j;
                    if (__any_sync(kFull, mine != 0u)) {
                        TopEntry te = lane < kTopK ? sL[u * kTopK + lane] : TopEntry{-INFINITY, INT_MAX};
                        for (int round = 0; round < kTopK; ++round) {
                            float bv = -INFINITY;
                            int bi = INT_MAX, bj = -1;
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                if (((mine >> j) & 1u) && beats(x[j], base + 32 * j + lane, bv, bi)) {
                                    bv = x[j];
                                    bi = base + 32 * j + lane;
                                    bj = j;
                                }
                            }
                            float wv = bv;
                            int wi = bi;
#pragma unroll
                            for (int o2 = 16; o2 > 0; o2 >>= 1) {
                                const float ov = __shfl_xor_sync(kFull, wv, o2);
                                const int oi = __shfl_xor_sync(kFull, wi, o2);
                                if (beats(ov, oi, wv, wi)) {
                                    wv = ov;
                                    wi = oi;
                                }
                            }
                            const float tv = __shfl_sync(kFull, te.v, kTopK - 1);
                            const int ti = __shfl_sync(kFull, te.i, kTopK - 1);
                            if (wi == INT_MAX) break;  // no candidate left (wi, wv, tv, ti: the warp's)
                            if (!beats(wv, wi, tv, ti)) break;
                            warp_list_insert(te.v, te.i, wv, wi);
                            if (bi == wi) mine &= ~(1u << bj);  // its lane drops it (row ids are unique)
                        }
                        if (lane < kTopK) sL[u * kTopK + lane] = te;
                        __syncwarp();
                    }
                }
            }
        }
        if (cur_k >= 0) flush(cur_k);
    }

    // ---------------- teardown ----------------
    tc_fence_before();
    sync_block();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (a.merge_per_head) return;
    // many sequences: a grid barrier (every CTA's partials are written), then
    // the (sequence, head) merges spread over all warps of the grid
    __threadfence();
    sync_block();
    if (threadIdx.x == 0) {
        *last_flag = 0;
        atomicAdd(&a.ctr[1], 1u);
        const uint64_t t0 = global_ns();
        while (ld_acquire_u32(&a.ctr[1]) < gridDim.x) {
            if (global_ns() - t0 > wait_ns) {
                set_status(a.status, MEDUSA_STATUS_TIMEOUT);
                *last_flag = 1;
                break;
            }
            __nanosleep(64);
        }
    }
    sync_block();
    if (*last_flag) return;
    __threadfence();
    for (int p = blockIdx.x * kTcWarps + warp; p < B * K; p += gridDim.x * kTcWarps) {
        const int b = p % B, k = p / B;
        merge_head(a.part, gridDim.x, tph_l, nkb, B, b, b, a.V, K, k, a.tree.base ? a.tree.at(b) : nullptr, a.tree.T,
                   a.root_token, a.topk_idx, a.topk_prob, a.node_tokens, a.node_q, a.stats, a.status);
    }
}

template <int N>
size_t tc_smem_bytes(int stages, int B) {
    return 1024 + (size_t)stages * (kABytes + N * kTK * 2) + (2 * (size_t)stages + 5) * 8 + 16 +
           (size_t)((B * kTS + 3) & ~3) * 4 +
           (units_epilogue<N>() ? (size_t)B * row_blocks(B) * (sizeof(HeadState) + 32 * sizeof(float2) + kTopK * 8)
                                : (size_t)B * seg_per_col(B) * sizeof(HeadState));
}

// as many stages as shared memory holds (at most 16): the weight bytes in
// flight per SM set the stream rate
template <int N>
int tc_stages(int B) {
    int s = 16;
    while (s > 2 && tc_smem_bytes<N>(s, B) > (size_t)kSmemBudget) --s;
    return s;
}

template <int N>
cudaError_t launch_n(const TcHeadsArgs& args, cudaStream_t st) {
    TcHeadsArgs a = args;
    a.stages = tc_stages<N>(a.B);
    const size_t smem = tc_smem_bytes<N>(a.stages, a.B);
    auto kern = a.wait_ns == kWaitLimitNs ? heads_tc_kernel<N, false> : heads_tc_kernel<N, true>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    prefer_max_smem(kern);
    cudaLaunchConfig_t cfg = {};
    // one CTA per SM, or fewer when the caller leaves SMs to other streams
    const int cap = launch_heads_ctas();
    cfg.gridDim = dim3(cap > 0 && cap < num_sms() ? cap : num_sms());
    cfg.blockDim = dim3(kTcWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace

bool heads_tc_supported(int B, int d, medusa_dtype dt) { return dt == MEDUSA_BF16 && B >= 1 && B <= 64 && d % 8 == 0; }

cudaError_t heads_tc_launch(const HeadsArgs& x, void* hk, void* part, unsigned int* ctr, float* slots, float2* stats,
                            float* logits, cudaStream_t st) {
    TcHeadsArgs a;
    const uint64_t d = x.d, V = x.V, K = x.K, B = x.B;
    const int N = (x.B + 15) / 16 * 16;
    {
        const uint64_t dims[3] = {d, d, K}, strides[2] = {d * 2, d * d * 2};
        const uint32_t box[3] = {kTK, kTM, 1};
        if (!make_tmap_bf16(&a.mW_res, x.W_res, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[3] = {d, V, K}, strides[2] = {d * 2, V * d * 2};
        const uint32_t box[3] = {kTK, kTM, 1};
        if (!make_tmap_bf16(&a.mW_head, x.W_head, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[2] = {d, B}, strides[1] = {d * 2};
        const uint32_t box[2] = {kTK, (uint32_t)N};
        if (!make_tmap_bf16(&a.mh, x.h, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[3] = {d, K, B}, strides[2] = {d * 2, K * d * 2};
        const uint32_t box[3] = {kTK, 1, (uint32_t)N};
        if (!make_tmap_bf16(&a.mhk, hk, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    a.h = (const __nv_bfloat16*)x.h;
    a.hk = (__nv_bfloat16*)hk;
    a.hk_out = (__nv_bfloat16*)x.h_res_out;
    a.logits = logits;
    a.part = (HeadState*)part;
    a.ctr = ctr;
    a.slots = slots;
    a.tree = x.tree;
    a.root_token = x.root_token;
    a.topk_idx = x.topk_idx;
    a.topk_prob = x.topk_prob;
    a.node_tokens = x.node_tokens;
    a.node_q = x.node_q;
    a.stats = stats;
    a.status = x.status;
    a.B = x.B;
    a.d = x.d;
    a.V = x.V;
    a.K = x.K;
    a.merge_per_head = x.B <= kMergePerHeadMaxB;
    a.wait_ns = wait_limit_ns();
    cudaError_t e = cudaMemsetAsync(ctr, 0, (size_t)(2 + 2 * num_sms() + x.K) * sizeof(unsigned int), st);
    if (e != cudaSuccess) return e;
    switch (N) {
        case 16: return launch_n<16>(a, st);
        case 32: return launch_n<32>(a, st);
        case 48: return launch_n<48>(a, st);
        default: return launch_n<64>(a, st);
    }
}

}  // namespace medusa
