// Shared device-side definitions of libmedusa (B200, sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "medusa.h"

namespace medusa {

// Prefer the largest shared-memory carveout for a kernel: the heads and
// tensor-core attention kernels need it, and when every kernel of a step asks
// for the same split, an SM is never reconfigured between back-to-back
// launches.
template <typename Kernel>
inline void prefer_max_smem(Kernel kernel) {
    // a hint: if the driver refuses it, drop the error so the launch's own
    // status check does not report it
    if (cudaFuncSetAttribute(reinterpret_cast<const void*>(kernel), cudaFuncAttributePreferredSharedMemoryCarveout,
                             100) != cudaSuccess)
        (void)cudaGetLastError();
}

constexpr int kMaxTree = MEDUSA_MAX_TREE;  // nodes per tree
constexpr int kTopK = MEDUSA_TOPK;         // entries kept per head
constexpr unsigned kFull = 0xffffffffu;

// Candidate tree as the kernels read it (device memory, built once by
// medusa_tree_create).  Children of a node are child_idx[child_off[u] ..
// child_off[u+1]) in increasing index order.  anc[i] has bit j set when node j
// is node i or one of its ancestors (the tree attention mask row of node i).
struct TreeDev {
    int T;
    int max_depth;
    int max_children;
    int pad;
    int16_t parent[kMaxTree];
    uint8_t depth[kMaxTree];
    uint8_t rank[kMaxTree];
    uint8_t child_off[kMaxTree + 4];
    uint8_t child_idx[kMaxTree];
    uint32_t anc[kMaxTree][4];
};

// The tree(s) of a call: one tree shared by every sequence (stride 0) or one
// per sequence (stride 1).  T is the node dimension of the [B, T, ...] arrays
// of the call (the largest tree's node count); sequence b uses its own
// tree's first at(b)->T rows of them.
struct TreeRef {
    const TreeDev* base;
    int stride;
    int T;
    __host__ __device__ const TreeDev* at(int b) const { return base + (long)b * stride; }
};

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
    return x;
}

// 16-byte streaming load of read-only data that is used once (weights):
// bypasses L1 allocation and asks L2 for 256-byte sectors.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// 16-byte read-only load that may stay in L1 (small vectors reused by a CTA).
__device__ __forceinline__ uint4 ld_nc(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Element-type traits: number of elements in 16 bytes and conversions.
template <typename T>
struct Elt;
template <>
struct Elt<float> {
    static constexpr int kVec = 4;
    __device__ __forceinline__ static void unpack(const uint4& v, float* f) {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
    __device__ __forceinline__ static float to_float(float x) { return x; }
    __device__ __forceinline__ static float from_float(float x) { return x; }
    // the largest of the vector's elements; NaN only when all are NaN
    __device__ __forceinline__ static float vmax(const uint4& v) {
        return fmaxf(fmaxf(__uint_as_float(v.x), __uint_as_float(v.y)), fmaxf(__uint_as_float(v.z), __uint_as_float(v.w)));
    }
};
template <>
struct Elt<__nv_bfloat16> {
    static constexpr int kVec = 8;
    __device__ __forceinline__ static void unpack(const uint4& v, float* f) {
        f[0] = bf16lo(v.x);
        f[1] = bf16hi(v.x);
        f[2] = bf16lo(v.y);
        f[3] = bf16hi(v.y);
        f[4] = bf16lo(v.z);
        f[5] = bf16hi(v.z);
        f[6] = bf16lo(v.w);
        f[7] = bf16hi(v.w);
    }
    __device__ __forceinline__ static float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
    __device__ __forceinline__ static __nv_bfloat16 from_float(float x) { return __float2bfloat16_rn(x); }
    // the largest of the vector's elements (exact: a maximum rounds nothing);
    // the paired maximum returns the other operand when one is NaN, so the
    // result is NaN only when all eight are
    __device__ __forceinline__ static float vmax(const uint4& v) {
        const __nv_bfloat162 m = __hmax2(__hmax2(pair(v.x), pair(v.y)), __hmax2(pair(v.z), pair(v.w)));
        return fmaxf(__low2float(m), __high2float(m));
    }
    __device__ __forceinline__ static __nv_bfloat162 pair(uint32_t u) {
        __nv_bfloat162 r;
        memcpy(&r, &u, 4);
        return r;
    }
};

// ---------------------------------------------------------------------------
// mbarrier + bulk asynchronous copy (TMA engine, no tensor map)
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

// make initialised barriers visible to the async (bulk-copy) proxy
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

// kSuspend: the waiting thread is suspended until the phase completes or
// kSuspendHintNs pass.  Without the hint try_wait returns after a short
// hardware-chosen time and the wait loop spins.  In the heads kernel (deep
// buffering, waits of whole tiles) the spinning producer, MMA and epilogue
// threads cost 9% of the weight stream at llama8b (752 against 687 us on one
// box); in tree attention, whose softmax and MMA threads hand each chunk back
// and forth, the suspended threads woke too late (32k keys: 95 against 100 us),
// so there the waits spin.
constexpr uint32_t kSuspendHintNs = 2000;

template <bool kSuspend = false>
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    if (kSuspend)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_addr(bar)), "r"(parity), "r"(kSuspendHintNs)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_addr(bar)), "r"(parity)
            : "memory");
    return ok != 0;
}

// non-blocking test of the phase with the given parity
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Limit of every wait in the kernels: about two seconds.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Wait for the phase of `bar` with the given parity to complete, giving up
// after limit_ns (returns false then).  Used by every pipeline wait so that a
// protocol error ends the kernel instead of hanging the GPU.  limit_ns <= 1
// gives up at once unless the phase is already complete (a test of the
// error paths; see medusa_debug_set_wait_limit).
template <bool kSuspend = false>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
    if (limit_ns <= 1) return mbar_test(bar, parity);
    if (mbar_try_wait<kSuspend>(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait<kSuspend>(bar, parity)) return true;
        if ((i & (kSuspend ? 15u : 255u)) == 0 && global_ns() - t0 > limit_ns) return false;
    }
}

// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) from
// global to this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void set_status(int32_t* status, int bits) {
    if (status) atomicOr(status, bits);
}

// Total order of (value, index) candidates used by top-s and argmax: a larger
// value wins; among equal values the lower index wins; NaN never wins.
// Block-wide barrier after code in which the lanes of a warp took different
// paths (lane 0 running a producer or MMA loop while the others wait, say).
// The barrier behind __syncthreads is an aligned one: it must be reached by
// whole warps, and a warp that arrives with some lanes still elsewhere is
// counted wrongly (the barrier can release early).  Each warp reconverges
// first.
__device__ __forceinline__ void sync_block() {
    __syncwarp();
    __syncthreads();
}

__device__ __forceinline__ bool beats(float v, int i, float w, int j) { return v > w || (v == w && i < j); }

}  // namespace medusa
