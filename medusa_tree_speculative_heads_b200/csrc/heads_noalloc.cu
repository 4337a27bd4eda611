// medusa_heads without a caller-supplied workspace.
//
// Some callers cannot allocate device memory at all: a plug-in running
// inside a host framework that owns every byte of the GPU's memory and hands
// out no allocator, or a serving loop that must never call cudaMalloc /
// cudaFree because those calls synchronise the whole device.  For them this
// file keeps the heads' scratch in a fixed array in the library's own device
// memory (allocated by the driver when the library's code is loaded onto a
// GPU, and held by every GPU that loads it until the process exits), and
// forwards to medusa_heads with that array as the workspace.
#include <stdio.h>

#include "kernels.h"

namespace medusa {
int report_error(int code, const char* msg);
}

namespace {

// Largest workspace the scratch-free variant serves (32 MiB per GPU).
constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;

// The scratch itself.  Host code must not use this name as an address: on the
// host it is only a stand-in symbol; the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_heads_scratch[kNoAllocScratchBytes];

// Device address of g_heads_scratch on the current device, with that device
// current.  Looked up on every call (a host-side table lookup once the
// library's module is loaded), never cached: a primary context that was reset
// and re-created reloads the module, and an address kept from before would
// then point at memory the new context does not own.
int scratch_address(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_heads_scratch);
    if (e != cudaSuccess || !p) {
        char msg[256];
        snprintf(msg, sizeof msg, "medusa_heads_noalloc: cudaGetSymbolAddress of the scratch failed (%s)",
                 cudaGetErrorString(e));
        return medusa::report_error(MEDUSA_ERR_CUDA, msg);
    }
    *out = p;
    return MEDUSA_OK;
}

}  // namespace

extern "C" int medusa_heads_noalloc(const void* h, const void* W_res, const void* W_head, int B, int d, int V, int K,
                                    medusa_dtype dt, const medusa_tree* tree, const int32_t* root_token,
                                    int32_t* topk_idx, float* topk_prob, int32_t* node_tokens, float* node_q,
                                    void* h_res_out, float* logits_out, float* probs_out, int32_t* status,
                                    medusa_stream_t stream) {
    const size_t need = medusa_heads_workspace_size(B, d, V, K, dt);
    if (need > kNoAllocScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "medusa_heads_noalloc: these sizes need %zu bytes of scratch, above the fixed %zu-byte array; "
                 "use medusa_heads with a workspace",
                 need, kNoAllocScratchBytes);
        return medusa::report_error(MEDUSA_ERR_UNSUPPORTED, msg);
    }
    void* ws = nullptr;
    int rc = scratch_address(&ws);
    if (rc != MEDUSA_OK) return rc;
    return medusa_heads(h, W_res, W_head, B, d, V, K, dt, tree, root_token, topk_idx, topk_prob, node_tokens, node_q,
                        h_res_out, logits_out, probs_out, ws, kNoAllocScratchBytes, status, stream);
}
