// sv_verify_attention_noalloc: verify attention for callers that cannot
// allocate device memory.
//
// sv_verify_attention needs a caller-provided workspace for the partial
// results of the split-context pass. Some callers cannot obtain one: code
// that runs inside an engine or framework which owns every device buffer and
// forbids allocation while it executes, plugins that are handed only their
// input and output tensors, or host threads that must not call cudaMalloc
// because it can implicitly synchronise the device. This entry point serves
// them by using a fixed scratch array that is part of the library's device
// image instead of a workspace argument. It allocates nothing: no cudaMalloc,
// no cudaFree, no allocating library routine.
//
// Set-up: the first call on each device looks up that device's copy of the
// scratch array (cudaGetSymbolAddress, with the device current) and caches
// the address; make that first call before any stream capture. A lookup that
// fails is not cached: the call returns SV_ERR_CUDA and the next call tries
// again. All calls on
// a device share the one array and it keeps whatever the last call left in
// it; the kernels write every scratch word before they read it, so nothing
// needs clearing. Two calls whose executions overlap on the GPU (on different
// streams, say) race on the array and may both return wrong results: order
// them on one stream or with events.
#include <stdio.h>

#include <mutex>

#include "sv_internal.h"

namespace {

// Held by every GPU that loads the library, until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_lookup_mutex;
void *g_scratch_ptr[kMaxDevices];  // set once a lookup on that device succeeded

// The address of `dev`'s copy of the scratch array (dev is current), or null.
// Only a successful lookup is kept: a failed one (say, made while a stream was
// being captured) is retried by the next call, and its error is cleared from
// the runtime so that it is not reported later as another call's failure.
void *scratch_address(int dev) {
    std::lock_guard<std::mutex> lock(g_lookup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) == cudaSuccess) {
            g_scratch_ptr[dev] = ptr;
        } else {
            (void)cudaGetLastError();
        }
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" sv_status sv_verify_attention_noalloc(const sv_attn_desc *desc, const void *q,
                                                 const sv_paged_kv *paged_kv, const int32_t *block_table,
                                                 const int32_t *ctx_lens, const uint64_t *draft_mask,
                                                 void *out, int32_t *status_flags, void *stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        sv::record_error("cannot query the current device");
        return SV_ERR_CUDA;
    }
    // the caller's current device is `dev`; the symbol's address is per device
    void *scratch = scratch_address(dev);
    if (scratch == nullptr) {
        sv::record_error("cannot look up the scratch array on the current device");
        return SV_ERR_CUDA;
    }
    const size_t need = sv_verify_attention_workspace_size(desc);
    if (need > SV_NOALLOC_SCRATCH_BYTES) {
        // over the fixed scratch: refuse before anything is launched
        char msg[160];
        snprintf(msg, sizeof msg, "request needs %zu bytes of scratch, the built-in array holds %zu",
                 need, (size_t)SV_NOALLOC_SCRATCH_BYTES);
        sv::record_error(msg);
        return SV_ERR_WORKSPACE;
    }
    return sv_verify_attention(desc, q, paged_kv, block_table, ctx_lens, draft_mask, out,
                               scratch, SV_NOALLOC_SCRATCH_BYTES, status_flags, stream);
}
