// Test hooks of libspecverify (include/specverify_testing.h): the device Philox
// block function over a list of counters, and the attention call with one wait
// per CTA made to run out.
#include "../../include/specverify_testing.h"
#include "sv_device.cuh"
#include "sv_internal.h"

namespace sv {

// One thread per counter; the same philox4x32_10 that sv_accept's kernels use.
__global__ void philox_words_kernel(PhiloxKey key, const uint4 *__restrict__ ctr, uint4 *__restrict__ out,
                                    int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = philox4x32_10(ctr[i], key);
}

}  // namespace sv

extern "C" sv_status sv_testing_philox4x32_10(uint64_t key, const uint32_t *counters, uint32_t *out, int64_t n,
                                              void *stream) {
    if (n < 0 || n > ((int64_t)1 << 31)) {
        sv::record_error("n must be in [0, 2^31]");
        return SV_ERR_INVALID_ARG;
    }
    if (n == 0) return SV_OK;
    if (!counters || !out || (reinterpret_cast<uintptr_t>(counters) & 15) || (reinterpret_cast<uintptr_t>(out) & 15)) {
        sv::record_error("counters and out must be non-NULL and 16-byte aligned");
        return SV_ERR_INVALID_ARG;
    }
    const sv::PhiloxKey k{(uint32_t)(key & 0xFFFFFFFFull), (uint32_t)(key >> 32)};
    const int threads = 256;
    const int64_t want = (n + threads - 1) / threads;
    const unsigned blocks = (unsigned)(want < 4096 ? want : 4096);
    sv::philox_words_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
        k, reinterpret_cast<const uint4 *>(counters), reinterpret_cast<uint4 *>(out), n);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        sv::record_error(cudaGetErrorString(e));
        return SV_ERR_CUDA;
    }
    return SV_OK;
}

extern "C" sv_status sv_testing_verify_attention_stalled(const sv_attn_desc *desc, const void *q,
                                                         const sv_paged_kv *paged_kv, const int32_t *block_table,
                                                         const int32_t *ctx_lens, const uint64_t *draft_mask,
                                                         void *out, void *workspace, size_t workspace_bytes,
                                                         int32_t *status_flags, uint64_t wait_limit_ns,
                                                         void *stream) {
    if (wait_limit_ns < 1000000ull || wait_limit_ns > 2000000000ull) {
        sv::record_error("wait_limit_ns must be in [1 ms, 2 s]");
        return SV_ERR_INVALID_ARG;
    }
    return sv::verify_attention_entry(desc, q, paged_kv, block_table, ctx_lens, draft_mask, out, workspace,
                                      workspace_bytes, status_flags, stream, wait_limit_ns, 1);
}
