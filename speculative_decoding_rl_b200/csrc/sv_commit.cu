// sv_kv_commit: keep the root and the accepted draft nodes of every sequence,
// compacted behind the root in path order, in every layer and KV head (the
// verified tree's accepted path continues the sequence: SRT review,
// "Speculative Rollout integration"; results built on a rejected draft are
// discarded: TLT reading notes, "1. RL and SD").
//
// One CTA per (sequence, KV head, layer): the sequence is validated, then all
// accepted rows of K and V are staged in shared memory before any is written
// (a destination can be another move's source). A chain (path 1..a) moves
// nothing. Pure data movement: 16-byte loads and stores of whole rows.
#include "sv_device.cuh"
#include "sv_internal.h"

namespace sv {

constexpr int COMMIT_THREADS = 128;

struct CommitParams {
    const int32_t *block_table, *ctx_lens, *accept_len, *accept_path;
    int32_t *new_ctx, *status;
    int B, N, Hkv, D, max_blocks, num_blocks, L;
    uint16_t *k[SV_COMMIT_MAX_LAYERS];
    uint16_t *v[SV_COMMIT_MAX_LAYERS];
};

__global__ void __launch_bounds__(COMMIT_THREADS) kv_commit_kernel(const __grid_constant__ CommitParams P) {
    extern __shared__ uint4 stage[];  // [a][2][D/8]: K row, V row
    const int b = blockIdx.x, h = blockIdx.y, l = blockIdx.z, tid = threadIdx.x;
    const int N = P.N, D = P.D;
    const int C = P.ctx_lens[b];
    const int *tbl = P.block_table + (size_t)b * P.max_blocks;
    const int *path = P.accept_path + (size_t)b * (N > 1 ? N - 1 : 1);
    int f = 0;
    if (C < N || C > P.max_blocks * PAGE) f |= SV_FLAG_BAD_CONTEXT;
    if (!f)
        for (int pg = (C - N) / PAGE; pg <= (C - 1) / PAGE; ++pg)
            if (tbl[pg] < 0 || tbl[pg] >= P.num_blocks) { f |= SV_FLAG_BAD_BLOCK; break; }
    const int a = P.accept_len[b];
    if (a < 0 || a > N - 1) {
        f |= SV_FLAG_BAD_PATH;
    } else {
        for (int k = 0, prev = 0; k < a; ++k) {
            const int node = path[k];
            if (node < 1 || node > N - 1 || node <= prev) { f |= SV_FLAG_BAD_PATH; break; }
            prev = node;
        }
    }
    if (h == 0 && l == 0 && tid == 0) {
        P.new_ctx[b] = f ? C : C - N + 1 + a;
        if (P.status) P.status[b] = f;
    }
    if (f) return;
    bool moves = false;
    for (int k = 0; k < a; ++k) moves |= path[k] != k + 1;
    if (!moves) return;  // a chain: every accepted row is already in place

    const int v8 = D / 8;  // 16-byte vectors per row
    uint16_t *kp = P.k[l], *vp = P.v[l];
    auto row = [&](uint16_t *pool, int t) -> uint4 * {
        return reinterpret_cast<uint4 *>(pool + (((size_t)tbl[t / PAGE] * P.Hkv + h) * PAGE + t % PAGE) * D);
    };
    for (int e = tid; e < a * 2 * v8; e += COMMIT_THREADS) {
        const int k = e / (2 * v8), rem = e - k * 2 * v8, kv = rem / v8, x = rem - kv * v8;
        stage[e] = row(kv ? vp : kp, C - N + path[k])[x];
    }
    __syncthreads();
    for (int e = tid; e < a * 2 * v8; e += COMMIT_THREADS) {
        const int k = e / (2 * v8), rem = e - k * 2 * v8, kv = rem / v8, x = rem - kv * v8;
        row(kv ? vp : kp, C - N + 1 + k)[x] = stage[e];
    }
}

cudaError_t launch_kv_commit(const CommitLaunch &c, cudaStream_t stream) {
    CommitParams P;
    P.block_table = c.block_table;
    P.ctx_lens = c.ctx_lens;
    P.accept_len = c.accept_len;
    P.accept_path = c.accept_path;
    P.new_ctx = c.new_ctx;
    P.status = c.status;
    P.B = c.B;
    P.N = c.N;
    P.Hkv = c.Hkv;
    P.D = c.D;
    P.max_blocks = c.max_blocks;
    P.num_blocks = c.num_blocks;
    P.L = c.L;
    for (int i = 0; i < SV_COMMIT_MAX_LAYERS; ++i) {
        P.k[i] = i < c.L ? c.k[i] : nullptr;
        P.v[i] = i < c.L ? c.v[i] : nullptr;
    }
    const size_t smem = (size_t)(c.N - 1 > 0 ? c.N - 1 : 1) * 2 * c.D * sizeof(uint16_t);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kv_commit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kv_commit_kernel<<<dim3((unsigned)c.B, (unsigned)c.Hkv, (unsigned)c.L), COMMIT_THREADS, smem, stream>>>(P);
    return cudaGetLastError();
}

}  // namespace sv
