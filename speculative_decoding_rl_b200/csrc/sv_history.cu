// sv_history_draft: weight-free drafts from earlier responses (History Tree
// PR: drafts from earlier rollouts' high-reward responses of the same prompt,
// with a global fallback; SRT review: prefix lookup in earlier rollouts).
//
// One CTA per sequence. Its last K tokens are the key; every (response,
// position) pair is tested in parallel, first among the responses of the
// sequence's group, then among all responses if none matched. The winner is
// the highest reward, then the lowest response index (one 64-bit shared
// atomicMax over (order-preserving reward bits, ~h)), then the first position
// in that response (atomicMin). The up to gamma tokens after it are the
// drafts; each draft row of the one-hot draft probabilities is written too.
#include "sv_device.cuh"
#include "sv_internal.h"

namespace sv {

constexpr int HIST_THREADS = 256;

struct HistoryParams {
    const int32_t *htok, *hlen, *hgroup, *stok, *slen, *sgroup;
    const float *hreward;
    int32_t *drafts, *dlen;
    float *probs;
    int B, H, hstride, sstride, K, gamma, V;
};

// float -> uint32 whose unsigned order is the float order
SV_DEV uint32_t ordered_bits(float x) {
    const uint32_t u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(HIST_THREADS) history_draft_kernel(const HistoryParams P) {
    __shared__ int32_t key[64];
    __shared__ unsigned long long best;
    __shared__ int best_p;
    const int b = blockIdx.x, tid = threadIdx.x, K = P.K;
    // lengths are device data: clamp them to their rows so no read leaves a row
    const int L = min(P.slen[b], P.sstride);
    const bool has_key = L >= K;
    if (has_key && tid < K) key[tid] = P.stok[(size_t)b * P.sstride + L - K + tid];
    if (tid == 0) { best = 0ull; best_p = 0x7fffffff; }
    __syncthreads();
    const int g = P.sgroup[b];
    auto hl = [&](int h) { return max(0, min(P.hlen[h], P.hstride)); };
    auto match = [&](int h, int p) -> bool {
        if (p + K >= hl(h)) return false;  // a token must follow the key
        const int32_t *t = P.htok + (size_t)h * P.hstride + p;
        for (int i = 0; i < K; ++i)
            if (t[i] != key[i]) return false;
        return true;
    };
    const long long total = (long long)P.H * P.hstride;
    for (int pass = 0; pass < 2 && has_key; ++pass) {
        for (long long e = tid; e < total; e += HIST_THREADS) {
            const int h = (int)(e / P.hstride), p = (int)(e - (long long)h * P.hstride);
            if (pass == 0 && P.hgroup[h] != g) continue;
            if (match(h, p))
                atomicMax(&best, ((unsigned long long)ordered_bits(P.hreward[h]) << 32) | (0xffffffffu - (uint32_t)h));
        }
        __syncthreads();
        if (best != 0ull) break;  // uniform: every thread reads the same shared value
        __syncthreads();
    }
    const bool found = best != 0ull;
    const int hb = found ? (int)(0xffffffffu - (uint32_t)(best & 0xffffffffull)) : 0;
    if (found) {
        for (int p = tid; p < P.hstride; p += HIST_THREADS)
            if (match(hb, p)) atomicMin(&best_p, p);
    }
    __syncthreads();
    const int start = found ? best_p + K : 0;
    const int hlb = found ? hl(hb) : 0;
    if (tid < P.gamma) {
        const bool ok = found && start + tid < hlb;
        P.drafts[(size_t)b * P.gamma + tid] = ok ? P.htok[(size_t)hb * P.hstride + start + tid] : 0;
    }
    if (tid == 0) P.dlen[b] = found ? min(P.gamma, hlb - start) : 0;
    if (P.probs && P.V > 0) {
        float *rows = P.probs + (size_t)b * P.gamma * P.V;
        const size_t n = (size_t)P.gamma * P.V;
        for (size_t e = tid; e < n; e += HIST_THREADS) rows[e] = 0.f;
        __syncthreads();
        if (tid < P.gamma) {
            const bool ok = found && start + tid < hlb;
            const int t = ok ? P.htok[(size_t)hb * P.hstride + start + tid] : 0;
            if (t >= 0 && t < P.V) rows[(size_t)tid * P.V + t] = 1.f;
        }
    }
}

cudaError_t launch_history_draft(const HistoryLaunch &h, cudaStream_t stream) {
    HistoryParams P;
    P.htok = h.htok; P.hlen = h.hlen; P.hgroup = h.hgroup; P.hreward = h.hreward;
    P.stok = h.stok; P.slen = h.slen; P.sgroup = h.sgroup;
    P.drafts = h.drafts; P.dlen = h.dlen; P.probs = h.probs;
    P.B = h.B; P.H = h.H; P.hstride = h.hstride; P.sstride = h.sstride; P.K = h.K; P.gamma = h.gamma; P.V = h.V;
    history_draft_kernel<<<(unsigned)h.B, HIST_THREADS, 0, stream>>>(P);
    return cudaGetLastError();
}

}  // namespace sv
