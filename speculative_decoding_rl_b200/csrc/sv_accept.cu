// sv_accept: vocab-wide temperature softmax, accept test, tree/chain walk and
// residual resampling for the speculative-decoding verify step.
//
// One thread-block cluster of ACC_CLUSTER CTAs handles one sequence; CTA k of
// the cluster owns the vocabulary slice [k*chunk, (k+1)*chunk) of every row.
// Row statistics and every walk decision are reduced across the cluster
// through distributed shared memory (DSMEM), so the whole step is one launch,
// reads each logit once (plus the rows the walk rejects at, once more), and
// needs no workspace. Every CTA evaluates every decision from the same
// reduced values in the same order, so all CTAs of a cluster take identical
// control flow.
//
// The rule is the lossless one (Accelerating RL Post-Training Rollouts via
// System-Integrated Speculative Decoding, Abstract): accept draft i while
// u_i < min(1, p_i/q_i), drafts after the first rejection are discarded (TLT
// reading notes, "1. RL and SD"), and the emitted token is drawn from
// norm(max(0, p - q)) at the rejection, or from p after the last draft. Draft
// trees (SRT review, "Speculative Rollout integration", step 5) are walked as
// recursive rejection sampling over each accepted node's children in index
// order, which is the chain rule when every node has one child.
#include <cooperative_groups.h>

#include <algorithm>

#include "sv_device.cuh"
#include "sv_internal.h"
#include "sv_tc.cuh"

namespace cg = cooperative_groups;

namespace sv {

using namespace tc;

constexpr int ACC_CLUSTER = 8;
constexpr int ACC_THREADS = 512;
constexpr int ACC_WARPS = ACC_THREADS / 32;

struct RowStat {
    float m;    // T>0: max logit of the slice;  T=0: max logit
    float s;    // T>0: sum exp2((l - m) * c);    T=0: unused
    int idx;    // T=0: lowest index attaining the max
    int flag;   // SV_FLAG_NONFINITE seen in the slice
};

struct StepSlot {
    float sum;      // slice sum of the current weights
    float rnext;    // residual at the next sibling's draft token (owner only)
    int has_rnext;  // this slice owns that token
    int last_nz;    // last index of the slice with a positive weight, -1 if none
};

struct AcceptShared {
    RowStat rowstat[64];      // this CTA's partials (read by the cluster)
    StepSlot slot[2];         // per reduction step, double-buffered by parity
    float rowM[64], rowS[64];
    int rowArg[64];
    int path[64];
    float red_f[ACC_WARPS];
    float red_g[ACC_WARPS];
    int red_i[ACC_WARPS];
    int red_j[ACC_WARPS];
    // walk state (written by thread 0, read after a __syncthreads)
    int v, depth, last_tried, child, next_sib, action, r_is_p, parity, flags, tok, seqflag;
    float rZ, rnext, draw_t;
    int draw_owner, draw_fallback;
};

enum { ACT_CONTINUE = 0, ACT_REJECT = 1, ACT_DRAW = 2 };

SV_DEV void merge_sumexp(float &m, float &s, float m2, float s2, float c) {
    const float M = fmaxf(m, m2);
    if (M == -INFINITY) return;
    const float a = (m == -INFINITY) ? 0.f : s * exp2f((m - M) * c);
    const float b = (m2 == -INFINITY) ? 0.f : s2 * exp2f((m2 - M) * c);
    m = M;
    s = a + b;
}

SV_DEV void merge_argmax(float &m, int &i, float m2, int i2) {
    if (i2 >= 0 && (i < 0 || m2 > m || (m2 == m && i2 < i))) { m = m2; i = i2; }
}

// Per-element update of a thread's running (max, sum) or (max, argmax).
template <bool GREEDY>
SV_DEV void consume(float x, int idx, float &m, float &s, int &ai, int &flag, float c) {
    if (isnan(x) || x == INFINITY) { flag = 1; return; }
    if (GREEDY) {
        // a thread visits its indices in increasing order, so a strict '>'
        // keeps the lowest index among equal maxima
        if (x > m) { m = x; ai = idx; }
    } else {
        if (x == -INFINITY) return;
        if (x > m) {
            s = (m == -INFINITY) ? 1.f : s * exp2f((m - x) * c) + 1.f;
            m = x;
        } else {
            s += exp2f((x - m) * c);
        }
    }
}

// Next child of node v with index > after, or -1.
SV_DEV int next_child(const AcceptParams &p, int v, int after) {
    for (int c = after + 1; c < p.N; ++c)
        if (p.parent[c] == v) return c;
    return -1;
}

template <bool GREEDY, bool VEC>
__global__ void __launch_bounds__(ACC_THREADS, 1) accept_kernel(const AcceptParams p) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    extern __shared__ __align__(16) float rbuf[];  // chunk floats: residual / draw weights
    __shared__ AcceptShared S;

    const int lo = min(rank * p.chunk, p.V);
    const int hi = min(lo + p.chunk, p.V);
    const size_t rowV = (size_t)p.V;
    const float *lb = p.logits + (size_t)b * p.N * rowV;
    const float c = p.log2e_over_T;
    if (tid == 0) S.seqflag = 0;
    __syncthreads();

    // ---- phase 1: per-row statistics of this CTA's slice, all N rows ----
    for (int v = 0; v < p.N; ++v) {
        const float *row = lb + (size_t)v * rowV;
        float m = -INFINITY, s = 0.f;
        int ai = -1, flag = 0;
        if (VEC) {
            const float4 *r4 = reinterpret_cast<const float4 *>(row);
#pragma unroll 4
            for (int x = lo + 4 * tid; x < hi; x += 4 * ACC_THREADS) {
                const float4 f = __ldg(r4 + (x >> 2));
                consume<GREEDY>(f.x, x, m, s, ai, flag, c);
                consume<GREEDY>(f.y, x + 1, m, s, ai, flag, c);
                consume<GREEDY>(f.z, x + 2, m, s, ai, flag, c);
                consume<GREEDY>(f.w, x + 3, m, s, ai, flag, c);
            }
        } else {
#pragma unroll 4
            for (int x = lo + tid; x < hi; x += ACC_THREADS) consume<GREEDY>(__ldg(row + x), x, m, s, ai, flag, c);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
            const int i2 = __shfl_xor_sync(0xffffffffu, ai, o);
            if (GREEDY) merge_argmax(m, ai, m2, i2); else merge_sumexp(m, s, m2, s2, c);
        }
        flag = warp_or(flag);
        if (lane == 0) { S.red_f[warp] = m; S.red_g[warp] = s; S.red_i[warp] = ai; S.red_j[warp] = flag; }
        __syncthreads();
        if (tid == 0) {
            float M = S.red_f[0], Ssum = S.red_g[0];
            int I = S.red_i[0], F = S.red_j[0];
            for (int w = 1; w < ACC_WARPS; ++w) {
                if (GREEDY) merge_argmax(M, I, S.red_f[w], S.red_i[w]);
                else merge_sumexp(M, Ssum, S.red_f[w], S.red_g[w], c);
                F |= S.red_j[w];
            }
            S.rowstat[v] = RowStat{M, Ssum, I, F};
        }
        __syncthreads();
    }
    cluster.sync();

    // ---- combine row statistics over the cluster (rank order) ----
    if (tid < p.N) {
        const int v = tid;
        float M = -INFINITY, Ssum = 0.f;
        int I = -1, F = 0;
        for (int k = 0; k < ACC_CLUSTER; ++k) {
            const RowStat rs = *cluster.map_shared_rank(&S.rowstat[v], k);
            if (GREEDY) merge_argmax(M, I, rs.m, rs.idx); else merge_sumexp(M, Ssum, rs.m, rs.s, c);
            F |= rs.flag;
        }
        if (M == -INFINITY) F = 1;  // no finite logit in the row
        S.rowM[v] = M; S.rowS[v] = Ssum; S.rowArg[v] = I;
        if (F) atomicOr(&S.seqflag, 1);
    }
    if (tid == 0) {
        S.v = 0; S.depth = 0; S.last_tried = 0; S.r_is_p = 1; S.parity = 0; S.flags = 0;
        S.rZ = 1.f; S.tok = 0;
    }
    __syncthreads();
    const bool nonfinite = S.seqflag != 0;

    const int32_t *db = p.drafts + (size_t)b * (p.N - 1);

    if (nonfinite) {
        if (rank == 0 && tid == 0) {
            p.accept_len[b] = 0;
            p.next_token[b] = 0;
            if (p.accept_path) for (int k = 0; k < p.N - 1; ++k) p.accept_path[(size_t)b * (p.N - 1) + k] = -1;
            if (p.status) p.status[b] = SV_FLAG_NONFINITE;
        }
        cluster.sync();
        return;
    }

    if (GREEDY) {
        if (tid == 0) {
            int v = 0, depth = 0, flags = 0;
            for (;;) {
                const int am = S.rowArg[v];
                int moved = -1;
                for (int ch = next_child(p, v, v); ch >= 0; ch = next_child(p, v, ch)) {
                    const int d = db[ch - 1];
                    if (d < 0 || d >= p.V) { flags |= SV_FLAG_BAD_TOKEN; continue; }
                    if (d == am) { moved = ch; break; }
                }
                if (moved < 0) { S.tok = am; break; }
                S.path[depth++] = moved;
                v = moved;
            }
            S.depth = depth;
            S.flags = flags;
        }
        __syncthreads();
        if (rank == 0 && tid == 0) {
            p.accept_len[b] = S.depth;
            p.next_token[b] = S.tok;
            if (p.accept_path)
                for (int k = 0; k < p.N - 1; ++k)
                    p.accept_path[(size_t)b * (p.N - 1) + k] = k < S.depth ? S.path[k] : -1;
            if (p.status) p.status[b] = S.flags;
        }
        cluster.sync();
        return;
    }

    // ---- sampling walk ----
    const float *qb = p.q + (size_t)b * (p.N - 1) * rowV;
    const int n = hi - lo;
    for (;;) {
        if (tid == 0) {
            const int v = S.v;
            const int ch = next_child(p, v, S.last_tried);
            if (ch < 0) {
                S.action = ACT_DRAW;
            } else {
                const int d = db[ch - 1];
                bool acc = false;
                if (d < 0 || d >= p.V) {
                    S.flags |= SV_FLAG_BAD_TOKEN;
                } else {
                    const float u = philox_uniform(PhiloxKey{p.key.k0, p.key.k1}, (uint32_t)b, (uint32_t)ch, 0u);
                    const float qd = __ldg(qb + (size_t)(ch - 1) * rowV + d);
                    float rd;
                    if (S.r_is_p)
                        rd = exp2f((__ldg(lb + (size_t)v * rowV + d) - S.rowM[v]) * c) / S.rowS[v];
                    else
                        rd = S.rnext / S.rZ;
                    acc = u * qd < rd;
                }
                if (acc) {
                    S.path[S.depth++] = ch;
                    S.v = ch;
                    S.last_tried = ch;
                    S.r_is_p = 1;
                    S.rZ = 1.f;
                    S.action = ACT_CONTINUE;
                } else {
                    S.child = ch;
                    S.last_tried = ch;
                    S.next_sib = next_child(p, v, ch);
                    S.action = ACT_REJECT;
                }
            }
        }
        __syncthreads();
        const int action = S.action;
        if (action == ACT_CONTINUE) continue;
        if (action == ACT_DRAW) break;

        // Rejection at child S.child of node S.v: r <- max(0, r/rZ - q_child) over the slice.
        const int v = S.v, ch = S.child, sib = S.next_sib;
        const bool from_p = S.r_is_p != 0;
        const float rZ = S.rZ, Mv = S.rowM[v], Sv = S.rowS[v];
        const float *lrow = lb + (size_t)v * rowV;
        const float *qrow = qb + (size_t)(ch - 1) * rowV;
        int dsib = -1;
        if (sib >= 0) {
            dsib = db[sib - 1];
            if (dsib < lo || dsib >= hi) dsib = -1;
        }
        float part = 0.f;
        if (VEC) {
            // n and lo are multiples of 4 and the rows are 16-byte aligned
            const float4 *l4 = reinterpret_cast<const float4 *>(lrow + lo);
            const float4 *q4 = reinterpret_cast<const float4 *>(qrow + lo);
            float4 *r4 = reinterpret_cast<float4 *>(rbuf);
#pragma unroll 4
            for (int x = tid; x < (n >> 2); x += ACC_THREADS) {
                const float4 qv = __ldg(q4 + x);
                float4 rv;
                if (from_p) {
                    const float4 lv = __ldg(l4 + x);
                    rv = make_float4(exp2f((lv.x - Mv) * c) / Sv, exp2f((lv.y - Mv) * c) / Sv,
                                     exp2f((lv.z - Mv) * c) / Sv, exp2f((lv.w - Mv) * c) / Sv);
                } else {
                    rv = r4[x];
                    rv = make_float4(rv.x / rZ, rv.y / rZ, rv.z / rZ, rv.w / rZ);
                }
                const float4 w = make_float4(fmaxf(rv.x - qv.x, 0.f), fmaxf(rv.y - qv.y, 0.f),
                                             fmaxf(rv.z - qv.z, 0.f), fmaxf(rv.w - qv.w, 0.f));
                r4[x] = w;
                part += (w.x + w.y) + (w.z + w.w);
                const int d0 = lo + 4 * x;
                if (dsib >= d0 && dsib < d0 + 4)
                    S.slot[S.parity].rnext = dsib == d0 ? w.x : dsib == d0 + 1 ? w.y : dsib == d0 + 2 ? w.z : w.w;
            }
        } else {
#pragma unroll 4
            for (int x = tid; x < n; x += ACC_THREADS) {
                const float r = from_p ? exp2f((__ldg(lrow + lo + x) - Mv) * c) / Sv : rbuf[x] / rZ;
                const float w = fmaxf(r - __ldg(qrow + lo + x), 0.f);
                rbuf[x] = w;
                part += w;
                if (lo + x == dsib) S.slot[S.parity].rnext = w;
            }
        }
        part = warp_sum(part);
        if (lane == 0) S.red_f[warp] = part;
        __syncthreads();
        if (tid == 0) {
            float t = 0.f;
            for (int w = 0; w < ACC_WARPS; ++w) t += S.red_f[w];
            S.slot[S.parity].sum = t;
            S.slot[S.parity].has_rnext = dsib >= 0;
        }
        cluster.sync();
        if (tid == 0) {
            float Z = 0.f, rn = 0.f;
            for (int k = 0; k < ACC_CLUSTER; ++k) {
                const StepSlot sl = *cluster.map_shared_rank(&S.slot[S.parity], k);
                Z += sl.sum;
                if (sl.has_rnext) rn = sl.rnext;
            }
            if (Z > 0.f) { S.rZ = Z; S.r_is_p = 0; S.rnext = rn; }
            else { S.rZ = 1.f; S.r_is_p = 1; }
            S.parity ^= 1;
        }
        __syncthreads();
    }

    // ---- draw at node S.v from r (or p_v) ----
    {
        const int v = S.v;
        const bool from_p = S.r_is_p != 0;
        const float Mv = S.rowM[v];
        const float *lrow = lb + (size_t)v * rowV;
        if (from_p) {
            if (VEC) {
                const float4 *l4 = reinterpret_cast<const float4 *>(lrow + lo);
                float4 *r4 = reinterpret_cast<float4 *>(rbuf);
#pragma unroll 4
                for (int x = tid; x < (n >> 2); x += ACC_THREADS) {
                    const float4 lv = __ldg(l4 + x);
                    r4[x] = make_float4(exp2f((lv.x - Mv) * c), exp2f((lv.y - Mv) * c), exp2f((lv.z - Mv) * c),
                                        exp2f((lv.w - Mv) * c));
                }
            } else {
#pragma unroll 4
                for (int x = tid; x < n; x += ACC_THREADS) rbuf[x] = exp2f((__ldg(lrow + lo + x) - Mv) * c);
            }
        }
        __syncthreads();
        // contiguous segment per thread, summed in index order
        const int seg = (n + ACC_THREADS - 1) / ACC_THREADS;
        const int s0 = min(tid * seg, n), s1 = min(s0 + seg, n);
        float tsum = 0.f;
        int tlast = -1;
        for (int x = s0; x < s1; ++x) {
            const float w = rbuf[x];
            tsum += w;
            if (w > 0.f) tlast = x;
        }
        // block exclusive scan of thread sums (thread order)
        float incl = tsum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int wl = tlast;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wl = max(wl, __shfl_xor_sync(0xffffffffu, wl, o));
        if (lane == 31) S.red_f[warp] = incl;
        if (lane == 0) S.red_i[warp] = wl;
        __syncthreads();
        float wpre = 0.f;
        for (int w = 0; w < warp; ++w) wpre += S.red_f[w];
        const float excl = wpre + incl - tsum;
        if (tid == 0) {
            float tot = 0.f;
            int ln = -1;
            for (int w = 0; w < ACC_WARPS; ++w) { tot += S.red_f[w]; ln = max(ln, S.red_i[w]); }
            StepSlot &sl = S.slot[S.parity];
            sl.sum = tot;
            sl.last_nz = ln < 0 ? -1 : lo + ln;
            sl.has_rnext = 0;
        }
        cluster.sync();
        if (tid == 0) {
            StepSlot all[ACC_CLUSTER];
            float total = 0.f;
            for (int k = 0; k < ACC_CLUSTER; ++k) {
                all[k] = *cluster.map_shared_rank(&S.slot[S.parity], k);
                total += all[k].sum;
            }
            const float u = philox_uniform(PhiloxKey{p.key.k0, p.key.k1}, (uint32_t)b, (uint32_t)v, 1u);
            const float t = u * total;
            int owner = -1, gl = -1;
            float pre = 0.f, tk = 0.f;
            for (int k = 0; k < ACC_CLUSTER; ++k) {
                if (owner < 0 && t - pre < all[k].sum) { owner = k; tk = t - pre; }
                pre += all[k].sum;
                gl = max(gl, all[k].last_nz);
            }
            S.draw_owner = owner;
            S.draw_t = tk;
            S.draw_fallback = gl;
            S.tok = -1;
        }
        __syncthreads();
        if (S.draw_owner == rank) {
            const float tj = S.draw_t - excl;
            const bool sel = (s1 > s0) && (tj < tsum);
            // first thread (lowest tid) whose segment holds the threshold
            const unsigned bal = __ballot_sync(0xffffffffu, sel);
            if (lane == 0) S.red_j[warp] = bal ? (warp * 32 + __ffs(bal) - 1) : 0x7fffffff;
            __syncthreads();
            if (tid == 0) {
                int first = 0x7fffffff;
                for (int w = 0; w < ACC_WARPS; ++w) first = min(first, S.red_j[w]);
                S.red_i[0] = first;
            }
            __syncthreads();
            const int first = S.red_i[0];
            if (first == 0x7fffffff) {
                if (tid == 0) {
                    int ln = -1;
                    for (int x = n - 1; x >= 0; --x) if (rbuf[x] > 0.f) { ln = x; break; }
                    p.next_token[b] = lo + max(ln, 0);
                }
            } else if (tid == first) {
                float cl = 0.f;
                int tok = s1 - 1;
                for (int x = s0; x < s1; ++x) {
                    cl += rbuf[x];
                    if (cl > tj) { tok = x; break; }
                }
                p.next_token[b] = lo + tok;
            }
        } else if (S.draw_owner < 0 && rank == 0 && tid == 0) {
            p.next_token[b] = max(S.draw_fallback, 0);
        }
        if (rank == 0 && tid == 0) {
            p.accept_len[b] = S.depth;
            if (p.accept_path)
                for (int k = 0; k < p.N - 1; ++k)
                    p.accept_path[(size_t)b * (p.N - 1) + k] = k < S.depth ? S.path[k] : -1;
            if (p.status) p.status[b] = S.flags;
        }
    }
    cluster.sync();
}

// ===========================================================================
// Streamed variant (vocabulary a multiple of 4, 16-byte aligned rows): the
// same walk and arithmetic, with the slices fed through a ring of 16 KB
// shared-memory stages by bulk copies from a producer warp, so each CTA keeps
// up to STR_MAX_STAGES x 16 KB of loads in flight while 16 consumer warps
// reduce. The decision inputs of every draft (its draft probability and its
// logit in its parent's row) are loaded once at the start, so the walk itself
// issues no dependent global loads.
// ===========================================================================
constexpr int STR_CWARPS = 16;
constexpr int STR_CTHREADS = 32 * STR_CWARPS;      // consumer threads
constexpr int STR_THREADS = STR_CTHREADS + 32;     // + the producer warp
constexpr int STR_WARPS = STR_CWARPS + 1;
constexpr int STAGE_FLOATS = 8192;                 // 32 KB per ring stage (a bulk copy streams
                                                   // faster per SM the larger it is)
constexpr int HALF_STAGE = STAGE_FLOATS / 2;       // residual stages: p half, q half
constexpr int STR_MAX_STAGES = 6;
constexpr int STR_MAX_CLUSTER = 16;
constexpr uint64_t STR_WAIT_NS = 2000000000ull;    // 2 s per wait, then the CTA gives up

struct StreamShared {
    uint64_t full[STR_MAX_STAGES], empty[STR_MAX_STAGES];
    RowStat rowstat[64];
    StepSlot slot[2];
    float rowM[64], rowS[64];
    int rowArg[64];
    int path[64];
    int dr[64];       // draft token of node c (c >= 1)
    float Ld[64];     // logit of d_c in the row of c's parent
    float Qd[64];     // draft probability of d_c
    float red_f[STR_WARPS];
    float red_g[STR_WARPS];
    int red_i[STR_WARPS];
    int red_j[STR_WARPS];
    int v, depth, last_tried, child, next_sib, action, r_is_p, parity, flags, tok, seqflag;
    float rZ, rnext, draw_t;
    int draw_owner, draw_fallback;
    int abort;        // a bounded wait gave up
    StepSlot gath[STR_MAX_CLUSTER];  // the cluster's slots, gathered in parallel
};

template <bool GREEDY>
__global__ void __launch_bounds__(STR_THREADS, 1) accept_stream_kernel(const AcceptParams p, int nst) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int csize = (int)cluster.num_blocks();
    const int b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool producer = warp == STR_CWARPS;
    extern __shared__ __align__(16) float dyn[];
    float *ring = dyn;                                          // nst x STAGE_FLOATS
    float *rbuf = dyn + (size_t)nst * STAGE_FLOATS;             // chunk floats: residual / draw weights
    RowStat *wpart = reinterpret_cast<RowStat *>(rbuf + p.chunk);  // [N][STR_CWARPS] warp partials
    __shared__ StreamShared S;
    volatile int *abort_flag = &S.abort;

    const int lo = min(rank * p.chunk, p.V);
    const int hi = min(lo + p.chunk, p.V);
    const int n = hi - lo;
    const size_t rowV = (size_t)p.V;
    const float *lb = p.logits + (size_t)b * p.N * rowV;
    const float *qb = GREEDY ? nullptr : p.q + (size_t)b * (p.N - 1) * rowV;
    const float c = p.log2e_over_T;
    if (tid == 0) {
        for (int i = 0; i < nst; ++i) { mbar_init(&S.full[i], 1); mbar_init(&S.empty[i], STR_CWARPS); }
        S.seqflag = 0;
        S.abort = 0;
        fence_barrier_init();
    }
    // decision inputs of every draft node (independent loads, overlapping the stream)
    if (tid >= 1 && tid < p.N) {
        const int ch = tid, d = p.drafts[(size_t)b * (p.N - 1) + ch - 1];
        S.dr[ch] = d;
        if (d >= 0 && d < p.V) {
            S.Ld[ch] = __ldg(lb + (size_t)p.parent[ch] * rowV + d);
            if (!GREEDY) S.Qd[ch] = __ldg(qb + (size_t)(ch - 1) * rowV + d);
        }
    }
    __syncthreads();

    // ---- ring: the producer issues stages in order, consumers take them in order ----
    int g = 0;                               // stages issued (producer) / taken (consumers)
    int last_issue[STR_MAX_STAGES];          // producer: most recent stage index per slot
#pragma unroll
    for (int i = 0; i < STR_MAX_STAGES; ++i) last_issue[i] = -1;
    // one stage: nA floats from srcA at the stage start, nB floats from srcB at HALF_STAGE
    auto produce = [&](const float *srcA, int nA, const float *srcB, int nB) {
        const int sl = g % nst;
        if (mbar_wait(&S.empty[sl], ((g / nst) & 1) ^ 1, abort_flag, STR_WAIT_NS)) {
            mbar_arrive_expect_tx(&S.full[sl], (uint32_t)(nA + nB) * 4u);
            float *dst = ring + (size_t)sl * STAGE_FLOATS;
            if (nA > 0) bulk_load(dst, srcA, (uint32_t)nA * 4u, &S.full[sl]);
            if (nB > 0) bulk_load(dst + HALF_STAGE, srcB, (uint32_t)nB * 4u, &S.full[sl]);
            last_issue[sl] = g;
        }
        ++g;
    };
    // warp-uniform: the stage, or nullptr when the wait gave up (the stage is then skipped)
    auto acquire = [&]() -> const float * {
        const int sl = g % nst;
        const uint32_t par = (g / nst) & 1;
        const bool ok = mbar_test(&S.full[sl], par) || mbar_wait(&S.full[sl], par, abort_flag, STR_WAIT_NS);
        return __all_sync(0xffffffffu, ok) ? ring + (size_t)sl * STAGE_FLOATS : nullptr;
    };
    auto release = [&]() {
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[g % nst]);
        ++g;
    };

    // ---- phase 1: per-row statistics of this CTA's slice, all N rows in one stream ----
    const int npc = (n + STAGE_FLOATS - 1) / STAGE_FLOATS;  // stages per row
    if (producer) {
        if (lane == 0)
            for (int v = 0; v < p.N; ++v)
                for (int k = 0; k < npc; ++k)
                    produce(lb + (size_t)v * rowV + lo + k * STAGE_FLOATS, min(STAGE_FLOATS, n - k * STAGE_FLOATS),
                            nullptr, 0);
        __syncwarp();
    } else {
        for (int v = 0; v < p.N; ++v) {
            float m = -INFINITY, s = 0.f;
            int ai = -1, flag = 0;
            for (int k = 0; k < npc; ++k) {
                const float *st = acquire();
                const int len4 = min(STAGE_FLOATS, n - k * STAGE_FLOATS) >> 2;
                if (st) {
                    const float4 *s4 = reinterpret_cast<const float4 *>(st);
                    if (GREEDY) {
                        for (int i = tid; i < len4; i += STR_CTHREADS) {
                            const float4 f = s4[i];
                            const int x = lo + k * STAGE_FLOATS + 4 * i;
                            consume<true>(f.x, x, m, s, ai, flag, c);
                            consume<true>(f.y, x + 1, m, s, ai, flag, c);
                            consume<true>(f.z, x + 2, m, s, ai, flag, c);
                            consume<true>(f.w, x + 3, m, s, ai, flag, c);
                        }
                    } else {
                        // this thread's elements of the stage at once: their maximum,
                        // one rescale of the running sum, then independent exponentials
                        float e[STAGE_FLOATS / STR_CTHREADS];
#pragma unroll
                        for (int j = 0; j < STAGE_FLOATS / (4 * STR_CTHREADS); ++j) {
                            const int i = tid + j * STR_CTHREADS;
                            const float4 f = i < len4 ? s4[i] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
                            e[4 * j] = f.x; e[4 * j + 1] = f.y; e[4 * j + 2] = f.z; e[4 * j + 3] = f.w;
                        }
                        float lm = -INFINITY;
#pragma unroll
                        for (int j = 0; j < STAGE_FLOATS / STR_CTHREADS; ++j) {
                            if (isnan(e[j]) || e[j] == INFINITY) { flag = 1; e[j] = -INFINITY; }
                            lm = fmaxf(lm, e[j]);
                        }
                        if (lm > m) {
                            s = (m == -INFINITY) ? 0.f : s * exp2f((m - lm) * c);
                            m = lm;
                        }
                        if (m != -INFINITY) {
                            float add = 0.f;
#pragma unroll
                            for (int j = 0; j < STAGE_FLOATS / STR_CTHREADS; ++j) add += exp2f((e[j] - m) * c);
                            s += add;
                        }
                    }
                }
                release();
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
                const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
                const int i2 = __shfl_xor_sync(0xffffffffu, ai, o);
                if (GREEDY) merge_argmax(m, ai, m2, i2); else merge_sumexp(m, s, m2, s2, c);
            }
            flag = warp_or(flag);
            if (lane == 0) wpart[v * STR_CWARPS + warp] = RowStat{m, s, ai, flag};
        }
    }
    __syncthreads();
    if (tid < p.N) {
        const int v = tid;
        RowStat r = wpart[v * STR_CWARPS];
        for (int w = 1; w < STR_CWARPS; ++w) {
            const RowStat o = wpart[v * STR_CWARPS + w];
            if (GREEDY) merge_argmax(r.m, r.idx, o.m, o.idx); else merge_sumexp(r.m, r.s, o.m, o.s, c);
            r.flag |= o.flag;
        }
        S.rowstat[v] = r;
    }
    cluster.sync();

    // ---- combine row statistics over the cluster (rank order); the remote
    // partials are first gathered in parallel into the (now free) warp partials ----
    for (int idx = tid; idx < p.N * csize; idx += STR_THREADS) {
        const int v = idx / csize, k = idx - v * csize;
        wpart[v * STR_CWARPS + k] = *cluster.map_shared_rank(&S.rowstat[v], k);
    }
    __syncthreads();
    if (tid < p.N) {
        const int v = tid;
        float M = -INFINITY, Ssum = 0.f;
        int I = -1, F = 0;
        for (int k = 0; k < csize; ++k) {
            const RowStat rs = wpart[v * STR_CWARPS + k];
            if (GREEDY) merge_argmax(M, I, rs.m, rs.idx); else merge_sumexp(M, Ssum, rs.m, rs.s, c);
            F |= rs.flag;
        }
        if (M == -INFINITY) F = 1;  // no finite logit in the row
        S.rowM[v] = M; S.rowS[v] = Ssum; S.rowArg[v] = I;
        if (F) atomicOr(&S.seqflag, 1);
    }
    if (tid == 0) {
        S.v = 0; S.depth = 0; S.last_tried = 0; S.r_is_p = 1; S.parity = 0; S.flags = 0;
        S.rZ = 1.f; S.tok = 0;
    }
    __syncthreads();
    const bool nonfinite = S.seqflag != 0;

    if (nonfinite) {
        if (rank == 0 && tid == 0) {
            p.accept_len[b] = 0;
            p.next_token[b] = 0;
            if (p.accept_path) for (int k = 0; k < p.N - 1; ++k) p.accept_path[(size_t)b * (p.N - 1) + k] = -1;
            if (p.status) p.status[b] = SV_FLAG_NONFINITE;
        }
    } else if (GREEDY) {
        if (tid == 0) {
            int v = 0, depth = 0, flags = 0;
            for (;;) {
                const int am = S.rowArg[v];
                int moved = -1;
                for (int ch = next_child(p, v, v); ch >= 0; ch = next_child(p, v, ch)) {
                    const int d = S.dr[ch];
                    if (d < 0 || d >= p.V) { flags |= SV_FLAG_BAD_TOKEN; continue; }
                    if (d == am) { moved = ch; break; }
                }
                if (moved < 0) { S.tok = am; break; }
                S.path[depth++] = moved;
                v = moved;
            }
            S.depth = depth;
            S.flags = flags;
        }
        __syncthreads();
        if (rank == 0 && tid == 0) {
            p.accept_len[b] = S.depth;
            p.next_token[b] = S.tok;
            if (p.accept_path)
                for (int k = 0; k < p.N - 1; ++k)
                    p.accept_path[(size_t)b * (p.N - 1) + k] = k < S.depth ? S.path[k] : -1;
            if (p.status) p.status[b] = S.flags;
        }
    } else {
        // ---- sampling walk ----
        for (;;) {
            if (tid == 0) {
                const int v = S.v;
                const int ch = next_child(p, v, S.last_tried);
                if (ch < 0) {
                    S.action = ACT_DRAW;
                } else {
                    const int d = S.dr[ch];
                    bool acc = false;
                    if (d < 0 || d >= p.V) {
                        S.flags |= SV_FLAG_BAD_TOKEN;
                    } else {
                        const float u = philox_uniform(PhiloxKey{p.key.k0, p.key.k1}, (uint32_t)b, (uint32_t)ch, 0u);
                        const float rd = S.r_is_p ? exp2f((S.Ld[ch] - S.rowM[v]) * c) / S.rowS[v] : S.rnext / S.rZ;
                        acc = u * S.Qd[ch] < rd;
                    }
                    if (acc) {
                        S.path[S.depth++] = ch;
                        S.v = ch;
                        S.last_tried = ch;
                        S.r_is_p = 1;
                        S.rZ = 1.f;
                        S.action = ACT_CONTINUE;
                    } else {
                        S.child = ch;
                        S.last_tried = ch;
                        S.next_sib = next_child(p, v, ch);
                        S.action = ACT_REJECT;
                    }
                }
            }
            __syncthreads();
            const int action = S.action;
            if (action == ACT_CONTINUE) continue;
            if (action == ACT_DRAW) break;

            // Rejection at child S.child of node S.v: r <- max(0, r/rZ - q_child) over the slice.
            const int v = S.v, ch = S.child, sib = S.next_sib;
            const bool from_p = S.r_is_p != 0;
            const float rZ = S.rZ, Mv = S.rowM[v], Sv = S.rowS[v];
            const float *lrow = lb + (size_t)v * rowV + lo;
            const float *qrow = qb + (size_t)(ch - 1) * rowV + lo;
            const int npr = (n + HALF_STAGE - 1) / HALF_STAGE;
            const int dsib_all = sib >= 0 ? S.dr[sib] : -1;
            const bool owns_sib = dsib_all >= lo && dsib_all < hi;  // this slice holds the next sibling's token
            float part = 0.f;
            if (producer) {
                if (lane == 0)
                    for (int k = 0; k < npr; ++k) {
                        const int len = min(HALF_STAGE, n - k * HALF_STAGE);
                        produce(lrow + k * HALF_STAGE, from_p ? len : 0, qrow + k * HALF_STAGE, len);
                    }
                __syncwarp();
            } else {
                const int dsib = owns_sib ? dsib_all : -1;
                float4 *r4 = reinterpret_cast<float4 *>(rbuf);
                for (int k = 0; k < npr; ++k) {
                    const float *st = acquire();
                    const int len4 = min(HALF_STAGE, n - k * HALF_STAGE) >> 2;
                    if (st) {
                        const float4 *l4 = reinterpret_cast<const float4 *>(st);
                        const float4 *q4 = reinterpret_cast<const float4 *>(st + HALF_STAGE);
                        for (int i = tid; i < len4; i += STR_CTHREADS) {
                            const int x = k * (HALF_STAGE / 4) + i;  // float4 index in the slice
                            const float4 qv = q4[i];
                            float4 rv;
                            if (from_p) {
                                const float4 lv = l4[i];
                                rv = make_float4(exp2f((lv.x - Mv) * c) / Sv, exp2f((lv.y - Mv) * c) / Sv,
                                                 exp2f((lv.z - Mv) * c) / Sv, exp2f((lv.w - Mv) * c) / Sv);
                            } else {
                                rv = r4[x];
                                rv = make_float4(rv.x / rZ, rv.y / rZ, rv.z / rZ, rv.w / rZ);
                            }
                            const float4 w = make_float4(fmaxf(rv.x - qv.x, 0.f), fmaxf(rv.y - qv.y, 0.f),
                                                         fmaxf(rv.z - qv.z, 0.f), fmaxf(rv.w - qv.w, 0.f));
                            r4[x] = w;
                            part += (w.x + w.y) + (w.z + w.w);
                            const int d0 = lo + 4 * x;
                            if (dsib >= d0 && dsib < d0 + 4)
                                S.slot[S.parity].rnext = dsib == d0 ? w.x : dsib == d0 + 1 ? w.y : dsib == d0 + 2 ? w.z : w.w;
                        }
                    }
                    release();
                }
            }
            part = warp_sum(part);
            if (lane == 0) S.red_f[warp] = part;
            __syncthreads();
            if (tid == 0) {
                float t = 0.f;
                for (int w = 0; w < STR_WARPS; ++w) t += S.red_f[w];
                S.slot[S.parity].sum = t;
                S.slot[S.parity].has_rnext = owns_sib;
            }
            cluster.sync();
            if (tid < csize) S.gath[tid] = *cluster.map_shared_rank(&S.slot[S.parity], tid);  // one remote read each
            __syncthreads();
            if (tid == 0) {
                float Z = 0.f, rn = 0.f;
                for (int k = 0; k < csize; ++k) {
                    const StepSlot sl = S.gath[k];
                    Z += sl.sum;
                    if (sl.has_rnext) rn = sl.rnext;
                }
                if (Z > 0.f) { S.rZ = Z; S.r_is_p = 0; S.rnext = rn; }
                else { S.rZ = 1.f; S.r_is_p = 1; }
                S.parity ^= 1;
            }
            __syncthreads();
        }

        // ---- draw at node S.v from r (or p_v) ----
        const int v = S.v;
        const bool from_p = S.r_is_p != 0;
        const float Mv = S.rowM[v];
        const float *lrow = lb + (size_t)v * rowV + lo;
        if (from_p) {
            if (producer) {
                if (lane == 0)
                    for (int k = 0; k < npc; ++k)
                        produce(lrow + k * STAGE_FLOATS, min(STAGE_FLOATS, n - k * STAGE_FLOATS), nullptr, 0);
                __syncwarp();
            } else {
                float4 *r4 = reinterpret_cast<float4 *>(rbuf);
                for (int k = 0; k < npc; ++k) {
                    const float *st = acquire();
                    const int len4 = min(STAGE_FLOATS, n - k * STAGE_FLOATS) >> 2;
                    if (st) {
                        const float4 *l4 = reinterpret_cast<const float4 *>(st);
                        for (int i = tid; i < len4; i += STR_CTHREADS) {
                            const float4 lv = l4[i];
                            r4[k * (STAGE_FLOATS / 4) + i] = make_float4(exp2f((lv.x - Mv) * c), exp2f((lv.y - Mv) * c),
                                                                         exp2f((lv.z - Mv) * c), exp2f((lv.w - Mv) * c));
                        }
                    }
                    release();
                }
            }
        }
        __syncthreads();
        // contiguous segment per consumer thread, summed in index order
        const int seg = (n + STR_CTHREADS - 1) / STR_CTHREADS;
        const int s0 = min(tid * seg, n), s1 = min(s0 + seg, n);
        float tsum = 0.f;
        int tlast = -1;
        for (int x = s0; x < s1; ++x) {
            const float w = rbuf[x];
            tsum += w;
            if (w > 0.f) tlast = x;
        }
        // block exclusive scan of thread sums (thread order)
        float incl = tsum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int wl = tlast;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wl = max(wl, __shfl_xor_sync(0xffffffffu, wl, o));
        if (lane == 31) S.red_f[warp] = incl;
        if (lane == 0) S.red_i[warp] = wl;
        __syncthreads();
        float wpre = 0.f;
        for (int w = 0; w < warp; ++w) wpre += S.red_f[w];
        const float excl = wpre + incl - tsum;
        if (tid == 0) {
            float tot = 0.f;
            int ln = -1;
            for (int w = 0; w < STR_WARPS; ++w) { tot += S.red_f[w]; ln = max(ln, S.red_i[w]); }
            StepSlot &sl = S.slot[S.parity];
            sl.sum = tot;
            sl.last_nz = ln < 0 ? -1 : lo + ln;
            sl.has_rnext = 0;
        }
        cluster.sync();
        if (tid < csize) S.gath[tid] = *cluster.map_shared_rank(&S.slot[S.parity], tid);
        __syncthreads();
        if (tid == 0) {
            float total = 0.f;
            for (int k = 0; k < csize; ++k) total += S.gath[k].sum;
            const float u = philox_uniform(PhiloxKey{p.key.k0, p.key.k1}, (uint32_t)b, (uint32_t)v, 1u);
            const float t = u * total;
            int owner = -1, gl = -1;
            float pre = 0.f, tk = 0.f;
            for (int k = 0; k < csize; ++k) {
                const StepSlot sk = S.gath[k];
                if (owner < 0 && t - pre < sk.sum) { owner = k; tk = t - pre; }
                pre += sk.sum;
                gl = max(gl, sk.last_nz);
            }
            S.draw_owner = owner;
            S.draw_t = tk;
            S.draw_fallback = gl;
            S.tok = -1;
        }
        __syncthreads();
        if (S.draw_owner == rank) {
            const float tj = S.draw_t - excl;
            const bool sel = (s1 > s0) && (tj < tsum);
            // first thread (lowest tid) whose segment holds the threshold
            const unsigned bal = __ballot_sync(0xffffffffu, sel);
            if (lane == 0) S.red_j[warp] = bal ? (warp * 32 + __ffs(bal) - 1) : 0x7fffffff;
            __syncthreads();
            if (tid == 0) {
                int first = 0x7fffffff;
                for (int w = 0; w < STR_WARPS; ++w) first = min(first, S.red_j[w]);
                S.red_i[0] = first;
            }
            __syncthreads();
            const int first = S.red_i[0];
            if (first == 0x7fffffff) {
                if (tid == 0) {
                    int ln = -1;
                    for (int x = n - 1; x >= 0; --x) if (rbuf[x] > 0.f) { ln = x; break; }
                    p.next_token[b] = lo + max(ln, 0);
                }
            } else if (tid == first) {
                float cl = 0.f;
                int tok = s1 - 1;
                for (int x = s0; x < s1; ++x) {
                    cl += rbuf[x];
                    if (cl > tj) { tok = x; break; }
                }
                p.next_token[b] = lo + tok;
            }
        } else if (S.draw_owner < 0 && rank == 0 && tid == 0) {
            p.next_token[b] = max(S.draw_fallback, 0);
        }
        if (rank == 0 && tid == 0) {
            p.accept_len[b] = S.depth;
            if (p.accept_path)
                for (int k = 0; k < p.N - 1; ++k)
                    p.accept_path[(size_t)b * (p.N - 1) + k] = k < S.depth ? S.path[k] : -1;
            if (p.status) p.status[b] = S.flags;
        }
    }
    cluster.sync();  // no CTA leaves while another may still read its shared memory
    if (*abort_flag) {
        // let this CTA's own copies land before it exits, then report the timeout
        if (producer && lane == 0)
            for (int sl = 0; sl < nst; ++sl)
                if (last_issue[sl] >= 0) mbar_wait_time(&S.full[sl], (last_issue[sl] / nst) & 1, STR_WAIT_NS);
        if (tid == 0 && p.status) atomicOr(p.status + b, SV_FLAG_TIMEOUT);
    }
}

template <bool GREEDY, bool VEC>
static cudaError_t launch_one(const AcceptParams &p, size_t smem, cudaStream_t stream) {
    auto kfn = accept_kernel<GREEDY, VEC>;
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ACC_CLUSTER, (unsigned)p.B, 1);
    cfg.blockDim = dim3(ACC_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ACC_CLUSTER;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kfn, p);
}

int accept_max_vocab() { return ACC_CLUSTER * (ACC_MAX_CHUNK_FLOATS); }

template <bool GREEDY>
static cudaError_t launch_stream(const AcceptParams &p, int csize, int nst, size_t smem, cudaStream_t stream) {
    auto kfn = accept_stream_kernel<GREEDY>;
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (csize > 8) {
        e = cudaFuncSetAttribute(kfn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)csize, (unsigned)p.B, 1);
    cfg.blockDim = dim3(STR_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kfn, p, nst);
}

constexpr size_t STR_SMEM_LIMIT = 227 * 1024;

cudaError_t launch_accept(const AcceptParams &p0, cudaStream_t stream) {
    AcceptParams p = p0;
    auto a16 = [](const void *x) { return (reinterpret_cast<uintptr_t>(x) & 15) == 0; };
    const bool vec = (p.V % 4 == 0) && a16(p.logits) && (p.greedy || p.q == nullptr || a16(p.q));
    if (vec) {
        // cluster of 8 CTAs per sequence; 16 when a slice of 8 leaves too little
        // shared memory for a ring of at least two stages
        for (int csize = 8; csize <= STR_MAX_CLUSTER; csize *= 2) {
            const int chunk = (((p.V + csize - 1) / csize) + 3) & ~3;
            const size_t fixed = (size_t)chunk * sizeof(float) + (size_t)p.N * STR_CWARPS * sizeof(RowStat);
            const size_t avail = STR_SMEM_LIMIT - sizeof(StreamShared) - 1024;
            if (fixed >= avail) continue;
            const int nst = (int)std::min<size_t>(STR_MAX_STAGES, (avail - fixed) / (STAGE_FLOATS * sizeof(float)));
            if (nst < 2) continue;
            p.chunk = chunk;
            const size_t smem = fixed + (size_t)nst * STAGE_FLOATS * sizeof(float);
            return p.greedy ? launch_stream<true>(p, csize, nst, smem, stream)
                            : launch_stream<false>(p, csize, nst, smem, stream);
        }
    }
    int chunk = (p.V + ACC_CLUSTER - 1) / ACC_CLUSTER;
    chunk = (chunk + 3) & ~3;
    p.chunk = chunk;
    const size_t smem = (size_t)chunk * sizeof(float);
    return p.greedy ? launch_one<true, false>(p, smem, stream) : launch_one<false, false>(p, smem, stream);
}

}  // namespace sv
