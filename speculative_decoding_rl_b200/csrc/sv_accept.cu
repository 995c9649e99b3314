// sv_accept: vocab-wide temperature softmax, accept test, tree/chain walk and
// residual resampling for the speculative-decoding verify step.
//
// The rule is the lossless one (Accelerating RL Post-Training Rollouts via
// System-Integrated Speculative Decoding, Abstract): accept draft i while
// u_i < min(1, p_i/q_i), drafts after the first rejection are discarded (TLT
// reading notes, "1. RL and SD"), and the emitted token is drawn from
// norm(max(0, p - q)) at the rejection, or from p after the last draft. Draft
// trees (SRT review, "Speculative Rollout integration", step 5) are walked as
// recursive rejection sampling over each accepted node's children in index
// order, which is the chain rule when every node has one child.
//
// Work decomposition. Everything that spans the vocabulary is a wide pass of
// one CTA per (slice of ACC_SLICE entries, row, sequence) over every SM; the
// walk, which needs a handful of values per draft, runs per sequence between
// the passes:
//   1. stats  every logit once (16-byte loads): per (row, slice) the maximum
//             and the sum of 2^((l - max) log2(e) / T) (T = 0: the maximum and
//             its lowest index), and whether NaN or +inf occurs;
//   2. walk   one CTA per sequence: the row statistics are merged over the
//             slices, each draft's decision inputs (its draft probability and
//             its logit in its parent's row) are loaded, and the walk runs
//             until it needs a vocabulary-wide sum: the mass of the residual
//             left by a rejection, or the mass of p at a node without children;
//   3. pass   the per-slice parts of that sum, from the node's logit row and
//             the draft rows of the children rejected there (the residual is
//             rebuilt element by element from them);
//   4. walk   the walk resumes with the sum: it tries the next child (a tree's
//             next rejection needs another pass) or draws. The draw finds its
//             slice from the per-slice sums and re-reads and scans that slice
//             alone.
// A chain needs one pass; a tree as many as its worst walk has rejections;
// T = 0 needs none. Each kernel waits only for the kernel before it
// (programmatic dependent launch): there is no spin-wait anywhere.
#include <algorithm>

#include "sv_device.cuh"
#include "sv_internal.h"
#include "sv_tc.cuh"

namespace sv {

using tc::griddep_launch_dependents;
using tc::griddep_wait;

constexpr int ACC_THREADS = 256;                        // stats and pass kernels
constexpr int ACC_PER_THREAD = ACC_SLICE / ACC_THREADS;  // 32 entries per thread
constexpr int WALK_THREADS = 256;
constexpr int WALK_SEG = ACC_SLICE / WALK_THREADS;       // draw: contiguous entries per thread

// Pass requested by the walk of a sequence (AccState::mode).
enum { MODE_NONE = 0, MODE_RESID = 1, MODE_P = 2, MODE_DONE = 3 };

// Walk state of one sequence, kept in the workspace between kernels.
struct __align__(16) AccState {
    int mode;        // MODE_*
    int v;           // current node
    int depth;       // accepted drafts so far
    int flags;       // SV_FLAG_* bits
    int last_tried;  // last child of v tried (children have larger indices)
    int nchain;      // children rejected at v since r was last p_v
    int have_pass;   // the per-slice sums of the current r are in the workspace
    int pad;
    float Z[64];     // masses of the residuals after each rejection of the chain
    int chain[64];   // the rejected children, in order
    int path[64];
    float rowM[64], rowS[64];
    int rowArg[64];
    float Ld[64];    // logit of draft c's token in its parent's row
    float Qd[64];    // draft probability of draft c's token
    int dr[64];      // draft token of node c
};
static_assert(sizeof(AccState) % 16 == 0, "AccState is copied in 16-byte words");

struct AccWorkspace {
    size_t stats, state, rsum, total;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static AccWorkspace acc_workspace(int B, int N, int V) {
    const size_t S = (size_t)(V + ACC_SLICE - 1) / ACC_SLICE;
    AccWorkspace w;
    w.stats = 0;
    w.state = align256((size_t)B * N * S * sizeof(float4));
    w.rsum = w.state + align256((size_t)B * sizeof(AccState));
    w.total = w.rsum + align256((size_t)B * S * sizeof(float2));
    return w;
}

size_t accept_workspace_bytes(int B, int N, int V) { return acc_workspace(B, N, V).total; }

struct AccPtrs {
    float4 *stats;   // [B][N][S]: (max, sum | -, argmax bits, nonfinite bits)
    AccState *st;    // [B]
    float2 *rsum;    // [B][S]: (residual part, p part) of the pending pass
};

SV_DEV AccPtrs acc_ptrs(const AcceptParams &p) {
    const AccWorkspace w = {0, align256((size_t)p.B * p.N * p.S * sizeof(float4)), 0, 0};
    char *base = static_cast<char *>(p.workspace);
    AccPtrs r;
    r.stats = reinterpret_cast<float4 *>(base);
    r.st = reinterpret_cast<AccState *>(base + w.state);
    r.rsum = reinterpret_cast<float2 *>(base + w.state + align256((size_t)p.B * sizeof(AccState)));
    return r;
}

// (max, sum of 2^((x - max) c)) pairs; -inf maxima carry no mass.
SV_DEV void merge_sumexp(float &m, float &s, float m2, float s2, float c) {
    const float M = fmaxf(m, m2);
    if (M == -INFINITY) return;
    const float a = (m == -INFINITY) ? 0.f : s * exp2f((m - M) * c);
    const float b = (m2 == -INFINITY) ? 0.f : s2 * exp2f((m2 - M) * c);
    m = M;
    s = a + b;
}

// (max, lowest index attaining it); index -1 = nothing finite yet.
SV_DEV void merge_argmax(float &m, int &i, float m2, int i2) {
    if (i2 >= 0 && (i < 0 || m2 > m || (m2 == m && i2 < i))) { m = m2; i = i2; }
}

// Element arithmetic shared by the statistics, the pass, the walk's test and
// the draw, so that every kernel computes the same bits for the same weight:
//   e(x)  = 2^((l(x) - M) c)                        (pweight)
//   r_0   = e (1/S),  r_i = max(0, r_{i-1} - q_i) (1/Z_i)   (rstart, rstep)
//   weight after the chain c_1..c_k = max(0, r_{k-1} - q_k)  (rlast)
// The reciprocals are correctly rounded (one per row or chain entry), the
// products and differences are rounded once each and never contracted.
SV_DEV float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;  // results below 2^-126 of the row maximum's weight flush to zero
}
SV_DEV float pweight(float l, float M, float c) { return ex2_ftz(__fmul_rn(__fsub_rn(l, M), c)); }
SV_DEV float rstart(float e, float invS) { return __fmul_rn(e, invS); }
SV_DEV float rstep(float r, float q, float invZ) { return __fmul_rn(fmaxf(__fsub_rn(r, q), 0.f), invZ); }
SV_DEV float rlast(float r, float q) { return fmaxf(__fsub_rn(r, q), 0.f); }

// Next child of node v with index > after, or -1.
SV_DEV int next_child(const AcceptParams &p, int v, int after) {
    for (int c = after + 1; c < p.N; ++c)
        if (p.parent[c] == v) return c;
    return -1;
}

SV_DEV float block_sum(float v, float *red) {
    v = warp_sum(v);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = 0.f;
    if (threadIdx.x == 0)
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    __syncthreads();
    return t;  // valid in thread 0
}

// ---------------------------------------------------------------------------
// 1. Row statistics per (slice, row, sequence).
// ---------------------------------------------------------------------------
template <bool GREEDY, bool VEC>
__global__ void __launch_bounds__(ACC_THREADS) accept_stats_kernel(const AcceptParams p) {
    griddep_wait();
    griddep_launch_dependents();
    const int j = blockIdx.x, v = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float *row = p.logits + ((size_t)b * p.N + v) * p.V;
    const int x0 = j * ACC_SLICE;
    const int n = min(ACC_SLICE, p.V - x0);
    // entry k of this thread: slice index 4*(tid + 256*(k/4)) + k%4 (vector) or tid + 256*k;
    // either way a thread's entries come in increasing index order
    float e[ACC_PER_THREAD];
    if (VEC) {
        const float4 *r4 = reinterpret_cast<const float4 *>(row + x0);
#pragma unroll
        for (int k = 0; k < ACC_PER_THREAD / 4; ++k) {
            const int i = tid + k * ACC_THREADS;
            const float4 f = 4 * i < n ? __ldg(r4 + i) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            e[4 * k] = f.x; e[4 * k + 1] = f.y; e[4 * k + 2] = f.z; e[4 * k + 3] = f.w;
        }
    } else {
#pragma unroll
        for (int k = 0; k < ACC_PER_THREAD; ++k) {
            const int i = tid + k * ACC_THREADS;
            e[k] = i < n ? __ldg(row + x0 + i) : -INFINITY;
        }
    }
    auto index_of = [&](int k) { return VEC ? x0 + 4 * (tid + (k >> 2) * ACC_THREADS) + (k & 3) : x0 + tid + k * ACC_THREADS; };
    int flag = 0;
    float m = -INFINITY, s = 0.f;
    int ai = -1;
    const float c = p.log2e_over_T;
    if (GREEDY) {
#pragma unroll
        for (int k = 0; k < ACC_PER_THREAD; ++k) {
            if (isnan(e[k]) || e[k] == INFINITY) { flag = 1; e[k] = -INFINITY; }
            if (e[k] > m) { m = e[k]; ai = index_of(k); }  // strict: the lowest index among equals
        }
    } else {
        // fmaxf skips NaN; a NaN or +inf entry then shows as a NaN sum (or an
        // infinite maximum), and only such a thread redoes its entries with
        // the non-finite ones replaced by -inf
#pragma unroll
        for (int k = 0; k < ACC_PER_THREAD; ++k) m = fmaxf(m, e[k]);
        if (m > -INFINITY && m < INFINITY) {
#pragma unroll
            for (int k = 0; k < ACC_PER_THREAD; ++k) s += pweight(e[k], m, c);
        }
        if (!(m > -INFINITY && m < INFINITY) || isnan(s)) {
            m = -INFINITY;
            s = 0.f;
#pragma unroll
            for (int k = 0; k < ACC_PER_THREAD; ++k) {
                if (isnan(e[k]) || e[k] == INFINITY) { flag = 1; e[k] = -INFINITY; }
                m = fmaxf(m, e[k]);
            }
            if (m != -INFINITY) {
#pragma unroll
                for (int k = 0; k < ACC_PER_THREAD; ++k) s += pweight(e[k], m, c);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, ai, o);
        if (GREEDY) merge_argmax(m, ai, m2, i2); else merge_sumexp(m, s, m2, s2, c);
    }
    flag = warp_or(flag);
    __shared__ float4 part[ACC_THREADS / 32];
    if (lane == 0) part[warp] = make_float4(m, s, __int_as_float(ai), __int_as_float(flag));
    __syncthreads();
    if (tid == 0) {
        float4 r = part[0];
        int I = __float_as_int(r.z), F = __float_as_int(r.w);
        for (int w = 1; w < ACC_THREADS / 32; ++w) {
            const float4 o = part[w];
            if (GREEDY) merge_argmax(r.x, I, o.x, __float_as_int(o.z));
            else merge_sumexp(r.x, r.y, o.x, o.y, c);
            F |= __float_as_int(o.w);
        }
        acc_ptrs(p).stats[((size_t)b * p.N + v) * p.S + j] = make_float4(r.x, r.y, __int_as_float(I), __int_as_float(F));
    }
}

// ---------------------------------------------------------------------------
// Residual weights. For node v with chain c_1..c_k of rejected children:
//   e(x) = 2^((l_v(x) - M_v) c),  r_0 = e / S_v,
//   r_i = max(0, r_{i-1} - q_{c_i}) / Z_i   (i < k),
//   weight = max(0, r_{k-1} - q_{c_k})      (unnormalised; its sum is Z_k).
// With k = 0 the weight is e (p_v unnormalised). The pass and the draw compute
// every weight with the same fp32 operations (pweight, rstart, rstep, rlast:
// the divisions as products with correctly rounded reciprocals), so they agree
// bit for bit.
// ---------------------------------------------------------------------------
// 3. Per-slice parts of the pending pass of a sequence.
// ---------------------------------------------------------------------------
template <bool VEC>
__global__ void __launch_bounds__(ACC_THREADS) accept_pass_kernel(const AcceptParams p) {
    griddep_wait();
    griddep_launch_dependents();
    const int j = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const AccPtrs w = acc_ptrs(p);
    const AccState *st = w.st + b;
    __shared__ int s_mode, s_v, s_k;
    __shared__ float s_M, s_S;
    __shared__ float s_Z[64];  // 1/Z_i
    __shared__ const float *s_q[64];
    if (tid == 0) {
        s_mode = __ldcg(&st->mode);
        // the rest of the state is only defined while a pass is pending
        if (s_mode == MODE_RESID || s_mode == MODE_P) {
            s_v = __ldcg(&st->v);
            s_k = s_mode == MODE_RESID ? __ldcg(&st->nchain) : 0;
            s_M = __ldcg(&st->rowM[s_v]);
            s_S = __ldcg(&st->rowS[s_v]);
        }
    }
    __syncthreads();
    const int mode = s_mode;
    if (mode != MODE_RESID && mode != MODE_P) return;
    const int k = s_k;
    const int x0 = j * ACC_SLICE;
    const int n = min(ACC_SLICE, p.V - x0);
    if (tid < k) {
        s_Z[tid] = __frcp_rn(__ldcg(&st->Z[tid]));  // 1/Z_i (the last entry is unused)
        s_q[tid] = p.q + ((size_t)b * (p.N - 1) + __ldcg(&st->chain[tid]) - 1) * p.V + x0;
    }
    __syncthreads();
    const float *lrow = p.logits + ((size_t)b * p.N + s_v) * p.V + x0;
    const float M = s_M, invS = __frcp_rn(s_S), c = p.log2e_over_T;
    float wsum = 0.f, psum = 0.f;
    if (VEC && k <= 1) {
        // p alone, or the chain case (one draft row): 16-byte loads, all of a
        // thread's loads in flight before the first is used
        const float4 *l4 = reinterpret_cast<const float4 *>(lrow);
        const float4 *q4 = reinterpret_cast<const float4 *>(k ? s_q[0] : lrow);
        constexpr int J = ACC_PER_THREAD / 4;
        float4 lv[J], qv[J];
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int i = tid + j * ACC_THREADS;
            lv[j] = 4 * i < n ? __ldg(l4 + i) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            qv[j] = (k && 4 * i < n) ? __ldg(q4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const float e0 = pweight(lv[j].x, M, c), e1 = pweight(lv[j].y, M, c);
            const float e2 = pweight(lv[j].z, M, c), e3 = pweight(lv[j].w, M, c);
            psum += (e0 + e1) + (e2 + e3);
            if (k)
                wsum += (rlast(rstart(e0, invS), qv[j].x) + rlast(rstart(e1, invS), qv[j].y)) +
                        (rlast(rstart(e2, invS), qv[j].z) + rlast(rstart(e3, invS), qv[j].w));
        }
    } else {
        for (int x = tid; x < n; x += ACC_THREADS) {
            const float e = pweight(__ldg(lrow + x), M, c);
            psum += e;
            if (k) {
                float r = rstart(e, invS);
                for (int i = 0; i + 1 < k; ++i) r = rstep(r, __ldg(s_q[i] + x), s_Z[i]);
                wsum += rlast(r, __ldg(s_q[k - 1] + x));
            }
        }
    }
    __shared__ float red[2][ACC_THREADS / 32];
    const float ws = block_sum(wsum, red[0]);
    const float ps = block_sum(psum, red[1]);
    if (tid == 0) w.rsum[(size_t)b * p.S + j] = make_float2(ws, ps);
}

// ---------------------------------------------------------------------------
// 2 / 4. The walk of one sequence (one CTA; the walk itself on thread 0).
// ---------------------------------------------------------------------------
enum { ACT_PASS = 0, ACT_DRAW = 1 };

// Sampling walk from the state in S until a pass is needed or the draw.
SV_DEV int walk_sampling(const AcceptParams &p, AccState &S, int b) {
    const float c = p.log2e_over_T;
    const PhiloxKey key{p.key.k0, p.key.k1};
    for (;;) {
        const int v = S.v;
        const int ch = next_child(p, v, S.last_tried);
        if (ch < 0) {
            if (S.have_pass) return ACT_DRAW;  // every child was rejected: draw from that residual (or p_v)
            S.mode = MODE_P;                   // a node without children: the draw needs p_v's mass
            return ACT_PASS;
        }
        S.last_tried = ch;
        const int d = S.dr[ch];
        bool acc = false;
        if (d < 0 || d >= p.V) {
            S.flags |= SV_FLAG_BAD_TOKEN;  // counts as a rejection
        } else {
            const float u = philox_uniform(key, (uint32_t)b, (uint32_t)ch, 0u);
            float r = rstart(pweight(S.Ld[ch], S.rowM[v], c), __frcp_rn(S.rowS[v]));
            for (int i = 0; i < S.nchain; ++i) {
                const float qx = __ldg(p.q + ((size_t)b * (p.N - 1) + S.chain[i] - 1) * p.V + d);
                r = rstep(r, qx, __frcp_rn(S.Z[i]));
            }
            acc = u * S.Qd[ch] < r;
        }
        if (acc) {
            S.path[S.depth++] = ch;
            S.v = ch;
            S.nchain = 0;
            S.have_pass = 0;
            continue;
        }
        S.chain[S.nchain++] = ch;  // its residual's mass is the next pass
        S.have_pass = 0;
        S.mode = MODE_RESID;
        return ACT_PASS;
    }
}

SV_DEV void write_outputs(const AcceptParams &p, int b, int depth, const int *path, int tok, int flags) {
    p.accept_len[b] = depth;
    p.next_token[b] = tok;
    if (p.accept_path)
        for (int k = 0; k < p.N - 1; ++k) p.accept_path[(size_t)b * (p.N - 1) + k] = k < depth ? path[k] : -1;
    if (p.status) p.status[b] = flags;
}

template <bool GREEDY>
__global__ void __launch_bounds__(WALK_THREADS, 1) accept_walk_kernel(const AcceptParams p, int round) {
    griddep_wait();
    griddep_launch_dependents();
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const AccPtrs W = acc_ptrs(p);
    __shared__ AccState S;
    // draw: the weights of the drawn slice, one pad word after every 32 so that
    // a thread's contiguous segment of 32 sits in 32 different banks
    __shared__ float wbuf[ACC_SLICE + ACC_SLICE / 32];
    __shared__ float2 rs[ACC_MAX_VOCAB / ACC_SLICE];  // the pass's per-slice sums
    __shared__ int s_action, s_nonfinite, s_owner, s_first;
    __shared__ float s_t;
    __shared__ float red_f[WALK_THREADS / 32];
    __shared__ int red_i[WALK_THREADS / 32];
    const int N = p.N;
    const float c = p.log2e_over_T;

    if (round == 0) {
        if (tid == 0) s_nonfinite = 0;
        __syncthreads();
        // row statistics merged over the slices: one warp per row, the lanes'
        // loads in flight together, then a butterfly merge (a fixed order)
        for (int v = warp; v < N; v += WALK_THREADS / 32) {
            const float4 *sr = W.stats + ((size_t)b * N + v) * p.S;
            float M = -INFINITY, Ssum = 0.f;
            int I = -1, F = 0;
            for (int j = lane; j < p.S; j += 32) {
                const float4 x = __ldcg(sr + j);
                if (GREEDY) merge_argmax(M, I, x.x, __float_as_int(x.z));
                else merge_sumexp(M, Ssum, x.x, x.y, c);
                F |= __float_as_int(x.w);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float m2 = __shfl_xor_sync(0xffffffffu, M, o);
                const float s2 = __shfl_xor_sync(0xffffffffu, Ssum, o);
                const int i2 = __shfl_xor_sync(0xffffffffu, I, o);
                if (GREEDY) merge_argmax(M, I, m2, i2); else merge_sumexp(M, Ssum, m2, s2, c);
            }
            F = warp_or(F);
            if (lane == 0) {
                if (M == -INFINITY) F = 1;  // no finite logit in the row
                S.rowM[v] = M;
                S.rowS[v] = Ssum;
                S.rowArg[v] = I;
                if (F) atomicOr(&s_nonfinite, 1);
            }
        }
        if (tid >= 1 && tid < N) {
            // decision inputs of draft node c: independent loads, done once
            const int ch = tid, d = __ldg(p.drafts + (size_t)b * (N - 1) + ch - 1);
            S.dr[ch] = d;
            if (d >= 0 && d < p.V) {
                S.Ld[ch] = __ldg(p.logits + ((size_t)b * N + p.parent[ch]) * p.V + d);
                if (!GREEDY) S.Qd[ch] = __ldg(p.q + ((size_t)b * (N - 1) + ch - 1) * p.V + d);
            }
        }
        if (tid == 0) {
            S.mode = MODE_NONE; S.v = 0; S.depth = 0; S.flags = 0; S.last_tried = 0; S.nchain = 0;
            S.have_pass = 0;
        }
        __syncthreads();
        if (s_nonfinite) {
            if (tid == 0) {
                write_outputs(p, b, 0, S.path, 0, SV_FLAG_NONFINITE);
                W.st[b].mode = MODE_DONE;
            }
            return;
        }
        if (GREEDY) {
            if (tid == 0) {
                int v = 0, depth = 0, flags = 0, tok;
                for (;;) {
                    const int am = S.rowArg[v];
                    int moved = -1;
                    for (int ch = next_child(p, v, v); ch >= 0; ch = next_child(p, v, ch)) {
                        const int d = S.dr[ch];
                        if (d < 0 || d >= p.V) { flags |= SV_FLAG_BAD_TOKEN; continue; }
                        if (d == am) { moved = ch; break; }
                    }
                    if (moved < 0) { tok = am; break; }
                    S.path[depth++] = moved;
                    v = moved;
                }
                write_outputs(p, b, depth, S.path, tok, flags);
                W.st[b].mode = MODE_DONE;
            }
            return;
        }
    } else {
        // resume: the state, then the sum of the pass that was asked for
        const int4 *src = reinterpret_cast<const int4 *>(W.st + b);
        int4 *dst = reinterpret_cast<int4 *>(&S);
        for (int i = tid; i < (int)(sizeof(AccState) / 16); i += WALK_THREADS) dst[i] = __ldcg(src + i);
        for (int j = tid; j < p.S; j += WALK_THREADS) rs[j] = __ldcg(W.rsum + (size_t)b * p.S + j);
        __syncthreads();
        if (S.mode != MODE_RESID && S.mode != MODE_P) return;  // finished, or nothing asked
        if (tid == 0) {
            if (S.mode == MODE_RESID) {
                float Z = 0.f;
                for (int j = 0; j < p.S; ++j) Z += rs[j].x;
                if (Z > 0.f) S.Z[S.nchain - 1] = Z;
                else S.nchain = 0;  // no residual mass (rounding only): r falls back to p_v
            }
            S.mode = MODE_NONE;
            S.have_pass = 1;
        }
        __syncthreads();
    }

    if (tid == 0) s_action = walk_sampling(p, S, b);
    __syncthreads();
    if (s_action == ACT_PASS) {
        // hand the state to the pass kernel and the next walk
        const int4 *src = reinterpret_cast<const int4 *>(&S);
        int4 *dst = reinterpret_cast<int4 *>(W.st + b);
        for (int i = tid; i < (int)(sizeof(AccState) / 16); i += WALK_THREADS) dst[i] = src[i];
        return;
    }

    // ---- draw at node v from the residual of its rejected chain, or from p_v ----
    const int v = S.v, k = S.nchain;
    const bool use_w = k > 0;
    if (tid == 0) {
        float tot = 0.f;
        for (int j = 0; j < p.S; ++j) {
            const float2 x = rs[j];
            tot += use_w ? x.x : x.y;
        }
        const float u = philox_uniform(PhiloxKey{p.key.k0, p.key.k1}, (uint32_t)b, (uint32_t)v, 1u);
        const float t = u * tot;
        int owner = -1, lastpos = 0;
        float pre = 0.f, tk = 0.f;
        for (int j = 0; j < p.S; ++j) {
            const float2 x = rs[j];
            const float sj = use_w ? x.x : x.y;
            if (owner < 0 && t - pre < sj) { owner = j; tk = t - pre; }
            pre += sj;
            if (sj > 0.f) lastpos = j;
        }
        if (owner < 0) { owner = lastpos; tk = INFINITY; }  // rounding: the last token with weight
        s_owner = owner;
        s_t = tk;
    }
    __syncthreads();
    const int x0 = s_owner * ACC_SLICE;
    const int n = min(ACC_SLICE, p.V - x0);
    {
        // the drawn slice's weights, with the pass's arithmetic, staged in shared
        // memory; a thread's loads are all in flight before the first is used
        const float *lrow = p.logits + ((size_t)b * N + v) * p.V + x0;
        const float M = S.rowM[v], invS = __frcp_rn(S.rowS[v]);
        auto put = [&](int x, float wgt) { wbuf[x + (x >> 5)] = wgt; };
        if (p.vec && k <= 1) {
            const float4 *l4 = reinterpret_cast<const float4 *>(lrow);
            const float4 *q4 = k ? reinterpret_cast<const float4 *>(
                                       p.q + ((size_t)b * (N - 1) + S.chain[0] - 1) * p.V + x0)
                                 : l4;
            constexpr int J = ACC_SLICE / (4 * WALK_THREADS);
            float4 lv[J], qv[J];
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int i = tid + j * WALK_THREADS;
                lv[j] = 4 * i < n ? __ldg(l4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                qv[j] = (k && 4 * i < n) ? __ldg(q4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int i = tid + j * WALK_THREADS;
                if (4 * i >= n) continue;
                const float l[4] = {lv[j].x, lv[j].y, lv[j].z, lv[j].w};
                const float q[4] = {qv[j].x, qv[j].y, qv[j].z, qv[j].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float ex = pweight(l[e], M, c);
                    put(4 * i + e, k ? rlast(rstart(ex, invS), q[e]) : ex);
                }
            }
        } else {
            for (int x = tid; x < n; x += WALK_THREADS) {
                const float e = pweight(__ldg(lrow + x), M, c);
                float wgt = e;
                if (use_w) {
                    float r = rstart(e, invS);
                    for (int i = 0; i + 1 < k; ++i)
                        r = rstep(r, __ldg(p.q + ((size_t)b * (N - 1) + S.chain[i] - 1) * p.V + x0 + x),
                                  __frcp_rn(S.Z[i]));
                    wgt = rlast(r, __ldg(p.q + ((size_t)b * (N - 1) + S.chain[k - 1] - 1) * p.V + x0 + x));
                }
                put(x, wgt);
            }
        }
    }
    __syncthreads();
    // contiguous segment per thread, summed in index order, then an exclusive
    // scan of the segment sums in thread order
    const int s0 = min(tid * WALK_SEG, n), s1 = min(s0 + WALK_SEG, n);
    float tsum = 0.f;
    int tlast = -1;
    for (int x = s0; x < s1; ++x) {
        const float wv = wbuf[x + (x >> 5)];
        tsum += wv;
        if (wv > 0.f) tlast = x;
    }
    float incl = tsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    int wl = tlast;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wl = max(wl, __shfl_xor_sync(0xffffffffu, wl, o));
    if (lane == 31) red_f[warp] = incl;
    if (lane == 0) red_i[warp] = wl;
    __syncthreads();
    float wpre = 0.f;
    int slast = -1;
    for (int w = 0; w < WALK_THREADS / 32; ++w) {
        if (w < warp) wpre += red_f[w];
        slast = max(slast, red_i[w]);
    }
    const float tj = s_t - (wpre + incl - tsum);
    // the first thread (lowest tid) whose segment holds the threshold
    const unsigned bal = __ballot_sync(0xffffffffu, s1 > s0 && tj < tsum);
    __syncthreads();
    if (lane == 0) red_i[warp] = bal ? warp * 32 + __ffs(bal) - 1 : 0x7fffffff;
    __syncthreads();
    if (tid == 0) {
        int first = 0x7fffffff;
        for (int w = 0; w < WALK_THREADS / 32; ++w) first = min(first, red_i[w]);
        s_first = first;
    }
    __syncthreads();
    const int first = s_first;
    int tok = -1;
    if (first == 0x7fffffff) {
        if (tid == 0) tok = x0 + max(slast, 0);  // rounding: the slice's last token with weight
    } else if (tid == first) {
        float cl = 0.f;
        tok = x0 + max(tlast, s0);
        for (int x = s0; x < s1; ++x) {
            const float wv = wbuf[x + (x >> 5)];
            cl += wv;
            if (wv > 0.f && cl > tj) { tok = x0 + x; break; }
        }
    }
    if (tok >= 0) {
        write_outputs(p, b, S.depth, S.path, tok, S.flags);
        W.st[b].mode = MODE_DONE;
    }
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
int accept_rounds(const int8_t *parent, int N) {
    int best = 1;
    for (int v = 0; v < N; ++v) {
        int rej = 0;  // children rejected on the way to v: the earlier siblings of each node on the path
        for (int u = v; u > 0; u = parent[u])
            for (int c = 1; c < u; ++c) rej += parent[c] == parent[u];
        int kids = 0;
        for (int c = v + 1; c < N; ++c) kids += parent[c] == v;
        best = std::max(best, rej + std::max(kids, 1));
    }
    return best;
}

template <typename... Args>
static cudaError_t launch_pdl(void (*kfn)(Args...), dim3 grid, dim3 block, cudaStream_t stream, const Args &...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kfn, args...);
}

cudaError_t launch_accept(const AcceptParams &p0, int rounds, cudaStream_t stream, int *launches) {
    auto a16 = [](const void *x) { return (reinterpret_cast<uintptr_t>(x) & 15) == 0; };
    const bool vec = (p0.V % 4 == 0) && a16(p0.logits) && (p0.greedy || p0.q == nullptr || a16(p0.q));
    AcceptParams pv = p0;
    pv.vec = vec ? 1 : 0;
    const AcceptParams &p = pv;
    const dim3 sgrid((unsigned)p.S, (unsigned)p.N, (unsigned)p.B);
    cudaError_t e;
    int n = 0;
    if (p.greedy) {
        e = vec ? launch_pdl(accept_stats_kernel<true, true>, sgrid, dim3(ACC_THREADS), stream, p)
                : launch_pdl(accept_stats_kernel<true, false>, sgrid, dim3(ACC_THREADS), stream, p);
        if (e != cudaSuccess) return e;
        ++n;
        e = launch_pdl(accept_walk_kernel<true>, dim3((unsigned)p.B), dim3(WALK_THREADS), stream, p, 0);
        if (e != cudaSuccess) return e;
        if (launches) *launches = n + 1;
        return cudaSuccess;
    }
    e = vec ? launch_pdl(accept_stats_kernel<false, true>, sgrid, dim3(ACC_THREADS), stream, p)
            : launch_pdl(accept_stats_kernel<false, false>, sgrid, dim3(ACC_THREADS), stream, p);
    if (e != cudaSuccess) return e;
    e = launch_pdl(accept_walk_kernel<false>, dim3((unsigned)p.B), dim3(WALK_THREADS), stream, p, 0);
    if (e != cudaSuccess) return e;
    n = 2;
    for (int r = 1; r <= rounds; ++r) {
        const dim3 pgrid((unsigned)p.S, (unsigned)p.B);
        e = vec ? launch_pdl(accept_pass_kernel<true>, pgrid, dim3(ACC_THREADS), stream, p)
                : launch_pdl(accept_pass_kernel<false>, pgrid, dim3(ACC_THREADS), stream, p);
        if (e != cudaSuccess) return e;
        e = launch_pdl(accept_walk_kernel<false>, dim3((unsigned)p.B), dim3(WALK_THREADS), stream, p, r);
        if (e != cudaSuccess) return e;
        n += 2;
    }
    if (launches) *launches = n;
    return cudaSuccess;
}

}  // namespace sv
