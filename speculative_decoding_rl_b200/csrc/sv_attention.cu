// sv_verify_attention: GQA attention of every active sequence's N draft query
// rows over its paged bf16 KV cache, split over the context and combined.
//
// The target scores all gamma+1 positions in one pass (TLT reading notes,
// "1. RL and SD"); with a draft tree, row i sees only its ancestors among the
// new positions (SRT review, "Speculative Rollout integration", step 5:
// tree verification). The KV pool is the one the drafter shares with the
// target (EfficientRollout, "Key modules" 1).
//
// Work decomposition (one persistent CTA per SM):
//   unit  = (sequence b, KV head h, row chunk rc): the N*G query rows of the G
//           query heads that read KV head h, at most ROWS_MAX per chunk;
//   tile  = TILE_KEYS consecutive keys of one unit;
//   All tiles of all units are laid end to end and cut into num_ctas equal
//   ranges, so every SM streams the same number of KV bytes whatever the mix
//   of context lengths. Where a CTA's range covers part of a unit it writes a
//   partial (unnormalised O, running max m, running sum l) to workspace slot
//   unit + cta, which is unique because consecutive units can share at most
//   one CTA. The combine kernel merges a unit's partials by their log-sum-exp.
#include "sv_device.cuh"
#include "sv_internal.h"

namespace sv {

// ---------------------------------------------------------------------------
// Schedule helpers (attention and combine kernels agree on these).
// ---------------------------------------------------------------------------
SV_DEV int seq_tiles(const AttnParams &p, int b) {
    const int C = p.ctx_lens[b];
    const bool ok = C >= p.N && C <= p.max_blocks * PAGE;
    return ok ? (C + TILE_KEYS - 1) / TILE_KEYS : 0;
}

// Exclusive prefix of per-sequence tile counts into TP[0..B]; whole block participates.
SV_DEV void tile_prefix(const AttnParams &p, int *TP, int *scratch) {
    const int nt = blockDim.x, tid = threadIdx.x;
    const int per = (p.B + nt - 1) / nt;
    const int s0 = min(tid * per, p.B), s1 = min(s0 + per, p.B);
    int local = 0;
    for (int b = s0; b < s1; ++b) local += seq_tiles(p, b);
    // block exclusive scan of `local`
    const int lane = tid & 31, warp = tid >> 5;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    int wpre = 0;
    for (int w = 0; w < warp; ++w) wpre += scratch[w];
    int run = wpre + incl - local;
    for (int b = s0; b < s1; ++b) {
        TP[b] = run;
        run += seq_tiles(p, b);
    }
    if (tid == nt - 1) TP[p.B] = run;
    __syncthreads();
}

// Tile t -> sequence b (largest b with ups*TP[b] <= t), by binary search.
SV_DEV int tile_seq(const int *TP, int B, int ups, int t) {
    int lo = 0, hi = B;  // invariant: ups*TP[lo] <= t < ups*TP[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ups * TP[mid] <= t) lo = mid; else hi = mid;
    }
    return lo;
}

SV_DEV bool key_visible(const AttnParams &p, int b, int C, int i, int t) {
    if (t >= C) return false;
    const int j = t - (C - p.N);
    if (j < 0) return true;
    if (p.mask) return (p.mask[(size_t)b * p.N + i] >> j) & 1ull;
    return j <= i;
}

// ---------------------------------------------------------------------------
// Split-context attention on the CUDA cores: one page (16 keys) at a time,
// fp32 in shared memory. Straightforward and exact to fp32 rounding.
// ---------------------------------------------------------------------------
constexpr int V1_THREADS = 256;

__global__ void __launch_bounds__(V1_THREADS, 1) attn_split_kernel(const AttnParams p) {
    extern __shared__ __align__(16) float sm[];
    const int D = p.D, RU = p.rows_unit;
    int *TP = reinterpret_cast<int *>(sm);
    int *scratch = TP + ((p.B + 1 + 3) & ~3);
    float *Qs = reinterpret_cast<float *>(scratch + 32);
    float *Ks = Qs + RU * D;
    float *Vs = Ks + PAGE * (D + 1);
    float *Ps = Vs + PAGE * D;
    float *Os = Ps + RU * PAGE;
    float *mrow = Os + RU * D;
    float *lrow = mrow + RU;
    float *arow = lrow + RU;

    const int tid = threadIdx.x, nt = blockDim.x;
    tile_prefix(p, TP, scratch);
    const int ups = p.Hkv * p.RC;
    const int total = ups * TP[p.B];
    if (total == 0) {
        if (blockIdx.x == 0 && tid == 0) { p.ws_plan[0] = 1; p.ws_plan[1] = 0; }
        if (blockIdx.x == 0) for (int b = tid; b <= p.B; b += nt) p.ws_plan[2 + b] = TP[b];
        return;
    }
    const int W = (total + p.num_ctas - 1) / p.num_ctas;
    if (blockIdx.x == 0) {
        if (tid == 0) { p.ws_plan[0] = W; p.ws_plan[1] = total; }
        for (int b = tid; b <= p.B; b += nt) p.ws_plan[2 + b] = TP[b];
    }
    const int t_begin = blockIdx.x * W;
    const int t_end = min(t_begin + W, total);
    const size_t slot_floats = (size_t)RU * D + 2 * RU;

    int cur_u = -1, b = 0, h = 0, rc = 0, rows = 0, C = 0;
    for (int t = t_begin; t <= t_end; ++t) {
        int nb = 0, nhr = 0, j = 0, u = -1;
        if (t < t_end) {
            nb = tile_seq(TP, p.B, ups, t);
            const int Tb = TP[nb + 1] - TP[nb];
            const int off = t - ups * TP[nb];
            nhr = off / Tb;
            j = off - nhr * Tb;
            u = nb * ups + nhr;
        }
        if (u != cur_u) {
            if (cur_u >= 0) {  // flush the finished segment
                float *slot = p.ws_partial + (size_t)(cur_u + blockIdx.x) * slot_floats;
                for (int e = tid; e < rows * D; e += nt) slot[e] = Os[e];
                for (int r = tid; r < rows; r += nt) {
                    slot[(size_t)RU * D + r] = mrow[r];
                    slot[(size_t)RU * D + RU + r] = lrow[r];
                }
            }
            if (u < 0) break;
            cur_u = u;
            b = nb;
            h = nhr / p.RC;
            rc = nhr - h * p.RC;
            rows = min(ROWS_MAX, p.R - rc * ROWS_MAX);
            C = p.ctx_lens[b];
            __syncthreads();
            for (int e = tid; e < rows * D; e += nt) {
                const int r = e / D, d = e - r * D;
                const int ridx = rc * ROWS_MAX + r;
                const int i = ridx / p.G, hq = h * p.G + (ridx - i * p.G);
                Qs[e] = bf16_bits_to_float(p.q[(((size_t)b * p.N + i) * p.Hq + hq) * D + d]);
                Os[e] = 0.f;
            }
            for (int r = tid; r < rows; r += nt) { mrow[r] = -INFINITY; lrow[r] = 0.f; }
            __syncthreads();
        }
        // ---- tile j of the unit: up to 8 pages ----
        const int k0 = j * TILE_KEYS;
        for (int pg = k0 / PAGE; pg < (k0 + TILE_KEYS) / PAGE; ++pg) {
            const int t0 = pg * PAGE;
            if (t0 >= C) break;
            const int blk = p.block_table[(size_t)b * p.max_blocks + pg];
            const bool bad = blk < 0 || blk >= p.num_blocks;
            for (int e = tid; e < PAGE * D; e += nt) {
                const int n = e / D, d = e - n * D;
                float kv = 0.f, vv = 0.f;
                if (!bad && t0 + n < C) {
                    const size_t off = (((size_t)blk * p.Hkv + h) * PAGE + n) * D + d;
                    kv = bf16_bits_to_float(p.k_pool[off]);
                    vv = bf16_bits_to_float(p.v_pool[off]);
                }
                Ks[n * (D + 1) + d] = kv;
                Vs[n * D + d] = vv;
            }
            __syncthreads();
            for (int e = tid; e < rows * PAGE; e += nt) {
                const int r = e >> 4, n = e & 15;
                const int ridx = rc * ROWS_MAX + r;
                const int i = ridx / p.G;
                float s = -INFINITY;
                if (key_visible(p, b, C, i, t0 + n)) {
                    float acc = 0.f;
                    const float *qr = Qs + r * D;
                    const float *kr = Ks + n * (D + 1);
                    for (int d = 0; d < D; ++d) acc = fmaf(qr[d], kr[d], acc);
                    s = acc * p.scale_log2;
                }
                Ps[e] = s;
            }
            __syncthreads();
            for (int r = tid; r < rows; r += nt) {
                float mx = mrow[r];
                for (int n = 0; n < PAGE; ++n) mx = fmaxf(mx, Ps[r * PAGE + n]);
                float alpha = 1.f;
                if (mx == -INFINITY) {
                    for (int n = 0; n < PAGE; ++n) Ps[r * PAGE + n] = 0.f;
                } else {
                    alpha = exp2f(mrow[r] - mx);  // 0 when mrow is -inf
                    float sum = 0.f;
                    for (int n = 0; n < PAGE; ++n) {
                        const float e = exp2f(Ps[r * PAGE + n] - mx);
                        Ps[r * PAGE + n] = e;
                        sum += e;
                    }
                    lrow[r] = lrow[r] * alpha + sum;
                    mrow[r] = mx;
                }
                arow[r] = alpha;
            }
            __syncthreads();
            for (int e = tid; e < rows * D; e += nt) {
                const int r = e / D, d = e - r * D;
                float o = Os[e] * arow[r];
                const float *pr = Ps + r * PAGE;
#pragma unroll
                for (int n = 0; n < PAGE; ++n) o = fmaf(pr[n], Vs[n * D + d], o);
                Os[e] = o;
            }
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------------------
// Combine: merge a unit's partials, normalise, write bf16; one CTA per
// (row of a unit, unit), one thread per head dimension. The CTA of row 0 of
// each sequence's first unit also writes that sequence's status flags.
// ---------------------------------------------------------------------------
__global__ void attn_combine_kernel(const AttnParams p) {
    const int r = blockIdx.x, u = blockIdx.y, d = threadIdx.x;
    const int D = p.D, RU = p.rows_unit;
    const int ups = p.Hkv * p.RC;
    const int b = u / ups, hr = u - b * ups;
    const int h = hr / p.RC, rc = hr - h * p.RC;
    const int rows = min(ROWS_MAX, p.R - rc * ROWS_MAX);
    if (r >= rows) return;
    const int ridx = rc * ROWS_MAX + r;
    const int i = ridx / p.G, hq = h * p.G + (ridx - i * p.G);
    const int W = p.ws_plan[0];
    const int *TP = p.ws_plan + 2;
    const int Tb = TP[b + 1] - TP[b];
    const size_t slot_floats = (size_t)RU * D + 2 * RU;
    float res = 0.f;
    if (Tb > 0) {
        const int tpre = ups * TP[b] + hr * Tb;
        const int first = tpre / W, last = (tpre + Tb - 1) / W;
        float M = -INFINITY;
        for (int c = first; c <= last; ++c)
            M = fmaxf(M, p.ws_partial[(size_t)(u + c) * slot_floats + (size_t)RU * D + r]);
        if (M > -INFINITY) {
            float L = 0.f, acc = 0.f;
            for (int c = first; c <= last; ++c) {
                const float *slot = p.ws_partial + (size_t)(u + c) * slot_floats;
                const float m = slot[(size_t)RU * D + r];
                if (m == -INFINITY) continue;
                const float w = exp2f(m - M);
                L = fmaf(w, slot[(size_t)RU * D + RU + r], L);
                acc = fmaf(w, slot[(size_t)r * D + d], acc);
            }
            res = acc / L;
        }
    }
    const __nv_bfloat16 o = __float2bfloat16_rn(res);
    p.out[(((size_t)b * p.N + i) * p.Hq + hq) * D + d] = *reinterpret_cast<const uint16_t *>(&o);

    if (p.status && r == 0 && hr == 0) {
        const int C = p.ctx_lens[b];
        const bool ctx_ok = C >= p.N && C <= p.max_blocks * PAGE;
        int bad = 0;
        if (ctx_ok)
            for (int jb = d; jb < (C + PAGE - 1) / PAGE; jb += blockDim.x) {
                const int blk = p.block_table[(size_t)b * p.max_blocks + jb];
                bad |= (blk < 0 || blk >= p.num_blocks);
            }
        bad = __syncthreads_or(bad);
        if (d == 0) p.status[b] = (ctx_ok ? 0 : SV_FLAG_BAD_CONTEXT) | (bad ? SV_FLAG_BAD_BLOCK : 0);
    }
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
static size_t plan_bytes(int B) { return (((size_t)(B + 3) * 4) + 255) & ~(size_t)255; }

static int rows_per_unit(int N, int Hq, int Hkv) {
    const int R = N * (Hq / Hkv);
    return R < ROWS_MAX ? R : ROWS_MAX;
}

int attention_num_ctas() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return sms;
}

size_t attention_workspace_bytes(int B, int N, int Hq, int Hkv, int D, int num_ctas) {
    const int R = N * (Hq / Hkv);
    const int RC = (R + ROWS_MAX - 1) / ROWS_MAX;
    const int RU = rows_per_unit(N, Hq, Hkv);
    const size_t units = (size_t)B * Hkv * RC;
    const size_t slot_floats = (size_t)RU * D + 2 * RU;
    return plan_bytes(B) + (units + (size_t)num_ctas) * slot_floats * sizeof(float);
}

cudaError_t launch_attention(const AttnParams &p0, cudaStream_t stream) {
    AttnParams p = p0;
    const int D = p.D, RU = p.rows_unit;
    const size_t smem = sizeof(int) * ((size_t)((p.B + 1 + 3) & ~3) + 32) +
                        sizeof(float) * ((size_t)RU * D + PAGE * (D + 1) + PAGE * D + RU * PAGE +
                                         (size_t)RU * D + 3 * RU);
    cudaError_t e = cudaFuncSetAttribute(attn_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    attn_split_kernel<<<p.num_ctas, V1_THREADS, smem, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_combine_kernel<<<dim3(RU, p.units), D, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace sv
