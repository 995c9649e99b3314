// sv_cascade_verify_attention: verify attention for groups of rollouts that
// share a prompt's KV pages.
//
// The rollouts of one prompt share its prefix, stored once (SRT review,
// "Tree-Structured KV Cache": node sharing), and reusing that prefix's KV with
// fewer memory accesses is where the speed-up comes from (SRT review,
// "Speculative Rollout integration"). The plain call streams every member's
// whole context, so a group's prefix pages are fetched once per member (from
// L2 at best). Here the prefix is read once per group and KV head for the
// query rows of ALL the group's members, which turns it into a dense
// (members x N x G rows) by (prefix keys) product.
//
// Softmax over a union of key sets is the log-sum-exp merge of the softmaxes
// over the parts, so the result is attention over the whole context:
//   cascade_prep_kernel    one CTA per sequence: checks the prefix against the
//                          context, writes the member's suffix length and
//                          suffix block table (its own pages after the prefix)
//                          and flags bad block ids among the prefix pages;
//   cascade_prefix_kernel  one CTA per (group, KV head, prefix split, chunk of
//                          64 group rows): 4 warps x 16 rows; 64-key tiles of
//                          the shared pages, double-buffered through
//                          cp.async; S = Q K^T and O += P V with
//                          mma.sync m16n8k16 (bf16 in, fp32 accumulate),
//                          online softmax in the log2 domain; writes an
//                          unnormalised partial (O, running max, row sum) per
//                          row and split;
//   launch_attention       the split-context tcgen05 kernel over every
//                          member's suffix (own pages, draft rows and masks),
//                          every unit through a workspace slot, and the combine
//                          kernel that folds the prefix partials into each row.
#include <string.h>

#include "sv_internal.h"
#include "sv_tc.cuh"

namespace sv {
namespace {

using tc::ex2_approx;
using tc::smem_u32;

constexpr int PF_WARPS = CASCADE_ROWS / 16;  // one m16 row block per warp
constexpr int PF_THREADS = 32 * PF_WARPS;
constexpr int PREP_THREADS = 128;
constexpr int MAX_SPLITS = 8;
constexpr int PF_CTAS_PER_SM = 3;  // resident prefix CTAs per SM (launch bounds; 69.6 KB shared memory each)
// Running max of a row that has seen no key: finite, so that 2^(M_NONE - m) = 0.
constexpr float PF_M_NONE = -3.402823466e38f;

struct PrepParams {
    const int32_t *block_table, *ctx_lens;
    int32_t *sfx_ctx, *sfx_table, *pflag;
    int B, N, max_blocks, num_blocks;
    CascadePlan plan;
};

struct PrefixParams {
    const uint16_t *q, *k_pool, *v_pool;  // bf16 bits
    const int32_t *block_table;
    float *pp_o, *pp_ml;
    int B, N, Hq, Hkv, G, max_blocks, num_blocks;
    float scale_log2;
    CascadePlan plan;
};

// Largest g in [0, n) with x[g] <= v, for nondecreasing x with x[0] <= v.
SV_DEV int upper_index(const int *x, int n, int v) {
    int lo = 0, hi = n;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (x[mid] <= v) lo = mid; else hi = mid;
    }
    return lo;
}

SV_DEV void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    // src_bytes = 0 fills the 16 bytes with zeros and reads nothing
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
SV_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int n>
SV_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(n) : "memory"); }

SV_DEV void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
SV_DEV void ldsm_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
// c[16x8] += a[16x16] * b[16x8], bf16 operands, fp32 accumulators.
SV_DEV void mma_16816(float *c, const uint32_t *a, uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
SV_DEV uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // lo in the low half
    return *reinterpret_cast<const uint32_t *>(&v);
}

__global__ void __launch_bounds__(PREP_THREADS) cascade_prep_kernel(const __grid_constant__ PrepParams p) {
    const int b = blockIdx.x;
    const CascadePlan &pl = p.plan;
    const int g = upper_index(pl.off, pl.num_groups, b);  // off[g] <= b < off[g+1]
    const int P = pl.pre[g], first = pl.off[g];
    const int C = p.ctx_lens[b];
    const bool ok = C >= p.N && C <= p.max_blocks * PAGE && P <= C - p.N;
    if (!ok) {  // the attention kernel flags SV_FLAG_BAD_CONTEXT and writes zeros
        if (threadIdx.x == 0) {
            p.sfx_ctx[b] = -1;
            p.pflag[b] = 0;
        }
        return;
    }
    const int np = P / PAGE, ns = (C - P + PAGE - 1) / PAGE;  // np + ns <= max_blocks
    const int32_t *own = p.block_table + (size_t)b * p.max_blocks + np;
    int32_t *dst = p.sfx_table + (size_t)b * p.max_blocks;
    for (int j = threadIdx.x; j < ns; j += PREP_THREADS) dst[j] = __ldg(own + j);
    const int32_t *shared_pages = p.block_table + (size_t)first * p.max_blocks;
    int bad = 0;
    for (int j = threadIdx.x; j < np; j += PREP_THREADS) {
        const int blk = __ldg(shared_pages + j);
        bad |= blk < 0 || blk >= p.num_blocks;
    }
    bad = __syncthreads_or(bad);
    if (threadIdx.x == 0) {
        p.sfx_ctx[b] = C - P;
        p.pflag[b] = bad ? SV_FLAG_BAD_BLOCK : 0;
    }
}

template <int D>
__global__ void __launch_bounds__(PF_THREADS, PF_CTAS_PER_SM) cascade_prefix_kernel(const __grid_constant__ PrefixParams p) {
    constexpr int LD = D + 8;                   // padded row: ldmatrix rows land on distinct banks
    constexpr int TILE = CASCADE_KEYS * LD;     // bf16 elements of one K or V tile
    constexpr int NT = CASCADE_KEYS / 8;        // 8-key column blocks of S
    constexpr int KS = D / 16;                  // 16-dim steps of Q K^T
    extern __shared__ __align__(16) uint16_t pf_smem[];
    uint16_t *Ks = pf_smem;                     // [2][CASCADE_KEYS][LD]
    uint16_t *Vs = pf_smem + 2 * TILE;          // [2][CASCADE_KEYS][LD]

    // ---- work item -> (group, KV head, split, row chunk) ----
    const CascadePlan &pl = p.plan;
    const int it = blockIdx.x;
    const int g = upper_index(pl.item0, pl.num_groups, it);
    const int b0 = pl.off[g];
    const int NG = p.N * p.G;
    const int rows_g = (pl.off[g + 1] - b0) * NG;
    const int chunks = (rows_g + CASCADE_ROWS - 1) / CASCADE_ROWS;
    int rem = it - pl.item0[g];
    const int chunk = rem % chunks;
    rem /= chunks;
    const int s = rem % pl.splits, h = rem / pl.splits;
    const int P = pl.pre[g];
    const int nt_all = (P + CASCADE_KEYS - 1) / CASCADE_KEYS;
    const int tps = (nt_all + pl.splits - 1) / pl.splits;
    const int t0 = min(s * tps, nt_all), t1 = min(t0 + tps, nt_all);
    const int32_t *bt = p.block_table + (size_t)b0 * p.max_blocks;  // the group's pages

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;  // fragment row / column pair

    // this thread's rows gq and gq + 8 of the warp's 16: group row r = (member, i, j)
    // -> row (b, i, hq) of q / out; -1 past the group's rows
    auto row_of = [&](int k) -> long long {
        const int r = chunk * CASCADE_ROWS + warp * 16 + gq + 8 * k;
        if (r >= rows_g) return -1;
        const int m = r / NG, rr = r - m * NG, i = rr / p.G, j = rr - i * p.G;
        return ((long long)(b0 + m) * p.N + i) * p.Hq + (long long)h * p.G + j;
    };

    // Q as m16n8k16 A fragments, straight from global memory (rows past the group: zeros)
    uint32_t qa[KS][4];
    {
        const long long r0 = row_of(0), r1 = row_of(1);
        const uint32_t *q0 = reinterpret_cast<const uint32_t *>(p.q) + (r0 < 0 ? 0 : r0) * (D / 2);
        const uint32_t *q1 = reinterpret_cast<const uint32_t *>(p.q) + (r1 < 0 ? 0 : r1) * (D / 2);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            qa[ks][0] = r0 >= 0 ? __ldg(q0 + ks * 8 + tq) : 0u;
            qa[ks][1] = r1 >= 0 ? __ldg(q1 + ks * 8 + tq) : 0u;
            qa[ks][2] = r0 >= 0 ? __ldg(q0 + ks * 8 + 4 + tq) : 0u;
            qa[ks][3] = r1 >= 0 ? __ldg(q1 + ks * 8 + 4 + tq) : 0u;
        }
    }

    // K and V of prefix tile tt into stage st; keys past the prefix and bad
    // pages are zero-filled (the former are masked out of the softmax as well)
    auto load_tile = [&](int tt, int st) {
        uint16_t *kd = Ks + st * TILE, *vd = Vs + st * TILE;
        constexpr int CPR = D / 8;  // 16-byte chunks per key
        for (int e = tid; e < CASCADE_KEYS * CPR; e += PF_THREADS) {
            const int key = e / CPR, c = e - key * CPR;
            const int kk = tt * CASCADE_KEYS + key;
            const int blk = kk < P ? __ldg(bt + kk / PAGE) : -1;
            const bool ok = blk >= 0 && blk < p.num_blocks;
            const size_t off = ok ? (((size_t)blk * p.Hkv + h) * PAGE + (kk % PAGE)) * D + c * 8 : 0;
            cp_async16(smem_u32(kd + key * LD + c * 8), p.k_pool + off, ok ? 16u : 0u);
            cp_async16(smem_u32(vd + key * LD + c * 8), p.v_pool + off, ok ? 16u : 0u);
        }
    };

    float o[D / 8][4];
#pragma unroll
    for (int dn = 0; dn < D / 8; ++dn) o[dn][0] = o[dn][1] = o[dn][2] = o[dn][3] = 0.f;
    float mrow[2] = {PF_M_NONE, PF_M_NONE}, lrow[2] = {0.f, 0.f};
    const float sc = p.scale_log2;

    if (t0 < t1) load_tile(t0, 0);
    cp_async_commit();
    for (int tt = t0; tt < t1; ++tt) {
        const int st = (tt - t0) & 1;
        if (tt + 1 < t1) load_tile(tt + 1, st ^ 1);  // that stage was released at the end of tt - 1
        cp_async_commit();
        cp_async_wait<1>();  // tile tt has landed (this thread's copies) ...
        __syncthreads();     // ... and every thread's
        const uint16_t *kt = Ks + st * TILE, *vt = Vs + st * TILE;

        // S = Q K^T: 16 rows x 64 keys per warp
        float sacc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
                // matrices: keys +0..7 / +8..15 (lane bit 4) x dims +0..7 / +8..15 (lane bit 3)
                const int mi = lane >> 3;
                const int key = np * 16 + (mi >> 1) * 8 + (lane & 7);
                const int dim = ks * 16 + (mi & 1) * 8;
                uint32_t k0, k1, k2, k3;
                ldsm_x4(smem_u32(kt + key * LD + dim), k0, k1, k2, k3);
                mma_16816(sacc[2 * np], qa[ks], k0, k1);
                mma_16816(sacc[2 * np + 1], qa[ks], k2, k3);
            }
        }
        const int kbase = tt * CASCADE_KEYS;
        if (kbase + CASCADE_KEYS > P) {  // ragged last tile
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (kbase + nt * 8 + 2 * tq + (c & 1) >= P) sacc[nt][c] = -INFINITY;
        }

        // online softmax (log2 domain); c = 0, 1: row gq; c = 2, 3: row gq + 8.
        // Every tile holds at least one prefix key, and every row sees all of them.
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            mx[0] = fmaxf(mx[0], fmaxf(sacc[nt][0], sacc[nt][1]));
            mx[1] = fmaxf(mx[1], fmaxf(sacc[nt][2], sacc[nt][3]));
        }
        float alpha[2];
        bool raised = false;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 1));
            mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 2));
            const float mn = fmaxf(mrow[k], mx[k] * sc);
            raised |= mn > mrow[k];
            alpha[k] = ex2_approx(mrow[k] - mn);  // first tile: 2^(M_NONE - mn) = 0; unchanged: 1
            mrow[k] = mn;
        }
        uint32_t pa[NT / 2][4];  // P as A fragments of the PV product
        float ls[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float p0 = ex2_approx(fmaf(sacc[nt][0], sc, -mrow[0]));
            const float p1 = ex2_approx(fmaf(sacc[nt][1], sc, -mrow[0]));
            const float p2 = ex2_approx(fmaf(sacc[nt][2], sc, -mrow[1]));
            const float p3 = ex2_approx(fmaf(sacc[nt][3], sc, -mrow[1]));
            ls[0] += p0 + p1;
            ls[1] += p2 + p3;
            pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(p0, p1);  // row gq, keys 2tq (+8 for odd nt)
            pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(p2, p3);  // row gq + 8
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) lrow[k] = fmaf(lrow[k], alpha[k], ls[k]);  // this thread's columns only
        if (__any_sync(0xffffffffu, raised)) {  // an unchanged maximum leaves O as it is (alpha = 1)
#pragma unroll
            for (int dn = 0; dn < D / 8; ++dn) {
                o[dn][0] *= alpha[0];
                o[dn][1] *= alpha[0];
                o[dn][2] *= alpha[1];
                o[dn][3] *= alpha[1];
            }
        }

        // O += P V: V tiles [key][dim] read transposed as B fragments
#pragma unroll
        for (int kb = 0; kb < NT / 2; ++kb) {
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                // matrices: keys +0..7 / +8..15 (lane bit 3) x dims +0..7 / +8..15 (lane bit 4)
                const int key = kb * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int dim = dp * 16 + (lane >> 4) * 8;
                uint32_t v0, v1, v2, v3;
                ldsm_x4_trans(smem_u32(vt + key * LD + dim), v0, v1, v2, v3);
                mma_16816(o[2 * dp], pa[kb], v0, v1);
                mma_16816(o[2 * dp + 1], pa[kb], v2, v3);
            }
        }
        __syncthreads();  // stage st may be refilled
    }
    cp_async_wait<0>();

    // partial of rows gq, gq + 8 for split s: O unnormalised, (m, l)
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        lrow[k] += __shfl_xor_sync(0xffffffffu, lrow[k], 1);
        lrow[k] += __shfl_xor_sync(0xffffffffu, lrow[k], 2);
    }
    const size_t pstride = (size_t)p.B * p.N * p.Hq;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const long long rk = row_of(k);
        if (rk < 0) continue;
        const size_t row = (size_t)s * pstride + (size_t)rk;
        float *dst = p.pp_o + row * D;
#pragma unroll
        for (int dn = 0; dn < D / 8; ++dn)
            *reinterpret_cast<float2 *>(dst + dn * 8 + 2 * tq) = make_float2(o[dn][2 * k], o[dn][2 * k + 1]);
        if (tq == 0) *reinterpret_cast<float2 *>(p.pp_ml + 2 * row) = make_float2(mrow[k], lrow[k]);
    }
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

template <int D>
constexpr size_t prefix_smem_bytes() {
    return (size_t)2 * 2 * CASCADE_KEYS * (D + 8) * sizeof(uint16_t);
}

}  // namespace

void cascade_plan(const sv_cascade_desc *cd, int N, int Hq, int Hkv, int num_sms, CascadePlan *pl) {
    memset(pl, 0, sizeof *pl);
    const int G = Hq / Hkv;
    pl->num_groups = cd->num_groups;
    int base = 0, max_tiles = 0;
    for (int g = 0; g <= cd->num_groups; ++g) pl->off[g] = cd->group_offsets[g];
    for (int g = 0; g < cd->num_groups; ++g) {
        pl->pre[g] = cd->prefix_lens[g];
        const int rows = (pl->off[g + 1] - pl->off[g]) * N * G;
        base += (rows + CASCADE_ROWS - 1) / CASCADE_ROWS * Hkv;
        max_tiles = max(max_tiles, (pl->pre[g] + CASCADE_KEYS - 1) / CASCADE_KEYS);
    }
    // The most prefix splits whose items still fit one wave of resident CTAs
    // (three per SM: shared memory and registers). A second, partial wave costs
    // more than the latency the extra warps hide: at 448 items for 444 slots the
    // pass ran longer than at 224. Every split also adds a partial per row.
    int S = base > 0 ? (PF_CTAS_PER_SM * num_sms) / base : 1;
    S = max(1, min(S, min(MAX_SPLITS, max(1, max_tiles))));
    pl->splits = S;
    int acc = 0;
    for (int g = 0; g < cd->num_groups; ++g) {
        pl->item0[g] = acc;
        const int rows = (pl->off[g + 1] - pl->off[g]) * N * G;
        acc += (rows + CASCADE_ROWS - 1) / CASCADE_ROWS * Hkv * S;
    }
    pl->item0[cd->num_groups] = acc;
    pl->items = acc;
}

CascadeWorkspace cascade_workspace(int B, int N, int Hq, int Hkv, int D, int max_blocks, int num_ctas,
                                   int splits) {
    CascadeWorkspace w;
    size_t off = 0;
    w.slots = off;
    off += align256(attention_workspace_bytes(B, N, Hq, Hkv, D, num_ctas));
    w.sfx_ctx = off;
    off += align256((size_t)B * sizeof(int32_t));
    w.pflag = off;
    off += align256((size_t)B * sizeof(int32_t));
    w.sfx_table = off;
    off += align256((size_t)B * max_blocks * sizeof(int32_t));
    const size_t rows = (size_t)splits * B * N * Hq;
    w.pp_o = off;
    off += align256(rows * D * sizeof(float));
    w.pp_ml = off;
    off += align256(rows * 2 * sizeof(float));
    w.total = off;
    return w;
}

cudaError_t launch_cascade(const AttnParams &p, const CascadePlan &plan, cudaStream_t stream) {
    const CascadeWorkspace w = cascade_workspace(p.B, p.N, p.Hq, p.Hkv, p.D, p.max_blocks, p.num_ctas, plan.splits);
    char *base = reinterpret_cast<char *>(p.ws_partial);
    int32_t *sfx_ctx = reinterpret_cast<int32_t *>(base + w.sfx_ctx);
    int32_t *pflag = reinterpret_cast<int32_t *>(base + w.pflag);
    int32_t *sfx_table = reinterpret_cast<int32_t *>(base + w.sfx_table);
    float *pp_o = reinterpret_cast<float *>(base + w.pp_o);
    float *pp_ml = reinterpret_cast<float *>(base + w.pp_ml);

    PrepParams pp;
    pp.block_table = p.block_table;
    pp.ctx_lens = p.ctx_lens;
    pp.sfx_ctx = sfx_ctx;
    pp.sfx_table = sfx_table;
    pp.pflag = pflag;
    pp.B = p.B;
    pp.N = p.N;
    pp.max_blocks = p.max_blocks;
    pp.num_blocks = p.num_blocks;
    pp.plan = plan;
    cascade_prep_kernel<<<p.B, PREP_THREADS, 0, stream>>>(pp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    PrefixParams fp;
    fp.q = p.q;
    fp.k_pool = p.k_pool;
    fp.v_pool = p.v_pool;
    fp.block_table = p.block_table;
    fp.pp_o = pp_o;
    fp.pp_ml = pp_ml;
    fp.B = p.B;
    fp.N = p.N;
    fp.Hq = p.Hq;
    fp.Hkv = p.Hkv;
    fp.G = p.G;
    fp.max_blocks = p.max_blocks;
    fp.num_blocks = p.num_blocks;
    fp.scale_log2 = p.scale_log2;
    fp.plan = plan;
    if (p.D == 128) {
        constexpr size_t smem = prefix_smem_bytes<128>();
        e = cudaFuncSetAttribute(cascade_prefix_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        cascade_prefix_kernel<128><<<plan.items, PF_THREADS, smem, stream>>>(fp);
    } else {
        constexpr size_t smem = prefix_smem_bytes<64>();
        e = cudaFuncSetAttribute(cascade_prefix_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        cascade_prefix_kernel<64><<<plan.items, PF_THREADS, smem, stream>>>(fp);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    AttnParams a = p;
    a.block_table = sfx_table;
    a.ctx_lens = sfx_ctx;
    a.ws_partial = reinterpret_cast<float *>(base + w.slots);
    a.pp_o = pp_o;
    a.pp_ml = pp_ml;
    a.pflag = pflag;
    a.pp_splits = plan.splits;
    return launch_attention(a, stream);
}

}  // namespace sv
