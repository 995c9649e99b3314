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
//   cascade_prefix_kernel  one CTA per (group, KV head, 128 group rows, prefix
//                          split): tcgen05 products over 128-key tiles of the
//                          shared pages, an unnormalised partial (O, running
//                          max, row sum) per row and split; its prep warp
//                          writes each member's suffix length and suffix block
//                          table (its own pages after the prefix) and flags
//                          bad block ids among the prefix pages;
//   launch_attention       the split-context tcgen05 kernel over every
//                          member's suffix (own pages, draft rows and masks);
//                          a unit one CTA covers whole merges the rows' prefix
//                          partials before it writes the output, a split unit
//                          leaves slots that the combine kernel merges with
//                          the prefix partials.
#include <string.h>

#include "sv_internal.h"
#include "sv_tc.cuh"

namespace sv {
namespace {

using namespace tc;

constexpr int PF_ROWS = CASCADE_ROWS;  // group rows per CTA: the MMA M dimension, one TMEM lane each
constexpr int PF_KEYS = CASCADE_KEYS;  // keys per tile (8 pages): the N of S = Q K^T, the K of O += P V
static_assert(PF_ROWS == 128 && PF_KEYS == 128, "the prefix pass is written for 128 x 128 tiles");
constexpr int PF_WARP_LOAD = 0;   // TMA producer (K and V)
constexpr int PF_WARP_MMA = 1;    // TMEM allocator and MMA issuer
constexpr int PF_WARP_PREP = 2;   // members' suffix tables, lengths and prefix flags
constexpr int PF_WARP_SM0 = 3;    // softmax warps 3..6: thread = row (TMEM lane quadrant = warp % 4)
constexpr int PF_THREADS = 32 * (PF_WARP_SM0 + 4);
constexpr int MAX_SPLITS = 8;
constexpr uint32_t PF_ATOM = 16384;  // 128 rows x 128 bytes: one 128B-swizzle column of an operand
constexpr float PF_M_NONE = -3.402823466e38f;  // running max of a row that has seen no key
constexpr float PF_RESCALE_LOG2 = 8.f;         // O is rescaled only when a row max rises by more
constexpr uint64_t PF_DRAIN_NS = 2000000000ull;

struct PrefixParams {
    CUtensorMap tm_k, tm_v;
    const uint16_t *q;                // bf16 bits [B][N][Hq][D]
    const int32_t *block_table, *ctx_lens;
    float *pp_o, *pp_ml;
    int32_t *sfx_ctx, *sfx_table, *pflag;
    int B, N, Hq, Hkv, G, max_blocks, num_blocks;
    float scale_log2;
    uint64_t wait_limit_ns;
    int NK, NV, NP;
    CascadePlan plan;
};

struct PfLayout {
    uint32_t tile, off_q, off_k, off_v, off_p, off_bar, off_misc, total;
};

__host__ __device__ inline PfLayout pf_layout(int D, int NK, int NV, int NP) {
    PfLayout L;
    L.tile = (uint32_t)(D / 64) * PF_ATOM;  // 128 keys x D of K or V; also Q's 128 rows x D
    L.off_q = 0;
    L.off_k = L.off_q + L.tile;
    L.off_v = L.off_k + NK * L.tile;
    L.off_p = L.off_v + NV * L.tile;                    // P: 128 rows x 128 keys, two atoms
    L.off_bar = L.off_p + NP * 2 * PF_ATOM;
    const int nbar = 2 * NK + 2 * NV + 2 * 2 /*s*/ + 2 * NP /*p*/ + 2 /*o*/ + 1 /*q*/ + 1 /*done*/;
    L.off_misc = L.off_bar + 8u * nbar;
    L.total = L.off_misc + 16u;
    return L;
}

// Largest g in [0, n) with x[g] <= v, for nondecreasing x with x[0] <= v.
SV_DEV int upper_index(const int *x, int n, int v) {
    int lo = 0, hi = n;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (x[mid] <= v) lo = mid; else hi = mid;
    }
    return lo;
}

// Byte offset of 16-byte chunk c (8 bf16) of row r in a K-major operand tile of
// 128 rows: 64-element columns of PF_ATOM bytes, rows of 128 bytes in groups of
// eight, chunks xor-swizzled by the row (the 128-byte swizzle TMA and the MMA use).
SV_DEV uint32_t kmajor_off(int r, int c) {
    return (uint32_t)(c >> 3) * PF_ATOM + (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u +
           ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

// One CTA per (group, KV head, 128 group rows, prefix split). Rows (member, i, j)
// of every member of the group share the group's prefix pages, so each tile of
// those pages is read once for 128 rows: S = Q K^T (M = 128 rows, N = 128 keys)
// and O += P V (M = 128 rows, N = D) on tcgen05 with fp32 accumulators in TMEM,
// K and V tiles by TMA (a page id outside the pool, or a page past the prefix,
// becomes a coordinate past the pool: zeros), Q and P written into the
// swizzled operand layout by the softmax threads. The result per row and split
// is an unnormalised partial (O, running max m in the log2 domain, row sum l).
// The prep warp meanwhile writes each member's suffix length and table and the
// bad-prefix-page flags for the split-context pass that follows.
template <int D>
__global__ void __launch_bounds__(PF_THREADS, 1) cascade_prefix_kernel(const __grid_constant__ PrefixParams p) {
    constexpr int nDA = D / 64;
    const int NK = p.NK, NV = p.NV, NP = p.NP;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const PfLayout L = pf_layout(D, NK, NV, NP);
    uint64_t *bar = reinterpret_cast<uint64_t *>(base + L.off_bar);
    uint64_t *k_full = bar, *k_empty = bar + NK;
    uint64_t *v_full = bar + 2 * NK, *v_empty = v_full + NV;
    uint64_t *s_full = v_empty + NV, *s_empty = s_full + 2;
    uint64_t *p_full = s_empty + 2, *p_empty = p_full + NP;
    uint64_t *o_full = p_empty + NP;  // [2] by tile parity: that tile's P V has completed
    uint64_t *q_ready = o_full + 2, *done_bar = q_ready + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + L.off_misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + L.off_misc + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // ---- work item -> (group, KV head, split, row tile) ----
    const CascadePlan &pl = p.plan;
    const int it = blockIdx.x;
    const int g = upper_index(pl.item0, pl.num_groups, it);
    const int b0 = pl.off[g];
    const int NG = p.N * p.G;
    const int rows_g = (pl.off[g + 1] - b0) * NG;
    const int tiles_g = (rows_g + PF_ROWS - 1) / PF_ROWS;
    int rem = it - pl.item0[g];
    const int rt = rem % tiles_g;
    rem /= tiles_g;
    const int s = rem % pl.splits, h = rem / pl.splits;
    const int P = pl.pre[g];
    const int nt_all = (P + PF_KEYS - 1) / PF_KEYS;
    const int tps = (nt_all + pl.splits - 1) / pl.splits;
    const int t0 = min(s * tps, nt_all), t1 = min(t0 + tps, nt_all);
    const int ntiles = t1 - t0;

    if (tid == 0) {
        for (int i = 0; i < NK; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
        for (int i = 0; i < NV; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 4);
            mbar_init(&o_full[i], 1);
        }
        for (int i = 0; i < NP; ++i) { mbar_init(&p_full[i], 4); mbar_init(&p_empty[i], 1); }
        mbar_init(q_ready, 4);
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == PF_WARP_MMA) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (warp == PF_WARP_LOAD && lane == 0) {
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // shared memory, TMEM and parameters only so far: with a programmatic launch
    // this overlaps the previous kernel's tail
    griddep_wait();
    griddep_launch_dependents();

    if (warp == PF_WARP_LOAD) {
        // ------------------------- TMA producer -------------------------
        if (lane == 0) {
            const int32_t *bt = p.block_table + (size_t)b0 * p.max_blocks;  // the group's pages
            int issued_k = 0, issued_v = 0;
            for (int lt = 0; lt < ntiles; ++lt) {
                const int tile = t0 + lt;
                int blks[PF_KEYS / PAGE];
#pragma unroll
                for (int pg = 0; pg < PF_KEYS / PAGE; ++pg) {
                    const int page = tile * (PF_KEYS / PAGE) + pg;
                    const int blk = page * PAGE < P ? __ldg(bt + page) : -1;
                    blks[pg] = (blk >= 0 && blk < p.num_blocks) ? blk : p.num_blocks;  // past the pool: zeros
                }
                const int sk = lt % NK;
                if (!mbar_wait(&k_empty[sk], ((lt / NK) & 1) ^ 1, abort_flag, p.wait_limit_ns)) break;
                mbar_arrive_expect_tx(&k_full[sk], L.tile);
                uint8_t *kd = base + L.off_k + sk * L.tile;
#pragma unroll
                for (int pg = 0; pg < PF_KEYS / PAGE; ++pg)
                    for (int a = 0; a < nDA; ++a)
                        tma_load_4d(kd + a * PF_ATOM + pg * 2048, &p.tm_k, &k_full[sk], a * 64, 0, h, blks[pg]);
                issued_k = lt + 1;
                const int sv = lt % NV;
                if (!mbar_wait(&v_empty[sv], ((lt / NV) & 1) ^ 1, abort_flag, p.wait_limit_ns)) break;
                mbar_arrive_expect_tx(&v_full[sv], L.tile);
                uint8_t *vd = base + L.off_v + sv * L.tile;
#pragma unroll
                for (int pg = 0; pg < PF_KEYS / PAGE; ++pg)
                    for (int a = 0; a < nDA; ++a)
                        tma_load_4d(vd + a * PF_ATOM + pg * 2048, &p.tm_v, &v_full[sv], a * 64, 0, h, blks[pg]);
                issued_v = lt + 1;
            }
            if (*abort_flag) {
                // this CTA's own copies land before it can exit
                for (int lt = max(0, issued_k - NK); lt < issued_k; ++lt)
                    mbar_wait_time(&k_full[lt % NK], (lt / NK) & 1, PF_DRAIN_NS);
                for (int lt = max(0, issued_v - NV); lt < issued_v; ++lt)
                    mbar_wait_time(&v_full[lt % NV], (lt / NV) & 1, PF_DRAIN_NS);
            }
        }
    } else if (warp == PF_WARP_MMA) {
        // -------------------------- MMA issuer ---------------------------
        if (lane == 0 && ntiles > 0) {
            constexpr uint32_t ids = idesc_bf16(128, PF_KEYS, false, false);  // Q, K both K-major
            constexpr uint32_t idp = idesc_bf16(128, D, false, true);         // P K-major, V dims-major
            const uint32_t qa = smem_u32(base + L.off_q);
            bool ok = mbar_wait(q_ready, 0, abort_flag, p.wait_limit_ns);
            int nq = 0, np = 0;
            uint32_t idle = 0;
            uint64_t idle_since = 0;
            while (ok && np < ntiles) {
                bool progressed = false;
                if (nq < ntiles) {
                    const int sk = nq % NK, sb = nq & 1;
                    if (mbar_test(&k_full[sk], (nq / NK) & 1) && mbar_test(&s_empty[sb], ((nq >> 1) & 1) ^ 1)) {
                        tc_fence_after();
                        const uint32_t ka = smem_u32(base + L.off_k + sk * L.tile);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t ad = sw128_desc(qa + (kk >> 2) * PF_ATOM + (kk & 3) * 32, 16, 1024);
                            const uint64_t bd = sw128_desc(ka + (kk >> 2) * PF_ATOM + (kk & 3) * 32, 16, 1024);
                            mma_bf16_ss(tmem + sb * PF_KEYS, ad, bd, ids, kk > 0);
                        }
                        mma_commit(&s_full[sb]);
                        mma_commit(&k_empty[sk]);
                        ++nq;
                        progressed = true;
                    }
                }
                if (np < nq) {
                    const int sv = np % NV, pb = np % NP;
                    if (mbar_test(&p_full[pb], (np / NP) & 1) && mbar_test(&v_full[sv], (np / NV) & 1)) {
                        tc_fence_after();
                        const uint32_t va = smem_u32(base + L.off_v + sv * L.tile);
                        const uint32_t pa = smem_u32(base + L.off_p + pb * 2 * PF_ATOM);
#pragma unroll
                        for (int kk = 0; kk < PF_KEYS / 16; ++kk) {
                            const uint64_t ad = sw128_desc(pa + (kk >> 2) * PF_ATOM + (kk & 3) * 32, 16, 1024);
                            const uint64_t bd = sw128_desc(va + kk * 2048, PF_ATOM, 1024);
                            mma_bf16_ss(tmem + 2 * PF_KEYS, ad, bd, idp, (np > 0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(&o_full[np & 1]);
                        mma_commit(&p_empty[pb]);
                        mma_commit(&v_empty[sv]);
                        ++np;
                        progressed = true;
                    }
                }
                if (progressed) {
                    idle = 0;
                } else if (++idle > 8 && (__nanosleep(20), (idle & 63) == 0)) {
                    if (*abort_flag) break;
                    const uint64_t now = globaltimer_ns();
                    if (idle == 64) idle_since = now;
                    else if (now - idle_since > p.wait_limit_ns) { *abort_flag = 1; break; }
                }
            }
            mma_commit(done_bar);  // every MMA of this CTA has finished before TMEM is freed
            mbar_wait_time(done_bar, 0, PF_DRAIN_NS);
        }
    } else if (warp == PF_WARP_PREP) {
        // -------- members' suffix lengths and tables, prefix page flags --------
        // sequence b is handled by CTA b mod gridDim.x; a member whose context
        // is invalid or shorter than its group's prefix plus N gets length -1
        // (the attention kernel flags SV_FLAG_BAD_CONTEXT and writes zeros)
        for (int b = blockIdx.x; b < p.B; b += gridDim.x) {
            const int gb = upper_index(pl.off, pl.num_groups, b);
            const int Pb = pl.pre[gb], first = pl.off[gb];
            const int C = __ldg(p.ctx_lens + b);
            const bool okc = C >= p.N && C <= p.max_blocks * PAGE && Pb <= C - p.N;
            if (!okc) {
                if (lane == 0) p.sfx_ctx[b] = -1;
                continue;
            }
            const int npg = Pb / PAGE, ns = (C - Pb + PAGE - 1) / PAGE;
            const int32_t *own = p.block_table + (size_t)b * p.max_blocks + npg;
            int32_t *dst = p.sfx_table + (size_t)b * p.max_blocks;
            for (int j = lane; j < ns; j += 32) dst[j] = __ldg(own + j);
            const int32_t *shared_pages = p.block_table + (size_t)first * p.max_blocks;
            int bad = 0;
            for (int j = lane; j < npg; j += 32) {
                const int blk = __ldg(shared_pages + j);
                bad |= blk < 0 || blk >= p.num_blocks;
            }
            bad = __any_sync(0xffffffffu, bad);
            if (lane == 0) {
                p.sfx_ctx[b] = C - Pb;
                if (bad) atomicOr(p.pflag + b, SV_FLAG_BAD_BLOCK);
            }
        }
    } else {
        // ------------------- softmax: one thread per row -------------------
        const int quad = warp & 3;              // TMEM lane quadrant of this warp
        const int ell = quad * 32 + lane;       // row of the tile = TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const int r = rt * PF_ROWS + ell;       // group row (member, i, j)
        long long prow = -1;                    // row (b, i, hq) of q / out
        if (r < rows_g) {
            const int m = r / NG, rr = r - m * NG, i = rr / p.G, j = rr - i * p.G;
            prow = ((long long)(b0 + m) * p.N + i) * p.Hq + (long long)h * p.G + j;
        }
        auto warp_arrive = [&](uint64_t *b) {
            __syncwarp();
            if (lane == 0) mbar_arrive(b);
        };
        auto wait_w = [&](uint64_t *b, uint32_t parity) -> bool {
            const bool ok = mbar_test(b, parity) || mbar_wait(b, parity, abort_flag, p.wait_limit_ns);
            return __all_sync(0xffffffffu, ok);
        };
        {   // Q row into the swizzled K-major operand tile (zeros past the group's rows)
            const uint4 *src = reinterpret_cast<const uint4 *>(p.q + (prow < 0 ? 0 : prow) * D);
            uint8_t *qt = base + L.off_q;
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const uint4 v = prow >= 0 ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(qt + kmajor_off(ell, c)) = v;
            }
            fence_proxy_async_smem();
            warp_arrive(q_ready);
        }
        const float sc = p.scale_log2;
        float m_run = PF_M_NONE, l_run = 0.f;
        bool ok = true;
        for (int lt = 0; lt < ntiles && ok; ++lt) {
            const int sb = lt & 1, pb = lt % NP;
            const int valid = P - (t0 + lt) * PF_KEYS;  // keys of this tile inside the prefix
            if (!(ok = wait_w(&s_full[sb], (lt >> 1) & 1))) break;
            tc_fence_after();
            const uint32_t sa = lane_base + sb * PF_KEYS;
            float mx = -INFINITY;
#pragma unroll 1
            for (int c0 = 0; c0 < PF_KEYS; c0 += 32) {
                float v[32];
                tmem_ld32(sa + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) mx = fmaxf(mx, c0 + c < valid ? v[c] : -INFINITY);
            }
            // the running max is raised on a row's first tile, or when a score
            // beats it by more than 2^8; otherwise the tile folds in as it is
            const float cand = mx * sc;
            const bool raise = m_run == PF_M_NONE || cand > m_run + PF_RESCALE_LOG2;
            const float m_new = raise ? fmaxf(m_run, cand) : m_run;
            const float alpha = ex2_approx(m_run - m_new);  // first tile: 0; unchanged: 1
            l_run *= alpha;
            if (lt > 0 && __any_sync(0xffffffffu, raise)) {
                // O (this row, every dim) scaled once the previous tile's P V has landed
                if (!(ok = wait_w(&o_full[(lt - 1) & 1], ((lt - 1) >> 1) & 1))) break;
                tc_fence_after();
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 16) {
                    float o[16];
                    tmem_ld16(lane_base + 2 * PF_KEYS + c0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 16; ++c) o[c] *= alpha;
                    tmem_st16(lane_base + 2 * PF_KEYS + c0, o);
                }
                tmem_wait_st();
            }
            m_run = m_new;
            if (!(ok = wait_w(&p_empty[pb], ((lt / NP) & 1) ^ 1))) break;
            uint8_t *pt = base + L.off_p + pb * 2 * PF_ATOM;
#pragma unroll 1
            for (int c0 = 0; c0 < PF_KEYS; c0 += 32) {
                float v[32];
                tmem_ld32(sa + c0, v);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float p0 = c0 + c < valid ? ex2_approx(fmaf(v[c], sc, -m_run)) : 0.f;
                    const float p1 = c0 + c + 1 < valid ? ex2_approx(fmaf(v[c + 1], sc, -m_run)) : 0.f;
                    l_run += p0 + p1;
                    const __nv_bfloat162 hv = __floats2bfloat162_rn(p0, p1);
                    pk[c >> 1] = *reinterpret_cast<const uint32_t *>(&hv);
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    *reinterpret_cast<uint4 *>(pt + kmajor_off(ell, (c0 >> 3) + q4)) =
                        make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
            }
            tc_fence_before();
            warp_arrive(&s_empty[sb]);
            fence_proxy_async_smem();
            warp_arrive(&p_full[pb]);
        }
        // ---- partial of this row and split: O unnormalised, (m, l) ----
        const size_t pstride = (size_t)p.B * p.N * p.Hq;
        float *dst = prow >= 0 ? p.pp_o + ((size_t)s * pstride + (size_t)prow) * D : nullptr;
        if (ok && ntiles > 0) ok = wait_w(&o_full[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1);
        if (ok && ntiles > 0) {
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 16) {
                float o[16];
                tmem_ld16(lane_base + 2 * PF_KEYS + c0, o);
                tmem_wait_ld();
                if (dst)
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4)
                        *reinterpret_cast<float4 *>(dst + c0 + 4 * c4) =
                            make_float4(o[4 * c4], o[4 * c4 + 1], o[4 * c4 + 2], o[4 * c4 + 3]);
            }
        } else if (dst) {
            for (int c = 0; c < D; c += 4) *reinterpret_cast<float4 *>(dst + c) = make_float4(0.f, 0.f, 0.f, 0.f);
            m_run = PF_M_NONE;
            l_run = 0.f;
        }
        if (dst) *reinterpret_cast<float2 *>(p.pp_ml + 2 * ((size_t)s * pstride + (size_t)prow)) = make_float2(m_run, l_run);
    }

    // ----------------------------- teardown -------------------------------
    tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid < 32)
        for (int b = lane; b < p.B; b += 32) atomicOr(p.pflag + b, SV_FLAG_TIMEOUT);
    if (warp == PF_WARP_MMA) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

constexpr int PF_SMEM_LIMIT = 227 * 1024;

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
    // One CTA per SM (shared memory and TMEM): the most prefix splits whose
    // items still fit one wave. Every split adds a partial per row.
    int S = base > 0 ? num_sms / base : 1;
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

template <int D>
static cudaError_t launch_prefix(PrefixParams &fp, int items, cudaStream_t stream) {
    static const int choices[][3] = {{2, 3, 2}, {3, 2, 2}, {2, 2, 2}, {2, 2, 1}, {1, 2, 1}};
    int k = 0;
    PfLayout L;
    for (; k < 5; ++k) {
        L = pf_layout(D, choices[k][0], choices[k][1], choices[k][2]);
        if (L.total + 1024 <= (uint32_t)PF_SMEM_LIMIT) break;
    }
    if (k == 5) return cudaErrorInvalidConfiguration;
    fp.NK = choices[k][0];
    fp.NV = choices[k][1];
    fp.NP = choices[k][2];
    const size_t smem = L.total + 1024;
    auto kfn = cascade_prefix_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)items);
    cfg.blockDim = dim3(PF_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kfn, fp);
}

cudaError_t launch_cascade(const AttnParams &p, const CascadePlan &plan, cudaStream_t stream) {
    const CascadeWorkspace w = cascade_workspace(p.B, p.N, p.Hq, p.Hkv, p.D, p.max_blocks, p.num_ctas, plan.splits);
    char *base = reinterpret_cast<char *>(p.ws_partial);
    int32_t *sfx_ctx = reinterpret_cast<int32_t *>(base + w.sfx_ctx);
    int32_t *pflag = reinterpret_cast<int32_t *>(base + w.pflag);
    int32_t *sfx_table = reinterpret_cast<int32_t *>(base + w.sfx_table);
    float *pp_o = reinterpret_cast<float *>(base + w.pp_o);
    float *pp_ml = reinterpret_cast<float *>(base + w.pp_ml);

    // prefix flags are ORed in by the prefix kernel's CTAs
    cudaError_t e = cudaMemsetAsync(pflag, 0, (size_t)p.B * sizeof(int32_t), stream);
    if (e != cudaSuccess) return e;

    PrefixParams fp;
    memset(&fp, 0, sizeof fp);
    if (!encode_pool_map(&fp.tm_k, p.k_pool, p.num_blocks, p.Hkv, p.D) ||
        !encode_pool_map(&fp.tm_v, p.v_pool, p.num_blocks, p.Hkv, p.D))
        return cudaErrorInvalidValue;
    fp.q = p.q;
    fp.block_table = p.block_table;
    fp.ctx_lens = p.ctx_lens;
    fp.pp_o = pp_o;
    fp.pp_ml = pp_ml;
    fp.sfx_ctx = sfx_ctx;
    fp.sfx_table = sfx_table;
    fp.pflag = pflag;
    fp.B = p.B;
    fp.N = p.N;
    fp.Hq = p.Hq;
    fp.Hkv = p.Hkv;
    fp.G = p.G;
    fp.max_blocks = p.max_blocks;
    fp.num_blocks = p.num_blocks;
    fp.scale_log2 = p.scale_log2;
    fp.wait_limit_ns = p.wait_limit_ns;
    fp.plan = plan;
    e = p.D == 128 ? launch_prefix<128>(fp, plan.items, stream) : launch_prefix<64>(fp, plan.items, stream);
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
