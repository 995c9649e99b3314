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
//                          and flags bad block ids among the group's prefix
//                          pages;
//   launch_attention       the split-context tcgen05 kernel over every
//                          member's suffix (own pages, draft rows and masks),
//                          every unit leaving its partial in a workspace slot;
//   cascade_prefix_kernel  one CTA per (group, KV head, 128 group rows):
//                          tcgen05 products over 128-key tiles of the shared
//                          pages; its epilogue merges each row's prefix partial
//                          (in TMEM) with the row's suffix slots and writes the
//                          output, so no combine kernel runs.
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
constexpr int PF_WARP_SM0 = 2;    // softmax warps 2..9: quadrant warp % 4 (its TMEM lanes), half (warp - 2) / 4
constexpr int PF_SM_WARPS = 8;
constexpr int PF_THREADS = 32 * (PF_WARP_SM0 + PF_SM_WARPS);
constexpr int PREP_THREADS = 128;
constexpr uint32_t PF_ATOM = 16384;  // 128 rows x 128 bytes: one 128B-swizzle column of an operand
constexpr uint32_t COL_S = 0;        // TMEM: S double buffer (2 x 128 columns), O (D columns),
constexpr uint32_t COL_O = 2 * PF_KEYS;  // then exchange columns of the two warps sharing lanes
constexpr uint32_t COL_X = COL_O + 128;
constexpr float PF_M_NONE = -3.402823466e38f;  // running max of a row that has seen no key
constexpr float PF_RESCALE_LOG2 = 8.f;         // O is rescaled only when a row max rises by more
constexpr uint64_t PF_DRAIN_NS = 2000000000ull;

struct PrepParams {
    const int32_t *block_table, *ctx_lens;
    int32_t *sfx_ctx, *sfx_table, *pflag;
    int B, N, max_blocks, num_blocks;
    CascadePlan plan;
};

struct PrefixParams {
    CUtensorMap tm_k, tm_v;
    AttnParams a;                     // the suffix call: slots, suffix lengths, shapes, status
    const int32_t *block_table;       // the caller's table (the group's first member's prefix pages)
    const int32_t *pflag;
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
    const int nbar = 2 * NK + 2 * NV + 2 * 2 /*s*/ + 2 * NP /*p*/ + 2 /*o*/ + 1 /*q*/ + 1 /*done*/ + 4 /*pair*/;
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

// Split-context tiles of sequence b in the suffix call (the attention kernel's rule).
SV_DEV int suffix_tiles(const AttnParams &a, int b) {
    const int C = __ldcg(a.ctx_lens + b);
    return (C >= a.N && C <= a.max_blocks * PAGE) ? (C + TILE_KEYS - 1) / TILE_KEYS : 0;
}
// Its schedule positions (the tiles plus UNIT_COST per unit).
SV_DEV int suffix_slots(const AttnParams &a, int b) {
    const int t = suffix_tiles(a, b);
    return t > 0 ? t + UNIT_COST : 0;
}

__global__ void __launch_bounds__(PREP_THREADS) cascade_prep_kernel(const __grid_constant__ PrepParams p) {
    griddep_wait();
    griddep_launch_dependents();
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

// One CTA per (group, KV head, 128 group rows). Rows (member, i, j) of every
// member of the group share the group's prefix pages, so each tile of those
// pages is read once for 128 rows: S = Q K^T (M = 128 rows, N = 128 keys) and
// O += P V (M = 128 rows, N = D) on tcgen05 with fp32 accumulators in TMEM, K
// and V tiles by TMA (a page id outside the pool, or a page past the prefix,
// becomes a coordinate past the pool: zeros), Q and P written into the
// swizzled operand layout by the softmax threads. Two softmax warps share each
// TMEM lane quadrant, one per half of the keys (and of the head dims of O);
// they exchange row maxima and sums through TMEM columns, ordered by an
// mbarrier per pair. The epilogue merges each row's prefix partial with the
// row's suffix slots left by the split-context pass (log-sum-exp) and writes
// the row's output.
template <int D>
__global__ void __launch_bounds__(PF_THREADS, 1) cascade_prefix_kernel(const __grid_constant__ PrefixParams p) {
    constexpr int nDA = D / 64;
    constexpr int HD = D / 2;  // head dims of O per half
    const AttnParams &a = p.a;
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
    uint64_t *pair_bar = done_bar + 1;  // [4] by lane quadrant: the two warps of a quadrant
    // A two-slot K ring's slot of tile t is its S buffer t & 1, freed by the QK
    // product s_full[t & 1] marks; two P buffers are freed by tile t's P V, which
    // o_full[t & 1] marks: one commit fewer per tile each.
    uint64_t *k_free = NK == 2 ? s_full : k_empty;
    uint64_t *p_free = NP == 2 ? o_full : p_empty;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + L.off_misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + L.off_misc + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // ---- work item -> (group, KV head, row tile) ----
    const CascadePlan &pl = p.plan;
    const int it = blockIdx.x;
    const int g = upper_index(pl.item0, pl.num_groups, it);
    const int b0 = pl.off[g];
    const int G = a.G;
    const int NG = a.N * G;
    const int rows_g = (pl.off[g + 1] - b0) * NG;
    const int tiles_g = (rows_g + PF_ROWS - 1) / PF_ROWS;
    const int local = it - pl.item0[g];
    const int rt = local % tiles_g, h = local / tiles_g;
    const int P = pl.pre[g];
    const int ntiles = (P + PF_KEYS - 1) / PF_KEYS;

    if (tid == 0) {
        for (int i = 0; i < NK; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
        for (int i = 0; i < NV; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], PF_SM_WARPS);
            mbar_init(&o_full[i], 1);
        }
        for (int i = 0; i < NP; ++i) { mbar_init(&p_full[i], PF_SM_WARPS); mbar_init(&p_empty[i], 1); }
        mbar_init(q_ready, PF_SM_WARPS);
        mbar_init(done_bar, 1);
        for (int i = 0; i < 4; ++i) mbar_init(&pair_bar[i], 2);
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
    // Launched programmatically after the split-context kernel, which issues its
    // trigger only after its own wait on everything before the call: q, the KV
    // pools and the block table are complete when this kernel starts, so the
    // prefix products run while the split-context kernel's last CTAs finish.
    // Its outputs (the slots, the status) and the prep kernel's are read only
    // after griddep_wait.
    griddep_launch_dependents();

    if (warp == PF_WARP_LOAD) {
        // ------------------------- TMA producer -------------------------
        if (lane == 0) {
            const int32_t *bt = p.block_table + (size_t)b0 * a.max_blocks;  // the group's pages
            int issued_k = 0, issued_v = 0;
            int sk = 0, sv = 0;  // ring slots of tile lt and their phases (no runtime division)
            uint32_t kph = 0, vph = 0;
            for (int lt = 0; lt < ntiles; ++lt) {
                int blks[PF_KEYS / PAGE];
#pragma unroll
                for (int pg = 0; pg < PF_KEYS / PAGE; ++pg) {
                    const int page = lt * (PF_KEYS / PAGE) + pg;
                    const int blk = page * PAGE < P ? __ldg(bt + page) : -1;
                    blks[pg] = (blk >= 0 && blk < a.num_blocks) ? blk : a.num_blocks;  // past the pool: zeros
                }
                if (!mbar_wait(&k_free[sk], kph ^ 1u, abort_flag, a.wait_limit_ns)) break;
                mbar_arrive_expect_tx(&k_full[sk], L.tile);
                uint8_t *kd = base + L.off_k + sk * L.tile;
#pragma unroll
                for (int pg = 0; pg < PF_KEYS / PAGE; ++pg)
                    for (int q = 0; q < nDA; ++q)
                        tma_load_4d(kd + q * PF_ATOM + pg * 2048, &p.tm_k, &k_full[sk], q * 64, 0, h, blks[pg]);
                issued_k = lt + 1;
                if (++sk == NK) { sk = 0; kph ^= 1u; }
                if (!mbar_wait(&v_empty[sv], vph ^ 1u, abort_flag, a.wait_limit_ns)) break;
                mbar_arrive_expect_tx(&v_full[sv], L.tile);
                uint8_t *vd = base + L.off_v + sv * L.tile;
#pragma unroll
                for (int pg = 0; pg < PF_KEYS / PAGE; ++pg)
                    for (int q = 0; q < nDA; ++q)
                        tma_load_4d(vd + q * PF_ATOM + pg * 2048, &p.tm_v, &v_full[sv], q * 64, 0, h, blks[pg]);
                issued_v = lt + 1;
                if (++sv == NV) { sv = 0; vph ^= 1u; }
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
            // operand descriptors of the buffers; a product adds its stage's offset
            // in 16-byte units (shared addresses stay below 2^18 bytes, so the
            // 14-bit address field does not carry)
            const uint64_t qdesc = sw128_desc(smem_u32(base + L.off_q), 16, 1024);
            const uint64_t kdesc = sw128_desc(smem_u32(base + L.off_k), 16, 1024);
            const uint64_t pdesc = sw128_desc(smem_u32(base + L.off_p), 16, 1024);
            const uint64_t vdesc = sw128_desc(smem_u32(base + L.off_v), PF_ATOM, 1024);
            bool ok = mbar_wait(q_ready, 0, abort_flag, a.wait_limit_ns);
            int nq = 0, np = 0;
            int ks = 0, vs = 0, ps = 0;  // ring slots of tiles nq (K) and np (V, P) and their phases
            uint32_t kph = 0, vph = 0, pph = 0;
            uint32_t idle = 0;
            uint64_t idle_since = 0;
            while (ok && np < ntiles) {
                bool progressed = false;
                if (nq < ntiles) {
                    const int sk = ks, sb = nq & 1;
                    if (mbar_test(&k_full[sk], kph) && mbar_test(&s_empty[sb], ((nq >> 1) & 1) ^ 1)) {
                        tc_fence_after();
                        const uint64_t ka = kdesc + ((sk * L.tile) >> 4);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t off = ((kk >> 2) * PF_ATOM + (kk & 3) * 32) >> 4;
                            mma_bf16_ss(tmem + COL_S + sb * PF_KEYS, qdesc + off, ka + off, ids, kk > 0);
                        }
                        mma_commit(&s_full[sb]);
                        if (NK != 2) mma_commit(&k_empty[sk]);
                        if (++ks == NK) { ks = 0; kph ^= 1u; }
                        ++nq;
                        progressed = true;
                    }
                }
                if (np < nq) {
                    const int sv = vs, pb = ps;
                    if (mbar_test(&p_full[pb], pph) && mbar_test(&v_full[sv], vph)) {
                        tc_fence_after();
                        const uint64_t va = vdesc + ((sv * L.tile) >> 4);
                        const uint64_t pa = pdesc + ((pb * 2 * PF_ATOM) >> 4);
#pragma unroll
                        for (int kk = 0; kk < PF_KEYS / 16; ++kk) {
                            const uint64_t ad = pa + (((kk >> 2) * PF_ATOM + (kk & 3) * 32) >> 4);
                            const uint64_t bd = va + ((kk * 2048) >> 4);
                            mma_bf16_ss(tmem + COL_O, ad, bd, idp, (np > 0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(&o_full[np & 1]);
                        if (NP != 2) mma_commit(&p_empty[pb]);
                        mma_commit(&v_empty[sv]);
                        if (++vs == NV) { vs = 0; vph ^= 1u; }
                        if (++ps == NP) { ps = 0; pph ^= 1u; }
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
                    else if (now - idle_since > a.wait_limit_ns) { *abort_flag = 1; break; }
                }
            }
            mma_commit(done_bar);  // every MMA of this CTA has finished before TMEM is freed
            mbar_wait_time(done_bar, 0, PF_DRAIN_NS);
        }
    } else {
        // --------- softmax: two warps per lane quadrant, a thread per row ---------
        const int quad = warp & 3;                   // TMEM lane quadrant of this warp
        const int half = (warp - PF_WARP_SM0) >> 2;  // keys [64 half, +64), O dims [HD half, +HD)
        const int ell = quad * 32 + lane;            // row of the tile = TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const int r = rt * PF_ROWS + ell;            // group row (member, i, j)
        int mb = -1, mi = 0, mj = 0;                 // its sequence, query row and head offset
        if (r < rows_g) {
            const int m = r / NG, rr = r - m * NG;
            mb = b0 + m;
            mi = rr / G;
            mj = rr - mi * G;
        }
        const long long prow = mb < 0 ? -1 : ((long long)mb * a.N + mi) * a.Hq + (long long)h * G + mj;
        auto warp_arrive = [&](uint64_t *b) {
            __syncwarp();
            if (lane == 0) mbar_arrive(b);
        };
        auto wait_w = [&](uint64_t *b, uint32_t parity) -> bool {
            const bool okw = mbar_test(b, parity) || mbar_wait(b, parity, abort_flag, a.wait_limit_ns);
            return __all_sync(0xffffffffu, okw);
        };
        // the two warps of a quadrant swap one value per row through TMEM
        // columns COL_X + 2 slot + half (the partner writes the other one)
        uint32_t pair_phase = 0;
        auto swap = [&](float v, int slot, bool &okx) -> float {
            tmem_st1(lane_base + COL_X + 2 * slot + half, v);
            tmem_wait_st();
            tc_fence_before();
            warp_arrive(&pair_bar[quad]);
            okx = okx && wait_w(&pair_bar[quad], pair_phase);
            pair_phase ^= 1;
            tc_fence_after();
            return tmem_ld1(lane_base + COL_X + 2 * slot + (half ^ 1));
        };
        {   // Q row (this half's head dims) into the swizzled K-major operand tile
            const uint4 *src = reinterpret_cast<const uint4 *>(a.q + (prow < 0 ? 0 : prow) * D);
            uint8_t *qt = base + L.off_q;
#pragma unroll
            for (int c = half * (D / 16); c < (half + 1) * (D / 16); ++c) {
                const uint4 v = prow >= 0 ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(qt + kmajor_off(ell, c)) = v;
            }
            fence_proxy_async_smem();
            warp_arrive(q_ready);
        }
        const float sc = a.scale_log2;
        float m_run = PF_M_NONE, l_run = 0.f;  // l_run: this half's keys only
        bool ok = true;
        int pslot = 0;  // P buffer of tile lt, and its phase
        uint32_t pphase = 0;
        // One pass over this half's 64 scores of a tile: their maximum, and p =
        // 2^(s scale - m) against a given maximum, packed as bf16 pairs, with
        // their sum. Keys past the prefix get p = 0.
        auto scores_to_p = [&](uint32_t sa, int valid, float m, float &mx, float &tsum, uint32_t *pk) {
            mx = -INFINITY;
            tsum = 0.f;
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 32) {
                float v[32];
                tmem_ld32(sa + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    float v0 = v[c], v1 = v[c + 1];
                    if (valid < 64) {
                        v0 = c0 + c < valid ? v0 : -INFINITY;
                        v1 = c0 + c + 1 < valid ? v1 : -INFINITY;
                    }
                    mx = fmaxf(mx, fmaxf(v0, v1));
                    const float p0 = ex2_approx(fmaf(v0, sc, -m)), p1 = ex2_approx(fmaf(v1, sc, -m));
                    tsum += p0 + p1;
                    const __nv_bfloat162 hv = __floats2bfloat162_rn(p0, p1);
                    pk[(c0 + c) >> 1] = *reinterpret_cast<const uint32_t *>(&hv);
                }
            }
        };
        for (int lt = 0; lt < ntiles && ok; ++lt) {
            const int sb = lt & 1, pb = pslot;
            const int valid = P - lt * PF_KEYS - half * 64;  // keys of this half inside the prefix
            if (!(ok = wait_w(&s_full[sb], (lt >> 1) & 1))) break;
            tc_fence_after();
            const uint32_t sa = lane_base + COL_S + sb * PF_KEYS + half * 64;
            // p against the running maximum, which stays unless this tile raises
            // it: a row's first tile, or a score above it by more than 2^8 (rare
            // after the first tile); a raise reads the scores once more
            float mx, tsum;
            uint32_t pk[32];
            scores_to_p(sa, valid, m_run, mx, tsum, pk);
            mx = fmaxf(mx, swap(mx, lt & 1, ok));
            if (!ok) break;
            const float cand = mx * sc;
            const bool raise = m_run == PF_M_NONE || cand > m_run + PF_RESCALE_LOG2;
            const float m_new = raise ? fmaxf(m_run, cand) : m_run;
            const bool wraise = __any_sync(0xffffffffu, raise);
            if (wraise) {
                float mx2;
                scores_to_p(sa, valid, m_new, mx2, tsum, pk);
            }
            tc_fence_before();
            warp_arrive(&s_empty[sb]);  // this tile's scores are read
            const float alpha = ex2_approx(m_run - m_new);  // first tile: 0; unchanged: 1
            l_run = l_run * alpha + tsum;
            if (lt > 0 && wraise) {
                // this half's dims of O, once the previous tile's P V has landed
                if (!(ok = wait_w(&o_full[(lt - 1) & 1], ((lt - 1) >> 1) & 1))) break;
                tc_fence_after();
#pragma unroll
                for (int c0 = 0; c0 < HD; c0 += 16) {
                    float o[16];
                    tmem_ld16(lane_base + COL_O + half * HD + c0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 16; ++c) o[c] *= alpha;
                    tmem_st16(lane_base + COL_O + half * HD + c0, o);
                }
                tmem_wait_st();
            }
            m_run = m_new;
            if (!(ok = wait_w(&p_free[pb], pphase ^ 1u))) break;
            if (++pslot == NP) { pslot = 0; pphase ^= 1u; }
            uint8_t *pt = base + L.off_p + pb * 2 * PF_ATOM;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<uint4 *>(pt + kmajor_off(ell, half * 8 + q)) =
                    make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            tc_fence_before();
            fence_proxy_async_smem();
            warp_arrive(&p_full[pb]);
        }
        // ---- epilogue: prefix partial (O in TMEM, m_run, l) merged with the row's suffix slots ----
        griddep_wait();  // the split-context kernel has completed: its slots are visible
        if (ok && ntiles > 0) ok = wait_w(&o_full[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1);
        if (ok) {
            tc_fence_after();
            const float lo = swap(l_run, 2, ok);
            const float l_p = half == 0 ? l_run + lo : lo + l_run;  // the same sum in both halves
            const float m_p = ntiles > 0 ? m_run : PF_M_NONE;
            // split-context schedule of the suffix call (the attention kernel's
            // rule): the prefix of the sequences' schedule positions, one copy
            // per warp, in the P buffers, which the last P V has finished reading
            int *TP = reinterpret_cast<int *>(base + L.off_p) + (warp - PF_WARP_SM0) * (MAX_SEQS + 1);
            {
                const int per = (a.B + 31) / 32;
                const int s0 = min(lane * per, a.B), s1 = min(s0 + per, a.B);
                int loc = 0;
                for (int b = s0; b < s1; ++b) loc += suffix_slots(a, b);
                int incl = loc;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                int run = incl - loc;
                for (int b = s0; b < s1; ++b) {
                    TP[b] = run;
                    run += suffix_slots(a, b);
                }
                if (lane == 31) TP[a.B] = incl;
                __syncwarp();
            }
            const int ups = a.Hkv * a.RC;
            const int total = ups * TP[a.B];
            const int W = total > 0 ? (total + a.num_ctas - 1) / a.num_ctas : 1;
            const size_t sf = slot_stride(a.rows_unit, D);
            int n = 0, ru = 0;
            const float *seg = a.ws_partial;
            if (mb >= 0) {
                const int Nc = a.rows_unit / G;  // whole query rows per row chunk
                const int rc = mi / Nc;          // row chunk of the unit that holds query row mi
                ru = (mi - rc * Nc) * G + mj;
                const int T1 = TP[mb + 1] - TP[mb];
                const int Tb = T1 > 0 ? T1 - UNIT_COST : 0;
                if (Tb > 0) {
                    const int hr = h * a.RC + rc;
                    const int u = mb * ups + hr;
                    const int tpre = ups * TP[mb] + hr * T1;
                    const int first = tpre / W;
                    n = (tpre + Tb - 1) / W - first + 1;
                    seg = a.ws_partial + (size_t)(u + first) * sf;
                }
            }
            // weights of the prefix partial and of the n suffix segments
            const size_t ml_off = (size_t)a.rows_unit * D + ru;
            float M = m_p;
            for (int k = 0; k < n; ++k) M = fmaxf(M, __ldcg(seg + k * sf + ml_off));
            const float wp = ex2_approx(m_p - M);  // M_NONE - finite underflows to 0
            float Lsum = wp * l_p;
            for (int k = 0; k < n; ++k)
                Lsum += ex2_approx(__ldcg(seg + k * sf + ml_off) - M) * __ldcg(seg + k * sf + ml_off + a.rows_unit);
            const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
#pragma unroll 1
            for (int c0 = 0; c0 < HD; c0 += 16) {
                float o[16];
                tmem_ld16(lane_base + COL_O + half * HD + c0, o);
                tmem_wait_ld();
                if (n > 0) {
#pragma unroll
                    for (int c = 0; c < 16; ++c) o[c] = ntiles > 0 ? o[c] * wp : 0.f;
                    for (int k = 0; k < n; ++k) {
                        const float wk = ex2_approx(__ldcg(seg + k * sf + ml_off) - M);
                        const float4 *src = reinterpret_cast<const float4 *>(seg + k * sf + (size_t)ru * D + half * HD + c0);
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) {
                            const float4 x = __ldcg(src + c4);
                            o[4 * c4] = fmaf(wk, x.x, o[4 * c4]);
                            o[4 * c4 + 1] = fmaf(wk, x.y, o[4 * c4 + 1]);
                            o[4 * c4 + 2] = fmaf(wk, x.z, o[4 * c4 + 2]);
                            o[4 * c4 + 3] = fmaf(wk, x.w, o[4 * c4 + 3]);
                        }
                    }
                    uint32_t pk[8];
#pragma unroll
                    for (int c = 0; c < 16; c += 2) {
                        const __nv_bfloat162 hv = __floats2bfloat162_rn(o[c] * inv, o[c + 1] * inv);
                        pk[c >> 1] = *reinterpret_cast<const uint32_t *>(&hv);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(a.out + (size_t)prow * D + half * HD + c0);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
        }
    }

    // ----------------------------- teardown -------------------------------
    tc_fence_before();
    __syncthreads();
    if (a.status && tid < 32) {
        // flags of the group's members, after the split-context kernel's status
        // stores: bad prefix pages (the first row tile of head 0 reports them),
        // and a wait of this CTA that gave up
        griddep_wait();
        const bool report = rt == 0 && h == 0;
        const int aborted = *abort_flag;
        for (int b = b0 + lane; b < pl.off[g + 1]; b += 32) {
            const int f = (report ? __ldcg(p.pflag + b) : 0) | (aborted ? SV_FLAG_TIMEOUT : 0);
            if (f) atomicOr(a.status + b, f);
        }
    }
    if (warp == PF_WARP_MMA) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

constexpr int PF_SMEM_LIMIT = 227 * 1024;

}  // namespace

void cascade_plan(const sv_cascade_desc *cd, int N, int Hq, int Hkv, CascadePlan *pl) {
    memset(pl, 0, sizeof *pl);
    const int G = Hq / Hkv;
    pl->num_groups = cd->num_groups;
    for (int g = 0; g <= cd->num_groups; ++g) pl->off[g] = cd->group_offsets[g];
    int acc = 0;
    for (int g = 0; g < cd->num_groups; ++g) {
        pl->pre[g] = cd->prefix_lens[g];
        pl->item0[g] = acc;
        const int rows = (pl->off[g + 1] - pl->off[g]) * N * G;
        acc += (rows + CASCADE_ROWS - 1) / CASCADE_ROWS * Hkv;
    }
    pl->item0[cd->num_groups] = acc;
    pl->items = acc;
}

CascadeWorkspace cascade_workspace(int B, int N, int Hq, int Hkv, int D, int max_blocks, int num_ctas) {
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
    w.total = off;
    return w;
}

template <typename Params>
static cudaError_t launch_pdl(void (*kfn)(Params), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              const Params &prm) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kfn, prm);
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
    // the epilogue keeps one copy of the sequences' tile prefix per softmax warp in the P buffers
    if ((size_t)PF_SM_WARPS * (MAX_SEQS + 1) * sizeof(int) > (size_t)fp.NP * 2 * PF_ATOM)
        return cudaErrorInvalidConfiguration;
    const size_t smem = L.total + 1024;
    auto kfn = cascade_prefix_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kfn, dim3((unsigned)items), dim3(PF_THREADS), smem, stream, fp);
}

cudaError_t launch_cascade(const AttnParams &p, const CascadePlan &plan, cudaStream_t stream) {
    const CascadeWorkspace w = cascade_workspace(p.B, p.N, p.Hq, p.Hkv, p.D, p.max_blocks, p.num_ctas);
    char *base = reinterpret_cast<char *>(p.ws_partial);
    int32_t *sfx_ctx = reinterpret_cast<int32_t *>(base + w.sfx_ctx);
    int32_t *pflag = reinterpret_cast<int32_t *>(base + w.pflag);
    int32_t *sfx_table = reinterpret_cast<int32_t *>(base + w.sfx_table);

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
    cudaError_t e = launch_pdl(cascade_prep_kernel, dim3((unsigned)p.B), dim3(PREP_THREADS), 0, stream, pp);
    if (e != cudaSuccess) return e;

    // the members' suffixes: every unit leaves its partial in a slot
    AttnParams a = p;
    a.block_table = sfx_table;
    a.ctx_lens = sfx_ctx;
    a.ws_partial = reinterpret_cast<float *>(base + w.slots);
    a.all_slots = 1;
    e = launch_attention(a, stream);
    if (e != cudaSuccess) return e;

    // the shared prefixes, merged with the slots into the output
    PrefixParams fp;
    memset(&fp, 0, sizeof fp);
    if (!encode_pool_map(&fp.tm_k, p.k_pool, p.num_blocks, p.Hkv, p.D) ||
        !encode_pool_map(&fp.tm_v, p.v_pool, p.num_blocks, p.Hkv, p.D))
        return cudaErrorInvalidValue;
    fp.a = a;
    fp.block_table = p.block_table;
    fp.pflag = pflag;
    fp.plan = plan;
    return p.D == 128 ? launch_prefix<128>(fp, plan.items, stream) : launch_prefix<64>(fp, plan.items, stream);
}

}  // namespace sv
