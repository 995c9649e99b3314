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
//   unit  = (sequence b, KV head h, row chunk rc): the query rows (i, g) of the
//           G query heads that read KV head h; a chunk holds whole query rows
//           i, at most ROWS_MAX rows (i, g) in all;
//   tile  = TILE_KEYS consecutive keys of one unit;
//   all tiles of all units are laid end to end, each unit followed by
//   UNIT_COST empty positions for its fixed cost, and the positions are cut
//   into num_ctas equal ranges, so every SM carries the same load whatever the
//   mix of context lengths. A CTA writes one partial (unnormalised O, running
//   max m, running sum l; log2 domain) per unit it touches but does not cover
//   whole to workspace slot unit + cta, unique because consecutive units share
//   at most one CTA; the combine kernel merges a unit's partials by their
//   log-sum-exp. A unit one CTA covers whole is written out directly.
//
// Inside a CTA (warp-specialised, tcgen05 + TMA, sm_100a), with MATH_WARPS =
// 4 x the number of softmax warpgroups:
//   warps 0 .. MATH_WARPS-1  softmax warpgroups, each owning CW of the RP row
//                columns; warp w owns TMEM lane quadrant w % 4 (a key for S, a
//                head dim for O). Per tile: load S, mask, a warpgroup vote on
//                raising the running column maxima (rare after a unit's first
//                tile; then the maxima are reduced over the 128 keys and O^T in
//                TMEM is rescaled), p = 2^(s scale - m) as bf16 into a swizzled
//                shared tile for the PV product;
//   WARP_K       TMA producer of the query rows (one 3-D box per 64 dims when a
//                unit starts) and of K: per tile, 8 pages x (D/64) boxes of 16
//                keys x 64 dims into a 128B-swizzled ring slot;
//   WARP_MMA     TMEM allocator and MMA issuer: S^T = K Q^T (M = 128 keys,
//                N = padded rows RP, K = D) and O^T += V^T P^T (M = 128 dims,
//                N = RP, K = 128 keys), fp32 accumulators in TMEM, S and O
//                double-buffered; it polls both queues and issues whichever
//                product is ready;
//   WARP_V       TMA producer of V, as for K;
//   WARP_ST      per-sequence status flags (and zero output for invalid
//                sequences), then the V ring: the rows of keys past ctx_len in
//                a tile's last page are zeroed before the tile goes to its PV.
// Ring slots and barrier phases are counters advanced once per tile.
// Putting keys on the MMA M dimension keeps the tensor-core work at
// 2 * 128 * RP * D per tile however few rows N*G there are, instead of
// padding the rows to 128.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <string.h>

#include <atomic>
#include <mutex>

#include "sv_internal.h"
#include "sv_tc.cuh"

namespace sv {

using namespace tc;

// Softmax warpgroups: 4 warps each (one TMEM lane quadrant per warp), each
// owning tc_cw(RP) consecutive row columns; RP = tc_cw(RP) * NWG. 96-row units
// take 32 columns per warpgroup: half the warps, each with twice the registers
// (no spills) and its fixed per-tile costs paid half as often.
__host__ __device__ constexpr int tc_cw(int RP) { return RP == 96 ? 32 : 16; }
constexpr int WARPS_PER_WG = 4;
__host__ __device__ constexpr int tc_nwg(int RP) { return RP / tc_cw(RP); }
__host__ __device__ constexpr int tc_threads(int RP) { return 32 * (WARPS_PER_WG * tc_nwg(RP) + 4); }
// Running column maximum of a column that has seen no visible key: finite, so
// that s*scale - M_NONE is +huge for a visible score (it votes for a raise) and
// -inf for a masked one (p = 0), with no special case in the exponentials.
constexpr float M_NONE = -3.402823466e38f;
// Drain limit: after an abort, a role still waits this long for its own copies
// and products in flight. The limit of every other wait is AttnParams::wait_limit_ns
// (2 s; test hooks shorten it).
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;

// ---------------------------------------------------------------------------
// Schedule helpers (attention and combine kernels agree on these).
// ---------------------------------------------------------------------------
SV_DEV int seq_tiles(const AttnParams &p, int b) {
    const int C = p.ctx_lens[b];
    const bool ok = C >= p.N && C <= p.max_blocks * PAGE;
    return ok ? (C + TILE_KEYS - 1) / TILE_KEYS : 0;
}

// Schedule positions of one unit of sequence b: its tiles plus UNIT_COST.
SV_DEV int seq_slots(const AttnParams &p, int b) {
    const int t = seq_tiles(p, b);
    return t > 0 ? t + UNIT_COST : 0;
}

// Tiles of a sequence from its schedule positions.
SV_DEV int real_tiles(int positions) { return positions > 0 ? positions - UNIT_COST : 0; }

// Exclusive prefix of per-sequence schedule positions (seq_slots) into
// TP[0..B] (and, when CL is given, the context lengths into CL[0..B)); the
// whole block participates.
SV_DEV void tile_prefix(const AttnParams &p, int *TP, int *scratch, int *CL = nullptr) {
    const int nt = blockDim.x, tid = threadIdx.x;
    const int per = (p.B + nt - 1) / nt;
    const int s0 = min(tid * per, p.B), s1 = min(s0 + per, p.B);
    int local = 0;
    for (int b = s0; b < s1; ++b) {
        local += seq_slots(p, b);
        if (CL) CL[b] = p.ctx_lens[b];
    }
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
        run += seq_slots(p, b);
    }
    if (tid == nt - 1) TP[p.B] = run;
    __syncthreads();
}

// Schedule position t -> sequence b (largest b with ups*TP[b] <= t).
SV_DEV int tile_seq(const int *TP, int B, int ups, int t) {
    int lo = 0, hi = B;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ups * TP[mid] <= t) lo = mid; else hi = mid;
    }
    return lo;
}

// A tile: sequence b, head/row-chunk hr, tile j of the unit's Tb tiles.
struct TileInfo {
    int b, hr, j, Tb;
};

// The tile after ti in the end-to-end order (j, then head/row chunk, then
// sequence; sequences without tiles are skipped). Callers stop at their range's
// end, so running past the last sequence only has to be harmless.
SV_DEV void next_tile(TileInfo &ti, const int *TP, int B, int ups) {
    if (++ti.j < ti.Tb) return;
    ti.j = 0;
    if (++ti.hr < ups) return;
    ti.hr = 0;
    do {
        ++ti.b;
        ti.Tb = ti.b < B ? real_tiles(TP[ti.b + 1] - TP[ti.b]) : 1;
    } while (ti.b < B && ti.Tb == 0);
}

// The first tile a CTA owns and how many it owns: the tiles whose schedule
// positions fall in [v0, v1) (positions past a unit's tiles hold no work).
SV_DEV TileInfo cta_tiles(const int *TP, int B, int ups, int v0, int v1, int *ntiles) {
    TileInfo ti{0, 0, 0, 1};
    *ntiles = 0;
    if (v0 >= v1) return ti;
    ti.b = tile_seq(TP, B, ups, v0);
    const int T1 = TP[ti.b + 1] - TP[ti.b];  // positions per unit of b (> 0)
    const int off = v0 - ups * TP[ti.b];
    ti.hr = off / T1;
    ti.j = off - ti.hr * T1;
    ti.Tb = real_tiles(T1);
    if (ti.j >= ti.Tb) {  // a position past the unit's tiles: start at the next unit
        ti.j = ti.Tb - 1;
        next_tile(ti, TP, B, ups);
    }
    TileInfo w = ti;
    int n = 0;
    while (w.b < B) {
        const int pos = ups * TP[w.b] + w.hr * (w.Tb + UNIT_COST) + w.j;
        if (pos >= v1) break;
        const int here = min(w.Tb - w.j, v1 - pos);
        n += here;
        w.j = w.Tb - 1;
        next_tile(w, TP, B, ups);
    }
    *ntiles = n;
    return ti;
}

// ---------------------------------------------------------------------------
// Shared-memory plan of the tcgen05 kernel (host and device agree).
// ---------------------------------------------------------------------------
constexpr uint32_t ATOM = 16384;  // 128 rows x 128 bytes, one 128B-swizzle column of a tile

struct TcLayout {
    uint32_t tile_bytes, off_k, off_q, q_bytes, off_p, p_bytes, off_bar, off_tp, off_cl, off_red, off_ms, off_as,
        off_lred, off_rowi, off_umask, off_vote, off_fin, off_mfin, off_misc, total;
};

// V ring first (slots 0..NV-1), then the K ring: a V slot plus 16 KB is always
// inside the allocation (the D = 64 PV product reads one unused atom there).
__host__ __device__ inline TcLayout tc_layout(int D, int RP, int NK, int NV, int NP, int NQ, int B) {
    TcLayout L;
    const int nDA = D / 64;
    const int NWG = tc_nwg(RP);
    L.tile_bytes = (uint32_t)nDA * ATOM;  // 128 keys of K or of V
    L.off_k = NV * L.tile_bytes;
    L.off_q = L.off_k + NK * L.tile_bytes;
    L.q_bytes = (uint32_t)nDA * RP * 128u;
    L.off_p = L.off_q + (uint32_t)NQ * L.q_bytes;
    L.p_bytes = (uint32_t)((RP + 63) / 64) * ATOM;
    L.off_bar = L.off_p + NP * L.p_bytes;
    const int nbar = 2 * NK + 2 * NV + 2 * 2 /*q*/ + 2 * 2 /*s*/ + 2 * NP /*p*/ + 2 * 2 /*o*/ + 1 /*done*/ +
                     NWG /*wg*/ + NV /*vz*/;
    L.off_tp = L.off_bar + 8u * nbar;
    L.off_cl = L.off_tp + 4u * (B + 1);
    L.off_red = (L.off_cl + 4u * B + 15u) & ~15u;
    const int CW = tc_cw(RP);
    L.off_ms = L.off_red + 4u * 2 * NWG * WARPS_PER_WG * CW;  // [par][wg][warp][CW] tile column maxima
    L.off_as = L.off_ms + 4u * 2 * RP;                        // [par][RP] running maxima
    L.off_lred = L.off_as + 4u * 2 * RP;                      // [par][RP] rescale factors
    L.off_rowi = L.off_lred + 4u * NWG * WARPS_PER_WG * CW;   // [wg][warp][CW] row-sum partials
    L.off_umask = (L.off_rowi + 4u * RP + 15u) & ~15u;        // [RP] row r -> r / G
    L.off_vote = L.off_umask + 8u * NWG * 64;                 // [wg][64] mask words of the unit
    L.off_fin = L.off_vote + 4u * 2 * NWG * WARPS_PER_WG;     // [par][wg][warp] rescale votes
    L.off_mfin = L.off_fin + 4u * RP;                         // [RP] row sums of a finished unit
    L.off_misc = L.off_mfin + 4u * RP;                        // [RP] row maxima of a finished unit
    L.total = L.off_misc + 16u + 4u * 32;
    return L;
}

struct TcParams {
    CUtensorMap tm_k;
    CUtensorMap tm_v;
    CUtensorMap tm_q;
    AttnParams a;
    int NK, NV, NP, NQ, Nc;  // K / V / P slots, query buffers (1 or 2), query rows per chunk
};

// ---------------------------------------------------------------------------
// The tcgen05 split-context kernel.
// ---------------------------------------------------------------------------
template <int D, int RP>
__global__ void __launch_bounds__(tc_threads(RP), 1) attn_tc_kernel(const __grid_constant__ TcParams P) {
    constexpr int nDA = D / 64;
    constexpr int NWG = tc_nwg(RP);
    constexpr int CW = tc_cw(RP);
    constexpr int MATH_WARPS = WARPS_PER_WG * NWG;
    constexpr int NTHREADS = tc_threads(RP);
    constexpr int RPa = (RP + 31) / 32 * 32;  // TMEM columns per S / O buffer
    constexpr int WARP_K = MATH_WARPS, WARP_MMA = MATH_WARPS + 1, WARP_V = MATH_WARPS + 2,
                  WARP_ST = MATH_WARPS + 3;
    const AttnParams &p = P.a;
    const int NK = P.NK, NV = P.NV, NP = P.NP, NQ = P.NQ;
    // query buffer of the u-th unit and the phase of its barriers
    auto qbuf = [NQ](int u) { return NQ == 1 ? 0 : (u & 1); };
    auto qphase = [NQ](int u) -> uint32_t { return NQ == 1 ? (u & 1) : ((u >> 1) & 1); };

    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const TcLayout L = tc_layout(D, RP, NK, NV, NP, NQ, p.B);
    uint64_t *bar = reinterpret_cast<uint64_t *>(base + L.off_bar);
    uint64_t *k_full = bar, *k_empty = bar + NK;
    uint64_t *v_full = bar + 2 * NK, *v_empty = v_full + NV;
    uint64_t *q_full = v_empty + NV, *q_empty = q_full + 2;
    uint64_t *s_full = q_empty + 2, *s_empty = s_full + 2;
    uint64_t *p_full = s_empty + 2, *p_empty = p_full + NP;
    uint64_t *o_full = p_empty + NP;   // [2] by tile parity: the tile's PV has completed
    uint64_t *o_free = o_full + 2;     // [2] by unit parity: the unit's O buffer has been read out
    uint64_t *done_bar = o_free + 2;
    uint64_t *wg_bar = done_bar + 1;   // [NWG] warpgroup-local barriers
    uint64_t *vz = wg_bar + NWG;       // [NV] the tile's V is ready for its PV (rows past ctx_len zeroed)
    // With a two-slot K ring, tile t's K slot is its S buffer t & 1 and the QK
    // product that frees the slot is the one s_full[t & 1] marks: the K producer
    // waits on s_full. Likewise with two P buffers, buffer t & 1 is freed by
    // tile t's PV, which o_full[t & 1] marks. One commit fewer per tile each.
    uint64_t *k_free = NK == 2 ? s_full : k_empty;
    uint64_t *p_free = NP == 2 ? o_full : p_empty;
    int *TP = reinterpret_cast<int *>(base + L.off_tp);
    int *CL = reinterpret_cast<int *>(base + L.off_cl);
    float *red = reinterpret_cast<float *>(base + L.off_red);
    float *mS = reinterpret_cast<float *>(base + L.off_ms);
    float *aS = reinterpret_cast<float *>(base + L.off_as);
    float *lred = reinterpret_cast<float *>(base + L.off_lred);
    int *rowi = reinterpret_cast<int *>(base + L.off_rowi);
    uint64_t *umask = reinterpret_cast<uint64_t *>(base + L.off_umask);
    int *vote = reinterpret_cast<int *>(base + L.off_vote);
    float *lfin = reinterpret_cast<float *>(base + L.off_fin);  // [RP] row sums of the finished unit
    float *mfin = reinterpret_cast<float *>(base + L.off_mfin); // [RP] its row maxima
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + L.off_misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + L.off_misc + 4);
    uint64_t *stall_bar = reinterpret_cast<uint64_t *>(base + L.off_misc + 8);  // test hook: never arrived on
    int *scratch = reinterpret_cast<int *>(base + L.off_misc + 16);  // one int per warp (<= 28), used once

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < NK; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
        for (int s = 0; s < NV; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1); mbar_init(&q_empty[i], 1);
            mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], MATH_WARPS);
            mbar_init(&o_full[i], 1); mbar_init(&o_free[i], MATH_WARPS);
        }
        for (int i = 0; i < NP; ++i) { mbar_init(&p_full[i], MATH_WARPS); mbar_init(&p_empty[i], 1); }
        mbar_init(done_bar, 1);
        for (int s = 0; s < NV; ++s) mbar_init(&vz[s], 1);
        for (int g = 0; g < NWG; ++g) mbar_init(&wg_bar[g], WARPS_PER_WG);
        mbar_init(stall_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (warp == WARP_K && lane == 0) {
        tma_prefetch_desc(&P.tm_k);
        tma_prefetch_desc(&P.tm_v);
        tma_prefetch_desc(&P.tm_q);
    }
    for (int r = tid; r < RP; r += NTHREADS) rowi[r] = r / p.G;
    {  // zero both query buffers: rows past a unit's real rows stay zero
        uint4 *q4 = reinterpret_cast<uint4 *>(base + L.off_q);
        for (uint32_t e = tid; e < (uint32_t)NQ * L.q_bytes / 16u; e += NTHREADS) q4[e] = make_uint4(0, 0, 0, 0);
    }
    // Everything above touches only this CTA's shared memory, TMEM and the
    // kernel parameters, so with a programmatic launch it overlaps the previous
    // kernel's tail. No input is read, and nothing written, before this wait.
    griddep_wait();
    griddep_launch_dependents();  // the combine kernel may now be scheduled
    tile_prefix(p, TP, scratch, CL);  // contains __syncthreads
    const int ups = p.Hkv * p.RC;
    const int total = ups * TP[p.B];  // schedule positions of all units
    const int W = total > 0 ? (total + p.num_ctas - 1) / p.num_ctas : 1;
    if (tid == 0) {
        // this CTA's tiles: those at positions [cta*W, cta*W + W); published to
        // every role through the (now free) scratch words
        const int v0 = min((int)blockIdx.x * W, total), v1 = min(v0 + W, total);
        int n;
        const TileInfo t0 = cta_tiles(TP, p.B, ups, v0, v1, &n);
        scratch[0] = t0.b; scratch[1] = t0.hr; scratch[2] = t0.j; scratch[3] = t0.Tb; scratch[4] = n;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const TileInfo t_first{scratch[0], scratch[1], scratch[2], scratch[3]};
    const int ntiles = scratch[4];

    if (warp == WARP_K || warp == WARP_V) {
        // ------------------- TMA producers (Q and K; V) -------------------
        if (lane == 0) {
            const bool is_k = warp == WARP_K;
            const int NR = is_k ? NK : NV;
            uint64_t *full = is_k ? k_full : v_full;
            uint64_t *empty = is_k ? k_free : v_empty;
            const CUtensorMap *tm = is_k ? &P.tm_k : &P.tm_v;
            uint8_t *ring = base + (is_k ? L.off_k : 0u);
            const uint32_t q_box_bytes = 64u * p.G * P.Nc * 2u;
            int lu = -1, issued_tiles = 0;
            int rs = 0;  // ring slot of tile lt, and its phase
            uint32_t rph = 0;
            TileInfo ti = t_first;
            for (int lt = 0; lt < ntiles; ++lt, next_tile(ti, TP, p.B, ups)) {
                const int h = ti.hr / p.RC, rc = ti.hr - h * p.RC;
                // gather the tile's page ids first (independent loads), then wait for the slot
                const int C = CL[ti.b];
                int blks[TILE_KEYS / PAGE];
#pragma unroll
                for (int pg = 0; pg < TILE_KEYS / PAGE; ++pg) {
                    const int page = ti.j * (TILE_KEYS / PAGE) + pg;
                    blks[pg] = page * PAGE < C ? __ldg(p.block_table + (size_t)ti.b * p.max_blocks + page) : -1;
                }
                if (is_k && (lt == 0 || ti.j == 0)) {
                    ++lu;
                    const int qb = qbuf(lu);
                    if (!mbar_wait(&q_empty[qb], qphase(lu) ^ 1, abort_flag, p.wait_limit_ns)) break;
                    mbar_arrive_expect_tx(&q_full[qb], q_box_bytes * nDA);
                    uint8_t *qdst = base + L.off_q + qb * L.q_bytes;
                    for (int a = 0; a < nDA; ++a)
                        tma_load_3d(qdst + a * RP * 128, &P.tm_q, &q_full[qb], a * 64, h * p.G,
                                    ti.b * p.N + rc * P.Nc);
                }
                const int s = rs;
                if (!mbar_wait(&empty[s], rph ^ 1u, abort_flag, p.wait_limit_ns)) break;
                if (++rs == NR) { rs = 0; rph ^= 1u; }
                mbar_arrive_expect_tx(&full[s], L.tile_bytes);
                uint8_t *dst = ring + s * L.tile_bytes;
#pragma unroll
                for (int pg = 0; pg < TILE_KEYS / PAGE; ++pg) {
                    // out of range (or past ctx_len): a coordinate past the pool, which the TMA unit fills with zeros
                    const int blk = (blks[pg] >= 0 && blks[pg] < p.num_blocks) ? blks[pg] : p.num_blocks;
                    for (int a = 0; a < nDA; ++a)
                        tma_load_4d(dst + a * ATOM + pg * 2048, tm, &full[s], a * 64, 0, h, blk);
                }
                issued_tiles = lt + 1;
            }
            if (*abort_flag) {
                // let this CTA's own copies land before it can exit: the last
                // use of every slot and query buffer must have completed
                for (int lt = max(0, issued_tiles - NR); lt < issued_tiles; ++lt)
                    mbar_wait_time(&full[lt % NR], (lt / NR) & 1, WAIT_LIMIT_NS);
                if (is_k)
                    for (int u = max(0, lu - NQ + 1); u <= lu; ++u)
                        mbar_wait_time(&q_full[qbuf(u)], qphase(u), WAIT_LIMIT_NS);
            }
        }
    } else if (warp == WARP_ST) {
        // ---------------- per-sequence status (and invalid sequences) ----------------
        // Sequence b is handled by CTA b mod num_ctas: a context outside
        // [N, max_blocks*16] gets SV_FLAG_BAD_CONTEXT and a zero output; a valid
        // one is scanned for block ids outside the pool (SV_FLAG_BAD_BLOCK).
        for (int b = blockIdx.x; b < p.B; b += p.num_ctas) {
            const int C = CL[b];
            const bool ctx_ok = C >= p.N && C <= p.max_blocks * PAGE;
            int bad = 0;
            if (ctx_ok) {
                for (int jb = lane; jb < (C + PAGE - 1) / PAGE; jb += 32) {
                    const int blk = __ldg(p.block_table + (size_t)b * p.max_blocks + jb);
                    bad |= (blk < 0 || blk >= p.num_blocks);
                }
            } else {
                uint4 *o4 = reinterpret_cast<uint4 *>(p.out + (size_t)b * p.N * p.Hq * D);
                for (int e = lane; e < p.N * p.Hq * D / 8; e += 32) o4[e] = make_uint4(0, 0, 0, 0);
            }
            bad = __any_sync(0xffffffffu, bad);
            if (p.status && lane == 0)
                p.status[b] = (ctx_ok ? 0 : SV_FLAG_BAD_CONTEXT) | (bad ? SV_FLAG_BAD_BLOCK : 0);
        }
        // ------------------- V rows past ctx_len -------------------
        // Softmax gives keys past ctx_len p = 0, but 0 * NaN is NaN and the rows
        // of the last page past ctx_len hold whatever the pool holds; they are
        // zeroed here once the tile has landed, off the softmax path. Every tile
        // is released to its PV through vz, after its V has landed, so this warp
        // stays within one phase of the V ring.
        TileInfo ti = t_first;
        int vs = 0;  // V slot of tile lt, and its phase
        uint32_t vph = 0;
        for (int lt = 0; lt < ntiles; ++lt, next_tile(ti, TP, p.B, ups)) {
            const int s = vs;
            const uint32_t par = vph;
            if (++vs == NV) { vs = 0; vph ^= 1u; }
            const bool landed = mbar_test(&v_full[s], par) || mbar_wait(&v_full[s], par, abort_flag, p.wait_limit_ns);
            if (!__all_sync(0xffffffffu, landed)) break;
            // keys [k0, k1) of the tile: past ctx_len but inside its last page (pages
            // wholly past ctx_len were loaded as zeros by the TMA unit)
            const int k0 = max(0, CL[ti.b] - ti.j * TILE_KEYS);
            const int k1 = min(TILE_KEYS, (k0 + PAGE - 1) / PAGE * PAGE);
            if (k0 < k1) {
                uint8_t *vt = base + s * L.tile_bytes;
                for (int e = lane; e < (k1 - k0) * 8 * nDA; e += 32) {
                    const int key = k0 + e / (8 * nDA), rem = e - (key - k0) * (8 * nDA);
                    reinterpret_cast<uint4 *>(vt + (rem >> 3) * ATOM + key * 128)[rem & 7] = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&vz[s]);
        }
    } else if (warp == WARP_MMA) {
        // -------------------------- MMA issuer ----------------------------
        // Polls both queues and issues whichever product is ready: QK of the
        // next tile once its K slot, its query rows and an S buffer are ready;
        // PV of the oldest softmaxed tile once its P and V are ready (and, at
        // a unit's first tile, once the unit's O buffer has been read out).
        // PV accumulates a unit's tiles in place in TMEM.
        if (lane == 0) {
            constexpr uint32_t idq = idesc_bf16(128, RP, false, false);
            constexpr uint32_t idp = idesc_bf16(128, RP, true, true);
            int nq = 0, np = 0, lu = -1, qb = 0, lup = -1;
            // ring slots of tiles nq (K) and np (V, P) and their phases, advanced
            // by one per product (no division by the runtime ring sizes)
            int ks = 0, vs = 0, ps = 0;
            uint32_t kph = 0, vph = 0, pph = 0;
            // operand descriptors of the ring bases; a product adds its stage's
            // offset (in 16-byte units; shared addresses stay below 2^18 bytes,
            // so the 14-bit address field does not carry)
            const uint64_t kdesc = sw128_desc(smem_u32(base + L.off_k), 16, 1024);
            const uint64_t qdesc = sw128_desc(smem_u32(base + L.off_q), 16, 1024);
            const uint64_t vdesc = sw128_desc(smem_u32(base), ATOM, 1024);
            const uint64_t pdesc = sw128_desc(smem_u32(base + L.off_p), ATOM, 1024);
            TileInfo tq = t_first;
            TileInfo tp = tq;
            uint32_t idle = 0;
            uint64_t idle_since = 0;
            while (np < ntiles) {
                bool progressed = false;
                if (nq < ntiles) {
                    const bool newu = (nq == 0 || tq.j == 0);
                    const int lu_n = newu ? lu + 1 : lu;
                    const int qb_n = qbuf(lu_n);
                    const int s = ks, sb = nq & 1;
                    if ((!newu || mbar_test(&q_full[qb_n], qphase(lu_n))) &&
                        mbar_test(&k_full[s], kph) && mbar_test(&s_empty[sb], ((nq >> 1) & 1) ^ 1)) {
                        lu = lu_n;
                        qb = qb_n;
                        tc_fence_after();
                        const uint64_t ka = kdesc + ((s * L.tile_bytes) >> 4);
                        const uint64_t qa = qdesc + ((qb * L.q_bytes) >> 4);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t ad = ka + (((kk >> 2) * ATOM + (kk & 3) * 32) >> 4);
                            const uint64_t bd = qa + (((kk >> 2) * (RP * 128) + (kk & 3) * 32) >> 4);
                            mma_bf16_ss(tmem + sb * RPa, ad, bd, idq, kk > 0);
                        }
                        mma_commit(&s_full[sb]);
                        if (NK != 2) mma_commit(&k_empty[s]);
                        if (nq == ntiles - 1 || tq.j == tq.Tb - 1) mma_commit(&q_empty[qb]);
                        if (++ks == NK) { ks = 0; kph ^= 1u; }
                        ++nq;
                        if (nq < ntiles) next_tile(tq, TP, p.B, ups);
                        progressed = true;
                    }
                }
                if (np < nq) {
                    const bool newu = (np == 0 || tp.j == 0);
                    const int lup_n = newu ? lup + 1 : lup;
                    const int s = vs, pb = ps, ob = lup_n & 1;
                    // vz follows v_full: the status warp arrives on it after it has
                    // seen the tile's V land
                    if (mbar_test(&p_full[pb], pph) && mbar_test(&vz[s], vph) &&
                        (!newu || mbar_test(&o_free[ob], ((lup_n >> 1) & 1) ^ 1))) {
                        lup = lup_n;
                        tc_fence_after();
                        const uint64_t va = vdesc + ((s * L.tile_bytes) >> 4);
                        const uint64_t pa = pdesc + ((pb * L.p_bytes) >> 4);
#pragma unroll
                        for (int kk = 0; kk < TILE_KEYS / 16; ++kk) {
                            const uint64_t ad = va + ((kk * 2048) >> 4);
                            const uint64_t bd = pa + ((kk * 2048) >> 4);
                            mma_bf16_ss(tmem + (2 + ob) * RPa, ad, bd, idp, (kk > 0 || !newu) ? 1u : 0u);
                        }
                        mma_commit(&o_full[np & 1]);
                        if (NP != 2) mma_commit(&p_empty[pb]);
                        mma_commit(&v_empty[s]);
                        if (++vs == NV) { vs = 0; vph ^= 1u; }
                        if (++ps == NP) { ps = 0; pph ^= 1u; }
                        ++np;
                        if (np < ntiles) next_tile(tp, TP, p.B, ups);
                        progressed = true;
                    }
                }
                if (progressed) {
                    idle = 0;
                } else if (++idle > 8 && (__nanosleep(20), (idle & 63) == 0)) {
                    // bounded like every other wait: give up after the limit without progress
                    if (*abort_flag) break;
                    const uint64_t now = globaltimer_ns();
                    if (idle == 64) idle_since = now;
                    else if (now - idle_since > p.wait_limit_ns) { *abort_flag = 1; break; }
                }
            }
            mma_commit(done_bar);  // every MMA of this CTA has finished before TMEM is freed
            mbar_wait_time(done_bar, 0, WAIT_LIMIT_NS);
        }
    } else {
        // ------------------------------ softmax ------------------------------
        const int wg = warp >> 2;          // warpgroup: owns row columns [wg*CW, wg*CW + CW)
        const int wiw = warp & 3;          // warp within the warpgroup = TMEM lane quadrant
        const int ell = wiw * 32 + lane;   // key (S) / head dim (O) lane
        const int col0 = wg * CW;
        uint32_t wg_phase = 0;
        const uint32_t lane_base = tmem + ((uint32_t)(wiw * 32) << 16);
        float lsum[CW];
#pragma unroll
        for (int c = 0; c < CW; ++c) lsum[c] = 0.f;
        const size_t slot_floats = slot_stride(p.rows_unit, D);
        bool ok = true;

        int cur_u = -1, last_par = 0, lu = -1;
        int ub = 0, uh = 0, urc = 0, uC = 0, urows = 0;

        // one arrival per warp: every lane's prior work is ordered by __syncwarp
        auto warp_arrive = [&](uint64_t *b) {
            __syncwarp();
            if (lane == 0) mbar_arrive(b);
        };
        // warp-uniform bounded wait: the tcgen05 accesses that follow are .sync.aligned
        auto wait_w = [&](uint64_t *b, uint32_t parity) -> bool {
            const bool r = mbar_test(b, parity) || mbar_wait(b, parity, abort_flag, p.wait_limit_ns);
            return __all_sync(0xffffffffu, r);
        };
        auto wg_sync = [&]() -> bool {
            warp_arrive(&wg_bar[wg]);
            const bool r = wait_w(&wg_bar[wg], wg_phase);
            wg_phase ^= 1;
            return r;
        };
        // A unit ends in two steps. close_unit, at the boundary: the row sums of
        // p are reduced over the 128 key lanes and kept with the row maxima; no
        // wait on the tensor core. finish_unit, once the next unit's first tile
        // is through softmax (its last PV has landed by then, or nearly): O^T
        // (lane = head dim, column = row) is read from the unit's TMEM buffer,
        // which is then released. A unit this CTA covered whole is normalised
        // and written out; otherwise the CTA stores a partial (unnormalised O,
        // running maximum, row sum) in its workspace slot for the combine kernel.
        bool pending = false;
        int pend_u = 0, pend_ob = 0, pend_jt = 0;
        auto close_unit = [&](int jt_last) -> bool {
#pragma unroll
            for (int c = 0; c < CW; ++c) {
                const float v = warp_sum(lsum[c]);
                if (lane == 0) lred[(wg * 4 + wiw) * CW + c] = v;
                lsum[c] = 0.f;
            }
            if (!wg_sync()) return false;
            if (wiw == 0 && lane < CW) {
                float l = 0.f;
                for (int w = 0; w < 4; ++w) l += lred[(wg * 4 + w) * CW + lane];
                lfin[col0 + lane] = l;
                mfin[col0 + lane] = mS[last_par * RP + col0 + lane];
            }
            if (!wg_sync()) return false;
            pending = true;
            pend_u = cur_u;
            pend_ob = lu & 1;
            pend_jt = jt_last;
            return true;
        };
        auto finish_unit = [&]() -> bool {
            pending = false;
            if (!wait_w(&o_full[pend_jt & 1], (pend_jt >> 1) & 1)) return false;
            tc_fence_after();
            const int fb = pend_u / ups, fhr = pend_u - fb * ups;
            const int fh = fhr / p.RC, frc = fhr - fh * p.RC;
            const int frows = min(p.rows_unit, p.R - frc * p.rows_unit);
            const int Tb = real_tiles(TP[fb + 1] - TP[fb]);
            const int tpre = ups * TP[fb] + fhr * (Tb + UNIT_COST);  // the unit's first position
            const int first_cta = tpre / W;
            const int nseg = (tpre + Tb - 1) / W - first_cta + 1;
            // a cascade call leaves every unit in a slot for the shared-prefix merge
            const bool to_slot = nseg > 1 || p.all_slots;
            float *slot = p.ws_partial + (size_t)(pend_u + blockIdx.x) * slot_floats;
            // O^T in chunks of 16 columns (few live registers)
#pragma unroll 1
            for (int c0 = 0; c0 < CW; c0 += 16) {
                float o[16];
                tmem_ld16(lane_base + (2 + pend_ob) * RPa + col0 + c0, o);
                tmem_wait_ld();
                if (ell >= D) continue;
                if (!to_slot) {
                    // row r of the unit is query row frc*Nc + r/G, head fh*G + r%G;
                    // rowi holds r/G (no division here: this code runs once per
                    // unit and is kept short)
                    uint16_t *orow = p.out + (((size_t)fb * p.N + frc * P.Nc) * p.Hq + fh * p.G) * D + ell;
                    const size_t hqd = (size_t)p.Hq * D;
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const int r = col0 + c0 + c;
                        if (r < frows) {
                            const int i = rowi[r];
                            const float l = lfin[r];
                            const __nv_bfloat16 v = __float2bfloat16_rn(l > 0.f ? __fdividef(o[c], l) : 0.f);
                            orow[i * hqd + (size_t)(r - i * p.G) * D] = *reinterpret_cast<const uint16_t *>(&v);
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        if (col0 + c0 + c < frows) slot[(size_t)(col0 + c0 + c) * D + ell] = o[c];
                }
            }
            tc_fence_before();
            warp_arrive(&o_free[pend_ob]);
            if (to_slot && wiw == 0 && lane < CW && col0 + lane < frows) {
                slot[(size_t)p.rows_unit * D + col0 + lane] = mfin[col0 + lane];
                slot[(size_t)p.rows_unit * D + p.rows_unit + col0 + lane] = lfin[col0 + lane];
            }
            return true;
        };

        // Test hook (p.stall): wait on a barrier nothing arrives on, so that the
        // bounded wait runs out, the CTA aborts through the same path as a real
        // timeout and every sequence is flagged SV_FLAG_TIMEOUT.
        if (p.stall) ok = wait_w(stall_bar, 0);

        // one pass past the last tile closes and finishes the CTA's last unit
        TileInfo tnext = t_first;
        int pslot = 0;  // P buffer of tile lt, and its phase
        uint32_t pphase = 0;
        for (int lt = 0; lt <= ntiles && ok; ++lt) {
            const bool end = lt == ntiles;
            const TileInfo ti = end ? TileInfo{0, 0, 0, 1} : tnext;
            if (!end) next_tile(tnext, TP, p.B, ups);
            const bool first = (lt == 0 || ti.j == 0 || end);
            if (first) {
                if (lt > 0 && !(ok = close_unit(lt - 1))) break;
                if (end) {
                    if (pending) ok = finish_unit();
                    break;
                }
                ++lu;
                cur_u = ti.b * ups + ti.hr;
                ub = ti.b;
                uh = ti.hr / p.RC;
                urc = ti.hr - uh * p.RC;
                uC = CL[ub];
                urows = min(p.rows_unit, p.R - urc * p.rows_unit);
                if (p.mask) {
                    for (int k = wiw * 32 + lane; k < p.N; k += 128)
                        umask[wg * 64 + k] = __ldg(p.mask + (size_t)ub * p.N + k);
                    if (!(ok = wg_sync())) break;
                }
            }
            const int sb = lt & 1, par = lt & 1;
            if (!(ok = wait_w(&s_full[sb], (lt >> 1) & 1))) break;
            tc_fence_after();
            float sv[CW];
            tmem_ld_cols<CW>(lane_base + sb * RPa + col0, sv);
            tmem_wait_ld();
            tc_fence_before();
            warp_arrive(&s_empty[sb]);

            // Scores stay unscaled here: the 1/sqrt(D) * log2(e) factor is positive,
            // so it is applied to the column maximum and folded into the exponent.
            const int key = ti.j * TILE_KEYS + ell;
            const bool valid = key < uC;
            const int newk = key - (uC - p.N);
            if (__any_sync(0xffffffffu, !valid || newk >= 0)) {
                // tile holds keys past ctx_len or new (masked) keys: per-element visibility
                const int ibase = urc * P.Nc;
#pragma unroll
                for (int c = 0; c < CW; ++c) {
                    bool vis = valid;
                    if (valid && newk >= 0 && col0 + c < urows) {
                        const int i = ibase + rowi[col0 + c];
                        vis = p.mask ? ((umask[wg * 64 + i] >> newk) & 1ull) != 0 : newk <= i;
                    }
                    if (!vis) sv[c] = -INFINITY;
                }
            }

            // Running maxima are only raised when a score exceeds its column's
            // current maximum by more than 2^RESCALE_LOG2 (after a unit's first
            // tile this is rare): p = 2^(s*scale - m) then stays below 2^8 and
            // the tile folds in with alpha = 1. Otherwise the tile's column
            // maxima are reduced over the 128 keys, the maxima raised, and the
            // unit's O in TMEM rescaled before this tile's PV adds to it.
            // The exponent s*scale - m against the current maxima decides the vote
            // and (when nothing is raised) feeds the exponentials. A column with no
            // visible key yet holds M_NONE: its first visible score votes for a
            // raise, and masked scores (-inf) give 2^-inf = 0.
            constexpr float RESCALE_LOG2 = 8.f;
            const float sc = p.scale_log2;
            const float4 *mo4 = reinterpret_cast<const float4 *>(mS + (par ^ 1) * RP + col0);
            bool need = first;
            if (!first) {
#pragma unroll
                for (int c4 = 0; c4 < CW / 4; ++c4) {
                    const float4 m4 = mo4[c4];
                    need |= fmaf(sv[c4 * 4 + 0], sc, -m4.x) > RESCALE_LOG2;
                    need |= fmaf(sv[c4 * 4 + 1], sc, -m4.y) > RESCALE_LOG2;
                    need |= fmaf(sv[c4 * 4 + 2], sc, -m4.z) > RESCALE_LOG2;
                    need |= fmaf(sv[c4 * 4 + 3], sc, -m4.w) > RESCALE_LOG2;
                }
            }
            const bool wneed = __any_sync(0xffffffffu, need);
            if (lane == 0) vote[(par * NWG + wg) * 4 + wiw] = wneed;
            if (!(ok = wg_sync())) break;
            const int *vt = vote + (par * NWG + wg) * 4;
            const bool rescale = (vt[0] | vt[1] | vt[2] | vt[3]) != 0;
            if (rescale) {
                float *rd = red + ((par * NWG + wg) * 4 + wiw) * CW;
#pragma unroll
                for (int c = 0; c < CW; ++c) {
                    float m;
                    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(m) : "f"(sv[c]));
                    if (lane == c) rd[c] = m;
                }
                if (!(ok = wg_sync())) break;
                if (wiw == 0 && lane < CW) {
                    const int c = lane;
                    const float m_old = first ? M_NONE : mS[(par ^ 1) * RP + col0 + c];
                    float rmax = -INFINITY;
                    for (int w = 0; w < 4; ++w) rmax = fmaxf(rmax, red[((par * NWG + wg) * 4 + w) * CW + c]);
                    const float mx = fmaxf(m_old, rmax * sc);  // stays M_NONE while nothing is visible
                    mS[par * RP + col0 + c] = mx;
                    aS[par * RP + col0 + c] = ex2_approx(m_old - mx);  // M_NONE - finite underflows to 0
                }
                if (!(ok = wg_sync())) break;
                {
                    // the running row sums follow the raised maxima
                    const float4 *an4 = reinterpret_cast<const float4 *>(aS + par * RP + col0);
#pragma unroll
                    for (int c4 = 0; c4 < CW / 4; ++c4) {
                        const float4 a4 = an4[c4];
                        lsum[c4 * 4 + 0] *= a4.x;
                        lsum[c4 * 4 + 1] *= a4.y;
                        lsum[c4 * 4 + 2] *= a4.z;
                        lsum[c4 * 4 + 3] *= a4.w;
                    }
                }
                if (!first) {
                    // scale the unit's O^T columns once the previous tile's PV has landed
                    if (!(ok = wait_w(&o_full[(lt - 1) & 1], ((lt - 1) >> 1) & 1))) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int c0 = 0; c0 < CW; c0 += 16) {  // chunks of 16 columns
                        float o[16];
                        const uint32_t oaddr = lane_base + (2 + (lu & 1)) * RPa + col0 + c0;
                        tmem_ld16(oaddr, o);
                        tmem_wait_ld();
                        const float4 *a4p = reinterpret_cast<const float4 *>(aS + par * RP + col0 + c0);
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) {
                            const float4 a4 = a4p[c4];
                            o[c4 * 4 + 0] *= a4.x;
                            o[c4 * 4 + 1] *= a4.y;
                            o[c4 * 4 + 2] *= a4.z;
                            o[c4 * 4 + 3] *= a4.w;
                        }
                        tmem_st16(oaddr, o);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                }
            } else if (wiw == 0 && lane < CW) {
                // keep the maxima: readers of these slots are past the next tile's vote sync
                mS[par * RP + col0 + lane] = mS[(par ^ 1) * RP + col0 + lane];
                aS[par * RP + col0 + lane] = 1.f;
            }
            last_par = par;
            const float4 *ms4 = reinterpret_cast<const float4 *>(mS + (rescale ? par : par ^ 1) * RP + col0);
            uint32_t packed[CW / 2];
#pragma unroll
            for (int c4 = 0; c4 < CW / 4; ++c4) {
                const float4 m4 = ms4[c4];
                const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
                float pp[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int c = c4 * 4 + k;
                    pp[k] = ex2_approx(fmaf(sv[c], sc, -mm[k]));  // p = 2^(s*scale - m)
                    lsum[c] += pp[k];
                }
                __nv_bfloat162 h0 = __floats2bfloat162_rn(pp[0], pp[1]);
                __nv_bfloat162 h1 = __floats2bfloat162_rn(pp[2], pp[3]);
                packed[c4 * 2] = *reinterpret_cast<uint32_t *>(&h0);
                packed[c4 * 2 + 1] = *reinterpret_cast<uint32_t *>(&h1);
            }
            const int pb = pslot;
            if (!(ok = wait_w(&p_free[pb], pphase ^ 1u))) break;
            if (++pslot == NP) { pslot = 0; pphase ^= 1u; }
            uint8_t *pbuf = base + L.off_p + pb * L.p_bytes;
#pragma unroll
            for (int c8 = 0; c8 < CW / 8; ++c8) {
                const int cc = col0 + c8 * 8;
                const int chunk = (cc & 63) >> 3;
                uint4 *dst = reinterpret_cast<uint4 *>(pbuf + (cc >> 6) * ATOM + (ell >> 3) * 1024 +
                                                       (ell & 7) * 128 + ((chunk ^ (ell & 7)) << 4));
                *dst = make_uint4(packed[c8 * 4], packed[c8 * 4 + 1], packed[c8 * 4 + 2], packed[c8 * 4 + 3]);
            }
            fence_proxy_async_smem();
            warp_arrive(&p_full[pb]);
            // the previous unit's last PV was issued before this tile's
            if (pending && !(ok = finish_unit())) break;
        }
    }

    // ----------------------------- teardown -------------------------------
    tc_fence_before();
    __syncthreads();
    if (*abort_flag && p.status)
        for (int b = tid; b < p.B; b += NTHREADS) atomicOr(p.status + b, SV_FLAG_TIMEOUT);
    if (warp == WARP_MMA) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

constexpr int COMBINE_ROWS = 8;       // rows per combine CTA, one warp each
constexpr int COMBINE_REG_SEGS = 8;   // segments whose partial row is loaded up front

// Block-wide integer sum for blockDim.x <= 32 * COMBINE_ROWS; red holds one slot per warp.
SV_DEV int block_sum_i(int v, int *red) {
    v = __reduce_add_sync(0xffffffffu, v);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    int t = 0;
    for (int w = 0; w < (int)(blockDim.x + 31) / 32; ++w) t += red[w];
    __syncthreads();
    return t;
}

// Merge the partials of every unit that was split over several CTAs (a unit one
// CTA covered whole was written by the attention kernel, and an invalid
// sequence by its status warp). One CTA per (COMBINE_ROWS rows, unit), one warp
// per row, four head dimensions per lane:
//   M = max_k m_k,  L = sum_k 2^(m_k - M) l_k,  out = sum_k 2^(m_k - M) O_k / L.
// Launched as a programmatic dependent of the attention kernel, which lets it
// launch only after its own wait on earlier work: the schedule is recomputed
// from ctx_lens (complete by then) before this kernel waits, so once the
// attention kernel completes one round of loads remains.
// MIN_CTAS: CTAs per SM the register budget is sized for. Two when there are at
// most a quarter as many units as attention CTAs (every unit is split about four
// ways or more, and the extra registers keep more of its partials' loads in
// flight); three otherwise (a unit has a few partials, and most of the
// combine's CTAs return after the schedule test, so CTA turnover counts).
template <int MIN_CTAS>
__global__ void __launch_bounds__(32 * COMBINE_ROWS, MIN_CTAS) attn_combine_kernel(const AttnParams p) {
    griddep_launch_dependents();  // the next call's attention kernel may run its prologue
    const int u = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D = p.D, RU = p.rows_unit;
    const int ups = p.Hkv * p.RC;
    const int b = u / ups, hr = u - b * ups;
    const int h = hr / p.RC, rc = hr - h * p.RC;
    const int rows = min(RU, p.R - rc * RU);
    const int r = blockIdx.x * COMBINE_ROWS + warp;
    __shared__ int red_i[COMBINE_ROWS];
    // the attention kernel's schedule: all positions, those before sequence b,
    // b's own tiles
    int tot = 0, before = 0, own = 0;
    for (int s = threadIdx.x; s < p.B; s += blockDim.x) {
        const int t = seq_slots(p, s);
        tot += t;
        before += s < b ? t : 0;
        own += s == b ? real_tiles(t) : 0;
    }
    tot = block_sum_i(tot, red_i);
    before = block_sum_i(before, red_i);
    const int Tb = block_sum_i(own, red_i);
    if (Tb == 0 || r >= rows) return;
    const int total = ups * tot;
    const int W = (total + p.num_ctas - 1) / p.num_ctas;
    const int tpre = ups * before + hr * (Tb + UNIT_COST);
    const int first = tpre / W, n = (tpre + Tb - 1) / W - first + 1;
    if (n == 1) return;  // written by the attention kernel
    const int ridx = rc * RU + r;
    const int i = ridx / p.G, hq = h * p.G + (ridx - i * p.G);
    const size_t sf = slot_stride(RU, D);
    const float *seg0 = p.ws_partial + (size_t)(u + first) * sf;
    const bool dl = lane < D / 4;  // this lane holds head dims 4*lane .. 4*lane+3

    griddep_wait();  // the partials are complete and visible
    // one round of loads: this lane's dims of the first partials, and segment lane's (m, l)
    float4 ov[COMBINE_REG_SEGS];
#pragma unroll
    for (int k = 0; k < COMBINE_REG_SEGS; ++k)
        ov[k] = (k < n && dl) ? __ldcg(reinterpret_cast<const float4 *>(seg0 + (size_t)k * sf + (size_t)r * D) + lane)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    float mk = -INFINITY, lk = 0.f;
    if (lane < n) {
        mk = __ldcg(seg0 + (size_t)lane * sf + (size_t)RU * D + r);
        lk = __ldcg(seg0 + (size_t)lane * sf + (size_t)RU * D + RU + r);
    }
    float M = mk;
    for (int k = lane + 32; k < n; k += 32) M = fmaxf(M, __ldcg(seg0 + (size_t)k * sf + (size_t)RU * D + r));
    M = warp_max(M);
    const float wl = lane < n ? exp2f(mk - M) : 0.f;  // an empty segment holds l = 0
    float L = wl * lk;
    for (int k = lane + 32; k < n; k += 32) {
        const float *sg = seg0 + (size_t)k * sf + (size_t)RU * D;
        L = fmaf(exp2f(__ldcg(sg + r) - M), __ldcg(sg + RU + r), L);
    }
    L = warp_sum(L);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < COMBINE_REG_SEGS; ++k) {
        const float w = __shfl_sync(0xffffffffu, wl, k);
        if (k < n) {
            acc.x = fmaf(w, ov[k].x, acc.x); acc.y = fmaf(w, ov[k].y, acc.y);
            acc.z = fmaf(w, ov[k].z, acc.z); acc.w = fmaf(w, ov[k].w, acc.w);
        }
    }
    // the rest (a unit split over many CTAs, at small B) four at a time, the
    // four loads in flight before the first is used
    const size_t sf4 = sf / 4;  // slot stride in float4 (slots are 256-byte multiples)
    const float4 *op = reinterpret_cast<const float4 *>(seg0 + (size_t)COMBINE_REG_SEGS * sf + (size_t)r * D) + lane;
#pragma unroll 1
    for (int k0 = COMBINE_REG_SEGS; k0 < n; k0 += 4, op += 4 * sf4) {
        float4 ob[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            ob[j] = (k0 + j < n && dl) ? __ldcg(op + j * sf4) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = k0 + j;  // partials past n were loaded as zeros
            const float w = k < 32 ? __shfl_sync(0xffffffffu, wl, k & 31)
                                   : (k < n ? exp2f(__ldcg(seg0 + (size_t)k * sf + (size_t)RU * D + r) - M) : 0.f);
            acc.x = fmaf(w, ob[j].x, acc.x); acc.y = fmaf(w, ob[j].y, acc.y);
            acc.z = fmaf(w, ob[j].z, acc.z); acc.w = fmaf(w, ob[j].w, acc.w);
        }
    }
    if (!dl) return;
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const __nv_bfloat162 o01 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    const __nv_bfloat162 o23 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 packed;
    packed.x = *reinterpret_cast<const uint32_t *>(&o01);
    packed.y = *reinterpret_cast<const uint32_t *>(&o23);
    *reinterpret_cast<uint2 *>(p.out + (((size_t)b * p.N + i) * p.Hq + hq) * D + 4 * lane) = packed;
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
// Workspace: the partial slots (the combine kernel recomputes the schedule).

void row_chunks(int N, int G, int *rows_unit, int *RC, int *Nc) {
    const int R = N * G;
    if (R <= ROWS_MAX) {
        *rows_unit = R;
        *RC = 1;
        *Nc = N;
    } else {
        const int nc = ROWS_MAX / G;  // whole query rows per chunk (G <= ROWS_MAX is validated)
        *Nc = nc;
        *rows_unit = nc * G;
        *RC = (N + nc - 1) / nc;
    }
}

int attention_num_ctas() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return sms;
}

size_t attention_workspace_bytes(int B, int N, int Hq, int Hkv, int D, int num_ctas) {
    int RU, RC, Nc;
    row_chunks(N, Hq / Hkv, &RU, &RC, &Nc);
    const size_t units = (size_t)B * Hkv * RC;
    const size_t slot_floats = slot_stride(RU, D);
    return (units + (size_t)num_ctas) * slot_floats * sizeof(float);
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// Pool map: boxes of 16 keys x 64 dims, 128B-swizzled, for the shared-memory
// tiles; with whole_page, 16 keys x D dims un-swizzled, for L2 prefetches.
bool encode_pool_map(CUtensorMap *m, const void *pool, int num_blocks, int Hkv, int D, bool whole_page) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)PAGE, (cuuint64_t)Hkv, (cuuint64_t)num_blocks};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)PAGE * D * 2, (cuuint64_t)Hkv * PAGE * D * 2};
    const cuuint32_t box[4] = {whole_page ? (cuuint32_t)D : 64u, PAGE, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(pool), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, whole_page ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool encode_q_map(CUtensorMap *m, const void *q, int B, int N, int Hq, int D, int G, int Nc) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)B * N};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)Nc};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int SMEM_LIMIT = 227 * 1024;

// Launch with programmatic stream serialization: the kernel may start while the
// previous kernel in the stream finishes; it waits (griddep_wait) before it
// reads any input or writes anything.
template <typename... Args>
static cudaError_t launch_programmatic(void (*kfn)(Args...), dim3 grid, dim3 block, size_t smem,
                                       cudaStream_t stream, const Args &...args) {
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
    return cudaLaunchKernelEx(&cfg, kfn, args...);
}

template <int D, int RP>
static cudaError_t launch_tc(TcParams &P, cudaStream_t stream) {
    // deepest K/V rings, P and query buffering that fit, in order of preference
    // (K, V, P, Q); a single query buffer stalls a unit's first product on its
    // query load, which costs less than a shallower ring, or a single P buffer
    // (the softmax then waits on every P.V), when units are long
    static const int choices[][4] = {{3, 4, 2, 2}, {2, 4, 2, 2}, {2, 3, 2, 2}, {2, 3, 2, 1}, {2, 3, 1, 2},
                                     {2, 2, 2, 2}, {2, 2, 2, 1}, {2, 2, 1, 2}, {2, 2, 1, 1}};
    constexpr int nchoices = sizeof(choices) / sizeof(choices[0]);
    TcLayout L;
    int k = 0;
    for (; k < nchoices; ++k) {
        L = tc_layout(D, RP, choices[k][0], choices[k][1], choices[k][2], choices[k][3], P.a.B);
        if (L.total + 1024 <= (uint32_t)SMEM_LIMIT) break;
    }
    if (k == nchoices) return cudaErrorInvalidConfiguration;
    P.NK = choices[k][0];
    P.NV = choices[k][1];
    P.NP = choices[k][2];
    P.NQ = choices[k][3];
    const size_t smem = L.total + 1024;
    auto kfn = attn_tc_kernel<D, RP>;
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_programmatic(kfn, dim3(P.a.num_ctas), dim3(tc_threads(RP)), smem, stream, P);
}

template <int D>
static cudaError_t launch_tc_rp(TcParams &P, int RP, cudaStream_t stream) {
    switch (RP) {
        case 16: return launch_tc<D, 16>(P, stream);
        case 32: return launch_tc<D, 32>(P, stream);
        case 48: return launch_tc<D, 48>(P, stream);
        case 64: return launch_tc<D, 64>(P, stream);
        case 96: return launch_tc<D, 96>(P, stream);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_attention(const AttnParams &p, cudaStream_t stream) {
    TcParams P;
    memset(&P, 0, sizeof P);
    P.a = p;
    int RU, RC, Nc;
    row_chunks(p.N, p.G, &RU, &RC, &Nc);
    P.Nc = Nc;
    if (!encode_pool_map(&P.tm_k, p.k_pool, p.num_blocks, p.Hkv, p.D) ||
        !encode_pool_map(&P.tm_v, p.v_pool, p.num_blocks, p.Hkv, p.D) ||
        !encode_q_map(&P.tm_q, p.q, p.B, p.N, p.Hq, p.D, p.G, Nc))
        return cudaErrorInvalidValue;
    // rows padded to a multiple of 16; 65-80 rows run on the 96-row kernel (three
    // 32-column warpgroups) rather than five 16-column ones at 768 threads
    const int RP = RU > 64 ? 96 : (RU + 15) / 16 * 16;
    cudaError_t e = p.D == 128 ? launch_tc_rp<128>(P, RP, stream) : launch_tc_rp<64>(P, RP, stream);
    if (e != cudaSuccess || p.all_slots) return e;  // a cascade call merges in the shared-prefix kernel
    return launch_programmatic(4 * p.units <= p.num_ctas ? attn_combine_kernel<2> : attn_combine_kernel<3>,
                               dim3((RU + COMBINE_ROWS - 1) / COMBINE_ROWS, p.units),
                               dim3(32 * COMBINE_ROWS), 0, stream, p);
}

}  // namespace sv
