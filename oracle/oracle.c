/*
 * Plain CPU oracle for the speculative-decoding verify step.
 *
 * TEST INFRASTRUCTURE ONLY. Tests, the smoke check and the bench's CPU
 * baseline leg call it; the library under speculative_decoding_rl_b200/ never
 * does, and this file shares no code with it.
 *
 * Everything is computed in fp64, single-threaded, straight from the
 * definitions, with no blocking, splitting or fusion:
 *
 *  - Verify attention: each active sequence scores its N = gamma+1 draft query
 *    rows against its whole paged KV cache in one target pass (TLT reading
 *    notes, "1. RL and SD", paragraph on why the target can check several
 *    positions at once). Prefix keys are visible to every row; among the N
 *    new keys, row i sees key j iff bit j of its ancestor mask is set (a chain
 *    when no mask is given). Scores are q.k/sqrt(D) and the output is the
 *    softmax-weighted sum of V. GQA: query head hq reads KV head hq/(Hq/Hkv).
 *
 *  - Cascade verify attention: the same attention for groups of rollouts
 *    that share a prompt's KV pages (SRT review, "Tree-Structured KV
 *    Cache"): the group's prefix keys come from one set of pages.
 *
 *  - Accept / resample: the lossless rule (Accelerating RL Post-Training
 *    Rollouts via System-Integrated Speculative Decoding, Abstract: speculative
 *    decoding preserves the target's output distribution), with drafts after
 *    the first rejection discarded (TLT reading notes, "1. RL and SD"). For a
 *    draft tree (SRT review, "Speculative Rollout integration", step 5: accept
 *    or reject by tree verification) the walk is recursive rejection sampling
 *    over the children of each accepted node in index order; a chain is the
 *    tree whose every node has at most one child.
 *
 *  - Random numbers: Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel
 *    random numbers: as easy as 1, 2, 3", SC'11), key = 64-bit seed, counter =
 *    {sequence, node, tag, 0}; tag 0 draws the accept uniform of a draft node,
 *    tag 1 the resampling uniform at the node where the walk stops. A uniform
 *    is the top 24 bits of output word 0 times 2^-24, exact in fp32 and fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_TIE_EPS 1e-5

/* ------------------------------------------------------------------------ */
/* Philox4x32-10                                                             */
/* ------------------------------------------------------------------------ */

/* Round multipliers and Weyl key increments of Philox-4x32 as given in the
 * SC'11 paper (multipliers chosen for avalanche; key increments are the
 * golden ratio and sqrt(3)-1 in 0.32 fixed point). */
static const uint32_t PHILOX_M0 = 0xD2511F53u;
static const uint32_t PHILOX_M1 = 0xCD9E8D57u;
static const uint32_t PHILOX_W0 = 0x9E3779B9u;
static const uint32_t PHILOX_W1 = 0xBB67AE85u;

void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += PHILOX_W0; k1 += PHILOX_W1; }
        uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)x0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)x2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t y0 = hi1 ^ x1 ^ k0;
        uint32_t y1 = lo1;
        uint32_t y2 = hi0 ^ x3 ^ k1;
        uint32_t y3 = lo0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* The block function applied to n counters (ctr and out: [n][4]) under one key. */
void orc_philox4x32_10_many(long n, const uint32_t *ctr, const uint32_t key[2], uint32_t *out)
{
    for (long i = 0; i < n; ++i) orc_philox4x32_10(ctr + 4 * i, key, out + 4 * i);
}

double orc_uniform(uint64_t seed, uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3)
{
    uint32_t ctr[4] = {c0, c1, c2, c3};
    uint32_t key[2] = {(uint32_t)(seed & 0xFFFFFFFFu), (uint32_t)(seed >> 32)};
    uint32_t out[4];
    orc_philox4x32_10(ctr, key, out);
    return (double)(out[0] >> 8) * (1.0 / 16777216.0);
}

/* ------------------------------------------------------------------------ */
/* bf16                                                                      */
/* ------------------------------------------------------------------------ */

double orc_bf16_to_double(uint16_t h)
{
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* Verify attention                                                          */
/* ------------------------------------------------------------------------ */

/* A sequence is valid when N <= ctx_len <= max_blocks*bs and every block id
 * of its ceil(ctx_len/bs) pages lies in [0, num_blocks). */
static int seq_valid(int N, int bs, int max_blocks, int num_blocks, const int32_t *block_table,
                     const int32_t *ctx_lens, int b)
{
    const int C = ctx_lens[b];
    if (C < N || C > max_blocks * bs) return 0;
    for (int j = 0; j < (C + bs - 1) / bs; ++j) {
        int blk = block_table[(size_t)b * max_blocks + j];
        if (blk < 0 || blk >= num_blocks) return 0;
    }
    return 1;
}

/* One output row of a valid sequence: sequence b, query row i, query head hq.
 * out_row has D entries (all zero if the row sees no key). */
static void attention_row(int N, int Hq, int Hkv, int D, int bs, int max_blocks,
                         const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                         const int32_t *block_table, const int32_t *ctx_lens,
                         const uint64_t *mask, int b, int i, int hq, double *out_row,
                         double *scratch)
{
    const int G = Hq / Hkv;
    const int h = hq / G;
    const int C = ctx_lens[b];
    for (int d = 0; d < D; ++d) out_row[d] = 0.0;
    const int prefix = C - N;
    const uint16_t *qv = q + (((size_t)b * N + i) * Hq + hq) * D;
    const double scale = 1.0 / sqrt((double)D);
    double mx = -INFINITY;
    int any = 0;
    for (int t = 0; t < C; ++t) {
        int visible;
        if (t < prefix) visible = 1;
        else {
            int j = t - prefix;
            if (mask) visible = (int)((mask[(size_t)b * N + i] >> j) & 1u);
            else visible = (j <= i);
        }
        if (!visible) { scratch[t] = -INFINITY; continue; }
        int blk = block_table[(size_t)b * max_blocks + t / bs];
        const uint16_t *kv = k_pool + (((size_t)blk * Hkv + h) * bs + (t % bs)) * D;
        double s = 0.0;
        for (int d = 0; d < D; ++d) s += orc_bf16_to_double(qv[d]) * orc_bf16_to_double(kv[d]);
        s *= scale;
        scratch[t] = s;
        if (s > mx) mx = s;
        any = 1;
    }
    if (!any) return;
    double z = 0.0;
    for (int t = 0; t < C; ++t) {
        if (scratch[t] == -INFINITY) continue;
        double e = exp(scratch[t] - mx);
        scratch[t] = e;
        z += e;
        int blk = block_table[(size_t)b * max_blocks + t / bs];
        const uint16_t *vv = v_pool + (((size_t)blk * Hkv + h) * bs + (t % bs)) * D;
        for (int d = 0; d < D; ++d) out_row[d] += e * orc_bf16_to_double(vv[d]);
    }
    for (int d = 0; d < D; ++d) out_row[d] /= z;
}

/* Full attention. out: fp64 [B][N][Hq][D]. flags[b] (may be NULL) gets 1 when
 * sequence b has an invalid context or block id. Returns 0 on success. */
int orc_attention(int B, int N, int Hq, int Hkv, int D, int bs, int max_blocks, int num_blocks,
                  const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                  const int32_t *block_table, const int32_t *ctx_lens, const uint64_t *mask,
                  double *out, int32_t *flags)
{
    if (B < 0 || N < 1 || N > 64 || Hq < 1 || Hkv < 1 || Hq % Hkv || D < 1) return -2;
    int cmax = 1;
    for (int b = 0; b < B; ++b) if (ctx_lens[b] > cmax) cmax = ctx_lens[b];
    double *scratch = (double *)malloc(sizeof(double) * (size_t)cmax);
    if (!scratch) return -3;
    for (int b = 0; b < B; ++b) {
        int ok = seq_valid(N, bs, max_blocks, num_blocks, block_table, ctx_lens, b);
        for (int i = 0; i < N; ++i)
            for (int hq = 0; hq < Hq; ++hq) {
                double *o = out + (((size_t)b * N + i) * Hq + hq) * D;
                if (ok)
                    attention_row(N, Hq, Hkv, D, bs, max_blocks, q, k_pool, v_pool,
                                  block_table, ctx_lens, mask, b, i, hq, o, scratch);
                else
                    for (int d = 0; d < D; ++d) o[d] = 0.0;
            }
        if (flags) flags[b] = !ok;
    }
    free(scratch);
    return 0;
}

/* Selected rows only: rows[3*r .. 3*r+2] = (b, i, hq); out: fp64 [nrows][D]. */
int orc_attention_rows(int B, int N, int Hq, int Hkv, int D, int bs, int max_blocks, int num_blocks,
                       const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                       const int32_t *block_table, const int32_t *ctx_lens, const uint64_t *mask,
                       const int32_t *rows, int nrows, double *out)
{
    if (B < 0 || N < 1 || N > 64 || Hq < 1 || Hkv < 1 || Hq % Hkv || D < 1) return -2;
    int cmax = 1;
    for (int b = 0; b < B; ++b) if (ctx_lens[b] > cmax) cmax = ctx_lens[b];
    double *scratch = (double *)malloc(sizeof(double) * (size_t)cmax);
    if (!scratch) return -3;
    for (int r = 0; r < nrows; ++r) {
        int b = rows[3 * r], i = rows[3 * r + 1], hq = rows[3 * r + 2];
        double *o = out + (size_t)r * D;
        if (seq_valid(N, bs, max_blocks, num_blocks, block_table, ctx_lens, b))
            attention_row(N, Hq, Hkv, D, bs, max_blocks, q, k_pool, v_pool, block_table,
                          ctx_lens, mask, b, i, hq, o, scratch);
        else
            for (int d = 0; d < D; ++d) o[d] = 0.0;
    }
    free(scratch);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Cascade (shared-prefix) verify attention                                  */
/* ------------------------------------------------------------------------ */

/* Rollouts of one prompt share its KV pages: a shared prefix node is stored
 * once and every rollout that passes through it reads it (SRT review, "Core
 * idea" and "Tree-Structured KV Cache", node sharing). The operation is plain
 * verify attention over each member's whole context, where the first
 * prefix_lens[g] keys of every member of group g come from the pages of the
 * group's first member and the rest from the member's own block table row.
 *
 * Groups are consecutive: group g holds sequences [off[g], off[g+1]), with
 * off[0] = 0, off[G] = B, nondecreasing. A member is valid when prefix_lens[g]
 * is a non-negative multiple of bs, prefix_lens[g] <= ctx_len - N, and its
 * effective table row passes seq_valid. An invalid member gets zeros and flag 1.
 *
 * rows == NULL: out is fp64 [B][N][Hq][D] and flags [B] (may be NULL).
 * rows != NULL: rows[3r..3r+2] = (b, i, hq); out is fp64 [nrows][D]. */
int orc_cascade_attention(int B, int N, int Hq, int Hkv, int D, int bs, int max_blocks,
                          int num_blocks, int num_groups, const int32_t *group_offsets,
                          const int32_t *prefix_lens, const uint16_t *q, const uint16_t *k_pool,
                          const uint16_t *v_pool, const int32_t *block_table,
                          const int32_t *ctx_lens, const uint64_t *mask, const int32_t *rows,
                          int nrows, double *out, int32_t *flags)
{
    if (B < 0 || N < 1 || N > 64 || Hq < 1 || Hkv < 1 || Hq % Hkv || D < 1 || bs < 1) return -2;
    if (num_groups < 0 || group_offsets[0] != 0 || group_offsets[num_groups] != B) return -2;
    for (int g = 0; g < num_groups; ++g)
        if (group_offsets[g + 1] < group_offsets[g]) return -2;
    int32_t *eff = (int32_t *)malloc(sizeof(int32_t) * ((size_t)B * max_blocks + 1));
    int *ok = (int *)malloc(sizeof(int) * ((size_t)B + 1));
    int cmax = 1;
    for (int b = 0; b < B; ++b) if (ctx_lens[b] > cmax) cmax = ctx_lens[b];
    double *scratch = (double *)malloc(sizeof(double) * (size_t)cmax);
    if (!eff || !ok || !scratch) { free(eff); free(ok); free(scratch); return -3; }
    /* each member's effective page list: the group's prefix pages, then its own */
    for (int g = 0; g < num_groups; ++g) {
        const int first = group_offsets[g], P = prefix_lens[g];
        for (int b = group_offsets[g]; b < group_offsets[g + 1]; ++b) {
            const int pre_ok = P >= 0 && P % bs == 0 && P <= ctx_lens[b] - N;
            for (int j = 0; j < max_blocks; ++j) {
                const int from = (pre_ok && j < P / bs) ? first : b;
                eff[(size_t)b * max_blocks + j] = block_table[(size_t)from * max_blocks + j];
            }
            ok[b] = pre_ok && seq_valid(N, bs, max_blocks, num_blocks, eff, ctx_lens, b);
        }
    }
    if (!rows) {
        for (int b = 0; b < B; ++b) {
            for (int i = 0; i < N; ++i)
                for (int hq = 0; hq < Hq; ++hq) {
                    double *o = out + (((size_t)b * N + i) * Hq + hq) * D;
                    if (ok[b])
                        attention_row(N, Hq, Hkv, D, bs, max_blocks, q, k_pool, v_pool, eff,
                                      ctx_lens, mask, b, i, hq, o, scratch);
                    else
                        for (int d = 0; d < D; ++d) o[d] = 0.0;
                }
            if (flags) flags[b] = !ok[b];
        }
    } else {
        for (int r = 0; r < nrows; ++r) {
            const int b = rows[3 * r], i = rows[3 * r + 1], hq = rows[3 * r + 2];
            double *o = out + (size_t)r * D;
            if (ok[b])
                attention_row(N, Hq, Hkv, D, bs, max_blocks, q, k_pool, v_pool, eff, ctx_lens,
                              mask, b, i, hq, o, scratch);
            else
                for (int d = 0; d < D; ++d) o[d] = 0.0;
        }
    }
    free(eff);
    free(ok);
    free(scratch);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Accept / resample                                                         */
/* ------------------------------------------------------------------------ */

/* Target distribution of one row: p = softmax(l / T), fp64, for a row with
 * at least one finite logit and no NaN/+inf (checked by the caller). */
static void target_probs(const float *l, int V, double T, double *p)
{
    double mx = -INFINITY;
    for (int x = 0; x < V; ++x) {
        double v = (double)l[x];
        if (v > mx) mx = v;
    }
    double z = 0.0;
    for (int x = 0; x < V; ++x) {
        double e = exp(((double)l[x] - mx) / T);
        p[x] = e;
        z += e;
    }
    for (int x = 0; x < V; ++x) p[x] /= z;
}

/* argmax with the lowest index on exact ties; -1 when the row has NaN/+inf or no finite entry. */
static int row_argmax(const float *l, int V)
{
    int best = -1;
    float bv = -INFINITY;
    for (int x = 0; x < V; ++x) {
        float v = l[x];
        if (isnan(v) || v == INFINITY) return -1;
        if (best < 0 ? v > -INFINITY : v > bv) { best = x; bv = v; }
    }
    return best;
}

/* Smallest x with sum_{y<=x} w(y) > t (t absolute), else the last x with w(x) > 0. */
static int first_above(const double *w, int V, double t)
{
    double c = 0.0;
    for (int x = 0; x < V; ++x) {
        c += w[x];
        if (c > t) return x;
    }
    for (int x = V - 1; x >= 0; --x)
        if (w[x] > 0.0) return x;
    return V - 1;
}

/* Inverse CDF over unnormalised weights w >= 0: the smallest x with
 * sum_{y<=x} w(y) > u * sum(w); if rounding leaves none, the last x with
 * w(x) > 0. *gap gets the distance from u*sum(w) to the nearer end of x's
 * interval, divided by sum(w). */
static int inv_cdf(const double *w, int V, double u, double *gap)
{
    double total = 0.0;
    for (int x = 0; x < V; ++x) total += w[x];
    double t = u * total;
    double c = 0.0;
    for (int x = 0; x < V; ++x) {
        double prev = c;
        c += w[x];
        if (c > t) {
            double g1 = t - prev, g2 = c - t;
            *gap = (g1 < g2 ? g1 : g2) / total;
            return x;
        }
    }
    for (int x = V - 1; x >= 0; --x)
        if (w[x] > 0.0) { *gap = 0.0; return x; }
    *gap = 0.0;
    return V - 1;
}

/*
 * Verify-step accept for B sequences.
 *
 * Rows: logits row v (0 <= v < N) is the target's next-token distribution
 * after node v (row 0: after the last accepted token). Draft node c >= 1
 * carries token drafts[b][c-1], drawn from draft_probs[b][c-1]; its parent
 * node is parents[c] (parents == NULL means a chain: parents[c] = c-1).
 *
 * T > 0: at node v (starting at the root) the residual r starts as
 * p_v = softmax(l_v / T). Children c of v are tried in index order; with
 * u = U(seed; b, c, 0, 0) child c is accepted iff u * q_c(d_c) < r(d_c). On
 * acceptance the walk moves to c with r = p_c. On rejection
 * r <- max(0, r - q_c) / sum(max(0, r - q_c)) (or p_v if that sum is 0) and
 * the next child is tried. When no child is accepted (or v is a leaf) the
 * next token is InvCDF(r, U(seed; b, v, 1, 0)).
 * T == 0: the walk moves to the first child whose token is argmax l_v; the
 * next token is argmax l_v at the final node. Draft probabilities are unused.
 * A draft token outside [0, V) counts as a rejection and sets flag bit 2.
 * A sequence with a NaN or +inf logit, or a row with no finite logit, in any
 * of its N rows gets flag bit 0 and outputs accept_len 0, next_token 0.
 *
 * Outputs per sequence: accept_len (depth of the final node), accept_path
 * [B][N-1] (the accepted nodes, -1 after the end), next_token, and for
 * parity accounting tie_depth (depth of the node at which the first accept
 * test with |u - r(d)/q(d)| < 1e-5 happened, else -1), tie_draw (1 if the
 * final draw's gap < 1e-5 and no accept test was a near tie), draw_lo /
 * draw_hi (the tokens the draw picks at thresholds (u -/+ 1e-5) * sum(w):
 * every token a rounding of the threshold within that band can give) and flags
 * (bit 0: non-finite logits, bit 2: bad draft token).
 * Returns 0, or a negative value on bad arguments / allocation failure.
 */
int orc_accept(int B, int N, int V, const int32_t *parents, const float *logits,
               const float *draft_probs, const int32_t *drafts, double T, uint64_t seed,
               int32_t *accept_len, int32_t *accept_path, int32_t *next_token,
               int32_t *tie_depth, int32_t *tie_draw, int32_t *draw_lo, int32_t *draw_hi,
               int32_t *flags)
{
    if (B < 0 || N < 1 || N > 64 || V < 1 || T < 0.0) return -2;
    int *par = (int *)malloc(sizeof(int) * (size_t)N);
    double *r = (double *)malloc(sizeof(double) * (size_t)V);
    double *pv = (double *)malloc(sizeof(double) * (size_t)V);
    if (!par || !r || !pv) { free(par); free(r); free(pv); return -3; }
    par[0] = -1;
    for (int c = 1; c < N; ++c) {
        par[c] = parents ? parents[c] : c - 1;
        if (par[c] < 0 || par[c] >= c) { free(par); free(r); free(pv); return -2; }
    }
    for (int b = 0; b < B; ++b) {
        const float *lb = logits + (size_t)b * N * V;
        const float *qb = draft_probs + (size_t)b * (N - 1) * V;
        const int32_t *db = drafts + (size_t)b * (N - 1);
        int32_t *path = accept_path + (size_t)b * (N - 1);
        for (int k = 0; k < N - 1; ++k) path[k] = -1;
        int v = 0, depth = 0, flag = 0, tdepth = -1, tdraw = 0, tok = 0, dlo = 0, dhi = 0;
        for (int row = 0; row < N; ++row)
            if (row_argmax(lb + (size_t)row * V, V) < 0) flag |= 1;
        if (flag) goto done;

        if (T == 0.0) {
            for (;;) {
                int am = row_argmax(lb + (size_t)v * V, V);
                int moved = 0;
                for (int c = v + 1; c < N; ++c) {
                    if (par[c] != v) continue;
                    int d = db[c - 1];
                    if (d < 0 || d >= V) { flag |= 4; continue; }
                    if (d == am) { path[depth++] = c; v = c; moved = 1; break; }
                }
                if (!moved) { tok = am; break; }
            }
        } else {
            target_probs(lb + (size_t)v * V, V, T, pv);
            memcpy(r, pv, sizeof(double) * (size_t)V);
            for (;;) {
                int moved = 0;
                for (int c = v + 1; c < N; ++c) {
                    if (par[c] != v) continue;
                    int d = db[c - 1];
                    const float *qc = qb + (size_t)(c - 1) * V;
                    int accept = 0;
                    if (d < 0 || d >= V) flag |= 4;
                    else {
                        double u = orc_uniform(seed, (uint32_t)b, (uint32_t)c, 0u, 0u);
                        double qd = (double)qc[d];
                        accept = (u * qd < r[d]);
                        if (tdepth < 0 && qd > 0.0 && fabs(u - r[d] / qd) < ORC_TIE_EPS) tdepth = depth;
                    }
                    if (accept) {
                        path[depth++] = c;
                        v = c;
                        moved = 1;
                        break;
                    }
                    double z = 0.0;
                    for (int x = 0; x < V; ++x) {
                        double w = r[x] - (double)qc[x];
                        r[x] = w > 0.0 ? w : 0.0;
                        z += r[x];
                    }
                    if (z > 0.0) for (int x = 0; x < V; ++x) r[x] /= z;
                    else memcpy(r, pv, sizeof(double) * (size_t)V);
                }
                if (!moved) break;
                target_probs(lb + (size_t)v * V, V, T, pv);
                memcpy(r, pv, sizeof(double) * (size_t)V);
            }
            double gap;
            double u = orc_uniform(seed, (uint32_t)b, (uint32_t)v, 1u, 0u);
            tok = inv_cdf(r, V, u, &gap);
            if (tdepth < 0 && gap < ORC_TIE_EPS) tdraw = 1;
            double total = 0.0;
            for (int x = 0; x < V; ++x) total += r[x];
            dlo = first_above(r, V, (u - ORC_TIE_EPS) * total);
            dhi = first_above(r, V, (u + ORC_TIE_EPS) * total);
        }
    done:
        accept_len[b] = depth;
        next_token[b] = tok;
        if (tie_depth) tie_depth[b] = tdepth;
        if (tie_draw) tie_draw[b] = tdraw;
        if (draw_lo) draw_lo[b] = T == 0.0 ? tok : dlo;
        if (draw_hi) draw_hi[b] = T == 0.0 ? tok : dhi;
        if (flags) flags[b] = flag;
    }
    free(par); free(r); free(pv);
    return 0;
}

/* Inverse-CDF helper exposed for tests: returns the chosen index, *gap as above. */
int orc_inv_cdf(const double *w, int V, double u, double *gap)
{
    return inv_cdf(w, V, u, gap);
}

/* ------------------------------------------------------------------------ */
/* KV commit after accept                                                    */
/* ------------------------------------------------------------------------ */
/*
 * After verification the cache keeps the last accepted token's row (the tree
 * root, position C - N) and the accepted draft nodes; rejected drafts are
 * dropped (TLT reading notes, "1. RL and SD": results computed on top of a
 * rejected token are discarded; SRT review, "Speculative Rollout integration":
 * the accepted path of the verified tree continues the sequence). The
 * accepted nodes are compacted behind the root in path order:
 *   K/V at position C - N + path[k]  ->  position C - N + 1 + k,  k < a,
 *   new ctx_len = C - N + 1 + a,
 * for every layer and KV head. Positions past the new length keep whatever
 * they held. A chain's path is 1..a, so nothing moves.
 * A sequence is left untouched (new ctx_len = ctx_len) and flagged when
 * ctx_len is outside [N, max_blocks*bs] (bit 1), a page holding one of its N
 * new positions has a block id outside the pool (bit 3), or accept_len is
 * outside [0, N-1] or the path is not strictly increasing within [1, N-1]
 * (bit 5).
 * pools: num_layers (k, v) pairs of bf16 [num_blocks][Hkv][bs][D], in place.
 */
int orc_kv_commit(int B, int N, int Hkv, int D, int bs, int max_blocks, int num_blocks, int num_layers,
                  uint16_t *const *k_pools, uint16_t *const *v_pools, const int32_t *block_table,
                  const int32_t *ctx_lens, const int32_t *accept_len, const int32_t *accept_path,
                  int32_t *new_ctx_lens, int32_t *flags)
{
    if (B < 0 || N < 1 || N > 64 || Hkv < 1 || D < 1 || bs < 1 || num_layers < 0) return -2;
    uint16_t *row = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)D * 64);
    if (!row) return -3;
    for (int b = 0; b < B; ++b) {
        const int C = ctx_lens[b];
        int f = 0;
        if (C < N || C > max_blocks * bs) f |= 2;
        if (!f)
            for (int t = C - N; t < C; ++t) {
                const int blk = block_table[(size_t)b * max_blocks + t / bs];
                if (blk < 0 || blk >= num_blocks) { f |= 8; break; }
            }
        const int a = accept_len[b];
        if (a < 0 || a > N - 1) f |= 32;
        else
            for (int k = 0; k < a; ++k) {
                const int node = accept_path[(size_t)b * (N > 1 ? N - 1 : 1) + k];
                const int prev = k > 0 ? accept_path[(size_t)b * (N - 1) + k - 1] : 0;
                if (node < 1 || node > N - 1 || node <= prev) { f |= 32; break; }
            }
        flags[b] = f;
        if (f) { new_ctx_lens[b] = C; continue; }
        new_ctx_lens[b] = C - N + 1 + a;
        for (int l = 0; l < num_layers; ++l)
            for (int kv = 0; kv < 2; ++kv) {
                uint16_t *pool = kv ? v_pools[l] : k_pools[l];
                for (int h = 0; h < Hkv; ++h) {
                    /* gather every source row first, then write: a destination can be
                     * another move's source */
                    for (int k = 0; k < a; ++k) {
                        const int t = C - N + accept_path[(size_t)b * (N - 1) + k];
                        const int blk = block_table[(size_t)b * max_blocks + t / bs];
                        memcpy(row + (size_t)k * D, pool + (((size_t)blk * Hkv + h) * bs + t % bs) * D,
                               sizeof(uint16_t) * (size_t)D);
                    }
                    for (int k = 0; k < a; ++k) {
                        const int t = C - N + 1 + k;
                        const int blk = block_table[(size_t)b * max_blocks + t / bs];
                        memcpy(pool + (((size_t)blk * Hkv + h) * bs + t % bs) * D, row + (size_t)k * D,
                               sizeof(uint16_t) * (size_t)D);
                    }
                }
            }
    }
    free(row);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Weight-free drafts from earlier rollouts                                  */
/* ------------------------------------------------------------------------ */
/*
 * History drafts (History Tree PR: drafts taken from earlier rollouts' high
 * reward responses of the same prompt, with a global fallback; the SRT review's
 * tree cache looks a sequence's prefix up in earlier rollouts). For sequence b
 * the key is its last K tokens. A candidate is a response h and a position p
 * with history[h][p..p+K-1] == key and at least one token after the key. The
 * first pass considers responses of the sequence's group; when none matches,
 * a second pass considers every response. The chosen candidate has the
 * highest reward, then the lowest h, then the lowest p. Drafts are the up to
 * gamma tokens after the key (draft_len), padded with token 0; a sequence
 * shorter than K, or without a candidate, gets draft_len 0 and all padding.
 * When probs is given (vocab > 0) each of the gamma rows is one-hot at its
 * draft token.
 */
int orc_history_draft(int B, int H, int hstride, int sstride, int K, int gamma, int vocab,
                      const int32_t *htok, const int32_t *hlen, const float *hreward, const int32_t *hgroup,
                      const int32_t *stok, const int32_t *slen, const int32_t *sgroup,
                      int32_t *drafts, int32_t *draft_len, float *probs)
{
    if (B < 0 || H < 0 || K < 1 || gamma < 1 || vocab < 0) return -2;
    for (int b = 0; b < B; ++b) {
        int best_h = -1, best_p = -1;
        const int L = slen[b];
        if (L >= K) {
            const int32_t *key = stok + (size_t)b * sstride + (L - K);
            for (int pass = 0; pass < 2 && best_h < 0; ++pass)
                for (int h = 0; h < H; ++h) {
                    if (pass == 0 && hgroup[h] != sgroup[b]) continue;
                    for (int p = 0; p + K < hlen[h]; ++p) {
                        int eq = 1;
                        for (int i = 0; i < K && eq; ++i) eq = htok[(size_t)h * hstride + p + i] == key[i];
                        if (!eq) continue;
                        if (best_h < 0 || hreward[h] > hreward[best_h]) { best_h = h; best_p = p; }
                        break;  /* the lowest p of this response */
                    }
                }
        }
        int n = 0;
        for (int k = 0; k < gamma; ++k) {
            int t = 0;
            if (best_h >= 0 && best_p + K + k < hlen[best_h]) {
                t = htok[(size_t)best_h * hstride + best_p + K + k];
                ++n;
            }
            drafts[(size_t)b * gamma + k] = t;
        }
        draft_len[b] = n;
        if (probs && vocab > 0)
            for (int k = 0; k < gamma; ++k) {
                float *row = probs + ((size_t)b * gamma + k) * vocab;
                memset(row, 0, sizeof(float) * (size_t)vocab);
                const int t = drafts[(size_t)b * gamma + k];
                if (t >= 0 && t < vocab) row[t] = 1.f;
            }
    }
    return 0;
}
