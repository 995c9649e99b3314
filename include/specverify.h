/*
 * libspecverify -- the speculative-decoding verify step on one NVIDIA B200 (sm_100a).
 *
 * The verify step is the one target-model pass that scores all gamma+1 draft
 * positions of every active rollout at once and then keeps the longest
 * acceptable prefix (TLT reading notes, "1. RL and SD": the target scores
 * d1..dgamma in one pass; once d1 fails, the results for later positions are
 * discarded). Speculative decoding is used in RL rollouts because this step
 * is lossless: it leaves the target's output distribution unchanged
 * (Accelerating RL Post-Training Rollouts via System-Integrated Speculative
 * Decoding, Abstract). The library implements the two parts of the step that
 * touch every KV and logit byte:
 *
 *   sv_verify_attention  GQA attention of each sequence's N query rows (a
 *                        causal chain of gamma+1 positions, or 1+nodes of a
 *                        draft tree with per-row ancestor masks; SRT review,
 *                        "Speculative Rollout integration", step 5) over a
 *                        paged bf16 KV cache shared with the drafter
 *                        (EfficientRollout, "Key modules" 1).
 *   sv_accept            temperature softmax of the target logits, the accept
 *                        test of each draft, the walk to the longest accepted
 *                        path, and one token drawn from the residual
 *                        norm(max(0, p - q)) (or from p when every draft on
 *                        the path is accepted).
 *
 * Conventions for every call:
 *   - Tensor pointers are DEVICE pointers owned by the caller, unless a
 *     comment says host. Nothing is allocated, freed or retained by a call.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). Argument errors are detected on the host before any
 *     launch and returned as sv_status; nothing is launched then.
 *   - Data errors (bad context lengths, block ids, tokens, non-finite logits)
 *     are reported per sequence in `status_flags` (SV_FLAG_* bits), written by
 *     the kernels; read them after the stream is synchronised. Outputs of a
 *     flagged sequence are defined below but carry no meaning.
 *   - Calls that share a workspace must not overlap on the device.
 *   - The library never reads or writes memory outside the ranges described
 *     here; out-of-range block ids are never dereferenced.
 */
#ifndef SPECVERIFY_H
#define SPECVERIFY_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SV_API __attribute__((visibility("default")))
#else
#define SV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SV_OK = 0,
    SV_ERR_INVALID_ARG = 1,   /* NULL/unaligned pointer, bad size or shape */
    SV_ERR_UNSUPPORTED = 2,   /* valid request outside what the kernels handle */
    SV_ERR_CUDA = 3,          /* a CUDA runtime call failed (see sv_last_error) */
    SV_ERR_WORKSPACE = 4      /* workspace NULL or smaller than the size query */
} sv_status;

/* Per-sequence data-error bits written to status_flags[b]. */
#define SV_FLAG_NONFINITE   1  /* accept: a NaN or +inf logit, or a row without a finite logit */
#define SV_FLAG_BAD_CONTEXT 2  /* attention: ctx_len < N or ctx_len > max_blocks_per_seq*16 */
#define SV_FLAG_BAD_TOKEN   4  /* accept: a draft token outside [0, vocab) */
#define SV_FLAG_BAD_BLOCK   8  /* attention: a block id outside [0, num_blocks) */
#define SV_FLAG_TIMEOUT    16  /* attention: a bounded device-side wait gave up; outputs invalid */
#define SV_FLAG_BAD_PATH   32  /* kv commit: accept_len outside [0, N-1] or a path not strictly
                                  increasing within [1, N-1] */

/* ------------------------------------------------------------------------
 * Verify attention
 * ------------------------------------------------------------------------
 * Shapes (all row-major, contiguous):
 *   q            bf16  [B][N][Hq][D]       query rows, RoPE already applied
 *   k_pool/v_pool bf16 [num_blocks][Hkv][16][D]   paged KV pool (pages of 16 tokens)
 *   block_table  int32 [B][max_blocks_per_seq]    page ids of each sequence
 *   ctx_lens     int32 [B]                 keys of sequence b, INCLUDING its N new rows,
 *                                          whose K/V the caller has already written
 *   draft_mask   uint64 [B][N] or NULL     bit j of draft_mask[b][i]: row i sees new key j
 *                                          (new key j = position ctx_len-N+j); NULL = chain
 *                                          (row i sees new keys 0..i)
 *   out          bf16  [B][N][Hq][D]
 *   status_flags int32 [B] or NULL
 * Query head hq reads KV head hq / (Hq/Hkv). Every row sees all prefix keys
 * t < ctx_len - N. Scores are q.k / sqrt(D); out = softmax(scores) . V,
 * accumulated in fp32 (P is rounded to bf16 for the P.V tensor-core product).
 * Limits: 1 <= N <= 64, D in {64, 128}, block_size 16, Hq % Hkv == 0,
 * Hq/Hkv <= 96, B <= 512. q, out and the pools must be 16-byte aligned.
 * A sequence flagged SV_FLAG_BAD_CONTEXT gets out = 0; one flagged
 * SV_FLAG_BAD_BLOCK reads zeros for the bad pages. A row that sees no key
 * gets out = 0.
 * The work is split over the context across all SMs (tcgen05 tensor cores,
 * TMA page loads) and then combined in a second kernel; `workspace` holds the
 * per-split partials. Device-side waits are bounded: if one gives up, every
 * sequence of the call gets SV_FLAG_TIMEOUT.
 */
typedef struct {
    int32_t num_seqs;            /* B */
    int32_t num_q_rows;          /* N = gamma+1 (chain) or 1+nodes (tree) */
    int32_t num_q_heads;         /* Hq */
    int32_t num_kv_heads;        /* Hkv */
    int32_t head_dim;            /* D */
    int32_t block_size;          /* tokens per page; must be 16 */
    int32_t max_blocks_per_seq;  /* columns of block_table */
    int32_t num_blocks;          /* pages in each pool */
} sv_attn_desc;

typedef struct {
    const void *k_pool;          /* bf16 [num_blocks][Hkv][16][D] */
    const void *v_pool;          /* bf16 [num_blocks][Hkv][16][D] */
} sv_paged_kv;

/* Bytes of device workspace sv_verify_attention needs for `desc` on the
 * current device; 0 on an invalid desc. */
SV_API size_t sv_verify_attention_workspace_size(const sv_attn_desc *desc);

SV_API sv_status sv_verify_attention(const sv_attn_desc *desc, const void *q, const sv_paged_kv *paged_kv,
                              const int32_t *block_table, const int32_t *ctx_lens,
                              const uint64_t *draft_mask, void *out, void *workspace,
                              size_t workspace_bytes, int32_t *status_flags, void *stream);

/* ------------------------------------------------------------------------
 * Cascade verify attention (rollout groups that share a prompt's KV pages)
 * ------------------------------------------------------------------------
 * The rollouts of one prompt share its prefix, whose KV is stored once and
 * read by every rollout that passes through it (SRT review, "Core idea" and
 * "Tree-Structured KV Cache": node sharing; "Speculative Rollout
 * integration": shared-prefix KV reuse and fewer memory accesses as the
 * speed-up sources). This call returns what sv_verify_attention returns for
 * each member's whole context, except that the first prefix_lens[g] keys of
 * every member of group g are read from the pages of the group's FIRST member
 * (block_table row group_offsets[g]); the other members' first
 * prefix_lens[g]/16 table entries are not read. Those shared keys are read once
 * per group and KV head for all the group's query rows (a tensor-core pass over
 * the group's rows), the members' own keys by the split-context pass of
 * sv_verify_attention, and the two partial softmaxes are merged by log-sum-exp.
 *
 * cdesc and both of its arrays are HOST memory, read during the call:
 *   num_groups      1 .. SV_CASCADE_MAX_GROUPS
 *   group_offsets   int32 [num_groups + 1]: group g is sequences
 *                   [group_offsets[g], group_offsets[g+1]); group_offsets[0] = 0,
 *                   group_offsets[num_groups] = num_seqs, nondecreasing
 *   prefix_lens     int32 [num_groups]: shared keys of each group, a multiple
 *                   of 16 in [0, max_blocks_per_seq * 16]
 * When it pays: the plain call already reads a shared page once per member,
 * from L2 after the first member while the group's shared pages fit there, at
 * little cost; this call saves the DRAM traffic of shared pages that do not fit
 * (long prompts, many groups) and the tensor and softmax work of every member's
 * pass over them. Measured on one B200: 8 groups of 16 sharing 8192-token
 * prompts, 0.55 of the plain call's time; 4 groups of 16 sharing 1024-token
 * prompts under 2-12k tokens of their own, the same time as the plain call.
 * Every other argument, limit and error as sv_verify_attention, with the
 * workspace size from sv_cascade_attention_workspace_size. On the device, a
 * member whose context is invalid or shorter than prefix_lens[g] + N gets
 * SV_FLAG_BAD_CONTEXT and out = 0; a block id outside the pool among the
 * group's prefix pages gives every member SV_FLAG_BAD_BLOCK (zeros are read
 * for that page).
 */
#define SV_CASCADE_MAX_GROUPS 128
typedef struct {
    int32_t num_groups;
    const int32_t *group_offsets;  /* HOST [num_groups + 1] */
    const int32_t *prefix_lens;    /* HOST [num_groups] */
} sv_cascade_desc;

/* Bytes of device workspace sv_cascade_verify_attention needs; 0 on an invalid
 * desc or cdesc. */
SV_API size_t sv_cascade_attention_workspace_size(const sv_attn_desc *desc, const sv_cascade_desc *cdesc);

SV_API sv_status sv_cascade_verify_attention(const sv_attn_desc *desc, const sv_cascade_desc *cdesc,
                                             const void *q, const sv_paged_kv *paged_kv,
                                             const int32_t *block_table, const int32_t *ctx_lens,
                                             const uint64_t *draft_mask, void *out, void *workspace,
                                             size_t workspace_bytes, int32_t *status_flags, void *stream);

/* ------------------------------------------------------------------------
 * Accept / resample
 * ------------------------------------------------------------------------
 * Shapes:
 *   target_logits fp32 [B][N][V]   row v: target logits of the token after node v
 *                                  (row 0: after the last accepted token)
 *   draft_probs   fp32 [B][N-1][V] row c-1: distribution draft token c was drawn from
 *   draft_tokens  int32 [B][N-1]   token of draft node c at column c-1
 *   accept_len    int32 [B]        out: number of accepted drafts (depth of the final node)
 *   next_token    int32 [B]        out: the token emitted after the accepted path
 *   accept_path   int32 [B][N-1] or NULL   out: accepted node ids, then -1
 *   status_flags  int32 [B] or NULL        out: SV_FLAG_* bits
 *   workspace     device memory of sv_accept_workspace_size(desc) bytes, 256-byte
 *                 aligned; nothing in it needs clearing (every word is written
 *                 before it is read); calls sharing it must not overlap
 * tree_parents is a HOST array of N entries (tree_parents[0] = -1,
 * 0 <= tree_parents[c] < c), copied at the call; NULL = chain (parent c-1).
 *
 * Rule (temperature T > 0): p_v = softmax(l_v / T). The walk starts at the
 * root with residual r = p_0. Children c of the current node v are tried in
 * index order with u = U(seed; b, c, 0): accept iff u * q_c(d_c) < r(d_c)
 * (i.e. u < min(1, r/q)); accepting moves to c with r = p_c; rejecting sets
 * r = norm(max(0, r - q_c)) (p_v if that has no mass) and tries the next
 * child. When no child is accepted, next_token = InvCDF(r, U(seed; b, v, 1)).
 * For a chain this is: accept drafts while u_i < min(1, p_i/q_i), then draw
 * from norm(max(0, p - q)) at the first rejection, or from p after the last
 * draft. T == 0 (greedy): move to the first child whose token is argmax l_v
 * (lowest index on ties); next_token = argmax at the final node; draft_probs
 * is not read and may be NULL.
 * U(seed; b, c, tag) = (w0 >> 8) * 2^-24 where w0 is word 0 of
 * Philox4x32-10 with key {seed_lo32, seed_hi32} and counter {b, c, tag, 0}
 * (Salmon et al., SC'11). InvCDF(w, u) is the smallest x with
 * sum_{y<=x} w(y) > u * sum(w), else the last x with w(x) > 0.
 * Arithmetic is fp32: 2^x by the hardware approximation, divisions by a row's
 * or a residual's mass as products with its correctly rounded reciprocal, sums
 * in a fixed order, so a call's results depend only on its inputs and seed.
 * A sequence flagged SV_FLAG_NONFINITE gets
 * accept_len 0, next_token 0; a bad draft token counts as rejected.
 * The work is spread over every SM: one pass reads every logit once for the
 * row statistics, a per-sequence walk takes the decisions, and each rejection
 * (a chain has one, a tree at most its worst walk's count) costs one more pass
 * over that node's logit row and the rejected children's draft rows; the draw
 * re-reads one slice of 8192 entries. The kernels follow one another on
 * `stream` with no device-side wait of their own.
 * Limits: 1 <= N <= 64, 1 <= V <= 4194304, 0 <= B <= 65535.
 */
typedef struct {
    int32_t num_seqs;             /* B */
    int32_t num_rows;             /* N = drafts + 1 */
    int32_t vocab;                /* V */
    const int32_t *tree_parents;  /* HOST [N] or NULL (chain) */
} sv_accept_desc;

/* Bytes of device workspace sv_accept needs for `desc`; 0 on an invalid desc. */
SV_API size_t sv_accept_workspace_size(const sv_accept_desc *desc);

SV_API sv_status sv_accept(const sv_accept_desc *desc, const float *target_logits, const float *draft_probs,
                    const int32_t *draft_tokens, float temperature, uint64_t philox_seed,
                    int32_t *accept_len, int32_t *next_token, int32_t *accept_path,
                    int32_t *status_flags, void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------
 * KV commit after accept
 * ------------------------------------------------------------------------
 * After verification the cache keeps the row of the last accepted token (the
 * tree root, position ctx_len - N) and the accepted draft nodes, and drops the
 * rest: results computed on top of a rejected draft are discarded (TLT reading
 * notes, "1. RL and SD"), and the verified tree's accepted path continues the
 * sequence (SRT review, "Speculative Rollout integration"). The accepted
 * nodes are compacted behind the root in path order, in every layer and KV
 * head:
 *   K/V at position C - N + accept_path[b][k]  ->  position C - N + 1 + k,
 *   new_ctx_lens[b] = C - N + 1 + accept_len[b]          (C = ctx_lens[b]).
 * A chain's path is 1..a, so nothing moves and only the length changes.
 * Positions past the new length keep what they held and the block table is
 * not changed: pages past ceil(new_ctx_len / 16) are the caller's to reuse.
 *   desc          the attention descriptor of the verify call (num_q_heads is
 *                 unused; the pools' shape is [num_blocks][Hkv][16][D])
 *   layers        HOST array of num_layers {k_pool, v_pool} device pointers,
 *                 written in place; 1 <= num_layers <= SV_COMMIT_MAX_LAYERS
 *   block_table, ctx_lens   as for sv_verify_attention
 *   accept_len    int32 [B], accept_path int32 [B][N-1] (-1 padded), as
 *                 sv_accept returns them
 *   new_ctx_lens  int32 [B] out; status_flags int32 [B] or NULL
 * A sequence is left untouched (new_ctx_len = ctx_len) and flagged when its
 * ctx_len is outside [N, max_blocks*16] (SV_FLAG_BAD_CONTEXT), a page of its N
 * new positions has a block id outside the pool (SV_FLAG_BAD_BLOCK), or its
 * accept_len or path is malformed (SV_FLAG_BAD_PATH). Every source row is read
 * before any row is written, so overlapping moves are safe. Limits: D a
 * multiple of 8 up to 256, N <= 64. Pools 16-byte aligned.
 * new_ctx_lens and status_flags are written while the other CTAs of a
 * sequence still read the inputs, so neither may overlap block_table,
 * ctx_lens, accept_len, accept_path or each other (an in-place update of
 * ctx_lens is refused with SV_ERR_INVALID_ARG before any launch; use a
 * second buffer).
 * The pages have no interface for this step; its arguments follow the verify
 * and accept calls whose results it applies.
 */
#define SV_COMMIT_MAX_LAYERS 128
typedef struct {
    void *k_pool;                /* bf16 [num_blocks][Hkv][16][D], written in place */
    void *v_pool;
} sv_kv_layer;

SV_API sv_status sv_kv_commit(const sv_attn_desc *desc, int32_t num_layers, const sv_kv_layer *layers,
                              const int32_t *block_table, const int32_t *ctx_lens, const int32_t *accept_len,
                              const int32_t *accept_path, int32_t *new_ctx_lens, int32_t *status_flags,
                              void *stream);

/* ------------------------------------------------------------------------
 * Weight-free drafts from earlier responses
 * ------------------------------------------------------------------------
 * Chain drafts looked up in earlier rollouts' responses instead of drawn from
 * a draft model (History Tree PR: drafts from earlier high-reward responses of
 * the same prompt, with a global fallback; SRT review: prefix lookup in
 * earlier rollouts). For sequence b the key is its last key_len tokens. A
 * candidate is a response h and position p with history[h][p..p+key_len-1]
 * equal to the key and at least one token after it; candidates are first
 * sought among responses of the sequence's group, and among all responses if
 * none matched. The chosen one has the highest reward, then the lowest h, then
 * the lowest p. The drafts are the up to gamma tokens after it (draft_len),
 * padded with token 0; a sequence shorter than key_len or without a candidate
 * gets draft_len 0. With vocab > 0, draft_probs receives one-hot rows at the
 * draft tokens (padding included): a draft drawn from that q, as the accept
 * rule requires. Lengths are clamped to their rows' strides.
 *   history_tokens int32 [H][history_stride], history_lens [H],
 *   history_reward fp32 [H], history_group int32 [H]
 *   seq_tokens int32 [B][seq_stride], seq_lens [B], seq_group [B]
 *   draft_tokens int32 [B][gamma] out, draft_len int32 [B] out,
 *   draft_probs fp32 [B][gamma][vocab] out or NULL
 * Limits: 1 <= key_len <= 64, 1 <= gamma <= 63.
 */
typedef struct {
    int32_t num_seqs;            /* B */
    int32_t num_history;         /* H */
    int32_t history_stride;      /* columns of history_tokens */
    int32_t seq_stride;          /* columns of seq_tokens */
    int32_t key_len;             /* tokens matched */
    int32_t gamma;               /* drafts per sequence */
    int32_t vocab;               /* columns of draft_probs; 0 = no probabilities written */
} sv_history_desc;

SV_API sv_status sv_history_draft(const sv_history_desc *desc, const int32_t *history_tokens,
                                  const int32_t *history_lens, const float *history_reward,
                                  const int32_t *history_group, const int32_t *seq_tokens, const int32_t *seq_lens,
                                  const int32_t *seq_group, int32_t *draft_tokens, int32_t *draft_len,
                                  float *draft_probs, void *stream);

/* ------------------------------------------------------------------------
 * Host speculative-decoding controller
 * ------------------------------------------------------------------------
 * Host logic (no GPU work) that decides, for each decode step of a batch,
 * whether to speculate, how many drafts to verify and which drafter to use,
 * from costs measured with this library and the acceptance it observes:
 *  - elastic enable: no speculation while more than elastic_max_batch
 *    requests are active (TLT reading notes, "Elastic enable");
 *  - roofline toggle: speculate only when a verify step is expected to
 *    advance more tokens per millisecond than a plain decode step. The
 *    target's forward pass over T tokens costs max(weight bytes / HBM rate,
 *    T x flops per token / tensor rate) (memory-bound at small T, compute-bound
 *    at large T), plus the measured verify-path cost of the bucket
 *    (EfficientRollout, "System-aware SD toggle policy");
 *  - draft length, either acceptance-aware: the gamma maximising expected
 *    tokens per millisecond, sum_{k<=gamma} beta^k per sequence, under a
 *    running per-token acceptance estimate beta (EfficientRollout,
 *    "Acceptance-aware draft-length adaptation"); or BEG-MAB: per batch
 *    bucket, the draft length with the best median of accepted tokens per
 *    millisecond over a recent window, with occasional random exploration
 *    (TLT reading notes, "BEG-MAB");
 *  - drafter: timing_guard between a weight-free history drafter and a model
 *    drafter, per batch bucket, with the History Tree PR's defaults
 *    (sv_ctl_default_config) for EMA weight, switch margin, probe length,
 *    comparison delay and cooldown ("dynamic_rl default policy timing_guard").
 * The pages give no interface for this; the structures below carry what those
 * policies need. A controller object is not thread-safe.
 */
#define SV_CTL_GAMMA_ACCEPTANCE 0   /* draft length from the acceptance estimate */
#define SV_CTL_GAMMA_MAB        1   /* draft length from BEG-MAB per bucket */
#define SV_DRAFTER_NONE    0
#define SV_DRAFTER_HISTORY 1        /* weight-free drafts from earlier rollouts */
#define SV_DRAFTER_MODEL   2        /* a draft model (EAGLE-style head, small model) */
#define SV_CTL_MAX_BUCKETS 64
#define SV_CTL_MAX_GAMMA   63

typedef struct {
    /* target forward pass (roofline) */
    double target_weight_bytes;      /* bytes of target weights one forward pass reads */
    double target_flops_per_token;   /* ~2 x target parameters */
    double hbm_gbs;                  /* HBM GB/s */
    double tensor_tflops;            /* dense tensor TFLOP/s */
    double model_draft_ms;           /* model drafter: ms per drafted position (whole batch) */
    double history_draft_ms;         /* history drafter: ms per step (lookup) */
    /* verify-path cost measured with this library, per batch bucket */
    int32_t num_buckets;             /* 1..SV_CTL_MAX_BUCKETS */
    int32_t bucket_max_batch[SV_CTL_MAX_BUCKETS];   /* inclusive upper batch size, increasing */
    int32_t gamma_max;               /* draft lengths 1..gamma_max considered */
    const double *verify_ms;         /* HOST [num_buckets][gamma_max+1]: all layers' attention + accept at
                                        gamma drafts; index 0 = plain decode (one row per sequence) */
    /* policies */
    int32_t elastic_max_batch;       /* 0 = no limit */
    int32_t gamma_policy;            /* SV_CTL_GAMMA_* */
    double accept_prior;             /* initial per-token acceptance estimate, in (0, 1) */
    double accept_decay;             /* per-step decay of the acceptance counts, in [0, 1) */
    int32_t mab_window;              /* BEG-MAB: recent steps kept per (bucket, gamma) */
    double mab_explore;              /* BEG-MAB: probability of a random draft length */
    uint64_t seed;                   /* exploration random numbers */
    /* timing_guard */
    int32_t use_model_drafter;       /* 0: history drafter only */
    int32_t history_upper_batch;     /* history drafter only below this batch size */
    int32_t model_max_batch;         /* model drafter considered at batch <= this */
    int32_t model_probe_max_batch;   /* a probe of the model drafter starts only at batch <= this */
    int32_t history_warmup_records;  /* history records before the history cache counts as warm */
    int32_t model_cold_start_guard;  /* no model drafter before the history cache is warm */
    int32_t compare_after_steps;     /* history steps in a bucket before the model drafter is probed */
    int32_t model_probe_steps;       /* steps of one probe */
    double score_ema_alpha;          /* weight of a new tokens/ms sample in a branch's score */
    double switch_margin;            /* the model drafter needs score > history score x margin */
    int32_t cooldown_steps;          /* steps on history after a bad probe */
    int32_t max_cooldown_steps;
    double cooldown_growth;          /* cooldown multiplier after consecutive bad probes */
    double bad_step_ratio;           /* a model step below history score x ratio is a bad step */
} sv_ctl_config;

typedef struct {
    int32_t speculate;               /* 0: plain decode step */
    int32_t gamma;                   /* drafts per sequence (0 when not speculating) */
    int32_t drafter;                 /* SV_DRAFTER_* */
    int32_t bucket;                  /* batch bucket index */
    double expected_tokens_per_ms;   /* the model's estimate for the chosen step */
} sv_ctl_decision;

typedef struct {
    int32_t batch;                   /* sequences in the step */
    int32_t gamma;                   /* drafts per sequence verified (0: plain step) */
    int32_t drafter;                 /* SV_DRAFTER_* used */
    int64_t accepted_drafts;         /* sum of accept_len over the batch */
    int64_t rejections;              /* sequences whose accept_len < gamma */
    double step_ms;                  /* measured time of the whole step */
} sv_ctl_step;

typedef struct sv_ctl sv_ctl;

/* The History Tree PR's timing_guard defaults and neutral values for the rest. */
SV_API void sv_ctl_default_config(sv_ctl_config *config);
/* NULL with sv_last_error set on an invalid config; verify_ms is copied. */
SV_API sv_ctl *sv_ctl_create(const sv_ctl_config *config);
SV_API void sv_ctl_destroy(sv_ctl *ctl);
/* Decision for a step of `batch` active requests with `history_records`
 * records in the history drafter's cache. */
SV_API sv_status sv_ctl_decide(sv_ctl *ctl, int32_t batch, int32_t history_records, sv_ctl_decision *out);
/* Feed back a finished step (the decision it followed may differ: the caller decides). */
SV_API sv_status sv_ctl_observe(sv_ctl *ctl, const sv_ctl_step *step);
/* Current per-token acceptance estimate. */
SV_API double sv_ctl_acceptance(const sv_ctl *ctl);

/* ------------------------------------------------------------------------
 * Verify attention without a workspace argument
 * ------------------------------------------------------------------------
 * The source pages have no counterpart to this call; it exists for callers
 * that cannot allocate device memory (an engine or framework that owns every
 * device buffer and forbids allocation while it runs, a plugin handed only
 * its inputs and outputs, a host thread that must not call cudaMalloc because
 * it can synchronise the device). Same arguments and results as
 * sv_verify_attention minus the workspace: the split-context partials go to a
 * scratch array of SV_NOALLOC_SCRATCH_BYTES built into the library's device
 * image (every GPU that loads the library holds it until the process exits).
 * The call allocates nothing. A request whose workspace size
 * (sv_verify_attention_workspace_size) exceeds the scratch is refused with
 * SV_ERR_WORKSPACE before any launch.
 * The first call on a device looks up that device's scratch address; make it
 * before any stream capture (a lookup that fails returns SV_ERR_CUDA and is
 * retried by the next call). All calls on a device share the scratch, which
 * keeps the last call's contents (nothing in it needs clearing); calls whose
 * executions overlap on the GPU race on it and must be ordered by the caller.
 */
#define SV_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

SV_API sv_status sv_verify_attention_noalloc(const sv_attn_desc *desc, const void *q,
                                             const sv_paged_kv *paged_kv, const int32_t *block_table,
                                             const int32_t *ctx_lens, const uint64_t *draft_mask,
                                             void *out, int32_t *status_flags, void *stream);

/* Diagnostics. */
SV_API const char *sv_status_string(sv_status s);
SV_API const char *sv_last_error(void);   /* detail of the calling thread's last non-OK return */
SV_API int32_t sv_version(void);          /* major*10000 + minor*100 + patch */

#ifdef __cplusplus
}
#endif
#endif /* SPECVERIFY_H */
