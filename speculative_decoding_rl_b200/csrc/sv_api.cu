// C-ABI entry points of libspecverify: argument validation on the host, then
// asynchronous launches on the caller's stream. See include/specverify.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "sv_internal.h"

namespace {

thread_local char g_last_error[512] = "";

sv_status fail(sv_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// True when the byte ranges [a, a+na) and [b, b+nb) share a byte.
bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

sv_status check_attn_desc(const sv_attn_desc *d) {
    if (!d) return fail(SV_ERR_INVALID_ARG, "desc is NULL");
    if (d->num_seqs < 0) return fail(SV_ERR_INVALID_ARG, "num_seqs < 0");
    if (d->num_q_rows < 1 || d->num_q_rows > 64) return fail(SV_ERR_INVALID_ARG, "num_q_rows must be in [1, 64]");
    if (d->num_q_heads < 1 || d->num_kv_heads < 1 || d->num_q_heads % d->num_kv_heads)
        return fail(SV_ERR_INVALID_ARG, "num_q_heads must be a positive multiple of num_kv_heads");
    if (d->head_dim != 64 && d->head_dim != 128) return fail(SV_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
    if (d->block_size != sv::PAGE) return fail(SV_ERR_UNSUPPORTED, "block_size must be 16");
    if (d->max_blocks_per_seq < 1) return fail(SV_ERR_INVALID_ARG, "max_blocks_per_seq < 1");
    if (d->num_blocks < 1) return fail(SV_ERR_INVALID_ARG, "num_blocks < 1");
    if (d->num_seqs > sv::MAX_SEQS) return fail(SV_ERR_UNSUPPORTED, "num_seqs > 512");
    if (d->num_q_heads / d->num_kv_heads > sv::ROWS_MAX)
        return fail(SV_ERR_UNSUPPORTED, "more than 96 query heads per KV head");
    if ((long long)d->max_blocks_per_seq * sv::PAGE > (1LL << 30)) return fail(SV_ERR_UNSUPPORTED, "context too long");
    int ru, rc, nc;
    sv::row_chunks(d->num_q_rows, d->num_q_heads / d->num_kv_heads, &ru, &rc, &nc);
    const long long units = (long long)d->num_seqs * d->num_kv_heads * rc;
    if (units > 65535) return fail(SV_ERR_UNSUPPORTED, "num_seqs * num_kv_heads * row chunks above 65535");
    return SV_OK;
}

sv_status check_cascade_desc(const sv_attn_desc *d, const sv_cascade_desc *c) {
    if (!c) return fail(SV_ERR_INVALID_ARG, "cascade desc is NULL");
    if (c->num_groups < 1 || c->num_groups > SV_CASCADE_MAX_GROUPS)
        return fail(SV_ERR_INVALID_ARG, "num_groups must be in [1, %d]", SV_CASCADE_MAX_GROUPS);
    if (!c->group_offsets || !c->prefix_lens) return fail(SV_ERR_INVALID_ARG, "group_offsets or prefix_lens is NULL");
    if (c->group_offsets[0] != 0 || c->group_offsets[c->num_groups] != d->num_seqs)
        return fail(SV_ERR_INVALID_ARG, "group_offsets must run from 0 to num_seqs");
    for (int g = 0; g < c->num_groups; ++g) {
        if (c->group_offsets[g + 1] < c->group_offsets[g])
            return fail(SV_ERR_INVALID_ARG, "group_offsets must be nondecreasing");
        const int P = c->prefix_lens[g];
        if (P < 0 || P % sv::PAGE || (long long)P > (long long)d->max_blocks_per_seq * sv::PAGE)
            return fail(SV_ERR_INVALID_ARG, "prefix_lens[%d] must be a multiple of 16 in [0, max_blocks_per_seq*16]", g);
    }
    return SV_OK;
}

// Pointer checks shared by the plain and the cascade call.
sv_status check_attn_ptrs(const void *q, const sv_paged_kv *kv, const int32_t *block_table,
                          const int32_t *ctx_lens, const uint64_t *draft_mask, const void *out,
                          const int32_t *status_flags) {
    if (!q || !kv || !kv->k_pool || !kv->v_pool || !block_table || !ctx_lens || !out)
        return fail(SV_ERR_INVALID_ARG, "a required pointer is NULL");
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(kv->k_pool, 16) || !aligned(kv->v_pool, 16))
        return fail(SV_ERR_INVALID_ARG, "q, out and the KV pools must be 16-byte aligned");
    if (!aligned(block_table, 4) || !aligned(ctx_lens, 4) || (status_flags && !aligned(status_flags, 4)) ||
        (draft_mask && !aligned(draft_mask, 8)))
        return fail(SV_ERR_INVALID_ARG, "misaligned table, length, mask or status pointer");
    return SV_OK;
}

sv::AttnParams attn_params(const sv_attn_desc *d, const void *q, const sv_paged_kv *kv,
                           const int32_t *block_table, const int32_t *ctx_lens, const uint64_t *draft_mask,
                           void *out, void *workspace, int32_t *status_flags, int ctas) {
    sv::AttnParams p = {};
    p.q = static_cast<const uint16_t *>(q);
    p.k_pool = static_cast<const uint16_t *>(kv->k_pool);
    p.v_pool = static_cast<const uint16_t *>(kv->v_pool);
    p.block_table = block_table;
    p.ctx_lens = ctx_lens;
    p.mask = draft_mask;
    p.out = static_cast<uint16_t *>(out);
    p.status = status_flags;
    p.B = d->num_seqs;
    p.N = d->num_q_rows;
    p.Hq = d->num_q_heads;
    p.Hkv = d->num_kv_heads;
    p.D = d->head_dim;
    p.G = p.Hq / p.Hkv;
    p.R = p.N * p.G;
    int nc = 0;
    sv::row_chunks(p.N, p.G, &p.rows_unit, &p.RC, &nc);
    p.max_blocks = d->max_blocks_per_seq;
    p.num_blocks = d->num_blocks;
    p.units = p.B * p.Hkv * p.RC;
    p.num_ctas = ctas;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)p.D));
    p.ws_partial = static_cast<float *>(workspace);
    p.wait_limit_ns = 2000000000ull;
    p.stall = 0;
    p.all_slots = 0;
    return p;
}

}  // namespace

namespace sv {
void record_error(const char *msg) { snprintf(g_last_error, sizeof g_last_error, "%s", msg); }
}  // namespace sv

extern "C" {

const char *sv_status_string(sv_status s) {
    switch (s) {
        case SV_OK: return "SV_OK";
        case SV_ERR_INVALID_ARG: return "SV_ERR_INVALID_ARG";
        case SV_ERR_UNSUPPORTED: return "SV_ERR_UNSUPPORTED";
        case SV_ERR_CUDA: return "SV_ERR_CUDA";
        case SV_ERR_WORKSPACE: return "SV_ERR_WORKSPACE";
    }
    return "SV_ERR_UNKNOWN";
}

const char *sv_last_error(void) { return g_last_error; }

int32_t sv_version(void) { return 100; }

size_t sv_verify_attention_workspace_size(const sv_attn_desc *d) {
    if (check_attn_desc(d) != SV_OK) return 0;
    const int ctas = sv::attention_num_ctas();
    if (ctas <= 0) return 0;
    return sv::attention_workspace_bytes(d->num_seqs, d->num_q_rows, d->num_q_heads, d->num_kv_heads,
                                         d->head_dim, ctas);
}

sv_status sv_verify_attention(const sv_attn_desc *d, const void *q, const sv_paged_kv *kv,
                              const int32_t *block_table, const int32_t *ctx_lens,
                              const uint64_t *draft_mask, void *out, void *workspace,
                              size_t workspace_bytes, int32_t *status_flags, void *stream) {
    return sv::verify_attention_entry(d, q, kv, block_table, ctx_lens, draft_mask, out, workspace,
                                      workspace_bytes, status_flags, stream, 2000000000ull, 0);
}

}  // extern "C"

namespace sv {

sv_status verify_attention_entry(const sv_attn_desc *d, const void *q, const sv_paged_kv *kv,
                                 const int32_t *block_table, const int32_t *ctx_lens,
                                 const uint64_t *draft_mask, void *out, void *workspace,
                                 size_t workspace_bytes, int32_t *status_flags, void *stream,
                                 uint64_t wait_limit_ns, int stall) {
    sv_status s = check_attn_desc(d);
    if (s != SV_OK) return s;
    if (d->num_seqs == 0) return SV_OK;
    if ((s = check_attn_ptrs(q, kv, block_table, ctx_lens, draft_mask, out, status_flags)) != SV_OK) return s;
    const int ctas = sv::attention_num_ctas();
    if (ctas <= 0) return fail(SV_ERR_CUDA, "cannot query the current device");
    const size_t need = sv::attention_workspace_bytes(d->num_seqs, d->num_q_rows, d->num_q_heads,
                                                      d->num_kv_heads, d->head_dim, ctas);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
        return fail(SV_ERR_WORKSPACE, "workspace must be 256-byte aligned and hold %zu bytes", need);

    sv::AttnParams p =
        attn_params(d, q, kv, block_table, ctx_lens, draft_mask, out, workspace, status_flags, ctas);
    p.wait_limit_ns = wait_limit_ns;
    p.stall = stall;
    cudaError_t e = sv::launch_attention(p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(SV_ERR_CUDA, "attention launch: %s", cudaGetErrorString(e));
    return SV_OK;
}

}  // namespace sv

extern "C" {

size_t sv_cascade_attention_workspace_size(const sv_attn_desc *d, const sv_cascade_desc *c) {
    if (check_attn_desc(d) != SV_OK || check_cascade_desc(d, c) != SV_OK) return 0;
    const int ctas = sv::attention_num_ctas();
    if (ctas <= 0) return 0;
    return sv::cascade_workspace(d->num_seqs, d->num_q_rows, d->num_q_heads, d->num_kv_heads, d->head_dim,
                                 d->max_blocks_per_seq, ctas)
        .total;
}

sv_status sv_cascade_verify_attention(const sv_attn_desc *d, const sv_cascade_desc *c, const void *q,
                                      const sv_paged_kv *kv, const int32_t *block_table,
                                      const int32_t *ctx_lens, const uint64_t *draft_mask, void *out,
                                      void *workspace, size_t workspace_bytes, int32_t *status_flags,
                                      void *stream) {
    sv_status s = check_attn_desc(d);
    if (s != SV_OK) return s;
    if ((s = check_cascade_desc(d, c)) != SV_OK) return s;
    if (d->num_seqs == 0) return SV_OK;
    if ((s = check_attn_ptrs(q, kv, block_table, ctx_lens, draft_mask, out, status_flags)) != SV_OK) return s;
    const int ctas = sv::attention_num_ctas();
    if (ctas <= 0) return fail(SV_ERR_CUDA, "cannot query the current device");
    sv::CascadePlan plan;
    sv::cascade_plan(c, d->num_q_rows, d->num_q_heads, d->num_kv_heads, &plan);
    const size_t need = sv::cascade_workspace(d->num_seqs, d->num_q_rows, d->num_q_heads, d->num_kv_heads,
                                              d->head_dim, d->max_blocks_per_seq, ctas)
                            .total;
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
        return fail(SV_ERR_WORKSPACE, "workspace must be 256-byte aligned and hold %zu bytes", need);
    const sv::AttnParams p =
        attn_params(d, q, kv, block_table, ctx_lens, draft_mask, out, workspace, status_flags, ctas);
    cudaError_t e = sv::launch_cascade(p, plan, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(SV_ERR_CUDA, "cascade attention launch: %s", cudaGetErrorString(e));
    return SV_OK;
}

}  // extern "C"

namespace {

// Checks every argument of sv_accept that the workspace size depends on; fills p.
sv_status check_accept_desc(const sv_accept_desc *d, float temperature, sv::AcceptParams *p) {
    if (!d) return fail(SV_ERR_INVALID_ARG, "desc is NULL");
    if (d->num_seqs < 0) return fail(SV_ERR_INVALID_ARG, "num_seqs < 0");
    if (d->num_rows < 1 || d->num_rows > 64) return fail(SV_ERR_INVALID_ARG, "num_rows must be in [1, 64]");
    if (d->vocab < 1) return fail(SV_ERR_INVALID_ARG, "vocab < 1");
    if (d->vocab > sv::ACC_MAX_VOCAB) return fail(SV_ERR_UNSUPPORTED, "vocab above %d", sv::ACC_MAX_VOCAB);
    if (d->num_seqs > 65535) return fail(SV_ERR_UNSUPPORTED, "num_seqs above 65535");
    if (!(temperature >= 0.f) || isinf(temperature)) return fail(SV_ERR_INVALID_ARG, "temperature must be finite and >= 0");
    *p = sv::AcceptParams{};
    p->parent[0] = -1;
    for (int c = 1; c < d->num_rows; ++c) {
        const int par = d->tree_parents ? d->tree_parents[c] : c - 1;
        if (par < 0 || par >= c) return fail(SV_ERR_INVALID_ARG, "tree_parents[%d] = %d is not in [0, %d)", c, par, c);
        p->parent[c] = (int8_t)par;
    }
    if (d->tree_parents && d->tree_parents[0] != -1) return fail(SV_ERR_INVALID_ARG, "tree_parents[0] must be -1");
    p->B = d->num_seqs;
    p->N = d->num_rows;
    p->V = d->vocab;
    p->S = (d->vocab + sv::ACC_SLICE - 1) / sv::ACC_SLICE;
    return SV_OK;
}

}  // namespace

extern "C" {

size_t sv_accept_workspace_size(const sv_accept_desc *d) {
    sv::AcceptParams p;
    if (check_accept_desc(d, 1.f, &p) != SV_OK) return 0;
    return sv::accept_workspace_bytes(p.B, p.N, p.V);
}

sv_status sv_accept(const sv_accept_desc *d, const float *target_logits, const float *draft_probs,
                    const int32_t *draft_tokens, float temperature, uint64_t philox_seed,
                    int32_t *accept_len, int32_t *next_token, int32_t *accept_path,
                    int32_t *status_flags, void *workspace, size_t workspace_bytes, void *stream) {
    sv::AcceptParams p;
    sv_status s = check_accept_desc(d, temperature, &p);
    if (s != SV_OK) return s;
    const bool greedy = temperature == 0.f;
    if (d->num_seqs == 0) return SV_OK;
    if (!target_logits || !accept_len || !next_token) return fail(SV_ERR_INVALID_ARG, "a required pointer is NULL");
    if (d->num_rows > 1 && !draft_tokens) return fail(SV_ERR_INVALID_ARG, "draft_tokens is NULL");
    if (d->num_rows > 1 && !greedy && !draft_probs) return fail(SV_ERR_INVALID_ARG, "draft_probs is NULL");
    if (!aligned(target_logits, 4) || (draft_probs && !aligned(draft_probs, 4)) ||
        (draft_tokens && !aligned(draft_tokens, 4)) || !aligned(accept_len, 4) || !aligned(next_token, 4) ||
        (accept_path && !aligned(accept_path, 4)) || (status_flags && !aligned(status_flags, 4)))
        return fail(SV_ERR_INVALID_ARG, "misaligned pointer");
    const size_t need = sv::accept_workspace_bytes(p.B, p.N, p.V);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
        return fail(SV_ERR_WORKSPACE, "workspace must be 256-byte aligned and hold %zu bytes", need);
    p.logits = target_logits;
    p.q = draft_probs;
    p.drafts = draft_tokens;
    p.accept_len = accept_len;
    p.next_token = next_token;
    p.accept_path = accept_path;
    p.status = status_flags;
    p.greedy = greedy ? 1 : 0;
    p.log2e_over_T = greedy ? 0.f : (float)(1.4426950408889634 / (double)temperature);
    p.key.k0 = (uint32_t)(philox_seed & 0xFFFFFFFFull);
    p.key.k1 = (uint32_t)(philox_seed >> 32);
    p.workspace = workspace;
    const int rounds = greedy ? 0 : sv::accept_rounds(p.parent, p.N);
    cudaError_t e = sv::launch_accept(p, rounds, static_cast<cudaStream_t>(stream), nullptr);
    if (e != cudaSuccess) return fail(SV_ERR_CUDA, "accept launch: %s", cudaGetErrorString(e));
    return SV_OK;
}

sv_status sv_kv_commit(const sv_attn_desc *d, int32_t num_layers, const sv_kv_layer *layers,
                       const int32_t *block_table, const int32_t *ctx_lens, const int32_t *accept_len,
                       const int32_t *accept_path, int32_t *new_ctx_lens, int32_t *status_flags, void *stream) {
    if (!d) return fail(SV_ERR_INVALID_ARG, "desc is NULL");
    if (d->num_seqs < 0) return fail(SV_ERR_INVALID_ARG, "num_seqs < 0");
    if (d->num_q_rows < 1 || d->num_q_rows > 64) return fail(SV_ERR_INVALID_ARG, "num_q_rows must be in [1, 64]");
    if (d->num_kv_heads < 1 || d->num_kv_heads > 65535) return fail(SV_ERR_INVALID_ARG, "num_kv_heads must be in [1, 65535]");
    if (d->head_dim < 8 || d->head_dim > 256 || d->head_dim % 8)
        return fail(SV_ERR_UNSUPPORTED, "head_dim must be a multiple of 8 in [8, 256]");
    if (d->block_size != sv::PAGE) return fail(SV_ERR_UNSUPPORTED, "block_size must be 16");
    if (d->max_blocks_per_seq < 1) return fail(SV_ERR_INVALID_ARG, "max_blocks_per_seq < 1");
    if (d->num_blocks < 1) return fail(SV_ERR_INVALID_ARG, "num_blocks < 1");
    if ((long long)d->max_blocks_per_seq * sv::PAGE > (1LL << 30)) return fail(SV_ERR_UNSUPPORTED, "context too long");
    if (num_layers < 1 || num_layers > SV_COMMIT_MAX_LAYERS)
        return fail(SV_ERR_INVALID_ARG, "num_layers must be in [1, %d]", SV_COMMIT_MAX_LAYERS);
    if (!layers) return fail(SV_ERR_INVALID_ARG, "layers is NULL");
    for (int l = 0; l < num_layers; ++l)
        if (!layers[l].k_pool || !layers[l].v_pool || !aligned(layers[l].k_pool, 16) || !aligned(layers[l].v_pool, 16))
            return fail(SV_ERR_INVALID_ARG, "layer %d: pool NULL or not 16-byte aligned", l);
    if (d->num_seqs == 0) return SV_OK;
    if (!block_table || !ctx_lens || !accept_len || !new_ctx_lens)
        return fail(SV_ERR_INVALID_ARG, "a required pointer is NULL");
    if (d->num_q_rows > 1 && !accept_path) return fail(SV_ERR_INVALID_ARG, "accept_path is NULL");
    if (!aligned(block_table, 4) || !aligned(ctx_lens, 4) || !aligned(accept_len, 4) || !aligned(new_ctx_lens, 4) ||
        (accept_path && !aligned(accept_path, 4)) || (status_flags && !aligned(status_flags, 4)))
        return fail(SV_ERR_INVALID_ARG, "misaligned pointer");
    {
        // every CTA of a sequence reads its table row, length, accept length and
        // path while one of them writes the new length and the status: the
        // outputs must not alias any input (an in-place length update would let
        // late CTAs read the new length)
        const size_t B4 = (size_t)d->num_seqs * 4;
        const void *in[] = {block_table, ctx_lens, accept_len, accept_path};
        const size_t in_bytes[] = {B4 * (size_t)d->max_blocks_per_seq, B4, B4,
                                   B4 * (size_t)(d->num_q_rows > 1 ? d->num_q_rows - 1 : 1)};
        for (int i = 0; i < 4; ++i)
            if (overlaps(new_ctx_lens, B4, in[i], in_bytes[i]) || overlaps(status_flags, B4, in[i], in_bytes[i]))
                return fail(SV_ERR_INVALID_ARG, "new_ctx_lens and status_flags must not overlap an input array");
        if (overlaps(new_ctx_lens, B4, status_flags, B4))
            return fail(SV_ERR_INVALID_ARG, "new_ctx_lens and status_flags overlap");
    }
    sv::CommitLaunch c;
    memset(&c, 0, sizeof c);
    c.block_table = block_table;
    c.ctx_lens = ctx_lens;
    c.accept_len = accept_len;
    c.accept_path = accept_path;
    c.new_ctx = new_ctx_lens;
    c.status = status_flags;
    c.B = d->num_seqs;
    c.N = d->num_q_rows;
    c.Hkv = d->num_kv_heads;
    c.D = d->head_dim;
    c.max_blocks = d->max_blocks_per_seq;
    c.num_blocks = d->num_blocks;
    c.L = num_layers;
    for (int l = 0; l < num_layers; ++l) {
        c.k[l] = static_cast<uint16_t *>(layers[l].k_pool);
        c.v[l] = static_cast<uint16_t *>(layers[l].v_pool);
    }
    cudaError_t e = sv::launch_kv_commit(c, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(SV_ERR_CUDA, "kv commit launch: %s", cudaGetErrorString(e));
    return SV_OK;
}

sv_status sv_history_draft(const sv_history_desc *d, const int32_t *history_tokens, const int32_t *history_lens,
                           const float *history_reward, const int32_t *history_group, const int32_t *seq_tokens,
                           const int32_t *seq_lens, const int32_t *seq_group, int32_t *draft_tokens,
                           int32_t *draft_len, float *draft_probs, void *stream) {
    if (!d) return fail(SV_ERR_INVALID_ARG, "desc is NULL");
    if (d->num_seqs < 0 || d->num_history < 0) return fail(SV_ERR_INVALID_ARG, "negative count");
    if (d->key_len < 1 || d->key_len > 64) return fail(SV_ERR_INVALID_ARG, "key_len must be in [1, 64]");
    if (d->gamma < 1 || d->gamma > 63) return fail(SV_ERR_INVALID_ARG, "gamma must be in [1, 63]");
    if (d->history_stride < 1 || d->seq_stride < 1) return fail(SV_ERR_INVALID_ARG, "strides must be positive");
    if (d->vocab < 0) return fail(SV_ERR_INVALID_ARG, "vocab < 0");
    if (d->num_seqs == 0) return SV_OK;
    if (!seq_tokens || !seq_lens || !seq_group || !draft_tokens || !draft_len)
        return fail(SV_ERR_INVALID_ARG, "a required pointer is NULL");
    if (d->num_history > 0 && (!history_tokens || !history_lens || !history_reward || !history_group))
        return fail(SV_ERR_INVALID_ARG, "a history pointer is NULL");
    if (d->vocab > 0 && !draft_probs) return fail(SV_ERR_INVALID_ARG, "draft_probs is NULL with vocab > 0");
    const void *ptrs[] = {history_tokens, history_lens, history_reward, history_group, seq_tokens,
                          seq_lens, seq_group, draft_tokens, draft_len, draft_probs};
    for (const void *q : ptrs)
        if (q && !aligned(q, 4)) return fail(SV_ERR_INVALID_ARG, "misaligned pointer");
    if ((long long)d->num_history * d->history_stride > (1LL << 40)) return fail(SV_ERR_UNSUPPORTED, "history too large");
    sv::HistoryLaunch h;
    h.htok = history_tokens; h.hlen = history_lens; h.hgroup = history_group; h.hreward = history_reward;
    h.stok = seq_tokens; h.slen = seq_lens; h.sgroup = seq_group;
    h.drafts = draft_tokens; h.dlen = draft_len; h.probs = d->vocab > 0 ? draft_probs : nullptr;
    h.B = d->num_seqs; h.H = d->num_history; h.hstride = d->history_stride; h.sstride = d->seq_stride;
    h.K = d->key_len; h.gamma = d->gamma; h.V = d->vocab;
    cudaError_t e = sv::launch_history_draft(h, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(SV_ERR_CUDA, "history draft launch: %s", cudaGetErrorString(e));
    return SV_OK;
}

}  // extern "C"
