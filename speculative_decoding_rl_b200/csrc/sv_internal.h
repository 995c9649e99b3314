// Internal declarations shared by the libspecverify translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/specverify.h"

namespace sv {

// ----------------------------- accept ---------------------------------------
// The vocabulary is cut into slices of ACC_SLICE entries; every pass over a
// row is one CTA per (row, slice).
constexpr int ACC_SLICE = 8192;
constexpr int ACC_MAX_VOCAB = 1 << 22;

struct AcceptParams {
    const float *logits;
    const float *q;
    const int32_t *drafts;
    int32_t *accept_len;
    int32_t *next_token;
    int32_t *accept_path;
    int32_t *status;
    int B, N, V, S;        // S = slices per row
    float log2e_over_T;    // log2(e) / T for T > 0
    int greedy;
    int vec;               // V % 4 == 0 and 16-byte aligned rows: 16-byte loads
    struct { uint32_t k0, k1; } key;
    int8_t parent[64];
    void *workspace;       // accept_workspace_bytes(B, N, V), 256-byte aligned
};

size_t accept_workspace_bytes(int B, int N, int V);
// Passes over rejected rows (each a pass kernel and a walk kernel) the walk
// can need for this tree: the largest number of rejections on the way to a
// node, plus that node's children (one pass for a node without children).
int accept_rounds(const int8_t *parent, int N);
// Launches the whole accept (stats, walk, then `rounds` pass + walk pairs;
// greedy: stats and walk only). Returns the number of kernels launched in *launches.
cudaError_t launch_accept(const AcceptParams &p, int rounds, cudaStream_t stream, int *launches);

// ----------------------------- attention ------------------------------------
// Keys per work tile: the split-context schedule hands out tiles of TILE_KEYS
// keys of one (sequence, KV head, row chunk) unit.
constexpr int TILE_KEYS = 128;
// The split-context schedule charges every unit UNIT_COST tiles on top of its
// own, for the fixed work of a unit's start and end (its query rows, the first
// tile's rescale, the read-out of O), so that CTAs that touch many units get
// fewer tiles. A unit occupies Tb + UNIT_COST positions of the schedule; the
// last UNIT_COST hold no work.
constexpr int UNIT_COST = 2;
constexpr int PAGE = 16;
constexpr int ROWS_MAX = 96;       // query rows (N*G) one unit carries
constexpr int MAX_SEQS = 512;

struct AttnParams {
    const uint16_t *q;         // bf16 bits [B][N][Hq][D]
    const uint16_t *k_pool;    // bf16 bits [num_blocks][Hkv][16][D]
    const uint16_t *v_pool;
    const int32_t *block_table;
    const int32_t *ctx_lens;
    const uint64_t *mask;      // [B][N] or null
    uint16_t *out;             // bf16 bits [B][N][Hq][D]
    int32_t *status;           // [B] or null
    float *ws_partial;         // partial slots (see slot_stride)
    int B, N, Hq, Hkv, D, G, R, RC, rows_unit, max_blocks, num_blocks;
    int units;                 // B * Hkv * RC
    int num_ctas;
    float scale_log2;          // log2(e) / sqrt(D)
    // Cascade call: every unit leaves its partial in a slot and no combine
    // kernel runs; the shared-prefix kernel that follows merges each row.
    int all_slots;
    // Bound of every device-side wait (2 s). Test hooks shorten it, and with
    // stall set make one wait per CTA run out (see sv_testing_*).
    uint64_t wait_limit_ns;
    int stall;
};

size_t attention_workspace_bytes(int B, int N, int Hq, int Hkv, int D, int num_ctas);
#ifdef __CUDACC__
// Floats per workspace partial slot: O [rows][D], running max [rows], row sum
// [rows], padded to 256 bytes so every slot (and every O row) is 16-byte aligned.
// The partial of a unit's k-th CTA segment is slot unit + (first CTA) + k.
__host__ __device__ inline size_t slot_stride(int rows_unit, int D) {
    return ((size_t)rows_unit * D + 2 * (size_t)rows_unit + 63) & ~(size_t)63;
}
#endif
// TMA map of a K or V pool [num_blocks][Hkv][16][D]: boxes of 16 keys x 64 dims,
// 128-byte swizzled (whole_page: 16 keys x D, unswizzled). A block id of
// num_blocks addresses past the pool and loads zeros.
bool encode_pool_map(CUtensorMap *m, const void *pool, int num_blocks, int Hkv, int D, bool whole_page = false);
// Row chunks of a unit: rows_unit rows (i, g) per chunk, RC chunks, Nc whole query rows i per chunk.
void row_chunks(int N, int G, int *rows_unit, int *RC, int *Nc);
int attention_num_ctas();
cudaError_t launch_attention(const AttnParams &p, cudaStream_t stream);

// ------------------------------ cascade ------------------------------------
// Shared-prefix pass: one CTA of CASCADE_ROWS query rows per (group, KV head,
// row tile), CASCADE_KEYS keys per tile.
constexpr int CASCADE_ROWS = 128;
constexpr int CASCADE_KEYS = 128;

struct CascadePlan {
    int num_groups, items;
    int off[SV_CASCADE_MAX_GROUPS + 1];    // group member offsets
    int pre[SV_CASCADE_MAX_GROUPS];        // shared keys per group
    int item0[SV_CASCADE_MAX_GROUPS + 1];  // first work item of each group
};

// Work items of a validated cascade descriptor.
void cascade_plan(const sv_cascade_desc *cd, int N, int Hq, int Hkv, CascadePlan *plan);
// Workspace: the attention slots, then suffix lengths, prefix flags and the
// suffix block table, each 256-byte aligned.
struct CascadeWorkspace {
    size_t slots, sfx_ctx, pflag, sfx_table, total;
};
CascadeWorkspace cascade_workspace(int B, int N, int Hq, int Hkv, int D, int max_blocks, int num_ctas);
// p describes the whole call with the caller's block table and lengths; p's
// workspace pointer is the base of a CascadeWorkspace.
cudaError_t launch_cascade(const AttnParams &p, const CascadePlan &plan, cudaStream_t stream);

// ------------------------------- kv commit ----------------------------------
struct CommitLaunch {
    const int32_t *block_table, *ctx_lens, *accept_len, *accept_path;
    int32_t *new_ctx, *status;
    int B, N, Hkv, D, max_blocks, num_blocks, L;
    uint16_t *k[SV_COMMIT_MAX_LAYERS];
    uint16_t *v[SV_COMMIT_MAX_LAYERS];
};
cudaError_t launch_kv_commit(const CommitLaunch &c, cudaStream_t stream);

// ---------------------------- history drafts --------------------------------
struct HistoryLaunch {
    const int32_t *htok, *hlen, *hgroup, *stok, *slen, *sgroup;
    const float *hreward;
    int32_t *drafts, *dlen;
    float *probs;
    int B, H, hstride, sstride, K, gamma, V;
};
cudaError_t launch_history_draft(const HistoryLaunch &h, cudaStream_t stream);

// Sets the text sv_last_error() returns on the calling thread.
void record_error(const char *msg);

// sv_verify_attention with its wait bound and the stall test hook exposed.
sv_status verify_attention_entry(const sv_attn_desc *d, const void *q, const sv_paged_kv *kv,
                                 const int32_t *block_table, const int32_t *ctx_lens,
                                 const uint64_t *draft_mask, void *out, void *workspace,
                                 size_t workspace_bytes, int32_t *status_flags, void *stream,
                                 uint64_t wait_limit_ns, int stall);

}  // namespace sv
