// Internal declarations shared by the libspecverify translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/specverify.h"

namespace sv {

// ----------------------------- accept ---------------------------------------
constexpr int ACC_MAX_CHUNK_FLOATS = 55 * 1024;  // per-CTA vocabulary slice held in shared memory

struct PhiloxKeyHost { uint32_t k0, k1; };

struct AcceptParams {
    const float *logits;
    const float *q;
    const int32_t *drafts;
    int32_t *accept_len;
    int32_t *next_token;
    int32_t *accept_path;
    int32_t *status;
    int B, N, V, chunk;
    float log2e_over_T;   // log2(e) / T for T > 0
    int greedy;
    struct { uint32_t k0, k1; } key;
    int8_t parent[64];
};

int accept_max_vocab();
cudaError_t launch_accept(const AcceptParams &p, cudaStream_t stream);

// ----------------------------- attention ------------------------------------
// Keys per work tile: the split-context schedule hands out tiles of TILE_KEYS
// keys of one (sequence, KV head, row chunk) unit.
constexpr int TILE_KEYS = 128;
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
};

size_t attention_workspace_bytes(int B, int N, int Hq, int Hkv, int D, int num_ctas);
// Row chunks of a unit: rows_unit rows (i, g) per chunk, RC chunks, Nc whole query rows i per chunk.
void row_chunks(int N, int G, int *rows_unit, int *RC, int *Nc);
int attention_num_ctas();
cudaError_t launch_attention(const AttnParams &p, cudaStream_t stream);

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

}  // namespace sv
