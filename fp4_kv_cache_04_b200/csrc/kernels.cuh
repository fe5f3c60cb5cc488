// Internal launcher interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace csa2 {

struct IndexParams {
    int batch;
    int q_per_seq;
    int ratio;
    int64_t max_n;
    const int64_t* kv_offsets;
    const int64_t* q_pos;
    const uint16_t* idx_q;
    const float* idx_w;
    const uint8_t* idx_k;
    const float* idx_kscale;
    const int32_t* pool_blocks;
    RowMap rows;              // cache row of (sequence, position)
};

struct AttnParams {
    int batch;
    int q_per_seq;
    int ratio;
    int n_split;              // CTAs per query row (one cluster)
    int64_t swa_rows;
    float sm_scale;
    const int64_t* kv_offsets;
    const int64_t* q_pos;
    const uint8_t* codes;
    const uint8_t* scales;
    const int32_t* topk_idx;
    const uint16_t* q;
    const uint16_t* swa_kv;
    float* out;
    unsigned* err;            // device error word (ERR_* bits); word 1: the caller's wait bound
    int swa_fp8;              // SWA rows are E4M3 + per-row scale
    const uint8_t* swa_kv8;   // [B][swa_rows][512] E4M3 (swa_fp8)
    const float* swa_kscale;  // [B][swa_rows] (swa_fp8)
    RowMap rows;              // cache row of (sequence, position)
    int q_nvfp4;              // NVFP4 query variant (each head quantised in the kernel)
};

csa2_status launch_quantize(const uint16_t* x, int64_t n_in, int ratio, const int64_t* dst_row,
                            uint8_t* codes, uint8_t* scales, cudaStream_t stream);
csa2_status launch_append(const uint16_t* latent, const float* proj, int64_t n, const int64_t* dst_row,
                          uint8_t* codes, uint8_t* scales, uint8_t* idx_k, float* idx_kscale,
                          cudaStream_t stream);

// Scores [rows][ld] (column j = position j, or pool slot j); optional per-sequence block
// maxima [B][bm_ld] (decode rows only).
csa2_status launch_index_score(const IndexParams& p, float* scores, int64_t ld, float* blockmax,
                               int64_t bm_ld, cudaStream_t stream);

// Top-k of each row of a score matrix, as ascending positions (-1 padded).  With
// pool_kv_offsets (HSI pool selection over block maxima, one row per sequence) a row
// only considers its sequence's ceil(N_b/8) blocks.
csa2_status launch_topk_rows(const float* scores, int64_t ld, int64_t n_cols, int rows, int k,
                             const int32_t* pool_blocks, int q_per_seq, int32_t* idx_out,
                             cudaStream_t stream, const int64_t* pool_kv_offsets = nullptr);

// Fused decode indexer (one query per sequence, whole context visible).
constexpr int SCAN_CHUNK = 4096;          // max candidate columns per CTA (four CTAs per SM)
constexpr int REINDEX_CHUNK = 2816;       // pool columns per CTA: 6 per sequence, 384 CTAs at B = 64 (one wave)

struct ScanSelectArgs {
    IndexParams p;
    int chunk;                // candidate columns per CTA (multiple of 128, <= SCAN_CHUNK)
    int n_chunks;             // CTAs per sequence
    float* cand_s;            // [B][n_chunks][512]
    int32_t* cand_p;          // [B][n_chunks][512]
    float* bm;                // [B][bm_ld] block maxima (Full layer building the pool)
    int64_t bm_ld;
    unsigned* err;            // device error word (bounded waits)
    float* chunk_thr;         // [B][n_chunks] each chunk's 512th score (-inf if fewer)
    const float* pool_kscale; // Reindex over contiguous pool rows: [B][16384] scales (else null)
};

// The pool's indexer rows and scales gathered contiguously: pool_k [B][16384][64],
// pool_kscale [B][16384], slot j of sequence b = position 8 pool[b][j / 8] + j % 8.
csa2_status launch_pool_gather(const int32_t* pool_blocks, const int64_t* kv_offsets, int batch,
                               const uint8_t* idx_k, const float* idx_kscale, uint8_t* pool_k,
                               float* pool_kscale, RowMap rows, cudaStream_t stream);

// tmap: 2-D TMA map over idx_k as [total rows][64] bytes with the 64-byte swizzle; boxes
// of 128 rows (Full) or 8 rows (Reindex, one HSI block); with a.pool_kscale (Reindex over
// contiguous pool rows) a map over pool_k as [B * 16384][64], boxes of 128 rows.
csa2_status launch_scan_select(const ScanSelectArgs& a, const CUtensorMap& tmap, bool pool, bool want_bm,
                               cudaStream_t stream);
// Chunked-prefill Full indexer (many queries per sequence): scores and a streaming
// Top-512 per query in one kernel, no score matrix.  tmap: idx_k as for the decode scan,
// boxes of 128 rows.
csa2_status launch_prefill_index(const IndexParams& p, const CUtensorMap& tmap, int32_t* topk_out, unsigned* err,
                                 cudaStream_t stream);
csa2_status launch_merge_select(const float* cand_s, const int32_t* cand_p, const float* chunk_thr,
                                int n_chunks, int rows, int32_t* out, cudaStream_t stream);

// Block maxima of decode score rows: bm[b][blk] = max of positions 8blk..8blk+7 < N_b.
csa2_status launch_block_max(const float* scores, int64_t ld, const int64_t* kv_offsets, int batch,
                             int64_t max_n, float* bm, int64_t bm_ld, cudaStream_t stream);

// Attention of single query rows (decode rows, or prefill rows with their own causal
// Top-512 and 128-row SWA window): a row's key tiles (8 main tiles of 64 slots, then the
// SWA tiles of 32 bf16 / 64 E4M3 rows) dealt round robin over n_split CTAs (one cluster),
// two CTAs per SM; the row's CTAs merge their partials over distributed shared memory.
// tmap_q: q as [rows*16][512] bf16, boxes of 16 x 64, 128-byte swizzle.
// tmap_swa: swa_kv as [B][swa_rows][512] bf16, boxes of 1 x 32 x 64, 128-byte swizzle.
int attend_rows_swa_tiles(int64_t swa_rows, bool prefill, bool swa_fp8);
int attend_rows_split(int64_t rows, int swa_tiles, bool swa_fp8);
csa2_status launch_attend_rows(const AttnParams& p, const CUtensorMap& tmap_q, const CUtensorMap& tmap_swa,
                               cudaStream_t stream);

}  // namespace csa2
