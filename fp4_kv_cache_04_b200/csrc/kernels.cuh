// Internal launcher interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

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
};

struct AttnParams {
    int batch;
    int q_per_seq;
    int ratio;
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
    unsigned* err;            // device error word (ERR_* bits)
};

csa2_status launch_quantize(const uint16_t* x, int64_t n_in, int ratio, const int64_t* dst_row,
                            uint8_t* codes, uint8_t* scales, cudaStream_t stream);

// Scores [rows][ld] (column j = position j, or pool slot j); optional per-sequence block
// maxima [B][bm_ld] (decode rows only).
csa2_status launch_index_score(const IndexParams& p, float* scores, int64_t ld, float* blockmax,
                               int64_t bm_ld, cudaStream_t stream);

// Top-k of each row of a score matrix, as ascending positions (-1 padded).
csa2_status launch_topk_rows(const float* scores, int64_t ld, int64_t n_cols, int rows, int k,
                             const int32_t* pool_blocks, int q_per_seq, int32_t* idx_out,
                             cudaStream_t stream);

// Block maxima of decode score rows: bm[b][blk] = max of positions 8blk..8blk+7 < N_b.
csa2_status launch_block_max(const float* scores, int64_t ld, const int64_t* kv_offsets, int batch,
                             int64_t max_n, float* bm, int64_t bm_ld, cudaStream_t stream);

csa2_status launch_attend(const AttnParams& p, cudaStream_t stream);

}  // namespace csa2
