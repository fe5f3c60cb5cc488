// Indexer scan: scores every candidate position of a sequence for its indexer queries.
//
// The CSA2 section of the thecryptopost.io DeepSeek-V4.1-Flash article has a Full layer
// derive indexer K from the main KV and pick a new Top-512, and a Reindex layer score
// the same indexer K again with its own indexer Q (the decoder's Reindex layers
// only over the Hierarchical Sparse Indexer's pool).  The pages give no formula; the
// score computed here is
//     score(t, s) = kscale[s] * sum_h w[t,h] * ReLU( q[t,h] . e4m3(k8[s]) ),
// 4 heads x 64 dims, FP8 E4M3 K with one fp32 scale per row.
//
// Design (decode is a skinny GEMV: 64 FP8 bytes + 4 scale bytes per position against
// 4 heads): a warp covers 16 consecutive positions with two fully coalesced 512-byte
// loads, whose 16-byte chunks land exactly in the A fragments of four m16n8k16 f16
// tensor-core MMAs (the 64-wide dot product is permuted consistently in A and B, so a
// thread's contiguous 16 bytes serve all four k-slices).  E4M3 -> f16 is exact, bf16 q
// -> f16 is exact in the normal f16 range, and the MMA accumulates in fp32.  The
// 4 heads x 2 queries fill the n=8 columns.  The FP32-ALU alternative needs 256 FMA +
// 64 conversions per position, above the SM issue budget at HBM speed.
#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

namespace {

constexpr int SCAN_WARPS = 8;
constexpr int SCAN_TILES = 4;          // 16-position tiles per warp per iteration
constexpr int SCAN_COLS_PER_BLOCK = SCAN_WARPS * SCAN_TILES * 16;   // 512

// Sequence-local position of candidate column j (-1 = absent).
__device__ __forceinline__ int64_t column_position(const IndexParams& p, int b, int64_t j,
                                                   int64_t n_b) {
    if (p.pool_blocks == nullptr) return j < n_b ? j : -1;
    if (j >= POOL_POSITIONS) return -1;
    const int32_t blk = p.pool_blocks[static_cast<int64_t>(b) * POOL_BLOCKS + (j >> 3)];
    if (blk < 0) return -1;
    const int64_t pos = static_cast<int64_t>(blk) * POOL_BLOCK + (j & 7);
    return pos < n_b ? pos : -1;
}

// Loads the B fragments (indexer query, 4 slices x {b0, b1}) of column n = g of query
// pair `qp`: column n is query 2*qp + n/4, head n%4; the thread needs dims
// 16t .. 16t+15 of that head.
__device__ __forceinline__ void load_q_frags(const IndexParams& p, int b, int qp, int g, int t,
                                             uint32_t (&bq)[8]) {
    const int qi = 2 * qp + (g >> 2);
    if (qi >= p.q_per_seq) {
#pragma unroll
        for (int i = 0; i < 8; ++i) bq[i] = 0u;
        return;
    }
    const int64_t qrow = static_cast<int64_t>(b) * p.q_per_seq + qi;
    const uint16_t* src = p.idx_q + (qrow * IDX_HEADS + (g & 3)) * IDX_DIM + 16 * t;
    const uint4 v0 = *reinterpret_cast<const uint4*>(src);
    const uint4 v1 = *reinterpret_cast<const uint4*>(src + 8);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) bq[i] = bf16x2_to_f16x2(w[i]);
}

__global__ void __launch_bounds__(SCAN_WARPS * 32)
index_score_kernel(IndexParams p, float* __restrict__ scores, int64_t ld,
                   float* __restrict__ blockmax, int64_t bm_ld, int64_t n_cols) {
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;
    const int t = lane & 3;
    const int64_t seq_off = p.kv_offsets[b];
    const int64_t n_b = p.kv_offsets[b + 1] - seq_off;
    const int64_t col0 = static_cast<int64_t>(blockIdx.x) * SCAN_COLS_PER_BLOCK +
                         warp * (SCAN_TILES * 16);
    if (col0 >= n_cols) return;

    // A fragments: per tile, rows g and g+8, the thread's 16-byte chunk t of each row.
    uint4 ra[SCAN_TILES], rb[SCAN_TILES];
    int64_t pos_a[SCAN_TILES], pos_b[SCAN_TILES];
    float ks_a[SCAN_TILES], ks_b[SCAN_TILES];
#pragma unroll
    for (int u = 0; u < SCAN_TILES; ++u) {
        const int64_t ja = col0 + u * 16 + g;
        const int64_t jb = ja + 8;
        pos_a[u] = ja < n_cols ? column_position(p, b, ja, n_b) : -1;
        pos_b[u] = jb < n_cols ? column_position(p, b, jb, n_b) : -1;
        ra[u] = make_uint4(0, 0, 0, 0);
        rb[u] = make_uint4(0, 0, 0, 0);
        ks_a[u] = 0.0f;
        ks_b[u] = 0.0f;
        if (pos_a[u] >= 0) {
            ra[u] = ldg_stream(p.idx_k + (seq_off + pos_a[u]) * IDX_DIM + 16 * t);
            ks_a[u] = p.idx_kscale[seq_off + pos_a[u]];
        }
        if (pos_b[u] >= 0) {
            rb[u] = ldg_stream(p.idx_k + (seq_off + pos_b[u]) * IDX_DIM + 16 * t);
            ks_b[u] = p.idx_kscale[seq_off + pos_b[u]];
        }
    }
    // Convert to f16 A fragments: slice s uses word s of each chunk; its low byte pair
    // feeds a0/a1 and its high byte pair a2/a3.
    uint32_t fa[SCAN_TILES][4][4];
#pragma unroll
    for (int u = 0; u < SCAN_TILES; ++u) {
        const uint32_t wa[4] = {ra[u].x, ra[u].y, ra[u].z, ra[u].w};
        const uint32_t wb[4] = {rb[u].x, rb[u].y, rb[u].z, rb[u].w};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            fa[u][s][0] = e4m3x2_to_f16x2(static_cast<uint16_t>(wa[s] & 0xFFFFu));
            fa[u][s][1] = e4m3x2_to_f16x2(static_cast<uint16_t>(wb[s] & 0xFFFFu));
            fa[u][s][2] = e4m3x2_to_f16x2(static_cast<uint16_t>(wa[s] >> 16));
            fa[u][s][3] = e4m3x2_to_f16x2(static_cast<uint16_t>(wb[s] >> 16));
        }
    }

    const int n_pairs = (p.q_per_seq + 1) / 2;
    for (int qp = 0; qp < n_pairs; ++qp) {
        uint32_t bq[8];
        load_q_frags(p, b, qp, g, t, bq);
        // this thread's output columns: query qi = 2*qp + t/2, heads 2(t%2), 2(t%2)+1
        const int qi = 2 * qp + (t >> 1);
        const bool q_ok = qi < p.q_per_seq;
        const int64_t qrow = static_cast<int64_t>(b) * p.q_per_seq + (q_ok ? qi : 0);
        const float w0 = q_ok ? p.idx_w[qrow * IDX_HEADS + 2 * (t & 1)] : 0.0f;
        const float w1 = q_ok ? p.idx_w[qrow * IDX_HEADS + 2 * (t & 1) + 1] : 0.0f;
        int64_t vis = n_b;
        if (p.q_pos != nullptr && q_ok) {
            const int64_t tok = p.q_pos[b] + qi;
            vis = min(n_b, (tok + 1) / p.ratio);
            if (vis < 0) vis = 0;
        }
#pragma unroll
        for (int u = 0; u < SCAN_TILES; ++u) {
            float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int s = 0; s < 4; ++s) mma_16816(c, fa[u][s], bq[2 * s], bq[2 * s + 1]);
            float sa = w0 * fmaxf(c[0], 0.0f) + w1 * fmaxf(c[1], 0.0f);
            float sb = w0 * fmaxf(c[2], 0.0f) + w1 * fmaxf(c[3], 0.0f);
            sa += __shfl_xor_sync(0xFFFFFFFFu, sa, 1);
            sb += __shfl_xor_sync(0xFFFFFFFFu, sb, 1);
            sa = (pos_a[u] >= 0 && pos_a[u] < vis) ? ks_a[u] * sa : -INFINITY;
            sb = (pos_b[u] >= 0 && pos_b[u] < vis) ? ks_b[u] * sb : -INFINITY;
            const int64_t ja = col0 + u * 16 + g;
            if ((t & 1) == 0 && q_ok) {
                float* dst = scores + qrow * ld;
                if (ja < n_cols) dst[ja] = sa;
                if (ja + 8 < n_cols) dst[ja + 8] = sb;
            }
            if (blockmax != nullptr) {
                // decode only (one query): lanes with t == 0 hold query 0's scores of
                // rows g (block 2u) and g+8 (block 2u+1); reduce over g.
                float ma = sa, mb = sb;
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    ma = fmaxf(ma, __shfl_xor_sync(0xFFFFFFFFu, ma, off));
                    mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, off));
                }
                const int64_t blk = (col0 + u * 16) >> 3;
                if (lane == 0) {
                    float* bm = blockmax + static_cast<int64_t>(b) * bm_ld;
                    if (blk < bm_ld) bm[blk] = ma;
                    if (blk + 1 < bm_ld) bm[blk + 1] = mb;
                }
            }
        }
    }
}

}  // namespace

csa2_status launch_index_score(const IndexParams& p, float* scores, int64_t ld, float* blockmax,
                               int64_t bm_ld, cudaStream_t stream) {
    const int64_t n_cols = p.pool_blocks ? POOL_POSITIONS : p.max_n;
    if (n_cols <= 0) return CSA2_OK;
    dim3 grid(static_cast<unsigned>(ceil_div(n_cols, SCAN_COLS_PER_BLOCK)),
              static_cast<unsigned>(p.batch));
    index_score_kernel<<<grid, SCAN_WARPS * 32, 0, stream>>>(p, scores, ld, blockmax, bm_ld, n_cols);
    return check_launch("index_score_kernel");
}

}  // namespace csa2
