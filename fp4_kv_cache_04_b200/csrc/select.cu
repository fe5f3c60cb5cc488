// Top-K selection and the Hierarchical Sparse Indexer pool.
//
// CSA2 section of the thecryptopost.io DeepSeek-V4.1-Flash article: a Full or Reindex
// layer "selects fresh Top-512 indices"; the decoder's Full layer also builds a
// candidate pool of up to 16,384 positions (2,048 blocks of 8) that later Reindex
// layers score instead of the whole context.  Tie rule (the pages give none): equal
// scores go to the lower column; results are ascending positions, -1 padded.
//
// One CTA per row: an MSB-first radix select over the monotone 32-bit key of each
// score (4 passes of 8 bits, shared-memory histograms) finds the k-th key exactly; a
// stable compaction in column order then emits every larger key and the lowest-column
// equal keys, so the output comes out ascending without a sort.
#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

namespace {

constexpr int SEL_THREADS = 512;
constexpr int SEL_WARPS = SEL_THREADS / 32;

// Exclusive prefix sum over the CTA (SEL_THREADS threads); `total` gets the sum.
__device__ int block_exclusive_scan(int v, int* s_warp, int& total) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int y = lane < SEL_WARPS ? s_warp[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int z = __shfl_up_sync(0xFFFFFFFFu, y, off);
            if (lane >= off) y += z;
        }
        if (lane < SEL_WARPS) s_warp[lane] = y;
    }
    __syncthreads();
    const int before = (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
    total = s_warp[SEL_WARPS - 1];
    __syncthreads();
    return before;
}

__device__ __forceinline__ int32_t map_column(int64_t i, const int32_t* pool, int64_t seq) {
    if (pool == nullptr) return static_cast<int32_t>(i);
    const int32_t blk = pool[seq * POOL_BLOCKS + (i >> 3)];
    return blk * POOL_BLOCK + static_cast<int32_t>(i & 7);
}

__global__ void __launch_bounds__(SEL_THREADS)
topk_rows_kernel(const float* __restrict__ scores, int64_t ld, int64_t n_cols, int k,
                 const int32_t* __restrict__ pool, int q_per_seq, int32_t* __restrict__ out) {
    __shared__ unsigned hist[256];
    __shared__ int s_warp[32];
    __shared__ unsigned s_digit, s_above, s_total;

    const int64_t row = blockIdx.x;
    const float* src = scores + row * ld;
    const int tid = threadIdx.x;

    unsigned prefix = 0u, mask = 0u;
    int remaining = k;
    bool take_all = false;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = tid; i < 256; i += SEL_THREADS) hist[i] = 0u;
        __syncthreads();
        for (int64_t i = tid; i < n_cols; i += SEL_THREADS) {
            const unsigned key = score_key(src[i]);
            if (key != 0u && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            // lane l owns bins 255-8l .. 248-8l (descending)
            const int lane = tid;
            unsigned part = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) part += hist[255 - 8 * lane - i];
            unsigned incl = part;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const unsigned y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (lane >= off) incl += y;
            }
            const unsigned excl = incl - part;
            if (lane == 31) s_total = incl;
            if (excl < static_cast<unsigned>(remaining) && static_cast<unsigned>(remaining) <= incl) {
                unsigned cum = excl;
                for (int i = 0; i < 8; ++i) {
                    const unsigned bin = 255 - 8 * lane - i;
                    if (cum + hist[bin] >= static_cast<unsigned>(remaining)) {
                        s_digit = bin;
                        s_above = cum;
                        break;
                    }
                    cum += hist[bin];
                }
            }
        }
        __syncthreads();
        if (pass == 0 && s_total <= static_cast<unsigned>(k)) {
            take_all = true;
            break;
        }
        remaining -= static_cast<int>(s_above);
        prefix |= s_digit << shift;
        mask |= 0xFFu << shift;
        __syncthreads();
    }

    const unsigned T = take_all ? 0u : prefix;       // select keys > T ...
    const int need_eq = take_all ? 0 : remaining;    // ... and this many keys == T

    const int64_t seg = ceil_div(n_cols, SEL_THREADS);
    const int64_t lo = min(static_cast<int64_t>(tid) * seg, n_cols);
    const int64_t hi = min(lo + seg, n_cols);
    int gt = 0, eq = 0;
    for (int64_t i = lo; i < hi; ++i) {
        const unsigned key = score_key(src[i]);
        gt += key > T;
        eq += (T != 0u && key == T);
    }
    int dummy;
    const int eq_before = block_exclusive_scan(eq, s_warp, dummy);
    const int take_eq = max(0, min(need_eq - eq_before, eq));
    int n_sel;
    int off = block_exclusive_scan(gt + take_eq, s_warp, n_sel);

    const int64_t seq = row / q_per_seq;
    int32_t* dst = out + row * k;
    int eq_seen = 0;
    for (int64_t i = lo; i < hi; ++i) {
        const unsigned key = score_key(src[i]);
        bool sel = key > T;
        if (T != 0u && key == T) {
            sel = eq_seen < take_eq;
            ++eq_seen;
        }
        if (sel) dst[off++] = map_column(i, pool, seq);
    }
    for (int i = n_sel + tid; i < k; i += SEL_THREADS) dst[i] = -1;
}

__global__ void block_max_kernel(const float* __restrict__ scores, int64_t ld,
                                 const int64_t* __restrict__ kv_offsets, int64_t max_n,
                                 float* __restrict__ bm, int64_t bm_ld) {
    const int b = blockIdx.y;
    const int64_t blk = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (blk >= bm_ld) return;
    const int64_t n_b = kv_offsets[b + 1] - kv_offsets[b];
    float m = -INFINITY;
    const float* src = scores + static_cast<int64_t>(b) * ld;
    for (int r = 0; r < POOL_BLOCK; ++r) {
        const int64_t pos = blk * POOL_BLOCK + r;
        if (pos < n_b && pos < max_n) m = fmaxf(m, src[pos]);
    }
    bm[static_cast<int64_t>(b) * bm_ld + blk] = m;
}

}  // namespace

csa2_status launch_topk_rows(const float* scores, int64_t ld, int64_t n_cols, int rows, int k,
                             const int32_t* pool_blocks, int q_per_seq, int32_t* idx_out,
                             cudaStream_t stream) {
    if (rows == 0) return CSA2_OK;
    topk_rows_kernel<<<rows, SEL_THREADS, 0, stream>>>(scores, ld, n_cols, k, pool_blocks,
                                                        q_per_seq, idx_out);
    return check_launch("topk_rows_kernel");
}

csa2_status launch_block_max(const float* scores, int64_t ld, const int64_t* kv_offsets, int batch,
                             int64_t max_n, float* bm, int64_t bm_ld, cudaStream_t stream) {
    dim3 grid(static_cast<unsigned>(ceil_div(bm_ld, 256)), static_cast<unsigned>(batch));
    block_max_kernel<<<grid, 256, 0, stream>>>(scores, ld, kv_offsets, max_n, bm, bm_ld);
    return check_launch("block_max_kernel");
}

}  // namespace csa2
