// Top-K selection over score rows and the Hierarchical Sparse Indexer pool.
//
// CSA2 section of the thecryptopost.io DeepSeek-V4.1-Flash article: a Full or Reindex
// layer picks a new set of 512 indices; the decoder's Full layer also builds a
// candidate pool of up to 16,384 positions (2,048 blocks of 8) that later Reindex layers
// score instead of the whole context.  Block score (the pages give none): the max of
// the block's position scores.  Ties go to the lower column; results are ascending
// positions, -1 padded.
//
// One CTA per row runs the shared radix select (select.cuh) over the row read from
// global memory (L2-resident after the producing kernel) and emits in column order.
#include "common.cuh"
#include "kernels.cuh"
#include "select.cuh"

namespace csa2 {

namespace {

constexpr int SEL_THREADS = 1024;
constexpr int SEL_SMEM_KEYS = 32768;      // rows up to this long are staged in shared memory
constexpr int SEL_KPT = SEL_SMEM_KEYS / SEL_THREADS;   // staged keys per thread
static_assert(sizeof(RegSelectShared<SEL_THREADS, SEL_KPT>) <= sizeof(GlobalSelectShared<SEL_THREADS>),
              "the register select's scratch fits the kernel's shared memory");
static_assert(sizeof(GlobalSelectShared<SEL_THREADS>) % 16 == 0, "staged keys start 16-byte aligned");

__global__ void __launch_bounds__(SEL_THREADS)
topk_rows_kernel(const float* __restrict__ scores, int64_t ld, int64_t n_cols, int k,
                 const int32_t* __restrict__ pool, int q_per_seq,
                 const int64_t* __restrict__ kv_offsets, int32_t* __restrict__ out) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    auto& sh = *reinterpret_cast<GlobalSelectShared<SEL_THREADS>*>(smem_raw);
    float* keys = reinterpret_cast<float*>(smem_raw + sizeof(GlobalSelectShared<SEL_THREADS>));
    const int64_t row = blockIdx.x;
    const float* src = scores + row * ld;
    const int64_t seq = row / q_per_seq;
    int64_t n = n_cols;
    if (kv_offsets != nullptr) {              // pool rows: the sequence's blocks only
        const int64_t n_b = kv_offsets[seq + 1] - kv_offsets[seq];
        n = min(n, ceil_div(n_b, POOL_BLOCK));
    }
    const int ni = static_cast<int>(n);
    int32_t* dst = out + row * k;
    const auto emit_pos = [&](int i, int slot) {
        if (pool == nullptr) {
            dst[slot] = i;
        } else {
            const int32_t blk = __ldg(pool + seq * POOL_BLOCKS + (i >> 3));
            dst[slot] = blk * POOL_BLOCK + (i & 7);
        }
    };
    const bool staged = ni <= SEL_SMEM_KEYS;
    if (staged) {                          // one batched load of the row into shared memory
        stage_floats<SEL_THREADS>(keys, src, ni);
        __syncthreads();
        // one exact select over the staged keys
        const auto key_at = [&](int u) {
            const int i = u * SEL_THREADS + static_cast<int>(threadIdx.x);
            return i < ni ? score_key(keys[i]) : 0u;
        };
        auto& rs = *reinterpret_cast<RegSelectShared<SEL_THREADS, SEL_KPT>*>(smem_raw);
        unsigned T;
        const int n_sel = reg_select<SEL_THREADS, SEL_KPT>(key_at, ni, k, 0u, rs, T, emit_pos);
        if (n_sel >= 0) {
            for (int i = n_sel + threadIdx.x; i < k; i += SEL_THREADS) dst[i] = -1;
            return;
        }
    }
    const auto key_of = [&](int i) { return score_key(staged ? keys[i] : __ldg(src + i)); };
    const int n_sel = global_select<SEL_THREADS>(key_of, ni, k, sh, emit_pos);
    for (int i = n_sel + threadIdx.x; i < k; i += SEL_THREADS) dst[i] = -1;
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
                             cudaStream_t stream, const int64_t* pool_kv_offsets) {
    if (rows == 0) return CSA2_OK;
    const int base = static_cast<int>(sizeof(GlobalSelectShared<SEL_THREADS>));
    const int smem = base + (n_cols <= SEL_SMEM_KEYS ? static_cast<int>(n_cols) * 4 : 0);
    if (!opt_in_smem(reinterpret_cast<const void*>(topk_rows_kernel), base + SEL_SMEM_KEYS * 4))
        return check_launch("topk_rows_kernel smem attribute");
    topk_rows_kernel<<<rows, SEL_THREADS, smem, stream>>>(scores, ld, n_cols, k, pool_blocks,
                                                           q_per_seq, pool_kv_offsets, idx_out);
    return check_launch("topk_rows_kernel");
}

csa2_status launch_block_max(const float* scores, int64_t ld, const int64_t* kv_offsets, int batch,
                             int64_t max_n, float* bm, int64_t bm_ld, cudaStream_t stream) {
    dim3 grid(static_cast<unsigned>(ceil_div(bm_ld, 256)), static_cast<unsigned>(batch));
    block_max_kernel<<<grid, 256, 0, stream>>>(scores, ld, kv_offsets, max_n, bm, bm_ld);
    return check_launch("block_max_kernel");
}

}  // namespace csa2
