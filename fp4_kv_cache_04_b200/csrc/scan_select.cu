// Fused decode indexer: scan + chunk-local Top-512, then a per-sequence merge.
//
// CSA2 section of the thecryptopost.io DeepSeek-V4.1-Flash article: a Full layer scores
// the context with its indexer and selects fresh Top-512 indices; a Reindex layer
// rescores the Hierarchical Sparse Indexer's pool (2,048 blocks of 8) with its own
// indexer Q.  Score (the pages give no formula):
//     score(s) = kscale[s] * sum_h w[h] * ReLU(q[h] . e4m3(k8[s])).
//
// scan_select_kernel: one CTA per (chunk of candidate columns, sequence), warp-specialised
// on the tensor cores.  Warp 0 streams 128-row tiles of FP8 K (8 KB) with TMA into a
// 4-stage shared-memory ring (64-byte swizzle); warp 1 owns 32 TMEM columns and issues
// tcgen05.mma kind::f8f6f4 with M = 128 positions, N = 16 columns and K = 64, where the
// bf16 indexer query is split exactly into two E4M3 pieces per head under a per-head
// power-of-two scale (columns h and 4+h); warps 2-5 read each position's 8 accumulator
// columns back with tcgen05.ld, recombine the pieces, apply ReLU, the head weights and
// the row scale, and keep the scores in shared memory.  The MMA accumulates the exact
// FP8 products in fp32.  Every mbarrier wait is bounded (ERR_TIMEOUT, no hang).  The
// CTA then keeps its own Top-512 (every position of the sequence's Top-512 is in the
// Top-512 of its chunk) and writes 512 (score, position) candidates.  A Full layer
// that builds the pool also writes each 8-position block's max score.
//
// merge_select_kernel: one CTA per sequence selects the Top-512 of its chunks'
// candidates; candidates arrive in position order, so the stable selection writes the
// final indices ascending with no sort.
#include "common.cuh"
#include "kernels.cuh"
#include "select.cuh"
#include "tc.cuh"

namespace csa2 {

namespace {

constexpr int TC_THREADS = 192;            // warp 0: TMA, warp 1: MMA, warps 2-5: epilogue
constexpr int TC_STAGES = 4;               // shared-memory ring of K tiles
constexpr int TC_TILE = 128;               // positions per MMA (M)
constexpr int TC_N = 16;                   // MMA columns: 4 heads x 2 query pieces + 8 zero
constexpr int TC_TILE_BYTES = TC_TILE * IDX_DIM;
constexpr int MERGE_THREADS = 512;

struct __align__(1024) TcShared {
    uint8_t a[TC_STAGES][TC_TILE_BYTES];    // FP8 K tiles (64-byte swizzle), 1 KB aligned
    uint8_t b[TC_N * IDX_DIM];              // query pieces (64-byte swizzle)
    float score[SCAN_CHUNK];
    int32_t pool_blk[SCAN_CHUNK / POOL_BLOCK];
    SelectShared<TC_THREADS> sel;
    float wq[IDX_HEADS];                    // head weight times 2^-s_h
    int qsh[IDX_HEADS];                     // s_h
    uint64_t full[TC_STAGES], empty[TC_STAGES], tfull[2], tempty[2];
    uint32_t tmem;
};

__device__ __forceinline__ int64_t pool_pos(const TcShared& sm, int j, int64_t n_b) {
    const int32_t blk = sm.pool_blk[j >> 3];
    if (blk < 0) return -1;
    const int64_t pos = static_cast<int64_t>(blk) * POOL_BLOCK + (j & 7);
    return pos < n_b ? pos : -1;
}

template <bool POOL>
__device__ __forceinline__ int64_t chunk_pos(const TcShared& sm, int64_t col0, int j, int cnt, int64_t n_b) {
    if (j >= cnt) return -1;
    return POOL ? pool_pos(sm, j, n_b) : col0 + j;
}

template <bool POOL, bool WANT_BM>
__global__ void __launch_bounds__(TC_THREADS, 1)
scan_select_kernel(const __grid_constant__ CUtensorMap tmap, ScanSelectArgs a) {
    extern __shared__ uint8_t smem_raw[];
    TcShared& sm = *reinterpret_cast<TcShared*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const IndexParams& p = a.p;
    const int b = blockIdx.y;
    const int chunk = blockIdx.x;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    const int64_t seq_off = p.kv_offsets[b];
    const int64_t n_b = p.kv_offsets[b + 1] - seq_off;
    const int64_t n_cols = POOL ? POOL_POSITIONS : n_b;
    const int64_t col0 = static_cast<int64_t>(chunk) * a.chunk;
    const int cnt = static_cast<int>(max(static_cast<int64_t>(0),
                                         min(static_cast<int64_t>(a.chunk), n_cols - col0)));
    const int n_tiles = (cnt + TC_TILE - 1) / TC_TILE;

    if (POOL) {
        const int32_t* pool_b = p.pool_blocks + static_cast<int64_t>(b) * POOL_BLOCKS + (col0 >> 3);
        for (int i = tid; i < (cnt + 7) / 8; i += TC_THREADS) sm.pool_blk[i] = __ldg(pool_b + i);
    }
    // ---- query pieces: q_h * 2^s_h = p1 + p2/16 exactly (max|q_h| * 2^s_h in [128, 256));
    //      column h holds p1 of head h, column 4+h holds p2, columns 8..15 are zero.
    const uint16_t* qb = p.idx_q + static_cast<int64_t>(b) * IDX_HEADS * IDX_DIM;
    if (warp < IDX_HEADS) {
        const uint32_t two = *reinterpret_cast<const uint32_t*>(qb + warp * IDX_DIM + 2 * lane);
        float m = fmaxf(fabsf(__uint_as_float(two << 16)), fabsf(__uint_as_float(two & 0xFFFF0000u)));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
        if (lane == 0) {
            int ex = 0;
            frexpf(m, &ex);                               // m = f * 2^ex, f in [0.5, 1)
            const int sh = (m > 0.0f) ? 8 - ex : 0;
            sm.qsh[warp] = sh;
            sm.wq[warp] = ldexpf(p.idx_w[static_cast<int64_t>(b) * IDX_HEADS + warp], -sh);
        }
    }
    if (tid == 0) {
        for (int s = 0; s < TC_STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int j = 0; j < 2; ++j) {
            mbar_init(&sm.tfull[j], 1);
            mbar_init(&sm.tempty[j], 4);
        }
        mbar_fence_init();
    }
    if (warp == 1) tmem_alloc(&sm.tmem, 32);
    __syncthreads();
    for (int i = tid; i < TC_N * IDX_DIM; i += TC_THREADS) {
        const int n = i / IDX_DIM, k = i % IDX_DIM;
        uint32_t code = 0;
        if (n < 2 * IDX_HEADS) {
            const int h = n & 3;
            const float x = ldexpf(__uint_as_float(static_cast<uint32_t>(qb[h * IDX_DIM + k]) << 16), sm.qsh[h]);
            const uint32_t c1 = e4m3_encode_rne_sat(fabsf(x)) | (x < 0.0f ? 0x80u : 0u);
            code = c1;
            if (n >= IDX_HEADS) {
                const float r = x - e4m3_to_float(static_cast<uint8_t>(c1));   // exact
                code = e4m3_encode_rne_sat(fabsf(r) * 16.0f) | (r < 0.0f ? 0x80u : 0u);
            }
        }
        sm.b[sw64_offset(n, k)] = static_cast<uint8_t>(code);
    }
    fence_proxy_async_smem();                            // query pieces -> tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    unsigned* err = a.err;

    if (warp == 0 && lane == 0) {
        // ---- TMA producer: one 128-row K tile per stage
        int issued = 0;
        for (int it = 0; it < n_tiles; ++it) {
            const int s = it % TC_STAGES;
            if (!mbar_wait(&sm.empty[s], ((it / TC_STAGES) & 1) ^ 1, err)) break;
            mbar_arrive_expect_tx(&sm.full[s], TC_TILE_BYTES);
            if (POOL) {
#pragma unroll 1
                for (int j = 0; j < TC_TILE / POOL_BLOCK; ++j) {
                    const int jc = it * TC_TILE + j * POOL_BLOCK;
                    const int32_t blk = jc < cnt ? sm.pool_blk[jc >> 3] : -1;
                    const int64_t row = seq_off + (blk >= 0 && static_cast<int64_t>(blk) * POOL_BLOCK < n_b
                                                       ? static_cast<int64_t>(blk) * POOL_BLOCK : 0);
                    tma_load_2d(sm.a[s] + j * POOL_BLOCK * IDX_DIM, &tmap, 0, static_cast<int>(row), &sm.full[s]);
                }
            } else {
                tma_load_2d(sm.a[s], &tmap, 0, static_cast<int>(seq_off + col0 + it * TC_TILE), &sm.full[s]);
            }
            ++issued;
        }
        for (int it = max(0, issued - TC_STAGES); it < issued; ++it)   // copies landed
            mbar_wait(&sm.full[it % TC_STAGES], (it / TC_STAGES) & 1, err);
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer: D[buf] = K_tile * pieces^T over K = 64 (two K=32 steps)
        const uint32_t idesc = idesc_e4m3_f32(TC_TILE, TC_N);
        const uint64_t bdesc = umma_desc_sw64(smem_u32(sm.b));
        int done = 0;
        for (int it = 0; it < n_tiles; ++it) {
            const int s = it % TC_STAGES, buf = it & 1;
            if (!mbar_wait(&sm.full[s], (it / TC_STAGES) & 1, err)) break;
            if (!mbar_wait(&sm.tempty[buf], ((it >> 1) & 1) ^ 1, err)) break;
            tc_fence_after();
            const uint64_t adesc = umma_desc_sw64(smem_u32(sm.a[s]));
            const uint32_t d = tmem + buf * TC_N;
            mma_e4m3(d, adesc, bdesc, idesc, false);
            mma_e4m3(d, adesc + 2, bdesc + 2, idesc, true);          // +32 bytes of K
            mma_commit(&sm.empty[s]);
            mma_commit(&sm.tfull[buf]);
            ++done;
        }
        if (done > 0)                                    // every MMA has completed
            mbar_wait(&sm.tfull[(done - 1) & 1], ((done - 1) >> 1) & 1, err);
    } else if (warp >= 2) {
        // ---- epilogue: TMEM lanes 32*(warp%4) .. +31 = this thread's tile row
        const int q = warp & 3;
        const float* ksseq = p.idx_kscale + seq_off;
        const float w0 = sm.wq[0], w1 = sm.wq[1], w2 = sm.wq[2], w3 = sm.wq[3];
        int j = q * 32 + lane;
        int64_t pos = chunk_pos<POOL>(sm, col0, j, cnt, n_b);
        float ks = pos >= 0 ? __ldg(ksseq + pos) : 0.0f;
        for (int it = 0; it < n_tiles; ++it) {
            const int buf = it & 1;
            // prefetch the next tile's row scale while this tile's MMA runs
            const int jn = j + TC_TILE;
            const int64_t pos_n = it + 1 < n_tiles ? chunk_pos<POOL>(sm, col0, jn, cnt, n_b) : -1;
            const float ks_n = pos_n >= 0 ? __ldg(ksseq + pos_n) : 0.0f;
            if (!mbar_wait(&sm.tfull[buf], (it >> 1) & 1, err)) break;
            tc_fence_after();
            uint32_t v[8];
            tmem_ld8(tmem + (static_cast<uint32_t>(32 * q) << 16) + buf * TC_N, v);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.tempty[buf]);
            if (j < cnt) {
                float sc = -INFINITY;
                if (pos >= 0) {
                    const float d0 = __uint_as_float(v[0]) + 0.0625f * __uint_as_float(v[4]);
                    const float d1 = __uint_as_float(v[1]) + 0.0625f * __uint_as_float(v[5]);
                    const float d2 = __uint_as_float(v[2]) + 0.0625f * __uint_as_float(v[6]);
                    const float d3 = __uint_as_float(v[3]) + 0.0625f * __uint_as_float(v[7]);
                    sc = ks * (w0 * fmaxf(d0, 0.0f) + w1 * fmaxf(d1, 0.0f) +
                               w2 * fmaxf(d2, 0.0f) + w3 * fmaxf(d3, 0.0f));
                }
                sm.score[j] = sc;
            }
            j = jn;
            pos = pos_n;
            ks = ks_n;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 32);
    }

    if (WANT_BM) {                       // HSI block maxima of this chunk's positions
        float* bm_b = a.bm + static_cast<int64_t>(b) * a.bm_ld;
        for (int blk = tid; blk < (cnt + 7) / 8; blk += TC_THREADS) {
            float m = -INFINITY;
            for (int r = 8 * blk; r < min(8 * blk + 8, cnt); ++r) m = fmaxf(m, sm.score[r]);
            bm_b[(col0 >> 3) + blk] = m;
        }
    }

    // chunk-local Top-512 -> candidates (score, position), padded with (-inf, -1)
    const auto key_of = [&](int i) { return score_key(sm.score[i]); };
    unsigned T;
    int need_eq;
    radix_threshold<TC_THREADS>(key_of, cnt, TOPK, sm.sel, T, need_eq);
    const int64_t cbase = (static_cast<int64_t>(b) * a.n_chunks + chunk) * TOPK;
    float* cs = a.cand_s + cbase;
    int32_t* cp = a.cand_p + cbase;
    const int n_sel = stable_emit<TC_THREADS>(key_of, cnt, T, need_eq, sm.sel, [&](int i, int slot) {
        cs[slot] = sm.score[i];
        cp[slot] = static_cast<int32_t>(chunk_pos<POOL>(sm, col0, i, cnt, n_b));
    });
    for (int i = n_sel + tid; i < TOPK; i += TC_THREADS) {
        cs[i] = -INFINITY;
        cp[i] = -1;
    }
}

__global__ void __launch_bounds__(MERGE_THREADS)
merge_select_kernel(const float* __restrict__ cand_s, const int32_t* __restrict__ cand_p,
                    int n_cand, int32_t* __restrict__ out) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    auto& sh = *reinterpret_cast<GlobalSelectShared<MERGE_THREADS>*>(smem_raw);
    const int64_t r = blockIdx.x;
    const float* cs = cand_s + r * n_cand;
    const int32_t* cp = cand_p + r * n_cand;
    int32_t* dst = out + r * TOPK;
    const auto key_of = [&](int i) { return score_key(__ldg(cs + i)); };
    const int n_sel = global_select<MERGE_THREADS>(key_of, n_cand, TOPK, sh,
                                                   [&](int i, int slot) { dst[slot] = __ldg(cp + i); });
    for (int i = n_sel + threadIdx.x; i < TOPK; i += MERGE_THREADS) dst[i] = -1;
}

}  // namespace

csa2_status launch_scan_select(const ScanSelectArgs& a, const CUtensorMap& tmap, bool pool, bool want_bm,
                               cudaStream_t stream) {
    dim3 grid(static_cast<unsigned>(a.n_chunks), static_cast<unsigned>(a.p.batch));
    const int smem = static_cast<int>(sizeof(TcShared)) + 1024;     // + alignment slack
    const void* k = pool ? reinterpret_cast<const void*>(scan_select_kernel<true, false>)
                  : want_bm ? reinterpret_cast<const void*>(scan_select_kernel<false, true>)
                            : reinterpret_cast<const void*>(scan_select_kernel<false, false>);
    if (!opt_in_smem(k, smem)) return check_launch("scan_select_kernel smem attribute");
    if (pool) {
        scan_select_kernel<true, false><<<grid, TC_THREADS, smem, stream>>>(tmap, a);
    } else if (want_bm) {
        scan_select_kernel<false, true><<<grid, TC_THREADS, smem, stream>>>(tmap, a);
    } else {
        scan_select_kernel<false, false><<<grid, TC_THREADS, smem, stream>>>(tmap, a);
    }
    return check_launch("scan_select_kernel");
}

csa2_status launch_merge_select(const float* cand_s, const int32_t* cand_p, int n_cand, int rows,
                                int32_t* out, cudaStream_t stream) {
    const int smem = static_cast<int>(sizeof(GlobalSelectShared<MERGE_THREADS>));
    if (!opt_in_smem(reinterpret_cast<const void*>(merge_select_kernel), smem))
        return check_launch("merge_select_kernel smem attribute");
    merge_select_kernel<<<rows, MERGE_THREADS, smem, stream>>>(cand_s, cand_p, n_cand, out);
    return check_launch("merge_select_kernel");
}

}  // namespace csa2
