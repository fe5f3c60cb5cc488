// Fused decode indexer: scan + chunk-local Top-512, then a per-sequence merge.
//
// CSA2 section of the thecryptopost.io DeepSeek-V4.1-Flash article: a Full layer scores
// the context with its indexer and selects fresh Top-512 indices; a Reindex layer
// rescores the Hierarchical Sparse Indexer's pool (2,048 blocks of 8) with its own
// indexer Q.  Score (the pages give no formula):
//     score(s) = kscale[s] * sum_h w[h] * ReLU(q[h] . e4m3(k8[s])).
//
// scan_select_kernel: one CTA per (chunk of candidate columns, sequence).  Warps take
// 16-column tiles (1 KB of FP8 K).  Each warp streams its tiles through a 4-stage
// cp.async ring in shared memory; every lane copies, and later reads back, exactly the
// two 16-byte pieces it needs, so the ring needs no barrier and keeps ~8 KB per warp in
// flight.  Those pieces are exactly the A fragments of four m16n8k16 MMAs (the 64-dim
// dot product is permuted identically in A and B); E4M3 -> f16 is exact and the
// tensor cores accumulate in fp32.  Scores stay in shared memory; the CTA then
// keeps its own Top-512 (every position of the sequence's Top-512 is in the Top-512 of
// its chunk) and writes 512 (score, position) candidates.  A Full layer that builds the
// pool also writes each 8-position block's max score.
//
// merge_select_kernel: one CTA per sequence selects the Top-512 of its chunks'
// candidates; candidates arrive in position order, so the stable selection writes the
// final indices ascending with no sort.
#include "common.cuh"
#include "kernels.cuh"
#include "select.cuh"

namespace csa2 {

namespace {

constexpr int SS_THREADS = 256;
constexpr int SS_WARPS = SS_THREADS / 32;
constexpr int STAGES = 4;                  // cp.async ring depth per warp
constexpr int TPS = 2;                     // 16-row tiles per warp per stage
constexpr int TILE_BYTES = 16 * IDX_DIM;   // one tile of FP8 K rows
constexpr int MERGE_THREADS = 512;

struct ScanShared {
    uint8_t ring[SS_WARPS][STAGES][TPS][TILE_BYTES];   // FP8 K tiles in flight
    float kring[SS_WARPS][STAGES][TPS][16];            // their row scales
    float score[SCAN_CHUNK];
    int32_t pool_blk[SCAN_CHUNK / POOL_BLOCK];
    SelectShared<SS_THREADS> sel;
};

// Sequence-local position of chunk column j (-1 = absent).
template <bool POOL>
__device__ __forceinline__ int64_t column_pos(const ScanShared& sm, int64_t col0, int j, int cnt,
                                              int64_t n_b) {
    if (j >= cnt) return -1;
    if (!POOL) return col0 + j;
    const int32_t blk = sm.pool_blk[j >> 3];
    if (blk < 0) return -1;
    const int64_t pos = static_cast<int64_t>(blk) * POOL_BLOCK + (j & 7);
    return pos < n_b ? pos : -1;
}

template <bool POOL, bool WANT_BM>
__global__ void __launch_bounds__(SS_THREADS, 2)
scan_select_kernel(ScanSelectArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    ScanShared& sm = *reinterpret_cast<ScanShared*>(smem_raw);
    const IndexParams& p = a.p;
    const int b = blockIdx.y;
    const int chunk = blockIdx.x;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;
    const int t = lane & 3;

    const int64_t seq_off = p.kv_offsets[b];
    const int64_t n_b = p.kv_offsets[b + 1] - seq_off;
    const int64_t n_cols = POOL ? POOL_POSITIONS : n_b;
    const int64_t col0 = static_cast<int64_t>(chunk) * a.chunk;
    const int cnt = static_cast<int>(max(static_cast<int64_t>(0),
                                         min(static_cast<int64_t>(a.chunk), n_cols - col0)));

    if (POOL) {
        const int32_t* pool_b = p.pool_blocks + static_cast<int64_t>(b) * POOL_BLOCKS + (col0 >> 3);
        for (int i = threadIdx.x; i < (cnt + 7) / 8; i += SS_THREADS) sm.pool_blk[i] = __ldg(pool_b + i);
        __syncthreads();
    }

    // B fragments.  The bf16 query is split exactly into two E4M3 pieces per head,
    // q_h * 2^s_h = p1 + p2 / 16, with 2^s_h putting max|q_h| in [128, 256); column
    // n = g of the MMA holds piece g/4 of head g%4.  Lane (g, t) builds the bytes of
    // dims 16t .. 16t+15 (the same permutation as the A fragments).
    uint32_t bq[4];
    float w0, w1;
    {
        const int h = g & 3;
        const uint16_t* src = p.idx_q + (static_cast<int64_t>(b) * IDX_HEADS + h) * IDX_DIM + 16 * t;
        const uint4 v0 = *reinterpret_cast<const uint4*>(src);
        const uint4 v1 = *reinterpret_cast<const uint4*>(src + 8);
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        float qv[16];
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            qv[2 * i] = __uint_as_float(w[i] << 16);
            qv[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            m = fmaxf(m, fmaxf(fabsf(qv[2 * i]), fabsf(qv[2 * i + 1])));
        }
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
        int ex = 0;
        frexpf(m, &ex);                                   // m = f * 2^ex, f in [0.5, 1)
        const int sh = (m > 0.0f) ? 8 - ex : 0;           // max|q| * 2^sh in [128, 256)
        uint32_t bytes[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float x = ldexpf(qv[i], sh);            // exact
            const uint32_t c1 = e4m3_encode_rne_sat(fabsf(x)) | (x < 0.0f ? 0x80u : 0u);
            uint32_t code = c1;
            if (g >= 4) {
                const float r = x - e4m3_to_float(static_cast<uint8_t>(c1));   // exact
                code = e4m3_encode_rne_sat(fabsf(r) * 16.0f) | (r < 0.0f ? 0x80u : 0u);
            }
            bytes[i >> 2] |= code << (8 * (i & 3));
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) bq[i] = bytes[i];
        // lanes t = 0, 1 own heads {0,1} / {2,3}: weights with the 2^-s of their heads
        const int sh0 = __shfl_sync(0xFFFFFFFFu, sh, 4 * ((2 * t) & 3));
        const int sh1 = __shfl_sync(0xFFFFFFFFu, sh, 4 * ((2 * t + 1) & 3));
        w0 = (t < 2) ? ldexpf(p.idx_w[static_cast<int64_t>(b) * IDX_HEADS + 2 * t], -sh0) : 0.0f;
        w1 = (t < 2) ? ldexpf(p.idx_w[static_cast<int64_t>(b) * IDX_HEADS + 2 * t + 1], -sh1) : 0.0f;
    }

    const uint8_t* kseq = p.idx_k + seq_off * IDX_DIM + 16 * t;
    const float* ksseq = p.idx_kscale + seq_off;
    float* bm_b = WANT_BM ? a.bm + static_cast<int64_t>(b) * a.bm_ld : nullptr;

    // this warp's tiles: warp, warp + 8, ...; stage i holds its tiles i*TPS .. i*TPS+TPS-1
    const int n_tiles = (cnt + 15) / 16;
    const int my_tiles = n_tiles > warp ? (n_tiles - warp + SS_WARPS - 1) / SS_WARPS : 0;
    const int n_stages = (my_tiles + TPS - 1) / TPS;

    const auto issue = [&](int i) {
        if (i < n_stages) {
            const int slot = i % STAGES;
#pragma unroll
            for (int u = 0; u < TPS; ++u) {
                const int tile = warp + SS_WARPS * (i * TPS + u);
                const int ra = tile * 16 + g, rb = ra + 8;
                const int64_t pa = column_pos<POOL>(sm, col0, ra, cnt, n_b);
                const int64_t pb = column_pos<POOL>(sm, col0, rb, cnt, n_b);
                uint8_t* dst = sm.ring[warp][slot][u];
                cp_async_16(smem_u32(dst + g * IDX_DIM + 16 * t), kseq + (pa >= 0 ? pa : 0) * IDX_DIM,
                            pa >= 0 ? 16 : 0);
                cp_async_16(smem_u32(dst + (g + 8) * IDX_DIM + 16 * t), kseq + (pb >= 0 ? pb : 0) * IDX_DIM,
                            pb >= 0 ? 16 : 0);
                if (t == 0) {
                    cp_async_4(smem_u32(&sm.kring[warp][slot][u][g]), ksseq + (pa >= 0 ? pa : 0),
                               pa >= 0 ? 4 : 0);
                    cp_async_4(smem_u32(&sm.kring[warp][slot][u][g + 8]), ksseq + (pb >= 0 ? pb : 0),
                               pb >= 0 ? 4 : 0);
                }
            }
        }
        cp_async_commit();                   // empty groups keep the count uniform
    };

#pragma unroll
    for (int i = 0; i < STAGES - 1; ++i) issue(i);

    for (int i = 0; i < n_stages; ++i) {
        issue(i + STAGES - 1);
        cp_async_wait<STAGES - 1>();         // this lane's copies of stage i have landed
        const int slot = i % STAGES;
#pragma unroll
        for (int u = 0; u < TPS; ++u) {
            const int tile = warp + SS_WARPS * (i * TPS + u);
            if (tile >= n_tiles) break;      // warp-uniform
            const int ra = tile * 16 + g, rb = ra + 8;
            const uint8_t* src = sm.ring[warp][slot][u];
            const uint4 va4 = *reinterpret_cast<const uint4*>(src + g * IDX_DIM + 16 * t);
            const uint4 vb4 = *reinterpret_cast<const uint4*>(src + (g + 8) * IDX_DIM + 16 * t);
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            // k-half 0: bytes 16t..16t+7 of rows g / g+8; k-half 1: bytes 16t+8..16t+15
            mma_16832_e4m3(c, va4.x, vb4.x, va4.y, vb4.y, bq[0], bq[1]);
            mma_16832_e4m3(c, va4.z, vb4.z, va4.w, vb4.w, bq[2], bq[3]);
            // lanes t = 2, 3 hold the second pieces of the heads of lanes t = 0, 1
            float d[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) d[j] = c[j] + 0.0625f * __shfl_xor_sync(0xFFFFFFFFu, c[j], 2);
            float sa = w0 * fmaxf(d[0], 0.0f) + w1 * fmaxf(d[1], 0.0f);
            float sb = w0 * fmaxf(d[2], 0.0f) + w1 * fmaxf(d[3], 0.0f);
            sa += __shfl_xor_sync(0xFFFFFFFFu, sa, 1);
            sb += __shfl_xor_sync(0xFFFFFFFFu, sb, 1);
            if (t == 0) {
                const bool va = POOL ? column_pos<POOL>(sm, col0, ra, cnt, n_b) >= 0 : ra < cnt;
                const bool vb = POOL ? column_pos<POOL>(sm, col0, rb, cnt, n_b) >= 0 : rb < cnt;
                if (ra < cnt) sm.score[ra] = va ? sm.kring[warp][slot][u][g] * sa : -INFINITY;
                if (rb < cnt) sm.score[rb] = vb ? sm.kring[warp][slot][u][g + 8] * sb : -INFINITY;
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    if (WANT_BM) {                       // HSI block maxima of this chunk's positions
        for (int blk = threadIdx.x; blk < (cnt + 7) / 8; blk += SS_THREADS) {
            float m = -INFINITY;
            for (int r = 8 * blk; r < min(8 * blk + 8, cnt); ++r) m = fmaxf(m, sm.score[r]);
            bm_b[(col0 >> 3) + blk] = m;
        }
    }

    // chunk-local Top-512 -> candidates (score, position), padded with (-inf, -1)
    const auto key_of = [&](int i) { return score_key(sm.score[i]); };
    unsigned T;
    int need_eq;
    radix_threshold<SS_THREADS>(key_of, cnt, TOPK, sm.sel, T, need_eq);
    const int64_t cbase = (static_cast<int64_t>(b) * a.n_chunks + chunk) * TOPK;
    float* cs = a.cand_s + cbase;
    int32_t* cp = a.cand_p + cbase;
    const int n_sel = stable_emit<SS_THREADS>(key_of, cnt, T, need_eq, sm.sel, [&](int i, int slot) {
        cs[slot] = sm.score[i];
        cp[slot] = static_cast<int32_t>(column_pos<POOL>(sm, col0, i, cnt, n_b));
    });
    for (int i = n_sel + threadIdx.x; i < TOPK; i += SS_THREADS) {
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

csa2_status launch_scan_select(const ScanSelectArgs& a, bool pool, bool want_bm, cudaStream_t stream) {
    dim3 grid(static_cast<unsigned>(a.n_chunks), static_cast<unsigned>(a.p.batch));
    const int smem = static_cast<int>(sizeof(ScanShared));
    const void* k = pool ? reinterpret_cast<const void*>(scan_select_kernel<true, false>)
                  : want_bm ? reinterpret_cast<const void*>(scan_select_kernel<false, true>)
                            : reinterpret_cast<const void*>(scan_select_kernel<false, false>);
    if (!opt_in_smem(k, smem)) return check_launch("scan_select_kernel smem attribute");
    if (pool) {
        scan_select_kernel<true, false><<<grid, SS_THREADS, smem, stream>>>(a);
    } else if (want_bm) {
        scan_select_kernel<false, true><<<grid, SS_THREADS, smem, stream>>>(a);
    } else {
        scan_select_kernel<false, false><<<grid, SS_THREADS, smem, stream>>>(a);
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
