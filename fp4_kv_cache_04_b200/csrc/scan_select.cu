// Fused decode indexer: scan + chunk-local Top-512, then a per-sequence merge.
//
// CSA2 section of the thecryptopost.io DeepSeek-V4.1-Flash article: a Full layer scores
// the context with its indexer and selects fresh Top-512 indices; a Reindex layer
// rescores the Hierarchical Sparse Indexer's pool (2,048 blocks of 8) with its own
// indexer Q.  Score (the pages give no formula):
//     score(s) = kscale[s] * sum_h w[h] * ReLU(q[h] . e4m3(k8[s])).
//
// scan_select_kernel: one CTA per (chunk of 8,192 candidate columns, sequence).  Warps
// take 16-column tiles; for each tile a warp issues two fully coalesced 512-byte loads
// whose 16-byte pieces are exactly the A fragments of four m16n8k16 MMAs (the 64-dim
// dot product is permuted identically in A and B), converts E4M3 -> f16 (exact), and
// accumulates in fp32 on the tensor cores.  Scores stay in shared memory; the CTA then
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
constexpr int SS_UNROLL = 2;
constexpr int MERGE_THREADS = 512;

struct ScanShared {
    float score[SCAN_CHUNK];
    SelectShared<SS_THREADS> sel;
};

__device__ __forceinline__ int64_t pool_position(const int32_t* pool_b, int64_t col, int64_t n_b) {
    const int32_t blk = pool_b[col >> 3];
    if (blk < 0) return -1;
    const int64_t pos = static_cast<int64_t>(blk) * POOL_BLOCK + (col & 7);
    return pos < n_b ? pos : -1;
}

template <bool POOL, bool WANT_BM>
__global__ void __launch_bounds__(SS_THREADS, 2)
scan_select_kernel(ScanSelectArgs a) {
    __shared__ ScanShared sm;
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
    const int64_t col0 = static_cast<int64_t>(chunk) * SCAN_CHUNK;
    const int cnt = static_cast<int>(max(static_cast<int64_t>(0),
                                         min(static_cast<int64_t>(SCAN_CHUNK), n_cols - col0)));
    const int32_t* pool_b = POOL ? p.pool_blocks + static_cast<int64_t>(b) * POOL_BLOCKS : nullptr;

    // B fragments: column n = g is head g (g < 4) of this sequence's single query.
    uint32_t bq[8];
    if (g < IDX_HEADS) {
        const uint16_t* src = p.idx_q + (static_cast<int64_t>(b) * IDX_HEADS + g) * IDX_DIM + 16 * t;
        const uint4 v0 = *reinterpret_cast<const uint4*>(src);
        const uint4 v1 = *reinterpret_cast<const uint4*>(src + 8);
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) bq[i] = bf16x2_to_f16x2(w[i]);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) bq[i] = 0u;
    }
    // lanes t = 0, 1 own heads {0,1} / {2,3} of the query (columns 2t, 2t+1)
    const float w0 = (t < 2) ? p.idx_w[static_cast<int64_t>(b) * IDX_HEADS + 2 * t] : 0.0f;
    const float w1 = (t < 2) ? p.idx_w[static_cast<int64_t>(b) * IDX_HEADS + 2 * t + 1] : 0.0f;

    const uint8_t* kseq = p.idx_k + seq_off * IDX_DIM + 16 * t;
    const float* ksseq = p.idx_kscale + seq_off;
    float* bm_b = WANT_BM ? a.bm + static_cast<int64_t>(b) * a.bm_ld : nullptr;

    for (int tile0 = warp * 16; tile0 < cnt; tile0 += SS_WARPS * 16 * SS_UNROLL) {
        uint4 ra[SS_UNROLL], rb[SS_UNROLL];
        float ka[SS_UNROLL], kb[SS_UNROLL];
        bool va[SS_UNROLL], vb[SS_UNROLL];
#pragma unroll
        for (int u = 0; u < SS_UNROLL; ++u) {
            const int ja = tile0 + u * SS_WARPS * 16 + g;
            const int jb = ja + 8;
            int64_t pa, pb;
            if (POOL) {
                pa = ja < cnt ? pool_position(pool_b, col0 + ja, n_b) : -1;
                pb = jb < cnt ? pool_position(pool_b, col0 + jb, n_b) : -1;
            } else {
                pa = ja < cnt ? col0 + ja : -1;
                pb = jb < cnt ? col0 + jb : -1;
            }
            va[u] = pa >= 0;
            vb[u] = pb >= 0;
            ra[u] = va[u] ? ldg_stream(kseq + pa * IDX_DIM) : make_uint4(0, 0, 0, 0);
            rb[u] = vb[u] ? ldg_stream(kseq + pb * IDX_DIM) : make_uint4(0, 0, 0, 0);
            ka[u] = va[u] ? __ldg(ksseq + pa) : 0.0f;
            kb[u] = vb[u] ? __ldg(ksseq + pb) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < SS_UNROLL; ++u) {
            const int tile = tile0 + u * SS_WARPS * 16;
            if (tile >= cnt) break;                  // warp-uniform
            const uint32_t wa[4] = {ra[u].x, ra[u].y, ra[u].z, ra[u].w};
            const uint32_t wb[4] = {rb[u].x, rb[u].y, rb[u].z, rb[u].w};
            float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint32_t af[4] = {e4m3x2_to_f16x2(static_cast<uint16_t>(wa[s] & 0xFFFFu)),
                                        e4m3x2_to_f16x2(static_cast<uint16_t>(wb[s] & 0xFFFFu)),
                                        e4m3x2_to_f16x2(static_cast<uint16_t>(wa[s] >> 16)),
                                        e4m3x2_to_f16x2(static_cast<uint16_t>(wb[s] >> 16))};
                mma_16816(c, af, bq[2 * s], bq[2 * s + 1]);
            }
            float sa = w0 * fmaxf(c[0], 0.0f) + w1 * fmaxf(c[1], 0.0f);
            float sb = w0 * fmaxf(c[2], 0.0f) + w1 * fmaxf(c[3], 0.0f);
            sa += __shfl_xor_sync(0xFFFFFFFFu, sa, 1);
            sb += __shfl_xor_sync(0xFFFFFFFFu, sb, 1);
            sa = va[u] ? ka[u] * sa : -INFINITY;
            sb = vb[u] ? kb[u] * sb : -INFINITY;
            if (t == 0) {
                if (tile + g < cnt) sm.score[tile + g] = sa;
                if (tile + g + 8 < cnt) sm.score[tile + g + 8] = sb;
            }
            if (WANT_BM) {
                float ma = sa, mb = sb;
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    ma = fmaxf(ma, __shfl_xor_sync(0xFFFFFFFFu, ma, off));
                    mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, off));
                }
                if (lane == 0) {
                    const int64_t blk = (col0 + tile) >> 3;
                    bm_b[blk] = ma;
                    if (tile + 8 < cnt) bm_b[blk + 1] = mb;
                }
            }
        }
    }
    __syncthreads();

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
        cp[slot] = static_cast<int32_t>(POOL ? pool_position(pool_b, col0 + i, n_b) : col0 + i);
    });
    for (int i = n_sel + threadIdx.x; i < TOPK; i += SS_THREADS) {
        cs[i] = -INFINITY;
        cp[i] = -1;
    }
}

__global__ void __launch_bounds__(MERGE_THREADS)
merge_select_kernel(const float* __restrict__ cand_s, const int32_t* __restrict__ cand_p,
                    int n_cand, int32_t* __restrict__ out) {
    __shared__ SelectShared<MERGE_THREADS> sel;
    const int64_t r = blockIdx.x;
    const float* cs = cand_s + r * n_cand;
    const int32_t* cp = cand_p + r * n_cand;
    const auto key_of = [&](int i) { return score_key(__ldg(cs + i)); };
    unsigned T;
    int need_eq;
    radix_threshold<MERGE_THREADS>(key_of, n_cand, TOPK, sel, T, need_eq);
    int32_t* dst = out + r * TOPK;
    const int n_sel = stable_emit<MERGE_THREADS>(key_of, n_cand, T, need_eq, sel,
                                                 [&](int i, int slot) { dst[slot] = __ldg(cp + i); });
    for (int i = n_sel + threadIdx.x; i < TOPK; i += MERGE_THREADS) dst[i] = -1;
}

}  // namespace

csa2_status launch_scan_select(const ScanSelectArgs& a, bool pool, bool want_bm, cudaStream_t stream) {
    dim3 grid(static_cast<unsigned>(a.n_chunks), static_cast<unsigned>(a.p.batch));
    if (pool) {
        scan_select_kernel<true, false><<<grid, SS_THREADS, 0, stream>>>(a);
    } else if (want_bm) {
        scan_select_kernel<false, true><<<grid, SS_THREADS, 0, stream>>>(a);
    } else {
        scan_select_kernel<false, false><<<grid, SS_THREADS, 0, stream>>>(a);
    }
    return check_launch("scan_select_kernel");
}

csa2_status launch_merge_select(const float* cand_s, const int32_t* cand_p, int n_cand, int rows,
                                int32_t* out, cudaStream_t stream) {
    merge_select_kernel<<<rows, MERGE_THREADS, 0, stream>>>(cand_s, cand_p, n_cand, out);
    return check_launch("merge_select_kernel");
}

}  // namespace csa2
