// Fused decode indexer: scan + chunk-local Top-512, then a per-sequence merge.
//
// CSA2 section of the thecryptopost.io DeepSeek-V4.1-Flash article: a Full layer scores
// the context with its indexer and picks a new Top-512; a Reindex layer
// rescores the Hierarchical Sparse Indexer's pool (2,048 blocks of 8) with its own
// indexer Q.  Score (the pages give no formula):
//     score(s) = kscale[s] * sum_h w[h] * ReLU(q[h] . e4m3(k8[s])).
//
// scan_select_kernel: one CTA per (chunk of candidate columns, sequence), warp-specialised
// on the tensor cores.  Warp 0 streams 128-row tiles of FP8 K (8 KB) with TMA into a
// 4-stage shared-memory ring (64-byte swizzle): one 128-row box for a Full scan (its row
// scales by cp.async into the stage), sixteen 8-row boxes (one per HSI block, issued by
// sixteen lanes) for a Reindex scan (its row scales read by the epilogue threads two
// tiles ahead); warp 1 owns 32 TMEM columns and issues
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
//
// Both kernels are launched as programmatic dependents of the kernel before them on the
// stream: their barrier and TMEM set-up overlap its tail, and nothing is read from global
// memory before griddepcontrol.wait.
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
static_assert(sizeof(FastSelectShared<TC_THREADS>) <= TC_STAGES * TC_TILE_BYTES,
              "the chunk select's scratch lives in the TMA ring");
// merge threads: 1,024 for many candidates (a Full scan's 32 x 512; measured 25 against 32 us
// with 512 at B = 64), 512 for few (a Reindex scan's 4 x 512: 9.7 against 10.6 us)
constexpr int MERGE_THREADS_SMALL = 512;
constexpr int MERGE_THREADS_LARGE = 1024;
constexpr int MERGE_SMALL_CANDS = 4096;    // up to this many candidates: the 512-thread merge
constexpr int MERGE_SMEM_KEYS = 32768;     // candidates staged in shared memory
template <int NT>
__host__ __device__ constexpr int merge_kpt() { return MERGE_SMEM_KEYS / NT; }   // staged keys per thread
static_assert(sizeof(RegSelectShared<MERGE_THREADS_SMALL, merge_kpt<MERGE_THREADS_SMALL>()>) <=
                  sizeof(GlobalSelectShared<MERGE_THREADS_SMALL>) &&
              sizeof(RegSelectShared<MERGE_THREADS_LARGE, merge_kpt<MERGE_THREADS_LARGE>()>) <=
                  sizeof(GlobalSelectShared<MERGE_THREADS_LARGE>),
              "the exact select's scratch fits below the staged keys");
static_assert(sizeof(GlobalSelectShared<MERGE_THREADS_SMALL>) % 16 == 0 &&
              sizeof(GlobalSelectShared<MERGE_THREADS_LARGE>) % 16 == 0, "staged keys start 16-byte aligned");

struct __align__(1024) TcShared {
    uint8_t a[TC_STAGES][TC_TILE_BYTES];    // FP8 K tiles (64-byte swizzle), 1 KB aligned
    uint8_t b[TC_N * IDX_DIM];              // query pieces (64-byte swizzle)
    float ks[TC_STAGES][TC_TILE];           // the tiles' row scales (staged with the rows)
    float score[SCAN_CHUNK];
    int32_t pool_blk[SCAN_CHUNK / POOL_BLOCK];
    SelectShared<TC_THREADS> sel;
    float wq[IDX_HEADS];                    // head weight times 2^-s_h
    float t4[4];                            // per epilogue warp: min of the lanes' 4th best
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

// CONTIG (with POOL): the pool's rows were gathered contiguously (pool slot order) by
// pool_gather_kernel, so a Reindex tile is one 128-row TMA box and its row scales come by
// cp.async, as in a Full scan; the positions still come from the pool blocks.
template <bool POOL, bool WANT_BM, bool CONTIG>
__global__ void __launch_bounds__(TC_THREADS, 4)
scan_select_kernel(const __grid_constant__ CUtensorMap tmap, ScanSelectArgs a) {
    constexpr bool SCATTERED = POOL && !CONTIG;           // one 8-row TMA box per HSI block
    extern __shared__ uint8_t smem_raw[];
    // aligned by pointer arithmetic on the shared array (keeps the shared address space)
    TcShared& sm = *reinterpret_cast<TcShared*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const IndexParams& p = a.p;
    const int b = blockIdx.y;
    const int chunk = blockIdx.x;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // ---- set-up that reads nothing written by earlier kernels, then the programmatic
    //      dependency on the previous kernel (launched with programmatic serialization)
    if (tid == 0) {
        for (int s = 0; s < TC_STAGES; ++s) {
            // Full: 32 producer lanes (cp.async of the scales) + the TMA's expect_tx arrive;
            // pool: the expect_tx arrive of the block loads only (the epilogue loads scales)
            mbar_init(&sm.full[s], SCATTERED ? 1 : 33);
            // freed by the MMA's commit and by the 4 epilogue warps (done with the scales)
            mbar_init(&sm.empty[s], 5);
        }
        for (int j = 0; j < 2; ++j) {
            mbar_init(&sm.tfull[j], 1);
            mbar_init(&sm.tempty[j], 4);
        }
        mbar_fence_init();
    }
    if (warp == 1) tmem_alloc(&sm.tmem, 32);
    __syncthreads();
    griddep_launch_dependents();
    griddep_wait();

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
    __syncthreads();                                     // query scales and pool blocks
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
    const uint32_t limit = wait_limit(err);             // the caller's bound (drains keep the default)

    if (warp == 0) {
        // ---- producer warp: the K rows (one TMA tile, or one 8-row TMA box per HSI block
        //      of the pool) and the 128 row scales of each tile (cp.async)
        int issued = 0;
        for (int it = 0; it < n_tiles; ++it, ++issued) {
            const int s = it % TC_STAGES;
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&sm.empty[s], ((it / TC_STAGES) & 1) ^ 1, err, limit);
            if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) break;
            if (SCATTERED) {
                // one 8-row TMA box per HSI block (x = 0: 16-byte aligned), issued by lane bk
                // (16 independent issues, not a chain of dependent ones); lane 0 arms the
                // stage's bytes first.  An unused slot loads row 0 (in bounds, masked).
                if (lane == 0) mbar_arrive_expect_tx(&sm.full[s], TC_TILE_BYTES);
                __syncwarp();
                if (lane < TC_TILE / POOL_BLOCK) {
                    const int j = it * TC_TILE + lane * POOL_BLOCK;
                    const int32_t blk = j < cnt ? sm.pool_blk[j >> 3] : -1;
                    const int64_t row0 = blk >= 0 ? p.rows.row(b, seq_off, static_cast<int64_t>(blk) * POOL_BLOCK) : 0;
                    tma_load_2d(sm.a[s] + lane * POOL_BLOCK * IDX_DIM, &tmap, 0, static_cast<int>(row0), &sm.full[s]);
                }
            } else {
                // the tile's first row: Full: the cache row of column col0 + 128 it (the
                // tile lies in one page); contiguous pool: row b * 16384 + slot
                const int64_t tile_row = CONTIG ? static_cast<int64_t>(b) * POOL_POSITIONS + col0 + it * TC_TILE
                                                : p.rows.row(b, seq_off, col0 + it * TC_TILE);
                const float* kss = CONTIG ? a.pool_kscale : p.idx_kscale;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sm.full[s], TC_TILE_BYTES);
                    tma_load_2d(sm.a[s], &tmap, 0, static_cast<int>(tile_row), &sm.full[s]);
                }
                // the tile's 128 row scales
#pragma unroll
                for (int i = 0; i < TC_TILE / 32; ++i) {
                    const int row = lane + 32 * i;
                    const bool in = it * TC_TILE + row < cnt;
                    cp_async_4(smem_u32(&sm.ks[s][row]), kss + (in ? tile_row + row : 0), in ? 4 : 0);
                }
                cp_async_mbar_arrive_noinc(&sm.full[s]);
            }
        }
        cp_async_wait<0>();                                 // own copies landed
        if (lane == 0) {                                    // the issued TMA tiles landed too
            for (int it = max(0, issued - TC_STAGES); it < issued; ++it)
                mbar_wait(&sm.full[it % TC_STAGES], (it / TC_STAGES) & 1, err);
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer: D[buf] = K_tile * pieces^T over K = 64 (two K=32 steps)
        const uint32_t idesc = idesc_e4m3_f32(TC_TILE, TC_N);
        const uint64_t bdesc = umma_desc_sw64(smem_u32(sm.b));
        int done = 0;
        for (int it = 0; it < n_tiles; ++it) {
            const int s = it % TC_STAGES, buf = it & 1;
            if (!mbar_wait(&sm.full[s], (it / TC_STAGES) & 1, err, limit)) break;
            if (!mbar_wait(&sm.tempty[buf], ((it >> 1) & 1) ^ 1, err, limit)) break;
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
        const float w0 = sm.wq[0], w1 = sm.wq[1], w2 = sm.wq[2], w3 = sm.wq[3];
        float t1 = -INFINITY, t2 = -INFINITY, t3 = -INFINITY, t4 = -INFINITY;   // this thread's best 4
        // pool: this thread's row scale of tile it, loaded two tiles ahead (the producer warp
        // only issues the block copies)
        const auto pool_scale = [&](int it) {
            const int64_t pos = it < n_tiles ? chunk_pos<POOL>(sm, col0, it * TC_TILE + q * 32 + lane, cnt, n_b) : -1;
            return pos >= 0 ? __ldg(p.idx_kscale + p.rows.row(b, seq_off, pos)) : 0.0f;
        };
        float ks_a = 0.0f, ks_b = 0.0f;
        if (SCATTERED) {
            ks_a = pool_scale(0);
            ks_b = pool_scale(1);
        }
        for (int it = 0; it < n_tiles; ++it) {
            const int buf = it & 1;
            const int row = q * 32 + lane;
            const int j = it * TC_TILE + row;
            // (a failed wait ends the warp's loop as a whole: the loop body has warp-wide steps)
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.tfull[buf], (it >> 1) & 1, err, limit))) break;
            tc_fence_after();
            uint32_t v[8];
            tmem_ld8(tmem + (static_cast<uint32_t>(32 * q) << 16) + buf * TC_N, v);
            // Full: the stage's scales; its full barrier completed before the MMA ran (this
            // wait returns at once; the stage cannot be refilled before this warp releases it).
            // The pool's scales come from registers.
            if (!SCATTERED && !__all_sync(0xFFFFFFFFu, mbar_wait(&sm.full[it % TC_STAGES], (it / TC_STAGES) & 1, err, limit)))
                break;
            float ks;
            if (SCATTERED) {
                ks = ks_a;
                ks_a = ks_b;
                ks_b = pool_scale(it + 2);
            } else {
                ks = sm.ks[it % TC_STAGES][row];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.tempty[buf]);
                mbar_arrive(&sm.empty[it % TC_STAGES]);
            }
            const int64_t pos = chunk_pos<POOL>(sm, col0, j, cnt, n_b);
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
                float x = sc, hi;                             // branch-free insertion
                hi = fmaxf(t1, x); x = fminf(t1, x); t1 = hi;
                hi = fmaxf(t2, x); x = fminf(t2, x); t2 = hi;
                hi = fmaxf(t3, x); x = fminf(t3, x); t3 = hi;
                t4 = fmaxf(t4, x);
            }
        }
        // 4 x 128 scores are >= min over the epilogue threads of their 4th best, so that
        // minimum is a lower bound on the chunk's 512th score.
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) t4 = fminf(t4, __shfl_xor_sync(0xFFFFFFFFu, t4, off));
        if (lane == 0) sm.t4[q] = t4;
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

    // ---- chunk-local Top-512 -> candidates (score, position), padded with (-inf, -1)
    const auto key_of = [&](int i) { return score_key(sm.score[i]); };
    const float lb = fminf(fminf(sm.t4[0], sm.t4[1]), fminf(sm.t4[2], sm.t4[3]));
    const unsigned lb_key = score_key(lb);
    // keys >= lb_key (every valid key when lb is -inf) survive; the rest cannot be selected
    const int64_t cbase = (static_cast<int64_t>(b) * a.n_chunks + chunk) * TOPK;
    float* cs = a.cand_s + cbase;
    int32_t* cp = a.cand_p + cbase;
    // the TMA ring is idle now: it holds the select's survivors and histogram
    auto& fs = *reinterpret_cast<FastSelectShared<TC_THREADS>*>(&sm.a[0][0]);
    unsigned T;
    int n_sel = fast_select<TC_THREADS>(key_of, cnt, TOPK, lb_key, fs, T, [&](int i, int slot) {
        cs[slot] = sm.score[i];
        cp[slot] = static_cast<int32_t>(chunk_pos<POOL>(sm, col0, i, cnt, n_b));
    });
    if (n_sel < 0) {                     // too many survivors or a crowded boundary bin
        int need_eq;
        radix_threshold<TC_THREADS>(key_of, cnt, TOPK, sm.sel, T, need_eq);
        n_sel = stable_emit<TC_THREADS>(key_of, cnt, T, need_eq, sm.sel, [&](int i, int slot) {
            cs[slot] = sm.score[i];
            cp[slot] = static_cast<int32_t>(chunk_pos<POOL>(sm, col0, i, cnt, n_b));
        });
    }
    for (int i = n_sel + tid; i < TOPK; i += TC_THREADS) {
        cs[i] = -INFINITY;
        cp[i] = -1;
    }
    // this chunk's 512th score (the radix threshold), a lower bound on the sequence's
    if (tid == 0)
        a.chunk_thr[static_cast<int64_t>(b) * a.n_chunks + chunk] =
            (n_sel == TOPK && T != 0u) ? key_score(T) : -INFINITY;
}

template <int MERGE_THREADS>
__global__ void __launch_bounds__(MERGE_THREADS)
merge_select_kernel(const float* __restrict__ cand_s, const int32_t* __restrict__ cand_p,
                    const float* __restrict__ chunk_thr, int n_chunks, int32_t* __restrict__ out) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    auto& sh = *reinterpret_cast<GlobalSelectShared<MERGE_THREADS>*>(smem_raw);
    float* keys = reinterpret_cast<float*>(smem_raw + sizeof(GlobalSelectShared<MERGE_THREADS>));
    __shared__ float s_lb;
    griddep_launch_dependents();
    griddep_wait();                                      // the scan's candidates
    const int64_t r = blockIdx.x;
    const int n_cand = n_chunks * TOPK;
    const float* cs = cand_s + r * n_cand;
    const int32_t* cp = cand_p + r * n_cand;
    // the sequence's 512th score is >= every chunk's 512th score
    if (threadIdx.x < 32) {
        float lb = -INFINITY;
        for (int c = threadIdx.x; c < n_chunks; c += 32) lb = fmaxf(lb, chunk_thr[r * n_chunks + c]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) lb = fmaxf(lb, __shfl_xor_sync(0xFFFFFFFFu, lb, off));
        if (threadIdx.x == 0) s_lb = lb;
    }
    __syncthreads();
    const unsigned lb_key = score_key(s_lb);
    int32_t* dst = out + r * TOPK;
    const bool staged = n_cand <= MERGE_SMEM_KEYS;
    if (staged) stage_floats<MERGE_THREADS>(keys, cs, n_cand);   // one batched, coalesced load
    __syncthreads();
    if (staged) {                                   // one exact select over the staged keys
        const auto key_at = [&](int u) {
            const int i = u * MERGE_THREADS + static_cast<int>(threadIdx.x);
            return i < n_cand ? score_key(keys[i]) : 0u;
        };
        constexpr int MERGE_KPT = merge_kpt<MERGE_THREADS>();
        auto& rs = *reinterpret_cast<RegSelectShared<MERGE_THREADS, MERGE_KPT>*>(smem_raw);
        unsigned T;
        const int n_sel = reg_select<MERGE_THREADS, MERGE_KPT>(key_at, n_cand, TOPK, lb_key, rs, T,
                                                               [&](int i, int slot) { dst[slot] = __ldg(cp + i); });
        if (n_sel >= 0) {
            for (int i = n_sel + threadIdx.x; i < TOPK; i += MERGE_THREADS) dst[i] = -1;
            return;
        }
    }
    const auto key_of = [&](int i) {
        const unsigned k = score_key(staged ? keys[i] : __ldg(cs + i));
        return k >= lb_key ? k : 0u;
    };
    const int n_sel = global_select<MERGE_THREADS>(key_of, n_cand, TOPK, sh,
                                                   [&](int i, int slot) { dst[slot] = __ldg(cp + i); });
    for (int i = n_sel + threadIdx.x; i < TOPK; i += MERGE_THREADS) dst[i] = -1;
}

// The pool's indexer rows, contiguous in pool slot order: warp w of CTA (x, b) copies HSI
// block slot 8x + w of sequence b (8 rows x 64 B, one 16-byte chunk per lane) and its 8
// row scales; an absent block or a row past the context is written as zeros (the Reindex
// scan masks those slots by position anyway).
__global__ void __launch_bounds__(256)
pool_gather_kernel(const int32_t* __restrict__ pool_blocks, const int64_t* __restrict__ kv_offsets,
                   const uint8_t* __restrict__ idx_k, const float* __restrict__ idx_kscale,
                   uint8_t* __restrict__ pool_k, float* __restrict__ pool_kscale, RowMap rows) {
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t slot = static_cast<int64_t>(b) * POOL_BLOCKS + blockIdx.x * 8 + warp;
    const int64_t seq_off = kv_offsets[b];
    const int64_t n_b = kv_offsets[b + 1] - seq_off;
    const int32_t blk = pool_blocks[slot];
    const int64_t pos0 = static_cast<int64_t>(blk) * POOL_BLOCK;
    const int64_t row0 = blk >= 0 ? rows.row(b, seq_off, pos0) : 0;   // the block lies in one page
    const int r = lane >> 2, c = lane & 3;
    const bool in = blk >= 0 && pos0 + r < n_b;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (in) v = __ldg(reinterpret_cast<const uint4*>(idx_k + (row0 + r) * IDX_DIM) + c);
    reinterpret_cast<uint4*>(pool_k + slot * POOL_BLOCK * IDX_DIM)[lane] = v;
    if (lane < POOL_BLOCK) {
        const bool ok = blk >= 0 && pos0 + lane < n_b;
        pool_kscale[slot * POOL_BLOCK + lane] = ok ? __ldg(idx_kscale + row0 + lane) : 0.0f;
    }
}

}  // namespace

csa2_status launch_pool_gather(const int32_t* pool_blocks, const int64_t* kv_offsets, int batch,
                               const uint8_t* idx_k, const float* idx_kscale, uint8_t* pool_k,
                               float* pool_kscale, RowMap rows, cudaStream_t stream) {
    pool_gather_kernel<<<dim3(POOL_BLOCKS / 8, static_cast<unsigned>(batch)), 256, 0, stream>>>(
        pool_blocks, kv_offsets, idx_k, idx_kscale, pool_k, pool_kscale, rows);
    return check_launch("pool_gather_kernel");
}

csa2_status launch_scan_select(const ScanSelectArgs& a, const CUtensorMap& tmap, bool pool, bool want_bm,
                               cudaStream_t stream) {
    dim3 grid(static_cast<unsigned>(a.n_chunks), static_cast<unsigned>(a.p.batch));
    const int smem = static_cast<int>(sizeof(TcShared)) + 1024;     // + alignment slack
    const bool contig = pool && a.pool_kscale != nullptr;
    const void* k = contig ? reinterpret_cast<const void*>(scan_select_kernel<true, false, true>)
                  : pool ? reinterpret_cast<const void*>(scan_select_kernel<true, false, false>)
                  : want_bm ? reinterpret_cast<const void*>(scan_select_kernel<false, true, false>)
                            : reinterpret_cast<const void*>(scan_select_kernel<false, false, false>);
    if (!opt_in_smem(k, smem)) return check_launch("scan_select_kernel smem attribute");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(TC_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (contig) {
        cudaLaunchKernelEx(&cfg, scan_select_kernel<true, false, true>, tmap, a);
    } else if (pool) {
        cudaLaunchKernelEx(&cfg, scan_select_kernel<true, false, false>, tmap, a);
    } else if (want_bm) {
        cudaLaunchKernelEx(&cfg, scan_select_kernel<false, true, false>, tmap, a);
    } else {
        cudaLaunchKernelEx(&cfg, scan_select_kernel<false, false, false>, tmap, a);
    }
    return check_launch("scan_select_kernel");
}

csa2_status launch_merge_select(const float* cand_s, const int32_t* cand_p, const float* chunk_thr,
                                int n_chunks, int rows, int32_t* out, cudaStream_t stream) {
    const int n_cand = n_chunks * TOPK;
    const bool small = n_cand <= MERGE_SMALL_CANDS;
    const int nt = small ? MERGE_THREADS_SMALL : MERGE_THREADS_LARGE;
    const int gsel = static_cast<int>(small ? sizeof(GlobalSelectShared<MERGE_THREADS_SMALL>)
                                            : sizeof(GlobalSelectShared<MERGE_THREADS_LARGE>));
    const int smem = gsel + (n_cand <= MERGE_SMEM_KEYS ? n_cand * 4 : 0);
    const void* fn = small ? reinterpret_cast<const void*>(merge_select_kernel<MERGE_THREADS_SMALL>)
                           : reinterpret_cast<const void*>(merge_select_kernel<MERGE_THREADS_LARGE>);
    if (!opt_in_smem(fn, gsel + MERGE_SMEM_KEYS * 4)) return check_launch("merge_select_kernel smem attribute");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(rows));
    cfg.blockDim = dim3(static_cast<unsigned>(nt));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (small) cudaLaunchKernelEx(&cfg, merge_select_kernel<MERGE_THREADS_SMALL>, cand_s, cand_p, chunk_thr, n_chunks, out);
    else cudaLaunchKernelEx(&cfg, merge_select_kernel<MERGE_THREADS_LARGE>, cand_s, cand_p, chunk_thr, n_chunks, out);
    return check_launch("merge_select_kernel");
}

}  // namespace csa2
