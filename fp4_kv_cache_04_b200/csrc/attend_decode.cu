// Decode attention (one query per sequence, every position and SWA row visible).
//
// CSA2 section of the thecryptopost.io DeepSeek-V4.1-Flash article: every layer keeps its
// own main Q and SWA KV and attends over its Top-512 selection of the shared FP4 main KV;
// the Causal Encoder-Decoder section fixes the 128-token window; tldrocket.com: one
// 512-dim latent serves as both key and value.  Per head h:
//     out_h = softmax_j(sm_scale * q_h . row_j) . rows,  rows = selected FP4 rows
//                                                        (dequantised) ++ SWA rows.
//
// Work split: a sequence's keys form up to 8 main tiles (64 selected rows each) and
// ceil(swa_rows/64) SWA tiles.  CTA (row, sp) takes tiles_per_cta consecutive tiles of
// ONE kind: sp < n_split_main -> main tiles, otherwise SWA tiles.  The row's CTAs form
// one thread-block cluster.  Each keeps an unnormalised partial (reference max m, sum l,
// O) in registers; at the end it pushes every 64-dim block of O, and its m and l, into
// the shared memory of the cluster CTA that owns that block, and after a cluster barrier
// each CTA merges its own blocks from local shared memory:
//     out = sum_s e^(m_s - M) O_s / sum_s e^(m_s - M) l_s.
//
// One 64 KB shared tile holds a tile's 64 rows x 512 dims as 64-column blocks of
// [64 rows][128 B] with the 128-byte swizzle (the TMA layout), read with ldmatrix for
// both products, since key = value:
//  - S^T = K Q^T with mma.sync m16n8k16: warp w takes keys 16(w%4).. and dims of half
//    w/4; the two halves are summed in shared memory.
//  - O = P V: warp w owns output dims 64w .. 64w+63 for all 16 heads (32 fp32 registers).
// The tensor-core work per tile is 2 x 64 x 16 x 512 MACs; with only 16 heads the warp
// MMAs keep the tensor pipe busier than tcgen05 MMAs with N = 16 would (measured on B200:
// about 2 cycles per m16n8k16 per SM against about 71 cycles per 128x16x16 tcgen05.mma).
//
//  - main tiles: cp.async gathers the rows' E2M1 codes into a staging buffer and each
//    thread loads its row's 32 E4M3 scale bytes into registers (the next tile's loads run
//    during this tile's products); each thread turns
//    16-channel groups into f16 (hardware e2m1 -> f16, times the e4m3 scale: exact); the
//    products run in f16 with the query converted to f16 (exact in the normal range).
//    With the cross-layer reuse cache a Full/Reindex layer stores each finished tile
//    (one bulk copy) and Reuse layers load it back with one bulk copy.
//  - SWA tiles: TMA loads the bf16 rows straight into the tile; products in bf16 with the
//    bf16 query (exact); P is split into bf16 hi + lo pieces, so P V keeps ~16 bits.
//  - softmax: per head over the tile's 64 keys, two heads per warp.  A head's reference
//    max only moves when a score exceeds it by more than RESCALE_GAP (then its O rows are
//    rescaled); any reference gives the same normalised result.
// Every mbarrier wait is bounded (ERR_TIMEOUT set, the CTA stops computing, no hang).
#include <cuda_fp4.h>

#include <algorithm>
#include <cstddef>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace csa2 {

namespace {

constexpr int DT_THREADS = 256;
constexpr int DT_WARPS = DT_THREADS / 32;
constexpr int DT_KEYS = 64;                               // keys per tile
constexpr int DT_TILE_BYTES = DT_KEYS * D * 2;            // 64 KB
constexpr int DT_BLOCK_BYTES = DT_KEYS * 128;             // one 64-dim block of the tile
constexpr int DT_Q_BYTES = HEADS * D * 2;                 // 16 KB
constexpr int DT_P_BYTES = HEADS * DT_KEYS * 2;           // 2 KB
constexpr int DT_MAX_CLUSTER = 8;                         // portable cluster size
constexpr int DT_OBLOCK_FLOATS = HEADS * 64;              // one 64-dim block of O
constexpr float RESCALE_GAP = 8.0f;                       // lazy O rescale threshold (nats)

struct alignas(1024) DecodeSmem {
    uint8_t tile[DT_TILE_BYTES];          // SW128 [8][64 rows][128 B]; at the end, the
                                          // partial O blocks pushed by the cluster
    uint8_t q[DT_Q_BYTES];                // SW128 [8][16 heads][128 B]
    uint8_t p[2][DT_P_BYTES];             // P (f16) or P hi / lo (bf16): SW128 [16][64]
    float s2[2][DT_KEYS][HEADS + 1];      // S partials of the two dim halves
    uint8_t stage[DT_KEYS][ROW_CODES];    // gathered E2M1 codes (scales go to registers)
    int32_t main_pos[TOPK];
    float m[HEADS], l[HEADS], alpha[HEADS];
    float swa_s[DT_KEYS];                 // FP8 SWA tiles: the rows' scales
    float swa_smax;                       //   and their max over the tile
    int32_t warp_cnt[DT_WARPS];
    uint64_t bar_q, bar_load;
    int rescale, fail;
};

// After the tiles, the tile buffer receives the cluster's pushes: the 64-dim O blocks this
// CTA owns (slot (w / n_split) * n_split + sender; at most 14 slots for n_split <= 8) and
// every sender's m and l.
constexpr int DT_PUSH_SLOTS = 14;
constexpr int DT_PM_OFFSET = DT_PUSH_SLOTS * DT_OBLOCK_FLOATS * 4;
constexpr int DT_PL_OFFSET = DT_PM_OFFSET + DT_MAX_CLUSTER * HEADS * 4;
static_assert(DT_PL_OFFSET + DT_MAX_CLUSTER * HEADS * 4 <= DT_TILE_BYTES, "pushes fit in the tile buffer");
static_assert(sizeof(DecodeSmem) + 1024 <= 113 * 1024, "two CTAs must fit on one SM");

__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    const __half2_raw h = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(byte), __NV_E2M1);
    return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

// Byte offset of 8-element chunk `chunk` (0..63) of row `row` in a SW128 tile of `rows` rows.
__device__ __forceinline__ uint32_t sw_chunk(uint32_t rows, uint32_t row, uint32_t chunk) {
    return (chunk >> 3) * rows * 128u + row * 128u + (((chunk & 7u) ^ (row & 7u)) << 4);
}

template <bool BF16>
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (BF16) mma_16816_bf16(c, a, b0, b1);
    else mma_16816(c, a, b0, b1);
}

// S^T partial (this warp's 16 keys x 16 heads over its dim half) -> s2.
template <bool BF16>
__device__ __forceinline__ void s_partial(DecodeSmem& sm, int warp, int lane) {
    const int mi = lane >> 3, mj = lane & 7, g = lane >> 2, t = lane & 3;
    const int kg = warp & 3, dh = warp >> 2;
    const uint32_t k_base = smem_u32(sm.tile), q_base = smem_u32(sm.q);
    const int arow = kg * 16 + ((mi & 1) << 3) + mj;
    const int brow = ((mi >> 1) << 3) + mj;
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 4
    for (int ks = dh * 16; ks < dh * 16 + 16; ++ks) {
        uint32_t a[4], bq[4];
        ldmatrix_x4(a, k_base + sw_chunk(DT_KEYS, arow, 2 * ks + (mi >> 1)));
        ldmatrix_x4(bq, q_base + sw_chunk(HEADS, brow, 2 * ks + (mi & 1)));
        mma16816<BF16>(s[0], a, bq[0], bq[1]);
        mma16816<BF16>(s[1], a, bq[2], bq[3]);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int h = 8 * nt + 2 * t;
        sm.s2[dh][kg * 16 + g][h] = s[nt][0];
        sm.s2[dh][kg * 16 + g][h + 1] = s[nt][1];
        sm.s2[dh][kg * 16 + g + 8][h] = s[nt][2];
        sm.s2[dh][kg * 16 + g + 8][h + 1] = s[nt][3];
    }
}

// O += P V over the tile for this warp's 64 dims (bf16 tiles: P in hi and lo pieces).
template <bool BF16>
__device__ __forceinline__ void pv(DecodeSmem& sm, int warp, int lane, float (&o)[8][4]) {
    const int mi = lane >> 3, mj = lane & 7;
    const uint32_t k_base = smem_u32(sm.tile);
    const uint32_t p0 = smem_u32(sm.p[0]), p1 = smem_u32(sm.p[1]);
    const int prow = ((mi & 1) << 3) + mj;
#pragma unroll
    for (int ks = 0; ks < DT_KEYS / 16; ++ks) {
        uint32_t a[4], alo[4];
        ldmatrix_x4(a, p0 + sw_chunk(HEADS, prow, 2 * ks + (mi >> 1)));
        if (BF16) ldmatrix_x4(alo, p1 + sw_chunk(HEADS, prow, 2 * ks + (mi >> 1)));
        const int key = ks * 16 + ((mi & 1) << 3) + mj;
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
            uint32_t bv[4];
            ldmatrix_x4_trans(bv, k_base + sw_chunk(DT_KEYS, key, warp * 8 + 2 * pp + (mi >> 1)));
            mma16816<BF16>(o[2 * pp], a, bv[0], bv[1]);
            mma16816<BF16>(o[2 * pp + 1], a, bv[2], bv[3]);
            if (BF16) {
                mma16816<BF16>(o[2 * pp], alo, bv[0], bv[1]);
                mma16816<BF16>(o[2 * pp + 1], alo, bv[2], bv[3]);
            }
        }
    }
}

__global__ void __launch_bounds__(DT_THREADS, 2)
attend_decode_kernel(AttnParams p, const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_swa) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    DecodeSmem& sm = *reinterpret_cast<DecodeSmem*>(
        smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));

    const int64_t r = blockIdx.x;                     // row = sequence
    const int sp = blockIdx.y;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int g = lane >> 2;
    const bool swa_cta = sp >= p.n_split_main;
    const bool swa8 = swa_cta && p.swa_fp8 != 0;       // FP8 SWA rows: f16 tiles like main
    const bool bf16_tiles = swa_cta && !swa8;
    const int64_t seq_off = p.kv_offsets[r];
    const int64_t n_b = p.kv_offsets[r + 1] - seq_off;
    const bool use_cache = !swa_cta && p.cache_mode == CSA2_CACHE_USE;
    const bool fill_cache = !swa_cta && p.cache_mode == CSA2_CACHE_FILL;

    if (tid == 0) {
        mbar_init(&sm.bar_q, 1);
        mbar_init(&sm.bar_load, 1);
        mbar_fence_init();
        sm.fail = 0;
        sm.rescale = 0;
        mbar_arrive_expect_tx(&sm.bar_q, DT_Q_BYTES);
        for (int cb = 0; cb < D / 64; ++cb)
            tma_load_2d(sm.q + cb * HEADS * 128, &tmap_q, 64 * cb, static_cast<int>(r * HEADS), &sm.bar_q);
    }
    if (tid < HEADS) {
        sm.m[tid] = -INFINITY;
        sm.l[tid] = 0.0f;
    }

    // ---- valid main positions, compacted in order (2 per thread)
    int n_main = 0;
    if (!swa_cta) {
        const int32_t* idx = p.topk_idx + r * TOPK;
        const int32_t v0 = idx[2 * tid], v1 = idx[2 * tid + 1];
        const bool bad0 = v0 >= n_b, bad1 = v1 >= n_b;
        if ((bad0 || bad1) && sp == 0 && p.err) atomicOr(p.err, ERR_DEVICE);
        const bool ok0 = v0 >= 0 && !bad0, ok1 = v1 >= 0 && !bad1;
        const int cnt = static_cast<int>(ok0) + static_cast<int>(ok1);
        int incl = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off) incl += y;
        }
        if (lane == 31) sm.warp_cnt[warp] = incl;
        __syncthreads();
        int before = incl - cnt;
        for (int w = 0; w < DT_WARPS; ++w) {
            const int c = sm.warp_cnt[w];
            if (w < warp) before += c;
            n_main += c;
        }
        if (ok0) sm.main_pos[before++] = v0;
        if (ok1) sm.main_pos[before] = v1;
    }
    const int n_keys_kind = swa_cta ? static_cast<int>(p.swa_rows) : n_main;
    const int n_tiles = (n_keys_kind + DT_KEYS - 1) / DT_KEYS;
    const int t_begin = (swa_cta ? sp - p.n_split_main : sp) * p.tiles_per_cta;
    const int t_end = min(n_tiles, t_begin + p.tiles_per_cta);
    __syncthreads();

    const bool fp4_path = !swa_cta && !use_cache;
    // Main tile t: cp.async gathers its rows' codes into the staging buffer (one commit
    // group) and this thread loads the 32 scale bytes of its dequant row kk = tid / 4 into
    // registers (consumed by the dequant of tile t, latency hidden behind the tile before).
    uint4 scl0 = make_uint4(0, 0, 0, 0), scl1 = make_uint4(0, 0, 0, 0);
    auto gather = [&](int t) {
        constexpr int PIECES = ROW_CODES / 16;
        const int key0 = t * DT_KEYS;
        const int rows_t = min(DT_KEYS, n_keys_kind - key0);
        for (int id = tid; id < rows_t * PIECES; id += DT_THREADS) {
            const int kk = id / PIECES, c = id - kk * PIECES;
            const int64_t grow = seq_off + sm.main_pos[key0 + kk];
            cp_async_16(smem_u32(&sm.stage[kk][16 * c]), p.codes + grow * ROW_CODES + 16 * c);
        }
        cp_async_commit();
        const int kk = tid >> 2;
        if (kk < rows_t) {
            const uint4* src = reinterpret_cast<const uint4*>(p.scales + (seq_off + sm.main_pos[key0 + kk]) * ROW_SCALES);
            scl0 = __ldg(src);
            scl1 = __ldg(src + 1);
        }
    };
    if (fp4_path && t_begin < t_end) gather(t_begin);      // overlaps the query load

    uint32_t n_load = 0;                              // completed load phases waited on
    bool load_pending = false;
    // Bounded wait on the next phase of bar by every thread; a timeout marks the CTA failed.
    auto wait_next = [&](uint64_t* bar, uint32_t& count, bool& pending) {
        if (!mbar_wait(bar, count & 1u, p.err)) sm.fail = 1;
        else {
            ++count;
            pending = false;
        }
    };

    bool q_ok;
    {
        bool q_pending = true;
        uint32_t n_q = 0;
        wait_next(&sm.bar_q, n_q, q_pending);
        q_ok = !q_pending;
    }
    if (q_ok && !bf16_tiles && t_begin < t_end) {       // the query as f16 for f16 tiles
        for (int c = tid; c < DT_Q_BYTES / 16; c += DT_THREADS) {
            uint4* qp = reinterpret_cast<uint4*>(sm.q + 16 * c);
            uint4 v = *qp;
            v.x = bf16x2_to_f16x2(v.x);
            v.y = bf16x2_to_f16x2(v.y);
            v.z = bf16x2_to_f16x2(v.z);
            v.w = bf16x2_to_f16x2(v.w);
            *qp = v;
        }
    }
    __syncthreads();

    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m_ref[2] = {-INFINITY, -INFINITY};             // heads 2w, 2w+1 (warp-uniform)
    float l_lane[2] = {0.0f, 0.0f};                      // this lane's share of their sums

    for (int t = t_begin; t < t_end && !sm.fail; ++t) {
        const int key0 = t * DT_KEYS;
        const int tile_keys = min(DT_KEYS, n_keys_kind - key0);
        // ---- 1. every warp is done with the previous tile; its cache store has read it
        if (fill_cache && tid == 0 && t > t_begin) bulk_store_wait_read();
        __syncthreads();

        // ---- 2. load the tile (FP4: its gather was issued during the previous tile)
        if (fp4_path) {
            cp_async_wait<0>();
            __syncthreads();
            // thread -> (row kk, group quad j); 8 groups of 16 channels, one per 64-dim block
            const int kk = tid >> 2, j = tid & 3;
            const bool live = kk < tile_keys;
            const uint32_t scw[8] = {scl0.x, scl0.y, scl0.z, scl0.w, scl1.x, scl1.y, scl1.z, scl1.w};
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) {
                const int grp = 4 * cb + j;                  // scale byte grp = byte j of word cb
                uint32_t w[8];
                if (live) {
                    const uint2 cw = *reinterpret_cast<const uint2*>(&sm.stage[kk][8 * grp]);
                    const __half_raw sh = __nv_cvt_fp8_to_halfraw(
                        static_cast<__nv_fp8_storage_t>((scw[cb] >> (8 * j)) & 0xFFu), __NV_E4M3);
                    const __half2 s2 = __half2half2(__half(sh));
#pragma unroll
                    for (int bi = 0; bi < 8; ++bi) {
                        uint32_t e = e2m1x2_to_f16x2(((bi < 4 ? cw.x : cw.y) >> (8 * (bi & 3))) & 0xFFu);
                        __half2 v = __hmul2(*reinterpret_cast<__half2*>(&e), s2);
                        w[bi] = *reinterpret_cast<uint32_t*>(&v);
                    }
                } else {
#pragma unroll
                    for (int bi = 0; bi < 8; ++bi) w[bi] = 0u;
                }
                uint8_t* row = sm.tile + cb * DT_BLOCK_BYTES + kk * 128;
                *reinterpret_cast<uint4*>(row + (((2 * j) ^ (kk & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
                *reinterpret_cast<uint4*>(row + (((2 * j + 1) ^ (kk & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
            }
            if (fill_cache) fence_proxy_async_smem();      // the bulk store reads the tile
            __syncthreads();
            if (fill_cache && tid == 0)
                bulk_store(p.sel_cache + (r * (TOPK / DT_KEYS) + t) * (DT_TILE_BYTES / 2), sm.tile, DT_TILE_BYTES);
            if (t + 1 < t_end) gather(t + 1);                // staging is free again
        } else if (swa8) {
            // FP8 SWA rows: E4M3 codes staged 256 bytes of each row at a time, exact E4M3 ->
            // f16 into the tile (row scale applied to the logits and to P, not here)
            if (tid < DT_KEYS) {
                const int row = key0 + tid;
                sm.swa_s[tid] = row < n_keys_kind ? __ldg(p.swa_kscale + r * p.swa_rows + row) : 0.0f;
            }
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                for (int id = tid; id < DT_KEYS * 16; id += DT_THREADS) {
                    const int kk = id >> 4, c = id & 15, row = key0 + kk;
                    const bool in = row < n_keys_kind;
                    const uint8_t* src = p.swa_kv8 + (r * p.swa_rows + (in ? row : 0)) * D + 256 * half + 16 * c;
                    cp_async_16(smem_u32(&sm.stage[kk][16 * c]), src, in ? 16 : 0);
                }
                cp_async_commit();
                cp_async_wait<0>();
                __syncthreads();
                // thread (row kk, block j): 64 codes -> 64 f16 = 8 swizzled 16-byte chunks
                const int kk = tid >> 2, j = tid & 3, cb = 4 * half + j;
                const uint4* src4 = reinterpret_cast<const uint4*>(&sm.stage[kk][64 * j]);
                uint8_t* row_out = sm.tile + cb * DT_BLOCK_BYTES + kk * 128;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint4 v = src4[q4];
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                    uint32_t o[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        o[2 * e] = e4m3x2_to_f16x2(static_cast<uint16_t>(w[e] & 0xFFFFu));
                        o[2 * e + 1] = e4m3x2_to_f16x2(static_cast<uint16_t>(w[e] >> 16));
                    }
                    *reinterpret_cast<uint4*>(row_out + (((2 * q4) ^ (kk & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<uint4*>(row_out + (((2 * q4 + 1) ^ (kk & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
                }
                __syncthreads();                          // staging is reused by the next half
            }
            if (warp == 0) {
                float mx = fmaxf(sm.swa_s[lane], sm.swa_s[lane + 32]);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
                if (lane == 0) sm.swa_smax = mx;
            }
            __syncthreads();
        } else {
            if (tid == 0) {
                fence_proxy_async_smem();                  // order earlier generic reads of the tile
                mbar_arrive_expect_tx(&sm.bar_load, DT_TILE_BYTES);
                if (use_cache) {
                    bulk_load(sm.tile, p.sel_cache + (r * (TOPK / DT_KEYS) + t) * (DT_TILE_BYTES / 2),
                              DT_TILE_BYTES, &sm.bar_load);
                } else {
                    for (int cb = 0; cb < D / 64; ++cb)
                        tma_load_3d(sm.tile + cb * DT_BLOCK_BYTES, &tmap_swa, 64 * cb, key0, static_cast<int>(r),
                                    &sm.bar_load);
                }
            }
            load_pending = true;
            wait_next(&sm.bar_load, n_load, load_pending);
            __syncthreads();
            if (sm.fail) break;
        }

        // ---- 3. S^T partials -> shared
        if (bf16_tiles) s_partial<true>(sm, warp, lane);
        else s_partial<false>(sm, warp, lane);
        __syncthreads();

        // ---- 4. softmax: warp w owns heads 2w, 2w+1; lane owns keys lane, lane+32.  The
        //      reference max m_ref (uniform in the warp) only moves when a score exceeds it
        //      by more than RESCALE_GAP (P <= e^RESCALE_GAP is still exact-width in f16 /
        //      bf16), found with one vote; row sums stay per lane until the end.
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int h = 2 * warp + hh;
            float sv[2];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int key = lane + 32 * jj;
                sv[jj] = key < tile_keys ? (sm.s2[0][key][h] + sm.s2[1][key][h]) * p.sm_scale : -INFINITY;
                if (swa8 && key < tile_keys) sv[jj] *= sm.swa_s[key];
            }
            const float lm = fmaxf(sv[0], sv[1]);
            float alpha = 1.0f;
            if (__any_sync(0xFFFFFFFFu, lm > m_ref[hh] + RESCALE_GAP)) {   // also m_ref = -inf
                float mt = lm;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, off));
                if (m_ref[hh] != -INFINITY) alpha = __expf(m_ref[hh] - mt);
                m_ref[hh] = mt;
                l_lane[hh] *= alpha;
            }
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int key = lane + 32 * jj;
                const float pv = (sv[jj] == -INFINITY) ? 0.0f : __expf(sv[jj] - m_ref[hh]);
                l_lane[hh] += pv;
                const uint32_t off = sw_chunk(HEADS, h, key >> 3) + (key & 7) * 2;
                if (swa8) {                              // P * s_key / max s: <= P, in f16
                    const float smax = sm.swa_smax;
                    const float pw = smax > 0.0f ? pv * (sm.swa_s[key] / smax) : 0.0f;
                    *reinterpret_cast<__half*>(sm.p[0] + off) = __float2half_rn(pw);
                } else if (!swa_cta) {
                    *reinterpret_cast<__half*>(sm.p[0] + off) = __float2half_rn(pv);
                } else {
                    const __nv_bfloat16 hi = __float2bfloat16_rn(pv);
                    *reinterpret_cast<__nv_bfloat16*>(sm.p[0] + off) = hi;
                    *reinterpret_cast<__nv_bfloat16*>(sm.p[1] + off) = __float2bfloat16_rn(pv - __bfloat162float(hi));
                }
            }
            if (lane == 0) {
                sm.alpha[h] = alpha;
                if (alpha != 1.0f) sm.rescale = 1;
            }
        }
        __syncthreads();

        // ---- 5. O = alpha * O + P V (alpha is 1 unless a reference max moved)
        const bool rescale = sm.rescale != 0;
        // FP8 SWA: O += smax * (P' V') is done as O = (O / smax + P' V') * smax
        const float smax = swa8 && sm.swa_smax > 0.0f ? sm.swa_smax : 1.0f;
        if (rescale || swa8) {
            const float inv = 1.0f / smax;
            const float al = (rescale ? sm.alpha[g] : 1.0f) * inv, ah = (rescale ? sm.alpha[g + 8] : 1.0f) * inv;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                o[nt][0] *= al;
                o[nt][1] *= al;
                o[nt][2] *= ah;
                o[nt][3] *= ah;
            }
        }
        if (bf16_tiles) pv<true>(sm, warp, lane, o);
        else pv<false>(sm, warp, lane, o);
        if (swa8) {
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                o[nt][0] *= smax;
                o[nt][1] *= smax;
                o[nt][2] *= smax;
                o[nt][3] *= smax;
            }
        }
        // every thread has read sm.rescale; the next tile's writers run after its first barrier
        __syncthreads();
        if (tid == 0) sm.rescale = 0;
    }

    // ---- row sums of this warp's heads; m and l of all heads into shared memory
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float l = l_lane[hh];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, off);
        if (lane == 0) {
            sm.m[2 * warp + hh] = m_ref[hh];
            sm.l[2 * warp + hh] = l;
        }
    }

    // ---- drain in-flight copies
    cp_async_wait<0>();
    if (load_pending) wait_next(&sm.bar_load, n_load, load_pending);
    if (fill_cache && tid == 0) bulk_store_wait_all();
    __syncthreads();
    const bool have = t_begin < t_end && !sm.fail && q_ok;

    // ---- push this CTA's partial into the cluster: warp w's O fragment (64-dim block w)
    //      goes to CTA w % n_split, slot (w / n_split) * n_split + rank, lane-major
    //      (lane * 32 + 4 nt + c holds o[nt][c]); m and l go to every CTA
    const uint32_t rank = cluster_ctarank();
    const int ns = p.n_split;
    cluster_sync();                                   // every CTA is done with its tile buffer
    {
        const uint32_t owner = static_cast<uint32_t>(warp % ns);
        const int slot = (warp / ns) * ns + static_cast<int>(rank);
        const uint32_t base = dsmem_addr(smem_u32(sm.tile), owner) + (slot * DT_OBLOCK_FLOATS + lane * 32) * 4;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            if (have) dsmem_st_f32x4(base + 16 * nt, o[nt][0], o[nt][1], o[nt][2], o[nt][3]);
            else dsmem_st_f32x4(base + 16 * nt, 0.0f, 0.0f, 0.0f, 0.0f);
        }
        if (tid < HEADS * ns) {
            const int h = tid & 15, dst = tid >> 4;
            const uint32_t mine = smem_u32(sm.tile) + (rank * HEADS + h) * 4;
            dsmem_st_f32(dsmem_addr(mine + DT_PM_OFFSET, static_cast<uint32_t>(dst)), have ? sm.m[h] : -INFINITY);
            dsmem_st_f32(dsmem_addr(mine + DT_PL_OFFSET, static_cast<uint32_t>(dst)), have ? sm.l[h] : 0.0f);
        }
    }
    cluster_sync();

    // ---- merge the blocks this CTA owns (w = rank + k * n_split): thread tid takes
    //      fragment float4 (lane tid / 8, nt = tid % 8) of every sender's slot
    const float* recv = reinterpret_cast<const float*>(sm.tile);
    const float (*pm)[HEADS] = reinterpret_cast<const float (*)[HEADS]>(sm.tile + DT_PM_OFFSET);
    const float (*pl)[HEADS] = reinterpret_cast<const float (*)[HEADS]>(sm.tile + DT_PL_OFFSET);
    const int src_lane = tid >> 3, nt = tid & 7;
    const int hg = src_lane >> 2, dd = 8 * nt + 2 * (src_lane & 3);     // heads hg, hg + 8
    float wa[DT_MAX_CLUSTER], wb[DT_MAX_CLUSTER];
    float inv_a, inv_b;
    {
        float Ma = -INFINITY, Mb = -INFINITY;
        for (int s2i = 0; s2i < ns; ++s2i) {
            Ma = fmaxf(Ma, pm[s2i][hg]);
            Mb = fmaxf(Mb, pm[s2i][hg + 8]);
        }
        float La = 0.0f, Lb = 0.0f;
#pragma unroll
        for (int s2i = 0; s2i < DT_MAX_CLUSTER; ++s2i) {
            wa[s2i] = (s2i < ns && pm[s2i][hg] != -INFINITY) ? __expf(pm[s2i][hg] - Ma) : 0.0f;
            wb[s2i] = (s2i < ns && pm[s2i][hg + 8] != -INFINITY) ? __expf(pm[s2i][hg + 8] - Mb) : 0.0f;
            if (s2i < ns) {
                La += wa[s2i] * pl[s2i][hg];
                Lb += wb[s2i] * pl[s2i][hg + 8];
            }
        }
        inv_a = 1.0f / La;
        inv_b = 1.0f / Lb;
    }
    for (int w = static_cast<int>(rank), k = 0; w < D / 64; w += ns, ++k) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int s2i = 0; s2i < DT_MAX_CLUSTER; ++s2i) {
            if (s2i < ns) {
                const float4 v = *reinterpret_cast<const float4*>(recv + (k * ns + s2i) * DT_OBLOCK_FLOATS + 4 * tid);
                acc.x += wa[s2i] * v.x;
                acc.y += wa[s2i] * v.y;
                acc.z += wb[s2i] * v.z;
                acc.w += wb[s2i] * v.w;
            }
        }
        float* out_r = p.out + r * HEADS * D + 64 * w + dd;
        *reinterpret_cast<float2*>(out_r + hg * D) = make_float2(acc.x * inv_a, acc.y * inv_a);
        *reinterpret_cast<float2*>(out_r + (hg + 8) * D) = make_float2(acc.z * inv_b, acc.w * inv_b);
    }
}

}  // namespace

void attend_decode_split(int64_t rows, int64_t swa_rows, int& n_split_main, int& n_split,
                         int& tiles_per_cta) {
    const int main_tiles = TOPK / DT_KEYS;
    const int swa_tiles = static_cast<int>(ceil_div(swa_rows, DT_KEYS));
    const int64_t resident = 2 * 148;           // two CTAs per SM: keep the grid to one wave
    int tpc = 1;
    for (;; ++tpc) {
        const int n = static_cast<int>(ceil_div(main_tiles, tpc) + ceil_div(swa_tiles, tpc));
        if (n <= DT_MAX_CLUSTER && (rows * n <= resident || tpc >= std::max(main_tiles, swa_tiles))) break;
    }
    tiles_per_cta = tpc;
    n_split_main = static_cast<int>(ceil_div(main_tiles, tpc));
    n_split = n_split_main + static_cast<int>(ceil_div(swa_tiles, tpc));
}

csa2_status launch_attend_decode(const AttnParams& p, const CUtensorMap& tmap_q, const CUtensorMap& tmap_swa,
                                 cudaStream_t stream) {
    const int64_t rows = p.batch;
    if (rows == 0) return CSA2_OK;
    if (p.n_split < 2 || p.n_split > DT_MAX_CLUSTER || p.n_split_main < 1) return CSA2_ERR_UNSUPPORTED;
    const int smem = static_cast<int>(sizeof(DecodeSmem) + 1024);
    if (!opt_in_smem(reinterpret_cast<const void*>(attend_decode_kernel), smem))
        return check_launch("attend_decode_kernel smem attribute");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(rows), static_cast<unsigned>(p.n_split));
    cfg.blockDim = dim3(DT_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = static_cast<unsigned>(p.n_split);
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, attend_decode_kernel, p, tmap_q, tmap_swa);
    return check_launch("attend_decode_kernel");
}

}  // namespace csa2
