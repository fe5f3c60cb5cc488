// Decode attention (one query per sequence, every position and SWA row visible) on the
// Blackwell tensor cores: tcgen05 MMAs with TMEM accumulators.
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
// one thread-block cluster; each keeps an unnormalised partial (running max m, sum l, O)
// in its shared memory and, after a cluster barrier, merges a slice of the row's output
// from all partials through distributed shared memory:
//     out = sum_s e^(m_s - M) O_s / sum_s e^(m_s - M) l_s.
//
// One 64 KB shared tile holds a tile's 64 rows x 512 dims as 64-column blocks of
// [64 rows][128 B] with the 128-byte swizzle.  The same bytes are the K-major A operand
// of S^T = K Q^T (M = 128 rows of which 64 are real, N = 16 heads, K = 512) and the
// MN-major A operand of O^T = V^T P^T (M = 128 dims per MMA, N = 16 heads, K = 64 keys),
// since key = value.  TMEM: S^T in columns 0..15, O^T in 16..79 (four 128-dim blocks).
//
//  - main tiles: cp.async gathers the rows' FP4 codes and E4M3 scales; each thread turns
//    16-channel groups into f16 (hardware e2m1 -> f16, times the e4m3 scale: exact) in
//    the tile; MMAs in f16 with the query converted to f16 (exact in the normal range).
//    With the cross-layer reuse cache a Full/Reindex layer stores each finished tile
//    (one bulk copy) and Reuse layers load it back with one bulk copy.
//  - SWA tiles: TMA loads the bf16 rows straight into the tile; MMAs in bf16 with the
//    bf16 query (exact); P is split into bf16 hi + lo pieces, so P V keeps ~16 bits.
//  - softmax: the S^T columns are read from TMEM, transposed through shared memory and
//    reduced per head by all 8 warps; when a head's running max grows, its O^T column is
//    rescaled in TMEM before the next P V.
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
constexpr int DT_STAGE_ROW = ROW_CODES + ROW_SCALES;      // 288 B per FP4 row
constexpr int DT_P_BYTES = HEADS * DT_KEYS * 2;           // 2 KB
constexpr int DT_TMEM_COLS = 128;                         // S^T: 0..15, O^T: 16..79
constexpr int DT_S_LD = DT_KEYS + 1;
constexpr int DT_MAX_CLUSTER = 8;                      // portable cluster size

struct alignas(1024) DecodeSmem {
    uint8_t tile[DT_TILE_BYTES];          // SW128 [8][64 rows][128 B]
    uint8_t q[DT_Q_BYTES];                // SW128 [8][16 heads][128 B]; also read (unused
                                          // rows) by the M = 128 S MMA of the last block
    union {
        uint8_t stage[DT_KEYS][DT_STAGE_ROW];   // gathered FP4 rows: codes | scales
        struct {
            uint8_t p[2][DT_P_BYTES];     // P (f16) or P hi / lo (bf16): SW128 [16][64]
            float s_t[HEADS][DT_S_LD];    // S transposed, scaled
        } sm;
    } u;
    int32_t main_pos[TOPK];
    float m[HEADS], l[HEADS], alpha[HEADS];
    float pm[HEADS], pl[HEADS];           // this CTA's partial max / sum, read by the cluster
    int32_t warp_cnt[DT_WARPS];
    uint64_t bar_q, bar_load, bar_mma;
    uint32_t tmem;
    int rescale, fail;
};

static_assert(offsetof(DecodeSmem, u) % 1024 == 0, "P tiles need 1024-byte alignment");
static_assert(sizeof(DecodeSmem) + 1024 <= 113 * 1024, "two CTAs must fit on one SM");

__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    const __half2_raw h = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(byte), __NV_E2M1);
    return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
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
    const bool swa_cta = sp >= p.n_split_main;
    const int64_t seq_off = p.kv_offsets[r];
    const int64_t n_b = p.kv_offsets[r + 1] - seq_off;
    const bool use_cache = !swa_cta && p.cache_mode == CSA2_CACHE_USE;
    const bool fill_cache = !swa_cta && p.cache_mode == CSA2_CACHE_FILL;

    if (tid == 0) {
        mbar_init(&sm.bar_q, 1);
        mbar_init(&sm.bar_load, 1);
        mbar_init(&sm.bar_mma, 1);
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
    if (warp == 0) tmem_alloc(&sm.tmem, DT_TMEM_COLS);

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

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = sm.tmem;

    uint32_t n_load = 0, n_mma = 0;                   // completed phases waited on so far
    bool load_pending = false, mma_pending = false;
    // Bounded wait on the next phase of bar by every thread; a timeout marks the CTA failed.
    auto wait_next = [&](uint64_t* bar, uint32_t& count, bool& pending) {
        if (!mbar_wait(bar, count & 1u, p.err)) sm.fail = 1;
        else {
            ++count;
            pending = false;
        }
    };

    bool q_ok = true;
    {
        bool q_pending = true;
        uint32_t n_q = 0;
        wait_next(&sm.bar_q, n_q, q_pending);
        q_ok = !q_pending;
    }
    if (q_ok && !swa_cta && t_begin < t_end) {          // the query as f16 for the main MMAs
        for (int c = tid; c < DT_Q_BYTES / 16; c += DT_THREADS) {
            uint4* qp = reinterpret_cast<uint4*>(sm.q + 16 * c);
            uint4 v = *qp;
            v.x = bf16x2_to_f16x2(v.x);
            v.y = bf16x2_to_f16x2(v.y);
            v.z = bf16x2_to_f16x2(v.z);
            v.w = bf16x2_to_f16x2(v.w);
            *qp = v;
        }
        fence_proxy_async_smem();
    }
    __syncthreads();

    const uint32_t tile_s = smem_u32(sm.tile);
    const uint32_t q_s = smem_u32(sm.q);
    const uint32_t p_s0 = smem_u32(sm.u.sm.p[0]);
    const uint32_t p_s1 = smem_u32(sm.u.sm.p[1]);
    const uint32_t id_s = idesc_f16_f32(128, HEADS, swa_cta, false);
    const uint32_t id_o = idesc_f16_f32(128, HEADS, swa_cta, true);
    const uint32_t lane_quarter = static_cast<uint32_t>(32 * (warp & 3)) << 16;

    for (int t = t_begin; t < t_end && !sm.fail; ++t) {
        const int key0 = t * DT_KEYS;
        const int tile_keys = min(DT_KEYS, n_keys_kind - key0);
        // ---- 1. the previous tile's P V must be done before its tile / P are overwritten
        if (mma_pending) wait_next(&sm.bar_mma, n_mma, mma_pending);
        if (fill_cache && tid == 0 && t > t_begin) bulk_store_wait_read();
        __syncthreads();
        if (sm.fail) break;

        // ---- 2. load the tile
        if (!swa_cta && !use_cache) {
            constexpr int PIECES = DT_STAGE_ROW / 16;      // 16 code + 2 scale pieces per row
            for (int id = tid; id < tile_keys * PIECES; id += DT_THREADS) {
                const int kk = id / PIECES, c = id - kk * PIECES;
                const int64_t grow = seq_off + sm.main_pos[key0 + kk];
                const uint8_t* src = c < ROW_CODES / 16 ? p.codes + grow * ROW_CODES + 16 * c
                                                        : p.scales + grow * ROW_SCALES + 16 * (c - ROW_CODES / 16);
                cp_async_16(smem_u32(&sm.u.stage[kk][16 * c]), src);
            }
            cp_async_commit();
            cp_async_wait<0>();
            __syncthreads();
            // thread -> (row kk, group quad j); 8 groups of 16 channels, one per 64-dim block
            const int kk = tid >> 2, j = tid & 3;
            const bool live = kk < tile_keys;
#pragma unroll 2
            for (int cb = 0; cb < D / 64; ++cb) {
                const int grp = 4 * cb + j;
                uint32_t w[8];
                if (live) {
                    const uint2 cw = *reinterpret_cast<const uint2*>(&sm.u.stage[kk][8 * grp]);
                    const __half_raw sh = __nv_cvt_fp8_to_halfraw(
                        static_cast<__nv_fp8_storage_t>(sm.u.stage[kk][ROW_CODES + grp]), __NV_E4M3);
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
            fence_proxy_async_smem();
            __syncthreads();
            if (fill_cache && tid == 0)
                bulk_store(p.sel_cache + (r * (TOPK / DT_KEYS) + t) * (DT_TILE_BYTES / 2), sm.tile, DT_TILE_BYTES);
        } else {
            if (tid == 0) {
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

        // ---- 3. S^T = K Q^T into TMEM columns 0..15
        if (tid == 0) {
            tc_fence_after();
#pragma unroll 1
            for (int cb = 0; cb < D / 64; ++cb) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t a = umma_desc_sw128(tile_s + cb * DT_BLOCK_BYTES + ks * 32, 16, 1024);
                    const uint64_t b = umma_desc_sw128(q_s + cb * HEADS * 128 + ks * 32, 16, 1024);
                    mma_f16(tm, a, b, id_s, (cb | ks) != 0);
                }
            }
            mma_commit(&sm.bar_mma);
        }
        mma_pending = true;
        wait_next(&sm.bar_mma, n_mma, mma_pending);
        tc_fence_after();

        // ---- 4. softmax: scaled S^T -> shared (transposed), then two heads per warp
        if (warp < 2 && !mma_pending) {
            uint32_t v[16];
            tmem_ld16(tm + lane_quarter, v);
            const int key = 32 * warp + lane;
            const bool live = key < tile_keys;
#pragma unroll
            for (int h = 0; h < HEADS; ++h)
                sm.u.sm.s_t[h][key] = live ? __uint_as_float(v[h]) * p.sm_scale : -INFINITY;
        }
        __syncthreads();
        if (sm.fail) break;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int h = 2 * warp + hh;
            const float sv0 = sm.u.sm.s_t[h][lane], sv1 = sm.u.sm.s_t[h][lane + 32];
            float mt = fmaxf(sv0, sv1);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, off));
            const float m_old = sm.m[h];
            const float m_new = fmaxf(m_old, mt);
            const float alpha = (m_new == -INFINITY) ? 1.0f : __expf(m_old - m_new);
            const float p0 = (sv0 == -INFINITY) ? 0.0f : __expf(sv0 - m_new);
            const float p1 = (sv1 == -INFINITY) ? 0.0f : __expf(sv1 - m_new);
            float sum = p0 + p1;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
            const uint32_t o0 = sw128_offset(HEADS, h, lane), o1 = sw128_offset(HEADS, h, lane + 32);
            if (!swa_cta) {
                *reinterpret_cast<__half*>(sm.u.sm.p[0] + o0) = __float2half_rn(p0);
                *reinterpret_cast<__half*>(sm.u.sm.p[0] + o1) = __float2half_rn(p1);
            } else {
                const __nv_bfloat16 h0 = __float2bfloat16_rn(p0), h1 = __float2bfloat16_rn(p1);
                *reinterpret_cast<__nv_bfloat16*>(sm.u.sm.p[0] + o0) = h0;
                *reinterpret_cast<__nv_bfloat16*>(sm.u.sm.p[0] + o1) = h1;
                *reinterpret_cast<__nv_bfloat16*>(sm.u.sm.p[1] + o0) = __float2bfloat16_rn(p0 - __bfloat162float(h0));
                *reinterpret_cast<__nv_bfloat16*>(sm.u.sm.p[1] + o1) = __float2bfloat16_rn(p1 - __bfloat162float(h1));
            }
            __syncwarp();
            if (lane == 0) {
                sm.m[h] = m_new;
                sm.alpha[h] = alpha;
                sm.l[h] = alpha * sm.l[h] + sum;
                if (alpha != 1.0f) sm.rescale = 1;
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- 5. rescale O^T columns whose max grew (the previous P V has completed)
        if (t > t_begin && sm.rescale) {
            const uint32_t taddr = tm + lane_quarter + 16 + 32 * (warp >> 2);
            uint32_t v[32];
            tmem_ld32(taddr, v);
#pragma unroll
            for (int c = 0; c < 32; ++c) v[c] = __float_as_uint(__uint_as_float(v[c]) * sm.alpha[c & 15]);
            tmem_st32(taddr, v);
            tc_fence_before();
        }
        __syncthreads();

        // ---- 6. O^T += V^T P^T (bf16 tiles: P in hi and lo pieces)
        if (tid == 0) {
            tc_fence_after();
            sm.rescale = 0;
#pragma unroll 1
            for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t a = umma_desc_sw128(tile_s + 2 * mb * DT_BLOCK_BYTES + ks * 2048,
                                                       DT_BLOCK_BYTES, 1024);
                    mma_f16(tm + 16 + 16 * mb, a, umma_desc_sw128(p_s0 + ks * 32, 16, 1024), id_o,
                            t > t_begin || ks > 0);
                    if (swa_cta)
                        mma_f16(tm + 16 + 16 * mb, a, umma_desc_sw128(p_s1 + ks * 32, 16, 1024), id_o, true);
                }
            }
            mma_commit(&sm.bar_mma);
        }
        mma_pending = true;
    }

    // ---- drain: the last P V, in-flight loads and cache stores
    if (mma_pending) wait_next(&sm.bar_mma, n_mma, mma_pending);
    if (load_pending) wait_next(&sm.bar_load, n_load, load_pending);
    if (fill_cache && tid == 0) bulk_store_wait_all();
    tc_fence_after();
    __syncthreads();
    const bool have = t_begin < t_end && !sm.fail && q_ok;

    // ---- partial (or final) output from TMEM: thread = one dim of a 128-dim block
    const int mb0 = 2 * (warp >> 2);
    uint32_t v[32];
    if (have) {
        tmem_ld32(tm + lane_quarter + 16 + 32 * (warp >> 2), v);
    } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = 0u;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, DT_TMEM_COLS);

    // ---- this CTA's partial into its own shared memory ([16][512] fp32 in the free tile)
    float* o_part = reinterpret_cast<float*>(sm.tile);
    const int dim_in = 32 * (warp & 3) + lane;
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        const int h = c & 15, dim = 128 * (mb0 + (c >> 4)) + dim_in;
        o_part[h * D + dim] = __uint_as_float(v[c]);
    }
    if (tid < HEADS) {
        sm.pm[tid] = have ? sm.m[tid] : -INFINITY;
        sm.pl[tid] = have ? sm.l[tid] : 0.0f;
    }
    cluster_sync();

    // ---- cluster merge: CTA `rank` writes float4 chunks rank, rank + n_split, ... of the
    //      row's [16][512] output, reading every CTA's partial through DSMEM
    const uint32_t rank = cluster_ctarank();
    const int ns = p.n_split;
    uint32_t o_base[DT_MAX_CLUSTER], m_base[DT_MAX_CLUSTER], l_base[DT_MAX_CLUSTER];
#pragma unroll
    for (int s = 0; s < DT_MAX_CLUSTER; ++s) {
        const uint32_t peer = static_cast<uint32_t>(s < ns ? s : 0);
        o_base[s] = dsmem_addr(smem_u32(o_part), peer);
        m_base[s] = dsmem_addr(smem_u32(sm.pm), peer);
        l_base[s] = dsmem_addr(smem_u32(sm.pl), peer);
    }
    constexpr int CHUNKS = HEADS * D / 4;
    for (int i = static_cast<int>(rank) + ns * tid; i < CHUNKS; i += ns * DT_THREADS) {
        const int h = i / (D / 4);
        float ms[DT_MAX_CLUSTER], ls[DT_MAX_CLUSTER];
        float4 os[DT_MAX_CLUSTER];
#pragma unroll
        for (int s = 0; s < DT_MAX_CLUSTER; ++s) {     // all loads in flight at once
            if (s < ns) {
                ms[s] = dsmem_ld_f32(m_base[s] + 4 * h);
                ls[s] = dsmem_ld_f32(l_base[s] + 4 * h);
                os[s] = dsmem_ld_f32x4(o_base[s] + 16 * i);
            }
        }
        float M = -INFINITY;
#pragma unroll
        for (int s = 0; s < DT_MAX_CLUSTER; ++s)
            if (s < ns) M = fmaxf(M, ms[s]);
        float L = 0.0f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int s = 0; s < DT_MAX_CLUSTER; ++s) {
            if (s < ns && ms[s] != -INFINITY) {
                const float wgt = __expf(ms[s] - M);
                L += wgt * ls[s];
                acc.x += wgt * os[s].x;
                acc.y += wgt * os[s].y;
                acc.z += wgt * os[s].z;
                acc.w += wgt * os[s].w;
            }
        }
        const float inv = 1.0f / L;
        *reinterpret_cast<float4*>(p.out + r * HEADS * D + 4 * i) =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
    cluster_sync();                                   // peers may still be reading this CTA
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
