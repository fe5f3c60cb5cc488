// Chunked-prefill indexer of a Full layer: scores and Top-512 of many queries per
// sequence, fused, with no score matrix.
//
// CSA2 section of the thecryptopost.io DeepSeek-V4.1-Flash article: a Full layer scores
// the context with its indexer and picks a new Top-512 per query; in the encoder every
// query sees the compressed positions that end at or before its token.  Score (the pages
// give no formula):
//     score(t, s) = kscale[s] * sum_h w[t,h] * ReLU(q[t,h] . e4m3(k8[s])),
// and the Top-512 keeps the largest scores, ties to the lower position, ascending.
//
// prefill_index_kernel: one CTA per (block of 16 queries, sequence).  The prefill indexer
// is a real contraction (2,048 queries x 4 heads x 64 dims against every position of the
// sequence), so it runs on tcgen05:
//  - warp 0 streams 128-position FP8 K tiles (8 KB, 64-byte swizzle) with TMA into an
//    8-stage ring (a stage is free again once its MMAs complete; the epilogue threads
//    read their positions' row scales from global memory two tiles ahead);
//  - warp 1 owns the 512 TMEM columns (four accumulators) and issues
//    tcgen05.mma.kind::f8f6f4 with M = 128 positions, N = 128 columns (16 queries x 4
//    heads x 2 pieces) and K = 64: each bf16 query head is split exactly into two E4M3
//    pieces under a power-of-two scale, p1 + p2 / 16 (the split the decode scan uses);
//  - warps 2-17 read the accumulator back (tcgen05.ld; warp w reads TMEM lanes
//    32 (w % 4) .., four warps per group of 4 queries: 32 columns per warp and tile),
//    form each visible position's score and keep a streaming Top-512 per query in shared
//    memory.
// Streaming Top-512: each query has a buffer of up to 1,024 (score, position) candidates
// kept in position order and a threshold (-inf until the first compaction).  A tile
// appends the positions whose score beats the threshold, in position order (ballots, and
// per-quadrant counts exchanged between the four warps of a query group); when a buffer
// could overflow on the next tile, one warp compacts it: a bound T with 512 .. 640
// candidates at or above it (from 32 sorted samples and counting passes) becomes the
// threshold and only candidates >= T stay.  At least 512 kept candidates then score >= T and come
// earlier, so a later position with a score <= T can never enter the Top-512: only
// strictly larger scores are appended afterwards.  At the end each buffer's exact Top-512
// (four radix passes, ties to the lower position, i.e. the earlier entry) is written in
// buffer order, which is ascending position order.
// Every mbarrier wait is bounded (ERR_TIMEOUT set, no hang); after a failed wait a warp
// stops waiting but keeps taking part in the named barriers, so no warp waits forever.
#include "common.cuh"
#include "kernels.cuh"
#include "select.cuh"
#include "tc.cuh"

namespace csa2 {

namespace {

constexpr int PI_QB = 16;                      // queries per CTA
constexpr int PI_N = PI_QB * 8;                // MMA columns: query q, piece p, head h -> 8q + 4p + h
constexpr int PI_TILE = 128;                   // positions per tile (MMA M)
constexpr int PI_STAGES = 8;
constexpr int PI_EPI_WARPS = 16;
constexpr int PI_THREADS = 64 + 32 * PI_EPI_WARPS;   // warp 0: TMA, warp 1: MMA, 2..17: epilogue
constexpr int PI_QPW = 4;                      // queries per epilogue warp (one TMEM load of 32 columns)
constexpr int PI_CAP = 1024;                   // candidates per query
constexpr int PI_COMPACT_AT = PI_CAP - PI_TILE;   // compact before a tile could overflow
constexpr int PI_ACC = 4;                      // TMEM accumulators (the MMA runs up to 3 tiles ahead)
constexpr int PI_TMEM_COLS = PI_ACC * PI_N;    // all 512 columns (one CTA per SM)
constexpr int PI_TILE_BYTES = PI_TILE * IDX_DIM;

struct __align__(1024) PiShared {
    uint8_t a[PI_STAGES][PI_TILE_BYTES];       // FP8 K tiles (64-byte swizzle), 1 KB aligned
    uint8_t b[PI_N * IDX_DIM];                 // query pieces (64-byte swizzle)
    float cs[PI_QB][PI_CAP];                   // candidate scores, position order
    int32_t cp[PI_QB][PI_CAP];                 // candidate positions
    uint32_t hist[PI_EPI_WARPS][256];          // per-warp radix histograms
    float wq[PI_QB][IDX_HEADS];                // head weight times 2^-s
    int qsh[PI_QB][IDX_HEADS];                 // s of each query head
    int64_t lim[PI_QB];                        // visible positions of each query
    float thr[PI_QB];                          // append threshold (strict)
    int cnt[PI_QB];                            // candidates held
    int wcnt[4][PI_QB];                        // a tile's appends per TMEM quadrant
    uint64_t full[PI_STAGES], empty[PI_STAGES], tfull[PI_ACC], tempty[PI_ACC];
    uint32_t tmem;
    int fail;
};

// The k-th best (k >= 1) of the n candidates of one buffer, by (score desc, position asc)
// where buffer order is position order, found 8 key bits per pass from the top.  With
// all 4 passes: T is the key of the k-th best score and need_eq how many of the entries
// with key T are kept (the first ones in buffer order).  With fewer passes: T is the
// lowest key of the bin holding the k-th best, a lower bound of it (need_eq is then
// meaningless: every entry >= T is kept).  One warp; hist is this warp's 256-bin scratch;
// lanes with equal bins add once (__match_any_sync), so a crowded bin does not serialise.
__device__ __forceinline__ void warp_kth(const float* cs, int n, int k, uint32_t* hist, int passes, uint32_t& T,
                                         int& need_eq) {
    const int lane = threadIdx.x & 31;
    uint32_t prefix = 0, mask = 0;
    int rem = k;                                 // rank still to find among keys matching prefix
    for (int pass = 0; pass < passes; ++pass) {
        const int shift = 24 - 8 * pass;
#pragma unroll
        for (int j = 0; j < 8; ++j) hist[lane * 8 + j] = 0;
        __syncwarp();
        for (int i0 = 0; i0 < n; i0 += 32) {
            const int i = i0 + lane;
            const uint32_t key = i < n ? score_key(cs[i]) : 0u;
            const bool in = i < n && (key & mask) == prefix;
            const uint32_t bin = in ? ((key >> shift) & 255u) : 256u;
            const unsigned same = __match_any_sync(0xFFFFFFFFu, bin);
            if (in && (__ffs(same) - 1) == lane) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(same)));
        }
        __syncwarp();
        // lane owns bins 8*lane .. 8*lane+7
        uint32_t c[8];
        uint32_t mine = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            c[j] = hist[lane * 8 + j];
            mine += c[j];
        }
        uint32_t suf = mine;                     // inclusive suffix sum over lanes ...
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, suf, off);
            if (lane + off < 32) suf += y;
        }
        suf -= mine;                             // ... made exclusive: keys in higher bins
        // the bin holding rank rem: the lane whose suffix range covers it
        int found_bin = -1;
        uint32_t cum_above = 0;
        if (suf < static_cast<uint32_t>(rem) && suf + mine >= static_cast<uint32_t>(rem)) {
            uint32_t acc = suf;
#pragma unroll
            for (int j = 7; j >= 0; --j) {
                if (found_bin < 0 && acc + c[j] >= static_cast<uint32_t>(rem)) {
                    found_bin = lane * 8 + j;
                    cum_above = acc;
                }
                acc += c[j];
            }
        }
        const unsigned who = __ballot_sync(0xFFFFFFFFu, found_bin >= 0);
        const int src = who ? __ffs(who) - 1 : 0;         // (always found: rem <= matching keys)
        const int bin = max(0, __shfl_sync(0xFFFFFFFFu, found_bin, src));
        const uint32_t ab = __shfl_sync(0xFFFFFFFFu, cum_above, src);
        prefix |= static_cast<uint32_t>(bin) << shift;
        mask |= 255u << shift;
        rem -= static_cast<int>(ab);
        __syncwarp();
    }
    T = prefix;
    need_eq = passes == 4 ? rem : INT32_MAX;
}

// Keeps, in place and in order, the entries with key > T and the first need_eq entries
// with key == T; returns how many remain.  One warp.
__device__ __forceinline__ int warp_compact(float* cs, int32_t* cp, int n, uint32_t T, int need_eq) {
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    int kept = 0, eq_seen = 0;
    for (int base = 0; base < n; base += 128) {          // 4 chunks of 32 per round, read first
        float s[4];
        int32_t pos[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + 32 * u + lane;
            s[u] = i < n ? cs[i] : -INFINITY;
            pos[u] = i < n ? cp[i] : -1;
        }
        __syncwarp();                                    // every lane has read before any writes
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + 32 * u + lane;
            const bool in = i < n;
            const uint32_t key = in ? score_key(s[u]) : 0u;
            const bool eq = in && key == T;
            const unsigned eqm = __ballot_sync(0xFFFFFFFFu, eq);
            const int eq_rank = eq_seen + __popc(eqm & lt);
            const bool keep = in && (key > T || (eq && eq_rank < need_eq));
            const unsigned km = __ballot_sync(0xFFFFFFFFu, keep);
            if (keep) {
                const int o = kept + __popc(km & lt);
                cs[o] = s[u];
                cp[o] = pos[u];
            }
            kept += __popc(km);
            eq_seen += __popc(eqm);
        }
        __syncwarp();
    }
    return kept;
}

// A key T with at least `k` and at most `most` of the n candidates at or above it (k <=
// most, n > most), found without atomics: 32 samples of the buffer sorted across the warp
// give candidate bounds, and counting passes (ballots) test them; if no sample bound fits,
// the exact k-th key (four radix passes) is returned.  One warp.
__device__ __forceinline__ uint32_t warp_bound(const float* cs, int n, int k, int most, uint32_t* hist) {
    const int lane = threadIdx.x & 31;
    // sample lane: entry lane * n / 32, sorted descending across the warp (bitonic)
    uint32_t v = score_key(cs[(lane * n) >> 5]);
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const uint32_t o = __shfl_xor_sync(0xFFFFFFFFu, v, stride);
            const bool up = ((lane & size) == 0);            // descending runs first
            const bool lower = (lane & stride) == 0;
            const uint32_t hi = max(v, o), lo = min(v, o);
            v = (lower == up) ? hi : lo;
        }
    }
    // v at lane j is the (j+1)-th largest sample: about (j+1) n / 32 candidates are >= it;
    // start from the first sample expected to reach k and move by one sample at a time
    int j = max(0, min(31, (k * 32) / n));
    for (int tries = 0; tries < 6; ++tries) {
        const uint32_t b = __shfl_sync(0xFFFFFFFFu, v, j);
        int c = 0;
        for (int base = 0; base < n; base += 128) {
            float x[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) x[u] = base + 32 * u + lane < n ? cs[base + 32 * u + lane] : -INFINITY;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                c += __popc(__ballot_sync(0xFFFFFFFFu, base + 32 * u + lane < n && score_key(x[u]) >= b));
        }
        if (c >= k && c <= most) return b;
        if (c < k) {
            if (j == 31) break;
            ++j;
        } else {
            if (j == 0) break;
            --j;
        }
    }
    uint32_t T;
    int need_eq;
    warp_kth(cs, n, k, hist, 4, T, need_eq);
    return T;
}

__global__ void __launch_bounds__(PI_THREADS, 1)
prefill_index_kernel(const __grid_constant__ CUtensorMap tmap, IndexParams p, int32_t* __restrict__ topk_out,
                     unsigned* err) {
    extern __shared__ uint8_t smem_raw[];
    PiShared& sm = *reinterpret_cast<PiShared*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int b = blockIdx.y;
    const int q0 = blockIdx.x * PI_QB;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < PI_STAGES; ++s) {
            mbar_init(&sm.full[s], 1);           // the TMA's expect_tx
            mbar_init(&sm.empty[s], 1);          // the MMA's commit
        }
        for (int j = 0; j < PI_ACC; ++j) {
            mbar_init(&sm.tfull[j], 1);
            mbar_init(&sm.tempty[j], PI_EPI_WARPS);
        }
        mbar_fence_init();
        sm.fail = 0;
    }
    if (warp == 1) tmem_alloc(&sm.tmem, PI_TMEM_COLS);
    __syncthreads();
    griddep_launch_dependents();
    griddep_wait();

    const int64_t seq_off = p.kv_offsets[b];
    const int64_t n_b = p.kv_offsets[b + 1] - seq_off;
    const uint32_t limit = wait_limit(err);
    // ---- per query: visible positions, head scales s (max|q_h| * 2^s in [128, 256)), weights
    if (tid < PI_QB) {
        const int qq = tid;
        int64_t lim = 0;
        if (q0 + qq < p.q_per_seq) {
            lim = n_b;
            if (p.q_pos) {
                const int64_t t = p.q_pos[b] + q0 + qq;
                lim = min(n_b, max(static_cast<int64_t>(0), (t + 1) / p.ratio));
            }
        }
        sm.lim[qq] = lim;
        sm.thr[qq] = -INFINITY;
        sm.cnt[qq] = 0;
    }
    if (warp >= 2) {                             // 16 warps x 4 (query, head) pairs each
        const int e = warp - 2;
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
            const int pair = e * 4 + k;          // 64 pairs = 16 queries x 4 heads
            const int qq = pair >> 2, h = pair & 3;
            const int64_t row = static_cast<int64_t>(b) * p.q_per_seq + q0 + qq;
            float m = 0.0f;
            if (q0 + qq < p.q_per_seq) {
                const uint32_t two = *reinterpret_cast<const uint32_t*>(p.idx_q + (row * IDX_HEADS + h) * IDX_DIM + 2 * lane);
                m = fmaxf(fabsf(__uint_as_float(two << 16)), fabsf(__uint_as_float(two & 0xFFFF0000u)));
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
            if (lane == 0) {
                int ex = 0;
                frexpf(m, &ex);
                const int sh = (m > 0.0f) ? 8 - ex : 0;
                sm.qsh[qq][h] = sh;
                sm.wq[qq][h] = (q0 + qq < p.q_per_seq) ? ldexpf(p.idx_w[row * IDX_HEADS + h], -sh) : 0.0f;
            }
        }
    }
    __syncthreads();
    // ---- query pieces: row 8 qq + h = p1 of head h, row 8 qq + 4 + h = p2 (q 2^s = p1 + p2/16)
    for (int i = tid; i < PI_N * IDX_DIM; i += PI_THREADS) {
        const int n = i / IDX_DIM, k = i % IDX_DIM;
        const int qq = n >> 3, piece = (n >> 2) & 1, h = n & 3;
        uint32_t code = 0;
        if (q0 + qq < p.q_per_seq) {
            const int64_t row = static_cast<int64_t>(b) * p.q_per_seq + q0 + qq;
            const float x = ldexpf(bf16_bits_to_float(p.idx_q[(row * IDX_HEADS + h) * IDX_DIM + k]), sm.qsh[qq][h]);
            const uint32_t c1 = e4m3_encode_rne_sat(fabsf(x)) | (x < 0.0f ? 0x80u : 0u);
            code = c1;
            if (piece) {
                const float r = x - e4m3_to_float(static_cast<uint8_t>(c1));   // exact
                code = e4m3_encode_rne_sat(fabsf(r) * 16.0f) | (r < 0.0f ? 0x80u : 0u);
            }
        }
        sm.b[sw64_offset(n, k)] = static_cast<uint8_t>(code);
    }
    fence_proxy_async_smem();                    // query pieces -> tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    int64_t lim_top = 0;
    for (int qq = 0; qq < PI_QB; ++qq) lim_top = max(lim_top, sm.lim[qq]);
    const int n_tiles = static_cast<int>((lim_top + PI_TILE - 1) / PI_TILE);

    if (warp == 0) {
        // ---- producer: K tiles (TMA)
        int issued = 0;
        for (int it = 0; it < n_tiles; ++it, ++issued) {
            const int s = it % PI_STAGES;
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&sm.empty[s], ((it / PI_STAGES) & 1) ^ 1, err, limit);
            if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&sm.full[s], PI_TILE_BYTES);
                tma_load_2d(sm.a[s], &tmap, 0, static_cast<int>(p.rows.row(b, seq_off, static_cast<int64_t>(it) * PI_TILE)),
                            &sm.full[s]);
            }
        }
        if (lane == 0) {                                    // the issued tiles landed
            for (int it = max(0, issued - PI_STAGES); it < issued; ++it)
                mbar_wait(&sm.full[it % PI_STAGES], (it / PI_STAGES) & 1, err);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer: D[buf] = K_tile * pieces^T over K = 64 (two K = 32 steps)
            const uint32_t idesc = idesc_e4m3_f32(PI_TILE, PI_N);
            const uint64_t bdesc = umma_desc_sw64(smem_u32(sm.b));
            int done = 0;
            for (int it = 0; it < n_tiles; ++it) {
                const int s = it % PI_STAGES, buf = it % PI_ACC;
                if (!mbar_wait(&sm.full[s], (it / PI_STAGES) & 1, err, limit)) break;
                if (!mbar_wait(&sm.tempty[buf], ((it / PI_ACC) & 1) ^ 1, err, limit)) break;
                tc_fence_after();
                const uint64_t adesc = umma_desc_sw64(smem_u32(sm.a[s]));
                const uint32_t d = tmem + buf * PI_N;
                mma_e4m3(d, adesc, bdesc, idesc, false);
                mma_e4m3(d, adesc + 2, bdesc + 2, idesc, true);       // +32 bytes of K
                mma_commit(&sm.empty[s]);
                mma_commit(&sm.tfull[buf]);
                ++done;
            }
            if (done > 0) mbar_wait(&sm.tfull[(done - 1) % PI_ACC], ((done - 1) / PI_ACC) & 1, err);
        }
        __syncwarp();
    } else {
        // ---- epilogue: warp (quadrant qd, quarter hq) = TMEM lanes 32 qd .., queries 4 hq ..
        const int e = warp - 2;
        const int qd = warp & 3, hq = e >> 2;
        const int bar_id = 1 + hq;
        const int row = 32 * qd + lane;
        const unsigned lt = (1u << lane) - 1u;
        uint32_t* hist = sm.hist[e];
        float wq[PI_QPW][IDX_HEADS], thr[PI_QPW];
        int64_t lim[PI_QPW];
        int64_t lim_min = INT64_MAX;
#pragma unroll
        for (int k = 0; k < PI_QPW; ++k) {
            const int qq = PI_QPW * hq + k;
#pragma unroll
            for (int h = 0; h < IDX_HEADS; ++h) wq[k][h] = sm.wq[qq][h];
            thr[k] = -INFINITY;
            lim[k] = sm.lim[qq];
            lim_min = min(lim_min, lim[k]);
        }
        // this thread's row scale of tile it, loaded two tiles ahead
        const auto row_scale = [&](int it) {
            const int64_t pos = static_cast<int64_t>(it) * PI_TILE + row;
            return (it < n_tiles && pos < n_b) ? __ldg(p.idx_kscale + p.rows.row(b, seq_off, pos)) : 0.0f;
        };
        float ks_a = row_scale(0), ks_b = row_scale(1);
        bool failed = false;
        for (int it = 0; it < n_tiles; ++it) {
            const int buf = it % PI_ACC;
            failed = failed || sm.fail;
            const bool ok = !failed && __all_sync(0xFFFFFFFFu, mbar_wait(&sm.tfull[buf], (it / PI_ACC) & 1, err, limit));
            const float ks = ks_a;
            ks_a = ks_b;
            ks_b = row_scale(it + 2);
            if (!ok && !failed) {
                failed = true;
                sm.fail = 1;
            }
            unsigned pass[PI_QPW] = {};
            float sc[PI_QPW];
            const int64_t pos = static_cast<int64_t>(it) * PI_TILE + row;
            if (!failed) {
                tc_fence_after();
                uint32_t v[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(32 * qd) << 16) + buf * PI_N + 32 * hq, v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.tempty[buf]);
                const bool all_vis = static_cast<int64_t>(it + 1) * PI_TILE <= lim_min;
#pragma unroll
                for (int k = 0; k < PI_QPW; ++k) {
                    float x = 0.0f;
#pragma unroll
                    for (int h = 0; h < IDX_HEADS; ++h) {
                        const float d = __uint_as_float(v[8 * k + h]) + 0.0625f * __uint_as_float(v[8 * k + 4 + h]);
                        x += wq[k][h] * fmaxf(d, 0.0f);
                    }
                    sc[k] = ks * x;
                    pass[k] = __ballot_sync(0xFFFFFFFFu, (all_vis || pos < lim[k]) && sc[k] > thr[k]);
                }
            }
#pragma unroll
            for (int k = 0; k < PI_QPW; ++k)
                if (lane == k) sm.wcnt[qd][PI_QPW * hq + k] = __popc(pass[k]);
            named_barrier(bar_id, 128);                              // A: the tile's counts
            int tot[PI_QPW];
#pragma unroll
            for (int k = 0; k < PI_QPW; ++k) {
                const int qq = PI_QPW * hq + k;
                const int c0 = sm.cnt[qq];
                const int w0 = sm.wcnt[0][qq], w1 = sm.wcnt[1][qq], w2 = sm.wcnt[2][qq], w3 = sm.wcnt[3][qq];
                const int before = c0 + (qd > 0 ? w0 : 0) + (qd > 1 ? w1 : 0) + (qd > 2 ? w2 : 0);
                tot[k] = c0 + w0 + w1 + w2 + w3;
                if (pass[k] & (1u << lane)) {
                    const int o = before + __popc(pass[k] & lt);
                    sm.cs[qq][o] = sc[k];
                    sm.cp[qq][o] = static_cast<int32_t>(pos);
                }
            }
            named_barrier(bar_id, 128);                              // B: the tile's appends
            bool any = false;
#pragma unroll
            for (int k = 0; k < PI_QPW; ++k) any |= tot[k] > PI_COMPACT_AT;
            if (any) {
                // warp qd compacts query 4 hq + qd if it needs it: keep every candidate at or
                // above a bound T with 512 .. 640 candidates >= T (so T is at most the 512th
                // score), and append only larger scores from now on
                const int qq = PI_QPW * hq + qd;
                int my_tot = 0;
#pragma unroll
                for (int k = 0; k < PI_QPW; ++k)
                    if (k == qd) my_tot = tot[k];
                if (my_tot > PI_COMPACT_AT) {
                    uint32_t T = warp_bound(sm.cs[qq], my_tot, TOPK, PI_COMPACT_AT - 2 * PI_TILE, hist);
                    int kept = warp_compact(sm.cs[qq], sm.cp[qq], my_tot, T, INT32_MAX);
                    if (kept > PI_COMPACT_AT) {                  // ties at the bound: exact select
                        int need_eq;
                        warp_kth(sm.cs[qq], kept, TOPK, hist, 4, T, need_eq);
                        kept = warp_compact(sm.cs[qq], sm.cp[qq], kept, T, need_eq);
                    }
                    if (lane == 0) {
                        sm.cnt[qq] = kept;
                        sm.thr[qq] = key_score(T);
                    }
                }
                named_barrier(bar_id, 128);                          // C: compactions done
#pragma unroll
                for (int k = 0; k < PI_QPW; ++k) thr[k] = sm.thr[PI_QPW * hq + k];
            }
#pragma unroll
            for (int k = 0; k < PI_QPW; ++k)
                if (qd == 0 && lane == k && tot[k] <= PI_COMPACT_AT) sm.cnt[PI_QPW * hq + k] = tot[k];
            // (the counts are read again only after the next tile's barrier A; a compacted
            // query's count was written before barrier C)
        }
        named_barrier(bar_id, 128);
        // ---- each query's exact Top-512, ascending (buffer order), -1 padded
        {
            const int qq = PI_QPW * hq + qd;
            if (q0 + qq < p.q_per_seq) {
                const int n = sm.cnt[qq];
                int kept = n;
                if (n > TOPK && !sm.fail) {
                    uint32_t T;
                    int need_eq;
                    warp_kth(sm.cs[qq], n, TOPK, hist, 4, T, need_eq);
                    kept = warp_compact(sm.cs[qq], sm.cp[qq], n, T, need_eq);
                }
                int32_t* dst = topk_out + (static_cast<int64_t>(b) * p.q_per_seq + q0 + qq) * TOPK;
                for (int i = lane; i < TOPK; i += 32) dst[i] = (i < kept && !sm.fail) ? sm.cp[qq][i] : -1;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, PI_TMEM_COLS);
    }
}

}  // namespace

csa2_status launch_prefill_index(const IndexParams& p, const CUtensorMap& tmap, int32_t* topk_out, unsigned* err,
                                 cudaStream_t stream) {
    const int smem = static_cast<int>(sizeof(PiShared)) + 1024;
    if (!opt_in_smem(reinterpret_cast<const void*>(prefill_index_kernel), smem))
        return check_launch("prefill_index_kernel smem attribute");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ceil_div(p.q_per_seq, PI_QB)), static_cast<unsigned>(p.batch));
    cfg.blockDim = dim3(PI_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, prefill_index_kernel, tmap, p, topk_out, err);
    return check_launch("prefill_index_kernel");
}

}  // namespace csa2
