// Decode attention (one query per sequence, every position and SWA row visible).
//
// CSA2 section of the thecryptopost.io DeepSeek-V4.1-Flash article: every layer keeps its
// own main Q and SWA KV and attends over its Top-512 selection of the shared FP4 main KV;
// the Causal Encoder-Decoder section fixes the 128-token window; tldrocket.com: one
// 512-dim latent serves as both key and value.  Per head h:
//     out_h = softmax_j(sm_scale * q_h . row_j) . rows,  rows = selected FP4 rows
//                                                        (dequantised) ++ SWA rows.
//
// Work split: a sequence's keys form a list of tiles of 64 keys: 8 main tiles (the
// Top-512 slots; those past the valid selections are absent) followed by
// ceil(swa_rows / 64) SWA tiles.  CTA (row, sp) takes tiles [sp * tiles_per_cta, ...)
// of that list, main and SWA alike; the row's CTAs form one thread-block cluster.  One
// CTA per SM, the grid sized to one wave where possible.
//
// The rows are never expanded in shared memory: they stay in their storage format there
// (E2M1 codes + E4M3 group scales, bf16 SWA rows, or E4M3 SWA rows) and every consumer
// lane converts exactly the elements of its own MMA fragments in registers (hardware
// e2m1 / e4m3 -> f16 conversion; e2m1 x e4m3 scale is exact in f16).  Shared-memory
// traffic per 64-key FP4 tile is then about 100 KB instead of the ~290 KB of an f16 tile
// written once and read by both products.
//  - Tile i lives in stage i % 3 (3 stages of 64 KB), loaded by cp.async gathers of the
//    FP4 rows (codes + scales, 16-byte chunks XOR-swizzled) or of the E4M3 SWA rows
//    completing on an mbarrier (cp.async.mbarrier.arrive.noinc), or by TMA for bf16 SWA
//    rows.  The 8 warps issue tile i + 2 once every warp is past tile i - 1 (the first
//    barrier of tile i), so two tiles are in flight while one is computed.
//  - 8 warps, mma.sync m16n8k16 with fp32 accumulation:
//      S = Q K^T: warp (kq, dq) takes keys 32kq .. 32kq+31 and dims 128dq .. 128dq+127; the
//        query's A fragments for those dims live in registers for the whole CTA; the
//        k-slots of an MMA are a fixed permutation of 16 dims chosen so that lane t reads
//        one 16-byte chunk per key row for 8 k-steps; the four dim quarters are summed in
//        shared memory.
//      softmax per head over the tile's keys, two heads per warp; a head's reference max
//        only moves when a score exceeds it by more than RESCALE_GAP (then O is rescaled).
//      O = P V: warp w owns output dims 64w .. 64w+63 for all 16 heads; column c of n-tile
//        n is dim 64w + 8c + n, so lane g converts 8 contiguous dims of 4 keys per k-step
//        and pairs keys with byte permutes into the B fragments.
//    FP4 and FP8 tiles run in f16 (query converted to f16: exact in the normal range);
//    bf16 SWA tiles run in bf16 with P split into bf16 hi + lo pieces; FP8 SWA row scales
//    are applied to the logits and to P.
//    With only 16 heads, warp MMAs keep the tensor pipe busier than tcgen05 MMAs with
//    N = 16 would (measured on B200: about 2 cycles per m16n8k16 per SM against about 71
//    cycles per 128x16x16 tcgen05.mma).
//  - Merge: each CTA keeps an unnormalised partial (reference max m, sum l, O); at the end
//    every consumer warp pushes its 64-dim block of O, and m and l, into the shared memory
//    of the cluster CTA that owns that block; after a cluster barrier each CTA merges its
//    blocks: out = sum_s e^(m_s - M) O_s / sum_s e^(m_s - M) l_s.
// Every mbarrier wait is bounded (ERR_TIMEOUT set, the CTA stops computing, no hang).
#include <algorithm>
#include <cstddef>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace csa2 {

namespace {

constexpr int DT_THREADS = 256;                           // 8 warps
constexpr int DT_STAGES = 3;
constexpr int DT_KEYS = 64;                               // keys per tile
constexpr int DT_STAGE_BYTES = DT_KEYS * D * 2;           // 64 KB: one bf16 SWA tile
constexpr int DT_Q_BYTES = HEADS * D * 2;                 // 16 KB
constexpr int DT_P_BYTES = HEADS * DT_KEYS * 2;           // 2 KB
constexpr int DT_MAX_CLUSTER = 8;                         // portable cluster size
constexpr int DT_OBLOCK_FLOATS = HEADS * 64;              // one 64-dim block of O
constexpr int DT_MAIN_TILES = TOPK / DT_KEYS;             // 8
constexpr int DT_SMS = 148;                               // one CTA per SM
constexpr float RESCALE_GAP = 8.0f;                       // lazy O rescale threshold (nats)
// stage layouts
constexpr int ST_SCALE_OFF = DT_KEYS * ROW_CODES;         // FP4: codes [64][256], scales [64][48]
constexpr int ST_SCALE_LD = 48;                           //   (row pitch: conflict-free reads)
constexpr int ST8_SCALE_OFF = DT_KEYS * D;                // FP8 SWA: codes [64][512], f32 scales [64]
constexpr int SP_LD = 72;                                 // score partials: [4][16 heads][72]

enum TileKind { TK_FP4 = 0, TK_SWA16 = 1, TK_SWA8 = 2 };

struct alignas(1024) DecodeSmem {
    uint8_t stage[DT_STAGES][DT_STAGE_BYTES];   // at the end, stage[0] receives the pushes
    union {
        uint8_t q[DT_Q_BYTES];                  // bf16 query (TMA, SW128 [8][16][128 B]),
                                                // read once into registers
        struct {
            float s[4][HEADS][SP_LD];           // S partials of the four dim quarters
            uint8_t p[2][DT_P_BYTES];           // P (f16) or P hi / lo (bf16): SW128 [16][64]
        } w;
    } u;
    int32_t main_pos[TOPK];
    float m[HEADS], l[HEADS], alpha[HEADS];
    int32_t warp_cnt[DT_THREADS / 32];
    uint64_t bar_q, full[DT_STAGES];
    int fail;
};

// After the tiles, stage[0] receives the cluster's pushes: the 64-dim O blocks this CTA
// owns (slot (w / n_split) * n_split + sender; at most 14 slots for n_split <= 8) and
// every sender's m and l.
constexpr int DT_PUSH_SLOTS = 14;
constexpr int DT_PM_OFFSET = DT_PUSH_SLOTS * DT_OBLOCK_FLOATS * 4;
constexpr int DT_PL_OFFSET = DT_PM_OFFSET + DT_MAX_CLUSTER * HEADS * 4;
static_assert(DT_PL_OFFSET + DT_MAX_CLUSTER * HEADS * 4 <= DT_STAGE_BYTES, "pushes fit in a stage");
static_assert(ST_SCALE_OFF + DT_KEYS * ST_SCALE_LD <= DT_STAGE_BYTES, "FP4 tile fits a stage");
static_assert(ST8_SCALE_OFF + DT_KEYS * 4 <= DT_STAGE_BYTES, "FP8 SWA tile fits a stage");
static_assert(sizeof(DecodeSmem) + 1024 <= 227 * 1024, "one CTA per SM");

// Position of 16-byte chunk c (0..15) of FP4 code row `row` in the stage: the XOR keeps
// both products' reads conflict-free (S: rows r, r+1 x 4 chunks; PV: 4 rows x one chunk).
__device__ __forceinline__ uint32_t fp4_chunk(uint32_t row, uint32_t c) {
    return c ^ (((row & 1u) << 2) ^ (((row >> 1) & 3u) << 1));
}

// Byte offset of 8-element chunk `chunk` (0..63) of row `row` in a SW128 tile of `rows` rows.
__device__ __forceinline__ uint32_t sw_chunk(uint32_t rows, uint32_t row, uint32_t chunk) {
    return (chunk >> 3) * rows * 128u + row * 128u + (((chunk & 7u) ^ (row & 7u)) << 4);
}

// Four E2M1 pairs (the bytes of w, low byte first) -> four f16x2 (low nibble in the low half).
__device__ __forceinline__ void e2m1x8_to_f16(uint32_t w, uint32_t (&h)[4]) {
    asm("{ .reg .b8 b0, b1, b2, b3;\n"
        "  mov.b32 {b0, b1, b2, b3}, %4;\n"
        "  cvt.rn.f16x2.e2m1x2 %0, b0;\n"
        "  cvt.rn.f16x2.e2m1x2 %1, b1;\n"
        "  cvt.rn.f16x2.e2m1x2 %2, b2;\n"
        "  cvt.rn.f16x2.e2m1x2 %3, b3; }"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(w));
}

// Two E4M3 pairs (the 16-bit halves of w) -> two f16x2 (exact).
__device__ __forceinline__ void e4m3x4_to_f16(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{ .reg .b16 s0, s1;\n"
        "  mov.b32 {s0, s1}, %2;\n"
        "  cvt.rn.f16x2.e4m3x2 %0, s0;\n"
        "  cvt.rn.f16x2.e4m3x2 %1, s1; }"
        : "=r"(lo), "=r"(hi) : "r"(w));
}

// An E4M3 scale byte -> f16x2 (s, s), exact.
__device__ __forceinline__ uint32_t e4m3_scale_f16x2(uint32_t byte) {
    uint32_t r;
    const uint16_t two = static_cast<uint16_t>(byte | (byte << 8));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(two));
    return r;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

template <bool BF16>
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (BF16) mma_16816_bf16(c, a, b0, b1);
    else mma_16816(c, a, b0, b1);
}

// ---- S = Q K^T for this warp's 32 keys (4 n-tiles) over its 128 dims (8 k-steps).
//      k-step ks, lane t: k-slots 2t, 2t+1, 2t+8, 2t+9 <-> dims d0 .. d0+3,
//      d0 = 128 dq + 32 t + 4 ks.
__device__ __forceinline__ void s_fp4(const uint8_t* sb, const uint32_t (&qf)[8][4], int kq, int dq, int g, int t,
                                      float (&acc)[4][4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t row = 32 * kq + 8 * j + g;
        const uint4 cw = *reinterpret_cast<const uint4*>(sb + row * ROW_CODES + (fp4_chunk(row, 4 * dq + t) << 4));
        const uint32_t sc = *reinterpret_cast<const uint16_t*>(sb + ST_SCALE_OFF + row * ST_SCALE_LD + 8 * dq + 2 * t);
        const uint32_t sa = e4m3_scale_f16x2(sc & 0xFFu), sbb = e4m3_scale_f16x2(sc >> 8);
        const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {                  // word wi: k-steps 2wi, 2wi+1
            uint32_t h[4];
            e2m1x8_to_f16(words[wi], h);
            const uint32_t s = wi < 2 ? sa : sbb;         // group 8dq + 2t (+1 from k-step 4)
            mma16816<false>(acc[j], qf[2 * wi], hmul2_u32(h[0], s), hmul2_u32(h[1], s));
            mma16816<false>(acc[j], qf[2 * wi + 1], hmul2_u32(h[2], s), hmul2_u32(h[3], s));
        }
    }
}

__device__ __forceinline__ void s_swa16(const uint8_t* sb, const uint32_t (&qf)[8][4], int kq, int dq, int g, int t,
                                        float (&acc)[4][4]) {
    const uint32_t cb = 2 * dq + (t >> 1);                // 64-dim block of dims 128dq + 32t ..
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t row = 32 * kq + 8 * j + g;
#pragma unroll
        for (int c = 0; c < 4; ++c) {                     // chunk: dims 128dq + 32t + 8c ..
            const uint4 v = *reinterpret_cast<const uint4*>(sb + sw_chunk(DT_KEYS, row, 8 * cb + 4 * (t & 1) + c));
            mma16816<true>(acc[j], qf[2 * c], v.x, v.y);
            mma16816<true>(acc[j], qf[2 * c + 1], v.z, v.w);
        }
    }
}

__device__ __forceinline__ void s_swa8(const uint8_t* sb, const uint32_t (&qf)[8][4], int kq, int dq, int g, int t,
                                       float (&acc)[4][4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t row = 32 * kq + 8 * j + g;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {                  // chunk: dims 128dq + 32t + 16cc ..
            const uint32_t chunk = (8 * dq + 2 * t + cc) ^ (row & 7u);
            const uint4 v = *reinterpret_cast<const uint4*>(sb + row * D + (chunk << 4));
            const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {              // word wi: k-step 4cc + wi
                uint32_t lo, hi;
                e4m3x4_to_f16(words[wi], lo, hi);
                mma16816<false>(acc[j], qf[4 * cc + wi], lo, hi);
            }
        }
    }
}

// ---- O += P V for this warp's 64 dims: k-step ks covers keys 16ks .. 16ks+15, lane (g, t)
//      converts keys 16ks + 8kp + 2t, +1 (kp = 0, 1) at dims 64w + 8g .. 64w + 8g + 7.
__device__ __forceinline__ void pv_fp4(const uint8_t* sb, const DecodeSmem& sm, int warp, int lane, float (&o)[8][4]) {
    const int g = lane >> 2, t = lane & 3, mi = lane >> 3, mj = lane & 7;
    const uint32_t p0 = smem_u32(sm.u.w.p[0]);
    const int prow = ((mi & 1) << 3) + mj;
#pragma unroll
    for (int ks = 0; ks < DT_KEYS / 16; ++ks) {
        uint32_t a[4];
        ldmatrix_x4(a, p0 + sw_chunk(HEADS, prow, 2 * ks + (mi >> 1)));
        uint32_t bf[2][8];
#pragma unroll
        for (int kp = 0; kp < 2; ++kp) {
            uint32_t x[2][4];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const uint32_t key = 16 * ks + 8 * kp + 2 * t + e;
                const uint32_t cw = *reinterpret_cast<const uint32_t*>(
                    sb + key * ROW_CODES + (fp4_chunk(key, 2 * warp + (g >> 2)) << 4) + 4 * (g & 3));
                const uint32_t s = e4m3_scale_f16x2(sb[ST_SCALE_OFF + key * ST_SCALE_LD + 4 * warp + (g >> 1)]);
                uint32_t h[4];
                e2m1x8_to_f16(cw, h);
#pragma unroll
                for (int q = 0; q < 4; ++q) x[e][q] = hmul2_u32(h[q], s);
            }
#pragma unroll
            for (int n = 0; n < 8; ++n) bf[kp][n] = prmt(x[0][n >> 1], x[1][n >> 1], (n & 1) ? 0x7632u : 0x5410u);
        }
#pragma unroll
        for (int n = 0; n < 8; ++n) mma16816<false>(o[n], a, bf[0][n], bf[1][n]);
    }
}

__device__ __forceinline__ void pv_swa16(const uint8_t* sb, const DecodeSmem& sm, int warp, int lane,
                                         float (&o)[8][4]) {
    const int g = lane >> 2, t = lane & 3, mi = lane >> 3, mj = lane & 7;
    const uint32_t p0 = smem_u32(sm.u.w.p[0]), p1 = smem_u32(sm.u.w.p[1]);
    const int prow = ((mi & 1) << 3) + mj;
#pragma unroll
    for (int ks = 0; ks < DT_KEYS / 16; ++ks) {
        uint32_t a[4], alo[4];
        ldmatrix_x4(a, p0 + sw_chunk(HEADS, prow, 2 * ks + (mi >> 1)));
        ldmatrix_x4(alo, p1 + sw_chunk(HEADS, prow, 2 * ks + (mi >> 1)));
        uint32_t bf[2][8];
#pragma unroll
        for (int kp = 0; kp < 2; ++kp) {
            const uint32_t key = 16 * ks + 8 * kp + 2 * t;
            const uint4 v0 = *reinterpret_cast<const uint4*>(sb + sw_chunk(DT_KEYS, key, 8 * warp + g));
            const uint4 v1 = *reinterpret_cast<const uint4*>(sb + sw_chunk(DT_KEYS, key + 1, 8 * warp + g));
            const uint32_t x0[4] = {v0.x, v0.y, v0.z, v0.w}, x1[4] = {v1.x, v1.y, v1.z, v1.w};
#pragma unroll
            for (int n = 0; n < 8; ++n) bf[kp][n] = prmt(x0[n >> 1], x1[n >> 1], (n & 1) ? 0x7632u : 0x5410u);
        }
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            mma16816<true>(o[n], a, bf[0][n], bf[1][n]);
            mma16816<true>(o[n], alo, bf[0][n], bf[1][n]);
        }
    }
}

__device__ __forceinline__ void pv_swa8(const uint8_t* sb, const DecodeSmem& sm, int warp, int lane,
                                        float (&o)[8][4]) {
    const int g = lane >> 2, t = lane & 3, mi = lane >> 3, mj = lane & 7;
    const uint32_t p0 = smem_u32(sm.u.w.p[0]);
    const int prow = ((mi & 1) << 3) + mj;
#pragma unroll
    for (int ks = 0; ks < DT_KEYS / 16; ++ks) {
        uint32_t a[4];
        ldmatrix_x4(a, p0 + sw_chunk(HEADS, prow, 2 * ks + (mi >> 1)));
        uint32_t bf[2][8];
#pragma unroll
        for (int kp = 0; kp < 2; ++kp) {
            uint32_t x[2][4];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const uint32_t key = 16 * ks + 8 * kp + 2 * t + e;
                const uint32_t chunk = (4 * warp + (g >> 1)) ^ (key & 7u);
                const uint2 v = *reinterpret_cast<const uint2*>(sb + key * D + (chunk << 4) + 8 * (g & 1));
                e4m3x4_to_f16(v.x, x[e][0], x[e][1]);
                e4m3x4_to_f16(v.y, x[e][2], x[e][3]);
            }
#pragma unroll
            for (int n = 0; n < 8; ++n) bf[kp][n] = prmt(x[0][n >> 1], x[1][n >> 1], (n & 1) ? 0x7632u : 0x5410u);
        }
#pragma unroll
        for (int n = 0; n < 8; ++n) mma16816<false>(o[n], a, bf[0][n], bf[1][n]);
    }
}

__global__ void __launch_bounds__(DT_THREADS, 1)
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
    const int64_t seq_off = p.kv_offsets[r];
    const int64_t n_b = p.kv_offsets[r + 1] - seq_off;
    const int swa_tiles = static_cast<int>((p.swa_rows + DT_KEYS - 1) / DT_KEYS);
    const int t_first = sp * p.tiles_per_cta;
    const int t_last = min(DT_MAIN_TILES + swa_tiles, t_first + p.tiles_per_cta);
    const bool has_main = t_first < DT_MAIN_TILES && t_first < t_last;

    if (tid == 0) {
        mbar_init(&sm.bar_q, 1);
        for (int s = 0; s < DT_STAGES; ++s) mbar_init(&sm.full[s], DT_THREADS);
        mbar_fence_init();
        sm.fail = 0;
        mbar_arrive_expect_tx(&sm.bar_q, DT_Q_BYTES);
        for (int cb = 0; cb < D / 64; ++cb)
            tma_load_2d(sm.u.q + cb * HEADS * 128, &tmap_q, 64 * cb, static_cast<int>(r * HEADS), &sm.bar_q);
    }
    if (tid < HEADS) {
        sm.m[tid] = -INFINITY;
        sm.l[tid] = 0.0f;
    }

    // ---- valid main positions, compacted in order (2 per thread of the first 256)
    int n_main = 0;
    if (has_main) {
        int cnt = 0;
        bool ok0 = false, ok1 = false;
        int32_t v0 = 0, v1 = 0;
        if (tid < TOPK / 2) {
            const int32_t* idx = p.topk_idx + r * TOPK;
            v0 = idx[2 * tid];
            v1 = idx[2 * tid + 1];
            const bool bad0 = v0 >= n_b, bad1 = v1 >= n_b;
            if ((bad0 || bad1) && sp == 0 && p.err) atomicOr(p.err, ERR_DEVICE);
            ok0 = v0 >= 0 && !bad0;
            ok1 = v1 >= 0 && !bad1;
            cnt = static_cast<int>(ok0) + static_cast<int>(ok1);
        }
        int incl = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off) incl += y;
        }
        if (lane == 31) sm.warp_cnt[warp] = incl;
        __syncthreads();
        int before = incl - cnt;
        for (int w = 0; w < DT_THREADS / 32; ++w) {
            const int c = sm.warp_cnt[w];
            if (w < warp) before += c;
            n_main += c;
        }
        if (ok0) sm.main_pos[before++] = v0;
        if (ok1) sm.main_pos[before] = v1;
    }
    __syncthreads();

    // the CTA's tiles: main tile t exists while it holds valid selections
    const int main_tiles = (n_main + DT_KEYS - 1) / DT_KEYS;
    const auto exists = [&](int t) { return t < DT_MAIN_TILES ? t < main_tiles : true; };
    const auto kind_of = [&](int t) {
        if (t < DT_MAIN_TILES) return TK_FP4;
        return p.swa_fp8 ? TK_SWA8 : TK_SWA16;
    };
    const auto keys_of = [&](int t) {
        return t < DT_MAIN_TILES ? min(DT_KEYS, n_main - t * DT_KEYS)
                                 : static_cast<int>(min(static_cast<int64_t>(DT_KEYS),
                                                        p.swa_rows - static_cast<int64_t>(t - DT_MAIN_TILES) * DT_KEYS));
    };
    const auto next_tile = [&](int t) {
        for (int u = t + 1; u < t_last; ++u)
            if (exists(u)) return u;
        return -1;
    };
    const int t0 = (t_first < t_last && exists(t_first)) ? t_first : next_tile(t_first);
    int n_tiles = 0;
    for (int t = t0; t >= 0; t = next_tile(t)) ++n_tiles;

    // ---- tile loads: every thread issues its share and arrives on full[st] when its own
    //      copies land (bf16 SWA: thread 0 arms the TMA bytes, the others arrive at once)
    const auto issue = [&](int t, int st) {
        uint8_t* sb = sm.stage[st];
        const TileKind kind = kind_of(t);
        const int tile_keys = keys_of(t);
        if (kind == TK_FP4) {                            // codes + scales of 64 rows, absent rows zero
            // thread -> code chunk c = tid % 16 of rows tid / 16 + 16k, and (first 128 threads)
            // scale half tid % 2 of row tid / 2; the row indices are read before any copy is
            // issued, so the copies do not wait on them one by one
            constexpr int CPT = DT_KEYS * (ROW_CODES / 16) / DT_THREADS;   // 4
            static_assert(DT_KEYS * (ROW_SCALES / 16) <= DT_THREADS, "one scale chunk per thread");
            const int key0 = t * DT_KEYS;
            const int c = tid & 15, kk0 = tid >> 4;
            int64_t row[CPT];
#pragma unroll
            for (int k = 0; k < CPT; ++k) {
                const int kk = kk0 + 16 * k;
                row[k] = kk < tile_keys ? seq_off + sm.main_pos[key0 + kk] : -1;
            }
            const int skk = tid >> 1, sc = tid & 1;
            const int64_t srow = (tid < 2 * DT_KEYS && skk < tile_keys) ? seq_off + sm.main_pos[key0 + skk] : -1;
#pragma unroll
            for (int k = 0; k < CPT; ++k) {
                const int kk = kk0 + 16 * k;
                cp_async_16(smem_u32(sb + kk * ROW_CODES + (fp4_chunk(kk, c) << 4)),
                            p.codes + (row[k] >= 0 ? row[k] * ROW_CODES + 16 * c : 0), row[k] >= 0 ? 16 : 0);
            }
            if (tid < 2 * DT_KEYS)
                cp_async_16(smem_u32(sb + ST_SCALE_OFF + skk * ST_SCALE_LD + 16 * sc),
                            p.scales + (srow >= 0 ? srow * ROW_SCALES + 16 * sc : 0), srow >= 0 ? 16 : 0);
            cp_async_mbar_arrive_noinc(&sm.full[st]);
        } else if (kind == TK_SWA8) {                    // E4M3 rows + f32 row scales
            const int64_t row0 = r * p.swa_rows + static_cast<int64_t>(t - DT_MAIN_TILES) * DT_KEYS;
            for (int id = tid; id < DT_KEYS * (D / 16); id += DT_THREADS) {
                const int kk = id >> 5, c = id & 31;
                const bool in = kk < tile_keys;
                const uint8_t* src = p.swa_kv8 + (in ? (row0 + kk) * D + 16 * c : 0);
                cp_async_16(smem_u32(sb + kk * D + ((c ^ (kk & 7)) << 4)), src, in ? 16 : 0);
            }
            if (tid < DT_KEYS) {
                const bool in = tid < tile_keys;
                cp_async_4(smem_u32(sb + ST8_SCALE_OFF + 4 * tid), p.swa_kscale + (in ? row0 + tid : 0), in ? 4 : 0);
            }
            cp_async_mbar_arrive_noinc(&sm.full[st]);
        } else if (tid == 0) {                           // bf16 rows by TMA
            fence_proxy_async_smem();                    // after earlier generic reads of the stage
            mbar_arrive_expect_tx(&sm.full[st], DT_STAGE_BYTES);
            const int key0 = (t - DT_MAIN_TILES) * DT_KEYS;
            for (int cb = 0; cb < D / 64; ++cb)
                tma_load_3d(sb + cb * DT_KEYS * 128, &tmap_swa, 64 * cb, key0, static_cast<int>(r), &sm.full[st]);
        } else {
            mbar_arrive(&sm.full[st]);
        }
    };
    int armed[DT_STAGES] = {};                           // full phases armed per stage
    int t_ahead = t0;                                    // next tile to issue
    for (int k = 0; k < DT_STAGES && t_ahead >= 0; ++k, t_ahead = next_tile(t_ahead)) {
        issue(t_ahead, k);
        ++armed[k];
    }

    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    const int t4 = lane & 3;
    const int kq = warp & 1, dq = warp >> 1;
    // the query's A fragments for this warp's dims, f16 and bf16 (rows g, g + 8)
    uint32_t qh[8][4], qb[8][4];
    if (!mbar_wait(&sm.bar_q, 0, p.err)) sm.fail = 1;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        const uint32_t d0 = 128 * dq + 32 * t4 + 4 * ks;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t h = g + 8 * hh;
            const uint2 v = *reinterpret_cast<const uint2*>(
                sm.u.q + (d0 >> 6) * HEADS * 128 + h * 128 + ((((d0 & 63) >> 3) ^ (h & 7)) << 4) + (d0 & 7) * 2);
            qb[ks][hh] = v.x;
            qb[ks][2 + hh] = v.y;
            qh[ks][hh] = bf16x2_to_f16x2(v.x);
            qh[ks][2 + hh] = bf16x2_to_f16x2(v.y);
        }
    }
    __syncthreads();                                     // the query's space now holds S and P
    float m_ref[2] = {-INFINITY, -INFINITY};             // heads 2w, 2w+1 (warp-uniform)
    float l_lane[2] = {0.0f, 0.0f};                      // this lane's share of their sums
    // stage 0 receives the cluster's pushes at the end: this CTA arrives on the cluster
    // barrier right after its last tile in stage 0 (once, at a CTA-uniform point), so a
    // partner that finishes first can push while this CTA computes its last tiles
    const int last_in_stage0 = n_tiles > 0 ? ((n_tiles - 1) / DT_STAGES) * DT_STAGES : -1;
    bool arrived = false;
    if (last_in_stage0 < 0) {
        cluster_arrive();
        arrived = true;
    }
    int i = 0;
    // sm.fail is read only right after a barrier (every write precedes it)
    for (int t = t0; t >= 0; t = next_tile(t), ++i) {
        const int st = i % DT_STAGES;
        const TileKind kind = kind_of(t);
        const int tile_keys = keys_of(t);
        const uint8_t* sb = sm.stage[st];
        // ---- 1. tile i is in stage st
        if (!mbar_wait(&sm.full[st], (i / DT_STAGES) & 1, p.err)) sm.fail = 1;

        // ---- 2. S partial of this warp's keys and dim quarter -> shared
        {
            float acc[4][4] = {};
            if (kind == TK_FP4) s_fp4(sb, qh, kq, dq, g, t4, acc);
            else if (kind == TK_SWA16) s_swa16(sb, qb, kq, dq, g, t4, acc);
            else s_swa8(sb, qh, kq, dq, g, t4, acc);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int key = 32 * kq + 8 * j + 2 * t4;
                *reinterpret_cast<float2*>(&sm.u.w.s[dq][g][key]) = make_float2(acc[j][0], acc[j][1]);
                *reinterpret_cast<float2*>(&sm.u.w.s[dq][g + 8][key]) = make_float2(acc[j][2], acc[j][3]);
            }
        }
        __syncthreads();
        if (sm.fail) break;
        // every warp is past tile i - 1: its stage takes tile i + 2
        if (i >= 1 && t_ahead >= 0) {
            const int sn = (i + 2) % DT_STAGES;
            issue(t_ahead, sn);
            ++armed[sn];
            t_ahead = next_tile(t_ahead);
        }

        // ---- 3. softmax: warp w owns heads 2w, 2w+1; lane owns keys lane, lane+32.  The
        //      reference max m_ref (uniform in the warp) only moves when a score exceeds
        //      it by more than RESCALE_GAP (P <= e^RESCALE_GAP is still exact-width in
        //      f16 / bf16), found with one vote; row sums stay per lane until the end.
        const bool swa8 = kind == TK_SWA8;
        const float* rs = reinterpret_cast<const float*>(sb + ST8_SCALE_OFF);
        float smax = 1.0f;
        if (swa8) {                                      // the tile's largest row scale
            smax = fmaxf(rs[lane], rs[lane + 32]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) smax = fmaxf(smax, __shfl_xor_sync(0xFFFFFFFFu, smax, off));
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int h = 2 * warp + hh;
            float sv[2];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int key = lane + 32 * jj;
                const float sum = ((sm.u.w.s[0][h][key] + sm.u.w.s[1][h][key]) + sm.u.w.s[2][h][key]) +
                                  sm.u.w.s[3][h][key];
                sv[jj] = key < tile_keys ? sum * p.sm_scale : -INFINITY;
                if (swa8 && key < tile_keys) sv[jj] *= rs[key];
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
                const float pvv = (sv[jj] == -INFINITY) ? 0.0f : __expf(sv[jj] - m_ref[hh]);
                l_lane[hh] += pvv;
                const uint32_t off = sw_chunk(HEADS, h, key >> 3) + (key & 7) * 2;
                if (swa8) {                              // P * s_key / max s: <= P, in f16
                    const float pw = smax > 0.0f ? pvv * (rs[key] / smax) : 0.0f;
                    *reinterpret_cast<__half*>(sm.u.w.p[0] + off) = __float2half_rn(pw);
                } else if (kind == TK_FP4) {
                    *reinterpret_cast<__half*>(sm.u.w.p[0] + off) = __float2half_rn(pvv);
                } else {
                    const __nv_bfloat16 hi = __float2bfloat16_rn(pvv);
                    *reinterpret_cast<__nv_bfloat16*>(sm.u.w.p[0] + off) = hi;
                    *reinterpret_cast<__nv_bfloat16*>(sm.u.w.p[1] + off) =
                        __float2bfloat16_rn(pvv - __bfloat162float(hi));
                }
            }
            if (lane == 0) sm.alpha[h] = alpha;
        }
        __syncthreads();

        // ---- 4. O = alpha * O + P V (alpha is 1 unless a reference max moved); FP8 SWA:
        //      O + smax * (P' V') is done as (O / smax + P' V') * smax
        {
            const float inv = swa8 && smax > 0.0f ? 1.0f / smax : 1.0f;
            const float al = sm.alpha[g] * inv, ah = sm.alpha[g + 8] * inv;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                o[nt][0] *= al;
                o[nt][1] *= al;
                o[nt][2] *= ah;
                o[nt][3] *= ah;
            }
        }
        if (kind == TK_FP4) pv_fp4(sb, sm, warp, lane, o);
        else if (kind == TK_SWA16) pv_swa16(sb, sm, warp, lane, o);
        else pv_swa8(sb, sm, warp, lane, o);
        if (swa8 && smax > 0.0f) {
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                o[nt][0] *= smax;
                o[nt][1] *= smax;
                o[nt][2] *= smax;
                o[nt][3] *= smax;
            }
        }
        if (i == last_in_stage0) {                       // this thread's reads of stage 0 are done
            cluster_arrive();                            // (release: they precede the partner's pushes)
            arrived = true;
        }
    }
    if (!arrived) cluster_arrive();                      // a failed wait ended the loop early
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
    // ---- drain: every armed tile load has landed (all were consumed unless a wait failed)
    cp_async_wait<0>();
    if (tid == 0) {
        for (int s2i = 0; s2i < DT_STAGES; ++s2i)
            if (armed[s2i] > 0) mbar_wait(&sm.full[s2i], (armed[s2i] - 1) & 1, p.err);
    }
    __syncthreads();
    const bool have = n_tiles > 0 && !sm.fail;

    // ---- push this CTA's partial into the cluster: consumer warp w's O fragment (64-dim
    //      block w) goes to CTA w % n_split, slot (w / n_split) * n_split + rank, lane-major
    //      (lane * 32 + 4 nt + c holds o[nt][c]); m and l go to every CTA
    const uint32_t rank = cluster_ctarank();
    const int ns = p.n_split;
    cluster_wait();                                   // every CTA is done with its stage 0
    {
        const uint32_t owner = static_cast<uint32_t>(warp % ns);
        const int slot = (warp / ns) * ns + static_cast<int>(rank);
        const uint32_t base = dsmem_addr(smem_u32(sm.stage[0]), owner) + (slot * DT_OBLOCK_FLOATS + lane * 32) * 4;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            if (have) dsmem_st_f32x4(base + 16 * nt, o[nt][0], o[nt][1], o[nt][2], o[nt][3]);
            else dsmem_st_f32x4(base + 16 * nt, 0.0f, 0.0f, 0.0f, 0.0f);
        }
        if (tid < HEADS * ns) {
            const int h = tid & 15, dst = tid >> 4;
            const uint32_t mine = smem_u32(sm.stage[0]) + (rank * HEADS + h) * 4;
            dsmem_st_f32(dsmem_addr(mine + DT_PM_OFFSET, static_cast<uint32_t>(dst)), have ? sm.m[h] : -INFINITY);
            dsmem_st_f32(dsmem_addr(mine + DT_PL_OFFSET, static_cast<uint32_t>(dst)), have ? sm.l[h] : 0.0f);
        }
    }
    cluster_sync();

    // ---- merge the blocks this CTA owns (w = rank + k * n_split): thread tid takes
    //      fragment float4 (lane tid / 8, nt = tid % 8) of every sender's slot; its
    //      values are heads hg, hg + 8 at dims 64w + 16 t' + nt and 64w + 16 t' + 8 + nt
    const float* recv = reinterpret_cast<const float*>(sm.stage[0]);
    const float (*pm)[HEADS] = reinterpret_cast<const float (*)[HEADS]>(sm.stage[0] + DT_PM_OFFSET);
    const float (*pl)[HEADS] = reinterpret_cast<const float (*)[HEADS]>(sm.stage[0] + DT_PL_OFFSET);
    const int src_lane = tid >> 3, nt = tid & 7;
    const int hg = src_lane >> 2, dd = 16 * (src_lane & 3) + nt;
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
        out_r[hg * D] = acc.x * inv_a;
        out_r[hg * D + 8] = acc.y * inv_a;
        out_r[(hg + 8) * D] = acc.z * inv_b;
        out_r[(hg + 8) * D + 8] = acc.w * inv_b;
    }
}

}  // namespace

void attend_decode_split(int64_t rows, int64_t swa_rows, int& n_split, int& tiles_per_cta) {
    const int total = DT_MAIN_TILES + static_cast<int>(ceil_div(swa_rows, DT_KEYS));
    // fewest tiles on the critical path (waves x tiles per CTA); among equals, fewer CTAs
    int64_t best_cost = INT64_MAX;
    tiles_per_cta = total;
    for (int tpc = 1; tpc <= total; ++tpc) {
        const int64_t n = ceil_div(total, tpc);
        if (n > DT_MAX_CLUSTER) continue;
        const int64_t cost = ceil_div(rows * n, DT_SMS) * tpc;
        if (cost < best_cost || (cost == best_cost && n < ceil_div(total, tiles_per_cta))) {
            best_cost = cost;
            tiles_per_cta = tpc;
        }
    }
    n_split = static_cast<int>(ceil_div(total, tiles_per_cta));
}

csa2_status launch_attend_decode(const AttnParams& p, const CUtensorMap& tmap_q, const CUtensorMap& tmap_swa,
                                 cudaStream_t stream) {
    const int64_t rows = p.batch;
    if (rows == 0) return CSA2_OK;
    if (p.n_split < 1 || p.n_split > DT_MAX_CLUSTER) return CSA2_ERR_UNSUPPORTED;
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
