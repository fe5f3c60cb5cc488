// Sparse attention of single query rows: the decode query of a sequence, or one query of
// a prefill chunk (its own causal Top-512 and its own 128-row window of the chunk's SWA
// buffer).
//
// CSA2 section of the thecryptopost.io DeepSeek-V4.1-Flash article: every layer keeps its
// own main Q and SWA KV and attends over its Top-512 selection of the shared FP4 main KV;
// the Causal Encoder-Decoder section fixes the 128-token window; tldrocket.com: one
// 512-dim latent serves as both key and value.  Per head h:
//     out_h = softmax_j(sm_scale * q_h . row_j) . rows,  rows = selected FP4 rows
//                                                        (dequantised) ++ SWA rows.
//
// Work split: a row's keys form a list of tiles: 8 main tiles of 64 keys (the Top-512
// slots; a slot holding -1 or a position past the context is masked) followed by the SWA
// tiles (32 rows of bf16, or 64 rows of E4M3; a tile outside the row's window is
// skipped).  The row's n_split CTAs form one thread-block cluster and deal the list round
// robin (CTA sp takes tiles sp, sp + n_split, ...), so every CTA gets the same mix of main
// and SWA tiles; a CTA runs its SWA tiles first (their loads need no index) and reads the
// indices of its first main tiles straight into the threads that gather those rows.  Two
// CTAs run per SM (8 warps each), so one CTA's barriers and memory waits overlap with the
// other's tensor-core work.
//
// The rows are never expanded in shared memory: they stay in their storage format there
// (E2M1 codes + E4M3 group scales, bf16 SWA rows, or E4M3 SWA rows) and every consumer
// lane converts exactly the elements of its own MMA fragments in registers (hardware
// e2m1 / e4m3 -> f16 conversion; e2m1 x e4m3 scale is exact in f16).
//  - Tile i lives in stage i % 2 (2 stages of 33 KB), loaded by cp.async gathers of the
//    FP4 rows (codes + scales, 16-byte chunks XOR-swizzled) or of the E4M3 SWA rows
//    completing on an mbarrier (cp.async.mbarrier.arrive.noinc), or by TMA for bf16 SWA
//    rows.  The 8 warps issue tile i + 1 once every warp is past tile i - 1.
//  - 8 warps, mma.sync m16n8k16 with fp32 accumulation:
//      S = Q K^T: warp (kq, dq) takes keys 32kq .. 32kq+31 (16kq .. of a 32-key tile) and
//        dims 128dq .. 128dq+127; the query's A fragments (f16, exact for bf16 queries in
//        the f16 normal range) sit in shared memory in fragment order, one 16-byte load per
//        lane and k-step; the k-slots of an MMA are a fixed permutation of 16 dims chosen
//        so that lane t reads one 16-byte chunk per key row for 8 k-steps; the four dim
//        quarters are summed in shared memory.
//      softmax per head over the tile's keys, two heads per warp; a head's reference max
//        only moves when a score exceeds it by more than RESCALE_GAP (then O is rescaled).
//      O = P V: warp w owns output dims 64w .. 64w+63 for all 16 heads; column c of n-tile
//        n is dim 64w + 8c + n, so lane g converts 8 contiguous dims of 4 keys per k-step;
//        FP4 tiles interleave two keys' codes nibble by nibble first, so that each
//        conversion yields a key-pair B fragment (bf16 / E4M3 SWA tiles pair keys with
//        byte permutes).
//    FP4 and FP8 tiles run in f16; bf16 SWA tiles run in bf16 (the f16 query fragments
//    converted back to bf16, exactly) with P split into bf16 hi + lo pieces; FP8 SWA row
//    scales are applied to the logits and to P.
//    With only 16 heads, warp MMAs keep the tensor pipe busier than tcgen05 MMAs with
//    N = 16 would (measured on B200: about 2 cycles per m16n8k16 per SM against about 71
//    cycles per dependent 128x16x16 tcgen05.mma).
//  - Merge: each CTA keeps an unnormalised partial (reference max m, sum l, O); at the end
//    every warp pushes its 64-dim block of O, and m and l, over distributed shared memory
//    into the (idle) stages of the cluster CTA that owns that block; after a cluster
//    barrier each CTA merges its blocks in sender order (bit-reproducible):
//    out = sum_s e^(m_s - M) O_s / sum_s e^(m_s - M) l_s.
//  - Block-scaled FP4 query variant (the FP4 KV section's NVFP4 format on the FP4 tensor
//    cores): with the query given as NVFP4 rows (one per head: E2M1 codes + one E4M3
//    scale per 16 dims), S of an FP4 tile is one tcgen05.mma.kind::mxf4nvf4 per 64 dims
//    (M = 128 rows of the tile, of which the first 64 are keys, N = 16 heads, K = 64),
//    reading the gathered FP4 codes straight from shared memory (128-byte swizzled K-major
//    panels) and both operands' E4M3 scales from tensor memory: scale word s of row m in
//    lane m % 32 of every lane quarter, column 4 s + m / 32 (the 16 heads' in column 4 s),
//    4-column aligned.  Once an FP4 tile has landed, warps 0-3 store its scale words
//    there (tcgen05.st), thread 0 issues its 8 MMAs, and warps 0-1 (lanes 0..63) read S^T
//    into the S buffer.  The query is quantised in the kernel from its bf16 copy in
//    shared memory.
//    The SWA tiles and P V are unchanged (exact query, f16 / bf16 MMAs).
//  - Launched as a programmatic dependent of the previous kernel on the stream: barrier
//    set-up (and the variant's tensor-memory allocation) overlaps that kernel's tail, and
//    nothing from global memory is read before griddepcontrol.wait.
// Every mbarrier wait is bounded (ERR_TIMEOUT set, the CTA stops computing, no hang).
#include <algorithm>
#include <cstddef>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace csa2 {

namespace {

constexpr int DT_THREADS = 256;                           // 8 warps
constexpr int DT_CTAS_PER_SM = 2;
constexpr int DT_STAGES = 2;
constexpr int DT_KEYS = 64;                               // keys of an FP4 / E4M3 tile
constexpr int DT_KEYS16 = 32;                             // keys of a bf16 SWA tile
constexpr int DT_STAGE_BYTES = 33 * 1024;                 // 32 KB of rows + scales
constexpr int DT_Q_BYTES = HEADS * D * 2;                 // 16 KB
constexpr int DT_P_BYTES = HEADS * DT_KEYS * 2;           // 2 KB
constexpr int DT_MAX_CLUSTER = 8;                         // portable cluster size
constexpr int DT_OBLOCK_FLOATS = HEADS * 64;              // one 64-dim block of O
constexpr int DT_MAIN_TILES = TOPK / DT_KEYS;             // 8
constexpr int DT_SMS = 148;
constexpr float RESCALE_GAP = 8.0f;                       // lazy O rescale threshold (nats)
// stage layouts
constexpr int ST_SCALE_OFF = DT_KEYS * ROW_CODES;         // FP4: codes [64][256], scales [64][48]
constexpr int ST_SCALE_LD = 48;                           //   (row pitch: conflict-free reads)
constexpr int ST8_SCALE_OFF = DT_KEYS * D;                // FP8 SWA: codes [64][512], f32 scales [64]
constexpr int SP_LD = 72;                                 // score partials: [4][16 heads][72]
// NVFP4-query variant: FP4 tile codes as two 128-byte swizzled K-major panels (bytes
// 0..127 and 128..255 of each row) 16 KB apart, so that an M = 128 MMA over the 64 keys
// reads in-stage bytes for its 64 unused rows; the scales sit in that unused span
constexpr int ST4_PANEL = 16384;
constexpr int ST4_SCALE_OFF = 8192;
constexpr uint32_t QT_COLS = 128;                         // tensor memory of the variant:
constexpr uint32_t QT_D = 0;                              //   S^T (16 columns)
constexpr uint32_t QT_SFA = 32;                           //   tile scales (32)
constexpr uint32_t QT_SFB = 64;                           //   query scales (32)

enum TileKind { TK_FP4 = 0, TK_SWA16 = 1, TK_SWA8 = 2 };

struct alignas(1024) DecodeSmem {
    uint8_t stage[DT_STAGES][DT_STAGE_BYTES];
    uint8_t qb[2][HEADS][128];                  // NVFP4 query codes: SW128 K-major panels
    uint4 qf[4][8][32];                         // query A fragments (f16): [dq][k-step][lane]
    union {
        uint8_t q[DT_Q_BYTES];                  // bf16 query (TMA, SW128 [8][16][128 B])
        float s[4][HEADS][SP_LD];               // S partials of the four dim quarters
    } u;
    uint8_t p[2][DT_P_BYTES];                   // P (f16) or P hi / lo (bf16): SW128 [16][64]
    int32_t main_pos[TOPK];                     // this CTA's main slots' cache rows (-1 = masked)
    float m[HEADS], l[HEADS], alpha[HEADS];     // m, l: the merge of a one-CTA row
    uint64_t bar_q, full[DT_STAGES], bar_mma;
    uint32_t tmem;
    int fail;
};

// After the tiles the stages receive the cluster's pushes: the O blocks this CTA merges
// (slot (w / n) * n + sender: at most 14 slots of 4 KB for n <= 8) and every sender's m
// and l.
constexpr int DT_PUSH_SLOTS = 14;
constexpr int DT_PM_OFFSET = DT_PUSH_SLOTS * DT_OBLOCK_FLOATS * 4;
constexpr int DT_PL_OFFSET = DT_PM_OFFSET + DT_MAX_CLUSTER * HEADS * 4;
static_assert(DT_PL_OFFSET + DT_MAX_CLUSTER * HEADS * 4 <= DT_STAGES * DT_STAGE_BYTES, "pushes fit the stages");
static_assert(ST_SCALE_OFF + DT_KEYS * ST_SCALE_LD <= DT_STAGE_BYTES, "FP4 tile fits a stage");
static_assert(ST8_SCALE_OFF + DT_KEYS * 4 <= DT_STAGE_BYTES, "FP8 SWA tile fits a stage");
static_assert(DT_KEYS16 * D * 2 <= DT_STAGE_BYTES, "bf16 SWA tile fits a stage");
static_assert(DT_STAGE_BYTES % 1024 == 0, "stages keep the 1 KB alignment of the swizzled TMA tiles");
static_assert(ST4_SCALE_OFF >= DT_KEYS * 128 && ST4_SCALE_OFF + DT_KEYS * ST_SCALE_LD <= ST4_PANEL,
              "variant scales in the first panel's unused rows");
static_assert(ST4_PANEL + 128 * 128 <= DT_STAGE_BYTES, "an M = 128 read of the second panel stays in the stage");
static_assert(offsetof(DecodeSmem, qb) % 1024 == 0, "query panels on a swizzle-atom boundary");
static_assert(DT_CTAS_PER_SM * (sizeof(DecodeSmem) + 1024 + 1024) <= 228 * 1024, "two CTAs per SM");

// Position of 16-byte chunk c (0..15) of FP4 code row `row` in the stage: the XOR keeps
// both products' reads conflict-free (S: rows r, r+1 x 4 chunks; PV: 4 rows x one chunk).
__device__ __forceinline__ uint32_t fp4_chunk(uint32_t row, uint32_t c) {
    return c ^ (((row & 1u) << 2) ^ (((row >> 1) & 3u) << 1));
}

// Byte offset of 16-byte chunk c (0..15) of FP4 code row `row` in a variant stage: panel
// c / 8, the 128-byte swizzle (chunk c % 8 xor row % 8) that the MMA descriptors expect.
__device__ __forceinline__ uint32_t fp4q_chunk(uint32_t row, uint32_t c) {
    return (c >> 3) * ST4_PANEL + row * 128u + (((c & 7u) ^ (row & 7u)) << 4);
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

// Two E4M3 bytes (the low 16 bits of w, low byte first) -> f16x2 (low byte in the low
// half), exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t w) {
    uint32_t r;
    const uint16_t two = static_cast<uint16_t>(w);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(two));
    return r;
}

// An E4M3 scale byte -> f16x2 (s, s), exact.
__device__ __forceinline__ uint32_t e4m3_scale_f16x2(uint32_t byte) { return e4m3x2_to_f16x2(byte | (byte << 8)); }

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// f16x2 that hold bf16 values (a bf16 query converted to f16) -> the same values as bf16x2.
__device__ __forceinline__ uint32_t f16x2_to_bf16x2(uint32_t h) {
    __half2 v = *reinterpret_cast<__half2*>(&h);
    const float2 f = __half22float2(v);
    __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<uint32_t*>(&b);
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

__device__ __forceinline__ void load_frag(const uint4* qf, int ks, int lane, uint32_t (&a)[4]) {
    const uint4 v = qf[ks * 32 + lane];
    a[0] = v.x;
    a[1] = v.y;
    a[2] = v.z;
    a[3] = v.w;
}

// ---- S = Q K^T for this warp's 32 keys (4 n-tiles) over its 128 dims (8 k-steps).
//      k-step ks, lane t: k-slots 2t, 2t+1, 2t+8, 2t+9 <-> dims d0 .. d0+3,
//      d0 = 128 dq + 32 t + 4 ks.  qf: this warp's dim quarter, [k-step][lane].
__device__ __forceinline__ void s_fp4(const uint8_t* sb, const uint4* qf, int kq, int dq, int g, int t,
                                      int lane, float (&acc)[4][4]) {
    uint4 cw[4];
    uint32_t sa[4], sbb[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t row = 32 * kq + 8 * j + g;
        cw[j] = *reinterpret_cast<const uint4*>(sb + row * ROW_CODES + (fp4_chunk(row, 4 * dq + t) << 4));
        const uint32_t sc = *reinterpret_cast<const uint16_t*>(sb + ST_SCALE_OFF + row * ST_SCALE_LD + 8 * dq + 2 * t);
        sa[j] = e4m3_scale_f16x2(sc & 0xFFu);           // group 8dq + 2t (k-steps 0..3)
        sbb[j] = e4m3_scale_f16x2(sc >> 8);             // group 8dq + 2t + 1 (k-steps 4..7)
    }
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {                      // word wi: k-steps 2wi, 2wi+1
        uint32_t a0[4], a1[4];
        load_frag(qf, 2 * wi, lane, a0);
        load_frag(qf, 2 * wi + 1, lane, a1);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t word = wi == 0 ? cw[j].x : wi == 1 ? cw[j].y : wi == 2 ? cw[j].z : cw[j].w;
            uint32_t h[4];
            e2m1x8_to_f16(word, h);
            const uint32_t s = wi < 2 ? sa[j] : sbb[j];
            mma16816<false>(acc[j], a0, hmul2_u32(h[0], s), hmul2_u32(h[1], s));
            mma16816<false>(acc[j], a1, hmul2_u32(h[2], s), hmul2_u32(h[3], s));
        }
    }
}

// bf16 SWA tile of 32 keys: warp (kq, dq) takes keys 16kq .. 16kq+15 (2 n-tiles).
__device__ __forceinline__ void s_swa16(const uint8_t* sb, const uint4* qf, int kq, int dq, int g, int t, int lane,
                                        float (&acc)[4][4]) {
    const uint32_t cb = 2 * dq + (t >> 1);                // 64-dim block of dims 128dq + 32t ..
#pragma unroll
    for (int c = 0; c < 4; ++c) {                         // chunk: dims 128dq + 32t + 8c ..
        uint32_t a0[4], a1[4];
        load_frag(qf, 2 * c, lane, a0);
        load_frag(qf, 2 * c + 1, lane, a1);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            a0[e] = f16x2_to_bf16x2(a0[e]);
            a1[e] = f16x2_to_bf16x2(a1[e]);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint32_t row = 16 * kq + 8 * j + g;
            const uint4 v = *reinterpret_cast<const uint4*>(sb + sw_chunk(DT_KEYS16, row, 8 * cb + 4 * (t & 1) + c));
            mma16816<true>(acc[j], a0, v.x, v.y);
            mma16816<true>(acc[j], a1, v.z, v.w);
        }
    }
}

__device__ __forceinline__ void s_swa8(const uint8_t* sb, const uint4* qf, int kq, int dq, int g, int t, int lane,
                                       float (&acc)[4][4]) {
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {                      // chunk: dims 128dq + 32t + 16cc ..
        uint32_t a[4][4];
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) load_frag(qf, 4 * cc + wi, lane, a[wi]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t row = 32 * kq + 8 * j + g;
            const uint32_t chunk = (8 * dq + 2 * t + cc) ^ (row & 7u);
            const uint4 v = *reinterpret_cast<const uint4*>(sb + row * D + (chunk << 4));
            const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {              // word wi: k-step 4cc + wi
                uint32_t lo, hi;
                e4m3x4_to_f16(words[wi], lo, hi);
                mma16816<false>(acc[j], a[wi], lo, hi);
            }
        }
    }
}

// ---- O += P V for this warp's 64 dims: k-step ks covers keys 16ks .. 16ks+15, lane (g, t)
//      converts keys k0 = 16ks + 8kp + 2t and k0 + 1 (kp = 0, 1) at dims 64w + 8g .. +7.
//      The B fragment of n-tile n holds (k0, k0 + 1) at dim 64w + 8g + n, so the two keys'
//      code words are first interleaved nibble by nibble (byte i of `ev`: dim 2i of k0 in
//      the low nibble, of k0 + 1 in the high one; `od`: dim 2i + 1): one conversion then
//      yields a fragment register, and the two keys' scales (same 16-dim group) multiply
//      it as one f16x2 pair.  Every product is the exact dequantised value, so the MMAs
//      see the same operands as with a per-key conversion.
template <bool QF4>
__device__ __forceinline__ void pv_fp4(const uint8_t* sb, const DecodeSmem& sm, int warp, int lane, float (&o)[8][4]) {
    const int g = lane >> 2, t = lane & 3, mi = lane >> 3, mj = lane & 7;
    const uint32_t p0 = smem_u32(sm.p[0]);
    const int prow = ((mi & 1) << 3) + mj;
    const uint32_t ci = 2 * warp + (g >> 2);             // the 16-byte code chunk of dims 64w + 8g ..
#pragma unroll
    for (int ks = 0; ks < DT_KEYS / 16; ++ks) {
        uint32_t a[4];
        ldmatrix_x4(a, p0 + sw_chunk(HEADS, prow, 2 * ks + (mi >> 1)));
        uint32_t bf[2][8];
#pragma unroll
        for (int kp = 0; kp < 2; ++kp) {
            const uint32_t k0 = 16 * ks + 8 * kp + 2 * t;
            const uint32_t w0 = *reinterpret_cast<const uint32_t*>(
                sb + (QF4 ? fp4q_chunk(k0, ci) : k0 * ROW_CODES + (fp4_chunk(k0, ci) << 4)) + 4 * (g & 3));
            const uint32_t w1 = *reinterpret_cast<const uint32_t*>(
                sb + (QF4 ? fp4q_chunk(k0 + 1, ci) : (k0 + 1) * ROW_CODES + (fp4_chunk(k0 + 1, ci) << 4)) + 4 * (g & 3));
            const uint8_t* sc = sb + (QF4 ? ST4_SCALE_OFF : ST_SCALE_OFF) + k0 * ST_SCALE_LD + 4 * warp + (g >> 1);
            const uint32_t s = e4m3x2_to_f16x2(static_cast<uint32_t>(sc[0]) | (static_cast<uint32_t>(sc[ST_SCALE_LD]) << 8));
            const uint32_t ev = (w0 & 0x0F0F0F0Fu) | ((w1 << 4) & 0xF0F0F0F0u);
            const uint32_t od = ((w0 >> 4) & 0x0F0F0F0Fu) | (w1 & 0xF0F0F0F0u);
            uint32_t he[4], ho[4];
            e2m1x8_to_f16(ev, he);
            e2m1x8_to_f16(od, ho);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                bf[kp][2 * i] = hmul2_u32(he[i], s);
                bf[kp][2 * i + 1] = hmul2_u32(ho[i], s);
            }
        }
#pragma unroll
        for (int n = 0; n < 8; ++n) mma16816<false>(o[n], a, bf[0][n], bf[1][n]);
    }
}

__device__ __forceinline__ void pv_swa16(const uint8_t* sb, const DecodeSmem& sm, int warp, int lane,
                                         float (&o)[8][4]) {
    const int g = lane >> 2, t = lane & 3, mi = lane >> 3, mj = lane & 7;
    const uint32_t p0 = smem_u32(sm.p[0]), p1 = smem_u32(sm.p[1]);
    const int prow = ((mi & 1) << 3) + mj;
#pragma unroll
    for (int ks = 0; ks < DT_KEYS16 / 16; ++ks) {
        uint32_t a[4], alo[4];
        ldmatrix_x4(a, p0 + sw_chunk(HEADS, prow, 2 * ks + (mi >> 1)));
        ldmatrix_x4(alo, p1 + sw_chunk(HEADS, prow, 2 * ks + (mi >> 1)));
        uint32_t bf[2][8];
#pragma unroll
        for (int kp = 0; kp < 2; ++kp) {
            const uint32_t key = 16 * ks + 8 * kp + 2 * t;
            const uint4 v0 = *reinterpret_cast<const uint4*>(sb + sw_chunk(DT_KEYS16, key, 8 * warp + g));
            const uint4 v1 = *reinterpret_cast<const uint4*>(sb + sw_chunk(DT_KEYS16, key + 1, 8 * warp + g));
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
    const uint32_t p0 = smem_u32(sm.p[0]);
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

template <bool QF4>
__global__ void __launch_bounds__(DT_THREADS, DT_CTAS_PER_SM)
attend_rows_kernel(AttnParams p, const __grid_constant__ CUtensorMap tmap_q,
                   const __grid_constant__ CUtensorMap tmap_swa) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    DecodeSmem& sm = *reinterpret_cast<DecodeSmem*>(
        smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));

    const int64_t r = blockIdx.x;                     // query row
    const int sp = blockIdx.y;                        // = rank in the row's cluster
    const int ns = p.n_split;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int g = lane >> 2;

    // ---- set-up that reads nothing written by earlier kernels (the variant's tensor memory
    //      is allocated before dependents may launch, so none of them can hold it first)
    if (tid == 0) {
        mbar_init(&sm.bar_q, 1);
        for (int s = 0; s < DT_STAGES; ++s) mbar_init(&sm.full[s], DT_THREADS);
        if (QF4) mbar_init(&sm.bar_mma, 1);
        mbar_fence_init();
        sm.fail = 0;
    }
    if (QF4 && warp == 0) tmem_alloc(&sm.tmem, QT_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    griddep_launch_dependents();
    griddep_wait();
    const uint32_t tm = QF4 ? sm.tmem : 0u;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;

    const int64_t b = r / p.q_per_seq;
    const int qi = static_cast<int>(r - b * p.q_per_seq);
    const uint32_t limit = wait_limit(p.err);
    // the row's SWA rows: buffer rows [swa_base, swa_base + span) of sequence b, visible in
    // [swa_lo, swa_hi] (decode: the whole buffer; prefill: the query's own window)
    const int swa_keys = p.swa_fp8 ? DT_KEYS : DT_KEYS16;
    int64_t swa_base = 0, swa_lo = 0, swa_hi = p.swa_rows - 1, span = p.swa_rows;
    if (p.q_pos) {
        const int64_t q0 = p.q_pos[b];
        swa_base = qi;
        swa_lo = max(static_cast<int64_t>(qi), static_cast<int64_t>(WINDOW - 1) - q0);
        swa_hi = qi + WINDOW - 1;
        span = WINDOW;
    }
    const int swa_tiles = static_cast<int>((span + swa_keys - 1) / swa_keys);
    const int total = DT_MAIN_TILES + swa_tiles;
    // this CTA's tiles: k = sp, sp + ns, ... of the row's list (main tiles 0..7, then the
    // SWA tiles), dealt round robin so every CTA gets the same mix.  Tile number u (0..)
    // of the CTA:
    const int n_mine = total > sp ? (total - sp + ns - 1) / ns : 0;
    const int n_main_mine = DT_MAIN_TILES > sp ? (DT_MAIN_TILES - sp + ns - 1) / ns : 0;
    const auto tile_of = [&](int u) { return sp + u * ns; };   // row tile of the CTA's u-th tile
    const auto exists = [&](int t) {
        if (t < DT_MAIN_TILES) return true;              // masked slots cost no gather
        const int64_t lo = swa_base + static_cast<int64_t>(t - DT_MAIN_TILES) * swa_keys;
        return lo + swa_keys - 1 >= swa_lo && lo <= swa_hi;
    };
    const auto next_u = [&](int u) {
        for (int v = u + 1; v < n_mine; ++v)
            if (exists(tile_of(v))) return v;
        return -1;
    };
    const int u0 = (n_mine > 0 && exists(tile_of(0))) ? 0 : next_u(0);

    if (tid == 0) {
        mbar_arrive_expect_tx(&sm.bar_q, DT_Q_BYTES);
        for (int cb = 0; cb < D / 64; ++cb)
            tma_load_2d(sm.u.q + cb * HEADS * 128, &tmap_q, 64 * cb, static_cast<int>(r * HEADS), &sm.bar_q);
    }
    const int64_t seq_off = p.kv_offsets[b];
    const int64_t n_b = p.kv_offsets[b + 1] - seq_off;
    // a main slot's cache row, or -1 (absent, or past the context: skipped and reported)
    const auto slot_pos = [&](int slot) {
        const int32_t v = __ldg(p.topk_idx + r * TOPK + slot);
        const bool bad = v >= n_b;
        if (bad && p.err) atomicOr(p.err, ERR_DEVICE);
        return (v >= 0 && !bad) ? static_cast<int32_t>(p.rows.row(b, seq_off, v)) : -1;
    };

    // ---- tile loads: every thread issues its share and arrives on full[st] when its own
    //      copies land (bf16 SWA: thread 0 arms the TMA bytes, the others arrive at once)
    const auto issue = [&](int t, int st) {
        uint8_t* sb = sm.stage[st];
        if (t < DT_MAIN_TILES) {                         // codes + scales of 64 rows, masked rows zero
            // thread -> code chunk c = tid % 16 of rows tid / 16 + 16k, and (first 128 threads)
            // scale half tid % 2 of row tid / 2; the slots are read before any copy is issued
            constexpr int CPT = DT_KEYS * (ROW_CODES / 16) / DT_THREADS;   // 4
            static_assert(DT_KEYS * (ROW_SCALES / 16) <= DT_THREADS, "one scale chunk per thread");
            const int key0 = t * DT_KEYS;
            const int c = tid & 15, kk0 = tid >> 4;
            int32_t v[CPT];
#pragma unroll
            for (int k = 0; k < CPT; ++k) v[k] = sm.main_pos[key0 + kk0 + 16 * k];
            const int skk = tid >> 1, sc = tid & 1;
            const int32_t sv = tid < 2 * DT_KEYS ? sm.main_pos[key0 + skk] : -1;
#pragma unroll
            for (int k = 0; k < CPT; ++k) {
                const int kk = kk0 + 16 * k;
                const int64_t row = v[k];                // cache row (-1: masked)
                cp_async_16(smem_u32(sb + (QF4 ? fp4q_chunk(kk, c) : kk * ROW_CODES + (fp4_chunk(kk, c) << 4))),
                            p.codes + (v[k] >= 0 ? row * ROW_CODES + 16 * c : 0), v[k] >= 0 ? 16 : 0);
            }
            if (tid < 2 * DT_KEYS)
                cp_async_16(smem_u32(sb + (QF4 ? ST4_SCALE_OFF : ST_SCALE_OFF) + skk * ST_SCALE_LD + 16 * sc),
                            p.scales + (sv >= 0 ? static_cast<int64_t>(sv) * ROW_SCALES + 16 * sc : 0), sv >= 0 ? 16 : 0);
            cp_async_mbar_arrive_noinc(&sm.full[st]);
        } else if (p.swa_fp8) {                          // E4M3 rows + f32 row scales
            const int64_t lo = swa_base + static_cast<int64_t>(t - DT_MAIN_TILES) * DT_KEYS;
            const int64_t row0 = b * p.swa_rows + lo;
            for (int id = tid; id < DT_KEYS * (D / 16); id += DT_THREADS) {
                const int kk = id >> 5, c = id & 31;
                const bool in = lo + kk < p.swa_rows;
                const uint8_t* src = p.swa_kv8 + (in ? (row0 + kk) * D + 16 * c : 0);
                cp_async_16(smem_u32(sb + kk * D + ((c ^ (kk & 7)) << 4)), src, in ? 16 : 0);
            }
            if (tid < DT_KEYS) {
                const bool in = lo + tid < p.swa_rows;
                cp_async_4(smem_u32(sb + ST8_SCALE_OFF + 4 * tid), p.swa_kscale + (in ? row0 + tid : 0), in ? 4 : 0);
            }
            cp_async_mbar_arrive_noinc(&sm.full[st]);
        } else if (tid == 0) {                           // bf16 rows by TMA (rows past the
            fence_proxy_async_smem();                    // buffer read as zero)
            mbar_arrive_expect_tx(&sm.full[st], DT_KEYS16 * D * 2);
            const int64_t lo = swa_base + static_cast<int64_t>(t - DT_MAIN_TILES) * DT_KEYS16;
            for (int cb = 0; cb < D / 64; ++cb)
                tma_load_3d(sb + cb * DT_KEYS16 * 128, &tmap_swa, 64 * cb, static_cast<int>(lo), static_cast<int>(b),
                            &sm.full[st]);
        } else {
            mbar_arrive(&sm.full[st]);
        }
    };
    // the slots of this CTA's main tiles (tiles sp, sp + ns, ... < 8)
    for (int j = tid; j < DT_KEYS * n_main_mine; j += DT_THREADS) {
        const int slot = (sp + (j / DT_KEYS) * ns) * DT_KEYS + (j % DT_KEYS);
        sm.main_pos[slot] = slot_pos(slot);
    }
    __syncthreads();
    int armed[DT_STAGES] = {};                           // full phases armed per stage
    int u_ahead = u0;                                    // next tile (CTA numbering) to issue
    for (int k = 0; k < DT_STAGES && u_ahead >= 0; ++k, u_ahead = next_u(u_ahead)) {
        issue(tile_of(u_ahead), k);
        ++armed[k];
    }

    // ---- the query's A fragments (f16) in fragment order: entry (dq, ks, lane) holds rows
    //      g, g + 8 at dims d0 .. d0+3, d0 = 128 dq + 32 (lane % 4) + 4 ks
    const bool q_ok = mbar_wait(&sm.bar_q, 0, p.err, limit);
    if (!q_ok) sm.fail = 1;
    {
        const int ks = tid >> 5, t = lane & 3;
#pragma unroll
        for (int dq = 0; dq < 4; ++dq) {
            const uint32_t d0 = 128 * dq + 32 * t + 4 * ks;
            uint32_t a[4];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const uint32_t h = g + 8 * hh;
                const uint2 v = *reinterpret_cast<const uint2*>(
                    sm.u.q + (d0 >> 6) * HEADS * 128 + h * 128 + ((((d0 & 63) >> 3) ^ (h & 7)) << 4) + (d0 & 7) * 2);
                a[hh] = bf16x2_to_f16x2(v.x);
                a[2 + hh] = bf16x2_to_f16x2(v.y);
            }
            sm.qf[dq][ks][lane] = make_uint4(a[0], a[1], a[2], a[3]);
        }
    }
    if (QF4) {
        // NVFP4 query, quantised here from the bf16 query in shared memory (the cache's own
        // rule): thread -> head tid / 16, dims 32 (tid % 16) .. +31 = code chunk tid % 16 of
        // the head's row, two 16-dim groups; the chunk goes to the MMA's query panels and
        // the two scale bytes to a scratch row in the P buffer (unused until the first tile)
        const int h = tid >> 4, c = tid & 15;
        uint4 chunk;
        uint8_t sc[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const uint32_t d0 = 32 * c + 16 * e;         // group 2c + e: dims d0 .. d0+15
            const uint8_t* src = sm.u.q + (d0 >> 6) * HEADS * 128 + h * 128;
            const uint4 v0 = *reinterpret_cast<const uint4*>(src + ((((d0 & 63) >> 3) ^ (h & 7)) << 4));
            const uint4 v1 = *reinterpret_cast<const uint4*>(src + (((((d0 & 63) >> 3) + 1) ^ (h & 7)) << 4));
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            uint16_t hv[16];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                hv[2 * k] = static_cast<uint16_t>(w[k] & 0xFFFFu);
                hv[2 * k + 1] = static_cast<uint16_t>(w[k] >> 16);
            }
            uint2 cw;
            sc[e] = nvfp4_group(hv, cw);
            if (e == 0) {
                chunk.x = cw.x;
                chunk.y = cw.y;
            } else {
                chunk.z = cw.x;
                chunk.w = cw.y;
            }
        }
        *reinterpret_cast<uint4*>(&sm.qb[c >> 3][h][((c & 7) ^ (h & 7)) << 4]) = chunk;
        fence_proxy_async_smem();                        // the query panels, to the tensor core
        sm.p[0][h * ROW_SCALES + 2 * c] = sc[0];
        sm.p[0][h * ROW_SCALES + 2 * c + 1] = sc[1];
        __syncthreads();
        // scale word s of head h -> lane h of every quarter, column QT_SFB + 4 s
        if (warp < 4) {
            uint32_t y[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) y[k] = 0u;
            if (lane < HEADS) {
#pragma unroll
                for (int k = 0; k < 8; ++k) y[4 * k] = *reinterpret_cast<const uint32_t*>(&sm.p[0][lane * ROW_SCALES + 4 * k]);
            }
            tmem_st32(tm + lane_base + QT_SFB, y);
        }
        tc_fence_before();
    }
    __syncthreads();                                     // the query's space now holds S
    if (QF4) tc_fence_after();
    uint32_t n_fp4 = 0;                                  // variant: FP4 tiles (= MMA batches) so far

    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    const int t4 = lane & 3;
    const int kq = warp & 1, dq = warp >> 1;
    const uint4* qf = &sm.qf[dq][0][0];
    float m_ref[2] = {-INFINITY, -INFINITY};             // heads 2w, 2w+1 (warp-uniform)
    float l_lane[2] = {0.0f, 0.0f};                      // this lane's share of their sums
    // ---- O = alpha * O + P V of a tile (alpha is 1 unless a reference max moved); FP8
    //      SWA: O + smax * (P' V') is done as (O / smax + P' V') * smax
    const auto pv_step = [&](TileKind kind, const uint8_t* sb, float smax) {
        const bool swa8 = kind == TK_SWA8;
        const float inv = swa8 && smax > 0.0f ? 1.0f / smax : 1.0f;
        const float al = sm.alpha[g] * inv, ah = sm.alpha[g + 8] * inv;
        if (al != 1.0f || ah != 1.0f) {                  // (a reference max rarely moves)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                o[nt][0] *= al;
                o[nt][1] *= al;
                o[nt][2] *= ah;
                o[nt][3] *= ah;
            }
        }
        if (kind == TK_FP4) pv_fp4<QF4>(sb, sm, warp, lane, o);
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
    };
    int i = 0;
    // sm.fail is read only right after a barrier (every write precedes it)
    for (int u = u0; u >= 0; u = next_u(u), ++i) {
        const int t = tile_of(u);
        const int st = i % DT_STAGES;
        const TileKind kind = t < DT_MAIN_TILES ? TK_FP4 : (p.swa_fp8 ? TK_SWA8 : TK_SWA16);
        const uint8_t* sb = sm.stage[st];
        // ---- 1. tile i is in stage st
        if (!mbar_wait(&sm.full[st], (i / DT_STAGES) & 1, p.err, limit)) sm.fail = 1;
        if (QF4 && kind == TK_FP4) {
            // variant: the tile's scale words to tensor memory (warps 0-3: rows lane and 32 +
            // lane; rows 64..127 of the M = 128 MMA get zero scales), then thread 0 issues the
            // 8 MMAs; the previous tile's MMAs are complete (observed before the last barrier)
            fence_proxy_async_smem();                    // the landed codes, to the tensor core
            if (warp < 4) {
                tc_fence_after();
                uint32_t y[32];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    y[4 * k] = *reinterpret_cast<const uint32_t*>(sb + ST4_SCALE_OFF + lane * ST_SCALE_LD + 4 * k);
                    y[4 * k + 1] =
                        *reinterpret_cast<const uint32_t*>(sb + ST4_SCALE_OFF + (32 + lane) * ST_SCALE_LD + 4 * k);
                    y[4 * k + 2] = 0u;
                    y[4 * k + 3] = 0u;
                }
                tmem_st32(tm + lane_base + QT_SFA, y);
            }
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            if (tid == 0) {
                constexpr uint32_t idesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(HEADS >> 3) << 17) |
                                           (static_cast<uint32_t>(128 >> 4) << 24);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint64_t da = umma_desc_sw128(smem_u32(sb) + (k >> 2) * ST4_PANEL + (k & 3) * 32, 16, 1024);
                    const uint64_t db =
                        umma_desc_sw128(smem_u32(&sm.qb[0][0][0]) + (k >> 2) * HEADS * 128 + (k & 3) * 32, 16, 1024);
                    mma_nvf4(tm + QT_D, da, db, idesc, tm + QT_SFA + 4 * k, tm + QT_SFB + 4 * k, k > 0);
                }
                mma_commit(&sm.bar_mma);
            }
        }

        // ---- 2. S partial of this warp's keys and dim quarter -> shared
        if (QF4 && kind == TK_FP4) {
            // S^T of this tile (rows = keys 32 warp + lane)
            if (warp < 2) {
                if (!mbar_wait(&sm.bar_mma, n_fp4 & 1, p.err, limit)) sm.fail = 1;
                tc_fence_after();
                uint32_t v[16];
                tmem_ld16(tm + lane_base + QT_D, v);
#pragma unroll
                for (int h = 0; h < HEADS; ++h) sm.u.s[0][h][32 * warp + lane] = __uint_as_float(v[h]);
                tc_fence_before();                       // before the next tile's MMAs overwrite S^T
            }
        } else {
            float acc[4][4] = {};
            if (kind == TK_FP4) s_fp4(sb, qf, kq, dq, g, t4, lane, acc);
            else if (kind == TK_SWA16) s_swa16(sb, qf, kq, dq, g, t4, lane, acc);
            else s_swa8(sb, qf, kq, dq, g, t4, lane, acc);
            const int kb = kind == TK_SWA16 ? 16 * kq : 32 * kq;
            const int nj = kind == TK_SWA16 ? 2 : 4;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (j < nj) {
                    const int key = kb + 8 * j + 2 * t4;
                    *reinterpret_cast<float2*>(&sm.u.s[dq][g][key]) = make_float2(acc[j][0], acc[j][1]);
                    *reinterpret_cast<float2*>(&sm.u.s[dq][g + 8][key]) = make_float2(acc[j][2], acc[j][3]);
                }
            }
        }
        if (kind == TK_FP4) ++n_fp4;
        __syncthreads();
        if (sm.fail) break;
        // every warp is past tile i - 1: its stage takes the tile after tile i
        if (i >= 1 && u_ahead >= 0) {
            const int sn = (i + 1) % DT_STAGES;
            issue(tile_of(u_ahead), sn);
            ++armed[sn];
            u_ahead = next_u(u_ahead);
        }

        // ---- 3. softmax: warp w owns heads 2w, 2w+1; lane owns keys lane, lane+32.  The
        //      reference max m_ref (uniform in the warp) only moves when a score exceeds
        //      it by more than RESCALE_GAP (P <= e^RESCALE_GAP is still exact-width in
        //      f16 / bf16), found with one vote; row sums stay per lane until the end.
        const bool swa8 = kind == TK_SWA8;
        const int tile_keys = kind == TK_SWA16 ? DT_KEYS16 : DT_KEYS;
        const float* rs = reinterpret_cast<const float*>(sb + ST8_SCALE_OFF);
        bool valid[2];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int key = lane + 32 * jj;
            if (kind == TK_FP4) {
                valid[jj] = sm.main_pos[t * DT_KEYS + key] >= 0;
            } else {
                const int64_t row = swa_base + static_cast<int64_t>(t - DT_MAIN_TILES) * tile_keys + key;
                valid[jj] = key < tile_keys && row >= swa_lo && row <= swa_hi;
            }
        }
        float smax = 1.0f;
        if (swa8) {                                      // the tile's largest (visible) row scale
            smax = fmaxf(valid[0] ? rs[lane] : 0.0f, valid[1] ? rs[lane + 32] : 0.0f);
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
                const float sum = (QF4 && kind == TK_FP4)
                                      ? sm.u.s[0][h][key]
                                      : ((sm.u.s[0][h][key] + sm.u.s[1][h][key]) + sm.u.s[2][h][key]) +
                                            sm.u.s[3][h][key];
                sv[jj] = valid[jj] ? sum * p.sm_scale : -INFINITY;
                if (swa8 && valid[jj]) sv[jj] *= rs[key];
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
                    *reinterpret_cast<__half*>(sm.p[0] + off) = __float2half_rn(pw);
                } else if (kind == TK_FP4) {
                    *reinterpret_cast<__half*>(sm.p[0] + off) = __float2half_rn(pvv);
                } else {
                    const __nv_bfloat16 hi = __float2bfloat16_rn(pvv);
                    *reinterpret_cast<__nv_bfloat16*>(sm.p[0] + off) = hi;
                    *reinterpret_cast<__nv_bfloat16*>(sm.p[1] + off) =
                        __float2bfloat16_rn(pvv - __bfloat162float(hi));
                }
            }
            if (lane == 0) sm.alpha[h] = alpha;
        }
        __syncthreads();

        // ---- 4. P V of this tile
        pv_step(kind, sb, smax);
    }
    // ---- drain: every armed tile load has landed (all were consumed unless a wait failed);
    //      these waits keep the library's default bound whatever the caller's limit
    cp_async_wait<0>();
    if (tid == 0) {
        if (!q_ok) mbar_wait(&sm.bar_q, 0, p.err);
        for (int s2i = 0; s2i < DT_STAGES; ++s2i)
            if (armed[s2i] > 0) mbar_wait(&sm.full[s2i], (armed[s2i] - 1) & 1, p.err);
        if (QF4 && n_fp4 > 0) mbar_wait(&sm.bar_mma, (n_fp4 - 1) & 1, p.err);   // the last MMAs
    }
    const bool failed = sm.fail != 0;                    // final: written before a barrier
    // ---- row sums of this warp's heads (m, l of heads 2w, 2w+1)
    float l_tot[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float l = l_lane[hh];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, off);
        l_tot[hh] = l;
    }

    // ---- push this CTA's partial into the cluster: warp w's O fragment (64-dim block w)
    //      goes to CTA w % n_split, slot (w / n_split) * n_split + rank, lane-major (lane * 32
    //      + 4 nt + c holds o[nt][c]); m and l of every head go to every CTA.  The stages are
    //      the receiving buffer: each CTA arrives once it is done with its own.
    const uint32_t push_base = smem_u32(&sm.stage[0][0]);
    cluster_arrive();
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        if (lane == 0) {
            sm.m[2 * warp + hh] = failed ? -INFINITY : m_ref[hh];
            sm.l[2 * warp + hh] = failed ? 0.0f : l_tot[hh];
        }
    }
    __syncthreads();
    cluster_wait();                                   // every CTA is done with its stages
    {
        const uint32_t owner = static_cast<uint32_t>(warp % ns);
        const int slot = (warp / ns) * ns + sp;
        const uint32_t base = dsmem_addr(push_base, owner) + (slot * DT_OBLOCK_FLOATS + lane * 32) * 4;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) dsmem_st_f32x4(base + 16 * nt, o[nt][0], o[nt][1], o[nt][2], o[nt][3]);
        if (tid < HEADS * ns) {
            const int h = tid & 15, dst = tid >> 4;
            const uint32_t mine = push_base + (sp * HEADS + h) * 4;
            dsmem_st_f32(dsmem_addr(mine + DT_PM_OFFSET, static_cast<uint32_t>(dst)), sm.m[h]);
            dsmem_st_f32(dsmem_addr(mine + DT_PL_OFFSET, static_cast<uint32_t>(dst)), sm.l[h]);
        }
    }
    cluster_sync();

    // ---- merge the blocks this CTA owns (w = rank + k * n_split): thread tid takes
    //      fragment float4 (lane tid / 8, nt = tid % 8) of every sender's slot; its values
    //      are heads hg, hg + 8 at dims 64w + 16 t' + nt and 64w + 16 t' + 8 + nt
    const float* recv = reinterpret_cast<const float*>(&sm.stage[0][0]);
    const float* pm = recv + DT_PM_OFFSET / 4;        // [sender][16]
    const float* pl = recv + DT_PL_OFFSET / 4;
    const int src_lane = tid >> 3, nt = tid & 7;
    const int hg = src_lane >> 2, dd = 16 * (src_lane & 3) + nt;
    float wa[DT_MAX_CLUSTER], wb[DT_MAX_CLUSTER];
    float inv_a, inv_b;
    {
        float Ma = -INFINITY, Mb = -INFINITY;
        for (int s2i = 0; s2i < ns; ++s2i) {
            Ma = fmaxf(Ma, pm[s2i * HEADS + hg]);
            Mb = fmaxf(Mb, pm[s2i * HEADS + hg + 8]);
        }
        float La = 0.0f, Lb = 0.0f;
#pragma unroll
        for (int s2i = 0; s2i < DT_MAX_CLUSTER; ++s2i) {
            const float ma = s2i < ns ? pm[s2i * HEADS + hg] : -INFINITY;
            const float mb = s2i < ns ? pm[s2i * HEADS + hg + 8] : -INFINITY;
            wa[s2i] = ma != -INFINITY ? __expf(ma - Ma) : 0.0f;
            wb[s2i] = mb != -INFINITY ? __expf(mb - Mb) : 0.0f;
            if (s2i < ns) {
                La += wa[s2i] * pl[s2i * HEADS + hg];
                Lb += wb[s2i] * pl[s2i * HEADS + hg + 8];
            }
        }
        inv_a = 1.0f / La;
        inv_b = 1.0f / Lb;
    }
    for (int w = sp, k = 0; w < D / 64; w += ns, ++k) {
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
    if (QF4) {                                           // every tensor-memory access is done
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 0) tmem_dealloc(tm, QT_COLS);
    }
}

}  // namespace

int attend_rows_swa_tiles(int64_t swa_rows, bool prefill, bool swa_fp8) {
    const int64_t span = prefill ? WINDOW : std::max<int64_t>(swa_rows, 1);
    return static_cast<int>(ceil_div(span, swa_fp8 ? DT_KEYS : DT_KEYS16));
}

int attend_rows_split(int64_t rows, int swa_tiles, bool swa_fp8) {
    // CTA sp of n takes the row's tiles sp, sp + n, ...; the cost of a row is its
    // busiest CTA's tiles (a bf16 SWA tile of 32 rows counts 0.7 of a 64-row tile) times
    // the waves of CTAs (two per SM); among equal costs, fewer CTAs
    const int total = DT_MAIN_TILES + swa_tiles;
    const double w_swa = swa_fp8 ? 1.0 : 0.7;
    double best = 1e300;
    int best_n = 1;
    for (int n = 1; n <= DT_MAX_CLUSTER && n <= total; ++n) {
        double busiest = 0.0;
        for (int sp = 0; sp < n; ++sp) {
            double c = 0.0;
            for (int k = sp; k < total; k += n) c += k < DT_MAIN_TILES ? 1.0 : w_swa;
            busiest = std::max(busiest, c);
        }
        const double cost = static_cast<double>(ceil_div(rows * n, DT_SMS * DT_CTAS_PER_SM)) * busiest;
        if (cost < best - 1e-9) {
            best = cost;
            best_n = n;
        }
    }
    return best_n;
}

csa2_status launch_attend_rows(const AttnParams& p, const CUtensorMap& tmap_q, const CUtensorMap& tmap_swa,
                               cudaStream_t stream) {
    const int64_t rows = static_cast<int64_t>(p.batch) * p.q_per_seq;
    if (rows == 0) return CSA2_OK;
    if (p.n_split < 1 || p.n_split > DT_MAX_CLUSTER) return CSA2_ERR_UNSUPPORTED;
    const int smem = static_cast<int>(sizeof(DecodeSmem) + 1024);
    const bool qf4 = p.q_nvfp4 != 0;
    const void* fn = qf4 ? reinterpret_cast<const void*>(attend_rows_kernel<true>)
                         : reinterpret_cast<const void*>(attend_rows_kernel<false>);
    if (!opt_in_smem(fn, smem)) return check_launch("attend_rows_kernel smem attribute");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(rows), static_cast<unsigned>(p.n_split));
    cfg.blockDim = dim3(DT_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = static_cast<unsigned>(p.n_split);
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (qf4) cudaLaunchKernelEx(&cfg, attend_rows_kernel<true>, p, tmap_q, tmap_swa);
    else cudaLaunchKernelEx(&cfg, attend_rows_kernel<false>, p, tmap_q, tmap_swa);
    return check_launch("attend_rows_kernel");
}

}  // namespace csa2
