// Shared device helpers of libcsa2: number-format conversions, warp-level tensor-core
// fragments (mma.sync / ldmatrix) and the launch-error plumbing.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa2.h"

namespace csa2 {

constexpr int D = CSA2_D;
constexpr int GROUP = CSA2_GROUP;
constexpr int ROW_CODES = CSA2_ROW_CODES;
constexpr int ROW_SCALES = CSA2_ROW_SCALES;
constexpr int HEADS = CSA2_HEADS;
constexpr int IDX_HEADS = CSA2_IDX_HEADS;
constexpr int IDX_DIM = CSA2_IDX_DIM;
constexpr int TOPK = CSA2_TOPK;
constexpr int WINDOW = CSA2_WINDOW;
constexpr int POOL_BLOCKS = CSA2_POOL_BLOCKS;
constexpr int POOL_BLOCK = CSA2_POOL_BLOCK;
constexpr int POOL_POSITIONS = POOL_BLOCKS * POOL_BLOCK;   // 16,384

// Device error word bits (kept in the first 16 bytes of a workspace).
constexpr unsigned ERR_TIMEOUT = 1u;
constexpr unsigned ERR_DEVICE = 2u;

// ------------------------------------------------------------------ formats

// E4M3 byte -> float (exact; cvt to f16 is exact for every finite E4M3 value).
__device__ __forceinline__ float e4m3_to_float(uint8_t b) {
    __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(b), __NV_E4M3);
    return __half2float(__half(h));
}

// Two E4M3 bytes (low byte = first element) -> packed f16x2 bits (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t two) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
    return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

// E4M3 code of a finite v >= 0: round to nearest, ties to even, saturating at 448.
// Written from the format: below 2^-6 the grid is m * 2^-9 (m = 0..8, and m = 8 is the
// smallest normal, code 8); at and above it, a binade 2^e holds 8 values
// 2^e * (1 + k/8) with code ((e + 7) << 3) | k.  Scaling by a power of two is exact in
// fp32 and rint() rounds half to even.
__device__ __forceinline__ uint8_t e4m3_encode_rne_sat(float v) {
    if (!(v < 448.0f)) return 126;                       // >= 448 (and +inf) -> 448
    if (v < 0.015625f) {                                 // 2^-6
        return static_cast<uint8_t>(__float2int_rn(v * 512.0f));   // 0 .. 8
    }
    const int e = static_cast<int>((__float_as_uint(v) >> 23) & 0xFFu) - 127;   // -6 .. 8
    int m = __float2int_rn(ldexpf(v, 3 - e));            // 8 .. 16
    int ee = e;
    if (m == 16) {
        m = 8;
        ++ee;
    }
    const int code = ((ee + 7) << 3) | (m - 8);
    return static_cast<uint8_t>(code > 126 ? 126 : code);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// E2M1 magnitude code of y >= 0 (finite): nearest of {0,.5,1,1.5,2,3,4,6}, ties to the
// even code, values above 6 saturate.  At each midpoint the comparison is strict when
// the lower neighbour's code is even and inclusive when the upper one's is.
__device__ __forceinline__ uint32_t e2m1_magnitude(float y) {
    return static_cast<uint32_t>(y > 0.25f) + static_cast<uint32_t>(y >= 0.75f) +
           static_cast<uint32_t>(y > 1.25f) + static_cast<uint32_t>(y >= 1.75f) +
           static_cast<uint32_t>(y > 2.5f) + static_cast<uint32_t>(y >= 3.5f) +
           static_cast<uint32_t>(y > 5.0f);
}

// One NVFP4 group of 16 bf16 values (the FP4 KV section's format without its global
// scale): scale = E4M3 RNE of amax/6 (saturating), codes = sign | E2M1 RNE of |x|/scale
// (saturating), the sign kept when the magnitude rounds to 0.  Returns the scale byte;
// codes gets the 16 nibbles, element i in bits 4i.. of the 64-bit pair (x low, y high).
// The divisions are IEEE fp32: both operands carry at most 8 significant bits, so the
// quotient lands exactly on a rounding midpoint iff the exact quotient does.
__device__ __forceinline__ uint8_t nvfp4_group(const uint16_t (&h)[16], uint2& codes) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(bf16_bits_to_float(h[i])));
    const uint8_t scale_code = e4m3_encode_rne_sat(amax / 6.0f);
    const float s = e4m3_to_float(scale_code);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t sign = (h[i] >> 15) & 1u;
        uint32_t mag = 0;
        if (s > 0.0f) mag = e2m1_magnitude(fabsf(bf16_bits_to_float(h[i])) / s);
        const uint32_t code = (sign << 3) | mag;
        if (i < 8) lo |= code << (4 * i);
        else       hi |= code << (4 * (i - 8));
    }
    codes.x = lo;
    codes.y = hi;
    return scale_code;
}

// Packed bf16x2 bits -> packed f16x2 bits (round to nearest; exact for the normal f16
// range, which holds every |x| in [2^-14, 65504] with <= 8 significant bits).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
    float lo = __uint_as_float(v << 16);
    float hi = __uint_as_float(v & 0xFFFF0000u);
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Monotone map of a float score to an unsigned key: a larger key is a larger score.
// -inf (an absent candidate) maps to 0, which no finite score reaches; -0 and +0 map
// to the same key.
__device__ __forceinline__ uint32_t score_key(float s) {
    if (s == -INFINITY) return 0u;
    s = s + 0.0f;                                   // -0 -> +0
    uint32_t b = __float_as_uint(s);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Inverse of score_key for keys of finite scores.
__device__ __forceinline__ float key_score(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// ------------------------------------------------------------------ mma.sync helpers

// D = A(16x16, row) * B(16x8, col) + C, f16 inputs, f32 accumulate.
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4],
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Same with bf16 inputs.
__device__ __forceinline__ void mma_16816_bf16(float (&c)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D = A(16x32, row) * B(32x8, col) + C, E4M3 inputs, f32 accumulate.
__device__ __forceinline__ void mma_16832_e4m3(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t smem_addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t smem_addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_addr));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 128-bit global load that bypasses L1 allocation (streamed once).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// cp.async (LDGSTS): global -> shared copies that complete asynchronously; a thread
// waits only for its own copies (wait_group), so a lane that reads back exactly what it
// copied needs no barrier.  src_bytes < size zero-fills the rest.
__device__ __forceinline__ void cp_async_16(uint32_t smem_addr, const void* gmem, int src_bytes = 16) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n"
                 :: "r"(smem_addr), "l"(gmem), "r"(src_bytes));
}

__device__ __forceinline__ void cp_async_4(uint32_t smem_addr, const void* gmem, int src_bytes = 4) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n"
                 :: "r"(smem_addr), "l"(gmem), "r"(src_bytes));
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" :: "n"(N)); }

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) {
    return (a + b - 1) / b;
}

// Cache row of position pos of sequence b: seq_off + pos (contiguous, packed by
// kv_offsets), or through a page table: page_table[b * pages_per_seq + pos / page_rows] *
// page_rows + pos % page_rows (page_rows a multiple of 128, so a 128-position tile and an
// 8-position HSI block never straddle two pages).
struct RowMap {
    const int32_t* page_table;       // nullptr: contiguous
    int32_t page_rows;
    int32_t pages_per_seq;
    __device__ __forceinline__ int64_t row(int64_t b, int64_t seq_off, int64_t pos) const {
        if (page_table == nullptr) return seq_off + pos;
        const int64_t pg = __ldg(page_table + b * pages_per_seq + pos / page_rows);
        return pg * page_rows + pos % page_rows;
    }
};

// Row pitch (in elements) of the library's padded score and block-maxima rows: a multiple
// of 64, so fp32 rows start 256-byte aligned.  Every scratch of those rows uses this rule.
__host__ __device__ __forceinline__ int64_t padded_ld(int64_t n) { return (n + 63) / 64 * 64; }

}  // namespace csa2

// Host-side launch helpers (defined in api.cu).
namespace csa2 {
csa2_status check_launch(const char* what);
// Records a failed CUDA runtime call for csa2_last_error() and returns CSA2_ERR_CUDA.
csa2_status fail_cuda(const char* what, cudaError_t e);
// Raises a kernel's dynamic shared-memory limit once per (kernel, device); the first
// call on a device should come before any stream capture.  False on failure.
bool opt_in_smem(const void* kernel, int bytes);
}
