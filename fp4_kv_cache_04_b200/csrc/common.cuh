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

// float -> E4M3 byte, round to nearest even, saturating to +-448 (hardware cvt).
__device__ __forceinline__ uint8_t float_to_e4m3_satfinite(float v) {
    return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
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

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) {
    return (a + b - 1) / b;
}

}  // namespace csa2

// Host-side launch helpers (defined in api.cu).
namespace csa2 {
csa2_status check_launch(const char* what);
// Raises a kernel's dynamic shared-memory limit once per (kernel, device); the first
// call on a device should come before any stream capture.  False on failure.
bool opt_in_smem(const void* kernel, int bytes);
}
