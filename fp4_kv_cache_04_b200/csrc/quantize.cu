// FP4 main-KV quantiser: bf16 latent rows -> E2M1 codes + one E4M3 scale per 16 channels
// ("FP4 KV, Bounded Replay, and Other Extensions" section of the thecryptopost.io
// DeepSeek-V4.1-Flash article: E2M1 with one E4M3 scale per 16 channels, NVFP4 without
// its global scale), optionally after ratio-2 merging of adjacent positions (CSA2
// section: the encoder compresses at ratio 2; tldrocket.com: merging of adjacent
// positions).
//
// One warp per output row, one lane per 16-channel group: a warp reads 1 KB (2 KB at
// ratio 2) of contiguous bf16 and writes 256 contiguous code bytes + 32 scale bytes.
// The rounding decisions use IEEE fp32 division (never a reciprocal multiply): both
// operands carry at most 8 significant bits, so the fp32 quotient lands exactly on a
// rounding midpoint iff the exact quotient does, and never crosses one.
#include "common.cuh"

namespace csa2 {

namespace {

// Round-to-nearest-even of a float64 value to bf16, through a round-to-odd float32
// intermediate (16 spare bits make the second rounding exact).
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double m) {
    float f = __double2float_rz(m);
    if (static_cast<double>(f) != m) f = __uint_as_float(__float_as_uint(f) | 1u);
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&h);
}

__device__ __forceinline__ void unpack8(const uint4& v, uint16_t (&h)[16], int base) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        h[base + 2 * i] = static_cast<uint16_t>(w[i] & 0xFFFFu);
        h[base + 2 * i + 1] = static_cast<uint16_t>(w[i] >> 16);
    }
}

// One 16-channel group (nvfp4_group): 8 packed code bytes and the scale byte stored.
__device__ __forceinline__ void store_group(const uint16_t (&h)[16], uint8_t* code_dst, uint8_t* scale_dst) {
    uint2 v;
    const uint8_t scale_code = nvfp4_group(h, v);
    *reinterpret_cast<uint2*>(code_dst) = v;
    *scale_dst = scale_code;
}

__global__ void __launch_bounds__(256)
quantize_kernel(const uint16_t* __restrict__ x, int64_t n_out, int ratio,
                const int64_t* __restrict__ dst_row, uint8_t* __restrict__ codes,
                uint8_t* __restrict__ scales) {
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
    if (row >= n_out) return;
    const int lane = threadIdx.x & 31;

    uint16_t h[16];                       // the group's 16 bf16 inputs (after merging)
    if (ratio == 1) {
        const uint16_t* src = x + row * D + lane * GROUP;
        unpack8(ldg_stream(src), h, 0);
        unpack8(ldg_stream(src + 8), h, 8);
    } else {
        uint16_t a[16], b[16];
        const uint16_t* s0 = x + (2 * row) * D + lane * GROUP;
        const uint16_t* s1 = s0 + D;
        unpack8(ldg_stream(s0), a, 0);
        unpack8(ldg_stream(s0 + 8), a, 8);
        unpack8(ldg_stream(s1), b, 0);
        unpack8(ldg_stream(s1 + 8), b, 8);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            // the pair sum is exact in float64; halving is exact; one rounding to bf16
            const double m = (static_cast<double>(bf16_bits_to_float(a[i])) +
                              static_cast<double>(bf16_bits_to_float(b[i]))) * 0.5;
            h[i] = f64_to_bf16_rne(m);
        }
    }

    const int64_t out_row = dst_row ? dst_row[row] : row;
    store_group(h, codes + out_row * ROW_CODES + lane * 8, scales + out_row * ROW_SCALES + lane);
}

// Cache append of new positions: warp per row.  Lane l quantises channels 16l..16l+15
// of the main-KV row (as above) and indexer values 2l, 2l+1: kscale = amax / 448 and
// code = sign | E4M3 RNE saturating of |k / kscale|, both quotients IEEE fp32; an
// all-zero row gets kscale 0 and zero codes.
__global__ void __launch_bounds__(256)
append_kernel(const uint16_t* __restrict__ latent, const float* __restrict__ proj, int64_t n,
              const int64_t* __restrict__ dst_row, uint8_t* __restrict__ codes,
              uint8_t* __restrict__ scales, uint8_t* __restrict__ idx_k, float* __restrict__ idx_kscale) {
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
    if (row >= n) return;
    const int lane = threadIdx.x & 31;
    const int64_t out_row = dst_row[row];

    uint16_t h[16];
    const uint16_t* src = latent + row * D + lane * GROUP;
    unpack8(ldg_stream(src), h, 0);
    unpack8(ldg_stream(src + 8), h, 8);
    store_group(h, codes + out_row * ROW_CODES + lane * 8, scales + out_row * ROW_SCALES + lane);

    const float2 k = __ldg(reinterpret_cast<const float2*>(proj + row * IDX_DIM) + lane);
    float amax = fmaxf(fabsf(k.x), fabsf(k.y));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
    const float ks = amax / 448.0f;
    uint32_t c0 = 0, c1 = 0;
    if (ks > 0.0f) {
        const float q0 = k.x / ks, q1 = k.y / ks;
        c0 = (signbit(q0) ? 0x80u : 0u) | e4m3_encode_rne_sat(fabsf(q0));
        c1 = (signbit(q1) ? 0x80u : 0u) | e4m3_encode_rne_sat(fabsf(q1));
    }
    reinterpret_cast<uint16_t*>(idx_k + out_row * IDX_DIM)[lane] = static_cast<uint16_t>(c0 | (c1 << 8));
    if (lane == 0) idx_kscale[out_row] = ks;
}

}  // namespace

csa2_status launch_append(const uint16_t* latent, const float* proj, int64_t n, const int64_t* dst_row,
                          uint8_t* codes, uint8_t* scales, uint8_t* idx_k, float* idx_kscale,
                          cudaStream_t stream) {
    if (n == 0) return CSA2_OK;
    const int rows_per_block = 8;
    append_kernel<<<static_cast<unsigned>(ceil_div(n, rows_per_block)), 32 * rows_per_block, 0, stream>>>(
        latent, proj, n, dst_row, codes, scales, idx_k, idx_kscale);
    return check_launch("append_kernel");
}

csa2_status launch_quantize(const uint16_t* x, int64_t n_in, int ratio, const int64_t* dst_row,
                            uint8_t* codes, uint8_t* scales, cudaStream_t stream) {
    const int64_t n_out = n_in / ratio;
    if (n_out == 0) return CSA2_OK;
    const int rows_per_block = 8;
    const int64_t grid = ceil_div(n_out, rows_per_block);
    quantize_kernel<<<static_cast<unsigned>(grid), 32 * rows_per_block, 0, stream>>>(
        x, n_out, ratio, dst_row, codes, scales);
    return check_launch("quantize_kernel");
}

}  // namespace csa2
