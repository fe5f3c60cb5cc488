// Sparse attention over the selected FP4 main-KV rows joined with the sliding window.
//
// CSA2 section of the thecryptopost.io DeepSeek-V4.1-Flash article: every layer keeps
// its own main Q and SWA KV and attends over its Top-512 selection of the shared main
// KV; the Causal Encoder-Decoder section fixes the 128-token window; tldrocket.com: one
// 512-dim latent serves as both key and value.  Per query and head h:
//     out_h = softmax_j(sm_scale * q_h . row_j) . rows,   rows = selected FP4 rows
//                                                         (dequantised) ++ SWA rows.
//
// One CTA per query row.  Keys are processed in tiles of 128: the tile's FP4 rows are
// gathered and dequantised exactly to f16 (e2m1 x e4m3 has <= 6 significant bits and
// lies in [2^-10, 2688]) and the SWA rows converted bf16 -> f16, into a shared-memory
// tile with 16-byte chunks XOR-swizzled by row so that ldmatrix reads are conflict
// free.  S^T = K Q^T puts 16 keys per warp on the MMA M axis with the 16 heads on N;
// O = P V puts the 16 heads on M with each warp owning 64 of the 512 output dims.
// Softmax is online across tiles (running max and sum per head) in fp32; P is rounded
// to f16 for the second MMA.  Both MMAs accumulate in fp32.
#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

namespace {

constexpr int AT_WARPS = 8;
constexpr int AT_THREADS = AT_WARPS * 32;
constexpr int AT_TILE = 128;                  // keys per tile (16 per warp)
constexpr int ROW_BYTES = D * 2;              // one f16 row in shared memory

struct AttnSmem {
    uint8_t k[AT_TILE * ROW_BYTES];           // [key][512] f16, swizzled
    uint8_t q[HEADS * ROW_BYTES];             // [head][512] f16, swizzled
    uint8_t p[HEADS * AT_TILE * 2];           // [head][128] f16, swizzled
    float red[AT_WARPS][HEADS];
    float m[HEADS], l[HEADS], alpha[HEADS];
    uint32_t lut[256];                        // byte -> f16x2 (e2m1 lo, e2m1 hi)
    int32_t main_pos[TOPK];
    int32_t warp_cnt[AT_WARPS];
};

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    return static_cast<uint32_t>(row) * ROW_BYTES + (static_cast<uint32_t>(chunk ^ (row & 7)) << 4);
}

// f16 bits of an E2M1 code (sign, 2 exponent bits with bias 1, 1 mantissa bit).
__device__ __forceinline__ uint32_t e2m1_f16_bits(uint32_t c) {
    const uint32_t mag = c & 7u, e = mag >> 1, m = mag & 1u;
    uint32_t bits = (e == 0u) ? (m ? 0x3800u : 0u) : (((e + 14u) << 10) | (m << 9));
    return bits | ((c & 8u) << 12);
}

__global__ void __launch_bounds__(AT_THREADS, 1)
attend_kernel(AttnParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw);

    const int64_t r = blockIdx.x;                      // query row
    const int b = static_cast<int>(r / p.q_per_seq);
    const int qi = static_cast<int>(r % p.q_per_seq);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int g = lane >> 2;
    const int t = lane & 3;

    const int64_t seq_off = p.kv_offsets[b];
    const int64_t n_b = p.kv_offsets[b + 1] - seq_off;

    // ---- decode table, running statistics
    {
        const uint32_t v = static_cast<uint32_t>(tid);
        sm.lut[tid] = e2m1_f16_bits(v & 15u) | (e2m1_f16_bits(v >> 4) << 16);
    }
    if (tid < HEADS) {
        sm.m[tid] = -INFINITY;
        sm.l[tid] = 0.0f;
    }

    // ---- valid main positions, compacted in order (2 per thread)
    int n_main;
    {
        const int32_t* idx = p.topk_idx + r * TOPK;
        int32_t v0 = idx[2 * tid], v1 = idx[2 * tid + 1];
        const bool bad0 = v0 >= n_b, bad1 = v1 >= n_b;
        if ((bad0 || bad1) && p.err) atomicOr(p.err, ERR_DEVICE);
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
        n_main = 0;
        for (int w = 0; w < AT_WARPS; ++w) {
            const int c = sm.warp_cnt[w];
            if (w < warp) before += c;
            n_main += c;
        }
        if (ok0) sm.main_pos[before++] = v0;
        if (ok1) sm.main_pos[before] = v1;
    }

    // ---- visible SWA rows [swa_lo, swa_hi]
    int64_t swa_lo = 0, swa_hi = p.swa_rows - 1;
    if (p.q_pos != nullptr) {
        const int64_t q0 = p.q_pos[b];
        swa_lo = max(static_cast<int64_t>(qi), static_cast<int64_t>(WINDOW - 1) - q0);
        swa_hi = min(static_cast<int64_t>(qi) + WINDOW - 1, p.swa_rows - 1);
    }
    const int n_swa = static_cast<int>(max(static_cast<int64_t>(0), swa_hi - swa_lo + 1));
    const int n_keys = n_main + n_swa;
    const uint16_t* swa_base = p.swa_kv + (static_cast<int64_t>(b) * p.swa_rows + swa_lo) * D;

    // ---- query, bf16 -> f16
    for (int id = tid; id < HEADS * (D / 8); id += AT_THREADS) {
        const int h = id / (D / 8), c = id % (D / 8);
        const uint4 v = *reinterpret_cast<const uint4*>(p.q + (r * HEADS + h) * D + 8 * c);
        uint4 o;
        o.x = bf16x2_to_f16x2(v.x);
        o.y = bf16x2_to_f16x2(v.y);
        o.z = bf16x2_to_f16x2(v.z);
        o.w = bf16x2_to_f16x2(v.w);
        *reinterpret_cast<uint4*>(sm.q + swz(h, c)) = o;
    }
    __syncthreads();

    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;

    const int half = tid >> 4;          // 16 half-warps fill 8 rows each
    const int hl = tid & 15;
    const uint32_t k_base = smem_u32(sm.k);
    const uint32_t q_base = smem_u32(sm.q);
    const uint32_t p_base = smem_u32(sm.p);
    const int mi = lane >> 3, mj = lane & 7;

    for (int tile0 = 0; tile0 < n_keys; tile0 += AT_TILE) {
        // ---- gather + dequantise the tile
        for (int rr = 0; rr < AT_TILE / 16; ++rr) {
            const int kk = half * (AT_TILE / 16) + rr;
            const int gk = tile0 + kk;
            if (gk < n_main) {
                const int64_t grow = seq_off + sm.main_pos[gk];
                const uint8_t* crow = p.codes + grow * ROW_CODES;
                const uint8_t* srow = p.scales + grow * ROW_SCALES;
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const int c = hl + 16 * qq;        // f16 chunk = dims 8c .. 8c+7
                    const uint32_t cw = *reinterpret_cast<const uint32_t*>(crow + 4 * c);
                    const __half_raw sh = __nv_cvt_fp8_to_halfraw(
                        static_cast<__nv_fp8_storage_t>(srow[c >> 1]), __NV_E4M3);
                    const __half2 s2 = __half2half2(__half(sh));
                    uint32_t w[4];
#pragma unroll
                    for (int bi = 0; bi < 4; ++bi) {
                        uint32_t e = sm.lut[(cw >> (8 * bi)) & 0xFFu];
                        __half2 v = __hmul2(*reinterpret_cast<__half2*>(&e), s2);
                        w[bi] = *reinterpret_cast<uint32_t*>(&v);
                    }
                    *reinterpret_cast<uint4*>(sm.k + swz(kk, c)) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            } else if (gk < n_keys) {
                const uint16_t* row = swa_base + static_cast<int64_t>(gk - n_main) * D;
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const int c = hl + 16 * qq;
                    const uint4 v = *reinterpret_cast<const uint4*>(row + 8 * c);
                    uint4 ov;
                    ov.x = bf16x2_to_f16x2(v.x);
                    ov.y = bf16x2_to_f16x2(v.y);
                    ov.z = bf16x2_to_f16x2(v.z);
                    ov.w = bf16x2_to_f16x2(v.w);
                    *reinterpret_cast<uint4*>(sm.k + swz(kk, c)) = ov;
                }
            } else {
#pragma unroll
                for (int qq = 0; qq < 4; ++qq)
                    *reinterpret_cast<uint4*>(sm.k + swz(kk, hl + 16 * qq)) = make_uint4(0, 0, 0, 0);
            }
        }
        __syncthreads();

        // ---- S^T = K Q^T: warp owns keys 16w .. 16w+15, both head octets
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
            const int arow = warp * 16 + ((mi & 1) << 3) + mj;
            const int brow = ((mi >> 1) << 3) + mj;
#pragma unroll 4
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t a[4], bq[4];
                ldmatrix_x4(a, k_base + swz(arow, 2 * ks + (mi >> 1)));
                ldmatrix_x4(bq, q_base + swz(brow, 2 * ks + (mi & 1)));
                mma_16816(s[0], a, bq[0], bq[1]);
                mma_16816(s[1], a, bq[2], bq[3]);
            }
        }
        const bool va = tile0 + warp * 16 + g < n_keys;
        const bool vb = tile0 + warp * 16 + g + 8 < n_keys;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            s[nt][0] = va ? s[nt][0] * p.sm_scale : -INFINITY;
            s[nt][1] = va ? s[nt][1] * p.sm_scale : -INFINITY;
            s[nt][2] = vb ? s[nt][2] * p.sm_scale : -INFINITY;
            s[nt][3] = vb ? s[nt][3] * p.sm_scale : -INFINITY;
        }
        // ---- per-head tile max
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float m = fmaxf(s[nt][j], s[nt][j + 2]);
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
                if (g == 0) sm.red[warp][8 * nt + 2 * t + j] = m;
            }
        }
        __syncthreads();
        if (tid < HEADS) {
            float mt = -INFINITY;
            for (int w = 0; w < AT_WARPS; ++w) mt = fmaxf(mt, sm.red[w][tid]);
            const float m_old = sm.m[tid];
            const float m_new = fmaxf(m_old, mt);
            sm.alpha[tid] = (m_new == -INFINITY) ? 1.0f : __expf(m_old - m_new);
            sm.m[tid] = m_new;
        }
        __syncthreads();
        // ---- P = exp(S - m) -> f16 [head][key]; row sums
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int h = 8 * nt + 2 * t + j;
                const float mh = sm.m[h];
                const float pa = (s[nt][j] == -INFINITY) ? 0.0f : __expf(s[nt][j] - mh);
                const float pb = (s[nt][j + 2] == -INFINITY) ? 0.0f : __expf(s[nt][j + 2] - mh);
                const int ka = warp * 16 + g, kb = ka + 8;
                *reinterpret_cast<__half*>(sm.p + h * (AT_TILE * 2) +
                                           (((ka >> 3) ^ (h & 7)) << 4) + (ka & 7) * 2) = __float2half_rn(pa);
                *reinterpret_cast<__half*>(sm.p + h * (AT_TILE * 2) +
                                           (((kb >> 3) ^ (h & 7)) << 4) + (kb & 7) * 2) = __float2half_rn(pb);
                float sum = pa + pb;
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
                if (g == 0) sm.red[warp][h] = sum;
            }
        }
        __syncthreads();
        if (tid < HEADS) {
            float add = 0.0f;
            for (int w = 0; w < AT_WARPS; ++w) add += sm.red[w][tid];
            sm.l[tid] = sm.alpha[tid] * sm.l[tid] + add;
        }
        // ---- O = alpha * O + P V: warp owns dims 64w .. 64w+63
        {
            const float al = sm.alpha[g], ah = sm.alpha[g + 8];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                o[nt][0] *= al;
                o[nt][1] *= al;
                o[nt][2] *= ah;
                o[nt][3] *= ah;
            }
            const int prow = ((mi & 1) << 3) + mj;
#pragma unroll 2
            for (int ks = 0; ks < AT_TILE / 16; ++ks) {
                uint32_t a[4];
                ldmatrix_x4(a, p_base + static_cast<uint32_t>(prow) * (AT_TILE * 2) +
                                   (static_cast<uint32_t>((2 * ks + (mi >> 1)) ^ (prow & 7)) << 4));
                const int key = ks * 16 + ((mi & 1) << 3) + mj;
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) {
                    uint32_t bv[4];
                    ldmatrix_x4_trans(bv, k_base + swz(key, warp * 8 + 2 * pp + (mi >> 1)));
                    mma_16816(o[2 * pp], a, bv[0], bv[1]);
                    mma_16816(o[2 * pp + 1], a, bv[2], bv[3]);
                }
            }
        }
        __syncthreads();
    }

    // ---- normalise and store fp32
    const float inv_a = 1.0f / sm.l[g];
    const float inv_b = 1.0f / sm.l[g + 8];
    float* out_a = p.out + (r * HEADS + g) * D + warp * 64 + 2 * t;
    float* out_b = p.out + (r * HEADS + g + 8) * D + warp * 64 + 2 * t;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        *reinterpret_cast<float2*>(out_a + 8 * nt) = make_float2(o[nt][0] * inv_a, o[nt][1] * inv_a);
        *reinterpret_cast<float2*>(out_b + 8 * nt) = make_float2(o[nt][2] * inv_b, o[nt][3] * inv_b);
    }
}

}  // namespace

csa2_status launch_attend(const AttnParams& p, cudaStream_t stream) {
    const int64_t rows = static_cast<int64_t>(p.batch) * p.q_per_seq;
    if (rows == 0) return CSA2_OK;
    const int smem = static_cast<int>(sizeof(AttnSmem));
    if (!opt_in_smem(reinterpret_cast<const void*>(attend_kernel), smem))
        return check_launch("attend_kernel smem attribute");
    attend_kernel<<<static_cast<unsigned>(rows), AT_THREADS, smem, stream>>>(p);
    return check_launch("attend_kernel");
}

}  // namespace csa2
