// Sparse attention over the selected FP4 main-KV rows joined with the sliding window.
//
// CSA2 section of the thecryptopost.io DeepSeek-V4.1-Flash article: every layer keeps
// its own main Q and SWA KV and attends over its Top-512 selection of the shared main
// KV; the Causal Encoder-Decoder section fixes the 128-token window; tldrocket.com: one
// 512-dim latent serves as both key and value.  Per query and head h:
//     out_h = softmax_j(sm_scale * q_h . row_j) . rows,   rows = selected FP4 rows
//                                                         (dequantised) ++ SWA rows.
//
// Work split: a query's key list (<= 512 + 128) is cut into 64-key tiles; CTA (row, sp)
// takes tiles [sp*tpc, (sp+1)*tpc).  With few query rows (decode: one per sequence) each
// CTA takes one tile so that every SM has work; CTAs write an unnormalised partial
// (running max m, sum l, O) and the last CTA of a row to finish (atomic ticket) merges
// them: out = sum_sp e^(m_sp - M) O_sp / sum_sp e^(m_sp - M) l_sp.  With many rows
// (prefill) one CTA runs all of a row's tiles and writes the output directly.
//
// Per tile: the FP4 rows are gathered and dequantised exactly to f16 (e2m1 x e4m3 has
// <= 6 significant bits in [2^-10, 2688]) and the SWA rows converted bf16 -> f16 into a
// shared tile whose 16-byte chunks are XOR-swizzled by row (conflict-free ldmatrix).
// S^T = K Q^T: warp w owns keys 16(w%4).. and dim half w/4 (the halves are summed in
// shared memory); O += P V: warp w owns output dims 64w .. 64w+63.  Softmax statistics
// are fp32; P is rounded to f16 for the second MMA; both MMAs accumulate in fp32.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

namespace {

constexpr int AT_WARPS = 8;
constexpr int AT_THREADS = AT_WARPS * 32;
constexpr int ROW_BYTES = D * 2;                  // one f16 row in shared memory
constexpr int P_ROW = ATT_TILE * 2;               // one head's P row (bytes)
constexpr int MAX_SPLIT = 16;

struct AttnSmem {
    uint8_t k[ATT_TILE * ROW_BYTES];              // [key][512] f16, swizzled
    uint8_t q[HEADS * ROW_BYTES];                 // [head][512] f16, swizzled
    uint8_t p[HEADS * P_ROW];                     // [head][64] f16, swizzled
    union {                                       // the staging is dead once dequantised
        uint8_t fp4[ATT_TILE][ROW_CODES + ROW_SCALES];  // staged FP4 rows (codes | scales)
        float s2[2][ATT_TILE][HEADS + 1];         // S partials of the two dim halves
    };
    float red[AT_WARPS][HEADS];
    float m[HEADS], l[HEADS], alpha[HEADS];
    float wsplit[MAX_SPLIT][HEADS];
    uint32_t lut[256];                            // byte -> f16x2 (e2m1 lo, e2m1 hi)
    int32_t main_pos[TOPK];
    int32_t warp_cnt[AT_WARPS];
    int last;
};

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    return static_cast<uint32_t>(row) * ROW_BYTES + (static_cast<uint32_t>(chunk ^ (row & 7)) << 4);
}

__device__ __forceinline__ uint32_t pswz(int row, int chunk) {
    return static_cast<uint32_t>(row) * P_ROW + (static_cast<uint32_t>(chunk ^ (row & 7)) << 4);
}

// f16 bits of an E2M1 code (sign, 2 exponent bits with bias 1, 1 mantissa bit).
__device__ __forceinline__ uint32_t e2m1_f16_bits(uint32_t c) {
    const uint32_t mag = c & 7u, e = mag >> 1, m = mag & 1u;
    uint32_t bits = (e == 0u) ? (m ? 0x3800u : 0u) : (((e + 14u) << 10) | (m << 9));
    return bits | ((c & 8u) << 12);
}

__global__ void __launch_bounds__(AT_THREADS, 2)
attend_kernel(AttnParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw);

    const int64_t r = blockIdx.x;                      // query row
    const int sp = blockIdx.y;                         // key split
    const int b = static_cast<int>(r / p.q_per_seq);
    const int qi = static_cast<int>(r % p.q_per_seq);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int g = lane >> 2;
    const int t = lane & 3;

    const int64_t seq_off = p.kv_offsets[b];
    const int64_t n_b = p.kv_offsets[b + 1] - seq_off;

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
        n_main = 0;
        for (int w = 0; w < AT_WARPS; ++w) {
            const int c = sm.warp_cnt[w];
            if (w < warp) before += c;
            n_main += c;
        }
        if (ok0) sm.main_pos[before++] = v0;
        if (ok1) sm.main_pos[before] = v1;
    }
    __syncthreads();                                   // main_pos is read by every thread

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
    const int key_begin = sp * p.tiles_per_cta * ATT_TILE;
    const int key_end = min(n_keys, key_begin + p.tiles_per_cta * ATT_TILE);

    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;

    const int half = tid >> 4;                         // 16 half-warps x 4 rows
    const int hl = tid & 15;
    const uint32_t k_base = smem_u32(sm.k);
    const uint32_t q_base = smem_u32(sm.q);
    const uint32_t p_base = smem_u32(sm.p);
    const int mi = lane >> 3, mj = lane & 7;
    const int kg = warp & 3, dh = warp >> 2;           // S: key group, dim half

    // ---- stage the query (bf16, converted in place later) with the first tile's rows
    if (key_begin < key_end) {
        for (int id = tid; id < HEADS * (D / 8); id += AT_THREADS) {
            const int h = id / (D / 8), c = id % (D / 8);
            cp_async_16(q_base + swz(h, c), p.q + (r * HEADS + h) * D + 8 * c);
        }
    }

    for (int tile0 = key_begin; tile0 < key_end; tile0 += ATT_TILE) {
        // ---- gather: FP4 rows -> staging, SWA rows (bf16) -> the tile, all in flight
        for (int id = tid; id < ATT_TILE * (D / 8); id += AT_THREADS) {
            const int kk = id / (D / 8), c = id % (D / 8);
            const int gk = tile0 + kk;
            if (gk < n_main) {
                if (c < (ROW_CODES + ROW_SCALES) / 16) {
                    const int64_t grow = seq_off + sm.main_pos[gk];
                    const uint8_t* src = c < ROW_CODES / 16 ? p.codes + grow * ROW_CODES + 16 * c
                                                            : p.scales + grow * ROW_SCALES + 16 * (c - ROW_CODES / 16);
                    cp_async_16(smem_u32(&sm.fp4[kk][16 * c]), src);
                }
            } else if (gk < key_end) {
                cp_async_16(k_base + swz(kk, c), swa_base + static_cast<int64_t>(gk - n_main) * D + 8 * c);
            } else {
                *reinterpret_cast<uint4*>(sm.k + swz(kk, c)) = make_uint4(0, 0, 0, 0);
            }
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        if (tile0 == key_begin) {                          // query: bf16 -> f16 in place
            for (int id = tid; id < HEADS * (D / 8); id += AT_THREADS) {
                const int h = id / (D / 8), c = id % (D / 8);
                uint4* qp = reinterpret_cast<uint4*>(sm.q + swz(h, c));
                const uint4 v = *qp;
                *qp = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z),
                                 bf16x2_to_f16x2(v.w));
            }
        }
        // ---- dequantise FP4 rows into the tile; SWA rows bf16 -> f16 in place
#pragma unroll
        for (int rr = 0; rr < ATT_TILE / 16; ++rr) {
            const int kk = half * (ATT_TILE / 16) + rr;
            const int gk = tile0 + kk;
            if (gk < n_main) {
                const uint8_t* crow = sm.fp4[kk];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const int c = hl + 16 * qq;        // f16 chunk = dims 8c .. 8c+7
                    const uint32_t cw = *reinterpret_cast<const uint32_t*>(crow + 4 * c);
                    const __half_raw sh = __nv_cvt_fp8_to_halfraw(
                        static_cast<__nv_fp8_storage_t>(crow[ROW_CODES + (c >> 1)]), __NV_E4M3);
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
            } else if (gk < key_end) {
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    uint4* kp = reinterpret_cast<uint4*>(sm.k + swz(kk, hl + 16 * qq));
                    const uint4 v = *kp;
                    *kp = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z),
                                     bf16x2_to_f16x2(v.w));
                }
            }
        }
        __syncthreads();

        // ---- S^T partial = K Q^T over this warp's dim half
        {
            float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            const int arow = kg * 16 + ((mi & 1) << 3) + mj;
            const int brow = ((mi >> 1) << 3) + mj;
#pragma unroll 4
            for (int ks = dh * 16; ks < dh * 16 + 16; ++ks) {
                uint32_t a[4], bq[4];
                ldmatrix_x4(a, k_base + swz(arow, 2 * ks + (mi >> 1)));
                ldmatrix_x4(bq, q_base + swz(brow, 2 * ks + (mi & 1)));
                mma_16816(s[0], a, bq[0], bq[1]);
                mma_16816(s[1], a, bq[2], bq[3]);
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
        __syncthreads();

        // ---- softmax: thread owns head h, keys 4kq .. 4kq+3
        const int h = tid & 15, kq = tid >> 4;
        float sv[4];
        float mloc = -INFINITY;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int key = 4 * kq + j;
            const bool ok = tile0 + key < key_end;
            sv[j] = ok ? (sm.s2[0][key][h] + sm.s2[1][key][h]) * p.sm_scale : -INFINITY;
            mloc = fmaxf(mloc, sv[j]);
        }
        mloc = fmaxf(mloc, __shfl_xor_sync(0xFFFFFFFFu, mloc, 16));
        if (lane < 16) sm.red[warp][h] = mloc;
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
        {
            const float mh = sm.m[h];
            float pv[4], sum = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                pv[j] = (sv[j] == -INFINITY) ? 0.0f : __expf(sv[j] - mh);
                sum += pv[j];
            }
            const __half2 p01 = __floats2half2_rn(pv[0], pv[1]);
            const __half2 p23 = __floats2half2_rn(pv[2], pv[3]);
            uint2 pk;
            pk.x = *reinterpret_cast<const uint32_t*>(&p01);
            pk.y = *reinterpret_cast<const uint32_t*>(&p23);
            *reinterpret_cast<uint2*>(sm.p + pswz(h, kq >> 1) + (kq & 1) * 8) = pk;
            sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 16);
            if (lane < 16) sm.red[warp][h] = sum;
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
#pragma unroll
            for (int ks = 0; ks < ATT_TILE / 16; ++ks) {
                uint32_t a[4];
                ldmatrix_x4(a, p_base + pswz(prow, 2 * ks + (mi >> 1)));
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

    if (p.n_split == 1) {
        const float inv_a = 1.0f / sm.l[g];
        const float inv_b = 1.0f / sm.l[g + 8];
        float* out_a = p.out + (r * HEADS + g) * D + warp * 64 + 2 * t;
        float* out_b = p.out + (r * HEADS + g + 8) * D + warp * 64 + 2 * t;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            *reinterpret_cast<float2*>(out_a + 8 * nt) = make_float2(o[nt][0] * inv_a, o[nt][1] * inv_a);
            *reinterpret_cast<float2*>(out_b + 8 * nt) = make_float2(o[nt][2] * inv_b, o[nt][3] * inv_b);
        }
        return;
    }

    // ---- partial: unnormalised O with this split's running max and sum
    const int64_t slot = r * p.n_split + sp;
    {
        float* po_a = p.part_o + (slot * HEADS + g) * D + warp * 64 + 2 * t;
        float* po_b = p.part_o + (slot * HEADS + g + 8) * D + warp * 64 + 2 * t;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            __stcg(reinterpret_cast<float2*>(po_a + 8 * nt), make_float2(o[nt][0], o[nt][1]));
            __stcg(reinterpret_cast<float2*>(po_b + 8 * nt), make_float2(o[nt][2], o[nt][3]));
        }
        if (tid < HEADS) {
            __stcg(p.part_ml + slot * 2 * HEADS + tid, sm.m[tid]);
            __stcg(p.part_ml + slot * 2 * HEADS + HEADS + tid, sm.l[tid]);
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned prev = atomicAdd(p.counters + r, 1u);
        sm.last = (prev == static_cast<unsigned>(p.n_split - 1));
    }
    __syncthreads();
    if (!sm.last) return;
    __threadfence();

    // ---- last CTA of the row: merge the n_split partials
    if (tid < HEADS) {
        float M = -INFINITY;
        for (int s = 0; s < p.n_split; ++s)
            M = fmaxf(M, __ldcg(p.part_ml + (r * p.n_split + s) * 2 * HEADS + tid));
        float L = 0.0f;
        for (int s = 0; s < p.n_split; ++s) {
            const float ms = __ldcg(p.part_ml + (r * p.n_split + s) * 2 * HEADS + tid);
            const float ls = __ldcg(p.part_ml + (r * p.n_split + s) * 2 * HEADS + HEADS + tid);
            const float wgt = (ms == -INFINITY) ? 0.0f : __expf(ms - M);
            sm.wsplit[s][tid] = wgt;
            L += wgt * ls;
        }
        sm.l[tid] = 1.0f / L;
    }
    __syncthreads();
    for (int e = tid * 4; e < HEADS * D; e += AT_THREADS * 4) {
        const int h = e / D;
        float4 v[MAX_SPLIT];
#pragma unroll
        for (int s = 0; s < MAX_SPLIT; ++s)                // all loads in flight at once
            if (s < p.n_split)
                v[s] = __ldcg(reinterpret_cast<const float4*>(p.part_o + (r * p.n_split + s) * HEADS * D + e));
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int s = 0; s < MAX_SPLIT; ++s) {
            if (s < p.n_split) {
                const float wgt = sm.wsplit[s][h];
                acc.x += wgt * v[s].x;
                acc.y += wgt * v[s].y;
                acc.z += wgt * v[s].z;
                acc.w += wgt * v[s].w;
            }
        }
        const float inv = sm.l[h];
        *reinterpret_cast<float4*>(p.out + r * HEADS * D + e) =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
    if (tid == 0) p.counters[r] = 0u;                  // ready for the next call
}

}  // namespace

void attend_split(int64_t rows, int64_t max_keys, int& n_split, int& tiles_per_cta) {
    const int n_tiles = static_cast<int>(ceil_div(max_keys, ATT_TILE));
    const int64_t target_ctas = 4 * 148;       // ~2 waves of 2 resident CTAs per SM
    int want = static_cast<int>(std::min<int64_t>(
        n_tiles, std::max<int64_t>(1, ceil_div(target_ctas, rows))));
    want = std::min(want, MAX_SPLIT);
    tiles_per_cta = static_cast<int>(ceil_div(n_tiles, want));
    n_split = static_cast<int>(ceil_div(n_tiles, tiles_per_cta));
}

static_assert(sizeof(AttnSmem) <= 112 * 1024, "two attention CTAs must fit on one SM");

csa2_status launch_attend(const AttnParams& p, cudaStream_t stream) {
    const int64_t rows = static_cast<int64_t>(p.batch) * p.q_per_seq;
    if (rows == 0) return CSA2_OK;
    const int smem = static_cast<int>(sizeof(AttnSmem));
    if (!opt_in_smem(reinterpret_cast<const void*>(attend_kernel), smem))
        return check_launch("attend_kernel smem attribute");
    dim3 grid(static_cast<unsigned>(rows), static_cast<unsigned>(p.n_split));
    attend_kernel<<<grid, AT_THREADS, smem, stream>>>(p);
    return check_launch("attend_kernel");
}

}  // namespace csa2
