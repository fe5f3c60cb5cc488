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
// takes tiles [sp*tpc, (sp+1)*tpc).  With few query rows (decode: one per sequence) the
// rows' tiles are spread over up to one wave of CTAs; CTAs write an unnormalised partial
// (running max m, sum l, O) and the last CTA of a row to finish (atomic ticket) merges
// them: out = sum_sp e^(m_sp - M) O_sp / sum_sp e^(m_sp - M) l_sp.  With many rows
// (prefill) one CTA runs all of a row's tiles and writes the output directly.
//
// Per tile: cp.async brings the selected FP4 rows (288 B each) into a staging area and
// the SWA rows (bf16) straight into the tile; FP4 rows are dequantised exactly to f16
// (hardware e2m1 -> f16 conversion, times the e4m3 scale: <= 6 significant bits in
// [2^-10, 2688]) and SWA rows converted bf16 -> f16 in place.  The tile's 16-byte chunks
// are XOR-swizzled by row (conflict-free ldmatrix).  S^T = K Q^T: warp w owns keys
// 16(w%4).. and dim half w/4 (halves summed in shared memory); the online softmax runs
// per warp on two heads with shuffles; O += P V: warp w owns output dims 64w .. 64w+63.
// Softmax statistics are fp32; P is rounded to f16; both MMAs accumulate in fp32.
#include <algorithm>

#include <cuda_fp4.h>

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
    float m[HEADS], l[HEADS], alpha[HEADS];
    float wsplit[MAX_SPLIT][HEADS];
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

// Two E2M1 codes (low nibble = first element) -> f16x2 bits (hardware cvt, exact).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    const __half2_raw h = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(byte), __NV_E2M1);
    return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4& v) {
    return make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z),
                      bf16x2_to_f16x2(v.w));
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

    const uint32_t k_base = smem_u32(sm.k);
    const uint32_t q_base = smem_u32(sm.q);
    const uint32_t p_base = smem_u32(sm.p);
    const int mi = lane >> 3, mj = lane & 7;
    const int kg = warp & 3, dh = warp >> 2;           // S: key group, dim half

    // ---- stage the query (bf16; converted in place with the first tile)
    if (key_begin < key_end) {
        for (int id = tid; id < HEADS * (D / 8); id += AT_THREADS)
            cp_async_16(q_base + swz(id >> 6, id & 63), p.q + (r * HEADS + (id >> 6)) * D + 8 * (id & 63));
    }

    constexpr int FP4_PIECES = (ROW_CODES + ROW_SCALES) / 16;   // 18 x 16 B per FP4 row
    const bool use_cache = p.cache_mode == CSA2_CACHE_USE;
    const bool fill_cache = p.cache_mode == CSA2_CACHE_FILL;
    for (int tile0 = key_begin; tile0 < key_end; tile0 += ATT_TILE) {
        const int tile_keys = min(ATT_TILE, key_end - tile0);
        const int main_rows = max(0, min(tile_keys, n_main - tile0));   // rows [0, main_rows)
        const int swa_first = main_rows;                                // rows [main_rows, tile_keys)
        // ---- gather: FP4 rows -> staging, SWA rows (bf16) -> the tile, all in flight
        if (use_cache) {                                   // rows dequantised by an earlier layer
            const uint16_t* crow = p.sel_cache + (r * TOPK + tile0) * D;
            for (int id = tid; id < main_rows * (D / 8); id += AT_THREADS) {
                const int kk = id >> 6, c = id & 63;
                cp_async_16(k_base + swz(kk, c), crow + static_cast<int64_t>(kk) * D + 8 * c);
            }
        } else {
            for (int id = tid; id < main_rows * FP4_PIECES; id += AT_THREADS) {
                const int kk = id / FP4_PIECES, c = id - kk * FP4_PIECES;
                const int64_t grow = seq_off + sm.main_pos[tile0 + kk];
                const uint8_t* src = c < ROW_CODES / 16 ? p.codes + grow * ROW_CODES + 16 * c
                                                        : p.scales + grow * ROW_SCALES + 16 * (c - ROW_CODES / 16);
                cp_async_16(smem_u32(&sm.fp4[kk][16 * c]), src);
            }
        }
        {
            const uint16_t* swa0 = swa_base + static_cast<int64_t>(tile0 + swa_first - n_main) * D;
            for (int id = tid; id < (tile_keys - swa_first) * (D / 8); id += AT_THREADS) {
                const int kk = swa_first + (id >> 6), c = id & 63;
                cp_async_16(k_base + swz(kk, c), swa0 + static_cast<int64_t>(id >> 6) * D + 8 * c);
            }
        }
        for (int id = tid; id < (ATT_TILE - tile_keys) * (D / 8); id += AT_THREADS) {
            const int kk = tile_keys + (id >> 6);
            *reinterpret_cast<uint4*>(sm.k + swz(kk, id & 63)) = make_uint4(0, 0, 0, 0);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        if (tile0 == key_begin) {                          // query: bf16 -> f16 in place
            for (int id = tid; id < HEADS * (D / 8); id += AT_THREADS) {
                uint4* qp = reinterpret_cast<uint4*>(sm.q + swz(id >> 6, id & 63));
                *qp = bf16x8_to_f16x8(*qp);
            }
        }
        // ---- FP4 rows -> f16 (e2m1 x e4m3, exact), one 16-channel scale group at a time;
        //      SWA rows bf16 -> f16 in place
        for (int id = tid; id < (use_cache ? 0 : main_rows * (D / GROUP)); id += AT_THREADS) {
            const int kk = id >> 5, grp = id & 31;         // dims 16grp .. 16grp+15
            const uint2 cw = *reinterpret_cast<const uint2*>(&sm.fp4[kk][8 * grp]);
            const __half_raw sh = __nv_cvt_fp8_to_halfraw(
                static_cast<__nv_fp8_storage_t>(sm.fp4[kk][ROW_CODES + grp]), __NV_E4M3);
            const __half2 s2 = __half2half2(__half(sh));
            uint32_t w[8];
#pragma unroll
            for (int bi = 0; bi < 8; ++bi) {
                uint32_t e = e2m1x2_to_f16x2(((bi < 4 ? cw.x : cw.y) >> (8 * (bi & 3))) & 0xFFu);
                __half2 v = __hmul2(*reinterpret_cast<__half2*>(&e), s2);
                w[bi] = *reinterpret_cast<uint32_t*>(&v);
            }
            *reinterpret_cast<uint4*>(sm.k + swz(kk, 2 * grp)) = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4*>(sm.k + swz(kk, 2 * grp + 1)) = make_uint4(w[4], w[5], w[6], w[7]);
        }
        for (int id = tid; id < (tile_keys - swa_first) * (D / 8); id += AT_THREADS) {
            uint4* kp = reinterpret_cast<uint4*>(sm.k + swz(swa_first + (id >> 6), id & 63));
            *kp = bf16x8_to_f16x8(*kp);
        }
        __syncthreads();
        if (fill_cache) {                                  // keep the dequantised rows for Reuse
            uint16_t* crow = p.sel_cache + (r * TOPK + tile0) * D;
            for (int id = tid; id < main_rows * (D / 8); id += AT_THREADS) {
                const int kk = id >> 6, c = id & 63;
                *reinterpret_cast<uint4*>(crow + static_cast<int64_t>(kk) * D + 8 * c) =
                    *reinterpret_cast<const uint4*>(sm.k + swz(kk, c));
            }
        }

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

        // ---- online softmax: warp w owns heads 2w, 2w+1; lane owns keys lane, lane+32
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int h = 2 * warp + hh;
            float sv[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int key = lane + 32 * j;
                sv[j] = key < tile_keys ? (sm.s2[0][key][h] + sm.s2[1][key][h]) * p.sm_scale : -INFINITY;
            }
            float mt = fmaxf(sv[0], sv[1]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, off));
            const float m_old = sm.m[h];
            const float m_new = fmaxf(m_old, mt);
            const float alpha = (m_new == -INFINITY) ? 1.0f : __expf(m_old - m_new);
            float sum = 0.0f;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int key = lane + 32 * j;
                const float pv = (sv[j] == -INFINITY) ? 0.0f : __expf(sv[j] - m_new);
                sum += pv;
                *reinterpret_cast<__half*>(sm.p + pswz(h, key >> 3) + (key & 7) * 2) = __float2half_rn(pv);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
            __syncwarp();
            if (lane == 0) {
                sm.m[h] = m_new;
                sm.alpha[h] = alpha;
                sm.l[h] = alpha * sm.l[h] + sum;
            }
        }
        __syncthreads();

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
    const int64_t resident = 2 * 148;          // two CTAs per SM: keep the grid to one wave
    int want = static_cast<int>(std::min<int64_t>(n_tiles, std::max<int64_t>(1, resident / rows)));
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
