// C-ABI entry points of libcsa2: host-side validation, workspace layout and the
// Full / Reindex / Reuse dispatch of a CSA2 layer (CSA2 section of the thecryptopost.io
// DeepSeek-V4.1-Flash article).  Every check runs before anything is enqueued.
#include <cuda.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

namespace {
thread_local char g_last_error[256] = "";

constexpr size_t WS_HEADER = 256;          // device error word + padding

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct WsLayout {
    bool fused = false;                    // decode indexer: scan + chunk Top-K + merge
    bool prefill_fused = false;            // many-query Full indexer with a streaming Top-K
    size_t scores = 0;                     // materialised scores [rows][scores_ld]
    int64_t scores_ld = 0;
    size_t cand_s = 0, cand_p = 0;         // fused: [B][n_chunks][512] candidates
    size_t chunk_thr = 0;                  // fused: [B][n_chunks] chunk 512th scores
    int n_chunks = 0, chunk = 0;
    size_t blockmax = 0;                   // [B][bm_ld] block maxima (FULL + want_pool)
    int64_t bm_ld = 0;
    int n_split = 1;                       // attention CTAs (one cluster) per query row
    size_t total = WS_HEADER;
};

WsLayout layer_layout(const csa2_layer_args* a) {
    WsLayout L;
    size_t off = WS_HEADER;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += align_up(bytes, 256);
        return at;
    };
    const int64_t rows = static_cast<int64_t>(a->batch) * a->q_per_seq;
    if (a->mode != CSA2_MODE_REUSE) {
        L.fused = (a->q_per_seq == 1 && a->q_pos == nullptr);
        L.prefill_fused = !L.fused && a->mode == CSA2_MODE_FULL;
        const int64_t ncols = (a->mode == CSA2_MODE_REINDEX) ? POOL_POSITIONS : a->max_n;
        if (L.prefill_fused) {
            // no scratch: scores and candidates stay in shared memory
        } else if (L.fused) {
            L.chunk = (a->mode == CSA2_MODE_REINDEX) ? REINDEX_CHUNK : SCAN_CHUNK;
            L.n_chunks = static_cast<int>(ceil_div(ncols, L.chunk));
            const size_t n = static_cast<size_t>(a->batch) * L.n_chunks * TOPK;
            L.cand_s = take(n * sizeof(float));
            L.cand_p = take(n * sizeof(int32_t));
            L.chunk_thr = take(static_cast<size_t>(a->batch) * L.n_chunks * sizeof(float));
        } else {
            L.scores_ld = padded_ld(ncols);
            L.scores = take(static_cast<size_t>(rows * L.scores_ld) * sizeof(float));
        }
        if (a->mode == CSA2_MODE_FULL && a->want_pool) {
            L.bm_ld = padded_ld(ceil_div(a->max_n, POOL_BLOCK));
            L.blockmax = take(static_cast<size_t>(a->batch * L.bm_ld) * sizeof(float));
        }
    }
    // every attention runs on the single-row kernel (decode rows and prefill rows alike);
    // a row's CTAs merge their partials in their cluster, so it needs no scratch
    const bool swa8 = a->swa_format == CSA2_SWA_FP8;
    L.n_split = attend_rows_split(rows, attend_rows_swa_tiles(a->swa_rows, a->q_pos != nullptr, swa8), swa8);
    L.total = off;
    return L;
}

// A second stream per device, for work of one call that may run beside the caller's
// stream (created on first use, outside stream capture; never destroyed).
cudaStream_t side_stream(cudaStream_t caller) {
    static std::mutex mu;
    static cudaStream_t streams[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!streams[dev]) {
        cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(caller, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) return nullptr;
        if (cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess) streams[dev] = nullptr;
    }
    return streams[dev];
}

// Fork / join of the side stream with events (inside a stream capture these become graph
// edges).  begin() returns the stream to use: the side stream, or the caller's own stream
// when no side stream is available (then join() has nothing to do).
struct SideFork {
    cudaEvent_t e_fork = nullptr, e_join = nullptr;
    cudaStream_t side = nullptr;
    cudaStream_t begin(cudaStream_t s) {
        cudaStream_t st = side_stream(s);
        if (!st || cudaEventCreateWithFlags(&e_fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&e_join, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventRecord(e_fork, s) != cudaSuccess || cudaStreamWaitEvent(st, e_fork, 0) != cudaSuccess) {
            (void)cudaGetLastError();
            return s;
        }
        side = st;
        return st;
    }
    // Instead of joining: records ev where the side work ends (the side stream, or s when
    // the work ran on s); whoever reads its outputs waits for ev.
    csa2_status defer(cudaStream_t s, cudaEvent_t ev) {
        const cudaError_t ce = cudaEventRecord(ev, side ? side : s);
        side = nullptr;
        return ce == cudaSuccess ? CSA2_OK : fail_cuda("csa2_attend ev_pool record", ce);
    }
    csa2_status join(cudaStream_t s) {
        cudaError_t ce = cudaSuccess;
        if (side) {
            ce = cudaEventRecord(e_join, side);
            if (ce == cudaSuccess) ce = cudaStreamWaitEvent(s, e_join, 0);
            side = nullptr;
        }
        return ce == cudaSuccess ? CSA2_OK : fail_cuda("csa2_attend side-stream join", ce);
    }
    ~SideFork() {
        if (e_fork) cudaEventDestroy(e_fork);
        if (e_join) cudaEventDestroy(e_join);
    }
};

csa2_status validate_index(const csa2_index_args* a) {
    if (!a) return CSA2_ERR_INVALID_ARG;
    if (a->batch < 1 || a->q_per_seq < 1 || a->q_per_seq > 65536) return CSA2_ERR_INVALID_ARG;
    if (a->ratio != 1 && a->ratio != 2) return CSA2_ERR_INVALID_ARG;
    if (a->reserved0 != 0 || a->max_n < 1) return CSA2_ERR_INVALID_ARG;
    if (!a->kv_offsets || !a->idx_q || !a->idx_w || !a->idx_k || !a->idx_kscale)
        return CSA2_ERR_INVALID_ARG;
    if (!aligned(a->idx_q, 16) || !aligned(a->idx_k, 16)) return CSA2_ERR_INVALID_ARG;
    return CSA2_OK;
}

IndexParams to_params(const csa2_index_args* a) {
    IndexParams p;
    p.batch = a->batch;
    p.q_per_seq = a->q_per_seq;
    p.ratio = a->ratio;
    p.max_n = a->max_n;
    p.kv_offsets = a->kv_offsets;
    p.q_pos = a->q_pos;
    p.idx_q = a->idx_q;
    p.idx_w = a->idx_w;
    p.idx_k = a->idx_k;
    p.idx_kscale = a->idx_kscale;
    p.pool_blocks = a->pool_blocks;
    p.rows = RowMap{nullptr, 0, 0};                      // the stage API reads packed rows
    return p;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<EncodeTiledFn>(f);
    }();
    return fn;
}

// TMA map over bf16 rows of 512: rank 2 = [rows][512] (boxes of box_rows x 64), rank 3 =
// [seqs][rows][512] (boxes of 1 x box_rows x 64); 128-byte swizzle.  The kernel's TMA
// instruction must have the same rank.
bool make_bf16_rows_map(const uint16_t* base, int64_t rows, int64_t seqs, int box_rows, int rank,
                        CUtensorMap* map) {
    const EncodeTiledFn enc = encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                                static_cast<cuuint64_t>(seqs)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(rows * D) * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (rank != 2 && rank != 3) return false;
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank), const_cast<uint16_t*>(base), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// TMA map over indexer K viewed as [rows][64] bytes, 64-byte swizzle, boxes of box_rows.
bool make_idx_k_map(const uint8_t* idx_k, int64_t rows, int box_rows, CUtensorMap* map) {
    const EncodeTiledFn enc = encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(IDX_DIM), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(IDX_DIM)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(IDX_DIM), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(idx_k), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool opt_in_smem(const void* kernel, int bytes) {
    constexpr int kMaxDev = 64, kMaxKernels = 16;
    static const void* kernels[kMaxKernels] = {};
    static bool done[kMaxKernels][kMaxDev] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return false;
    std::lock_guard<std::mutex> lock(mu);
    int slot = 0;
    while (slot < kMaxKernels && kernels[slot] != nullptr && kernels[slot] != kernel) ++slot;
    if (slot == kMaxKernels) return false;
    kernels[slot] = kernel;
    if (done[slot][dev]) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return false;
    done[slot][dev] = true;
    return true;
}

std::atomic<uint64_t> g_launches{0};

csa2_status fail_cuda(const char* what, cudaError_t e) {
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, cudaGetErrorString(e));
    cudaGetLastError();                       // clear a non-sticky error
    return CSA2_ERR_CUDA;
}

csa2_status check_launch(const char* what) {
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) {
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return CSA2_OK;
    }
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, cudaGetErrorString(e));
    return CSA2_ERR_CUDA;
}

}  // namespace csa2

using namespace csa2;

extern "C" {

const char* csa2_status_string(csa2_status s) {
    switch (s) {
        case CSA2_OK: return "CSA2_OK";
        case CSA2_ERR_INVALID_ARG: return "CSA2_ERR_INVALID_ARG";
        case CSA2_ERR_UNSUPPORTED: return "CSA2_ERR_UNSUPPORTED";
        case CSA2_ERR_WORKSPACE: return "CSA2_ERR_WORKSPACE";
        case CSA2_ERR_CUDA: return "CSA2_ERR_CUDA";
        case CSA2_ERR_TIMEOUT: return "CSA2_ERR_TIMEOUT";
        case CSA2_ERR_DEVICE: return "CSA2_ERR_DEVICE";
        default: return "CSA2_ERR_UNKNOWN";
    }
}

const char* csa2_last_error(void) { return g_last_error; }

int32_t csa2_abi_version(void) { return CSA2_ABI_VERSION; }

uint64_t csa2_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

csa2_status csa2_quantize_kv(const uint16_t* x, int64_t n_in, int32_t ratio, const int64_t* dst_row,
                             uint8_t* codes, uint8_t* scales, void* stream) {
    if (ratio != 1 && ratio != 2) return CSA2_ERR_INVALID_ARG;
    if (n_in < 0 || n_in % ratio != 0) return CSA2_ERR_INVALID_ARG;
    if (n_in == 0) return CSA2_OK;
    if (!x || !codes || !scales) return CSA2_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(codes, 8)) return CSA2_ERR_INVALID_ARG;
    if (n_in / ratio > (int64_t(1) << 36)) return CSA2_ERR_UNSUPPORTED;
    return launch_quantize(x, n_in, ratio, dst_row, codes, scales, static_cast<cudaStream_t>(stream));
}

csa2_status csa2_append_kv(const uint16_t* latent, const float* idx_proj, int64_t n, const int64_t* dst_row,
                           uint8_t* codes, uint8_t* scales, uint8_t* idx_k, float* idx_kscale, void* stream) {
    if (n < 0) return CSA2_ERR_INVALID_ARG;
    if (n == 0) return CSA2_OK;
    if (!latent || !idx_proj || !dst_row || !codes || !scales || !idx_k || !idx_kscale)
        return CSA2_ERR_INVALID_ARG;
    if (!aligned(latent, 16) || !aligned(idx_proj, 8) || !aligned(codes, 8) || !aligned(idx_k, 2) ||
        !aligned(idx_kscale, 4) || !aligned(dst_row, 8))
        return CSA2_ERR_INVALID_ARG;
    if (n > (int64_t(1) << 36)) return CSA2_ERR_UNSUPPORTED;
    return launch_append(latent, idx_proj, n, dst_row, codes, scales, idx_k, idx_kscale,
                         static_cast<cudaStream_t>(stream));
}

csa2_status csa2_index_score(const csa2_index_args* a, float* scores, int64_t ld, void* stream) {
    const csa2_status st = validate_index(a);
    if (st != CSA2_OK) return st;
    if (!scores) return CSA2_ERR_INVALID_ARG;
    const int64_t ncols = a->pool_blocks ? POOL_POSITIONS : a->max_n;
    if (ld < ncols) return CSA2_ERR_INVALID_ARG;
    return launch_index_score(to_params(a), scores, ld, nullptr, 0, static_cast<cudaStream_t>(stream));
}

csa2_status csa2_topk(const float* scores, int64_t ld, int64_t n_cols, int32_t rows, int32_t k,
                      const int32_t* pool_blocks, int32_t q_per_seq, int32_t* idx_out, void* stream) {
    if (rows < 0 || k < 1 || k > 4096 || q_per_seq < 1) return CSA2_ERR_INVALID_ARG;
    if (n_cols < 0 || n_cols > ld) return CSA2_ERR_INVALID_ARG;
    if (pool_blocks && n_cols > POOL_POSITIONS) return CSA2_ERR_INVALID_ARG;
    if (rows == 0) return CSA2_OK;
    if (!scores || !idx_out) return CSA2_ERR_INVALID_ARG;
    if (n_cols > (int64_t(1) << 31) - 1) return CSA2_ERR_UNSUPPORTED;
    return launch_topk_rows(scores, ld, n_cols, rows, k, pool_blocks, q_per_seq, idx_out,
                            static_cast<cudaStream_t>(stream));
}

size_t csa2_pool_workspace_size(int32_t batch, int64_t max_n) {
    if (batch < 1 || max_n < 1) return 0;
    const int64_t bm_ld = padded_ld(ceil_div(max_n, POOL_BLOCK));
    return WS_HEADER + align_up(static_cast<size_t>(batch * bm_ld) * sizeof(float), 256);
}

csa2_status csa2_build_pool(const float* scores, int64_t ld, const int64_t* kv_offsets, int32_t batch,
                            int64_t max_n, int32_t* pool_blocks, void* workspace,
                            size_t workspace_bytes, void* stream) {
    if (batch < 1 || max_n < 1 || ld < max_n) return CSA2_ERR_INVALID_ARG;
    if (!scores || !kv_offsets || !pool_blocks) return CSA2_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256) ||
        workspace_bytes < csa2_pool_workspace_size(batch, max_n))
        return CSA2_ERR_WORKSPACE;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t bm_ld = padded_ld(ceil_div(max_n, POOL_BLOCK));
    float* bm = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + WS_HEADER);
    csa2_status st = launch_block_max(scores, ld, kv_offsets, batch, max_n, bm, bm_ld, s);
    if (st != CSA2_OK) return st;
    return launch_topk_rows(bm, bm_ld, ceil_div(max_n, POOL_BLOCK), batch, POOL_BLOCKS, nullptr, 1,
                            pool_blocks, s, kv_offsets);
}

size_t csa2_workspace_size(const csa2_layer_args* a) {
    if (!a) return 0;
    if (a->batch < 1 || a->q_per_seq < 1 || a->max_n < 1) return WS_HEADER;
    return layer_layout(a).total;
}

csa2_status csa2_attend(const csa2_layer_args* a, void* stream) {
    if (!a) return CSA2_ERR_INVALID_ARG;
    if (a->mode != CSA2_MODE_FULL && a->mode != CSA2_MODE_REINDEX && a->mode != CSA2_MODE_REUSE)
        return CSA2_ERR_INVALID_ARG;
    if (a->batch < 1 || a->q_per_seq < 1 || a->q_per_seq > 65536) return CSA2_ERR_INVALID_ARG;
    if (a->ratio != 1 && a->ratio != 2) return CSA2_ERR_INVALID_ARG;
    if (a->reserved0 != 0 || a->reserved1 != 0 || a->max_n < 1) return CSA2_ERR_INVALID_ARG;
    if (a->swa_format != CSA2_SWA_BF16 && a->swa_format != CSA2_SWA_FP8) return CSA2_ERR_INVALID_ARG;
    if ((a->q_format != CSA2_Q_BF16 && a->q_format != CSA2_Q_NVFP4) || a->reserved2 != 0)
        return CSA2_ERR_INVALID_ARG;
    const bool swa8 = a->swa_format == CSA2_SWA_FP8;
    if (!a->kv_offsets || !a->codes || !a->scales || !a->topk_idx || !a->q || !a->out) return CSA2_ERR_INVALID_ARG;
    if (swa8 ? (!a->swa_kv8 || !a->swa_kscale) : !a->swa_kv) return CSA2_ERR_INVALID_ARG;
    if (swa8 && (!aligned(a->swa_kv8, 16) || !aligned(a->swa_kscale, 4))) return CSA2_ERR_INVALID_ARG;
    if (swa8 && (a->q_per_seq != 1 || a->q_pos != nullptr)) return CSA2_ERR_UNSUPPORTED;
    if (a->mode != CSA2_MODE_REUSE && (!a->idx_q || !a->idx_w || !a->idx_k || !a->idx_kscale))
        return CSA2_ERR_INVALID_ARG;
    if (a->mode == CSA2_MODE_REINDEX && !a->pool_blocks) return CSA2_ERR_INVALID_ARG;
    if (a->want_pool && (a->mode != CSA2_MODE_FULL || !a->pool_blocks || a->q_per_seq != 1))
        return CSA2_ERR_INVALID_ARG;
    if (a->swa_rows < 1) return CSA2_ERR_INVALID_ARG;
    if ((a->pool_k != nullptr) != (a->pool_kscale != nullptr)) return CSA2_ERR_INVALID_ARG;
    if (a->page_table) {
        if (a->page_rows < 128 || a->page_rows % 128 != 0 || a->page_rows > (1 << 24)) return CSA2_ERR_INVALID_ARG;
        if (a->pages_per_seq < ceil_div(a->max_n, a->page_rows)) return CSA2_ERR_INVALID_ARG;
        if (a->mode == CSA2_MODE_REINDEX && (a->q_per_seq != 1 || a->q_pos != nullptr))
            return CSA2_ERR_UNSUPPORTED;
    }
    if (a->pool_k && (!aligned(a->pool_k, 16) || !aligned(a->pool_kscale, 4))) return CSA2_ERR_INVALID_ARG;
    if (a->sel_cache_mode < CSA2_CACHE_OFF || a->sel_cache_mode > CSA2_CACHE_USE)
        return CSA2_ERR_INVALID_ARG;
    if (a->sel_cache_mode != CSA2_CACHE_OFF && (!a->sel_cache || !aligned(a->sel_cache, 16)))
        return CSA2_ERR_INVALID_ARG;
    if (a->sel_cache_mode == CSA2_CACHE_USE && a->mode != CSA2_MODE_REUSE) return CSA2_ERR_INVALID_ARG;
    if (a->mode != CSA2_MODE_REUSE && (a->total_n < 1 || a->total_n > INT32_MAX))
        return CSA2_ERR_INVALID_ARG;
    if (a->q_pos && a->swa_rows < static_cast<int64_t>(a->q_per_seq) + CSA2_WINDOW - 1)
        return CSA2_ERR_INVALID_ARG;
    if (!aligned(a->q, 16) || (!swa8 && !aligned(a->swa_kv, 16)) || !aligned(a->codes, 16) ||
        !aligned(a->scales, 16) ||
        !aligned(a->out, 8) || (a->idx_q && !aligned(a->idx_q, 16)) ||
        (a->idx_k && !aligned(a->idx_k, 16)))
        return CSA2_ERR_INVALID_ARG;
    const WsLayout L = layer_layout(a);
    if (!a->workspace || !aligned(a->workspace, 256) || a->workspace_bytes < L.total)
        return CSA2_ERR_WORKSPACE;

    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(a->workspace);
    unsigned* err = reinterpret_cast<unsigned*>(ws);
    const int rows = a->batch * a->q_per_seq;
    csa2_status st = CSA2_OK;
    SideFork fork;                                      // the HSI pool select's side stream

    if (a->mode == CSA2_MODE_REINDEX && a->ev_pool) {       // the pool of a deferred Full call
        const cudaError_t ce = cudaStreamWaitEvent(s, static_cast<cudaEvent_t>(a->ev_pool), 0);
        if (ce != cudaSuccess) return fail_cuda("csa2_attend ev_pool wait", ce);
    }
    if (a->mode != CSA2_MODE_REUSE) {
        IndexParams ip;
        ip.batch = a->batch;
        ip.q_per_seq = a->q_per_seq;
        ip.ratio = a->ratio;
        ip.max_n = a->max_n;
        ip.kv_offsets = a->kv_offsets;
        ip.q_pos = a->q_pos;
        ip.idx_q = a->idx_q;
        ip.idx_w = a->idx_w;
        ip.idx_k = a->idx_k;
        ip.idx_kscale = a->idx_kscale;
        ip.pool_blocks = (a->mode == CSA2_MODE_REINDEX) ? a->pool_blocks : nullptr;
        ip.rows = RowMap{a->page_table, a->page_rows, a->pages_per_seq};
        const bool want_bm = (a->mode == CSA2_MODE_FULL && a->want_pool);
        float* bm = want_bm ? reinterpret_cast<float*>(ws + L.blockmax) : nullptr;
        cudaError_t ce;
        // under stream capture the timing events must be event-record nodes of the graph
        cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
        if ((a->ev_index_begin || a->ev_index_end) && (ce = cudaStreamIsCapturing(s, &cap)) != cudaSuccess)
            return fail_cuda("csa2_attend cudaStreamIsCapturing", ce);
        const unsigned ev_flags = cap == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : 0u;
        if (a->ev_index_begin &&
            (ce = cudaEventRecordWithFlags(static_cast<cudaEvent_t>(a->ev_index_begin), s, ev_flags)) !=
                cudaSuccess)
            return fail_cuda("csa2_attend ev_index_begin", ce);
        if (L.fused) {
            ScanSelectArgs sa;
            sa.p = ip;
            sa.chunk = L.chunk;
            sa.n_chunks = L.n_chunks;
            sa.cand_s = reinterpret_cast<float*>(ws + L.cand_s);
            sa.cand_p = reinterpret_cast<int32_t*>(ws + L.cand_p);
            sa.bm = bm;
            sa.bm_ld = L.bm_ld;
            sa.err = err;
            sa.chunk_thr = reinterpret_cast<float*>(ws + L.chunk_thr);
            CUtensorMap tmap;
            const bool pool = a->mode == CSA2_MODE_REINDEX;
            const bool contig = pool && a->pool_k != nullptr;
            sa.pool_kscale = contig ? a->pool_kscale : nullptr;
            const bool map_ok = contig ? make_idx_k_map(a->pool_k, static_cast<int64_t>(a->batch) * POOL_POSITIONS,
                                                        128, &tmap)
                                       : make_idx_k_map(a->idx_k, a->total_n, pool ? POOL_BLOCK : 128, &tmap);
            if (!map_ok) {
                std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed");
                return CSA2_ERR_CUDA;
            }
            st = launch_scan_select(sa, tmap, pool, want_bm, s);
        } else if (L.prefill_fused) {
            CUtensorMap tmap;
            if (!make_idx_k_map(a->idx_k, a->total_n, 128, &tmap)) {
                std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed");
                return CSA2_ERR_CUDA;
            }
            st = launch_prefill_index(ip, tmap, a->topk_idx, err, s);
        } else {
            st = launch_index_score(ip, reinterpret_cast<float*>(ws + L.scores), L.scores_ld,
                                    bm, L.bm_ld, s);
        }
        if (st != CSA2_OK) return st;
        if (a->ev_index_end &&
            (ce = cudaEventRecordWithFlags(static_cast<cudaEvent_t>(a->ev_index_end), s, ev_flags)) !=
                cudaSuccess)
            return fail_cuda("csa2_attend ev_index_end", ce);
        // The HSI pool select (Top-2,048 blocks) does not depend on the Top-512 select: it
        // runs on a side stream forked from s, beside the merge and the attention (neither
        // reads the pool), and is joined back at the end of the call.
        const cudaStream_t ps = bm ? fork.begin(s) : s;
        if (bm) {
            st = launch_topk_rows(bm, L.bm_ld, ceil_div(a->max_n, POOL_BLOCK), a->batch, POOL_BLOCKS,
                                  nullptr, 1, a->pool_blocks, ps, a->kv_offsets);
            if (st == CSA2_OK && a->pool_k)            // the pool's rows, contiguous, for Reindex
                st = launch_pool_gather(a->pool_blocks, a->kv_offsets, a->batch, a->idx_k, a->idx_kscale,
                                        a->pool_k, a->pool_kscale, ip.rows, ps);
        }
        if (st == CSA2_OK && L.fused) {
            st = launch_merge_select(reinterpret_cast<float*>(ws + L.cand_s),
                                     reinterpret_cast<int32_t*>(ws + L.cand_p),
                                     reinterpret_cast<float*>(ws + L.chunk_thr), L.n_chunks, rows,
                                     a->topk_idx, s);
        } else if (st == CSA2_OK && !L.prefill_fused) {
            const int64_t ncols = (a->mode == CSA2_MODE_REINDEX) ? POOL_POSITIONS : a->max_n;
            st = launch_topk_rows(reinterpret_cast<float*>(ws + L.scores), L.scores_ld, ncols, rows,
                                  TOPK, ip.pool_blocks, a->q_per_seq, a->topk_idx, s);
        }
        if (st != CSA2_OK) {
            (void)fork.join(s);
            return st;
        }
    }

    AttnParams ap;
    ap.batch = a->batch;
    ap.q_per_seq = a->q_per_seq;
    ap.ratio = a->ratio;
    ap.n_split = L.n_split;
    ap.swa_rows = a->swa_rows;
    ap.sm_scale = a->sm_scale;
    ap.kv_offsets = a->kv_offsets;
    ap.q_pos = a->q_pos;
    ap.codes = a->codes;
    ap.scales = a->scales;
    ap.topk_idx = a->topk_idx;
    ap.q = a->q;
    ap.swa_kv = a->swa_kv;
    ap.out = a->out;
    ap.err = err;
    ap.swa_fp8 = swa8 ? 1 : 0;
    ap.swa_kv8 = a->swa_kv8;
    ap.swa_kscale = a->swa_kscale;
    ap.rows = RowMap{a->page_table, a->page_rows, a->pages_per_seq};
    ap.q_nvfp4 = a->q_format == CSA2_Q_NVFP4 ? 1 : 0;
    {
        CUtensorMap tq, tswa;
        memset(&tswa, 0, sizeof(tswa));                  // unused by the FP8 SWA tiles
        if (!make_bf16_rows_map(a->q, static_cast<int64_t>(rows) * HEADS, 1, HEADS, 2, &tq) ||
            (!swa8 && !make_bf16_rows_map(a->swa_kv, a->swa_rows, a->batch, 32, 3, &tswa))) {
            std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed (attention)");
            (void)fork.join(s);
            return CSA2_ERR_CUDA;
        }
        st = launch_attend_rows(ap, tq, tswa, s);
    }
    const bool defer = st == CSA2_OK && a->ev_pool && a->mode == CSA2_MODE_FULL && a->want_pool;
    const csa2_status js = defer ? fork.defer(s, static_cast<cudaEvent_t>(a->ev_pool)) : fork.join(s);
    return st != CSA2_OK ? st : js;
}

csa2_status csa2_set_wait_limit(void* workspace, uint32_t polls, void* stream) {
    if (!workspace || !aligned(workspace, 256)) return CSA2_ERR_WORKSPACE;
    // word 1 of the header (word 0 is the error word); a pageable source is staged by the
    // runtime before the call returns, so the local may go out of scope
    const unsigned v = polls;
    const cudaError_t ce = cudaMemcpyAsync(static_cast<unsigned*>(workspace) + 1, &v, sizeof(v),
                                           cudaMemcpyHostToDevice, static_cast<cudaStream_t>(stream));
    return ce == cudaSuccess ? CSA2_OK : fail_cuda("csa2_set_wait_limit", ce);
}

csa2_status csa2_check_device_status(void* workspace, void* stream) {
    if (!workspace || !aligned(workspace, 256)) return CSA2_ERR_WORKSPACE;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned h = 0;
    cudaError_t ce = cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, s);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(s);
    if (ce != cudaSuccess) return fail_cuda("csa2_check_device_status", ce);
    if (h != 0 && (ce = cudaMemsetAsync(workspace, 0, sizeof(unsigned), s)) != cudaSuccess)
        return fail_cuda("csa2_check_device_status", ce);
    if (h & ERR_TIMEOUT) return CSA2_ERR_TIMEOUT;
    if (h & ERR_DEVICE) return CSA2_ERR_DEVICE;
    return CSA2_OK;
}

}  // extern "C"
