// csa2_build_pool_noalloc: the Hierarchical Sparse Indexer pool ([CP] "DeepSeek AI Released
// DeepSeek-V4.1-Flash with 1M Context, FP4 KV Cache, and Cross-Layer Attention Reuse",
// section "Compressed Sparse Attention 2 (CSA2)": 2,048 blocks of 8 positions) built exactly
// as csa2_build_pool builds it, with the block maxima kept in a fixed array of this module
// instead of a caller workspace.  Nothing is allocated at call time.  The entry point itself
// has no counterpart on the pages (see csa2_build_pool_noalloc in include/csa2.h).
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

namespace {

constexpr int64_t NOALLOC_SCRATCH_FLOATS = CSA2_NOALLOC_POOL_SCRATCH_BYTES / sizeof(float);

// Block maxima [B][bm_ld] of the call in flight on this device.  Every entry a call reads
// is written earlier in the same call, so nothing here needs to start at zero.
static __device__ __align__(256) float g_pool_scratch[NOALLOC_SCRATCH_FLOATS];

constexpr int MAX_DEVICES = 64;

// Device address of g_pool_scratch on the current device, looked up once per device.
csa2_status scratch_address(float** out) {
    static float* addr[MAX_DEVICES] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail_cuda("csa2_build_pool_noalloc cudaGetDevice", e);
    if (dev < 0 || dev >= MAX_DEVICES) return CSA2_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_pool_scratch);
        if (e != cudaSuccess) return fail_cuda("csa2_build_pool_noalloc cudaGetSymbolAddress", e);
        addr[dev] = static_cast<float*>(p);
    }
    *out = addr[dev];
    return CSA2_OK;
}

}  // namespace

}  // namespace csa2

using namespace csa2;

extern "C" csa2_status csa2_build_pool_noalloc(const float* scores, int64_t ld,
                                               const int64_t* kv_offsets, int32_t batch,
                                               int64_t max_n, int32_t* pool_blocks, void* stream) {
    if (batch < 1 || max_n < 1 || ld < max_n) return CSA2_ERR_INVALID_ARG;
    if (!scores || !kv_offsets || !pool_blocks) return CSA2_ERR_INVALID_ARG;
    const int64_t n_blocks = ceil_div(max_n, POOL_BLOCK);
    const int64_t bm_ld = padded_ld(n_blocks);               // the pitch csa2_build_pool uses
    if (bm_ld > NOALLOC_SCRATCH_FLOATS / batch) return CSA2_ERR_UNSUPPORTED;
    float* bm = nullptr;
    const csa2_status st = scratch_address(&bm);
    if (st != CSA2_OK) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const csa2_status st1 = launch_block_max(scores, ld, kv_offsets, batch, max_n, bm, bm_ld, s);
    if (st1 != CSA2_OK) return st1;
    return launch_topk_rows(bm, bm_ld, n_blocks, batch, POOL_BLOCKS, nullptr, 1, pool_blocks, s,
                            kv_offsets);
}
