/*
 * csa2.h — C ABI of libcsa2.so: Compressed Sparse Attention 2 (CSA2) over an FP4 main
 * KV cache, as described for DeepSeek-V4.1-Flash, on NVIDIA B200 (sm_100a).
 *
 * Sources (web pages; none prints an equation, code or a kernel):
 *   [CP] "DeepSeek AI Released DeepSeek-V4.1-Flash with 1M Context, FP4 KV Cache, and
 *        Cross-Layer Attention Reuse" (thecryptopost.io): sections "Compressed Sparse
 *        Attention 2 (CSA2)", "FP4 KV, Bounded Replay, and Other Extensions",
 *        "Causal Encoder-Decoder: Half the Prefill".
 *   [AH] "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression"
 *        (agihunt.info digest of the technical report): the CSA2 / FP4 paragraph.
 *   [TR] "DeepSeek-V4.1 Flash: Pushing the Limits of KV Cache Compression"
 *        (tldrocket.com): the attention-design paragraph (512-dim shared latent).
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is a DEVICE pointer on the current CUDA device, owned by the
 *     caller, contiguous and row-major.  The library allocates no device memory: scratch
 *     comes from the caller's workspace, sized by csa2_workspace_size(), or, for
 *     csa2_build_pool_noalloc only, from a fixed array in the library's own module.
 *   - bf16 tensors are passed as uint16_t bit patterns; E2M1 / E4M3 data as uint8_t.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Every call is asynchronous on that stream: it enqueues kernels and returns.
 *   - Arguments are validated on the host before anything is enqueued; on any error
 *     nothing is enqueued and outputs are untouched.  CSA2_ERR_CUDA means a launch
 *     failed (cudaGetLastError); the CUDA error string is kept for csa2_last_error().
 *   - Ragged batches: kv_offsets[B+1] (device, int64) are prefix sums of each
 *     sequence's position count into the packed main-KV / indexer-K arrays.  Positions
 *     in index outputs are sequence-local, in [0, N_b).
 *   - max_n is a host-side upper bound on every N_b; the kernels clip to the true N_b.
 *     A sequence longer than max_n is not detected and is only partly processed.
 */
#ifndef CSA2_H_
#define CSA2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Fixed shape of the method: 512-dim shared latent [TR]; one E4M3 scale per 16
 * channels [CP, FP4 KV section]; Top-512 and 2,048 blocks of 8 [CP, CSA2 section];
 * 128-token window [CP, Causal Encoder-Decoder section]; 16 query heads and a
 * 4-head x 64-dim indexer (workload shape; the pages do not give the indexer's). */
#define CSA2_D           512
#define CSA2_GROUP       16
#define CSA2_ROW_CODES   256   /* bytes of E2M1 codes per main-KV row */
#define CSA2_ROW_SCALES  32    /* E4M3 scale bytes per main-KV row    */
#define CSA2_HEADS       16
#define CSA2_IDX_HEADS   4
#define CSA2_IDX_DIM     64
#define CSA2_TOPK        512
#define CSA2_WINDOW      128
#define CSA2_POOL_BLOCKS 2048
#define CSA2_POOL_BLOCK  8

typedef int32_t csa2_status;
#define CSA2_OK               0
#define CSA2_ERR_INVALID_ARG  1  /* NULL pointer, bad enum, inconsistent sizes        */
#define CSA2_ERR_UNSUPPORTED  2  /* a shape outside what the kernels implement        */
#define CSA2_ERR_WORKSPACE    3  /* workspace NULL, misaligned or smaller than needed */
#define CSA2_ERR_CUDA         4  /* a CUDA launch or runtime call failed             */
#define CSA2_ERR_TIMEOUT      5  /* a bounded device-side wait gave up (read back)    */
#define CSA2_ERR_DEVICE       6  /* a device-side check failed (read back)            */

/* Cross-layer reuse cache modes (csa2_layer_args.sel_cache: accepted, not used). */
#define CSA2_CACHE_OFF  0
#define CSA2_CACHE_FILL 1
#define CSA2_CACHE_USE  2

/* SWA KV storage (csa2_layer_args.swa_format).  The workloads store the 128-token window
 * in bf16; the agihunt.info digest keeps the SWA KV in FP8.  FP8 here (this library's
 * reading): E4M3 codes with one fp32 scale per row, scale = amax/448 and code = E4M3
 * round-to-nearest-even (saturating) of x/scale, the row used as e4m3(code) * scale. */
#define CSA2_SWA_BF16 0
#define CSA2_SWA_FP8  1

/* Query format of the main-row logits (csa2_layer_args.q_format).  CSA2_Q_BF16 is the
 * method as stated: the bf16 query against the exactly dequantised FP4 rows.
 * CSA2_Q_NVFP4 is the block-scaled FP4 variant (the thecryptopost.io FP4 KV section keeps
 * the main KV in NVFP4, which FP4 tensor cores consume directly): each head's 512-dim
 * query is quantised by the csa2_quantize_kv rule into one NVFP4 row (E2M1 codes + one
 * E4M3 scale per 16 dims), and the logits of the gathered FP4 rows are the block-scaled
 * FP4 MMA of the two; SWA logits, softmax and P V stay exact.  Its error against
 * CSA2_Q_BF16 is the query's FP4 rounding (reported on its own, not held to the
 * attention bound of the exact path). */
#define CSA2_Q_BF16  0
#define CSA2_Q_NVFP4 1

/* Layer modes [CP, CSA2 section; AH digest]: every CSA2 layer has one of three modes,
 * fixed ahead of time. */
#define CSA2_MODE_FULL    0  /* own indexer scores over the context, fresh Top-512    */
#define CSA2_MODE_REINDEX 1  /* rescore the HSI pool with this layer's indexer Q      */
#define CSA2_MODE_REUSE   2  /* reuse the latest Top-512 indices; no indexer at all   */

/* Human-readable name of a status code (static string, never NULL). */
const char* csa2_status_string(csa2_status s);

/* Text of the last CUDA error seen by this thread's calls, or "" (static per thread). */
const char* csa2_last_error(void);

/* Number of kernels this library has enqueued in this process (all devices, all
 * threads; counted after each successful launch). */
uint64_t csa2_kernel_launches(void);

/* ABI version of this header; bumped on any incompatible change. */
int32_t csa2_abi_version(void);
#define CSA2_ABI_VERSION 6

/* ---------------------------------------------------------------------------------
 * csa2_quantize_kv — quantise bf16 latent rows to the FP4 main-KV format.
 *
 * [CP, FP4 KV section]: the main KV is E2M1 with one E4M3 scale per 16 channels,
 * NVFP4 without its global scale.  Per 16-channel group: scale = E4M3 round-to-
 * nearest-even of amax/6 (saturating at 448); code = sign | E2M1 round-to-nearest-
 * even of |x|/scale (saturating at 6); a zero scale gives sign-only codes.  With
 * ratio 2 [CP, CSA2 section: encoder compression ratio of 2; TR: merging adjacent
 * positions] the row quantised is bf16((x[2j] + x[2j+1]) / 2), one rounding.
 *
 *   x       [n_in][512] bf16 latent rows.  n_in must be a multiple of `ratio`; with
 *           ratio 2 each sequence's rows must start at an even row so that pairs never
 *           straddle two sequences (the caller's layout guarantees it).
 *   n_in    number of input rows (>= 0; 0 enqueues nothing).
 *   ratio   1 or 2.
 *   dst_row NULL, or [n_in/ratio] int64 destination rows: output row i is written to
 *           row dst_row[i] of codes/scales (for appending into a larger cache).  The
 *           caller guarantees distinct, in-range rows.
 *   codes   [rows][256] uint8: byte b holds channel 2b in its low nibble and channel
 *           2b+1 in its high nibble; bit 3 of a nibble is the sign.
 *   scales  [rows][32] uint8 E4M3 bit patterns, one per 16 channels.
 * Non-finite inputs are outside the contract.
 * ------------------------------------------------------------------------------- */
csa2_status csa2_quantize_kv(const uint16_t* x, int64_t n_in, int32_t ratio,
                             const int64_t* dst_row, uint8_t* codes, uint8_t* scales,
                             void* stream);

/* ---------------------------------------------------------------------------------
 * csa2_append_kv — the cache append of new decode positions in one kernel: each new
 * position's FP4 main-KV row (as csa2_quantize_kv at ratio 1) and its FP8 indexer-K
 * row with per-row scale [CP, CSA2 section: a Full layer's indexer K is derived from
 * the main KV; FP4 KV section for the main row].  The projection that makes the
 * indexer values is model weights, outside this library: the caller passes its fp32
 * output.  Indexer row (the pages give no format; this library's reading): kscale =
 * amax/448 and code = sign | E4M3 round-to-nearest-even (saturating) of |k/kscale|,
 * both divisions IEEE fp32; an all-zero row gets kscale 0 and zero codes.
 *
 *   latent     [n][512] bf16 rows of the new positions (16-B aligned).
 *   idx_proj   [n][64] fp32 indexer values of the new positions (8-B aligned).
 *   n          rows to append (>= 0; 0 enqueues nothing).
 *   dst_row    [n] int64 destination rows in the packed caches (distinct, in range:
 *              not checked on the device).
 *   codes, scales          main-KV cache, as for csa2_quantize_kv (codes 8-B aligned).
 *   idx_k      [rows][64] uint8 E4M3 indexer K (2-B aligned); idx_kscale [rows] fp32.
 * Non-finite inputs are outside the contract.
 * ------------------------------------------------------------------------------- */
csa2_status csa2_append_kv(const uint16_t* latent, const float* idx_proj, int64_t n,
                           const int64_t* dst_row, uint8_t* codes, uint8_t* scales,
                           uint8_t* idx_k, float* idx_kscale, void* stream);

/* ---------------------------------------------------------------------------------
 * Indexer arguments shared by csa2_index_score and csa2_topk.
 * [CP, CSA2 section]: a Full layer derives indexer K from the main KV and picks a
 * new Top-512; a Reindex layer rescores the shared indexer K with its own
 * indexer Q.  The pages give no formula; this library computes
 *   score(t, s) = kscale[s] * sum_h w[t,h] * ReLU( sum_d q[t,h,d] * e4m3(k8[s,d]) )
 * (4 heads x 64 dims, FP8 E4M3 K with one fp32 scale per row; kscale >= 0).
 * ------------------------------------------------------------------------------- */
typedef struct csa2_index_args {
    int32_t batch;              /* B >= 1 sequences                                     */
    int32_t q_per_seq;          /* queries per sequence (1 = decode)                    */
    int32_t ratio;              /* compression ratio of the cache (1 or 2); only used
                                   with q_pos for causal visibility                     */
    int32_t reserved0;          /* must be 0                                            */
    int64_t max_n;              /* host upper bound on every N_b                        */
    const int64_t* kv_offsets;  /* [B+1] prefix sums of N_b                             */
    const int64_t* q_pos;       /* [B] token of each sequence's first query, or NULL.
                                   With q_pos, query i of sequence b is token
                                   t = q_pos[b] + i and sees compressed position j
                                   iff ratio*j + ratio - 1 <= t.  NULL: every
                                   position is visible (decode).                        */
    const uint16_t* idx_q;      /* [B*q_per_seq][4][64] bf16                            */
    const float* idx_w;         /* [B*q_per_seq][4] head weights                        */
    const uint8_t* idx_k;       /* [sum N_b][64] E4M3                                   */
    const float* idx_kscale;    /* [sum N_b] per-row fp32 scale (>= 0)                  */
    const int32_t* pool_blocks; /* [B][2048] HSI pool (ascending, -1 padded) or NULL    */
} csa2_index_args;

/* csa2_index_score — materialise indexer scores (stage entry point; csa2_attend runs
 * the fused path).  Row r = b*q_per_seq + i of `scores` holds, at column j:
 *   pool_blocks == NULL: the score of position j (j < max_n);
 *   pool_blocks != NULL: the score of position pool[b][j/8]*8 + j%8 (j < 16384).
 * Invisible, absent or out-of-range entries are written as -inf.
 *   scores  [B*q_per_seq][ld] float, ld >= number of columns (max_n or 16384). */
csa2_status csa2_index_score(const csa2_index_args* a, float* scores, int64_t ld,
                             void* stream);

/* csa2_topk — Top-k per row [CP, CSA2 section: Full and Reindex layers pick a new
 * Top-512 index set].
 * Keeps the k largest finite scores of each row (ties to the lower column), maps each
 * kept column to its position (identity, or through pool_blocks as in
 * csa2_index_score, with q_per_seq rows per sequence), and writes the positions in
 * ascending order, padded with -1.
 *   scores     [rows][ld] float (-inf = not a candidate); n_cols <= ld.
 *   pool_blocks NULL or [rows/q_per_seq][2048].
 *   idx_out    [rows][k] int32.
 *   k          1 .. 4096.
 * Workspace: none.  */
csa2_status csa2_topk(const float* scores, int64_t ld, int64_t n_cols, int32_t rows,
                      int32_t k, const int32_t* pool_blocks, int32_t q_per_seq,
                      int32_t* idx_out, void* stream);

/* csa2_build_pool — the Hierarchical Sparse Indexer's candidate pool [CP, CSA2 section:
 * the decoder's Full layer builds a pool of up to 16,384 positions (2,048 blocks of 8)
 * so later Reindex layers score a bounded set].  Block b of sequence s covers positions
 * 8b .. 8b+7 (< N_s); its score is the max of those positions' scores (-inf entries
 * ignored).  The 2,048 best blocks (ties to the lower block) are written ascending,
 * padded with -1; every block is kept when ceil(N_s/8) <= 2,048.
 *   scores      [B][ld] float, one decode row per sequence (column = position).
 *   kv_offsets  [B+1]; max_n as above (ld >= max_n).
 *   pool_blocks [B][2048] int32.
 *   workspace   >= csa2_pool_workspace_size(B, max_n) bytes, 256-byte aligned. */
size_t csa2_pool_workspace_size(int32_t batch, int64_t max_n);
csa2_status csa2_build_pool(const float* scores, int64_t ld, const int64_t* kv_offsets,
                            int32_t batch, int64_t max_n, int32_t* pool_blocks,
                            void* workspace, size_t workspace_bytes, void* stream);

/* csa2_build_pool_noalloc — csa2_build_pool with no workspace argument.  The pages have
 * no counterpart: this is an integration variant of the pool step above, with the same
 * arguments (minus the workspace), validation, semantics and results.
 * Its [B][bm_ld] fp32 block maxima (bm_ld = ceil(max_n/8) rounded up to 64) live in one
 * fixed array of the library's module, CSA2_NOALLOC_POOL_SCRATCH_BYTES per device (8 MiB:
 * B = 64 sequences of max_n = 262,144), so the call allocates nothing.  It serves
 * callers with no device allocator at hand: a plain C host without a memory pool, or a
 * serving loop that reserved the whole HBM for its KV cache at start-up, where a
 * cudaMalloc would fail or would synchronise the device in the middle of decoding.
 *   - B * bm_ld * 4 > CSA2_NOALLOC_POOL_SCRATCH_BYTES -> CSA2_ERR_UNSUPPORTED, nothing
 *     enqueued.
 *   - The scratch address is looked up (cudaGetSymbolAddress) on the first call on each
 *     device; make that first call before any stream capture.  A failed lookup returns
 *     CSA2_ERR_CUDA with the CUDA error in csa2_last_error().
 *   - Nothing in the scratch has to start at zero: each call writes every entry it reads.
 *   - The scratch is shared by all calls on a device.  Calls that may execute at the same
 *     time (streams not ordered with each other, or host threads without a common
 *     stream) race on it and can return wrong pools; order them on one stream or with
 *     events. */
#define CSA2_NOALLOC_POOL_SCRATCH_BYTES (8u << 20)
csa2_status csa2_build_pool_noalloc(const float* scores, int64_t ld, const int64_t* kv_offsets,
                                    int32_t batch, int64_t max_n, int32_t* pool_blocks,
                                    void* stream);

/* ---------------------------------------------------------------------------------
 * csa2_attend — one CSA2 layer [CP, CSA2 section; Causal Encoder-Decoder section]:
 *   FULL    : indexer scores over every visible position, Top-512 into topk_idx and,
 *             with want_pool, the HSI pool into pool_blocks (and, given pool_k, the
 *             pool's indexer rows contiguously); then attention.
 *   REINDEX : indexer scores over the positions of pool_blocks with this layer's
 *             idx_q / idx_w, Top-512 into topk_idx; then attention.
 *   REUSE   : attention with topk_idx as given.  topk_idx is only read: its bytes are
 *             identical after the call (cross-layer index reuse).
 * Attention, per query and head h: softmax over the union of the selected main-KV
 * rows (FP4 rows dequantised exactly, e2m1 * e4m3) and the visible SWA rows, with
 * logits sm_scale * q_h . row and key = value = the row [TR: a 512-dimensional latent
 * for shared key-value representation].  Every layer has its own q and SWA KV [CP].
 *
 * Visibility: q_pos == NULL (decode) -> all N_b positions and every SWA row.  With
 * q_pos, query i of sequence b is token t = q_pos[b] + i; it sees compressed positions
 * j with ratio*j + ratio - 1 <= t, and SWA buffer rows r whose token
 * q_pos[b] - 127 + r lies in [max(0, t-127), t].
 * ------------------------------------------------------------------------------- */
typedef struct csa2_layer_args {
    int32_t mode;               /* CSA2_MODE_*                                          */
    int32_t batch;              /* B >= 1                                               */
    int32_t q_per_seq;          /* queries per sequence, 1 .. 65536                     */
    int32_t ratio;              /* 1 or 2                                               */
    int32_t want_pool;          /* FULL: also build pool_blocks (decode only: q_per_seq
                                   must be 1)                                           */
    int32_t reserved0;          /* must be 0                                            */
    int64_t max_n;              /* host upper bound on every N_b (>= 1)                 */
    int64_t total_n;            /* host: rows of the packed main-KV / indexer-K arrays
                                   (= kv_offsets[B]); FULL/REINDEX decode bounds every
                                   TMA load of indexer K by it (1 .. 2^31-1)            */
    const int64_t* kv_offsets;  /* [B+1]                                                */
    const int64_t* q_pos;       /* [B] or NULL                                          */
    const uint8_t* codes;       /* [sum N_b][256] main-KV E2M1 codes (16-B aligned)     */
    const uint8_t* scales;      /* [sum N_b][32]  main-KV E4M3 scales (16-B aligned)    */
    const uint16_t* idx_q;      /* FULL/REINDEX: [B*q_per_seq][4][64] bf16              */
    const float* idx_w;         /* FULL/REINDEX: [B*q_per_seq][4]                       */
    const uint8_t* idx_k;       /* FULL/REINDEX: [sum N_b][64] E4M3                     */
    const float* idx_kscale;    /* FULL/REINDEX: [sum N_b]                              */
    int32_t* pool_blocks;       /* [B][2048]: written by FULL+want_pool, read by REINDEX */
    int32_t* topk_idx;          /* [B*q_per_seq][512]: written by FULL/REINDEX, read by
                                   REUSE (ascending positions, -1 padded)               */
    const uint16_t* q;          /* [B*q_per_seq][16][512] bf16 (|q| < 65504)            */
    const uint16_t* swa_kv;     /* CSA2_SWA_BF16: [B][swa_rows][512] bf16 (|x| < 65504);
                                   CSA2_SWA_FP8: ignored (may be NULL)                  */
    int64_t swa_rows;           /* rows per sequence: 128 (decode) or
                                   q_per_seq + 127 (prefill chunk)                      */
    float sm_scale;             /* logit scale                                          */
    int32_t reserved1;          /* must be 0                                            */
    float* out;                 /* [B*q_per_seq][16][512] fp32; must not alias inputs   */
    void* workspace;            /* >= csa2_workspace_size(this) bytes, 256-B aligned;
                                   its first 256 bytes hold the device error word and
                                   must be zeroed before first use                      */
    size_t workspace_bytes;
    uint16_t* sel_cache;        /* optional, B*q_per_seq * 512 KB (16-B aligned): a
                                   cross-layer cache of the selected rows dequantised to
                                   f16.  Validated (mode, pointer, alignment) but neither
                                   written nor read: every attention converts the FP4 rows
                                   in registers, and re-gathering 288 B per row costs less
                                   than writing and reading back the 1 KB f16 row.  Results
                                   are the same with or without it.                     */
    int32_t sel_cache_mode;     /* CSA2_CACHE_OFF, CSA2_CACHE_FILL or CSA2_CACHE_USE (USE:
                                   REUSE only); see sel_cache                           */
    int32_t swa_format;         /* CSA2_SWA_BF16 or CSA2_SWA_FP8 (decode only: q_per_seq
                                   1, q_pos NULL; else CSA2_ERR_UNSUPPORTED)            */
    void* ev_index_begin;       /* optional cudaEvent_t recorded on `stream` right before
                                   the indexer-scan kernel (FULL / REINDEX), or NULL;
                                   under stream capture both events become event-record
                                   nodes of the graph (cudaEventRecordExternal)         */
    void* ev_index_end;         /* optional cudaEvent_t recorded right after it, or NULL */
    const uint8_t* swa_kv8;     /* CSA2_SWA_FP8: [B][swa_rows][512] E4M3 (16-B aligned)  */
    const float* swa_kscale;    /* CSA2_SWA_FP8: [B][swa_rows] fp32 row scales          */
    uint8_t* pool_k;            /* optional (decode: q_per_seq 1, q_pos NULL), with
                                   pool_kscale: [B][16384][64] E4M3 (16-B aligned), the
                                   HSI pool's indexer rows in pool slot order (slot j of
                                   sequence b = position 8*pool_blocks[b][j/8] + j%8;
                                   absent slots zero).  A FULL call with want_pool writes
                                   them (beside the pool select, on the library's side
                                   stream, joined at the end of the call); a REINDEX call
                                   then streams them in 128-row tiles instead of gathering
                                   each 8-row block from idx_k.  Both NULL: not used.   */
    float* pool_kscale;         /* with pool_k: [B][16384] fp32 row scales              */
    const int32_t* page_table;  /* optional paged cache (device, [B][pages_per_seq]): row
                                   of position p of sequence b in codes / scales / idx_k /
                                   idx_kscale = page_table[b*pages_per_seq + p/page_rows] *
                                   page_rows + p % page_rows (the cache's own layout; the
                                   pages need not be in order or contiguous).  kv_offsets
                                   then only give the lengths N_b = kv_offsets[b+1] -
                                   kv_offsets[b].  NULL: positions are packed by
                                   kv_offsets.  Not supported (CSA2_ERR_UNSUPPORTED) by a
                                   prefill REINDEX call, the one indexer call that
                                   materialises scores.                                 */
    int32_t page_rows;          /* with page_table: rows per page, a multiple of 128    */
    int32_t pages_per_seq;      /* with page_table: its row stride, >= ceil(max_n /
                                   page_rows)                                           */
    int32_t q_format;           /* CSA2_Q_BF16 or CSA2_Q_NVFP4 (any mode, decode or
                                   prefill; the attention kernel quantises the query)   */
    int32_t reserved2;          /* must be 0                                            */
    void* ev_pool;              /* optional cudaEvent_t, or NULL.  FULL with want_pool:
                                   instead of joining the pool select and the pool-row
                                   gather back into `stream` at the end of the call, the
                                   library records ev_pool where they end (on its side
                                   stream); pool_blocks / pool_k / pool_kscale are then
                                   ready once ev_pool completes, so later readers must
                                   wait for it.  REINDEX: `stream` waits for ev_pool before
                                   the scan.  Under stream capture the wait must happen
                                   before the capture ends (a REINDEX call, or
                                   cudaStreamWaitEvent) so that the side work rejoins it.
                                   Ignored by other calls.                              */
} csa2_layer_args;

/* Workspace bytes csa2_attend needs for these arguments.  Reads mode, batch,
 * q_per_seq, max_n, want_pool, swa_rows, swa_format and whether q_pos is NULL; other
 * pointers are ignored.  Every mode needs one: its first 256 bytes hold the device error
 * word (word 0) and the wait bound of csa2_set_wait_limit (word 1).  Reuse calls need
 * nothing more (the attention merges its partials on chip).  Decode Full/Reindex
 * (q_per_seq == 1, q_pos == NULL) use the fused scan, whose candidates take
 * B * ceil(columns/4096) * 4 KB (Reindex: 2,816 columns per chunk), plus the block maxima
 * of a Full call with want_pool; a prefill Full call (many queries or q_pos) keeps its
 * streaming Top-512 on chip and needs nothing more; a prefill Reindex call materialises a
 * [rows][16384] fp32 score matrix.  A workspace must not be shared by calls that may run
 * concurrently. */
size_t csa2_workspace_size(const csa2_layer_args* a);

/* Enqueues the layer on `stream` (a cudaStream_t, NULL = the legacy default stream) and
 * returns without synchronising.  A FULL call with want_pool runs the HSI pool select on
 * a second stream the library keeps per device (forked from `stream` after the indexer
 * scan and joined back into it at the end of the call, after the attention, with events;
 * inside a stream capture both become graph edges), so work enqueued on `stream` after
 * the call still sees every output (unless ev_pool defers that join: see ev_pool).  The side stream is created by the first such call made outside a
 * stream capture; until then, and whenever it cannot be created, the pool select runs
 * on `stream`.  Concurrent calls from several host threads share the side stream (they
 * stay correct; their pool selects serialise), except that while one thread captures
 * such a call into a graph no other thread may make FULL want_pool calls on the same
 * device (their work would join the capture). */
csa2_status csa2_attend(const csa2_layer_args* a, void* stream);

/* Reads back (synchronising `stream`) and clears the device error word that bounded
 * waits and device checks of earlier csa2_attend calls with this workspace set (the
 * wait bound of csa2_set_wait_limit is kept).
 * Returns CSA2_OK, CSA2_ERR_TIMEOUT or CSA2_ERR_DEVICE. */
csa2_status csa2_check_device_status(void* workspace, void* stream);

/* Sets the bound, in non-blocking polls (a few tens of cycles each), of every pipelined
 * device-side wait of later calls that use this workspace (0 restores the library's
 * default: 2^24 polls that may each suspend the thread for a while).  The bound is
 * stored in the workspace header, on `stream`, so calls enqueued on `stream` after this
 * one see it.  A wait that runs out sets CSA2_ERR_TIMEOUT in the workspace's error word; its CTA
 * stops computing, waits (with the default bound) for the copies and tensor-core
 * operations it has already issued, frees its tensor memory and returns, so the context
 * stays usable and the next call runs normally.  The outputs of a call that timed out
 * are undefined.  This is a watchdog knob: a serving loop can trade a faster error for a
 * slow GPU, and tests can drive the timeout path on purpose.  No page section describes
 * it (it is part of this library's failure handling, not of the method). */
csa2_status csa2_set_wait_limit(void* workspace, uint32_t polls, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H_ */
