"""Float64 CPU oracle for Compressed Sparse Attention 2 (CSA2) over an FP4 main KV cache.

TEST INFRASTRUCTURE ONLY.  This module is the checker the CUDA library is compared
against.  Only the test suite, the smoke check and the CPU-baseline leg of the bench
may import it; the product path (the C-ABI library and its Python binding) never does,
and this module imports nothing from the product package.  It shares no code, table or
constant generator with the CUDA sources.

It is written for a reader to check by eye against the pages, not for speed: every step
is the plain definition, in float64, in the order the method states it.

Sources (web pages about DeepSeek-V4.1-Flash; none prints an equation or code):
  [CP]  "DeepSeek AI Released DeepSeek-V4.1-Flash with 1M Context, FP4 KV Cache, and
        Cross-Layer Attention Reuse" (thecryptopost.io), sections "Compressed Sparse
        Attention 2 (CSA2)", "FP4 KV, Bounded Replay, and Other Extensions" and
        "Causal Encoder-Decoder: Half the Prefill".
  [AH]  "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression" (agihunt.info
        digest of the technical report), the CSA2 / FP4 paragraph of the digest.
  [TR]  "DeepSeek-V4.1 Flash: Pushing the Limits of KV Cache Compression"
        (tldrocket.com), the attention-design paragraph (512-dim shared latent,
        merging of adjacent positions).

What the pages fix:
  * main KV = one 512-dim latent per position, shared as key and value [TR];
  * it is stored as E2M1 elements with one E4M3 scale per 16 channels, NVFP4 without
    its global scale [CP, FP4 KV section; AH];
  * each CSA2 layer is Full (own indexer scores, fresh Top-512), Reindex (rescores the
    shared indexer K with its own indexer Q) or Reuse (reuses the latest Top-K, no
    indexer) [CP, CSA2 section; AH];
  * the decoder's Full layer builds a candidate pool of up to 16,384 positions =
    2,048 blocks of 8 for the later Reindex layers [CP, CSA2 section];
  * every layer also attends over its own 128-token sliding window [CP, Causal
    Encoder-Decoder section];
  * the encoder merges adjacent positions at compression ratio 2 [CP; TR].

Stated assumptions where the pages are silent (each is listed in the design notes):
  A1  scale = E4M3 round-to-nearest-even of amax/6, saturating at 448; element code =
      E2M1 round-to-nearest-even of x/scale, saturating at 6; the element sign is kept
      even when the magnitude rounds to 0; a zero scale gives sign-only codes.
  A2  ratio-2 compression = mean of the two adjacent bf16 latents, rounded once to bf16.
  A3  indexer: 4 heads x 64 dims; K stored as FP8 E4M3 with one fp32 scale per row;
      score(t, s) = sum_h w[t,h] * ReLU(q[t,h] . k[s]) with k[s] = kscale[s] * e4m3(k8[s]).
  A4  Top-K keeps the K largest scores, ties to the lower position; indices are
      returned in ascending position order, padded with -1.
  A5  HSI block score = max of the (up to 8) position scores in the block; the top
      2,048 blocks are kept with the same tie rule.
  A6  attention: softmax over the union of the gathered main-KV rows and the visible
      SWA rows (no de-duplication), key = value = the row, logits scaled by sm_scale.
  A7  causal visibility at ratio r: a query at token t sees compressed position j when
      r*j + r - 1 <= t; it sees SWA tokens max(0, t-127) .. t.
  A8  indexer-K row of a new position (the cache append): from its fp32 indexer
      projection k[64], kscale = fp32(amax / 448) and k8 = E4M3 round-to-nearest-even,
      saturating, of fp32(k / kscale), both quotients in IEEE fp32 (the precision the
      stored scale has); an all-zero row gets kscale 0 and zero codes.
  A9  FP8 SWA KV (the variant the digest's "SWA KV stays FP8" suggests; the workloads
      use bf16): each 512-wide SWA row is stored as E4M3 codes with one fp32 scale per
      row, made from the bf16 row exactly as in A8; attention uses the dequantised row
      e4m3(code) * scale as key and value.
  A10 block-scaled FP4 query (the variant the FP4 KV section's NVFP4 format allows on
      FP4 tensor cores): each head's 512-dim query is quantised as one NVFP4 row by the
      A1 quantiser; the logits of the gathered main-KV rows use that quantised query
      (dequantised exactly), the SWA logits and the values are unchanged.  Its error
      against the exact path is reported on its own, not held to the attention bound.
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------------
# Shape constants of the method (fixed by the pages or by the stated assumptions).
# ----------------------------------------------------------------------------------
D_LATENT = 512      # shared latent width [TR]
GROUP = 16          # channels per E4M3 scale [CP, FP4 KV section]
N_HEADS = 16        # main query heads (workload shape)
IDX_HEADS = 4       # indexer heads (assumption A3)
IDX_DIM = 64        # indexer head dim (assumption A3)
TOPK = 512          # Top-512 [CP, CSA2 section]
SWA_WINDOW = 128    # sliding window [CP, Causal Encoder-Decoder section]
POOL_BLOCKS = 2048  # HSI pool = 2,048 blocks ... [CP, CSA2 section]
POOL_BLOCK = 8      # ... of 8 positions

FULL, REINDEX, REUSE = 0, 1, 2

# ----------------------------------------------------------------------------------
# Number formats, decoded from their bit fields.
# ----------------------------------------------------------------------------------


def e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit,
    no infinities or NaN.  Exponent field 0 is subnormal: 0.5 * mantissa."""
    sign = -1.0 if (code >> 3) & 1 else 1.0
    exp = (code >> 1) & 3
    man = code & 1
    if exp == 0:
        return sign * 0.5 * man
    return sign * 2.0 ** (exp - 1) * (1.0 + 0.5 * man)


def e4m3_value(code: int) -> float:
    """Value of an 8-bit E4M3 ("fn") code: 1 sign, 4 exponent bits (bias 7), 3 mantissa
    bits; exponent field 0 is subnormal (mantissa/8 * 2^-6); 0x7F / 0xFF are NaN; no
    infinities."""
    sign = -1.0 if (code >> 7) & 1 else 1.0
    exp = (code >> 3) & 15
    man = code & 7
    if exp == 15 and man == 7:
        return float("nan")
    if exp == 0:
        return sign * (man / 8.0) * 2.0 ** -6
    return sign * 2.0 ** (exp - 7) * (1.0 + man / 8.0)


E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def _nearest_even(y: np.ndarray, values: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """Code of the value nearest to each y (all inputs >= 0), ties to the even code.

    `values` is ascending and `codes` are the matching codes, whose low bit is the
    mantissa LSB; y above the largest value saturates to it (satfinite)."""
    # satfinite: anything above the largest value is that value (clamping first also
    # keeps huge inputs from making every float64 distance equal)
    y = np.minimum(np.asarray(y, dtype=np.float64), values[-1])
    dist = np.abs(y[..., None] - values)                 # [..., n_values]
    best = dist.min(axis=-1, keepdims=True)
    is_best = dist == best
    # Among equally near values prefer an even code; there are at most two candidates.
    even = (codes % 2 == 0)
    pick_even = is_best & even
    has_even = pick_even.any(axis=-1, keepdims=True)
    chosen = np.where(has_even, pick_even, is_best)
    idx = np.argmax(chosen, axis=-1)
    return codes[idx]


_E2M1_POS_CODES = np.arange(8)                           # magnitudes 0 .. 6
_E2M1_POS_VALUES = E2M1_TABLE[:8]
_E4M3_POS_CODES = np.arange(127)                         # 0 .. 448, NaN (0x7F) excluded
_E4M3_POS_VALUES = E4M3_TABLE[:127]


def e2m1_encode_magnitude(y: np.ndarray) -> np.ndarray:
    """E2M1 magnitude code (0..7) of y >= 0: round to nearest, ties to even, saturate."""
    return _nearest_even(y, _E2M1_POS_VALUES, _E2M1_POS_CODES).astype(np.uint8)


def e4m3_encode_positive(v: np.ndarray) -> np.ndarray:
    """E4M3 code (0..126) of v >= 0: round to nearest, ties to even, saturate at 448."""
    return _nearest_even(v, _E4M3_POS_VALUES, _E4M3_POS_CODES).astype(np.uint8)


# ----------------------------------------------------------------------------------
# bf16 as raw uint16 bits (numpy has no bf16 type).
# ----------------------------------------------------------------------------------


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (the upper half of an IEEE binary32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (8 significant bits, binary32 exponent range),
    nearest with ties to even, straight from float64 (one rounding).  Finite inputs
    inside the bf16 range only."""
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros(v.shape, dtype=np.float64)
    nz = v != 0
    _, e = np.frexp(np.abs(v[nz]))                        # |v| = m * 2^e, m in [0.5, 1)
    # bf16 keeps 8 significant bits: spacing 2^(e-8) in binade [2^(e-1), 2^e);
    # below the normal range the spacing stays at the subnormal step 2^-133.
    spacing = np.ldexp(1.0, np.maximum(e - 8, -133))
    out[nz] = np.round(v[nz] / spacing) * spacing        # np.round is half-to-even
    f32 = out.astype(np.float32)                          # exact: out has <= 8 bits
    bits = (f32.view(np.uint32) >> 16).astype(np.uint16)
    # keep the sign of zero
    bits = np.where(v == 0, np.where(np.signbit(v), 0x8000, 0), bits).astype(np.uint16)
    return bits


# ----------------------------------------------------------------------------------
# Step 1: FP4 main-KV quantisation [CP, FP4 KV section; assumption A1].
# Row layout: 256 bytes of codes (byte b = channel 2b in the low nibble, channel 2b+1
# in the high nibble) followed, in a separate array, by 32 E4M3 scale bytes.
# ----------------------------------------------------------------------------------


def quantize_rows(x_bits: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """bf16 latent rows [n][512] (uint16 bits) -> (codes uint8 [n][256], scales uint8 [n][32])."""
    x_bits = np.asarray(x_bits, dtype=np.uint16).reshape(-1, D_LATENT)
    if x_bits.shape[0] > 256:                 # bound the temporaries of _nearest_even
        parts = [quantize_rows(x_bits[i:i + 256]) for i in range(0, x_bits.shape[0], 256)]
        return (np.concatenate([c for c, _ in parts]), np.concatenate([s for _, s in parts]))
    x = bf16_to_f64(x_bits).reshape(-1, D_LATENT // GROUP, GROUP)   # [n][32][16]
    amax = np.abs(x).max(axis=-1)                                   # [n][32]
    scale_code = e4m3_encode_positive(amax / 6.0)                   # [n][32]
    scale = E4M3_TABLE[scale_code]                                  # exact value
    safe = np.where(scale > 0, scale, 1.0)
    mag = e2m1_encode_magnitude(np.abs(x) / safe[..., None])        # [n][32][16]
    mag = np.where(scale[..., None] > 0, mag, 0).astype(np.uint8)   # zero scale -> 0
    sign = np.signbit(x).astype(np.uint8)
    code = (sign << 3) | mag                                        # [n][32][16]
    code = code.reshape(-1, D_LATENT)
    packed = (code[:, 0::2] | (code[:, 1::2] << 4)).astype(np.uint8)
    return packed, scale_code.astype(np.uint8)


def dequantize_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """(codes [n][256], scales [n][32]) -> exact float64 rows [n][512]."""
    codes = np.asarray(codes, dtype=np.uint8)
    lo = codes & 0x0F
    hi = codes >> 4
    code = np.empty((codes.shape[0], D_LATENT), dtype=np.uint8)
    code[:, 0::2] = lo
    code[:, 1::2] = hi
    vals = E2M1_TABLE[code].reshape(-1, D_LATENT // GROUP, GROUP)
    s = E4M3_TABLE[np.asarray(scales, dtype=np.uint8)]
    return (vals * s[..., None]).reshape(-1, D_LATENT)


def compress_ratio2(x_bits: np.ndarray) -> np.ndarray:
    """Ratio-2 sequence compression [CP, CSA2 section; TR; assumption A2]: compressed
    row j = bf16(mean of rows 2j and 2j+1).  The sum of two bf16 values is exact in
    float64 and halving is exact, so the only rounding is the final one to bf16."""
    x = bf16_to_f64(x_bits)
    assert x.shape[0] % 2 == 0, "ratio-2 compression needs an even number of rows"
    return f64_to_bf16((x[0::2] + x[1::2]) / 2.0)


# ----------------------------------------------------------------------------------
# Step 2: indexer scores [CP, CSA2 section: indexer K is derived from the main KV; a
# Reindex layer scores the pool again with its own indexer Q; assumption A3].
# ----------------------------------------------------------------------------------


def quantize_e4m3_rows(k: np.ndarray, width: int) -> tuple[np.ndarray, np.ndarray]:
    """fp32 rows [n][width] -> (E4M3 codes uint8 [n][width], fp32 scales [n]) (A8, A9):
    scale = amax/448, code = RNE saturating E4M3 of x/scale, both divisions in IEEE
    fp32; an all-zero row gets scale 0 and zero codes."""
    k = np.asarray(k, dtype=np.float32).reshape(-1, width)
    amax = np.abs(k).max(axis=1)
    kscale = (amax / np.float32(448.0)).astype(np.float32)             # fp32 division
    safe = np.where(kscale > 0, kscale, np.float32(1.0)).astype(np.float32)
    q = (k / safe[:, None]).astype(np.float32)                         # fp32 division
    mag = e4m3_encode_positive(np.abs(q).astype(np.float64))
    code = (np.signbit(q).astype(np.uint8) << 7) | mag.astype(np.uint8)
    code = np.where(kscale[:, None] > 0, code, 0).astype(np.uint8)
    return code, kscale


def quantize_indexer_rows(k: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """fp32 indexer projections [n][64] -> (E4M3 codes [n][64], fp32 scales [n]) (A8)."""
    return quantize_e4m3_rows(k, IDX_DIM)


def quantize_swa_rows(x_bits: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """bf16 SWA rows [n][512] (uint16 bits) -> (E4M3 codes [n][512], fp32 scales [n]) (A9)."""
    return quantize_e4m3_rows(bf16_to_f64(np.asarray(x_bits)).astype(np.float32), D_LATENT)


def dequantize_e4m3_rows(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """(E4M3 codes [n][w], fp32 scales [n]) -> exact float64 rows [n][w]."""
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)] * np.asarray(scale, dtype=np.float64)[:, None]


def indexer_keys(idx_k: np.ndarray, idx_kscale: np.ndarray) -> np.ndarray:
    """FP8 E4M3 indexer K rows [n][64] with per-row fp32 scale -> float64 rows."""
    return E4M3_TABLE[np.asarray(idx_k, dtype=np.uint8)] * \
        np.asarray(idx_kscale, dtype=np.float64)[:, None]


def index_scores(idx_q_bits: np.ndarray, idx_w: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """Scores of one query against key rows.

    idx_q_bits: bf16 [4][64]; idx_w: [4]; keys: float64 [n][64] (from indexer_keys).
    Returns float64 [n]: sum over heads of w_h * ReLU(q_h . k)."""
    q = bf16_to_f64(idx_q_bits).reshape(IDX_HEADS, IDX_DIM)
    w = np.asarray(idx_w, dtype=np.float64).reshape(IDX_HEADS)
    dots = keys @ q.T                                   # [n][4]
    return (np.maximum(dots, 0.0) * w).sum(axis=1)


# ----------------------------------------------------------------------------------
# Step 3: Top-K and the HSI pool [CP, CSA2 section; assumptions A4, A5].
# ----------------------------------------------------------------------------------


def topk_select(scores: np.ndarray, positions: np.ndarray, k: int) -> np.ndarray:
    """The k best (score desc, position asc) of the candidates, as ascending positions,
    padded with -1 to length k."""
    scores = np.asarray(scores, dtype=np.float64)
    positions = np.asarray(positions, dtype=np.int64)
    order = np.lexsort((positions, -scores))           # primary: -score; then position
    keep = np.sort(positions[order[:k]])
    out = np.full(k, -1, dtype=np.int32)
    out[:keep.size] = keep
    return out


def block_scores(scores: np.ndarray) -> np.ndarray:
    """HSI block score: max over the positions of each block of 8 (last may be partial)."""
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.size
    nb = -(-n // POOL_BLOCK)
    padded = np.full(nb * POOL_BLOCK, -np.inf)
    padded[:n] = scores
    return padded.reshape(nb, POOL_BLOCK).max(axis=1)


def pool_select(scores: np.ndarray, n_blocks: int = POOL_BLOCKS) -> np.ndarray:
    """HSI candidate pool: the n_blocks best blocks by block score, ties to the lower
    block, ascending, padded with -1."""
    bs = block_scores(scores)
    return topk_select(bs, np.arange(bs.size), n_blocks)


def pool_positions(pool_blocks: np.ndarray, n: int) -> np.ndarray:
    """Positions covered by the pool's blocks (ascending), clipped to the context n."""
    blocks = np.asarray(pool_blocks, dtype=np.int64)
    blocks = blocks[blocks >= 0]
    pos = (blocks[:, None] * POOL_BLOCK + np.arange(POOL_BLOCK)).reshape(-1)
    return pos[pos < n]


# ----------------------------------------------------------------------------------
# Step 4: gather + dequantise + softmax attention over Top-K rows and the SWA window
# [CP, CSA2 and Causal Encoder-Decoder sections; TR; assumption A6].
# ----------------------------------------------------------------------------------


def attend(q_bits: np.ndarray, rows: np.ndarray, sm_scale: float) -> np.ndarray:
    """One query: q bf16 [16][512], rows float64 [m][512] (keys = values).
    Returns float64 [16][512]."""
    q = bf16_to_f64(q_bits).reshape(N_HEADS, D_LATENT)
    logits = sm_scale * (q @ rows.T)                    # [16][m]
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=1, keepdims=True)
    return p @ rows


def quantize_query_nvfp4(q_bits: np.ndarray) -> np.ndarray:
    """A10: a bf16 query [16][512] -> float64 [16][512], each head quantised as one NVFP4
    row by the A1 quantiser (quantize_rows) and dequantised exactly."""
    codes, scales = quantize_rows(np.asarray(q_bits, dtype=np.uint16).reshape(N_HEADS, D_LATENT))
    return dequantize_rows(codes, scales)


def attend_q_nvfp4(q_bits: np.ndarray, main_rows: np.ndarray, swa_rows: np.ndarray,
                   sm_scale: float) -> np.ndarray:
    """A10: one softmax over [main rows; SWA rows] (keys = values) whose main-row logits
    use the NVFP4 query and whose SWA logits use the bf16 query.  Returns [16][512]."""
    q = bf16_to_f64(q_bits).reshape(N_HEADS, D_LATENT)
    q4 = quantize_query_nvfp4(q_bits)
    logits = sm_scale * np.concatenate([q4 @ main_rows.T, q @ swa_rows.T], axis=1)
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=1, keepdims=True)
    return p @ np.concatenate([main_rows, swa_rows], axis=0)


def visible_main(t: int | None, ratio: int, n: int) -> int:
    """Number of compressed positions a query at token t sees (assumption A7);
    t = None means decode, where the whole context is visible."""
    if t is None:
        return n
    return max(0, min(n, (t + 1) // ratio))


def visible_swa_rows(t: int | None, t0: int | None, n_rows: int) -> np.ndarray:
    """Row indices of the SWA buffer a query sees.  Decode (t None): every row.  Prefill:
    the buffer row r holds token t0 - (W-1) + r; the query sees tokens
    max(0, t-W+1) .. t."""
    if t is None:
        return np.arange(n_rows)
    first_tok = t0 - (SWA_WINDOW - 1)
    tok = first_tok + np.arange(n_rows)
    return np.nonzero((tok >= max(0, t - SWA_WINDOW + 1)) & (tok <= t))[0]


# ----------------------------------------------------------------------------------
# Step 5: one CSA2 layer in Full / Reindex / Reuse mode [CP, CSA2 section].
# ----------------------------------------------------------------------------------


def csa2_layer(mode: int, *, codes, scales, idx_k=None, idx_kscale=None, idx_q=None,
               idx_w=None, q, swa, sm_scale=1.0, ratio=1, t=None, t0=None,
               topk_in=None, pool_in=None, want_pool=False, k=TOPK, swa_scale=None,
               q_nvfp4=False):
    """One query of one layer over one sequence.

    codes/scales: the sequence's FP4 main KV [n][256], [n][32]; idx_k/idx_kscale: its
    FP8 indexer K [n][64], [n]; idx_q: bf16 [4][64]; idx_w: [4]; q: bf16 [16][512];
    swa: bf16 [rows][512], or with swa_scale [rows] the FP8 variant's E4M3 codes
    [rows][512] (A9); t: the query's token (None = decode); t0: token of the chunk's
    first query (prefill SWA buffer origin); q_nvfp4: the block-scaled FP4 query
    variant (A10).

    Full    -> scores every visible position, Top-k, and (want_pool) the HSI pool.
    Reindex -> scores the positions of pool_in with this layer's idx_q/idx_w, Top-k.
    Reuse   -> uses topk_in unchanged; no indexer work.
    Returns (topk_idx int32 [k], pool int32 [2048] or None, out float64 [16][512])."""
    n = codes.shape[0]
    nv = visible_main(t, ratio, n)
    pool = None
    if mode == FULL:
        keys = indexer_keys(idx_k[:nv], idx_kscale[:nv])
        s = index_scores(idx_q, idx_w, keys)
        topk = topk_select(s, np.arange(nv), k)
        if want_pool:
            pool = pool_select(s)
    elif mode == REINDEX:
        pos = pool_positions(pool_in, nv)
        keys = indexer_keys(idx_k[pos], idx_kscale[pos])
        s = index_scores(idx_q, idx_w, keys)
        topk = topk_select(s, pos, k)
    elif mode == REUSE:
        topk = np.asarray(topk_in, dtype=np.int32)
    else:
        raise ValueError("mode must be FULL, REINDEX or REUSE")
    sel = topk[topk >= 0]
    main_rows = dequantize_rows(codes[sel], scales[sel])
    vis = visible_swa_rows(t, t0, swa.shape[0])
    if swa_scale is None:
        swa_rows = bf16_to_f64(np.asarray(swa)[vis])
    else:
        swa_rows = dequantize_e4m3_rows(np.asarray(swa)[vis], np.asarray(swa_scale)[vis])
    if q_nvfp4:
        out = attend_q_nvfp4(q, main_rows, swa_rows, sm_scale)
    else:
        out = attend(q, np.concatenate([main_rows, swa_rows], axis=0), sm_scale)
    return topk, pool, out


# ----------------------------------------------------------------------------------
# Byte accounting of the packed cache [CP intro and Key Takeaways: 890 bytes per token].
# ----------------------------------------------------------------------------------


def main_row_bytes() -> int:
    """Bytes of one packed FP4 main-KV row: 4-bit codes + one 1-byte scale per 16."""
    return D_LATENT * 4 // 8 + D_LATENT // GROUP


def indexer_row_bytes() -> int:
    """Bytes of one FP8 indexer-K row + its fp32 scale (assumption A3)."""
    return IDX_DIM * 1 + 4


def global_kv_bytes_per_token(encoder_full_layers: int = 3, encoder_ratio: int = 2,
                              decoder_full_layers: int = 1, decoder_ratio: int = 1) -> float:
    """Global-KV bytes per prompt token under the layer schedule of the CSA2 section:
    only Full layers own a main KV and an indexer K (Reindex/Reuse layers reuse them);
    the encoder's 3 groups each have one Full layer at ratio 2, the decoder's 5 groups
    share one main KV at ratio 1 whose only Full layer is the first."""
    per_pos = main_row_bytes() + indexer_row_bytes()
    return (encoder_full_layers * per_pos / encoder_ratio
            + decoder_full_layers * per_pos / decoder_ratio)
