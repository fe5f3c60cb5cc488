"""Pins for the float64 oracle: facts fixed by the pages, library routines, closed forms,
brute force on tiny inputs and invariants.  CPU only; the CUDA library is not involved.

Each test names what it pins the oracle to.  A plausible slip in the oracle (a dropped
term, a wrong sign, a transposed operand, a wrong tie rule) fails at least one of them.
"""
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import csa2_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append([float(t) for t in line.split()])
    return np.array(rows)


# ---------------------------------------------------------------- number formats


def test_e2m1_value_set_is_the_fp4_grid():
    # E2M1 (FP4 KV section): the value set is {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6}.
    got = sorted(set(np.abs(O.E2M1_TABLE).tolist()))
    assert got == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert all(np.signbit(O.E2M1_TABLE[8:]))          # codes 8..15 are the negatives


def test_e2m1_table_matches_library_decode():
    lib = np.frombuffer(np.arange(16, dtype=np.uint8).tobytes(),
                        dtype=ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(O.E2M1_TABLE, lib)
    np.testing.assert_array_equal(np.signbit(O.E2M1_TABLE), np.signbit(lib))


def test_e4m3_table_matches_torch_float8():
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(lib)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    np.testing.assert_array_equal(np.isnan(O.E4M3_TABLE), nan)
    np.testing.assert_array_equal(O.E4M3_TABLE[~nan], lib[~nan])


def test_e4m3_range_constants():
    pos = O.E4M3_TABLE[:127]
    assert pos.max() == 448.0
    assert pos[1] == 2.0 ** -9                          # smallest subnormal
    assert pos[8] == 2.0 ** -6                          # smallest normal
    assert np.all(np.diff(pos) > 0)                     # codes are ordered by value


def test_e2m1_rounding_golden_ties():
    for y, val, code in _load_golden("e2m1_rne_ties.txt"):
        c = int(O.e2m1_encode_magnitude(np.array([y]))[0])
        assert c == int(code), (y, c, code)
        assert O.E2M1_TABLE[c] == val


def test_e4m3_rounding_golden_cases():
    for v, val, code in _load_golden("e4m3_scale_cases.txt"):
        c = int(O.e4m3_encode_positive(np.array([v]))[0])
        assert c == int(code), (v, c, code)
        assert O.E4M3_TABLE[c] == val


def test_huge_values_saturate():
    # satfinite reading of the NVFP4 conversion: far above the largest finite value the
    # result is still the largest finite value (6 for E2M1, 448 for E4M3)
    huge = np.array([1e30, 2.0 ** 126 / 6, 1e300, 7.0, 465.0])
    assert (O.e2m1_encode_magnitude(huge) == 7).all()
    assert (O.e4m3_encode_positive(huge[[0, 1, 2, 4]]) == 126).all()
    x = np.zeros((1, 512))
    x[0, :16] = 2.0 ** 126
    x[0, 16] = 2.0 ** 126
    x[0, 17] = -1.0
    codes, scales = O.quantize_rows(O.f64_to_bf16(x))
    assert scales[0, 0] == 126 and scales[0, 1] == 126
    assert (codes[0, :8] == 0x77).all()
    assert codes[0, 8] == 0x07 | (0x8 << 4)      # 2^126 -> +6; -1 -> -(1/448 -> 0) = -0


def test_e2m1_rounding_matches_library_cast():
    rng = np.random.default_rng(11)
    grid = O.E2M1_TABLE[:8]
    mids = (grid[1:] + grid[:-1]) / 2
    y = np.concatenate([rng.uniform(0, 8, 20000), grid, mids, [100.0]]).astype(np.float32)
    lib = y.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    ours = O.E2M1_TABLE[O.e2m1_encode_magnitude(y.astype(np.float64))]
    np.testing.assert_array_equal(ours, lib)


def test_e4m3_rounding_matches_library_cast_in_range():
    rng = np.random.default_rng(12)
    grid = O.E4M3_TABLE[:127]
    mids = (grid[1:] + grid[:-1]) / 2
    v = np.concatenate([rng.uniform(0, 448, 20000), rng.uniform(0, 0.03, 20000),
                        grid, mids]).astype(np.float32)
    lib = v.astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    ours = O.E4M3_TABLE[O.e4m3_encode_positive(v.astype(np.float64))]
    np.testing.assert_array_equal(ours, lib)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(13)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.uniform(-30, 30, 20000),
                        [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -0.0, 0.0]])
    v = v.astype(np.float32).astype(np.float64)          # exactly f32 -> one rounding
    lib = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).view(torch.int16)
    lib = lib.numpy().view(np.uint16)
    np.testing.assert_array_equal(O.f64_to_bf16(v), lib)
    bits = rng.integers(0, 1 << 16, 5000).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]               # finite only
    lib_v = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(O.bf16_to_f64(bits), lib_v)


# ---------------------------------------------------------------- quantiser


def _bf16(x):
    return O.f64_to_bf16(np.asarray(x, dtype=np.float64))


def test_quantise_error_bound_and_scale_rule():
    rng = np.random.default_rng(1)
    x = _bf16(rng.standard_normal((64, 512)) * np.exp(rng.uniform(-4, 8, (64, 1))))
    codes, scales = O.quantize_rows(x)
    xv = O.bf16_to_f64(x).reshape(64, 32, 16)
    deq = O.dequantize_rows(codes, scales).reshape(64, 32, 16)
    s = O.E4M3_TABLE[scales]
    amax = np.abs(xv).max(-1)
    # scale is the E4M3 value nearest amax/6: no E4M3 value is strictly nearer
    grid = O.E4M3_TABLE[:127]
    nearest = np.abs(grid[None, None, :] - (amax / 6)[..., None]).min(-1)
    np.testing.assert_array_equal(np.abs(s - amax / 6), nearest)
    # every element within half a grid step of its scaled value, or saturated at 6*s
    assert (s > 0).all()
    y = np.abs(xv) / s[..., None]
    err = np.abs(np.abs(deq) - np.abs(xv)) / s[..., None]
    step = np.where(y < 2, 0.5, np.where(y < 4, 1.0, 2.0))
    ok = (err <= step / 2 + 1e-12) | (y > 6)
    assert ok.all()
    assert ((np.abs(deq) == 6 * s[..., None]) | (y <= 6)).all()
    np.testing.assert_array_equal(np.signbit(deq) | (deq == 0), np.signbit(xv) | (deq == 0))


def test_quantise_blocks_on_the_grid_roundtrip():
    # A block s * c with c on the E2M1 grid and one element at +-6 has amax/6 = s exactly,
    # so quantisation must return s and c unchanged.
    rng = np.random.default_rng(2)
    n = 200
    sc = rng.integers(1, 127, (n, 32)).astype(np.uint8)
    cc = rng.integers(0, 16, (n, 32, 16)).astype(np.uint8)
    cc[..., 0] = np.where(rng.integers(0, 2, (n, 32)) == 1, 15, 7)  # +-6 present
    x = (O.E2M1_TABLE[cc] * O.E4M3_TABLE[sc][..., None]).reshape(n, 512)
    codes, scales = O.quantize_rows(_bf16(x))
    np.testing.assert_array_equal(scales, sc)
    flat = cc.reshape(n, 512)
    expect = (flat[:, 0::2] | (flat[:, 1::2] << 4)).astype(np.uint8)
    # a zero magnitude keeps its sign bit: compare code values, not only magnitudes
    np.testing.assert_array_equal(codes, expect)


def test_quantise_special_blocks():
    x = np.zeros((1, 512))
    x[0, 16:32] = 1e-5                      # amax/6 below half the smallest subnormal
    x[0, 32:48] = -1e-5
    x[0, 48] = 6 * 448 * 4.0                # saturating scale
    x[0, 49] = 1.0
    x[0, 64:80] = 6 * 2.0 ** -9             # scale = smallest subnormal exactly
    codes, scales = O.quantize_rows(_bf16(x))
    assert scales[0, 0] == 0 and scales[0, 1] == 0 and scales[0, 2] == 0
    assert (codes[0, 0:8] == 0).all()
    assert (codes[0, 8:16] == 0).all()                    # +tiny -> +0
    assert (codes[0, 16:24] == 0x88).all()                # -tiny -> -0 (sign kept)
    assert scales[0, 3] == 126                            # 448
    assert codes[0, 24] & 0x0F == 7                       # 6 * 448 * 4 saturates to 6
    assert scales[0, 4] == 1
    assert (codes[0, 32:40] == 0x77).all()                # 6 * s


def test_ratio2_mean_rounds_once_to_bf16():
    a = _bf16([1.0, 1.0, 3.0, -2.0, 1.0])
    b = _bf16([1.0 + 2.0 ** -7, 2.0 ** -20, 3.0 + 2.0 ** -6, 2.0, -1.0])
    x = np.stack([a, b], axis=1).reshape(-1)
    x = np.tile(x[:, None], (1, 512))[:10]
    out = O.bf16_to_f64(O.compress_ratio2(x))[:, 0]
    # (1 + (1+2^-7))/2 = 1 + 2^-8: a bf16 midpoint between 1 and 1+2^-7 -> even = 1
    # (1 + 2^-20)/2: representable to 8 bits? 0.5 + 2^-21 -> rounds to 0.5
    # (3 + 3 + 2^-6)/2 = 3 + 2^-7: bf16 step at 3 is 2^-6 -> midpoint -> even (3.0)
    # (-2 + 2)/2 = 0
    np.testing.assert_array_equal(out, [1.0, 0.5, 3.0, 0.0, 0.0])


# ---------------------------------------------------------------- indexer


def test_index_score_closed_forms():
    rng = np.random.default_rng(3)
    keys = rng.standard_normal((50, 64))
    q = np.zeros((4, 64))
    q[0, 5] = 1.0
    q[1, 7] = -2.0
    w = np.array([0.5, 0.25, 0.0, 0.0])
    s = O.index_scores(_bf16(q), w, keys)
    expect = 0.5 * np.maximum(keys[:, 5], 0) + 0.25 * np.maximum(-2 * keys[:, 7], 0)
    np.testing.assert_allclose(s, expect, rtol=0, atol=1e-15)
    # every head independently ReLU'd: all-negative dots give zero
    assert (O.index_scores(_bf16(-np.abs(q) * 0 - 1), np.ones(4), np.abs(keys)) == 0).all()


def test_index_score_fp8_keys_and_row_scale():
    k8 = np.array([[0x38] + [0] * 63, [0xB8] + [0] * 63, [0x40] + [0] * 63], np.uint8)
    ks = np.array([2.0, 2.0, 0.5], np.float32)            # 0x38 = 1.0, 0xB8 = -1.0, 0x40 = 2.0
    keys = O.indexer_keys(k8, ks)
    np.testing.assert_array_equal(keys[:, 0], [2.0, -2.0, 1.0])
    q = np.zeros((4, 64))
    q[:, 0] = [1.0, 2.0, -1.0, 0.5]
    s = O.index_scores(_bf16(q), np.array([1.0, 1.0, 1.0, 1.0]), keys)
    np.testing.assert_array_equal(s, [2 + 4 + 0 + 1, 0 + 0 + 2 + 0, 1 + 2 + 0 + 0.5])


# ---------------------------------------------------------------- Top-K and pool


def _brute_topk(scores, positions, k):
    # position p is kept iff fewer than k candidates beat it (higher score, or equal
    # score at a lower position): the definition, evaluated pairwise.
    keep = []
    for i, (s, p) in enumerate(zip(scores, positions)):
        beaters = sum(1 for s2, p2 in zip(scores, positions) if s2 > s or (s2 == s and p2 < p))
        if beaters < k:
            keep.append(p)
    keep = sorted(keep)
    return keep + [-1] * (k - len(keep))


@pytest.mark.parametrize("n,k", [(1, 1), (5, 3), (12, 4), (12, 12), (7, 9), (30, 10)])
def test_topk_matches_pairwise_definition(n, k):
    rng = np.random.default_rng(n * 100 + k)
    for trial in range(20):
        scores = rng.integers(0, 4, n).astype(np.float64)    # many ties
        positions = rng.permutation(100)[:n]
        got = O.topk_select(scores, positions, k).tolist()
        assert got == _brute_topk(scores.tolist(), positions.tolist(), k)


def test_pool_rules():
    rng = np.random.default_rng(4)
    n = 8 * 3000 + 5                                          # partial last block
    s = rng.standard_normal(n) ** 2
    pool = O.pool_select(s)
    assert pool.size == 2048 and (pool >= 0).all() and (np.diff(pool) > 0).all()
    bs = O.block_scores(s)
    assert bs.size == 3001 and bs[-1] == s[-5:].max()
    kept = np.zeros(bs.size, bool)
    kept[pool] = True
    assert bs[kept].min() >= bs[~kept].max()
    # Top-512 lies inside the pool: each Top-512 position's block beats the 512th score,
    # and at most 512 blocks can hold a Top-512 position.
    top = O.topk_select(s, np.arange(n), 512)
    assert np.isin(top // 8, pool).all()
    # few blocks -> every block is kept
    small = O.pool_select(s[:8 * 100 + 3])
    np.testing.assert_array_equal(small[:101], np.arange(101))
    assert (small[101:] == -1).all()


def test_pool_matches_pairwise_definition():
    rng = np.random.default_rng(5)
    s = rng.integers(0, 3, 8 * 20 + 3).astype(np.float64)
    bs = O.block_scores(s)
    got = O.topk_select(bs, np.arange(bs.size), 6).tolist()
    assert got == _brute_topk(bs.tolist(), list(range(bs.size)), 6)


# ---------------------------------------------------------------- attention


def _rand_layer(seed, n, swa_rows=128, sm=1.0):
    rng = np.random.default_rng(seed)
    latent = _bf16(rng.standard_normal((n, 512)))
    codes, scales = O.quantize_rows(latent)
    k8 = torch.from_numpy(rng.standard_normal((n, 64)).astype(np.float32))
    ks = (k8.abs().amax(1) / 448).clamp_min(1e-12)
    idx_k = (k8 / ks[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return dict(codes=codes, scales=scales, idx_k=idx_k, idx_kscale=ks.numpy(),
                idx_q=_bf16(rng.standard_normal((4, 64))), idx_w=rng.uniform(0, 1, 4),
                q=_bf16(rng.standard_normal((16, 512)) / math.sqrt(512)),
                swa=_bf16(rng.standard_normal((swa_rows, 512))), sm_scale=sm)


def test_topk_covering_context_is_dense_softmax_attention():
    # With K >= N the selection keeps every position, so CSA2 reduces to dense softmax
    # attention over [all main rows; SWA rows] (keys = values): check against torch SDPA.
    L = _rand_layer(6, 300)
    topk, _, out = O.csa2_layer(O.FULL, **L)
    assert (topk[:300] == np.arange(300)).all() and (topk[300:] == -1).all()
    rows = np.concatenate([O.dequantize_rows(L["codes"], L["scales"]),
                           O.bf16_to_f64(L["swa"])])
    kv = torch.from_numpy(rows)[None, None]
    qq = torch.from_numpy(O.bf16_to_f64(L["q"]))[None, :, None, :]
    ref = torch.nn.functional.scaled_dot_product_attention(
        qq, kv.expand(1, 16, -1, -1), kv.expand(1, 16, -1, -1), scale=1.0)
    np.testing.assert_allclose(out, ref[0, :, 0].numpy(), rtol=1e-12, atol=1e-13)


def test_attention_closed_forms():
    k = np.zeros((2, 512))
    k[0, 0] = 1.0
    k[1, 1] = 1.0
    q = np.zeros((16, 512))
    q[:, 0] = math.log(3.0)          # logits (ln 3, 0): weights 3/4 and 1/4
    out = O.attend(_bf16(q), k, 1.0)
    lq = O.bf16_to_f64(_bf16(q))[0, 0]
    w0 = math.exp(lq) / (math.exp(lq) + 1)
    np.testing.assert_allclose(out[:, 0], w0, rtol=1e-14)
    np.testing.assert_allclose(out[:, 1], 1 - w0, rtol=1e-14)
    # a single key returns that key; identical keys return the key
    one = O.attend(_bf16(q), k[:1], 1.0)
    np.testing.assert_array_equal(one, np.tile(k[:1], (16, 1)))
    same = O.attend(_bf16(np.random.default_rng(0).standard_normal((16, 512))),
                    np.tile(k[1:2], (5, 1)), 1.0)
    np.testing.assert_allclose(same, np.tile(k[1:2], (16, 1)), rtol=1e-15, atol=1e-15)


def test_attention_is_permutation_invariant():
    rng = np.random.default_rng(7)
    rows = rng.standard_normal((40, 512))
    q = _bf16(rng.standard_normal((16, 512)) / 20)
    a = O.attend(q, rows, 1.0)
    b = O.attend(q, rows[rng.permutation(40)], 1.0)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- modes


def test_reuse_passes_indices_through_unchanged():
    L = _rand_layer(8, 2000)
    topk, _, _ = O.csa2_layer(O.FULL, **L)
    before = topk.copy()
    L2 = dict(L, q=_bf16(np.random.default_rng(9).standard_normal((16, 512)) / 22))
    t2, _, out2 = O.csa2_layer(O.REUSE, topk_in=topk, **L2)
    assert t2.tobytes() == before.tobytes()
    assert out2.shape == (16, 512)


def test_reindex_with_full_query_reproduces_full_selection():
    L = _rand_layer(10, 8 * 2048 * 2 + 3)          # more blocks than the pool holds
    topk, pool, _ = O.csa2_layer(O.FULL, want_pool=True, **L)
    t2, _, _ = O.csa2_layer(O.REINDEX, pool_in=pool, **L)
    np.testing.assert_array_equal(t2, topk)
    # pool smaller than the context: Reindex scores only 16,384 positions
    assert O.pool_positions(pool, L["codes"].shape[0]).size == 16384


def test_reindex_over_full_pool_equals_full_scan():
    L = _rand_layer(11, 5000)                        # ceil(5000/8) <= 2048 blocks
    rng = np.random.default_rng(12)
    _, pool, _ = O.csa2_layer(O.FULL, want_pool=True, **L)
    L2 = dict(L, idx_q=_bf16(rng.standard_normal((4, 64))), idx_w=rng.uniform(0, 1, 4))
    full, _, o1 = O.csa2_layer(O.FULL, **L2)
    rein, _, o2 = O.csa2_layer(O.REINDEX, pool_in=pool, **L2)
    np.testing.assert_array_equal(full, rein)
    np.testing.assert_array_equal(o1, o2)


def test_causal_visibility_ratio2():
    # compressed position j covers tokens 2j, 2j+1: visible once both have been seen
    assert [O.visible_main(t, 2, 100) for t in range(6)] == [0, 1, 1, 2, 2, 3]
    assert O.visible_main(10 ** 6, 2, 100) == 100
    # SWA rows of the first chunk (t0 = 0): query t sees tokens 0..t
    rows = [O.visible_swa_rows(t, 0, 127 + 200).size for t in (0, 1, 126, 127, 199)]
    assert rows == [1, 2, 127, 128, 128]


# ---------------------------------------------------------------- byte accounting


def test_global_kv_is_890_bytes_per_token():
    # The whole KV cache costs 890 bytes per token (intro and Key Takeaways of the
    # thecryptopost.io article; the agihunt.info digest gives the same figure).
    assert O.main_row_bytes() == 288
    assert O.indexer_row_bytes() == 68
    assert O.global_kv_bytes_per_token() == 890.0


# ---------------------------------------------------------------- indexer-K row append (A8)

def test_indexer_rows_match_library_fp8_cast():
    # the oracle's E4M3 rounding of the fp32 quotient against torch's float8_e4m3fn cast
    k = np.random.default_rng(11).standard_normal((2000, 64)).astype(np.float32)
    k[::7] *= np.float32(1e-3)
    k[::11] *= np.float32(3e4)
    codes, ks = O.quantize_indexer_rows(k)
    amax = np.abs(k).max(axis=1)
    ref_ks = torch.from_numpy(amax).div(448.0).numpy()                 # torch fp32 division
    assert np.array_equal(ks.view(np.uint32), ref_ks.view(np.uint32))
    q = torch.from_numpy(k) / torch.from_numpy(ref_ks)[:, None]
    ref = q.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)


def test_indexer_rows_closed_forms():
    k = np.zeros((4, 64), np.float32)
    k[0, 0], k[0, 1], k[0, 2], k[0, 3], k[0, 4] = 448.0, 17.0, 19.0, -17.0, 1.0
    k[1, 5] = -3.0                                     # one value: it maps to -448
    k[3, 0], k[3, 1] = 448.0, -0.0                     # the sign of zero is kept
    codes, ks = O.quantize_indexer_rows(k)
    assert ks[0] == 1.0                                # 448 / 448
    assert codes[0, 0] == 0x7E                         # 448 = largest finite E4M3
    assert codes[0, 1] == 0x58                         # 17: tie between 16 and 18 -> 16 (even)
    assert codes[0, 2] == 0x5A                         # 19: tie between 18 and 20 -> 20 (even)
    assert codes[0, 3] == 0xD8                         # -17 -> -16
    assert codes[0, 4] == 0x38                         # 1.0 = 2^0: exponent 7, mantissa 0
    assert (codes[0, 5:] == 0).all()
    assert ks[1] == np.float32(3.0) / np.float32(448.0) and codes[1, 5] == 0xFE
    assert ks[2] == 0.0 and (codes[2] == 0).all()      # all-zero row
    assert codes[3, 1] == 0x80


def test_indexer_rows_error_bound():
    # |e4m3(q) * kscale - k| <= half an E4M3 step of q, times kscale (unsaturated)
    k = np.random.default_rng(12).standard_normal((500, 64)).astype(np.float32)
    codes, ks = O.quantize_indexer_rows(k)
    deq = O.E4M3_TABLE[codes] * ks[:, None].astype(np.float64)
    q = np.abs(k.astype(np.float64)) / ks[:, None]
    step = np.where(q >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(q, 2.0 ** -6))) - 3), 2.0 ** -9)
    assert (np.abs(deq - k) <= 0.5 * step * ks[:, None] * (1 + 1e-6) + 1e-30).all()


# ---------------------------------------------------------------- FP8 SWA rows (A9)

def test_swa_rows_fp8_match_library_cast_and_bound():
    x = (torch.randn(300, 512, generator=torch.Generator().manual_seed(13)) * 2).to(torch.bfloat16)
    x[7] = 0.0
    codes, sc = O.quantize_swa_rows(x.view(torch.int16).numpy().view(np.uint16))
    xf = x.float()
    ref_sc = (xf.abs().amax(dim=1) / 448.0).numpy()
    assert np.array_equal(sc.view(np.uint32), ref_sc.view(np.uint32))
    safe = torch.from_numpy(np.where(ref_sc > 0, ref_sc, 1.0).astype(np.float32))
    ref = (xf / safe[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ref[7] = 0
    assert np.array_equal(codes, ref)
    deq = O.dequantize_e4m3_rows(codes, sc)
    assert (deq[7] == 0).all()
    # relative error of an unsaturated E4M3 element is at most 2^-4 of its magnitude
    xd = xf.double().numpy()
    big = np.abs(xd) >= sc[:, None] * 2.0 ** -6
    assert (np.abs(deq - xd)[big] <= np.abs(xd)[big] * 2.0 ** -4 + 1e-30).all()


def test_layer_with_fp8_swa_equals_dense_reference():
    # the FP8 SWA variant changes only the SWA rows: softmax over [main; dequantised SWA]
    rng = np.random.default_rng(14)
    lat = (torch.randn(40, 512, generator=torch.Generator().manual_seed(15))).to(torch.bfloat16)
    lb = lat.view(torch.int16).numpy().view(np.uint16)
    codes, scales = O.quantize_rows(lb)
    swa = (torch.randn(9, 512, generator=torch.Generator().manual_seed(16))).to(torch.bfloat16)
    s8, ss = O.quantize_swa_rows(swa.view(torch.int16).numpy().view(np.uint16))
    q = (torch.randn(16, 512, generator=torch.Generator().manual_seed(17)) / 22.6).to(torch.bfloat16)
    qb = q.view(torch.int16).numpy().view(np.uint16)
    sel = np.full(512, -1, np.int32)
    sel[:5] = np.sort(rng.choice(40, 5, replace=False))
    _, _, out = O.csa2_layer(O.REUSE, codes=codes, scales=scales, q=qb, swa=s8, swa_scale=ss, topk_in=sel)
    # keys/values: the FP4 rows (decoded by the ml_dtypes E2M1/E4M3 tables) and the FP8
    # SWA rows (decoded by torch's float8_e4m3fn), attention by torch's SDPA in float64
    def fp4_rows(c, sc):
        lo, hi = c & 0xF, c >> 4
        nib = np.stack([lo, hi], axis=-1).reshape(c.shape[0], 512)
        vals = np.array([float(ml_dtypes.float4_e2m1fn(v)) for v in
                         [0, .5, 1, 1.5, 2, 3, 4, 6, -0.0, -.5, -1, -1.5, -2, -3, -4, -6]])[nib]
        s16 = sc.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
        return vals * np.repeat(s16, 16, axis=1)
    main = fp4_rows(codes[sel[:5]], scales[sel[:5]])
    swa_d = torch.from_numpy(s8).view(torch.float8_e4m3fn).double().numpy() * ss.astype(np.float64)[:, None]
    kv = torch.from_numpy(np.concatenate([main, swa_d]))
    ref = torch.nn.functional.scaled_dot_product_attention(q.double()[None], kv[None], kv[None], scale=1.0)[0]
    assert np.allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- A10: NVFP4 query variant


def _fp4_decode(c, sc):
    """(codes, scales) -> float64 rows through the ml_dtypes E2M1 / E4M3 decoders."""
    lo, hi = c & 0xF, c >> 4
    nib = np.stack([lo, hi], axis=-1).reshape(c.shape[0], 512)
    vals = np.array([float(ml_dtypes.float4_e2m1fn(v)) for v in
                     [0, .5, 1, 1.5, 2, 3, 4, 6, -0.0, -.5, -1, -1.5, -2, -3, -4, -6]])[nib]
    return vals * np.repeat(sc.view(ml_dtypes.float8_e4m3fn).astype(np.float64), 16, axis=1)


def _variant_case(seed, n_main, n_swa):
    g = torch.Generator().manual_seed(seed)
    lat = torch.randn(max(n_main, 1), 512, generator=g).to(torch.bfloat16)
    codes, scales = O.quantize_rows(lat.view(torch.int16).numpy().view(np.uint16))
    swa = torch.randn(n_swa, 512, generator=g).to(torch.bfloat16)
    q = (torch.randn(16, 512, generator=g) * 0.7).to(torch.bfloat16)
    sel = np.full(512, -1, np.int32)
    sel[:n_main] = np.arange(n_main)
    return codes, scales, swa, q, sel


def test_nvfp4_query_variant_is_sdpa_over_an_augmented_key_space():
    # keys [main | 0] and [0 | swa], query [q4 | q]: one torch SDPA gives the softmax whose
    # main logits use the NVFP4 query (decoded by ml_dtypes) and SWA logits the bf16 one
    codes, scales, swa, q, sel = _variant_case(21, 37, 11)
    qb = q.view(torch.int16).numpy().view(np.uint16)
    _, _, out = O.csa2_layer(O.REUSE, codes=codes, scales=scales, q=qb, swa=swa.view(torch.int16).numpy()
                             .view(np.uint16), topk_in=sel, sm_scale=0.3, q_nvfp4=True)
    qc, qs = O.quantize_rows(qb)
    q4 = _fp4_decode(qc, qs)
    main = _fp4_decode(codes[:37], scales[:37])
    sw = swa.double().numpy()
    kaug = np.concatenate([np.concatenate([main, np.zeros_like(main)], axis=1),
                           np.concatenate([np.zeros_like(sw), sw], axis=1)])
    qaug = np.concatenate([q4, q.double().numpy()], axis=1)
    v = np.concatenate([main, sw])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qaug)[:, None], torch.from_numpy(kaug)[None].expand(16, -1, -1),
        torch.from_numpy(v)[None].expand(16, -1, -1), scale=0.3)[:, 0]
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-11, atol=1e-13)


def test_nvfp4_query_on_the_grid_is_the_exact_path():
    # a query whose every head is already an NVFP4 row (values on the E2M1 x E4M3 grid, exact
    # in bf16, every 16-block holding a +-6 element so that amax / 6 is its scale) quantises
    # to itself: the variant equals the exact layer
    codes, scales, swa, _, sel = _variant_case(22, 60, 20)
    rng = np.random.default_rng(23)
    qc = rng.integers(0, 256, (16, 256), dtype=np.uint8)
    qc[:, 0::8] = (qc[:, 0::8] & 0xF8) | 0x07          # element 16 j: magnitude code 7 (6.0)
    qs = rng.integers(0x20, 0x48, (16, 32), dtype=np.uint8)
    qv = _fp4_decode(qc, qs)
    qb = O.f64_to_bf16(qv)
    assert (O.bf16_to_f64(qb) == qv).all()
    np.testing.assert_array_equal(O.quantize_query_nvfp4(qb), qv)
    sb = swa.view(torch.int16).numpy().view(np.uint16)
    kw = dict(codes=codes, scales=scales, q=qb, swa=sb, topk_in=sel, sm_scale=0.05)
    _, _, exact = O.csa2_layer(O.REUSE, **kw)
    _, _, var = O.csa2_layer(O.REUSE, q_nvfp4=True, **kw)
    np.testing.assert_allclose(var, exact, rtol=1e-13, atol=1e-15)


def test_nvfp4_query_changes_only_the_main_logits():
    codes, scales, swa, q, sel = _variant_case(24, 25, 7)
    qb = q.view(torch.int16).numpy().view(np.uint16)
    sb = swa.view(torch.int16).numpy().view(np.uint16)
    empty = np.full(512, -1, np.int32)
    # no main row: the variant is the exact SWA-only attention
    _, _, a = O.csa2_layer(O.REUSE, codes=codes, scales=scales, q=qb, swa=sb, topk_in=empty, q_nvfp4=True)
    _, _, b = O.csa2_layer(O.REUSE, codes=codes, scales=scales, q=qb, swa=sb, topk_in=empty)
    np.testing.assert_array_equal(a, b)
    # no visible SWA row (prefill query before the window's first token): exact attention
    # of the dequantised NVFP4 query, which is itself exact in bf16
    q4 = O.quantize_query_nvfp4(qb)
    q4b = O.f64_to_bf16(q4)
    assert (O.bf16_to_f64(q4b) == q4).all()
    _, _, c = O.csa2_layer(O.REUSE, codes=codes, scales=scales, q=qb, swa=sb[:0], topk_in=sel, q_nvfp4=True)
    _, _, d = O.csa2_layer(O.REUSE, codes=codes, scales=scales, q=q4b, swa=sb[:0], topk_in=sel)
    np.testing.assert_allclose(c, d, rtol=1e-13, atol=1e-15)
    # and the quantised query is not the bf16 one (the variant is not a no-op)
    assert not np.array_equal(q4, O.bf16_to_f64(qb).reshape(16, 512))
