"""GPU parity: every stage of the CUDA path, called through the C ABI, against the
float64 oracle on the same seeded inputs (small sizes that span several tiles and a
ragged tail; full workload sizes live in test_gpu_workloads.py)."""
import math

import numpy as np
import pytest
import torch

from oracle import csa2_oracle as O
from tests.helpers import (SeqView, attention_check, bits, host, oracle_fp4, oracle_scores,
                           score_tolerance, topk_tie_check)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def csa2():
    from __graft_entry__ import build
    build()
    from fp4_kv_cache_04_b200 import csa2 as c
    return c


@pytest.fixture(scope="module")
def synth():
    from fp4_kv_cache_04_b200 import synth as s
    return s


def _bf16(x):
    return torch.from_numpy(O.f64_to_bf16(np.asarray(x, np.float64)).view(np.int16)).view(torch.bfloat16)


def _gpu_quantize(csa2, x, ratio=1):
    n = x.shape[0] // ratio
    codes = torch.full((n, 256), 0xAB, dtype=torch.uint8, device=DEV)
    scales = torch.full((n, 32), 0xAB, dtype=torch.uint8, device=DEV)
    csa2.quantize_kv(x.to(DEV), ratio, codes, scales)
    torch.cuda.synchronize()
    return host(codes), host(scales)


# ---------------------------------------------------------------- quantiser: bit exact


def test_quantize_bitexact_wide_range(csa2):
    g = torch.Generator().manual_seed(100)
    x = torch.randn(4096 + 37, 512, generator=g) * torch.exp(torch.empty(4133, 1).uniform_(-12, 12, generator=g))
    x = x.to(torch.bfloat16)
    c, s = _gpu_quantize(csa2, x)
    oc, os_ = O.quantize_rows(bits(x))
    assert np.array_equal(s, os_)
    assert np.array_equal(c, oc)


def test_quantize_bitexact_ties_and_special_blocks(csa2):
    rng = np.random.default_rng(101)
    n = 600
    sc = rng.integers(0, 127, (n, 32))
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.0, 6.0, 7.0, 0.5, 3.0])
    y = rng.choice(mids, (n, 32, 16)) * np.where(rng.integers(0, 2, (n, 32, 16)) == 1, -1, 1)
    y[..., 0] = 6.0                                   # amax/6 = scale exactly
    x = (y * O.E4M3_TABLE[sc][..., None]).reshape(n, 512)
    x[0, :] = 0.0
    x[1, :16] = -1e-30
    x[2, :16] = 6 * 448 * 8
    x[3] = np.ldexp(1.0, rng.integers(-133, 127, 512))           # every binade incl. subnormal bf16
    # amax/6 exactly at E4M3 midpoints
    grid = O.E4M3_TABLE[:127]
    x[4:4 + 8, :] = 0.0
    for i in range(8):
        j = rng.integers(0, 126, 32)
        x[4 + i, ::16] = 6 * (grid[j] + grid[j + 1]) / 2
    xb = _bf16(x)
    c, s = _gpu_quantize(csa2, xb)
    oc, os_ = O.quantize_rows(bits(xb))
    assert np.array_equal(s, os_)
    assert np.array_equal(c, oc)


def test_quantize_ratio2_and_scatter(csa2):
    g = torch.Generator().manual_seed(102)
    x = (torch.randn(2 * 777, 512, generator=g) * 3).to(torch.bfloat16)
    x[0] = -x[1]                                       # mean exactly zero
    c, s = _gpu_quantize(csa2, x, ratio=2)
    oc, os_ = O.quantize_rows(O.compress_ratio2(bits(x)))
    assert np.array_equal(c, oc) and np.array_equal(s, os_)
    # scatter into a larger cache through dst_row
    dst = torch.tensor([5, 0, 9], dtype=torch.int64, device=DEV)
    codes = torch.zeros(10, 256, dtype=torch.uint8, device=DEV)
    scales = torch.zeros(10, 32, dtype=torch.uint8, device=DEV)
    csa2.quantize_kv(x[:3].contiguous().to(DEV), 1, codes, scales, dst_row=dst)
    torch.cuda.synchronize()
    oc3, os3 = O.quantize_rows(bits(x[:3]))
    assert np.array_equal(host(codes)[[5, 0, 9]], oc3) and np.array_equal(host(scales)[[5, 0, 9]], os3)
    assert (host(codes)[[1, 2, 3, 4, 6, 7, 8]] == 0).all()


def test_append_kv_bitexact(csa2):
    """The fused cache append: FP4 main-KV rows and FP8 indexer-K rows + fp32 scales,
    scattered to their rows, bit-exact against the oracle (A1, A8)."""
    g = torch.Generator().manual_seed(103)
    n, rows = 37, 100
    lat = (torch.randn(n, 512, generator=g) * 3).to(torch.bfloat16)
    proj = torch.randn(n, 64, generator=g)
    proj[1] = 0.0                                          # all-zero row: scale 0
    proj[2, :] = torch.tensor([448.0, 17.0, 19.0, -17.0] + [1.0] * 60)   # E4M3 ties
    proj[3] *= 1e-30                                       # tiny
    proj[4] *= 3e30                                        # huge
    proj[5, 7] = -0.0
    dst = torch.randperm(rows, generator=g)[:n].to(torch.int64)
    codes = torch.full((rows, 256), 0xA5, dtype=torch.uint8, device=DEV)
    scales = torch.full((rows, 32), 0xA5, dtype=torch.uint8, device=DEV)
    k8 = torch.full((rows, 64), 0xA5, dtype=torch.uint8, device=DEV)
    ks = torch.full((rows,), 7.0, dtype=torch.float32, device=DEV)
    csa2.append_kv(lat.to(DEV), proj.to(DEV), dst.to(DEV), codes, scales, k8, ks)
    torch.cuda.synchronize()
    oc, osc = O.quantize_rows(bits(lat))
    ok8, oks = O.quantize_indexer_rows(proj.numpy())
    d = dst.numpy()
    assert np.array_equal(host(codes)[d], oc) and np.array_equal(host(scales)[d], osc)
    assert np.array_equal(host(k8)[d], ok8)
    assert np.array_equal(host(ks)[d].view(np.uint32), oks.view(np.uint32))
    rest = np.setdiff1d(np.arange(rows), d)               # other rows untouched
    assert (host(codes)[rest] == 0xA5).all() and (host(k8)[rest] == 0xA5).all()
    assert (host(ks)[rest] == 7.0).all()


# ---------------------------------------------------------------- indexer scores


def _index_problem(synth, lens, seed, qps=1, ratio=1):
    w = synth.Workload("t", seed, len(lens), lens, None, ratio, [synth.FULL], q_per_seq=qps)
    return synth.make_problem(w, device="cpu", with_latent=False)


@pytest.mark.parametrize("lens", [[1000, 4097, 517], [16], [1]])
def test_index_scores_decode(csa2, synth, lens):
    P = _index_problem(synth, lens, 200 + len(lens))
    li = P.layers[0]
    B, max_n = len(lens), max(lens)
    scores = torch.full((B, max_n + 64), 7.0, device=DEV)
    csa2.index_score(batch=B, q_per_seq=1, max_n=max_n, kv_offsets=P.kv_offsets.to(DEV),
                     idx_q=li.idx_q.to(DEV), idx_w=li.idx_w.to(DEV), idx_k=P.idx_k.to(DEV),
                     idx_kscale=P.idx_kscale.to(DEV), scores=scores)
    torch.cuda.synchronize()
    got = host(scores).astype(np.float64)
    offs = P.kv_offsets.tolist()
    for b in range(B):
        v = SeqView(np.zeros((0,)), np.zeros((0,)), host(P.idx_k), host(P.idx_kscale), offs, b)
        pos = np.arange(v.n)
        ref = oracle_scores(v, bits(li.idx_q[b]), li.idx_w[b].numpy(), pos)
        tol = score_tolerance(v, bits(li.idx_q[b]), li.idx_w[b].numpy(), pos)
        assert (np.abs(got[b, :v.n] - ref) <= tol).all()
        assert np.isneginf(got[b, v.n:max_n]).all()
        assert (got[b, max_n:] == 7.0).all()           # nothing written past the columns


def test_index_scores_prefill_causal(csa2, synth):
    lens, qps, ratio = [700, 1203], 37, 2
    P = _index_problem(synth, lens, 210, qps=qps, ratio=ratio)
    li = P.layers[0]
    q_pos = torch.tensor([5, 2 * 1203 - 20], dtype=torch.int64)
    B, max_n = 2, max(lens)
    scores = torch.empty(B * qps, max_n, device=DEV)
    csa2.index_score(batch=B, q_per_seq=qps, max_n=max_n, ratio=ratio, q_pos=q_pos.to(DEV),
                     kv_offsets=P.kv_offsets.to(DEV), idx_q=li.idx_q.to(DEV),
                     idx_w=li.idx_w.to(DEV), idx_k=P.idx_k.to(DEV),
                     idx_kscale=P.idx_kscale.to(DEV), scores=scores)
    torch.cuda.synchronize()
    got = host(scores).astype(np.float64)
    offs = P.kv_offsets.tolist()
    for b in range(B):
        v = SeqView(np.zeros((0,)), np.zeros((0,)), host(P.idx_k), host(P.idx_kscale), offs, b)
        for i in range(qps):
            r = b * qps + i
            nv = O.visible_main(int(q_pos[b]) + i, ratio, v.n)
            pos = np.arange(nv)
            ref = oracle_scores(v, bits(li.idx_q[r]), li.idx_w[r].numpy(), pos)
            tol = score_tolerance(v, bits(li.idx_q[r]), li.idx_w[r].numpy(), pos)
            assert (np.abs(got[r, :nv] - ref) <= tol).all(), (b, i)
            assert np.isneginf(got[r, nv:]).all(), (b, i)


def test_index_scores_pool(csa2, synth):
    lens = [30000, 9001]
    P = _index_problem(synth, lens, 220)
    li = P.layers[0]
    rng = np.random.default_rng(5)
    pool = np.full((2, 2048), -1, np.int32)
    pool[0] = np.sort(rng.choice(-(-30000 // 8), 2048, replace=False))
    pool[1, :1126] = np.arange(1126)                    # every block of a short sequence
    scores = torch.empty(2, 16384, device=DEV)
    csa2.index_score(batch=2, q_per_seq=1, max_n=max(lens), kv_offsets=P.kv_offsets.to(DEV),
                     idx_q=li.idx_q.to(DEV), idx_w=li.idx_w.to(DEV), idx_k=P.idx_k.to(DEV),
                     idx_kscale=P.idx_kscale.to(DEV), scores=scores,
                     pool_blocks=torch.from_numpy(pool).to(DEV))
    torch.cuda.synchronize()
    got = host(scores).astype(np.float64)
    offs = P.kv_offsets.tolist()
    for b in range(2):
        v = SeqView(np.zeros((0,)), np.zeros((0,)), host(P.idx_k), host(P.idx_kscale), offs, b)
        cols = np.arange(16384)
        blk = pool[b][cols // 8]
        pos = blk.astype(np.int64) * 8 + cols % 8
        ok = (blk >= 0) & (pos < v.n)
        ref = oracle_scores(v, bits(li.idx_q[b]), li.idx_w[b].numpy(), pos[ok])
        tol = score_tolerance(v, bits(li.idx_q[b]), li.idx_w[b].numpy(), pos[ok])
        assert (np.abs(got[b, ok] - ref) <= tol).all()
        assert np.isneginf(got[b, ~ok]).all()


# ---------------------------------------------------------------- Top-K and pool: exact on
# identical fp32 inputs (the oracle selects on the same fp32 values, widened exactly)


@pytest.mark.parametrize("n,k", [(5000, 512), (511, 512), (512, 512), (513, 512), (100000, 512),
                                 (37, 5), (20000, 2048)])
def test_topk_exact(csa2, n, k):
    rng = np.random.default_rng(n + k)
    rows = 3
    s = rng.standard_normal((rows, n)).astype(np.float32) ** 2
    s[1] = np.floor(s[1] * 4) / 4                      # heavy ties
    s[2, ::3] = -np.inf                                # absent candidates
    s[0, :7] = 0.0
    s[0, 7:9] = -0.0
    out = torch.empty(rows, k, dtype=torch.int32, device=DEV)
    csa2.topk(torch.from_numpy(s).to(DEV), n, k, out)
    torch.cuda.synchronize()
    got = host(out)
    for r in range(rows):
        valid = np.nonzero(~np.isneginf(s[r]))[0]
        ref = O.topk_select(s[r, valid].astype(np.float64), valid, k)
        assert np.array_equal(got[r], ref), r


@pytest.mark.parametrize("n,k", [(700, 512), (5000, 512), (30000, 2048)])
def test_topk_skewed_range(csa2, n, k):
    """One huge outlier stretches the key range, so the bin holding the k-th key gets
    hundreds (ranked by radix passes) or thousands (the full fallback) of distinct keys."""
    rng = np.random.default_rng(7 * n + k)
    s = (1.0 + rng.random((2, n))).astype(np.float32)
    s[:, n // 2] = 3.0e38
    s[1, ::5] = np.float32(1.5)                        # ties inside the crowded bin
    out = torch.empty(2, k, dtype=torch.int32, device=DEV)
    csa2.topk(torch.from_numpy(s).to(DEV), n, k, out)
    torch.cuda.synchronize()
    got = host(out)
    for r in range(2):
        ref = O.topk_select(s[r].astype(np.float64), np.arange(n), k)
        assert np.array_equal(got[r], ref), r


def test_topk_through_pool_map(csa2):
    rng = np.random.default_rng(9)
    pool = np.sort(rng.choice(5000, 2048, replace=False)).astype(np.int32)[None]
    s = rng.standard_normal((2, 16384)).astype(np.float32)
    out = torch.empty(2, 512, dtype=torch.int32, device=DEV)
    csa2.topk(torch.from_numpy(s).to(DEV), 16384, 512, out, pool_blocks=torch.from_numpy(pool).to(DEV),
              q_per_seq=2)
    torch.cuda.synchronize()
    pos = pool[0][np.arange(16384) // 8].astype(np.int64) * 8 + np.arange(16384) % 8
    for r in range(2):
        assert np.array_equal(host(out)[r], O.topk_select(s[r].astype(np.float64), pos, 512))


@pytest.mark.parametrize("lens", [[262144 // 4, 5000, 16384, 16391], [8 * 2048], [3]])
def test_build_pool_exact(csa2, lens):
    rng = np.random.default_rng(len(lens) + sum(lens))
    B, max_n = len(lens), max(lens)
    s = np.full((B, max_n), -np.inf, np.float32)
    for b, n in enumerate(lens):
        s[b, :n] = np.round(rng.standard_normal(n).astype(np.float32) ** 2, 2)   # ties
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    pool = torch.empty(B, 2048, dtype=torch.int32, device=DEV)
    ws = csa2.alloc_workspace(csa2.pool_workspace_size(B, max_n))
    csa2.build_pool(torch.from_numpy(s).to(DEV), torch.from_numpy(offs).to(DEV), max_n, pool, ws)
    torch.cuda.synchronize()
    for b, n in enumerate(lens):
        assert np.array_equal(host(pool)[b], O.pool_select(s[b, :n].astype(np.float64))), b


# ---------------------------------------------------------------- attention (Reuse mode fed
# the oracle's indices, so it checks the attention alone)


def _cache(csa2, latent, ratio=1):
    n = latent.shape[0] // ratio
    codes = torch.empty(n, 256, dtype=torch.uint8, device=DEV)
    scales = torch.empty(n, 32, dtype=torch.uint8, device=DEV)
    csa2.quantize_kv(latent.to(DEV), ratio, codes, scales)
    return codes, scales


@pytest.mark.parametrize("lens,n_sel", [([3000, 700], 512), ([300], 300), ([5000, 64, 1000], 200)])
def test_attend_decode_matches_oracle(csa2, synth, lens, n_sel):
    w = synth.Workload("t", 300 + len(lens), len(lens), lens, None, 1, [synth.REUSE])
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    oc, osc = oracle_fp4(P.latent, 1)
    rng = np.random.default_rng(1)
    B = len(lens)
    idx = np.full((B, 512), -1, np.int32)
    for b, n in enumerate(lens):
        m = min(n_sel, n)
        idx[b, :m] = np.sort(rng.choice(n, m, replace=False))
    li = P.layers[0]
    out = torch.empty(B, 16, 512, device=DEV)
    topk = torch.from_numpy(idx).to(DEV)
    kw = dict(mode=synth.REUSE, batch=B, q_per_seq=1, max_n=max(lens), kv_offsets=P.kv_offsets.to(DEV),
              codes=codes, scales=scales, topk_idx=topk, q=li.q.to(DEV), swa_kv=li.swa.to(DEV), out=out)
    ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)))
    csa2.attend(csa2.layer_args(workspace=ws, **kw))
    torch.cuda.synchronize()
    assert np.array_equal(host(topk), idx)
    offs = P.kv_offsets.tolist()
    for b in range(B):
        sl = slice(offs[b], offs[b + 1])
        _, _, ref = O.csa2_layer(O.REUSE, codes=oc[sl], scales=osc[sl], q=bits(li.q[b]),
                                 swa=bits(li.swa[b]), topk_in=idx[b])
        attention_check(host(out[b]), ref, f"seq {b}")


def test_attend_decode_holes_in_selection(csa2, synth):
    """A Reuse index list with -1 slots scattered through it, a wholly empty 64-slot tile
    between full ones, and positions in no particular order: the attention runs over
    exactly the valid positions (the softmax is order-free)."""
    lens = [5000, 700, 9000]
    w = synth.Workload("t", 560, len(lens), lens, None, 1, [synth.REUSE])
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    oc, osc = oracle_fp4(P.latent, 1)
    rng = np.random.default_rng(560)
    B = len(lens)
    idx = np.full((B, 512), -1, np.int32)
    for b, n in enumerate(lens):
        slots = rng.choice(512, 300, replace=False)
        slots = slots[(slots < 128) | (slots >= 192)]            # slots 128..191 stay empty
        idx[b, slots] = rng.choice(n, slots.size, replace=False)
    idx[1, :] = -1
    idx[1, 511] = 699                                            # one valid slot, the last
    li = P.layers[0]
    out = torch.empty(B, 16, 512, device=DEV)
    kw = dict(mode=synth.REUSE, batch=B, q_per_seq=1, max_n=max(lens), kv_offsets=P.kv_offsets.to(DEV),
              codes=codes, scales=scales, topk_idx=torch.from_numpy(idx).to(DEV), q=li.q.to(DEV),
              swa_kv=li.swa.to(DEV), out=out)
    ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)))
    csa2.attend(csa2.layer_args(workspace=ws, **kw))
    assert csa2.check_device_status(ws) == 0
    offs = P.kv_offsets.tolist()
    for b in range(B):
        sl = slice(offs[b], offs[b + 1])
        _, _, ref = O.csa2_layer(O.REUSE, codes=oc[sl], scales=osc[sl], q=bits(li.q[b]),
                                 swa=bits(li.swa[b]), topk_in=idx[b])
        attention_check(host(out[b]), ref, f"seq {b}")


@pytest.mark.parametrize("swa_rows,n_sel", [(1, 0), (63, 1), (64, 70), (65, 512), (200, 129), (128, 0)])
def test_attend_decode_swa_rows_and_short_sets(csa2, synth, swa_rows, n_sel):
    """Decode attention with SWA buffers that do not fill whole 64-row tiles and with
    selections of 0, 1 or a few rows (main tiles partly or wholly empty)."""
    lens = [3000, 129]
    w = synth.Workload("t", 500 + swa_rows, len(lens), lens, None, 1, [synth.REUSE], swa_rows=swa_rows)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    oc, osc = oracle_fp4(P.latent, 1)
    rng = np.random.default_rng(swa_rows)
    B = len(lens)
    idx = np.full((B, 512), -1, np.int32)
    for b, n in enumerate(lens):
        m = min(n_sel, n)
        idx[b, :m] = np.sort(rng.choice(n, m, replace=False))
    li = P.layers[0]
    out = torch.empty(B, 16, 512, device=DEV)
    kw = dict(mode=synth.REUSE, batch=B, q_per_seq=1, max_n=max(lens), kv_offsets=P.kv_offsets.to(DEV),
              codes=codes, scales=scales, topk_idx=torch.from_numpy(idx).to(DEV), q=li.q.to(DEV),
              swa_kv=li.swa.to(DEV), out=out, swa_rows=swa_rows)
    ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)))
    for _ in range(2):                                   # the row tickets reset themselves
        csa2.attend(csa2.layer_args(workspace=ws, **kw))
        torch.cuda.synchronize()
        offs = P.kv_offsets.tolist()
        for b in range(B):
            sl = slice(offs[b], offs[b + 1])
            _, _, ref = O.csa2_layer(O.REUSE, codes=oc[sl], scales=osc[sl], q=bits(li.q[b]),
                                     swa=bits(li.swa[b]), topk_in=idx[b])
            attention_check(host(out[b]), ref, f"seq {b}")
    assert csa2.check_device_status(ws) == 0


@pytest.mark.parametrize("sm_scale", [6.0, 40.0])
def test_attend_decode_large_logits(csa2, synth, sm_scale):
    """Logits spread over tens of units, so a tile's max often exceeds the running max by
    more than the lazy-rescale gap (the O rescale path) and softmax is nearly one-hot."""
    lens = [5000, 3000, 700]
    w = synth.Workload("t", 600 + int(sm_scale), len(lens), lens, None, 1, [synth.REUSE], sm_scale=sm_scale)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    oc, osc = oracle_fp4(P.latent, 1)
    rng = np.random.default_rng(int(sm_scale))
    B = len(lens)
    idx = np.full((B, 512), -1, np.int32)
    for b, n in enumerate(lens):
        idx[b] = np.sort(rng.choice(n, 512, replace=False))
    li = P.layers[0]
    out = torch.empty(B, 16, 512, device=DEV)
    kw = dict(mode=synth.REUSE, batch=B, q_per_seq=1, max_n=max(lens), kv_offsets=P.kv_offsets.to(DEV),
              codes=codes, scales=scales, topk_idx=torch.from_numpy(idx).to(DEV), q=li.q.to(DEV),
              swa_kv=li.swa.to(DEV), out=out, sm_scale=sm_scale)
    ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)))
    csa2.attend(csa2.layer_args(workspace=ws, **kw))
    torch.cuda.synchronize()
    offs = P.kv_offsets.tolist()
    for b in range(B):
        sl = slice(offs[b], offs[b + 1])
        _, _, ref = O.csa2_layer(O.REUSE, codes=oc[sl], scales=osc[sl], q=bits(li.q[b]),
                                 swa=bits(li.swa[b]), topk_in=idx[b], sm_scale=sm_scale)
        attention_check(host(out[b]), ref, f"seq {b}")


@pytest.mark.parametrize("swa_rows,n_sel,sm_scale", [(128, 512, 1.0), (1, 0, 1.0), (65, 70, 1.0),
                                                    (200, 512, 1.0), (128, 300, 30.0)])
def test_attend_decode_fp8_swa(csa2, synth, swa_rows, n_sel, sm_scale):
    """The FP8 SWA variant (E4M3 rows with one fp32 scale each) against the oracle fed the
    same FP8 inputs: every SWA tile size, empty selections, large logits."""
    lens = [3000, 129]
    w = synth.Workload("t", 700 + swa_rows, len(lens), lens, None, 1, [synth.REUSE], swa_rows=swa_rows,
                       sm_scale=sm_scale)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    oc, osc = oracle_fp4(P.latent, 1)
    li = P.layers[0]
    s8, ss = synth.fp8_swa(li.swa)
    s8[1, 0] = 0                                            # a zero row (scale 0) in the window
    ss[1, 0] = 0.0
    rng = np.random.default_rng(swa_rows + n_sel)
    B = len(lens)
    idx = np.full((B, 512), -1, np.int32)
    for b, n in enumerate(lens):
        m = min(n_sel, n)
        idx[b, :m] = np.sort(rng.choice(n, m, replace=False))
    out = torch.empty(B, 16, 512, device=DEV)
    kw = dict(mode=synth.REUSE, batch=B, q_per_seq=1, max_n=max(lens), kv_offsets=P.kv_offsets.to(DEV),
              codes=codes, scales=scales, topk_idx=torch.from_numpy(idx).to(DEV), q=li.q.to(DEV),
              swa_kv=None, swa_kv8=s8.to(DEV), swa_kscale=ss.to(DEV), out=out, sm_scale=sm_scale)
    ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)))
    csa2.attend(csa2.layer_args(workspace=ws, **kw))
    torch.cuda.synchronize()
    assert csa2.check_device_status(ws) == 0
    offs = P.kv_offsets.tolist()
    for b in range(B):
        sl = slice(offs[b], offs[b + 1])
        _, _, ref = O.csa2_layer(O.REUSE, codes=oc[sl], scales=osc[sl], q=bits(li.q[b]),
                                 swa=host(s8[b]), swa_scale=host(ss[b]), topk_in=idx[b], sm_scale=sm_scale)
        attention_check(host(out[b]), ref, f"seq {b}")


def test_attend_prefill_causal_matches_oracle(csa2, synth):
    lens, qps, ratio = [400, 2000], 150, 2
    w = synth.Workload("t", 310, 2, lens, None, ratio, [synth.REUSE], q_per_seq=qps, q_pos=[0, 3000],
                       q_std=1.0, sm_scale=1 / math.sqrt(512), swa_rows=qps + 127)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent, ratio)
    oc, osc = oracle_fp4(P.latent, ratio)
    rng = np.random.default_rng(2)
    idx = np.full((2 * qps, 512), -1, np.int32)
    for b in range(2):
        for i in range(qps):
            nv = O.visible_main(w.q_pos[b] + i, ratio, lens[b])
            m = min(nv, 512)
            if m:
                idx[b * qps + i, :m] = np.sort(rng.choice(nv, m, replace=False))
    li = P.layers[0]
    out = torch.empty(2 * qps, 16, 512, device=DEV)
    kw = dict(mode=synth.REUSE, batch=2, q_per_seq=qps, ratio=ratio, max_n=max(lens),
              kv_offsets=P.kv_offsets.to(DEV), q_pos=P.q_pos.to(DEV), codes=codes, scales=scales,
              topk_idx=torch.from_numpy(idx).to(DEV), q=li.q.to(DEV), swa_kv=li.swa.to(DEV),
              out=out, sm_scale=w.sm_scale)
    ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)))
    csa2.attend(csa2.layer_args(workspace=ws, **kw))
    torch.cuda.synchronize()
    offs = P.kv_offsets.tolist()
    for b in range(2):
        sl = slice(offs[b], offs[b + 1])
        for i in list(range(0, qps, 7)) + [qps - 1]:
            r = b * qps + i
            _, _, ref = O.csa2_layer(O.REUSE, codes=oc[sl], scales=osc[sl], q=bits(li.q[r]),
                                     swa=bits(li.swa[b]), topk_in=idx[r], t=w.q_pos[b] + i,
                                     t0=w.q_pos[b], ratio=ratio, sm_scale=w.sm_scale)
            attention_check(host(out[r]), ref, f"seq {b} query {i}")


# ---------------------------------------------------------------- NVFP4-query variant


def _rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("lens,n_sel,holes,swa8", [([3000, 700], 512, False, False), ([300], 300, False, False),
                                                   ([5000, 700, 9000], 300, True, False),
                                                   ([4000, 129], 512, False, True)],
                         ids=["full_sets", "short_set", "holes", "fp8_swa"])
def test_attend_nvfp4_query_decode(csa2, synth, lens, n_sel, holes, swa8):
    """Decode rows with the block-scaled FP4 query: against the oracle's variant (the same
    quantised query, float64 attention) at the attention bound; the variant's own error
    against the exact path is measured beside it."""
    B = len(lens)
    w = synth.Workload("t", 900 + B, B, lens, None, 1, [synth.REUSE])
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    oc, osc = oracle_fp4(P.latent, 1)
    rng = np.random.default_rng(901)
    idx = np.full((B, 512), -1, np.int32)
    for b, n in enumerate(lens):
        if holes:
            slots = rng.choice(512, n_sel, replace=False)
            slots = slots[(slots < 128) | (slots >= 192)]
            idx[b, slots] = rng.choice(n, slots.size, replace=False)
        else:
            m = min(n_sel, n)
            idx[b, :m] = np.sort(rng.choice(n, m, replace=False))
    li = P.layers[0]
    out = torch.empty(B, 16, 512, device=DEV)
    kw = dict(mode=synth.REUSE, batch=B, q_per_seq=1, max_n=max(lens), kv_offsets=P.kv_offsets.to(DEV),
              codes=codes, scales=scales, topk_idx=torch.from_numpy(idx).to(DEV), q=li.q.to(DEV), out=out,
              q_nvfp4=True)
    if swa8:
        s8, ss = synth.fp8_swa(li.swa)
        kw.update(swa_kv=None, swa_kv8=s8.to(DEV), swa_kscale=ss.to(DEV))
    else:
        kw.update(swa_kv=li.swa.to(DEV))
    ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)))
    csa2.attend(csa2.layer_args(workspace=ws, **kw))
    assert csa2.check_device_status(ws) == 0
    offs = P.kv_offsets.tolist()
    dev = []
    for b in range(B):
        sl = slice(offs[b], offs[b + 1])
        kw_o = dict(codes=oc[sl], scales=osc[sl], q=bits(li.q[b]), topk_in=idx[b])
        if swa8:
            kw_o.update(swa=host(kw["swa_kv8"][b]), swa_scale=host(kw["swa_kscale"][b]))
        else:
            kw_o.update(swa=bits(li.swa[b]))
        _, _, ref = O.csa2_layer(O.REUSE, q_nvfp4=True, **kw_o)
        g = host(out[b]).astype(np.float64)
        attention_check(g, ref, f"seq {b} (NVFP4 query)")
        _, _, exact = O.csa2_layer(O.REUSE, **kw_o)
        dev.append(_rel_l2(ref, exact))
    # the variant is not the exact path, and its FP4 query rounding stays a few percent
    assert all(1e-4 < d < 0.15 for d in dev), dev
    print("NVFP4-query variant vs exact (rel L2):", dev)


def test_attend_nvfp4_query_prefill(csa2, synth):
    lens, qps, ratio = [400, 2000], 150, 2
    w = synth.Workload("t", 910, 2, lens, None, ratio, [synth.REUSE], q_per_seq=qps, q_pos=[0, 3000],
                       q_std=1.0, sm_scale=1 / math.sqrt(512), swa_rows=qps + 127)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent, ratio)
    oc, osc = oracle_fp4(P.latent, ratio)
    rng = np.random.default_rng(911)
    idx = np.full((2 * qps, 512), -1, np.int32)
    for b in range(2):
        for i in range(qps):
            nv = O.visible_main(w.q_pos[b] + i, ratio, lens[b])
            m = min(nv, 512)
            if m:
                idx[b * qps + i, :m] = np.sort(rng.choice(nv, m, replace=False))
    li = P.layers[0]
    out = torch.empty(2 * qps, 16, 512, device=DEV)
    kw = dict(mode=synth.REUSE, batch=2, q_per_seq=qps, ratio=ratio, max_n=max(lens),
              kv_offsets=P.kv_offsets.to(DEV), q_pos=P.q_pos.to(DEV), codes=codes, scales=scales,
              topk_idx=torch.from_numpy(idx).to(DEV), q=li.q.to(DEV), swa_kv=li.swa.to(DEV),
              out=out, sm_scale=w.sm_scale, q_nvfp4=True)
    ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)))
    csa2.attend(csa2.layer_args(workspace=ws, **kw))
    assert csa2.check_device_status(ws) == 0
    offs = P.kv_offsets.tolist()
    dev = []
    for b in range(2):
        sl = slice(offs[b], offs[b + 1])
        for i in list(range(0, qps, 7)) + [qps - 1]:
            r = b * qps + i
            kw_o = dict(codes=oc[sl], scales=osc[sl], q=bits(li.q[r]), swa=bits(li.swa[b]), topk_in=idx[r],
                        t=w.q_pos[b] + i, t0=w.q_pos[b], ratio=ratio, sm_scale=w.sm_scale)
            _, _, ref = O.csa2_layer(O.REUSE, q_nvfp4=True, **kw_o)
            attention_check(host(out[r]).astype(np.float64), ref, f"seq {b} query {i} (NVFP4 query)")
            if (idx[r] >= 0).any():
                _, _, exact = O.csa2_layer(O.REUSE, **kw_o)
                dev.append(_rel_l2(ref, exact))
    assert max(dev) < 0.15 and np.median(dev) > 1e-4, (min(dev), max(dev))
    print("NVFP4-query variant vs exact, prefill (rel L2): median", np.median(dev), "max", max(dev))


# ---------------------------------------------------------------- whole layers and modes


def _paged(P, codes, scales, page_rows, seed):
    """The same cache in pages of page_rows rows placed in a shuffled order (with unused
    pages between them): returns the physical codes, scales, indexer rows and scales, the
    page table [B][pages] and each sequence's last-position row."""
    rng = np.random.default_rng(seed)
    offs = P.kv_offsets.tolist()
    B = len(P.lens)
    pages = [(n + page_rows - 1) // page_rows for n in P.lens]
    n_phys = sum(pages) + 7                                  # a few pages never used
    perm = rng.permutation(n_phys)
    table = np.zeros((B, max(pages)), np.int32)
    k = 0
    src, dst = [], []
    for b in range(B):
        for j in range(pages[b]):
            table[b, j] = perm[k]
            k += 1
            lo = j * page_rows
            n = min(page_rows, P.lens[b] - lo)
            src.append(torch.arange(offs[b] + lo, offs[b] + lo + n))
            dst.append(torch.arange(int(table[b, j]) * page_rows, int(table[b, j]) * page_rows + n))
    src, dst = torch.cat(src).to(DEV), torch.cat(dst).to(DEV)
    rows = n_phys * page_rows
    out = []
    for t, fill in ((codes, 0xEE), (scales, 0xEE), (P.idx_k.to(DEV), 0xEE), (P.idx_kscale.to(DEV), float("nan"))):
        phys = torch.full((rows,) + tuple(t.shape[1:]), fill, dtype=t.dtype, device=DEV)
        phys[dst] = t[src]
        out.append(phys)
    return (*out, torch.from_numpy(table).to(DEV))


def _run_layers(csa2, synth, P, dev_codes, dev_scales, reuse_cache=False, swa_fp8=False, contig_pool=False,
                paged=None, defer_pool=False, q_nvfp4=False):
    w = P.workload
    B, qps = w.batch, w.q_per_seq
    rows = B * qps
    kv = P.kv_offsets.to(DEV)
    topk = torch.full((rows, 512), -7, dtype=torch.int32, device=DEV)
    pool = torch.full((B, 2048), -7, dtype=torch.int32, device=DEV)
    # the pool's rows gathered contiguously by the Full layer (filled with garbage first)
    pool_k = torch.full((B, 16384, 64), 0xA5, dtype=torch.uint8, device=DEV) if contig_pool else None
    pool_ks = torch.full((B, 16384), float("nan"), dtype=torch.float32, device=DEV) if contig_pool else None
    cache = torch.full((rows, 512, 512), float("nan"), dtype=torch.float16, device=DEV) if reuse_cache else None
    ev_pool = torch.cuda.Event() if defer_pool else None
    res = []
    for li in P.layers:
        out = torch.empty(rows, 16, 512, device=DEV)
        kw = dict(mode=li.mode, batch=B, q_per_seq=qps, ratio=w.ratio, max_n=max(P.lens),
                  kv_offsets=kv, q_pos=None if P.q_pos is None else P.q_pos.to(DEV),
                  codes=dev_codes, scales=dev_scales, topk_idx=topk, q=li.q.to(DEV),
                  swa_kv=None if swa_fp8 else li.swa.to(DEV), out=out, sm_scale=w.sm_scale, pool_blocks=pool,
                  want_pool=(li.mode == synth.FULL and w.want_pool), pool_k=pool_k, pool_kscale=pool_ks,
                  q_nvfp4=q_nvfp4)
        if li.mode != synth.REUSE:
            kw.update(idx_q=li.idx_q.to(DEV), idx_w=li.idx_w.to(DEV), idx_k=P.idx_k.to(DEV),
                      idx_kscale=P.idx_kscale.to(DEV), ev_pool=ev_pool)
        if paged is not None:                                # (codes, scales, idx_k, idx_ks, table, rows)
            pc, ps_, pk, pks, table, page_rows = paged
            kw.update(codes=pc, scales=ps_, page_table=table, page_rows=page_rows, total_n=pc.shape[0])
            if li.mode != synth.REUSE:
                kw.update(idx_k=pk, idx_kscale=pks)
        if swa_fp8:
            s8, ss = synth.fp8_swa(li.swa)
            kw.update(swa_kv8=s8.to(DEV), swa_kscale=ss.to(DEV))
        if cache is not None:
            kw.update(sel_cache=cache,
                      sel_cache_mode=csa2.CACHE_USE if li.mode == synth.REUSE else csa2.CACHE_FILL)
        before = topk.clone()
        ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)))
        csa2.attend(csa2.layer_args(workspace=ws, **kw))
        assert csa2.check_device_status(ws) == 0
        torch.cuda.synchronize()
        if li.mode == synth.REUSE:
            assert host(topk).tobytes() == host(before).tobytes(), "Reuse wrote its indices"
        res.append((host(topk).copy(), host(pool).copy(), host(out).astype(np.float64)))
    return res


def _check_layers(P, oc, osc, res, queries=None, swa_fp8=False, q_nvfp4=False):
    """Runs the oracle layer by layer per sequence/query and checks every output."""
    w = P.workload
    offs = P.kv_offsets.tolist()
    stats = {"tie_swaps": 0}
    for b in range(w.batch):
        sl = slice(offs[b], offs[b + 1])
        view = SeqView(oc, osc, host(P.idx_k), host(P.idx_kscale), offs, b)
        qs = range(w.q_per_seq) if queries is None else queries
        for i in qs:
            r = b * w.q_per_seq + i
            t = None if P.q_pos is None else int(P.q_pos[b]) + i
            o_top = o_pool = None
            for li, (g_top, g_pool, g_out) in zip(P.layers, res):
                if swa_fp8:
                    from fp4_kv_cache_04_b200 import synth as sy
                    s8, ss = sy.fp8_swa(li.swa[b:b + 1])
                    swa_kw = dict(swa=host(s8[0]), swa_scale=host(ss[0]))
                else:
                    swa_kw = dict(swa=bits(li.swa[b]))
                kw = dict(codes=oc[sl], scales=osc[sl], idx_k=view.idx_k, idx_kscale=view.idx_kscale,
                          q=bits(li.q[r]), **swa_kw, ratio=w.ratio, t=t,
                          t0=None if t is None else int(P.q_pos[b]), sm_scale=w.sm_scale, q_nvfp4=q_nvfp4)
                if li.mode != O.REUSE:
                    kw.update(idx_q=bits(li.idx_q[r]), idx_w=li.idx_w[r].numpy().astype(np.float64))
                new_top, pool_b, o_out = O.csa2_layer(
                    li.mode, topk_in=o_top, pool_in=o_pool,
                    want_pool=(li.mode == O.FULL and w.want_pool), **kw)
                if li.mode == O.FULL and w.want_pool:
                    bs = O.block_scores(oracle_scores(view, kw["idx_q"], kw["idx_w"], np.arange(view.n)))
                    kth = np.sort(bs)[::-1][min(2048, bs.size) - 1]
                    stats["tie_swaps"] += topk_tie_check(g_pool[b], pool_b, lambda p: bs[p], kth,
                                                         f"pool seq {b}")
                    o_pool = g_pool[b].copy()          # later layers use the GPU's validated pool
                if li.mode != O.REUSE:
                    cand = (np.arange(O.visible_main(t, w.ratio, view.n)) if li.mode == O.FULL
                            else O.pool_positions(o_pool, view.n))
                    sc = oracle_scores(view, kw["idx_q"], kw["idx_w"], cand)
                    lookup = dict(zip(cand.tolist(), sc.tolist()))
                    kth = np.sort(sc)[::-1][min(512, sc.size) - 1] if sc.size else 0.0
                    d = topk_tie_check(g_top[r], new_top, lambda p: lookup[p], kth, f"topk row {r}")
                    stats["tie_swaps"] += d
                    if d:                              # a tie-band swap: attend with the GPU's indices
                        _, _, o_out = O.csa2_layer(O.REUSE, topk_in=g_top[r], **kw)
                else:
                    assert np.array_equal(g_top[r], o_top), f"row {r}: Reuse changed the indices"
                o_top = g_top[r].copy()
                attention_check(g_out[r], o_out, f"row {r} mode {li.mode}")
    return stats


@pytest.mark.parametrize("contig_pool", [False, True], ids=["scattered_pool", "contiguous_pool"])
def test_decoder_group_full_reuse_reindex(csa2, synth, contig_pool):
    modes = [synth.FULL, synth.REUSE, synth.REUSE, synth.REINDEX, synth.REUSE, synth.REINDEX]
    w = synth.Workload("t", 400, 3, [40000, 9000, 16385], None, 1, modes, want_pool=True)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    res = _run_layers(csa2, synth, P, codes, scales, contig_pool=contig_pool)
    _check_layers(P, *oracle_fp4(P.latent), res)


def test_decoder_group_nvfp4_query(csa2, synth):
    """The NVFP4-query variant through a decoder group (Full + pool, Reuse, Reindex) over a
    paged cache: every layer's selection and the variant's attention against the oracle."""
    modes = [synth.FULL, synth.REUSE, synth.REINDEX, synth.REUSE]
    w = synth.Workload("t", 403, 3, [40000, 9000, 16385], None, 1, modes, want_pool=True)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    res = _run_layers(csa2, synth, P, codes, scales, contig_pool=True,
                      paged=_paged(P, codes, scales, 256, 403) + (256,), q_nvfp4=True)
    _check_layers(P, *oracle_fp4(P.latent), res, q_nvfp4=True)


@pytest.mark.parametrize("contig_pool", [False, True], ids=["scattered_pool", "contiguous_pool"])
def test_deferred_pool_join_matches_joined(csa2, synth, contig_pool):
    """ev_pool: the Full layer's pool select and pool-row gather joined by the first Reindex
    layer instead of at the end of the Full call give the same pool, Top-512 and outputs."""
    modes = [synth.FULL, synth.REUSE, synth.REUSE, synth.REINDEX, synth.REUSE, synth.REINDEX]
    w = synth.Workload("t", 401, 3, [40000, 9000, 16385], None, 1, modes, want_pool=True)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    a = _run_layers(csa2, synth, P, codes, scales, contig_pool=contig_pool)
    b = _run_layers(csa2, synth, P, codes, scales, contig_pool=contig_pool, defer_pool=True)
    for i, (x, y) in enumerate(zip(a, b)):
        for u, v in zip(x, y):
            assert np.array_equal(u, v), f"layer {i}"


def test_deferred_pool_join_in_a_cuda_graph(csa2, synth):
    """The deferred join inside a stream capture: a decoder group (Full + pool, Reuse,
    Reindex, Reuse, Reindex) captured with ev_pool and replayed twice equals its eager run."""
    modes = [synth.FULL, synth.REUSE, synth.REINDEX, synth.REUSE, synth.REINDEX]
    w = synth.Workload("t", 402, 4, [30000, 20000, 9000, 70000], None, 1, modes, want_pool=True)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    B = w.batch
    kv = P.kv_offsets.to(DEV)
    topk = torch.full((B, 512), -1, dtype=torch.int32, device=DEV)
    pool = torch.full((B, 2048), -1, dtype=torch.int32, device=DEV)
    pool_k = torch.zeros(B, 16384, 64, dtype=torch.uint8, device=DEV)
    pool_ks = torch.zeros(B, 16384, dtype=torch.float32, device=DEV)
    outs = [torch.empty(B, 16, 512, device=DEV) for _ in modes]
    ev_pool = torch.cuda.Event()

    def make(defer):
        args = []
        for li, out in zip(P.layers, outs):
            kw = dict(mode=li.mode, batch=B, q_per_seq=1, max_n=max(P.lens), kv_offsets=kv, codes=codes,
                      scales=scales, topk_idx=topk, q=li.q.to(DEV), swa_kv=li.swa.to(DEV), out=out,
                      pool_blocks=pool, want_pool=li.mode == synth.FULL, pool_k=pool_k, pool_kscale=pool_ks)
            if li.mode != synth.REUSE:
                kw.update(idx_q=li.idx_q.to(DEV), idx_w=li.idx_w.to(DEV), idx_k=P.idx_k.to(DEV),
                          idx_kscale=P.idx_kscale.to(DEV), ev_pool=ev_pool if defer else None)
            ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)))
            args.append((csa2.layer_args(workspace=ws, **kw), ws, kw))   # kw keeps the inputs alive
        return args

    ref_args = make(False)
    for a_, _, _ in ref_args:
        csa2.attend(a_)
    torch.cuda.synchronize()
    ref = [host(o).copy() for o in outs] + [host(topk).copy(), host(pool).copy()]
    g_args = make(True)
    for a_, _, _ in g_args:                                     # eager once (creates the side stream)
        csa2.attend(a_)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for a_, _, _ in g_args:
            csa2.attend(a_)
    for _ in range(2):
        for o in outs:
            o.fill_(float("nan"))
        topk.fill_(-3)
        graph.replay()
        torch.cuda.synchronize()
        got = [host(o).copy() for o in outs] + [host(topk).copy(), host(pool).copy()]
        for i, (x, y) in enumerate(zip(ref, got)):
            assert np.array_equal(x, y), f"item {i}"
    for _, ws, _ in g_args:
        assert csa2.check_device_status(ws) == 0


@pytest.mark.parametrize("contig_pool", [False, True], ids=["scattered_pool", "contiguous_pool"])
def test_paged_cache_matches_packed_cache(csa2, synth, contig_pool):
    """A cache in shuffled pages of 256 rows (page table) gives the packed cache's pool,
    Top-512 and outputs bit for bit through Full (+ pool), Reuse and Reindex layers."""
    modes = [synth.FULL, synth.REUSE, synth.REINDEX, synth.REUSE]
    w = synth.Workload("t", 405, 3, [40000, 9000, 16385], None, 1, modes, want_pool=True)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    packed = _run_layers(csa2, synth, P, codes, scales, contig_pool=contig_pool)
    paged = _run_layers(csa2, synth, P, codes, scales, contig_pool=contig_pool,
                        paged=(*_paged(P, codes, scales, 256, 7), 256))
    for i, ((t1, p1, o1), (t2, p2, o2)) in enumerate(zip(packed, paged)):
        assert np.array_equal(t1, t2), f"layer {i}: Top-512"
        assert np.array_equal(p1, p2), f"layer {i}: pool"
        assert np.array_equal(o1, o2), f"layer {i}: output"
    _check_layers(P, *oracle_fp4(P.latent), paged)


def test_paged_cache_prefill_matches_packed_cache(csa2, synth):
    modes = [synth.FULL, synth.REUSE]
    w = synth.Workload("t", 415, 2, [1500, 900], None, 2, modes, q_per_seq=64, q_pos=[0, 1700],
                       q_std=1.0, sm_scale=1 / math.sqrt(512), swa_rows=64 + 127)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent, 2)
    packed = _run_layers(csa2, synth, P, codes, scales)
    paged = _run_layers(csa2, synth, P, codes, scales, paged=(*_paged(P, codes, scales, 128, 9), 128))
    for i, ((t1, _, o1), (t2, _, o2)) in enumerate(zip(packed, paged)):
        assert np.array_equal(t1, t2), f"layer {i}: Top-512"
        assert np.array_equal(o1, o2), f"layer {i}: output"


def test_paged_cache_rejects_bad_pages(csa2, synth):
    w = synth.Workload("t", 425, 1, [1000], None, 1, [synth.REUSE])
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    out = torch.empty(1, 16, 512, device=DEV)
    table = torch.zeros(1, 8, dtype=torch.int32, device=DEV)
    base = dict(mode=synth.REUSE, batch=1, q_per_seq=1, max_n=1000, kv_offsets=P.kv_offsets.to(DEV),
                codes=codes, scales=scales, topk_idx=torch.full((1, 512), -1, dtype=torch.int32, device=DEV),
                q=P.layers[0].q.to(DEV), swa_kv=P.layers[0].swa.to(DEV), out=out, page_table=table)
    ws = csa2.alloc_workspace(1 << 20)
    for rows in (0, 64, 200):                                 # not a multiple of 128
        assert csa2.attend_status(csa2.layer_args(workspace=ws, page_rows=rows, **base)) == 1
    small = dict(base, page_table=torch.zeros(1, 3, dtype=torch.int32, device=DEV))   # 3 x 128 < 1000
    assert csa2.attend_status(csa2.layer_args(workspace=ws, page_rows=128, **small)) == 1
    assert csa2.attend_status(csa2.layer_args(workspace=ws, page_rows=128, **base)) == 0


def test_decoder_group_fp8_swa(csa2, synth):
    # the FP8 SWA variant through Full, Reuse (with the reuse cache) and Reindex layers
    modes = [synth.FULL, synth.REUSE, synth.REINDEX, synth.REUSE]
    w = synth.Workload("t", 440, 3, [30000, 700, 9001], None, 1, modes, want_pool=True)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    res = _run_layers(csa2, synth, P, codes, scales, reuse_cache=True, swa_fp8=True)
    _check_layers(P, *oracle_fp4(P.latent), res, swa_fp8=True)


def test_decoder_group_with_reuse_cache(csa2, synth):
    # decode calls take the reuse-cache arguments (CSA2_CACHE_FILL / USE) but neither write
    # nor read the cache: they re-gather the FP4 rows; the results equal the run without
    modes = [synth.FULL, synth.REUSE, synth.REUSE, synth.REINDEX, synth.REUSE]
    w = synth.Workload("t", 430, 3, [20000, 700, 9001], None, 1, modes, want_pool=True)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    res = _run_layers(csa2, synth, P, codes, scales, reuse_cache=True)
    _check_layers(P, *oracle_fp4(P.latent), res)
    res_plain = _run_layers(csa2, synth, P, codes, scales, reuse_cache=False)
    for (t1, _, o1), (t2, _, o2) in zip(res, res_plain):
        assert np.array_equal(t1, t2)
        assert np.array_equal(o1, o2)


def test_decoder_group_one_cta_per_sequence(csa2, synth):
    # B = 296 fills both CTA slots of every SM with one CTA per row (a tie on the critical
    # path that the split breaks toward fewer CTAs), so each row's 12 key tiles run on one
    # CTA: a cluster of one, merging with itself
    modes = [synth.FULL, synth.REUSE]
    lens = [200 + 13 * (i % 120) for i in range(296)]
    w = synth.Workload("t", 480, 296, lens, None, 1, modes, want_pool=False)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    res = _run_layers(csa2, synth, P, codes, scales)
    _check_layers(P, *oracle_fp4(P.latent), res)


@pytest.mark.parametrize("pattern", ["ties3", "ties8", "outlier"])
def test_decoder_group_select_paths(csa2, synth, pattern):
    # indexer keys that steer the scan's chunk Top-512 down each of its paths: 3 distinct
    # key rows (a third of every chunk ties at the top: too many survivors, radix
    # fallback), 8 distinct rows (the survivors all share one score: the boundary bin is a
    # single value), and a few rows with a 1000x scale (every other survivor falls into one
    # histogram bin: crowded-bin fallback)
    modes = [synth.FULL, synth.REUSE, synth.REINDEX, synth.REUSE]
    w = synth.Workload("t", 470, 2, [40000, 12289], None, 1, modes, want_pool=True)
    P = synth.make_problem(w, device="cpu")
    rng = np.random.default_rng(471)
    n = P.idx_k.shape[0]
    if pattern.startswith("ties"):
        groups = int(pattern[4:])
        base = P.idx_k[:groups].clone()
        P.idx_k[:] = base[torch.from_numpy(rng.integers(0, groups, n))]
        P.idx_kscale[:] = P.idx_kscale[0]
    else:
        P.idx_kscale[torch.from_numpy(rng.choice(n, 16, replace=False))] *= 1000.0
    codes, scales = _cache(csa2, P.latent)
    res = _run_layers(csa2, synth, P, codes, scales)
    stats = _check_layers(P, *oracle_fp4(P.latent), res)
    if pattern.startswith("ties"):
        assert stats["tie_swaps"] == 0          # exact ties: both sides keep the lowest positions


@pytest.mark.parametrize("lens", [[1, 7, 511, 8193], [8192, 16], [100003], [16384 * 8 + 5, 3000]])
def test_decoder_group_edges(csa2, synth, lens):
    modes = [synth.FULL, synth.REUSE, synth.REINDEX, synth.REUSE]
    w = synth.Workload("t", 401 + len(lens), len(lens), lens, None, 1, modes, want_pool=True)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    res = _run_layers(csa2, synth, P, codes, scales)
    _check_layers(P, *oracle_fp4(P.latent), res)


def test_prefill_full_reuse_causal(csa2, synth):
    modes = [synth.FULL, synth.REUSE, synth.REUSE]
    w = synth.Workload("t", 410, 2, [1500, 900], None, 2, modes, q_per_seq=64, q_pos=[0, 1700],
                       q_std=1.0, sm_scale=1 / math.sqrt(512), swa_rows=64 + 127)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent, 2)
    res = _run_layers(csa2, synth, P, codes, scales)
    _check_layers(P, *oracle_fp4(P.latent, 2), res)


def test_prefill_with_reuse_cache(csa2, synth):
    # prefill (many causal queries per sequence): Reuse layers read the rows the Full layer
    # dequantised (CSA2_CACHE_USE); the results equal the run without the cache, bit for bit
    modes = [synth.FULL, synth.REUSE, synth.REUSE]
    w = synth.Workload("t", 412, 2, [1500, 900], None, 2, modes, q_per_seq=64, q_pos=[0, 1700],
                       q_std=1.0, sm_scale=1 / math.sqrt(512), swa_rows=64 + 127)
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent, 2)
    res = _run_layers(csa2, synth, P, codes, scales, reuse_cache=True)
    _check_layers(P, *oracle_fp4(P.latent, 2), res, queries=range(0, 64, 9))
    res_plain = _run_layers(csa2, synth, P, codes, scales, reuse_cache=False)
    for (t1, _, o1), (t2, _, o2) in zip(res, res_plain):
        assert np.array_equal(t1, t2)
        assert np.array_equal(o1, o2)            # the cache holds exactly the dequantised rows


def test_reuse_out_of_range_index_sets_device_error(csa2, synth):
    w = synth.Workload("t", 420, 1, [100], None, 1, [synth.REUSE])
    P = synth.make_problem(w, device="cpu")
    codes, scales = _cache(csa2, P.latent)
    idx = torch.full((1, 512), -1, dtype=torch.int32)
    idx[0, :3] = torch.tensor([1, 50, 100])            # 100 is past the context
    li = P.layers[0]
    out = torch.empty(1, 16, 512, device=DEV)
    kw = dict(mode=synth.REUSE, batch=1, q_per_seq=1, max_n=100, kv_offsets=P.kv_offsets.to(DEV),
              codes=codes, scales=scales, topk_idx=idx.to(DEV), q=li.q.to(DEV),
              swa_kv=li.swa.to(DEV), out=out)
    ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)))
    csa2.attend(csa2.layer_args(workspace=ws, **kw))
    assert csa2.check_device_status(ws) == 6
    assert csa2.check_device_status(ws) == 0            # read-and-clear
    oc, osc = oracle_fp4(P.latent)
    _, _, ref = O.csa2_layer(O.REUSE, codes=oc, scales=osc, q=bits(li.q[0]),
                             swa=bits(li.swa[0]), topk_in=np.array([1, 50] + [-1] * 510, np.int32))
    attention_check(host(out[0]), ref, "skipping the bad index")
