"""Every workload at its own size, in the launch configuration bench.py times, against the
oracle on sampled sequences (decode) or sampled queries (chunked prefill).

Decode workloads (one Full layer at 4,096 positions; Full + 3 Reuse over 8 x 32,768; the
HSI at 1,048,576 positions with 3 Reindex layers; the 20-layer decoder step over 64 x
262,144 positions and its ragged variant) run exactly as the bench runs them: one
csa2_append_kv, then csa2_attend per layer with the same arguments and workspaces.  The
step is replayed layer by layer to keep each layer's Top-512 and pool (the replay must
reproduce the first run bit for bit: the path is deterministic).  For sampled sequences
the float64 oracle runs the same schedule on its own quantisation of the same seeded
inputs; every layer's pool and Top-512 must agree up to the tie band, and every layer's
attention output (relative L2 <= 1e-3, max abs <= 5e-3) is checked.  After a Full or
Reindex layer the oracle carries the GPU's validated pool and Top-512 forward, so a
legitimate tie-band swap never ends the check: the attention of that layer and of every
later layer is computed by the oracle with the indices the GPU used.

The chunked-prefill workload (encoder group Full + 5 Reuse, the last 2,048-token chunk of
a 131,072-token prompt at ratio 2, B = 2) runs the bench's PrefillStep (the chunk's own
tokens quantised into the cache, then the six layers); sampled queries of both sequences
(the first, the last and those between) are checked on every layer.  A first-chunk run
(tokens 0 .. 2,047) checks the causal edges at the same scale.

The whole-prompt workload (a 131,072-token prompt at ratio 2 in 64 chunks of 2,048
tokens, three encoder groups of Full + 5 Reuse per chunk, B = 2) runs the bench's
PromptStep chunk by chunk; sampled queries of the first, second, a middle and the last
chunk are checked on all 18 layers (each group's Reuse layers with the Top-512 of that
group's Full layer), and every query of those chunks selects only what it can see.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import csa2_oracle as O
from tests.helpers import attention_check, topk_tie_check

pytestmark = pytest.mark.gpu

DECODE_SAMPLED = {
    "decode_full_4k": (0,),
    "decoder_group_32k": (0, 3, 7),
    "hsi_1m": (0,),
    "decoder_step_256k": (0, 37, 63),
    "decoder_step_ragged": (0, 37, 63),
}
PREFILL_QUERIES = (0, 1, 2, 127, 128, 300, 511, 777, 1023, 1024, 1301, 1535, 1792, 2000, 2046, 2047)


@pytest.fixture(scope="module")
def bench():
    from __graft_entry__ import build
    build()
    import bench as b
    return b


def check_decode_sequence(bench, step, w, b, tops, pools, outs):
    """Oracle check of every layer of sequence b (GPU state carried after validation)."""
    seq = bench.OracleSeq(step.P, step.latent_host[b], w.want_pool, w.sm_scale, b)
    n = seq.idx_k.shape[0]
    keys = O.indexer_keys(seq.idx_k, seq.idx_kscale)
    top = pool = None
    total_swaps = 0
    for i, d in enumerate(seq.layers):
        kw = dict(codes=seq.codes, scales=seq.scales, idx_k=seq.idx_k, idx_kscale=seq.idx_kscale,
                  q=d["q"], swa=d["swa"], sm_scale=seq.sm_scale)
        if "idx_q" in d:
            kw.update(idx_q=d["idx_q"], idx_w=d["idx_w"])
        want = d["mode"] == O.FULL and w.want_pool
        where = f"{w.name} seq {b} layer {i}"
        g_top = tops[i][b].numpy()
        o_top, o_pool, out = O.csa2_layer(d["mode"], topk_in=top, pool_in=pool, want_pool=want, **kw)
        if d["mode"] == O.REUSE:
            assert np.array_equal(g_top, top), f"{where}: Reuse changed the indices"
        else:
            scores = O.index_scores(d["idx_q"], d["idx_w"], keys)
            if want:
                bs = O.block_scores(scores)
                kth = np.sort(bs)[::-1][min(2048, bs.size) - 1]
                total_swaps += topk_tie_check(pools[i][b].numpy(), o_pool, lambda p: bs[p], kth,
                                              where + " pool")
                pool = pools[i][b].numpy().copy()        # the GPU's pool, validated
            # the candidates of this layer: every position, or the (GPU's) pool's positions
            cand = np.arange(n) if d["mode"] == O.FULL else O.pool_positions(pool, n)
            sc = scores[cand]
            kth = np.sort(sc)[::-1][min(512, sc.size) - 1]
            swaps = topk_tie_check(g_top, o_top, lambda p: scores[p], kth, where + " top-512")
            total_swaps += swaps
            if swaps:                                  # attend with the indices the GPU used
                _, _, out = O.csa2_layer(O.REUSE, topk_in=g_top, **kw)
        top = g_top.copy()
        attention_check(outs[i][b], out, where)
    return total_swaps


@pytest.mark.parametrize("name", list(DECODE_SAMPLED))
def test_decode_workload_sampled_sequences(bench, name):
    from fp4_kv_cache_04_b200 import synth
    w = synth.workloads()[name]
    sampled = DECODE_SAMPLED[name]
    step = bench.DecodeStep(w, torch.device("cuda", 0), keep_seqs=sampled)
    step.run()
    torch.cuda.synchronize()
    assert all(s == 0 for s in step.check_status())
    first = [o.cpu().clone() for o in step.outs]

    c = step.csa2
    c.append_kv(step.new_rows, step.new_proj, step.dst_row, step.codes, step.scales, step.P.idx_k,
                step.P.idx_kscale)
    tops, pools = [], []
    for _, a in step.args:
        c.attend(a)
        tops.append(step.topk.cpu().clone())
        pools.append(step.pool.cpu().clone())
    torch.cuda.synchronize()
    assert all(s == 0 for s in step.check_status())
    for i, (o1, o2) in enumerate(zip(first, step.outs)):
        assert torch.equal(o1, o2.cpu()), f"layer {i}: replay differs"
    outs = [o.numpy() for o in first]
    for b in sampled:
        check_decode_sequence(bench, step, w, b, tops, pools, outs)


def _prefill_check(bench, step, b, queries, ch=None, q0=None, tops=None, outs=None):
    """Every layer of the sampled queries of sequence b against the oracle: each Full
    layer's Top-512 up to the tie band, then each layer's attention with the indices the
    GPU used (the same as the oracle's unless a tie-band swap happened).  tops[layer] /
    outs[layer] (GPU rows of the sampled queries, in order) replace the step's buffers
    when a whole prompt ran; q0 is then the chunk's first token."""
    w = step.w
    ch = ch or bench.OracleChunk(step.P, step.latent_host[b], b)
    q0 = ch.q0 if q0 is None else q0
    keys = O.indexer_keys(ch.idx_k, ch.idx_kscale)
    topk = step.topk.cpu().numpy() if tops is None else None
    for j, i in enumerate(queries):
        r = b * step.Q + i
        t = q0 + i
        nv = O.visible_main(t, w.ratio, ch.idx_k.shape[0])
        for li_i, li in enumerate(step.P.layers):
            if li.mode == O.FULL:
                g_top = topk[r] if tops is None else tops[li_i][j]
            g_out = step.outs[li_i][r].cpu().numpy() if outs is None else outs[li_i][j]
            d = ch._layer(li_i, i)
            kw = dict(codes=ch.codes, scales=ch.scales, idx_k=ch.idx_k, idx_kscale=ch.idx_kscale,
                      q=d["q"], swa=d["swa"], sm_scale=w.sm_scale, ratio=w.ratio, t=t, t0=q0)
            where = f"prefill seq {b} query {i} (token {t}) layer {li_i}"
            if li.mode == O.FULL and nv == 0:          # token 0 at ratio 2 sees no position
                assert (g_top == -1).all(), where
            elif li.mode == O.FULL:
                scores = O.index_scores(d["idx_q"], d["idx_w"], keys[:nv])
                o_top = O.topk_select(scores, np.arange(nv), 512)
                kth = np.sort(scores)[::-1][min(512, nv) - 1]
                topk_tie_check(g_top, o_top, lambda p: scores[p], kth, where + " top-512")
            _, _, out = O.csa2_layer(O.REUSE, topk_in=g_top, **kw)
            attention_check(g_out, out, where)


@pytest.mark.parametrize("first_chunk", [False, True], ids=["last_chunk", "first_chunk"])
def test_prefill_chunk_sampled_queries(bench, first_chunk):
    from fp4_kv_cache_04_b200 import synth
    w = synth.workloads()["prefill_chunk_128k"]
    if first_chunk:
        w = synth.Workload(**{**w.__dict__, "q_pos": [0] * w.batch})
    step = bench.PrefillStep(w, torch.device("cuda", 0), keep_seqs=(0, 1))
    step.run()
    torch.cuda.synchronize()
    assert all(s == 0 for s in step.check_status())
    rows = [b * step.Q + i for b in range(step.B) for i in PREFILL_QUERIES]
    first = [o[rows].cpu().clone() for o in step.outs]
    top_first = step.topk.cpu().clone()
    step.run()                                         # the step is deterministic
    torch.cuda.synchronize()
    assert torch.equal(top_first, step.topk.cpu())
    for i, o in enumerate(step.outs):
        assert torch.equal(first[i], o[rows].cpu()), f"layer {i}: replay differs"
    # causal: no query selects a position it cannot see
    topk = step.topk.cpu().numpy()
    for b in range(step.B):
        vis = np.array(step.visible(b))
        tb = topk[b * step.Q:(b + 1) * step.Q]
        assert ((tb < vis[:, None]) | (tb == -1)).all()
        assert ((tb >= 0).sum(axis=1) == np.minimum(vis, 512)).all()
    for b in range(step.B):
        _prefill_check(bench, step, b, PREFILL_QUERIES)


PROMPT_CHUNKS = (0, 1, 31, 63)
PROMPT_QUERIES = (0, 1, 2, 127, 1023, 1024, 2046, 2047)


def test_prefill_prompt_sampled_queries(bench):
    """The whole prompt, chunk by chunk, as the bench's step runs it."""
    from fp4_kv_cache_04_b200 import synth
    w = synth.workloads()["prefill_prompt_128k"]
    step = bench.PromptStep(w, torch.device("cuda", 0), keep_seqs=(0, 1))
    assert step.n_chunks == 64 and len(step.P.layers) == 18
    rows = [b * step.Q + i for b in range(step.B) for i in PROMPT_QUERIES]
    snap = {}
    for c in range(step.n_chunks):
        if c not in PROMPT_CHUNKS:
            step.run_chunk(c)
            continue
        tops, outs = {}, {}

        def grab(li, tops=tops, outs=outs):
            outs[li] = step.outs[li][rows].cpu().numpy()
            if step.P.layers[li].mode == synth.FULL:
                tops[li] = step.topk.cpu().numpy()
        step.run_chunk(c, on_layer=grab)
        snap[c] = (tops, outs)
    torch.cuda.synchronize()
    assert all(s_ == 0 for s_ in step.check_status())
    chs = {b: bench.OracleChunk(step.P, step.latent_host[b], b) for b in range(step.B)}
    for c, (tops, outs) in snap.items():
        for li, tk in tops.items():                 # causal: nothing beyond what a query sees
            for b in range(step.B):
                vis = np.array(step.visible(b, c))
                tb = tk[b * step.Q:(b + 1) * step.Q]
                assert ((tb < vis[:, None]) | (tb == -1)).all(), f"chunk {c} layer {li}"
                assert ((tb >= 0).sum(axis=1) == np.minimum(vis, 512)).all(), f"chunk {c} layer {li}"
        n_q = len(PROMPT_QUERIES)
        for b in range(step.B):
            sel = [b * step.Q + i for i in PROMPT_QUERIES]
            t_b = {li: tk[sel] for li, tk in tops.items()}
            t_full = {}
            cur = None
            for li in range(len(step.P.layers)):      # each layer sees its group's Top-512
                cur = t_b.get(li, cur)
                t_full[li] = cur
            o_b = {li: o[b * n_q:(b + 1) * n_q] for li, o in outs.items()}
            _prefill_check(bench, step, b, PROMPT_QUERIES, ch=chs[b], q0=c * step.Q,
                           tops=t_full, outs=o_b)
