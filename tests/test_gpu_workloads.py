"""Full-size decode workloads, in the launch configuration bench.py times, against the
oracle on sampled sequences.

A 20-layer decoder step over 64 sequences of up to 262,144 positions (the headline
workload, and its ragged variant) runs exactly as the bench runs it: one csa2_append_kv
(the new position's FP4 main-KV and FP8 indexer-K rows), then csa2_attend per layer with
the same arguments and workspaces.  The step is
then replayed layer by layer to keep each layer's Top-512 and pool (the replay must
reproduce the first run's outputs bit for bit: the path is deterministic).  For a few
sampled sequences the float64 oracle runs the same schedule on its own quantisation of
the same seeded inputs; every layer's pool, Top-512 (up to the tie band) and attention
output (relative L2 <= 1e-3, max abs <= 5e-3) are compared.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import csa2_oracle as O
from tests.helpers import attention_check, topk_tie_check

pytestmark = pytest.mark.gpu

SAMPLED = (0, 37, 63)


@pytest.fixture(scope="module")
def bench():
    from __graft_entry__ import build
    build()
    import bench as b
    return b


@pytest.mark.parametrize("name", ["decoder_step_256k", "decoder_step_ragged"])
def test_decoder_step_sampled_sequences(bench, name):
    from fp4_kv_cache_04_b200 import synth
    w = synth.workloads()[name]
    step = bench.DecodeStep(w, torch.device("cuda", 0), keep_seqs=SAMPLED)
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
    for i, (o1, o2) in enumerate(zip(first, step.outs)):
        assert torch.equal(o1, o2.cpu()), f"layer {i}: replay differs"

    for b in SAMPLED:
        seq = bench.OracleSeq(step.P, step.latent_host[b], w.want_pool, w.sm_scale, b)
        n = seq.idx_k.shape[0]
        keys = O.indexer_keys(seq.idx_k, seq.idx_kscale)
        top = pool = None
        for i, d in enumerate(seq.layers):
            kw = dict(codes=seq.codes, scales=seq.scales, idx_k=seq.idx_k, idx_kscale=seq.idx_kscale,
                      q=d["q"], swa=d["swa"], sm_scale=seq.sm_scale)
            if "idx_q" in d:
                kw.update(idx_q=d["idx_q"], idx_w=d["idx_w"])
            want = d["mode"] == O.FULL and w.want_pool
            top, pool_i, out = O.csa2_layer(d["mode"], topk_in=top, pool_in=pool, want_pool=want, **kw)
            where = f"{name} seq {b} layer {i}"
            swaps = 0
            if d["mode"] != O.REUSE:
                scores = O.index_scores(d["idx_q"], d["idx_w"], keys)
                if want:
                    bs = O.block_scores(scores)
                    kth = np.sort(bs)[::-1][min(2048, bs.size) - 1]
                    swaps += topk_tie_check(pools[i][b].numpy(), pool_i, lambda p: bs[p], kth, where + " pool")
                    pool = pool_i
                cand = np.arange(n) if d["mode"] == O.FULL else O.pool_positions(pool, n)
                sc = scores[cand]
                kth = np.sort(sc)[::-1][min(512, sc.size) - 1]
                swaps += topk_tie_check(tops[i][b].numpy(), top, lambda p: scores[p], kth, where + " top-512")
            if swaps:
                break                      # a tie-band swap: later layers see other rows
            attention_check(step.outs[i][b].cpu().numpy(), out, where)
