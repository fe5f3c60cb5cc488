"""The bounded-wait failure path, driven on purpose without faulting or hanging the GPU.

csa2_set_wait_limit lowers the bound of every pipelined device-side wait to one
non-blocking poll, so the first wait of the indexer pipelines (the tensor-core warp polling
the first TMA tile right after it is issued) gives up while the copies are in flight.
Each kernel then records CSA2_ERR_TIMEOUT, waits with the library's default bound for
the copies and MMAs it had already issued, frees its tensor memory and returns.  The
test checks the error word, then restores the default bound and requires that the same
workspace gives CSA2_OK and results equal to the float64 oracle: the context is intact.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import csa2_oracle as O
from tests.helpers import attention_check, bits, host, oracle_fp4, topk_tie_check

pytestmark = pytest.mark.gpu

DEV = "cuda"
TIMEOUT = 5


@pytest.fixture(scope="module")
def lib():
    from __graft_entry__ import build
    build()
    from fp4_kv_cache_04_b200 import csa2, synth
    return csa2, synth


def _call_twice(csa2, args, ws, must_time_out=True):
    """One call with a 1-poll bound, then one with the default bound.  A scan or prefill
    indexer call must time out: its tensor-core warp polls the first tile right after the
    load is issued.  An attention-only call may not (its first waits come after the index
    reads, when the data has often landed), so either status is accepted there."""
    csa2.set_wait_limit(ws, 1)
    csa2.attend(args)
    st = csa2.check_device_status(ws)
    assert st == TIMEOUT if must_time_out else st in (0, TIMEOUT)
    csa2.set_wait_limit(ws, 0)
    csa2.attend(args)
    assert csa2.check_device_status(ws) == 0


def test_decode_layers_time_out_and_recover(lib):
    csa2, synth = lib
    modes = [synth.FULL, synth.REUSE, synth.REINDEX]
    w = synth.Workload("t", 900, 2, [20000, 1501], None, 1, modes, want_pool=True)
    P = synth.make_problem(w, device="cpu")
    total = sum(P.lens)
    codes = torch.empty(total, 256, dtype=torch.uint8, device=DEV)
    scales = torch.empty(total, 32, dtype=torch.uint8, device=DEV)
    csa2.quantize_kv(P.latent.to(DEV), 1, codes, scales)
    kv = P.kv_offsets.to(DEV)
    idx_k, ks = P.idx_k.to(DEV), P.idx_kscale.to(DEV)
    topk = torch.full((2, 512), -1, dtype=torch.int32, device=DEV)
    pool = torch.full((2, 2048), -1, dtype=torch.int32, device=DEV)
    outs, tops, pools = [], [], []
    for li in P.layers:
        out = torch.empty(2, 16, 512, dtype=torch.float32, device=DEV)
        kw = dict(mode=li.mode, batch=2, q_per_seq=1, max_n=max(P.lens), kv_offsets=kv, codes=codes,
                  scales=scales, topk_idx=topk, q=li.q.to(DEV), swa_kv=li.swa.to(DEV), out=out,
                  pool_blocks=pool, want_pool=li.mode == synth.FULL)
        if li.mode != synth.REUSE:
            kw.update(idx_q=li.idx_q.to(DEV), idx_w=li.idx_w.to(DEV), idx_k=idx_k, idx_kscale=ks)
        ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)))
        _call_twice(csa2, csa2.layer_args(workspace=ws, **kw), ws, must_time_out=li.mode != synth.REUSE)
        outs.append(host(out).astype(np.float64))
        tops.append(host(topk).copy())
        pools.append(host(pool).copy())

    oc, osc = oracle_fp4(P.latent)
    offs = P.kv_offsets.tolist()
    for b in range(2):
        sl = slice(offs[b], offs[b + 1])
        k8, k8s = P.idx_k[sl].numpy(), P.idx_kscale[sl].numpy()
        keys = O.indexer_keys(k8, k8s)
        o_top = o_pool = None
        for i, li in enumerate(P.layers):
            kw = dict(codes=oc[sl], scales=osc[sl], idx_k=k8, idx_kscale=k8s, q=bits(li.q[b]),
                      swa=bits(li.swa[b]))
            if li.mode != synth.REUSE:
                kw.update(idx_q=bits(li.idx_q[b]), idx_w=li.idx_w[b].numpy().astype(np.float64))
            new_top, pool_b, ref = O.csa2_layer(li.mode, topk_in=o_top, pool_in=o_pool,
                                                want_pool=li.mode == synth.FULL, **kw)
            if li.mode != synth.REUSE:
                sc = O.index_scores(kw["idx_q"], kw["idx_w"], keys)
                if li.mode == synth.FULL:
                    bs = O.block_scores(sc)
                    kth = np.sort(bs)[::-1][min(2048, bs.size) - 1]
                    topk_tie_check(pools[i][b], pool_b, lambda p: bs[p], kth, f"pool seq {b}")
                    o_pool = pools[i][b].copy()
                cand = np.arange(sc.size) if li.mode == synth.FULL else O.pool_positions(o_pool, sc.size)
                kth = np.sort(sc[cand])[::-1][min(512, cand.size) - 1]
                if topk_tie_check(tops[i][b], new_top, lambda p: sc[p], kth, f"layer {i} seq {b}"):
                    _, _, ref = O.csa2_layer(O.REUSE, topk_in=tops[i][b], **kw)
            o_top = tops[i][b].copy()
            attention_check(outs[i][b], ref, f"layer {i} seq {b} after a timed-out call")


def test_prefill_indexer_times_out_and_recovers(lib):
    csa2, synth = lib
    w = synth.Workload("t", 910, 2, [1500, 900], None, 2, [synth.FULL], q_per_seq=48, q_pos=[0, 1700],
                       q_std=1.0, sm_scale=1 / math.sqrt(512), swa_rows=48 + 127)
    P = synth.make_problem(w, device="cpu")
    total = sum(P.lens)
    codes = torch.empty(total, 256, dtype=torch.uint8, device=DEV)
    scales = torch.empty(total, 32, dtype=torch.uint8, device=DEV)
    csa2.quantize_kv(P.latent.to(DEV), 2, codes, scales)
    li = P.layers[0]
    rows = 2 * 48
    topk = torch.full((rows, 512), -1, dtype=torch.int32, device=DEV)
    out = torch.empty(rows, 16, 512, dtype=torch.float32, device=DEV)
    kw = dict(mode=synth.FULL, batch=2, q_per_seq=48, ratio=2, max_n=max(P.lens),
              kv_offsets=P.kv_offsets.to(DEV), q_pos=P.q_pos.to(DEV), codes=codes, scales=scales,
              topk_idx=topk, q=li.q.to(DEV), swa_kv=li.swa.to(DEV), out=out, sm_scale=w.sm_scale,
              idx_q=li.idx_q.to(DEV), idx_w=li.idx_w.to(DEV), idx_k=P.idx_k.to(DEV),
              idx_kscale=P.idx_kscale.to(DEV))
    ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)))
    _call_twice(csa2, csa2.layer_args(workspace=ws, **kw), ws)

    oc, osc = oracle_fp4(P.latent, 2)
    offs = P.kv_offsets.tolist()
    g_top, g_out = host(topk), host(out).astype(np.float64)
    for b in range(2):
        sl = slice(offs[b], offs[b + 1])
        k8, k8s = P.idx_k[sl].numpy(), P.idx_kscale[sl].numpy()
        keys = O.indexer_keys(k8, k8s)
        q0 = int(P.q_pos[b])
        for i in (0, 1, 17, 47):
            r, t = b * 48 + i, q0 + i
            nv = O.visible_main(t, 2, k8.shape[0])
            kw_o = dict(codes=oc[sl], scales=osc[sl], idx_k=k8, idx_kscale=k8s, q=bits(li.q[r]),
                        swa=bits(li.swa[b]), ratio=2, t=t, t0=q0, sm_scale=w.sm_scale)
            if nv:
                sc = O.index_scores(bits(li.idx_q[r]), li.idx_w[r].numpy().astype(np.float64), keys[:nv])
                o_top = O.topk_select(sc, np.arange(nv), 512)
                kth = np.sort(sc)[::-1][min(512, nv) - 1]
                topk_tie_check(g_top[r], o_top, lambda p: sc[p], kth, f"prefill row {r}")
            else:
                assert (g_top[r] == -1).all()
            _, _, ref = O.csa2_layer(O.REUSE, topk_in=g_top[r], **kw_o)
            attention_check(g_out[r], ref, f"prefill row {r} after a timed-out call")
