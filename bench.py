#!/usr/bin/env python
"""Benchmark of the CSA2-over-FP4-KV decode step.

Metric: CSA2 decode queries/s at 256K context (one query = one sequence's full 20-layer
decoder step: the cache append of its new latent row, the Full layer's indexer scan,
Top-512 and HSI pool, four Reindex layers over the 16,384-position pool, and 20
sparse attentions over 512 FP4 rows + 128 SWA rows), plus the achieved HBM bandwidth
of the dominant kernel (the Full layer's indexer scan) against the measured peak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Multi-GPU: one process per GPU (torchrun); every rank runs its own batch of 64
sequences (data parallel over sequences, no collective on the data path), so the work
scales weakly; timing is the max over ranks.  `--impl reference` times the float64
oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA2 decode queries/s at 256K ctx; achieved HBM GB/s as % of roofline"
HBM_FALLBACK_GBS = 6650.0

IDX_ROW_BYTES = 64 + 4          # FP8 indexer-K row + fp32 scale
MAIN_ROW_BYTES = 256 + 32       # E2M1 codes + E4M3 scales
SWA_ROW_BYTES = 512 * 2
Q_BYTES = 16 * 512 * 2
OUT_BYTES = 16 * 512 * 4
IDXQW_BYTES = 4 * 64 * 2 + 4 * 4
POOL_POS = 16384


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 300 for decode workloads, 50 for a prefill chunk, "
                         "3 for a whole prompt)")
    ap.add_argument("--warmup", type=int, default=None,
                    help="untimed warm-up steps (default: 10; 3 for a whole prompt)")
    ap.add_argument("--workload", default="decoder_step_256k")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (profiling captures on a smaller case)")
    ap.add_argument("--context", type=int, default=None,
                    help="override every sequence's context length (profiling captures)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="budget of the oracle CPU-baseline sample (N=1, rank 0)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--reuse-cache", action="store_true",
                    help="pass the f16 cross-layer reuse cache (decode calls do not use it: they "
                         "re-gather the FP4 rows and convert them in registers)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--swa-fp8", action="store_true",
                    help="the FP8 SWA KV variant (E4M3 rows with one fp32 scale each)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps one by one instead of replaying one CUDA graph")
    ap.add_argument("--join-pool", action="store_true",
                    help="join the Full layer's pool select at the end of its call instead of "
                         "at the first Reindex layer")
    ap.add_argument("--q-nvfp4", action="store_true",
                    help="the block-scaled FP4 query variant: main-row logits from the query "
                         "quantised to NVFP4 on the FP4 tensor cores (not the exact method)")
    ap.add_argument("--paged", type=int, default=0, metavar="ROWS",
                    help="keep the cache in pages of ROWS rows (a multiple of 128) placed in a "
                         "shuffled order, addressed through a page table")
    ap.add_argument("--scattered-pool", action="store_true",
                    help="Reindex layers gather each 8-row pool block from the indexer cache instead "
                         "of streaming the pool's rows gathered contiguously by the Full layer")
    args = ap.parse_args(argv)
    prompt = args.workload.startswith("prefill_prompt")
    chunk = args.workload.startswith("prefill_chunk")
    if args.steps is None:
        args.steps = 3 if prompt else 50 if chunk else 300
    if args.warmup is None:
        args.warmup = 3 if prompt else 10
    return args


# ------------------------------------------------------------------ accounting


def algorithmic_bytes_per_seq(n: int, modes: list[int], swa_row_bytes: int = SWA_ROW_BYTES) -> int:
    """Unique bytes one sequence's decode step must move (each byte counted once):
    indexer scan of the Full layer, the pool's indexer rows once for all Reindex
    layers, each distinct Top-512 selection's FP4 rows once, every layer's SWA rows,
    q and fp32 output, the indexer q/w, and the appended position (bf16 latent and fp32
    indexer values in, FP4 main-KV and FP8 indexer rows out)."""
    n_full = sum(1 for m in modes if m == 0)
    n_reindex = sum(1 for m in modes if m == 1)
    scan = n_full * n * IDX_ROW_BYTES
    pool = (min(POOL_POS, n) * IDX_ROW_BYTES) if n_reindex else 0
    selections = (n_full + n_reindex) * 512 * MAIN_ROW_BYTES
    per_layer = len(modes) * (128 * swa_row_bytes + Q_BYTES + OUT_BYTES)
    idx_qw = (n_full + n_reindex) * IDXQW_BYTES
    append = 512 * 2 + MAIN_ROW_BYTES + 64 * 4 + IDX_ROW_BYTES
    return scan + pool + selections + per_layer + idx_qw + append


PREFILL_METRIC = ("CSA2 chunked-prefill tokens/s (encoder group Full + 5 Reuse, 2,048-token chunk "
                  "over 65,536 ratio-2 positions); attention + indexer TFLOP/s vs tensor peak")
PROMPT_METRIC = ("CSA2 whole-prompt encoder prefill tokens/s (131,072-token prompt in 2,048-token "
                 "chunks, 3 x (Full + 5 Reuse) per chunk); attention + indexer TFLOP/s vs tensor peak")
PREFILL_INDEX_FLOPS_PER_POS = 2 * 4 * 64        # one query against one visible position
PREFILL_INDEX_KERNEL = ("prefill_index_kernel (tcgen05 kind::f8f6f4 indexer scores + streaming "
                        "Top-512 per query)")
PREFILL_INDEX_PEAK_RATIO = 2                    # E4M3 MMA: the bf16 peak x 2 (nominal ratio)


def attention_flops_per_query(n_main: int, n_swa: int) -> int:
    """Useful FLOPs of one query's 16-head attention over n_main + n_swa keys of 512
    dims: S = Q K^T and O = P V, two multiply-adds per key, head and dim."""
    return 2 * 2 * 16 * 512 * (n_main + n_swa)


def prefill_bytes_per_seq(n: int, q_per_seq: int, swa_rows: int, modes: list[int]) -> int:
    """Unique bytes one sequence's chunked-prefill step must move (each byte once): the
    chunk's latent tokens in and their compressed FP4 rows out, the indexer scan of the
    Full layer (every position once), the FP4 rows the Top-512 selections gather (at most
    every position once), and per layer the chunk's q in, fp32 out and SWA rows."""
    n_full = sum(1 for m in modes if m == 0)
    chunk = q_per_seq * 1024 + (q_per_seq // 2) * MAIN_ROW_BYTES
    scan = n_full * n * IDX_ROW_BYTES
    gathered = n_full * min(n, q_per_seq * 512) * MAIN_ROW_BYTES
    per_layer = len(modes) * (q_per_seq * (Q_BYTES + OUT_BYTES) + swa_rows * SWA_ROW_BYTES)
    idx_qw = n_full * q_per_seq * IDXQW_BYTES
    return chunk + scan + gathered + per_layer + idx_qw


def measured_tensor_peaks():
    """(bf16 TFLOP/s measured burst, kind): the dense bf16 figure of MEASURED_PEAKS.json."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def scan_traffic_per_launch(lens) -> int | None:
    """DRAM bytes per Full-scan launch from the committed ncu summary, scaled to this
    launch by positions; None unless the kernel sources still hash to the captured ones."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "scan_select_full_b8_256k.md")
    csrc = os.path.join(ROOT, "fp4_kv_cache_04_b200", "csrc")
    try:
        text = open(path).read()
        fields = dict(line.split(": ", 1) for line in text.splitlines()
                      if line.startswith(("traffic_per_launch_b64_bytes", "kernel_sources_sha256")))
        h = hashlib.sha256()
        for f in ("scan_select.cu", "select.cuh", "tc.cuh", "common.cuh", "kernels.cuh"):
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(fh.read())
        if h.hexdigest() != fields["kernel_sources_sha256"].strip():
            return None
        per_b64 = int(fields["traffic_per_launch_b64_bytes"])
    except (OSError, KeyError, ValueError):
        return None
    return int(round(per_b64 * sum(lens) / (64 * 262144)))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return HBM_FALLBACK_GBS, "fallback"


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons while running."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = os.path.join("/tmp", f"csa2_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) != len(self.FIELDS):
                    continue
                try:
                    sm.append(float(parts[0]))
                    mx.append(float(parts[1]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[4:]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ multi-process helpers


def max_over_ranks(value: float, world: int, device) -> float:
    """The max over all ranks of a per-rank scalar (a timed interval): every rank makes
    the same collective call; one process returns its own value."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank: int, steps: int, elapsed_ms: float) -> float:
    """Units per second of the whole job: every rank processes units_per_rank per step
    (weak scaling, data parallel over sequences), timed by the slowest rank."""
    return world * units_per_rank * steps / (elapsed_ms / 1e3)


def rank_seed_offset(rank: int) -> int:
    """Each rank draws its own sequences (distinct seeds), with the same shapes."""
    return 1000 * rank


# ------------------------------------------------------------------ the GPU arm


def page_cache(step, page_rows, seed=11):
    """Moves the step's cache (FP4 rows, scales, indexer rows and scales) into pages of
    page_rows rows in a shuffled order; returns the page table [B][pages] and a function
    mapping (sequence, position) to the physical row."""
    import torch
    dev = step.codes.device
    offs = step.kv.tolist()
    pages = [(n + page_rows - 1) // page_rows for n in step.lens]
    n_phys = sum(pages)
    perm = torch.randperm(n_phys, generator=torch.Generator().manual_seed(seed))
    table = torch.zeros(len(pages), max(pages), dtype=torch.int32)
    k = 0
    for b, np_ in enumerate(pages):
        table[b, :np_] = perm[k:k + np_]
        k += np_
    src, dst = [], []
    for b, np_ in enumerate(pages):
        for j in range(np_):
            lo, n = j * page_rows, min(page_rows, step.lens[b] - j * page_rows)
            src.append(torch.arange(offs[b] + lo, offs[b] + lo + n))
            pg = int(table[b, j])
            dst.append(torch.arange(pg * page_rows, pg * page_rows + n))
    src, dst = torch.cat(src).to(dev), torch.cat(dst).to(dev)
    rows = n_phys * page_rows
    P = step.P
    for name, owner in (("codes", step), ("scales", step), ("idx_k", P), ("idx_kscale", P)):
        t = getattr(owner, name)
        phys = torch.zeros((rows,) + tuple(t.shape[1:]), dtype=t.dtype, device=dev)
        phys[dst] = t[src]
        setattr(owner, name, phys)
        del t
    torch.cuda.empty_cache()
    table = table.to(dev)

    def phys_row(b, pos):
        return int(table[b, pos // page_rows]) * page_rows + pos % page_rows
    return table, phys_row


class DecodeStep:
    """Device buffers and per-layer arguments of one decode step on one GPU."""

    def __init__(self, w, dev, seed_offset=0, reuse_cache=False, keep_seqs=(0,), swa_fp8=False,
                 contig_pool=True, paged=0, q_nvfp4=False, defer_pool=True):
        import torch

        from fp4_kv_cache_04_b200 import csa2, synth
        self.csa2, self.synth, self.torch = csa2, synth, torch
        w = synth.Workload(**{**w.__dict__, "seed": w.seed + seed_offset})
        self.w = w
        P = synth.make_problem(w, device=dev)
        self.P = P
        self.swa_fp8 = swa_fp8
        if swa_fp8:                        # the FP8 SWA variant replaces each layer's bf16 rows
            for li in P.layers:
                li.swa8, li.swa_s = synth.fp8_swa(li.swa)
                li.swa = None
        self.lens = P.lens
        self.B = w.batch
        self.max_n = max(P.lens)
        total = sum(P.lens)
        self.kv = P.kv_offsets
        self.codes = torch.empty(total, 256, dtype=torch.uint8, device=dev)
        self.scales = torch.empty(total, 32, dtype=torch.uint8, device=dev)
        # cache build (not part of the step): quantise every latent row once
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        csa2.quantize_kv(P.latent, 1, self.codes, self.scales)
        torch.cuda.synchronize()
        self.cache_build_s = time.perf_counter() - t0
        self.cache_build_bytes = total * (1024 + MAIN_ROW_BYTES)
        offs = P.kv_offsets.tolist()                  # host copies for the oracle legs
        self.latent_host = {b: P.latent[offs[b]:offs[b + 1]].cpu() for b in keep_seqs}
        P.latent = None
        torch.cuda.empty_cache()
        # the step appends its new row at each sequence's last position
        self.dst_row = (P.kv_offsets[1:] - 1).contiguous()
        self.page_table, self.page_rows = None, 0
        if paged:                          # the cache in shuffled pages behind a page table
            self.page_table, phys = page_cache(self, paged)
            self.page_rows = paged
            self.dst_row = torch.tensor([phys(b, n - 1) for b, n in enumerate(self.lens)],
                                        dtype=torch.int64, device=dev)
            total = self.codes.shape[0]
        self.new_rows = P.new_rows.contiguous()
        self.new_proj = P.new_idx_proj.contiguous()
        self.topk = torch.full((self.B, 512), -1, dtype=torch.int32, device=dev)
        self.pool = torch.full((self.B, 2048), -1, dtype=torch.int32, device=dev)
        # the pool's indexer rows, contiguous (written by the Full layer, read by Reindex)
        with_pool = w.want_pool and any(li.mode == synth.REINDEX for li in P.layers)
        self.pool_k = (torch.zeros(self.B, POOL_POS, 64, dtype=torch.uint8, device=dev)
                       if with_pool and contig_pool else None)
        self.pool_kscale = (torch.zeros(self.B, POOL_POS, dtype=torch.float32, device=dev)
                            if self.pool_k is not None else None)
        self.outs = [torch.empty(self.B, 16, 512, dtype=torch.float32, device=dev)
                     for _ in P.layers]
        # the Full layer's pool work is joined by the first Reindex layer, not at the end of
        # the Full call, so that it runs beside the Reuse layers in between
        self.ev_pool = torch.cuda.Event() if with_pool and defer_pool else None
        self.args = []
        self.ws = []
        # optional cross-layer reuse cache of dequantised rows (ignored by decode calls)
        self.sel_cache = (torch.empty(self.B, 512, 512, dtype=torch.float16, device=dev)
                          if reuse_cache else None)
        for li, out in zip(P.layers, self.outs):
            kw = dict(mode=li.mode, batch=self.B, q_per_seq=1, max_n=self.max_n,
                      kv_offsets=self.kv, codes=self.codes, scales=self.scales,
                      topk_idx=self.topk, q=li.q, swa_kv=li.swa, out=out,
                      swa_kv8=getattr(li, "swa8", None), swa_kscale=getattr(li, "swa_s", None),
                      pool_blocks=self.pool, want_pool=(li.mode == synth.FULL and w.want_pool),
                      sm_scale=w.sm_scale, total_n=total, pool_k=self.pool_k, pool_kscale=self.pool_kscale,
                      page_table=self.page_table, page_rows=self.page_rows, q_nvfp4=q_nvfp4,
                      ev_pool=self.ev_pool if li.mode != synth.REUSE else None)
            if self.sel_cache is not None:
                kw.update(sel_cache=self.sel_cache,
                          sel_cache_mode=csa2.CACHE_USE if li.mode == synth.REUSE else csa2.CACHE_FILL)
            if li.mode != synth.REUSE:
                kw.update(idx_q=li.idx_q, idx_w=li.idx_w, idx_k=P.idx_k, idx_kscale=P.idx_kscale)
            ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)), dev)
            self.ws.append(ws)
            self.args.append((kw, csa2.layer_args(workspace=ws, **kw)))
        self.full_layer = next(i for i, li in enumerate(P.layers) if li.mode == synth.FULL)
        self.reindex_layer = next((i for i, li in enumerate(P.layers) if li.mode == synth.REINDEX), None)

    def set_index_events(self, ev_begin, ev_end, ev_rbegin=None, ev_rend=None):
        """Points the Full layer's indexer timing events (and, when given, the first Reindex
        layer's) at the given torch events."""
        kw, _ = self.args[self.full_layer]
        a = self.csa2.layer_args(workspace=self.ws[self.full_layer], ev_index_begin=ev_begin,
                                 ev_index_end=ev_end, **kw)
        self.args[self.full_layer] = (kw, a)
        ri = getattr(self, "reindex_layer", None)
        if ev_rbegin is not None and ri is not None:
            kw, _ = self.args[ri]
            self.args[ri] = (kw, self.csa2.layer_args(workspace=self.ws[ri], ev_index_begin=ev_rbegin,
                                                      ev_index_end=ev_rend, **kw))

    def run(self):
        c = self.csa2
        P = self.P
        # the step's cache append: FP4 main-KV row + FP8 indexer-K row of each new position
        c.append_kv(self.new_rows, self.new_proj, self.dst_row, self.codes, self.scales, P.idx_k,
                    P.idx_kscale)
        for _, a in self.args:
            c.attend(a)

    def check_status(self):
        return [self.csa2.check_device_status(ws) for ws in self.ws]


class PrefillStep:
    """Device buffers and per-layer arguments of one chunked-prefill step on one GPU: the
    chunk's own latent tokens quantised into the FP4 cache at ratio 2 (mean of adjacent
    tokens), then the encoder group's layers (Full + 5 Reuse) for the chunk's queries,
    each query seeing the compressed positions that end at or before its token and its
    own 128-token window."""

    def __init__(self, w, dev, seed_offset=0, keep_seqs=(0,), q_nvfp4=False):
        import torch

        from fp4_kv_cache_04_b200 import csa2, synth
        self.csa2, self.synth, self.torch = csa2, synth, torch
        w = synth.Workload(**{**w.__dict__, "seed": w.seed + seed_offset})
        self.w = w
        P = synth.make_problem(w, device=dev)
        self.P = P
        self.lens = P.lens
        self.B = w.batch
        self.Q = w.q_per_seq
        self.max_n = max(P.lens)
        total = sum(P.lens)
        self.kv = P.kv_offsets
        self.codes = torch.empty(total, 256, dtype=torch.uint8, device=dev)
        self.scales = torch.empty(total, 32, dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        csa2.quantize_kv(P.latent, w.ratio, self.codes, self.scales)   # cache build (not timed)
        torch.cuda.synchronize()
        self.cache_build_s = time.perf_counter() - t0
        self.cache_build_bytes = total * (w.ratio * 1024 + MAIN_ROW_BYTES)
        toks = [w.ratio * n for n in P.lens]
        tok_off = [0]
        for n in toks:
            tok_off.append(tok_off[-1] + n)
        qpos = [int(x) for x in P.q_pos.tolist()]
        # the chunk's tokens (q_pos[b] .. q_pos[b] + Q - 1) and their compressed rows
        self.chunk_latent = torch.cat([P.latent[tok_off[b] + qpos[b]: tok_off[b] + qpos[b] + self.Q]
                                       for b in range(self.B)]).contiguous()
        offs = P.kv_offsets.tolist()
        self.chunk_dst = torch.cat([torch.arange(offs[b] + qpos[b] // w.ratio,
                                                 offs[b] + (qpos[b] + self.Q) // w.ratio,
                                                 dtype=torch.int64, device=dev)
                                    for b in range(self.B)]).contiguous()
        self.latent_host = {b: P.latent[tok_off[b]:tok_off[b + 1]].cpu() for b in keep_seqs}
        P.latent = None
        torch.cuda.empty_cache()
        rows = self.B * self.Q
        self.topk = torch.full((rows, 512), -1, dtype=torch.int32, device=dev)
        self.outs = [torch.empty(rows, 16, 512, dtype=torch.float32, device=dev) for _ in P.layers]
        self.args, self.ws = [], []
        for li, out in zip(P.layers, self.outs):
            kw = dict(mode=li.mode, batch=self.B, q_per_seq=self.Q, ratio=w.ratio, max_n=self.max_n,
                      kv_offsets=self.kv, q_pos=P.q_pos, codes=self.codes, scales=self.scales,
                      topk_idx=self.topk, q=li.q, swa_kv=li.swa, out=out, sm_scale=w.sm_scale,
                      total_n=total, q_nvfp4=q_nvfp4)
            if li.mode != synth.REUSE:
                kw.update(idx_q=li.idx_q, idx_w=li.idx_w, idx_k=P.idx_k, idx_kscale=P.idx_kscale)
            ws = csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(**kw)), dev)
            self.ws.append(ws)
            self.args.append((kw, csa2.layer_args(workspace=ws, **kw)))
        self.full_layer = next(i for i, li in enumerate(P.layers) if li.mode == synth.FULL)

    set_index_events = DecodeStep.set_index_events
    check_status = DecodeStep.check_status

    def run(self):
        c = self.csa2
        c.quantize_kv(self.chunk_latent, self.w.ratio, self.codes, self.scales, dst_row=self.chunk_dst)
        for _, a in self.args:
            c.attend(a)

    def visible(self, b):
        """Visible compressed positions of each query of sequence b (causal, ratio r)."""
        r = self.w.ratio
        q0 = int(self.P.q_pos[b])
        return [min(self.lens[b], (q0 + i + 1) // r) for i in range(self.Q)]


class PromptStep:
    """A whole prompt's encoder prefill: chunk after chunk (q_per_seq tokens each), the
    chunk's own latent tokens are quantised into the cache at ratio 2, then the encoder
    groups (Full + 5 Reuse each) run for the chunk's queries, each seeing the compressed
    positions that end at or before its token and its own 128-token window.  Every chunk
    uses the same per-layer query / window / indexer-query tensors (synthetic inputs; the
    chunks differ in position), and the indexer K of the whole prompt is given."""

    def __init__(self, w, dev, seed_offset=0, keep_seqs=(0,), n_chunks=None, q_nvfp4=False):
        import torch

        from fp4_kv_cache_04_b200 import csa2, synth
        self.csa2, self.synth, self.torch = csa2, synth, torch
        w = synth.Workload(**{**w.__dict__, "seed": w.seed + seed_offset})
        self.w = w
        P = synth.make_problem(w, device=dev)
        self.P = P
        self.lens = P.lens
        self.B, self.Q = w.batch, w.q_per_seq
        self.max_n = max(P.lens)
        total = sum(P.lens)
        self.kv = P.kv_offsets
        tokens = [w.ratio * n for n in P.lens]
        self.n_chunks = n_chunks or tokens[0] // self.Q
        assert all(t == self.n_chunks * self.Q for t in tokens), "whole chunks per prompt"
        self.codes = torch.zeros(total, 256, dtype=torch.uint8, device=dev)
        self.scales = torch.zeros(total, 32, dtype=torch.uint8, device=dev)
        self.cache_build_s, self.cache_build_bytes = 1e-9, 0      # the step builds the cache
        tok_off = [0]
        for n in tokens:
            tok_off.append(tok_off[-1] + n)
        offs = P.kv_offsets.tolist()
        self.latent_host = {b: P.latent[tok_off[b]:tok_off[b + 1]].cpu() for b in keep_seqs}
        self.chunk_latent, self.chunk_dst, self.q_pos = [], [], []
        per = self.Q // w.ratio
        for c in range(self.n_chunks):
            self.chunk_latent.append(torch.cat([P.latent[tok_off[b] + c * self.Q: tok_off[b] + (c + 1) * self.Q]
                                                for b in range(self.B)]).contiguous())
            self.chunk_dst.append(torch.cat([torch.arange(offs[b] + c * per, offs[b] + (c + 1) * per,
                                                          dtype=torch.int64, device=dev) for b in range(self.B)]))
            self.q_pos.append(torch.full((self.B,), c * self.Q, dtype=torch.int64, device=dev))
        P.latent = None
        torch.cuda.empty_cache()
        rows = self.B * self.Q
        self.topk = torch.full((rows, 512), -1, dtype=torch.int32, device=dev)
        self.outs = [torch.empty(rows, 16, 512, dtype=torch.float32, device=dev) for _ in P.layers]
        self.ws = []
        self.kws = []
        for li, out in zip(P.layers, self.outs):
            kw = dict(mode=li.mode, batch=self.B, q_per_seq=self.Q, ratio=w.ratio, max_n=self.max_n,
                      kv_offsets=self.kv, codes=self.codes, scales=self.scales, topk_idx=self.topk, q=li.q,
                      swa_kv=li.swa, out=out, sm_scale=w.sm_scale, total_n=total, q_nvfp4=q_nvfp4)
            if li.mode != synth.REUSE:
                kw.update(idx_q=li.idx_q, idx_w=li.idx_w, idx_k=P.idx_k, idx_kscale=P.idx_kscale)
            self.kws.append(kw)
            self.ws.append(csa2.alloc_workspace(csa2.workspace_size(csa2.layer_args(q_pos=self.q_pos[0], **kw)), dev))
        # arguments per (chunk, layer): the same buffers, the chunk's q_pos
        self.chunk_args = [[csa2.layer_args(workspace=ws, q_pos=self.q_pos[c], **kw)
                            for kw, ws in zip(self.kws, self.ws)] for c in range(self.n_chunks)]
        last = self.n_chunks - 1
        self.full_layer = next(i for i, li in enumerate(P.layers) if li.mode == synth.FULL)
        self.args = [(dict(kw, q_pos=self.q_pos[last]), a) for kw, a in zip(self.kws, self.chunk_args[last])]

    def set_index_events(self, ev_begin, ev_end, ev_rbegin=None, ev_rend=None):
        """Times the last chunk's first Full layer (its indexer sees the whole prompt)."""
        last = self.n_chunks - 1
        kw = self.kws[self.full_layer]
        self.chunk_args[last][self.full_layer] = self.csa2.layer_args(
            workspace=self.ws[self.full_layer], q_pos=self.q_pos[last], ev_index_begin=ev_begin,
            ev_index_end=ev_end, **kw)

    check_status = DecodeStep.check_status

    def run_chunk(self, c, on_layer=None, latent=None, chunk_args=None):
        """Chunk c: its latent tokens into the cache, then every layer (on_layer(i) after
        layer i; latent / chunk_args replace the step's own input set)."""
        c_ = self.csa2
        c_.quantize_kv(self.chunk_latent[c] if latent is None else latent, self.w.ratio, self.codes,
                       self.scales, dst_row=self.chunk_dst[c])
        for i, a in enumerate((self.chunk_args if chunk_args is None else chunk_args)[c]):
            c_.attend(a)
            if on_layer is not None:
                on_layer(i)

    def run(self):
        for c in range(self.n_chunks):
            self.run_chunk(c)

    def visible(self, b, chunk=None):
        """Visible compressed positions of each query of sequence b in a chunk (last: default)."""
        c = self.n_chunks - 1 if chunk is None else chunk
        return [min(self.lens[b], (c * self.Q + i + 1) // self.w.ratio) for i in range(self.Q)]

    def flops(self):
        """(indexer, attention) FLOPs of a whole prompt: every Full layer scores each query's
        visible positions; every layer attends over min(512, visible) rows + the window."""
        n_full = sum(1 for li in self.P.layers if li.mode == self.synth.FULL)
        idx = att = 0
        for c in range(self.n_chunks):
            for b in range(self.B):
                vis = self.visible(b, c)
                idx += n_full * sum(vis) * PREFILL_INDEX_FLOPS_PER_POS
                for i, v in enumerate(vis):
                    t = c * self.Q + i
                    att += len(self.P.layers) * attention_flops_per_query(min(512, v), min(128, t + 1))
        return idx, att


def make_step(w, dev, **kw):
    """The step object of a workload: decode (one query per sequence) or chunked prefill."""
    if w.name.startswith("prefill_prompt"):
        for k_ in ("reuse_cache", "swa_fp8", "contig_pool", "paged", "defer_pool"):
            kw.pop(k_, None)
        return PromptStep(w, dev, **kw)
    if w.q_pos is not None:
        for k_ in ("reuse_cache", "swa_fp8", "contig_pool", "paged", "defer_pool"):
            kw.pop(k_, None)
        return PrefillStep(w, dev, **kw)
    return DecodeStep(w, dev, **kw)


def run_ours(args, rank, world, dev):
    import torch
    import torch.distributed as dist

    from fp4_kv_cache_04_b200 import csa2, synth

    w = synth.workloads()[args.workload]
    if args.batch is not None:
        w = synth.Workload(**{**w.__dict__, "batch": args.batch,
                              "lens": None if w.lens is None else w.lens[:1] * args.batch})
    if args.context is not None:
        w = synth.Workload(**{**w.__dict__, "lens": [args.context] * w.batch, "ragged": None})
    step = make_step(w, dev, seed_offset=rank_seed_offset(rank), reuse_cache=args.reuse_cache,
                     q_nvfp4=args.q_nvfp4, defer_pool=not args.join_pool,
                     swa_fp8=args.swa_fp8, contig_pool=not args.scattered_pool, paged=args.paged)
    B = step.B
    modes = w.modes
    prefill = w.q_pos is not None
    swa_row = 512 + 4 if args.swa_fp8 else SWA_ROW_BYTES
    prompt = isinstance(step, PromptStep)
    if prompt:
        n_ch = step.n_chunks
        bytes_per_step = n_ch * sum(prefill_bytes_per_seq(n // n_ch, w.q_per_seq, w.swa_rows, modes)
                                    for n in step.lens)
        index_flops, attn_flops = step.flops()
        last_index_flops = sum(v for b in range(B) for v in step.visible(b)) * PREFILL_INDEX_FLOPS_PER_POS
    elif prefill:
        bytes_per_step = sum(prefill_bytes_per_seq(n, w.q_per_seq, w.swa_rows, modes) for n in step.lens)
        vis = [v for b in range(B) for v in step.visible(b)]
        index_flops = sum(vis) * PREFILL_INDEX_FLOPS_PER_POS
        attn_flops = B * w.q_per_seq * len(modes) * attention_flops_per_query(512, 128)
        last_index_flops = index_flops
    else:
        bytes_per_step = sum(algorithmic_bytes_per_seq(n, modes, swa_row) for n in step.lens)
    scan_bytes = sum(n * IDX_ROW_BYTES for n in step.lens)
    K, W = args.steps, args.warmup

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    has_reindex = getattr(step, "reindex_layer", None) is not None
    revs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(K)] if has_reindex else [(None, None)] * K
    for b_ev, e_ev in evs + (revs if has_reindex else []):   # create the CUDA events up front
        b_ev.record()
        e_ev.record()
    for _ in range(W):
        step.run()
    torch.cuda.synchronize()
    status = step.check_status()
    assert all(s == 0 for s in status), f"device status {status}"
    graph = None
    if not args.no_graph:
        # the K timed steps, each with its own Full-scan events, as one CUDA graph
        graph = torch.cuda.CUDAGraph()
        before = csa2.kernel_launches()
        with torch.cuda.graph(graph):
            for i in range(K):
                step.set_index_events(*evs[i], *revs[i])
                step.run()
        launches_per_graph = csa2.kernel_launches() - before
        graph.replay()                     # one untimed replay (first-launch upload)
        torch.cuda.synchronize()
        status = step.check_status()
        assert all(s == 0 for s in status), f"device status {status}"

    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(dev.index)
    sampler = ClockSampler(gpu_id)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.15)                       # let the sampler take its first sample
    launches0 = csa2.kernel_launches()
    start.record()
    if graph is not None:
        graph.replay()
    else:
        for i in range(K):
            step.set_index_events(*evs[i], *revs[i])
            step.run()
    end.record()
    torch.cuda.synchronize()
    # kernels of the library in the timed region: counted at launch, or at capture for the graph
    launches = (csa2.kernel_launches() - launches0) if graph is None else launches_per_graph
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    elapsed_ms = start.elapsed_time(end)
    scan_ms = sum(b.elapsed_time(e) for b, e in evs) / K
    reindex_ms = sum(b.elapsed_time(e) for b, e in revs) / K if has_reindex else None
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    ms_per_step = elapsed_ms / K
    value = whole_job_rate(world, B, K, elapsed_ms)

    peak, peak_kind = measured_peaks()
    achieved = scan_bytes / (scan_ms / 1e3) / 1e9
    result = {
        "metric": PREFILL_METRIC if prefill else METRIC,
        "value": round(value * (step.n_chunks * w.q_per_seq if prompt else w.q_per_seq if prefill else 1), 2),
        "unit": "tokens/s" if prefill else "queries/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3 (indexer) and f16 (attention) MMA operands, f32 accumulate; FP4/FP8 storage",
        "data": "synthetic (seeded generators of fp4_kv_cache_04_b200/synth.py; no weights, no dataset)",
        "config": {
            "workload": w.name, "describe": w.describe, "batch_per_gpu": B,
            "contexts": f"all {step.lens[0]}" if len(set(step.lens)) == 1 else
            f"ragged {min(step.lens)}..{max(step.lens)}",
            "layers": len(modes), "schedule": "".join("FRU"[m] for m in modes),
            "parallelism": f"dp{world} over sequences (no collective on the data path)",
            "l2": "inputs larger than L2 (the Full scan alone reads "
                  f"{scan_bytes / 1e9:.2f} GB per step; no flush)" if not prefill else
                  "the step's q and fp32 outputs (1.15 GB) are larger than L2; no flush",
            "algorithmic_bytes_per_step": bytes_per_step,
            "step_hbm_gbs": round(bytes_per_step / (ms_per_step / 1e3) / 1e9, 1),
            "step_frac_of_measured_hbm": round(bytes_per_step / (ms_per_step / 1e3) / 1e9 / peak, 4),
            "step_frac_of_8TBs": round(bytes_per_step / (ms_per_step / 1e3) / 8e12, 4),
            "cache_build_gbs": round(step.cache_build_bytes / step.cache_build_s / 1e9, 1),
            "reuse_cache": args.reuse_cache,
            "cuda_graph": not args.no_graph,
            "query": "NVFP4 variant (block-scaled FP4 MMA for the main-row logits)" if args.q_nvfp4
            else "bf16 (exact)",
            "swa_kv": "fp8 (E4M3 + fp32 row scale)" if args.swa_fp8 else "bf16",
            "reindex_pool_rows": "contiguous (gathered by the Full layer)" if getattr(step, "pool_k", None)
            is not None else "scattered 8-row blocks",
            "cache_layout": f"pages of {args.paged} rows, shuffled (page table)" if args.paged else "packed",
            "pool_join": "at the first Reindex layer (ev_pool)" if getattr(step, "ev_pool", None) is not None
            else "at the end of the Full call",
            "full_scan_launch_us": round(scan_ms * 1e3, 2),
            "reindex_scan_launch_us": None if reindex_ms is None else round(reindex_ms * 1e3, 2),
        },
        "roofline": {
            "kernel": "scan_select_kernel (Full-layer indexer scan + chunk Top-512)",
            "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
            "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
            "traffic": scan_traffic_per_launch(step.lens), "avg_launch_us": round(scan_ms * 1e3, 2),
            "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of a B=8 capture "
                              "(profiles/scan_select_full_b8_256k.md), scaled by positions",
            "algorithmic_bytes_per_launch": scan_bytes,
        },
        "clocks": clocks,
        "gpu_launches": int(launches),
    }
    if prefill:
        tpeak, tkind = measured_tensor_peaks()
        step_tflops = (index_flops + attn_flops) / (ms_per_step / 1e3) / 1e12
        idx_tflops = last_index_flops / (scan_ms / 1e3) / 1e12
        result["config"].update({
            "tokens_per_step": B * w.q_per_seq, "q_pos": [int(x) for x in step.P.q_pos.tolist()],
            "flops_per_step": {"attention": attn_flops, "indexer": index_flops},
            "step_tflops": round(step_tflops, 1),
            "step_frac_of_f16_peak": round(step_tflops / tpeak, 4),
            "step_frac_of_fp4_peak": round(step_tflops / (4 * tpeak), 4),
            "peaks_note": f"f16 = bf16 {tkind} dense burst {tpeak} TFLOP/s; fp8 = 2x, fp4 = 4x "
                          "that (nominal ratios)",
        })
        result["roofline"] = {
            "kernel": PREFILL_INDEX_KERNEL, "bound": "tensor", "achieved": round(idx_tflops, 1),
            "peak": round(PREFILL_INDEX_PEAK_RATIO * tpeak, 1),
            "peak_kind": f"{tkind} bf16 x {PREFILL_INDEX_PEAK_RATIO} (nominal ratio of the MMA dtype)",
            "unit": "TFLOP/s", "frac": round(idx_tflops / (PREFILL_INDEX_PEAK_RATIO * tpeak), 4),
            "traffic": None, "avg_launch_us": round(scan_ms * 1e3, 2),
            "algorithmic_flops_per_launch": last_index_flops,
        }
        if prompt:
            result["metric"] = PROMPT_METRIC
            result["roofline"]["kernel"] += " (the last chunk's first Full layer)"
            result["config"]["chunks"] = step.n_chunks
            result["config"]["tokens_per_step"] = B * step.n_chunks * w.q_per_seq
            del result["config"]["q_pos"]
        for k_ in ("reuse_cache", "swa_kv", "reindex_pool_rows", "full_scan_launch_us", "reindex_scan_launch_us",
                   "cache_layout", "pool_join"):
            del result["config"][k_]
    if prompt:
        result["config"]["cache_build_gbs"] = None      # the step quantises every chunk itself
        result["config"]["l2"] = ("each chunk's q and fp32 outputs (2.4 GB over 18 layers) are larger "
                                  "than L2; no flush")
    if not args.no_e2e:
        result["e2e"] = (run_e2e_prompt(step, K, world, dev) if prompt else
                         run_e2e(step, K=min(K, 50), world=world, dev=dev))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = run_cpu_baseline(step, args.cpu_seconds)
    return result


def _twin_inputs(step):
    """A second set of the step's per-step device inputs and outputs (clones), with layer
    arguments pointing at them; everything else (caches, indices, workspaces) is shared:
    the two sets' steps run one after the other on the compute stream."""
    import copy
    twin = copy.copy(step)
    clone = {}

    def cl(t):
        if t is None:
            return None
        if id(t) not in clone:
            clone[id(t)] = t.clone()
        return clone[id(t)]

    twin.outs = [cl(o) for o in step.outs]
    if isinstance(step, PrefillStep):
        twin.chunk_latent = cl(step.chunk_latent)
    else:
        twin.new_rows, twin.new_proj = cl(step.new_rows), cl(step.new_proj)
    twin.args = []
    for (kw, _), ws in zip(step.args, step.ws):
        kw2 = dict(kw)
        for k in ("q", "swa_kv", "swa_kv8", "swa_kscale", "idx_q", "idx_w", "out"):
            if kw2.get(k) is not None:
                kw2[k] = cl(kw2[k])
        twin.args.append((kw2, step.csa2.layer_args(workspace=ws, **kw2)))
    return twin, cl


def _step_io(st, prefill):
    """(device input views, last output) of one input set: every layer's q, the indexer
    q / w, the new SWA row (decode) or the chunk's window rows (prefill), and the new
    latent rows + indexer values (decode) or the chunk's latent tokens (prefill)."""
    ins = []
    for kw, _ in st.args:
        ins.append(kw["q"])
        if kw.get("idx_q") is not None:
            ins += [kw["idx_q"], kw["idx_w"]]
        if prefill:
            ins.append(kw["swa_kv"])
        elif kw.get("swa_kv") is not None:
            ins.append(kw["swa_kv"][:, -1])
        else:                                            # FP8 SWA: codes and scale of the new row
            ins += [kw["swa_kv8"][:, -1], kw["swa_kscale"][:, -1:]]
    ins += [st.chunk_latent] if prefill else [st.new_rows, st.new_proj]
    return ins, st.outs[-1]


def run_e2e_prompt(step, K, world, dev):
    """The whole prompt through the public API with host buffers.  Every chunk uploads its
    inputs from pinned memory (every layer's q and window rows, the Full layers' indexer
    q / w, the chunk's latent tokens) into one of two device input sets on a copy stream
    while the compute stream runs the previous chunk on the other set; a second copy
    stream reads each chunk's last-layer output back.  Events order the three streams.
    A step is one prompt per sequence (every chunk); value = tokens / time."""
    import torch
    import torch.distributed as dist

    csa2 = step.csa2
    sets = []
    for s_i in range(2):
        memo = {}

        def cl(t):
            if t is None or s_i == 0:
                return t
            if id(t) not in memo:
                memo[id(t)] = t.clone()
            return memo[id(t)]

        kws = []
        for kw in step.kws:
            kw2 = dict(kw)
            for k in ("q", "swa_kv", "idx_q", "idx_w", "out"):
                if kw2.get(k) is not None:
                    kw2[k] = cl(kw2[k])
            kws.append(kw2)
        lat = torch.empty_like(step.chunk_latent[0])
        args_ = [[csa2.layer_args(workspace=ws, q_pos=step.q_pos[c], **kw) for kw, ws in zip(kws, step.ws)]
                 for c in range(step.n_chunks)]
        ins = []
        for kw in kws:
            ins += [kw["q"], kw["swa_kv"]] + ([kw["idx_q"], kw["idx_w"]] if kw.get("idx_q") is not None else [])
        ins.append(lat)
        sets.append((args_, ins, lat, kws[-1]["out"]))
    src = sets[0][1][:-1] + [step.chunk_latent[0]]       # the same host inputs every chunk
    offs, total = [], 0
    for t in src:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    stage_h = torch.empty(total, dtype=torch.uint8).pin_memory()
    views = []
    for t, o in zip(src, offs):
        n = t.numel() * t.element_size()
        stage_h[o:o + n].copy_(t.contiguous().cpu().view(-1).view(torch.uint8))
        views.append(stage_h[o:o + n])
    host_out = [sets[s][3].cpu().pin_memory() for s in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in src)
    d2h = host_out[0].numel() * host_out[0].element_size()
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def pipeline(n_prompts, start=None, end=None, n_chunks=None):
        n_ch = n_chunks or step.n_chunks
        if start is not None:
            start.record(up)
        for k in range(n_prompts * n_ch):
            c, s = k % n_ch, k % 2
            args_, ins, lat, out = sets[s]
            with torch.cuda.stream(up):                  # chunk k's inputs into set s
                if k >= 2:
                    up.wait_event(ev_done[s])            # chunk k-2 is done reading set s
                for t, v in zip(ins, views):
                    t.view(-1).view(torch.uint8).copy_(v, non_blocking=True)
                ev_in[s].record(up)
            comp.wait_event(ev_in[s])
            if k >= 2:
                comp.wait_event(ev_out[s])               # chunk k-2's result has left set s
            step.run_chunk(c, latent=lat, chunk_args=args_)
            ev_done[s].record(comp)
            with torch.cuda.stream(down):                # chunk k's result back
                down.wait_event(ev_done[s])
                host_out[s].copy_(out, non_blocking=True)
                ev_out[s].record(down)
        if end is not None:
            end.record(down)

    pipeline(1, n_chunks=4)                              # warm-up: the first chunks
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pipeline(K, t0, t1)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    assert all(s == 0 for s in step.check_status())
    tokens = world * step.B * step.n_chunks * step.Q * K
    return {"value": round(tokens / (ms / 1e3), 2), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d * step.n_chunks, "d2h_bytes_per_step": d2h * step.n_chunks,
            "steps": K, "ms_per_step": round(ms / K, 4),
            "path": "csa2_quantize_kv + csa2_attend per chunk and layer (eager launches), inputs "
                    "uploaded per chunk from pinned host memory on a copy stream, each chunk's "
                    "last-layer output read back on another"}


def run_e2e(step, K, world, dev):
    """The same step through the public API with host buffers.  Every step copies its
    inputs (every layer's q, the indexer q / w, the new SWA rows, the new latent rows and
    indexer values; for prefill the chunk's tokens and window rows) host -> device from
    pinned memory and reads its result (the last layer's output) back.  The inputs of a
    step travel packed in one pinned buffer (one cudaMemcpyAsync per step) into one of two
    device staging buffers: a copy stream uploads step k+1's inputs while the compute
    stream replays step k, whose captured graph first spreads its staging buffer into the
    layer inputs (device copies) and then runs the layers; a second copy stream reads
    step k's result back.  Events order the three streams."""
    import torch
    import torch.distributed as dist

    prefill = isinstance(step, PrefillStep)
    # plain layer arguments (the timed run attached its indexer timing events)
    step.args = [(kw, step.csa2.layer_args(workspace=ws, **kw)) for (kw, _), ws in zip(step.args, step.ws)]
    twin, _ = _twin_inputs(step)
    sets = [step, twin]
    io = [_step_io(st, prefill) for st in sets]
    # packed layout of one step's inputs (256-byte aligned pieces)
    offs, total = [], 0
    for t in io[0][0]:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    stage_h = torch.empty(total, dtype=torch.uint8).pin_memory()
    for t, o in zip(io[0][0], offs):                      # the same new inputs every step
        n = t.numel() * t.element_size()
        stage_h[o:o + n].copy_(t.contiguous().cpu().view(-1).view(torch.uint8))
    stage_d = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(2)]
    host_out = [io[s][1].cpu().pin_memory() for s in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in io[0][0])
    d2h = host_out[0].numel() * host_out[0].element_size()

    def spread(s):                                        # staging buffer -> layer inputs
        for t, o in zip(io[s][0], offs):
            n = t.numel() * t.element_size()
            t.copy_(stage_d[s][o:o + n].view(t.dtype).view(t.shape))

    comp = torch.cuda.current_stream()
    graphs = []
    for s_i, st in enumerate(sets):                       # one graph per input set
        stage_d[s_i].copy_(stage_h)
        spread(s_i)
        st.run()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            spread(s_i)
            st.run()
        graphs.append(g)
    torch.cuda.synchronize()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def pipeline(n, start=None, end=None):
        if start is not None:
            start.record(up)
        for k in range(n):
            s = k % 2
            with torch.cuda.stream(up):                  # step k's inputs into staging set s
                if k >= 2:
                    up.wait_event(ev_done[s])            # step k-2 is done reading set s
                stage_d[s].copy_(stage_h, non_blocking=True)
                ev_in[s].record(up)
            comp.wait_event(ev_in[s])
            if k >= 2:
                comp.wait_event(ev_out[s])               # step k-2's result has left set s
            graphs[s].replay()
            ev_done[s].record(comp)
            with torch.cuda.stream(down):                # step k's result back
                down.wait_event(ev_done[s])
                host_out[s].copy_(io[s][1], non_blocking=True)
                ev_out[s].record(down)
        if end is not None:
            end.record(down)

    pipeline(4)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pipeline(K, t0, t1)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    per = step.Q if prefill else 1
    return {"value": round(whole_job_rate(world, step.B * per, K, ms), 2),
            "unit": "tokens/s" if prefill else "queries/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "steps": K, "ms_per_step": round(ms / K, 4),
            "overlap": "each step's inputs packed in one pinned buffer, uploaded on a copy stream "
                       "into one of two device staging sets while the previous step runs (one CUDA "
                       "graph per set: device copies into the layer inputs, then the layers); "
                       "results read back on a second copy stream"}


# ------------------------------------------------------------------ oracle (CPU) legs


class LazyFP4Rows:
    """The oracle's own FP4 quantisation of a sequence's latent rows (after its ratio-2
    compression of token pairs when ratio is 2), computed on first use and kept (the
    cache is state, built before a step, not per step)."""

    def __init__(self, latent_bits, which, ratio=1):
        self.latent = latent_bits
        self.which = which
        self.ratio = ratio
        self.memo = {}
        self.shape = (latent_bits.shape[0] // ratio, 256 if which == 0 else 32)

    def fill(self, rows):
        import numpy as np

        from oracle import csa2_oracle as O
        need = sorted({int(r) for r in rows if int(r) not in self.memo})
        if need:
            if self.ratio == 1:
                x = self.latent[need]
            else:
                x = np.concatenate([O.compress_ratio2(self.latent[[2 * r, 2 * r + 1]]) for r in need])
            c, s = O.quantize_rows(x)
            for r, cr, sr in zip(need, c, s):
                self.memo[r] = (cr, sr)

    def __getitem__(self, rows):
        import numpy as np
        rows = np.asarray(rows)
        self.fill(rows.reshape(-1))
        return np.stack([self.memo[int(r)][self.which] for r in rows]) if rows.size else \
            np.zeros((0, self.shape[1]), np.uint8)


class OracleChunk:
    """Host inputs of one sequence's chunked-prefill step for the oracle (the same seeded
    inputs as the GPU arm's; nothing comes from the CUDA library).  query(i) runs the
    encoder group's layers for the chunk's query i and returns each layer's
    (Top-512, output)."""

    def __init__(self, P, latent_seq, b=0):
        import numpy as np

        from fp4_kv_cache_04_b200.synth import bf16_bits
        w = P.workload
        o0, o1 = int(P.kv_offsets[b]), int(P.kv_offsets[b + 1])
        lb = bf16_bits(latent_seq).copy()
        self.codes = LazyFP4Rows(lb, 0, w.ratio)
        self.scales = LazyFP4Rows(lb, 1, w.ratio)
        self.scales.memo = self.codes.memo
        self.idx_k = P.idx_k[o0:o1].cpu().numpy()
        self.idx_kscale = P.idx_kscale[o0:o1].cpu().numpy()
        self.Q, self.ratio, self.sm_scale = w.q_per_seq, w.ratio, w.sm_scale
        self.q0 = int(P.q_pos[b])
        self.b = b
        self.layers = P.layers
        self.layer_host = {}

    def _layer(self, li_i, i):
        import numpy as np

        from fp4_kv_cache_04_b200.synth import bf16_bits
        li = self.layers[li_i]
        r = self.b * self.Q + i
        if li_i not in self.layer_host:
            self.layer_host[li_i] = dict(swa=bf16_bits(li.swa[self.b]))
        d = dict(q=bf16_bits(li.q[r]), swa=self.layer_host[li_i]["swa"])
        if li.idx_q is not None:
            d.update(idx_q=bf16_bits(li.idx_q[r]), idx_w=li.idx_w[r].cpu().numpy().astype(np.float64))
        return d

    def query(self, i, topk_override=None, q0=None):
        """Runs every layer for query i of the chunk that starts at token q0 (default: the
        workload's chunk).  topk_override(layer, oracle_topk) may replace the index set
        carried to later layers (tests feed the GPU's indices after a tie-band swap).
        Returns [(mode, topk, out)] per layer."""
        from oracle import csa2_oracle as O
        q0 = self.q0 if q0 is None else q0
        t = q0 + i
        res, top = [], None
        for li_i, li in enumerate(self.layers):
            d = self._layer(li_i, i)
            kw = dict(codes=self.codes, scales=self.scales, idx_k=self.idx_k,
                      idx_kscale=self.idx_kscale, q=d["q"], swa=d["swa"], sm_scale=self.sm_scale,
                      ratio=self.ratio, t=t, t0=q0)
            if "idx_q" in d:
                kw.update(idx_q=d["idx_q"], idx_w=d["idx_w"])
            top_i, _, out = O.csa2_layer(li.mode, topk_in=top, **kw)
            if topk_override is not None:
                new = topk_override(li_i, top_i)
                if new is not top_i:
                    top_i = new
                    _, _, out = O.csa2_layer(O.REUSE, topk_in=top_i, **kw)
            top = top_i
            res.append((li.mode, top_i, out))
        return res


class OracleSeq:
    """Host inputs of one sequence for the oracle's decode step (drawn by the same
    seeded generator as the GPU arm's; nothing here comes from the CUDA library)."""

    def __init__(self, P, latent_seq, want_pool, sm_scale, b=0):
        import numpy as np

        from fp4_kv_cache_04_b200.synth import bf16_bits
        o0, o1 = int(P.kv_offsets[b]), int(P.kv_offsets[b + 1])
        latent_bits = bf16_bits(latent_seq).copy()
        latent_bits[-1] = bf16_bits(P.new_rows[b:b + 1].cpu())[0]      # the appended row
        codes = LazyFP4Rows(latent_bits, 0)
        scales = LazyFP4Rows(latent_bits, 1)
        codes.memo = scales.memo = {}
        self.codes, self.scales = codes, scales
        self.idx_k = P.idx_k[o0:o1].cpu().numpy().copy()
        self.idx_kscale = P.idx_kscale[o0:o1].cpu().numpy().copy()
        if P.new_idx_proj is not None:                     # the appended indexer row
            from oracle import csa2_oracle as O
            k8, ks = O.quantize_indexer_rows(P.new_idx_proj[b:b + 1].cpu().numpy())
            self.idx_k[-1], self.idx_kscale[-1] = k8[0], ks[0]
            self.new_proj = P.new_idx_proj[b:b + 1].cpu().numpy()
        self.layers = []
        for li in P.layers:
            if li.swa is not None:
                d = dict(mode=li.mode, q=bf16_bits(li.q[b]), swa=bf16_bits(li.swa[b]))
            else:
                d = dict(mode=li.mode, q=bf16_bits(li.q[b]), swa=li.swa8[b].cpu().numpy(),
                         swa_scale=li.swa_s[b].cpu().numpy())
            if li.idx_q is not None:
                d.update(idx_q=bf16_bits(li.idx_q[b]),
                         idx_w=li.idx_w[b].cpu().numpy().astype(np.float64))
            self.layers.append(d)
        self.want_pool = want_pool
        self.sm_scale = sm_scale
        self.state = {}

    def layer(self, i):
        """Runs layer i of the schedule (state carries Top-K and pool between layers)."""
        from oracle import csa2_oracle as O
        d = self.layers[i]
        kw = dict(codes=self.codes, scales=self.scales, idx_k=self.idx_k,
                  idx_kscale=self.idx_kscale, q=d["q"], swa=d["swa"], sm_scale=self.sm_scale,
                  swa_scale=d.get("swa_scale"))
        if "idx_q" in d:
            kw.update(idx_q=d["idx_q"], idx_w=d["idx_w"])
        top, pool, _ = O.csa2_layer(d["mode"], topk_in=self.state.get("topk"),
                                    pool_in=self.state.get("pool"),
                                    want_pool=d["mode"] == O.FULL and self.want_pool, **kw)
        self.state["topk"] = top
        if pool is not None:
            self.state["pool"] = pool

    def step(self):
        from oracle import csa2_oracle as O
        O.quantize_rows(self.codes.latent[-1:])          # the step's cache append
        if hasattr(self, "new_proj"):
            O.quantize_indexer_rows(self.new_proj)
        for i in range(len(self.layers)):
            self.layer(i)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def run_cpu_baseline(step, budget_s):
    """The oracle's full 20-layer step of one sequence, repeated for about budget_s (or,
    for a prefill chunk, the chunk's queries of sequence 0 one by one through all layers)."""
    if isinstance(step, PromptStep):
        ch = OracleChunk(step.P, step.latent_host[0], 0)
        n_tok = step.n_chunks * step.Q
        ch.query(step.Q - 1, q0=(step.n_chunks - 1) * step.Q)   # untimed: warms the lazy FP4 rows
        n, t0 = 0, time.perf_counter()
        while True:
            t = (n * 40503 + 17) % n_tok                 # tokens spread over the whole prompt
            ch.query(t % step.Q, q0=t - t % step.Q)
            n += 1
            el = time.perf_counter() - t0
            if el >= budget_s:
                break
        return {"value": round(n / el, 4), "unit": "tokens/s", "cores": blas_threads(),
                "kind": "oracle",
                "sample": f"{n} tokens of sequence 0's prompt, spread over its {step.n_chunks} chunks "
                          f"(every layer of the 3 encoder groups, causal visibility) in {el:.1f} s"}
    if isinstance(step, PrefillStep):
        ch = OracleChunk(step.P, step.latent_host[0], 0)
        ch.query(step.Q - 1)                             # untimed: warms the lazy FP4 rows
        n, t0 = 0, time.perf_counter()
        while True:
            ch.query((n * 131) % step.Q)
            n += 1
            el = time.perf_counter() - t0
            if el >= budget_s:
                break
        return {"value": round(n / el, 4), "unit": "tokens/s", "cores": blas_threads(),
                "kind": "oracle",
                "sample": f"{n} queries of sequence 0's chunk (every layer of the encoder group, "
                          f"about {step.lens[0]} visible positions each) in {el:.1f} s"}
    seq = OracleSeq(step.P, step.latent_host[0], step.w.want_pool, step.w.sm_scale, 0)
    seq.step()                                           # untimed: fills the lazy FP4 rows
    n, t0 = 0, time.perf_counter()
    while True:
        seq.step()
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": round(n / el, 4), "unit": "queries/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{n} x the float64 oracle's 20-layer decode step of sequence 0 "
                      f"({step.lens[0]} positions) in {el:.1f} s; numpy elementwise work is "
                      "single-threaded, matmuls use the BLAS threads counted in cores"}


def run_reference(args, rank, world):
    """--impl reference: the float64 oracle timed on the host cores (rank 0 only).  Each
    step runs a bounded sample of the same workload: u consecutive layers of sequence 0's
    decode schedule (u sized so the whole run ends within a few minutes); a query is
    20 layers, so value = (layers run / 20) / time."""
    if rank != 0:
        return None
    import torch
    from fp4_kv_cache_04_b200 import synth

    w = synth.workloads()[args.workload]
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else None
    if dev is None:
        return {"impl": "reference", "unavailable": "the oracle's inputs are drawn with the "
                "CUDA generator; no GPU visible"}
    # the same seeded inputs as the GPU arm (torch's CUDA generator), no library call
    P = synth.make_problem(w, device=dev)
    if w.q_pos is not None:
        return run_reference_prefill(args, world, w, P)
    latent0 = P.latent[: P.lens[0]].cpu()
    P.latent = None
    seq = OracleSeq(P, latent0, w.want_pool, w.sm_scale, 0)
    seq.step()                                           # fills the lazy FP4 rows
    t_layer = []
    for i in range(len(seq.layers)):
        t0 = time.perf_counter()
        seq.layer(i)
        t_layer.append(time.perf_counter() - t0)
    per_query = sum(t_layer)
    budget = 150.0
    n_layers = len(seq.layers)
    u = max(1, min(n_layers, int(budget / max(args.steps + args.warmup, 1) /
                                 (per_query / n_layers))))
    cursor = 0

    def one():
        nonlocal cursor
        for _ in range(u):
            seq.layer(cursor)
            cursor = (cursor + 1) % n_layers

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    el = time.perf_counter() - t0
    value = (args.steps * u / n_layers) / el
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "queries/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "describe": w.describe,
                       "sample_layers_per_step": u}}
    cpu = {"value": line["value"], "unit": "queries/s", "cores": blas_threads(), "kind": "oracle",
           "sample": f"{u} consecutive layer(s) of sequence 0's 20-layer schedule per step"}
    line["cpu_baseline"] = cpu
    line["e2e"] = {"value": line["value"], "unit": "queries/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}
    return line


def run_reference_prefill(args, world, w, P):
    """--impl reference for a prefill chunk: each step runs u of the chunk's queries of
    sequence 0 through every layer of the group on the oracle; value = tokens/s."""
    latent0 = P.latent[: w.ratio * P.lens[0]].cpu()
    P.latent = None
    ch = OracleChunk(P, latent0, 0)
    prompt = w.name.startswith("prefill_prompt")
    n_tok = w.ratio * P.lens[0] if prompt else w.q_per_seq   # tokens the sample cycles over
    t0 = time.perf_counter()
    ch.query(w.q_per_seq - 1, q0=n_tok - w.q_per_seq if prompt else None)
    per_query = time.perf_counter() - t0
    u = max(1, int(150.0 / max(args.steps + args.warmup, 1) / max(per_query, 1e-3)))
    cursor = [0]

    def one():
        for _ in range(u):
            t = cursor[0]
            if prompt:
                ch.query(t % w.q_per_seq, q0=t - t % w.q_per_seq)
            else:
                ch.query(t)
            cursor[0] = (cursor[0] + (40503 if prompt else 131)) % n_tok

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    el = time.perf_counter() - t0
    value = args.steps * u / el
    line = {"impl": "reference", "metric": PROMPT_METRIC if prompt else PREFILL_METRIC,
            "value": round(value, 4), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "describe": w.describe, "sample_queries_per_step": u}}
    line["cpu_baseline"] = {"value": line["value"], "unit": "tokens/s", "cores": blas_threads(),
                            "kind": "oracle",
                            "sample": f"{u} of the {'prompt' if prompt else 'chunk'}'s tokens "
                                      "(sequence 0, every layer) per step"}
    line["e2e"] = {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}
    return line


# ------------------------------------------------------------------ main


def main(argv=None):
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from __graft_entry__ import build
    if rank == 0:
        build()
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        dist.barrier()
        if rank != 0:
            build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    result = run_ours(args, rank, world, dev)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
