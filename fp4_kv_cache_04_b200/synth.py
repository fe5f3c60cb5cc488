"""Seeded synthetic inputs for the CSA2 workloads.

Shared by the tests, the bench and the smoke check; it holds none of the method's
arithmetic (no quantisation of the main KV, no scores, no selection, no attention).
The one conversion it performs is building the FP8 indexer K the workloads call for:
per-row fp32 scale = amax/448 and torch's own E4M3 cast of k/scale.

Recipe (distributions from the workload definitions; draws in this order from one
torch.Generator seeded with the workload's seed, on the generating device):
  1. ragged lengths (CPU generator, so identical on every device), when ragged;
  2. latent  ~ N(0,1) [tokens][512] -> bf16  (tokens = positions * ratio);
  3. indexer K ~ N(0,1) [positions][64] -> scale amax/448 per row, E4M3 bytes;
  4. per layer: q ~ N(0,1) * q_std [rows][16][512] -> bf16, SWA KV ~ N(0,1)
     [B][swa_rows][512] -> bf16, and for Full / Reindex layers idx_q ~ N(0,1)
     [rows][4][64] -> bf16, idx_w ~ U(0,1) [rows][4] f32;
  5. decode: one new latent row per sequence ~ N(0,1) (the step's cache append), then
     its indexer projection ~ N(0,1) [B][64] fp32 (quantised by the append itself).
Values differ between CPU and CUDA generators; each test states which it uses.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

D, IDX_HEADS, IDX_DIM, HEADS, WINDOW = 512, 4, 64, 16, 128
FULL, REINDEX, REUSE = 0, 1, 2
MODE_NAMES = {FULL: "full", REINDEX: "reindex", REUSE: "reuse"}


def decoder_schedule(n_groups: int = 5, group: int = 4) -> list[int]:
    """Decoder modes (CSA2 section: 5 groups of 4; the first is Full + 3 Reuse, the
    rest Reindex + 3 Reuse)."""
    modes = []
    for gi in range(n_groups):
        modes.append(FULL if gi == 0 else REINDEX)
        modes.extend([REUSE] * (group - 1))
    return modes


def encoder_group_schedule(group: int = 6) -> list[int]:
    """One encoder group (CSA2 section: groups of 6 = 1 Full + 5 Reuse)."""
    return [FULL] + [REUSE] * (group - 1)


@dataclass
class Workload:
    name: str
    seed: int
    batch: int
    lens: list[int] | None           # positions per sequence (None -> ragged, drawn)
    ragged: tuple[int, int] | None
    ratio: int
    modes: list[int]
    q_per_seq: int = 1
    q_pos: list[int] | None = None   # prefill: token of each sequence's first query
    q_std: float = 1.0 / math.sqrt(D)
    sm_scale: float = 1.0
    swa_rows: int = WINDOW
    want_pool: bool = False
    describe: str = ""


def workloads() -> dict[str, Workload]:
    """The workloads, named by what they are (a prompt workload's q_pos / q_per_seq describe
    its first chunk: every chunk has the same shape, its tokens follow the previous one's)."""
    w = {}
    w["decode_full_4k"] = Workload(
        "decode_full_4k", 0, 1, [4096], None, 1, [FULL],
        describe="one Full decode layer, B=1, 4,096 positions")
    w["decoder_group_32k"] = Workload(
        "decoder_group_32k", 1, 8, [32768] * 8, None, 1, [FULL, REUSE, REUSE, REUSE],
        describe="decoder group Full + 3 Reuse, B=8, 32,768 positions each")
    w["prefill_chunk_128k"] = Workload(
        "prefill_chunk_128k", 2, 2, [65536] * 2, None, 2, encoder_group_schedule(),
        q_per_seq=2048, q_pos=[131072 - 2048] * 2, q_std=1.0, sm_scale=1.0 / math.sqrt(D),
        swa_rows=2048 + WINDOW - 1,
        describe="encoder prefill, last 2,048-token chunk of a 131,072-token prompt "
                 "(65,536 ratio-2 positions), Full + 5 Reuse, B=2")
    w["prefill_prompt_128k"] = Workload(
        "prefill_prompt_128k", 5, 2, [65536] * 2, None, 2, encoder_group_schedule() * 3,
        q_per_seq=2048, q_pos=[0] * 2, q_std=1.0, sm_scale=1.0 / math.sqrt(D),
        swa_rows=2048 + WINDOW - 1,
        describe="encoder prefill of a whole 131,072-token prompt (65,536 ratio-2 positions) in "
                 "64 chunks of 2,048 tokens, 3 groups of Full + 5 Reuse per chunk, B=2")
    w["hsi_1m"] = Workload(
        "hsi_1m", 3, 1, [1 << 20], None, 1, [FULL, REINDEX, REINDEX, REINDEX],
        want_pool=True,
        describe="HSI at 1,048,576 positions: Full (pool + Top-512) + 3 Reindex, B=1")
    w["decoder_step_256k"] = Workload(
        "decoder_step_256k", 4, 64, [262144] * 64, None, 1, decoder_schedule(), want_pool=True,
        describe="20-layer decoder decode step, B=64, every context 262,144 positions")
    w["decoder_step_ragged"] = Workload(
        "decoder_step_ragged", 4, 64, None, (65536, 262144), 1, decoder_schedule(),
        want_pool=True,
        describe="20-layer decoder decode step, B=64, contexts ~U[65,536, 262,144]")
    return w


@dataclass
class LayerInputs:
    mode: int
    q: torch.Tensor
    swa: torch.Tensor
    idx_q: torch.Tensor | None = None
    idx_w: torch.Tensor | None = None


@dataclass
class Problem:
    workload: Workload
    lens: list[int]
    kv_offsets: torch.Tensor          # int64 [B+1]
    latent: torch.Tensor | None       # bf16 [tokens][512] (tokens = positions * ratio)
    idx_k: torch.Tensor               # uint8 [positions][64]
    idx_kscale: torch.Tensor          # f32 [positions]
    layers: list[LayerInputs] = field(default_factory=list)
    new_rows: torch.Tensor | None = None   # bf16 [B][512] (decode append)
    q_pos: torch.Tensor | None = None
    new_idx_proj: torch.Tensor | None = None   # fp32 [B][64] (decode append)


def draw_lens(w: Workload) -> list[int]:
    if w.lens is not None:
        return list(w.lens)
    g = torch.Generator().manual_seed(w.seed)
    lo, hi = w.ragged
    return torch.randint(lo, hi + 1, (w.batch,), generator=g).tolist()


def fp8_rows(k: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """FP8 E4M3 rows with a per-row fp32 scale amax/448 (torch's cast)."""
    scale = (k.abs().amax(dim=1) / 448.0).clamp_min(1e-30)
    k8 = (k / scale[:, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return k8.contiguous(), scale.to(torch.float32).contiguous()


def fp8_swa(swa: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """bf16 SWA KV [B][rows][512] -> FP8 variant: E4M3 codes [B][rows][512] and fp32 row
    scales [B][rows] (scale amax/448, torch's E4M3 cast of x/scale; zero rows get 0)."""
    x = swa.float().reshape(-1, swa.shape[-1])
    amax = x.abs().amax(dim=1)
    scale = amax / 448.0
    safe = torch.where(scale > 0, scale, torch.ones_like(scale))
    codes = (x / safe[:, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    codes = torch.where(scale[:, None] > 0, codes, torch.zeros_like(codes))
    return (codes.reshape(swa.shape).contiguous(),
            scale.reshape(swa.shape[:-1]).to(torch.float32).contiguous())


def make_problem(w: Workload, device="cpu", lens: list[int] | None = None,
                 with_latent: bool = True, layers: int | None = None,
                 chunk_rows: int = 1 << 22) -> Problem:
    """Draws a workload's inputs (optionally with overridden lengths / layer count)."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(w.seed)
    lens = list(lens) if lens is not None else draw_lens(w)
    offs = [0]
    for n in lens:
        offs.append(offs[-1] + n)
    total = offs[-1]
    kv_offsets = torch.tensor(offs, dtype=torch.int64, device=device)
    latent = None
    if with_latent:
        latent = torch.empty(total * w.ratio, D, dtype=torch.bfloat16, device=device)
        for r0 in range(0, total * w.ratio, chunk_rows):
            r1 = min(r0 + chunk_rows, total * w.ratio)
            latent[r0:r1] = torch.randn(r1 - r0, D, generator=g, device=device).to(torch.bfloat16)
    k8 = torch.empty(total, IDX_DIM, dtype=torch.uint8, device=device)
    ks = torch.empty(total, dtype=torch.float32, device=device)
    for r0 in range(0, total, chunk_rows):
        r1 = min(r0 + chunk_rows, total)
        k = torch.randn(r1 - r0, IDX_DIM, generator=g, device=device)
        k8[r0:r1], ks[r0:r1] = fp8_rows(k)
    rows = w.batch * w.q_per_seq
    modes = w.modes if layers is None else w.modes[:layers]
    ls = []
    for m in modes:
        q = (torch.randn(rows, HEADS, D, generator=g, device=device) * w.q_std).to(torch.bfloat16)
        swa = torch.randn(w.batch, w.swa_rows, D, generator=g, device=device).to(torch.bfloat16)
        li = LayerInputs(m, q, swa)
        if m != REUSE:
            li.idx_q = torch.randn(rows, IDX_HEADS, IDX_DIM, generator=g,
                                   device=device).to(torch.bfloat16)
            li.idx_w = torch.rand(rows, IDX_HEADS, generator=g, device=device)
        ls.append(li)
    new_rows = new_proj = None
    if w.q_pos is None:
        new_rows = torch.randn(w.batch, D, generator=g, device=device).to(torch.bfloat16)
        new_proj = torch.randn(w.batch, IDX_DIM, generator=g, device=device)
    q_pos = None
    if w.q_pos is not None:
        q_pos = torch.tensor(w.q_pos, dtype=torch.int64, device=device)
    return Problem(w, lens, kv_offsets, latent, k8, ks, ls, new_rows, q_pos, new_proj)


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
