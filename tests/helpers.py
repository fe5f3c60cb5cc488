"""Test-side glue: runs the float64 oracle on the same inputs as the CUDA library and
compares the two by the acceptance rules of the CSA2 path:
  * FP4 codes and E4M3 scales bit-exact;
  * Top-K index sets equal except for positions whose oracle score lies within 1e-5
    relative of the K-th oracle score (and the same number of valid entries);
  * attention outputs (fp32) with relative L2 <= 1e-3 and max abs error <= 5e-3.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import csa2_oracle as O

TIE_REL = 1e-5
ATT_REL_L2 = 1e-3
ATT_MAX_ABS = 5e-3


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def topk_tie_check(gpu_idx: np.ndarray, oracle_idx: np.ndarray, score_of, kth_score: float,
                   where: str = "") -> int:
    """Compares two Top-K lists (ascending, -1 padded).  score_of(pos) -> oracle score.
    Returns the number of positions that differ (all inside the tie band)."""
    g = set(int(x) for x in gpu_idx if x >= 0)
    o = set(int(x) for x in oracle_idx if x >= 0)
    assert len(g) == len(o), f"{where}: valid counts differ {len(g)} vs {len(o)}"
    assert list(gpu_idx[gpu_idx >= 0]) == sorted(g), f"{where}: GPU indices not ascending"
    assert (gpu_idx[len(g):] == -1).all(), f"{where}: padding"
    diff = g ^ o
    for p in diff:
        s = score_of(p)
        assert abs(s - kth_score) <= TIE_REL * abs(kth_score), \
            f"{where}: position {p} score {s} not within the tie band of {kth_score}"
    return len(diff)


def attention_check(gpu_out: np.ndarray, oracle_out: np.ndarray, where: str = "") -> tuple[float, float]:
    gpu_out = np.asarray(gpu_out, dtype=np.float64)
    err = gpu_out - oracle_out
    rel = np.linalg.norm(err) / max(np.linalg.norm(oracle_out), 1e-300)
    mx = np.abs(err).max()
    assert rel <= ATT_REL_L2, f"{where}: relative L2 {rel:.3e} > {ATT_REL_L2}"
    assert mx <= ATT_MAX_ABS, f"{where}: max abs {mx:.3e} > {ATT_MAX_ABS}"
    return rel, mx


class OracleFP4:
    """The oracle's own E2M1 codes (which=0) or E4M3 scales (which=1) of bf16 latent rows
    (after ratio-2 compression when ratio is 2), quantised on first use: a check only
    touches the rows it gathers, and no oracle input comes from the CUDA path.  Supports
    row slices (views sharing the memo) and index arrays, like the arrays it stands for."""

    def __init__(self, latent_bits, ratio=1, which=0, base=0, n=None, memo=None):
        self.latent = latent_bits
        self.ratio = ratio
        self.which = which
        self.base = base
        self.n = latent_bits.shape[0] // ratio if n is None else n
        self.memo = {} if memo is None else memo
        self.shape = (self.n, 256 if which == 0 else 32)

    def _fill(self, rows):
        need = sorted({int(r) for r in rows if int(r) not in self.memo})
        if not need:
            return
        if self.ratio == 1:
            x = self.latent[need]
        else:
            pairs = np.stack([self.latent[[2 * j, 2 * j + 1]] for j in need])
            x = np.concatenate([O.compress_ratio2(pr) for pr in pairs])
        c, sc = O.quantize_rows(x)
        for j, cj, sj in zip(need, c, sc):
            self.memo[j] = (cj, sj)

    def __len__(self):
        return self.n

    def __getitem__(self, idx):
        if isinstance(idx, slice):
            start, stop, step = idx.indices(self.n)
            assert step == 1
            return OracleFP4(self.latent, self.ratio, self.which, self.base + start, stop - start, self.memo)
        rows = np.asarray(idx)
        flat = rows.reshape(-1) + self.base
        self._fill(flat)
        if flat.size == 0:
            return np.zeros(rows.shape + (self.shape[1],), np.uint8)
        return np.stack([self.memo[int(r)][self.which] for r in flat]).reshape(rows.shape + (self.shape[1],))


def oracle_fp4(latent: torch.Tensor, ratio: int = 1) -> tuple[OracleFP4, OracleFP4]:
    """(codes, scales) of the oracle's own quantisation of a bf16 latent tensor."""
    lb = bits(latent)
    c = OracleFP4(lb, ratio, 0)
    return c, OracleFP4(lb, ratio, 1, memo=c.memo)


class SeqView:
    """Host copies of one sequence's caches, for the oracle."""

    def __init__(self, codes, scales, idx_k, idx_kscale, kv_offsets, b):
        o0, o1 = int(kv_offsets[b]), int(kv_offsets[b + 1])
        self.n = o1 - o0
        self.codes = codes[o0:o1]
        self.scales = scales[o0:o1]
        self.idx_k = idx_k[o0:o1]
        self.idx_kscale = idx_kscale[o0:o1]


def oracle_scores(view: SeqView, idx_q_bits, idx_w, positions) -> np.ndarray:
    keys = O.indexer_keys(view.idx_k[positions], view.idx_kscale[positions])
    return O.index_scores(idx_q_bits, idx_w, keys)


def score_tolerance(view: SeqView, idx_q_bits, idx_w, positions) -> np.ndarray:
    """Bound on the fp32 error of a score: 2e-6 * kscale * sum_h w_h sum_d |q k8| (64
    exact products summed in fp32, then the ReLU-weighted head sum and the row scale;
    2e-6 ~ 32 * 2^-24 covers the rounding steps with margin)."""
    q = np.abs(O.bf16_to_f64(idx_q_bits).reshape(4, 64))
    w = np.abs(np.asarray(idx_w, dtype=np.float64))
    k = np.abs(O.E4M3_TABLE[view.idx_k[positions]])
    mag = (k @ q.T) @ w * np.asarray(view.idx_kscale[positions], dtype=np.float64)
    return 2e-6 * mag + 1e-30
