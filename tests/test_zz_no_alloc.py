"""csa2_build_pool_noalloc (the pool step with its scratch in a fixed module array)
against csa2_build_pool (the same step with a caller workspace), through the C ABI.

Calls in a row on one stream: the first at the scratch's full size (64 sequences of up
to 262,144 positions), the second on a smaller ragged batch (a stale entry left by the
first call would show in the second), the third on two sequences of about a million
positions (a wider row pitch, so its rows land at other offsets of the scratch).  Pools
are index sets: compared exactly with the workspace path, and one sampled row of each
call with the float64 oracle's pool selection on the same scores.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import csa2_oracle as O

DEV = "cuda"


@pytest.fixture(scope="module")
def csa2():
    from __graft_entry__ import build
    build()
    from fp4_kv_cache_04_b200 import csa2 as c
    return c


def test_noalloc_pool_size_check_runs_on_the_host(csa2):
    """65 sequences of 262,144 positions need 8,519,680 scratch bytes > 8 MiB: rejected
    before any CUDA call (the pointers are never dereferenced)."""
    fake = 1 << 20
    st = csa2.lib().csa2_build_pool_noalloc(fake, 262144, fake, 65, 262144, fake, None)
    assert st == 2                                                   # CSA2_ERR_UNSUPPORTED
    st = csa2.lib().csa2_build_pool_noalloc(fake, 262144 + 512, fake, 64, 262144 + 512, fake, None)
    assert st == 2
    st = csa2.lib().csa2_build_pool_noalloc(fake, 4, fake, 1, 8, fake, None)
    assert st == 1                                                   # ld < max_n


def _scores(lens, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    B, max_n = len(lens), max(lens)
    s = torch.randn(B, max_n, generator=g, device=DEV).square().mul_(100).round_().div_(100)  # ties
    col = torch.arange(max_n, device=DEV)
    s[col[None, :] >= torch.tensor(lens, device=DEV)[:, None]] = -torch.inf
    offs = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int64, device=DEV)
    return s, offs, max_n


def _with_workspace(csa2, s, offs, max_n):
    pool = torch.full((s.shape[0], 2048), -7, dtype=torch.int32, device=DEV)
    ws = csa2.alloc_workspace(csa2.pool_workspace_size(s.shape[0], max_n))
    csa2.build_pool(s, offs, max_n, pool, ws)
    return pool


def _oracle_row(s, lens, b):
    """The oracle's pool of row b from the same fp32 scores (exact selection)."""
    return O.pool_select(s[b, :lens[b]].double().cpu().numpy())


@pytest.mark.gpu
def test_noalloc_pool_matches_workspace_pool_twice(csa2):
    rng = np.random.default_rng(2048)
    lens1 = [262144] + rng.integers(1, 262145, 63).tolist()
    lens2 = [3, 16391, 5000]
    lens3 = [1 << 20, (1 << 20) - 13]
    s1, o1, m1 = _scores(lens1, 11)
    s2, o2, m2 = _scores(lens2, 12)
    s3, o3, m3 = _scores(lens3, 13)
    assert 64 * m1 * 4 // 8 == csa2.NOALLOC_POOL_SCRATCH_BYTES
    p1 = torch.full((64, 2048), -7, dtype=torch.int32, device=DEV)
    p2 = torch.full((3, 2048), -7, dtype=torch.int32, device=DEV)
    p3 = torch.full((2, 2048), -7, dtype=torch.int32, device=DEV)
    csa2.build_pool_noalloc(s1, o1, m1, p1)
    csa2.build_pool_noalloc(s2, o2, m2, p2)
    csa2.build_pool_noalloc(s3, o3, m3, p3)
    r1 = _with_workspace(csa2, s1, o1, m1)
    r2 = _with_workspace(csa2, s2, o2, m2)
    r3 = _with_workspace(csa2, s3, o3, m3)
    torch.cuda.synchronize()
    assert torch.equal(p1, r1)
    assert torch.equal(p2, r2)
    assert torch.equal(p3, r3)
    assert (p2[0, :1] == 0).all() and (p2[0, 1:] == -1).all()      # 3 positions: block 0 only
    assert np.array_equal(p1[37].cpu().numpy(), _oracle_row(s1, lens1, 37))
    assert np.array_equal(p2[1].cpu().numpy(), _oracle_row(s2, lens2, 1))
    assert np.array_equal(p3[1].cpu().numpy(), _oracle_row(s3, lens3, 1))


@pytest.mark.gpu
def test_noalloc_pool_rejects_more_than_the_scratch(csa2):
    s = torch.zeros(65, 262144, dtype=torch.float32, device=DEV)
    offs = torch.arange(66, dtype=torch.int64, device=DEV) * 262144
    pool = torch.full((65, 2048), -7, dtype=torch.int32, device=DEV)
    st = csa2.lib().csa2_build_pool_noalloc(s.data_ptr(), s.stride(0), offs.data_ptr(), 65, 262144,
                                            pool.data_ptr(), None)
    assert st == 2                                                   # CSA2_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert (pool == -7).all()
