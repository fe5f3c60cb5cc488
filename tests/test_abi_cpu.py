"""CPU-only checks of the C ABI: the library loads, exports every entry point that
include/csa2.h declares, and its host-side validation rejects bad arguments before any
CUDA call (nothing here launches a kernel)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa2.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(csa2_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from __graft_entry__ import build
    build()
    from fp4_kv_cache_04_b200 import csa2
    return csa2


def test_header_declares_the_five_stage_entry_points():
    names = declared_functions()
    for n in ["csa2_quantize_kv", "csa2_index_score", "csa2_topk", "csa2_build_pool", "csa2_attend"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(lib.lib(), n)
    assert set(lib.EXPORTED) == set(names)


def test_abi_version_and_status_strings(lib):
    assert lib.abi_version() == 6
    assert lib.status_string(0) == "CSA2_OK"
    assert lib.status_string(3) == "CSA2_ERR_WORKSPACE"
    assert lib.status_string(99) == "CSA2_ERR_UNKNOWN"


def test_host_validation_rejects_before_launch(lib):
    L = lib.lib()
    vp = ctypes.c_void_p
    assert L.csa2_attend(None, None) == 1
    a = lib.LayerArgs()
    a.mode = 7
    assert L.csa2_attend(ctypes.byref(a), None) == 1
    a.mode = lib.MODE_REUSE
    a.batch = 1
    a.q_per_seq = 1
    a.ratio = 1
    a.max_n = 10
    assert L.csa2_attend(ctypes.byref(a), None) == 1          # NULL tensors
    # fake (never dereferenced) aligned addresses: validation must stop at the workspace
    for f in ["kv_offsets", "codes", "scales", "topk_idx", "q", "swa_kv", "out"]:
        setattr(a, f, 1 << 20)
    a.swa_rows = 128
    assert L.csa2_attend(ctypes.byref(a), None) == 3          # no workspace
    a.workspace = (1 << 20) + 8                               # misaligned workspace
    a.workspace_bytes = 1 << 12
    assert L.csa2_attend(ctypes.byref(a), None) == 3
    a.ratio = 3
    assert L.csa2_attend(ctypes.byref(a), None) == 1
    a.ratio = 1
    a.want_pool = 1                                           # pool only for FULL
    assert L.csa2_attend(ctypes.byref(a), None) == 1
    a.want_pool = 0
    a.mode = lib.MODE_REINDEX                                 # Reindex needs indexer + pool
    assert L.csa2_attend(ctypes.byref(a), None) == 1
    a.mode = lib.MODE_REUSE
    a.swa_format = 7                                          # unknown SWA format
    assert L.csa2_attend(ctypes.byref(a), None) == 1
    a.swa_format = lib.SWA_FP8                                # FP8 SWA needs its pointers
    assert L.csa2_attend(ctypes.byref(a), None) == 1
    a.swa_kv8, a.swa_kscale = (1 << 20) + 8, 1 << 20          # misaligned codes
    assert L.csa2_attend(ctypes.byref(a), None) == 1
    a.swa_kv8 = 1 << 20
    a.q_pos, a.q_per_seq = 1 << 20, 4                         # FP8 SWA is decode only
    assert L.csa2_attend(ctypes.byref(a), None) == 2
    a.q_pos, a.q_per_seq, a.swa_format = None, 1, lib.SWA_BF16
    a.q_format = 2                                            # unknown query format
    assert L.csa2_attend(ctypes.byref(a), None) == 1
    a.q_format, a.reserved2 = lib.Q_NVFP4, 1                  # reserved word must be 0
    assert L.csa2_attend(ctypes.byref(a), None) == 1
    a.q_format, a.reserved2 = lib.Q_BF16, 0
    # quantiser
    assert L.csa2_quantize_kv(None, 0, 1, None, None, None, None) == 0   # empty is a no-op
    assert L.csa2_quantize_kv(vp(1 << 20), 3, 2, None, vp(1 << 20), vp(1 << 20), None) == 1
    assert L.csa2_quantize_kv(vp(1 << 20), 4, 3, None, vp(1 << 20), vp(1 << 20), None) == 1
    assert L.csa2_quantize_kv(vp((1 << 20) + 2), 4, 1, None, vp(1 << 20), vp(1 << 20), None) == 1
    # cache append
    f = vp(1 << 20)
    assert L.csa2_append_kv(None, None, 0, None, None, None, None, None, None) == 0   # empty
    assert L.csa2_append_kv(f, f, -1, f, f, f, f, f, None) == 1
    assert L.csa2_append_kv(f, None, 4, f, f, f, f, f, None) == 1                     # NULL
    assert L.csa2_append_kv(vp((1 << 20) + 8), f, 4, f, f, f, f, f, None) == 1        # latent align
    assert L.csa2_append_kv(f, vp((1 << 20) + 4), 4, f, f, f, f, f, None) == 1        # proj align
    assert L.csa2_append_kv(f, f, 4, f, f, f, vp((1 << 20) + 1), f, None) == 1        # idx_k align
    # Top-K
    assert L.csa2_topk(vp(1 << 20), 100, 100, 1, 0, None, 1, vp(1 << 20), None) == 1
    assert L.csa2_topk(vp(1 << 20), 100, 101, 1, 5, None, 1, vp(1 << 20), None) == 1
    assert L.csa2_topk(vp(1 << 20), 100, 100, 0, 5, None, 1, vp(1 << 20), None) == 0
    # pool
    assert L.csa2_build_pool(vp(1 << 20), 64, vp(1 << 20), 1, 64, vp(1 << 20), None, 0, None) == 3


def test_workspace_sizes(lib):
    L = lib.lib()
    a = lib.LayerArgs()
    a.mode, a.batch, a.q_per_seq, a.ratio, a.max_n = lib.MODE_REUSE, 64, 1, 1, 262144
    a.swa_rows = 128
    reuse = L.csa2_workspace_size(ctypes.byref(a))
    assert reuse >= 256                                  # decode: partials merge in a cluster
    a.mode = lib.MODE_FULL
    full = L.csa2_workspace_size(ctypes.byref(a))
    assert full >= reuse + 64 * (262144 // 4096) * 512 * 8  # chunk candidates
    a.want_pool = 1
    assert L.csa2_workspace_size(ctypes.byref(a)) >= full + 64 * 262144 // 8 * 4
    a.mode, a.want_pool = lib.MODE_REINDEX, 0
    assert L.csa2_workspace_size(ctypes.byref(a)) >= reuse + 64 * 2 * 512 * 8
    a.mode, a.q_per_seq, a.q_pos = lib.MODE_FULL, 2048, 1 << 20      # prefill Full: streaming
    a.batch, a.max_n, a.swa_rows = 2, 65536, 2048 + 127             # Top-512, no score matrix
    assert L.csa2_workspace_size(ctypes.byref(a)) == 256
    a.mode, a.pool_blocks = lib.MODE_REINDEX, 1 << 20                # prefill Reindex: scores
    assert L.csa2_workspace_size(ctypes.byref(a)) >= 2 * 2048 * 16384 * 4
    a.pool_blocks = None
    a.mode = lib.MODE_REUSE                      # prefill rows also merge in their cluster
    a.batch, a.q_per_seq = 1, 4
    assert L.csa2_workspace_size(ctypes.byref(a)) == 256
    a.q_format = lib.Q_NVFP4                     # the kernel quantises the query on chip
    assert L.csa2_workspace_size(ctypes.byref(a)) == 256
    a.q_format = lib.Q_BF16
    assert L.csa2_pool_workspace_size(64, 262144) >= 64 * 32768 * 4
