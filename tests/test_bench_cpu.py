"""Host-side accounting of bench.py (no GPU): the DRAM-traffic gate, the peak file and
the default timing arguments."""
from __future__ import annotations

import json
import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


@pytest.fixture()
def bench():
    import bench as b
    return b


def _copy_tree(tmp_path):
    """A copy of the files the traffic gate reads: the profile and the scan sources."""
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    (root / "fp4_kv_cache_04_b200" / "csrc").mkdir(parents=True)
    shutil.copy(os.path.join(ROOT, "profiles", "scan_select_full_b8_256k.md"), root / "profiles")
    for f in ("scan_select.cu", "select.cuh", "tc.cuh", "common.cuh", "kernels.cuh"):
        shutil.copy(os.path.join(ROOT, "fp4_kv_cache_04_b200", "csrc", f), root / "fp4_kv_cache_04_b200" / "csrc")
    return root


def test_traffic_is_reported_for_the_captured_sources(bench):
    lens = [262144] * 64
    t = bench.scan_traffic_per_launch(lens)
    assert t is not None
    # the capture reads each indexer byte once: traffic within 10% above the algorithmic bytes
    algorithmic = sum(lens) * bench.IDX_ROW_BYTES
    assert algorithmic <= t <= 1.10 * algorithmic
    # scaled by positions
    assert bench.scan_traffic_per_launch([262144] * 32) == pytest.approx(t / 2, rel=1e-6)


def test_traffic_is_withheld_once_a_scan_source_changes(bench, tmp_path, monkeypatch):
    root = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.scan_traffic_per_launch([262144] * 64) is not None
    with open(root / "fp4_kv_cache_04_b200" / "csrc" / "select.cuh", "a") as f:
        f.write("\n// edited\n")
    assert bench.scan_traffic_per_launch([262144] * 64) is None


def test_traffic_is_withheld_without_the_profile(bench, tmp_path, monkeypatch):
    root = _copy_tree(tmp_path)
    os.remove(root / "profiles" / "scan_select_full_b8_256k.md")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.scan_traffic_per_launch([262144] * 64) is None


def test_measured_peak_file_and_fallback(bench, tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    gbs, kind = bench.measured_peaks()
    assert kind == "fallback" and gbs == bench.HBM_FALLBACK_GBS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6000.5}))
    gbs, kind = bench.measured_peaks()
    assert kind == "measured" and gbs == 6000.5


def test_default_timing_arguments(bench):
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.steps >= 1
    assert a.impl == "ours" and not a.reuse_cache and not a.no_graph
    # the step counts default by workload (a whole prompt is about a second per step);
    # every default keeps at least 3 warm-up steps, and explicit values always win
    for wl, steps, warmup in [("decoder_step_256k", 300, 10), ("prefill_chunk_128k", 50, 10),
                              ("prefill_prompt_128k", 3, 3)]:
        a = bench.parse_args(["--workload", wl])
        assert (a.steps, a.warmup) == (steps, warmup)
        a = bench.parse_args(["--workload", wl, "--steps", "7", "--warmup", "4"])
        assert (a.steps, a.warmup) == (7, 4)


def test_algorithmic_bytes_of_the_headline_step(bench):
    # decoder schedule FUUURUUURUUURUUURUUU at 262,144 positions, worked by hand:
    #   Full scan 262,144 x 68 B; the pool's 16,384 indexer rows once (4 Reindex layers);
    #   5 distinct Top-512 selections x 288 B rows; 20 layers x (128 SWA rows x 1 KB +
    #   16 KB q + 32 KB fp32 out); 5 x (indexer q 512 B + weights 16 B); the append
    #   (1 KB latent in, 288 B + 68 B rows out, 256 B indexer values in)
    modes = [0, 2, 2, 2, 1, 2, 2, 2, 1, 2, 2, 2, 1, 2, 2, 2, 1, 2, 2, 2]
    expected = (17825792 + 1114112 + 737280 + 20 * (131072 + 16384 + 32768) + 5 * 528
                + 1024 + 288 + 256 + 68)
    assert bench.algorithmic_bytes_per_seq(262144, modes) == expected


def test_whole_prompt_workload_shape():
    # a 131,072-token prompt at ratio 2 (65,536 positions) in 2,048-token chunks, three
    # encoder groups (Full + 5 Reuse) per chunk, starting at token 0
    from fp4_kv_cache_04_b200 import synth
    w = synth.workloads()["prefill_prompt_128k"]
    assert w.modes == ([synth.FULL] + [synth.REUSE] * 5) * 3
    assert all(w.ratio * n == 64 * w.q_per_seq for n in w.lens) and w.q_pos == [0] * w.batch
    assert w.swa_rows == w.q_per_seq + 127


def test_whole_prompt_flops(bench):
    # PromptStep.flops over a tiny prompt, worked by hand: 2 chunks of 4 tokens at ratio 2
    # (4 positions), one Full + one Reuse layer; token t sees min(4, (t + 1) // 2) positions
    # and min(128, t + 1) window rows
    from fp4_kv_cache_04_b200 import synth

    class Tiny:
        n_chunks, Q, lens, B = 2, 4, [4], 1
        w = type("W", (), {"ratio": 2})()
        P = type("P", (), {"layers": [type("L", (), {"mode": 0})(), type("L", (), {"mode": 2})()]})()
        visible = bench.PromptStep.visible
    Tiny.synth = synth
    vis = [0, 1, 1, 2, 2, 3, 3, 4]
    idx, att = bench.PromptStep.flops(Tiny())
    assert idx == sum(vis) * bench.PREFILL_INDEX_FLOPS_PER_POS
    assert att == 2 * sum(bench.attention_flops_per_query(v, t + 1) for t, v in enumerate(vis))
