"""Host-side accounting of the benchmark, on the CPU: the work share that scales the
oracle's timed subset to the whole workload, and the subsets themselves."""
import sys
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent.parent
sys.path.insert(0, str(ROOT))

import bench  # noqa: E402
from block_sparse_mixed_b200 import workloads as W  # noqa: E402


def brute_kept_keys(oracle_mod, w, hi, keep, b, h, t):
    """Keys u <= t whose tile with t's query block is kept, by the oracle's tile action."""
    i = t // w.T
    n = 0
    for u in range(t + 1):
        a = oracle_mod.action(i, u // w.T, int(hi[h]), int(keep[h]))
        n += a in (oracle_mod.INT8, oracle_mod.INT4)
    return n


def test_kept_keys_per_row_equal_brute_force(oracle_mod):
    w = W.scaled(W.WORKLOADS["llama_prefill"], S=1024, Hq=4, Hkv=1)
    hi, keep = np.array([1, 0, 3, 2], np.int32), np.array([3, 0, 9, 2], np.int32)
    rng = np.random.RandomState(0)
    picks = [(0, int(rng.randint(4)), int(rng.randint(w.S))) for _ in range(200)]
    picks += [(0, h, t) for h in range(4) for t in (0, 1, 63, 64, 65, 1023)]
    got = bench.kept_keys_of_rows(w, hi, keep, picks)
    want = [brute_kept_keys(oracle_mod, w, hi, keep, *p) for p in picks]
    assert got.tolist() == want


def test_subsets_are_fixed_and_small():
    w = W.WORKLOADS["max_prefill"]
    a = bench.prefill_subset(w, block_phase=15)
    assert a == bench.prefill_subset(w, block_phase=15)           # deterministic
    assert len(a) == w.B * w.Hq * (w.nb // 16) * (w.T // 8)
    assert all(t // w.T % 16 == 15 and t % 8 == 7 for _, _, t in a)
    ref = bench.prefill_subset(w, block_phase=3, row_stride=16)
    assert all(t // w.T % 16 == 3 for _, _, t in ref)
    tiny = W.WORKLOADS["tiny_prefill"]                              # small enough to take whole
    assert len(bench.prefill_subset(tiny, block_phase=0)) == tiny.B * tiny.Hq * tiny.S


def test_decode_bytes_count_union_of_planes():
    # one KV group of two heads, kv_len 3 blocks + 5 tokens (T = 64, D = 128)
    B, Hq, Hkv, D, T = 1, 2, 1, 128, 64
    kv = [3 * 64 + 5]
    hi, keep = [1, 0], [2, 4]
    # query block 3 (partial, 5 tokens): both heads int8 on blocks 0 and 3; head 0
    # int4 at d = 1 (block 2); head 1 int4 at d = 1, 2 (blocks 2, 1)
    full8, full4 = 2 * 64 * D + 2 * 64 * 4, 2 * 64 * D // 2 + 2 * 64 * 4
    part8 = 2 * 5 * D + 2 * 5 * 4
    want = full8 + part8 + 2 * full4 + B * Hq * D * 2 + B * Hq * (D * 2 + 4)
    assert bench.decode_bytes(B, Hq, Hkv, D, T, kv, hi, keep) == want


def test_peaks_file_read_or_fallback(tmp_path, monkeypatch):
    """A measured-peaks file with the expected keys is used; one without them (or
    unreadable) falls back to the fixed figures instead of stopping the run."""
    import json
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    assert bench.load_peaks()[1] == "fallback"
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 7000, "bf16_tflops": 1600}))
    peaks, src = bench.load_peaks()
    assert src == "measured" and peaks["hbm_gbs"] == 7000.0 and peaks["bf16_tflops_sustained"] == 1600.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm": 1}))
    assert bench.load_peaks()[1] == "fallback"
    (tmp_path / "MEASURED_PEAKS.json").write_text("not json")
    assert bench.load_peaks()[1] == "fallback"
