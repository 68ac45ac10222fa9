"""GPU parity at the benchmark's full sizes and launch configuration.

The inputs are drawn on the device (the same seeded recipe as the benchmark). The
fused prefill and the decode run exactly as bench.py runs them. The oracle then
recomputes sampled outputs one by one from copies of the same inputs: query rows
for prefill, whole sequences for decode.
"""
import numpy as np
import pytest
import torch

from block_sparse_mixed_b200 import workloads as W
from parity import compare_lse, compare_o, rows_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    from block_sparse_mixed_b200.build import build
    build()
    from block_sparse_mixed_b200 import tria
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return tria


def run_prefill_like_bench(T, w):
    Q, K, V = W.prefill_inputs(w, device="cuda")
    hi, keep = W.policy(w)
    cache = T.CompressedKVCache(w.B, w.Hkv, w.D, w.T, w.S)
    T.tria_quantize_kv(K, V, cache)
    ws = torch.empty(T.tria_prefill_workspace_bytes(w.B, w.Hq, w.Hkv, w.S, w.D, w.T), dtype=torch.uint8,
                     device="cuda")
    O, L = torch.empty_like(Q), torch.empty((w.B, w.Hq, w.S), dtype=torch.float32, device="cuda")
    T.tria_prefill_prepare(Q, cache, ws)
    T.tria_prefill_attend(cache, hi, keep, ws, O, L)
    torch.cuda.synchronize()
    assert T.tria_workspace_status(ws) == 0
    return Q, K, V, hi, keep, cache, O, L


def sampled_picks(w, n_random, seed):
    """Edge rows of the first and last head of every sequence, one whole 128-row query
    tile of every head (the last tile for even heads, where rows keep the most blocks;
    a tile spread over the sequence for odd heads; sequence b = head mod B), and
    random rows."""
    rng = np.random.RandomState(seed)
    edges = (0, 1, w.T - 1, w.T, w.S // 2, w.S - w.T, w.S - 1)
    picks = [(b, h, t) for b in range(w.B) for h in (0, w.Hq - 1) for t in edges]
    n_tiles = w.S // 128
    for h in range(w.Hq):
        tile = n_tiles - 1 if h % 2 == 0 else (h * 37 + 5) % n_tiles
        picks += [(h % w.B, h, tile * 128 + r) for r in range(128)]
    picks += [(int(rng.randint(w.B)), int(rng.randint(w.Hq)), int(rng.randint(w.S))) for _ in range(n_random)]
    return picks


def check_rows(oracle_mod, w, Q, K, V, hi, keep, O, L, picks, name):
    rows = rows_of(w.B, w.Hq, w.S, picks)
    O_ref, L_ref = oracle_mod.prefill_rows(Q.cpu(), K.cpu(), V.cpu(), w.T, hi, keep, rows=rows)
    idx = torch.from_numpy(rows)
    compare_o(O.reshape(-1, w.D).cpu()[idx], O_ref, name)
    compare_lse(L.reshape(-1).cpu()[idx], L_ref, name)


def test_long_prefill_full_size_sampled_rows(T, oracle_mod):
    """Batch 2 x 32768 tokens, T = 128, a quarter of the causal tiles kept."""
    w = W.WORKLOADS["long_prefill"]
    Q, K, V, hi, keep, _, O, L = run_prefill_like_bench(T, w)
    check_rows(oracle_mod, w, Q, K, V, hi, keep, O, L, sampled_picks(w, 96, 1), "long_prefill sampled")


def test_max_prefill_gqa_full_size_sampled_rows(T, oracle_mod):
    """65536 tokens, T = 128, one (hi, keep) per KV head: the GQA-shared kernel at the
    longest context, on the same sampled rows as the per-head case."""
    w = W.WORKLOADS["max_prefill_gqa"]
    hi, keep = W.policy(w)
    G = w.Hq // w.Hkv
    assert all(hi[h] == hi[h + 1] and keep[h] == keep[h + 1] for h in range(0, w.Hq, 2)) and G % 2 == 0
    Q, K, V, hi, keep, _, O, L = run_prefill_like_bench(T, w)
    check_rows(oracle_mod, w, Q, K, V, hi, keep, O, L, sampled_picks(w, 64, 4), "max_prefill_gqa sampled")


def test_max_prefill_full_size_sampled_rows_and_cache(T, oracle_mod):
    """65536 tokens, T = 128; also the compressed cache it writes, bit for bit on sampled tokens."""
    w = W.WORKLOADS["max_prefill"]
    Q, K, V, hi, keep, cache, O, L = run_prefill_like_bench(T, w)
    check_rows(oracle_mod, w, Q, K, V, hi, keep, O, L, sampled_picks(w, 96, 2), "max_prefill sampled")
    rng = np.random.RandomState(3)
    toks = np.unique(np.concatenate([[0, w.S - 1], rng.randint(0, w.S, 62)]))
    for X, p in ((K, "k"), (V, "v")):
        for kvh in (0, w.Hkv - 1):
            rows = X[0, kvh, torch.from_numpy(toks).cuda()].cpu()
            c8, s8, c4, s4 = oracle_mod.quantize_rows(rows, w.D)
            sel = torch.from_numpy(toks)
            assert np.array_equal(cache.plane(p + "8")[0, kvh].cpu()[sel].numpy(), c8)
            assert np.array_equal(cache.plane(p + "4")[0, kvh].cpu()[sel].numpy(), oracle_mod.pack_int4(c4))
            assert np.array_equal(cache.plane(p + "8_scale")[0, kvh].cpu()[sel].numpy().view(np.uint32),
                                  s8.view(np.uint32))
            assert np.array_equal(cache.plane(p + "4_scale")[0, kvh].cpu()[sel].numpy().view(np.uint32),
                                  s4.view(np.uint32))


def test_decode_full_batch_all_sequences(T, oracle_mod):
    """All 64 sequences of 32768 tokens in one launch (the benchmark's item plan), each
    recomputed by the oracle over its whole kept cache."""
    w = W.WORKLOADS["decode"]
    q, K, V, kv_len = W.decode_inputs(w, device="cuda")
    hi, keep = W.policy(w)
    cache = T.CompressedKVCache(w.B, w.Hkv, w.D, w.T, w.S)
    T.tria_quantize_kv(K, V, cache)
    ws = torch.empty(T.tria_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, w.T, w.S), dtype=torch.uint8,
                     device="cuda")
    O, L = T.tria_decode(q, cache, kv_len, hi, keep, workspace=ws)
    torch.cuda.synchronize()
    assert T.tria_workspace_status(ws) == 0
    O_ref = np.empty((w.B, w.Hq, w.D))
    L_ref = np.empty((w.B, w.Hq))
    for b in range(w.B):      # one sequence per oracle call bounds its host memory
        O_ref[b:b + 1], L_ref[b:b + 1] = oracle_mod.decode(q[b:b + 1].cpu(), K[b:b + 1].cpu(), V[b:b + 1].cpu(),
                                                           w.T, kv_len[b:b + 1], hi, keep)
    compare_o(O, O_ref, "decode all 64 sequences")
    compare_lse(L, L_ref, "decode all 64 sequences")
