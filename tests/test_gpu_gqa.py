"""GPU parity of the GQA-shared fused prefill.

When the query heads of a KV group share their boundaries (hi, keep), one CTA
serves two of them and brings every kept K/V block on chip once for both (llmis.ru
chapter 3.5, section 4: the heads of a group read the same K and V). The result
must be the per-head computation's: every case here is checked against the
oracle element by element, with the shared kernel allowed and then forbidden
(tria_prefill_gqa), and both outputs must agree with each other within the
parity bound. Cases cover both block sizes and head dims, 2 and 4 query heads per
KV head, ragged query tiles, hi = 0, a 4-bit-only band and the 8,192-token shapes
with one policy per KV head (sampled rows).
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


def seeded(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


CASES = {
    # B, Hq, Hkv, D, T, S, per-KV-head (hi, keep)
    "t64_d128_g4": (1, 8, 2, 128, 64, 1216, [(1, 3), (0, 9)]),
    "t128_d128_g2": (2, 4, 2, 128, 128, 1024, [(2, 5), (1, 1)]),
    "t64_d64_g2": (1, 4, 2, 64, 64, 640, [(0, 0), (3, 40)]),
    "t128_d64_g4": (1, 4, 1, 64, 128, 768, [(1, 6)]),
    "t64_int4_band": (1, 4, 1, 128, 64, 896, [(1, 100)]),
}


@pytest.mark.parametrize("name", list(CASES))
def test_gqa_shared_prefill_matches_oracle_and_per_head(T, oracle_mod, name):
    B, Hq, Hkv, D, Tb, S, pol = CASES[name]
    G = Hq // Hkv
    hi = np.array([pol[h // G][0] for h in range(Hq)], np.int32)
    keep = np.array([pol[h // G][1] for h in range(Hq)], np.int32)
    Q, K, V = seeded((B, Hq, S, D), 61), seeded((B, Hkv, S, D), 62), seeded((B, Hkv, S, D), 63)
    cache = T.CompressedKVCache(B, Hkv, D, Tb, S)
    T.tria_quantize_kv(K.cuda(), V.cuda(), cache)
    prev = T.tria_prefill_gqa(True)
    try:
        O_s, L_s = T.tria_prefill(Q.cuda(), cache, hi, keep)
        T.tria_prefill_gqa(False)
        O_h, L_h = T.tria_prefill(Q.cuda(), cache, hi, keep)
        torch.cuda.synchronize()
    finally:
        T.tria_prefill_gqa(prev)
    O_ref, L_ref = oracle_mod.prefill_rows(Q, K, V, Tb, hi, keep)
    compare_o(O_s, O_ref.reshape(B, Hq, S, D), f"gqa shared {name}")
    compare_lse(L_s, L_ref.reshape(B, Hq, S), f"gqa shared {name}")
    compare_o(O_h, O_ref.reshape(B, Hq, S, D), f"gqa per head {name}")
    d = (O_s.float() - O_h.float()).abs().max().item()
    assert d <= 2e-2, f"shared and per-head outputs differ by {d}"


def test_gqa_shared_prefill_full_size_sampled_rows(T, oracle_mod):
    """The 8,192-token shapes with one policy per KV head, as the benchmark runs them."""
    w = W.WORKLOADS["llama_prefill_gqa"]
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
    rng = np.random.RandomState(7)
    picks = [(0, h, t) for h in (0, 1, 2, 3, w.Hq - 2, w.Hq - 1) for t in (0, 1, w.T - 1, w.T, w.S // 2, w.S - 1)]
    for h in range(0, w.Hq, 5):      # one whole 128-row query tile of every fifth head
        tile = (h * 29 + 3) % (w.S // 128)
        picks += [(0, h, tile * 128 + r) for r in range(128)]
    picks += [(0, int(rng.randint(w.Hq)), int(rng.randint(w.S))) for _ in range(200)]
    rows = rows_of(w.B, w.Hq, w.S, picks)
    O_ref, L_ref = oracle_mod.prefill_rows(Q.cpu(), K.cpu(), V.cpu(), w.T, hi, keep, rows=rows)
    idx = torch.from_numpy(rows)
    compare_o(O.reshape(-1, w.D).cpu()[idx], O_ref, "gqa shared llama sampled")
    compare_lse(L.reshape(-1).cpu()[idx], L_ref, "gqa shared llama sampled")
