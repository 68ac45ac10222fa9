"""GPU parity of step-by-step generation over the compressed cache.

The rit.work TriAttention page (section "Как калибровка распределяет вычисления
между головами", last paragraph) has the prepared K/V of the prompt written to a
compressed cache that step-by-step generation then reads, with the same per-head
boundaries. This test runs that loop through the C ABI: a fused prefill of S0
tokens, then for more than two blocks' worth of steps one token is appended to
the cache (tria_quantize_kv with S = 1 at its position) and decoded
(tria_decode with kv_len = position + 1). Every step is checked against the
oracle's decode over the same tokens, so the loop crosses into new diagonal
blocks (kv_len % T == 1), runs through partial blocks and moves every head's
bands by one block at each boundary. The appended cache rows are compared bit
for bit with the oracle's codec.
"""
import numpy as np
import pytest
import torch

from parity import compare_lse, compare_o

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
    # (B, Hq, Hkv, D, T, S0, steps, hi per head, keep per head)
    "T64": (2, 4, 2, 128, 64, 128, 2 * 64 + 7, [0, 1, 2, 1], [1, 3, 4, 2]),
    "T128": (1, 8, 2, 128, 128, 256, 2 * 128 + 3, [1, 2, 0, 3, 1, 1, 2, 4], [2, 3, 1, 5, 1, 4, 2, 4]),
}


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_then_generate_matches_oracle(T, oracle_mod, name):
    B, Hq, Hkv, D, Tb, S0, steps, hi, keep = CASES[name]
    hi, keep = np.array(hi, np.int32), np.array(keep, np.int32)
    cap = ((S0 + steps + Tb - 1) // Tb) * Tb
    K = seeded((B, Hkv, cap, D), 1)
    V = seeded((B, Hkv, cap, D), 2)
    Q0 = seeded((B, Hq, S0, D), 3)
    Qg = seeded((B, Hq, steps, D), 4)       # the query of each generated token
    cache = T.CompressedKVCache(B, Hkv, D, Tb, cap)

    # prompt: cache write and fused prefill
    T.tria_quantize_kv(K[:, :, :S0].contiguous().cuda(), V[:, :, :S0].contiguous().cuda(), cache)
    O, L = T.tria_prefill(Q0.cuda(), cache, hi, keep)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle_mod.prefill_rows(Q0, K[:, :, :S0].contiguous(), V[:, :, :S0].contiguous(), Tb, hi, keep)
    compare_o(O, O_ref.reshape(B, Hq, S0, D), f"{name} prompt")
    compare_lse(L, L_ref.reshape(B, Hq, S0), f"{name} prompt")

    ws = torch.empty(T.tria_decode_workspace_bytes(B, Hq, Hkv, D, Tb, cap), dtype=torch.uint8, device="cuda")
    Kd, Vd = K.cuda(), V.cuda()
    crossings = 0
    for s in range(steps):
        pos = S0 + s
        T.tria_quantize_kv(Kd[:, :, pos:pos + 1].contiguous(), Vd[:, :, pos:pos + 1].contiguous(), cache, start=pos)
        kv_len = np.full(B, pos + 1, np.int32)
        q = Qg[:, :, s].contiguous()
        Od, Ld = T.tria_decode(q.cuda(), cache, kv_len, hi, keep, workspace=ws)
        torch.cuda.synchronize()
        assert T.tria_workspace_status(ws) == 0
        Or, Lr = oracle_mod.decode(q, K, V, Tb, kv_len, hi, keep)
        compare_o(Od, Or, f"{name} step {s} (kv_len {pos + 1})")
        compare_lse(Ld, Lr, f"{name} step {s} (kv_len {pos + 1})")
        crossings += (pos + 1) % Tb == 1

    assert crossings >= 2
    # the appended rows, bit for bit
    gen = slice(S0, S0 + steps)
    for X, p in ((K, "k"), (V, "v")):
        c8, s8, c4, s4 = oracle_mod.quantize_rows(X[:, :, gen].contiguous(), D)
        c8 = c8.reshape(B, Hkv, steps, D)
        assert np.array_equal(cache.plane(p + "8")[:, :, gen].cpu().numpy(), c8)
        assert np.array_equal(cache.plane(p + "4")[:, :, gen].cpu().numpy(),
                              oracle_mod.pack_int4(c4).reshape(B, Hkv, steps, D // 2))
        assert np.array_equal(cache.plane(p + "8_scale")[:, :, gen].cpu().numpy().view(np.uint32),
                              s8.reshape(B, Hkv, steps).view(np.uint32))
        assert np.array_equal(cache.plane(p + "4_scale")[:, :, gen].cpu().numpy().view(np.uint32),
                              s4.reshape(B, Hkv, steps).view(np.uint32))
