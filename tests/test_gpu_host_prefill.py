"""GPU parity of the prefill from host buffers (tria_prefill_host).

The call splits a prompt by (batch, KV head) group and overlaps each group's copies
in and out with the kernels of its neighbours; it computes exactly what
tria_quantize_kv followed by tria_prefill computes on device buffers. So the cache
it writes and the O and LSE it copies out must equal that path's bit for bit (with
the same fused kernel: per-head policies that differ within every head pair, or
pairs that agree in every group so both paths take the GQA-shared kernel), and O
and LSE must match the oracle on sampled rows. Shapes cover several groups per
sequence, B > 1, both block sizes, two to four staging slots and more groups than
slots.
"""
import numpy as np
import pytest
import torch

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
    # B, Hq, Hkv, S, D, T, per-query-head (hi, keep), staging slots
    "per_head_t64": (2, 8, 2, 1024, 128, 64, [(1, 3), (2, 9), (0, 4), (3, 5), (1, 2), (4, 12), (2, 2), (0, 7)], 2),
    "pairs_t128": (1, 8, 4, 1280, 128, 128, [(1, 4), (1, 4), (2, 6), (2, 6), (0, 3), (0, 3), (3, 8), (3, 8)], 3),
    "d64_g1_t64": (3, 2, 2, 576, 64, 64, [(1, 5), (2, 3)], 4),
}


@pytest.mark.parametrize("name", list(CASES))
def test_host_prefill_equals_device_path(T, oracle_mod, name):
    B, Hq, Hkv, S, D, Tb, pol, slots = CASES[name]
    hi = np.array([p[0] for p in pol], np.int32)
    keep = np.array([p[1] for p in pol], np.int32)
    seed = sum(map(ord, name))
    Q, K, V = seeded((B, Hq, S, D), seed), seeded((B, Hkv, S, D), seed + 1), seeded((B, Hkv, S, D), seed + 2)

    # the device path
    ref_cache = T.CompressedKVCache(B, Hkv, D, Tb, S)
    T.tria_quantize_kv(K.cuda(), V.cuda(), ref_cache)
    O_d, L_d = T.tria_prefill(Q.cuda(), ref_cache, hi, keep)

    # the host path, into a cache whose rows start as garbage
    cache = T.CompressedKVCache(B, Hkv, D, Tb, S)
    cache.buffer[256:].fill_(0x5A)
    hQ, hK, hV = (t.pin_memory() for t in (Q, K, V))
    hO = torch.full((B, Hq, S, D), float("nan"), dtype=torch.bfloat16).pin_memory()
    hL = torch.full((B, Hq, S), float("nan"), dtype=torch.float32).pin_memory()
    run = T.HostPrefill(B, Hq, Hkv, S, D, Tb, slots=slots)
    for _ in range(2):   # twice: the second call reuses the staging slots and workspace
        run(hQ, hK, hV, cache, hi, keep, hO, hL)
    torch.cuda.current_stream().synchronize()
    assert T.tria_workspace_status(run.workspace) == 0
    assert cache.status() == 0

    for p in ("k8", "k4", "k8_scale", "k4_scale", "v8", "v4", "v8_scale", "v4_scale"):
        a, b = cache.plane(p).cpu(), ref_cache.plane(p).cpu()
        assert torch.equal(a.view(torch.uint8) if a.dtype != torch.float32 else a.view(torch.int32),
                           b.view(torch.uint8) if b.dtype != torch.float32 else b.view(torch.int32)), p
    assert torch.equal(hO.view(torch.int16), O_d.cpu().view(torch.int16))
    assert torch.equal(hL.view(torch.int32), L_d.cpu().view(torch.int32))

    # and the oracle, on rows of every head: the first, a middle and the last token
    picks = [(b, h, t) for b in range(B) for h in range(Hq) for t in (0, S // 2 + 3, S - 1)]
    rows = rows_of(B, Hq, S, picks)
    O_ref, L_ref = oracle_mod.prefill_rows(Q, K, V, Tb, hi, keep, rows=rows)
    got_o = torch.stack([hO[b, h, t] for b, h, t in picks])
    got_l = torch.stack([hL[b, h, t] for b, h, t in picks])
    compare_o(got_o, O_ref, f"host prefill {name}")
    compare_lse(got_l, L_ref, f"host prefill {name}")


def test_host_prefill_rejects_bad_arguments_before_any_work(T):
    B, Hq, Hkv, S, D, Tb = 1, 4, 2, 256, 128, 64
    cache = T.CompressedKVCache(B, Hkv, D, Tb, S)
    run = T.HostPrefill(B, Hq, Hkv, S, D, Tb)
    hQ = torch.zeros((B, Hq, S, D), dtype=torch.bfloat16).pin_memory()
    hK = torch.zeros((B, Hkv, S, D), dtype=torch.bfloat16).pin_memory()
    hO = torch.empty_like(hQ)
    hL = torch.empty((B, Hq, S), dtype=torch.float32).pin_memory()
    hi = np.ones(Hq, np.int32)
    keep = np.full(Hq, 3, np.int32)
    # one stream for both copies
    run.copy_out = run.copy_in
    with pytest.raises(T.TriaError) as e:
        run(hQ, hK, hK, cache, hi, keep, hO, hL)
    assert e.value.status == T.TRIA_ERR_INVALID_ARG
    # a cache with fewer tokens than the prompt
    run = T.HostPrefill(B, Hq, Hkv, S, D, Tb)
    small = T.CompressedKVCache(B, Hkv, D, Tb, S // 2)
    with pytest.raises(T.TriaError) as e:
        run(hQ, hK, hK, small, hi, keep, hO, hL)
    assert e.value.status == T.TRIA_ERR_INVALID_ARG
    torch.cuda.synchronize()
