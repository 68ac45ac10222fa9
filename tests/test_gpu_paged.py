"""GPU parity of the paged compressed cache.

The rit.work TriAttention page (section "Когда TriAttention меняет планы
инфраструктуры", paragraph four) names a special KV-cache layout as part of what a
deployment must support. The library's paged layout keeps pages of T tokens x Hkv
heads in a pool and finds logical block j of sequence b through a device block
table. Paging changes only where tokens are stored, so every result here is
checked against the oracle on the logical (unpaged) K/V: cache pages bit for bit
against the oracle's codec, prefill and decode outputs within the parity
tolerances. Page ids are a seeded random permutation of a pool larger than the
sequences need; sequences have different lengths, and a generation loop takes a
new page each time it crosses a block boundary.
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


def paged_cache(T, B, Hkv, D, Tb, max_blocks, spare, seed):
    """A paged cache whose block table maps every logical block to a distinct page of a
    shuffled pool with `spare` unused pages."""
    pages = B * max_blocks + spare
    perm = np.random.RandomState(seed).permutation(pages)[:B * max_blocks].astype(np.int32)
    table = torch.from_numpy(perm.reshape(B, max_blocks)).cuda()
    return T.PagedKVCache(B, Hkv, D, Tb, pages, table), perm.reshape(B, max_blocks)


def check_pages(oracle_mod, cache, table, K, V, S):
    """Every written token's page row against the oracle's codec of the logical row."""
    B, Hkv, _, D = K.shape
    Tb = cache.T
    for X, p in ((K, "k"), (V, "v")):
        c8, s8, c4, s4 = oracle_mod.quantize_rows(X[:, :, :S].contiguous(), D)
        c8 = c8.reshape(B, Hkv, S, D)
        c4p = oracle_mod.pack_int4(c4).reshape(B, Hkv, S, D // 2)
        s8 = s8.reshape(B, Hkv, S)
        s4 = s4.reshape(B, Hkv, S)
        planes = {n: cache.plane(p + n).cpu() for n in ("8", "4", "8_scale", "4_scale")}
        for b in range(B):
            for j in range((S + Tb - 1) // Tb):
                pg = int(table[b, j])
                n = min(Tb, S - j * Tb)
                tok = slice(j * Tb, j * Tb + n)
                assert np.array_equal(planes["8"][pg, :, :n].numpy(), c8[b, :, tok])
                assert np.array_equal(planes["4"][pg, :, :n].numpy(), c4p[b, :, tok])
                assert np.array_equal(planes["8_scale"][pg, :, :n].numpy().view(np.uint32), s8[b, :, tok].view(np.uint32))
                assert np.array_equal(planes["4_scale"][pg, :, :n].numpy().view(np.uint32), s4[b, :, tok].view(np.uint32))


PREFILL = {
    # B, Hq, Hkv, D, T, S, max_blocks, hi, keep
    "D128_T64": (2, 4, 2, 128, 64, 640, 12, [0, 2, 1, 3], [1, 5, 9, 4]),
    "D128_T128": (2, 4, 1, 128, 128, 768, 7, [1, 0, 2, 1], [3, 1, 4, 6]),
    "D64_T64": (1, 2, 1, 64, 64, 512, 9, [1, 2], [3, 5]),
    # head pairs with equal boundaries: the GQA-shared kernel reads the paged cache
    "D128_T64_gqa_pairs": (2, 4, 2, 128, 64, 640, 12, [2, 2, 0, 0], [5, 5, 9, 9]),
    "D128_T128_gqa_pairs": (2, 4, 1, 128, 128, 896, 8, [1, 1, 3, 3], [4, 4, 6, 6]),
    "D64_T128_gqa_pairs": (1, 4, 2, 64, 128, 640, 6, [0, 0, 2, 2], [2, 2, 5, 5]),
}


@pytest.mark.parametrize("name", list(PREFILL))
def test_paged_cache_write_and_prefill(T, oracle_mod, name):
    B, Hq, Hkv, D, Tb, S, mb, hi, keep = PREFILL[name]
    hi, keep = np.array(hi, np.int32), np.array(keep, np.int32)
    Q, K, V = seeded((B, Hq, S, D), 21), seeded((B, Hkv, S, D), 22), seeded((B, Hkv, S, D), 23)
    cache, table = paged_cache(T, B, Hkv, D, Tb, mb, spare=5, seed=24)
    T.tria_quantize_kv(K.cuda(), V.cuda(), cache)
    O, L = T.tria_prefill(Q.cuda(), cache, hi, keep)
    torch.cuda.synchronize()
    assert cache.status() == 0
    check_pages(oracle_mod, cache, table, K, V, S)
    O_ref, L_ref = oracle_mod.prefill_rows(Q, K, V, Tb, hi, keep)
    compare_o(O, O_ref.reshape(B, Hq, S, D), f"paged prefill {name}")
    compare_lse(L, L_ref.reshape(B, Hq, S), f"paged prefill {name}")


def test_paged_decode_ragged_and_generation(T, oracle_mod):
    """Ragged sequences decoded through the block table, then generation steps that
    append one token per sequence and take a fresh page at each block boundary."""
    B, Hq, Hkv, D, Tb, mb = 3, 8, 2, 128, 64, 10
    hi = np.array([1, 0, 2, 3, 1, 4, 0, 2], np.int32)
    keep = np.array([4, 2, 3, 6, 1, 9, 5, 2], np.int32)
    cap = mb * Tb
    K, V = seeded((B, Hkv, cap, D), 31), seeded((B, Hkv, cap, D), 32)
    lens = np.array([Tb * 4 + 7, Tb * 2 - 1, Tb * 6], np.int32)
    rng = np.random.RandomState(33)
    pool = list(rng.permutation(B * mb + 4).astype(np.int32))
    table = np.full((B, mb), -1, np.int32)
    for b in range(B):               # pages for the prompt only; the rest are handed out as the sequence grows
        for j in range((int(lens[b]) + Tb - 1) // Tb):
            table[b, j] = pool.pop()
    bt = torch.from_numpy(table).cuda()
    cache = T.PagedKVCache(B, Hkv, D, Tb, B * mb + 4, bt)
    # the prompts, one sequence at a time through a one-sequence view of the same pool
    for b in range(B):
        one = T.tria_kv_cache.from_buffer_copy(cache.struct)
        one.B = 1
        one.block_table = bt[b:b + 1].data_ptr()
        n = int(lens[b])
        Kb, Vb = K[b:b + 1, :, :n].contiguous().cuda(), V[b:b + 1, :, :n].contiguous().cuda()   # alive until the copy ran
        st = T.lib().tria_quantize_kv(Kb.data_ptr(), Vb.data_ptr(), n, 0, T.ctypes.byref(one), T._stream())
        assert st == 0
        torch.cuda.synchronize()
    torch.cuda.synchronize()
    ws = torch.empty(T.tria_decode_workspace_bytes(B, Hq, Hkv, D, Tb, cap), dtype=torch.uint8, device="cuda")
    Kd, Vd = K.cuda(), V.cuda()
    for step in range(Tb + 3):
        if step > 0:                 # append one token to every sequence
            for b in range(B):
                pos = int(lens[b])
                if table[b, pos // Tb] < 0:
                    table[b, pos // Tb] = pool.pop()
                    bt[b, pos // Tb] = int(table[b, pos // Tb])
            for b in range(B):
                one = T.tria_kv_cache.from_buffer_copy(cache.struct)
                one.B = 1
                one.block_table = bt[b:b + 1].data_ptr()
                pos = int(lens[b])
                Kb, Vb = Kd[b:b + 1, :, pos:pos + 1].contiguous(), Vd[b:b + 1, :, pos:pos + 1].contiguous()
                st = T.lib().tria_quantize_kv(Kb.data_ptr(), Vb.data_ptr(), 1, pos, T.ctypes.byref(one), T._stream())
                assert st == 0
                torch.cuda.synchronize()
            lens += 1
        q = seeded((B, Hq, D), 100 + step)
        Od, Ld = T.tria_decode(q.cuda(), cache, lens, hi, keep, workspace=ws)
        torch.cuda.synchronize()
        assert T.tria_workspace_status(ws) == 0
        Or, Lr = oracle_mod.decode(q, K, V, Tb, lens, hi, keep)
        compare_o(Od, Or, f"paged decode step {step}")
        compare_lse(Ld, Lr, f"paged decode step {step}")
    assert cache.status() == 0


def test_page_id_out_of_range_is_reported(T):
    """A block-table entry outside the pool is caught by the kernels' own check: the
    write is skipped, reads go to page 0, and the cache's status word says so."""
    B, Hq, Hkv, D, Tb, mb = 1, 2, 1, 128, 64, 4
    table = torch.tensor([[2, 0, 1, 3]], dtype=torch.int32, device="cuda")
    cache = T.PagedKVCache(B, Hkv, D, Tb, 4, table)
    K, V = seeded((B, Hkv, 4 * Tb, D), 41).cuda(), seeded((B, Hkv, 4 * Tb, D), 42).cuda()
    T.tria_quantize_kv(K, V, cache)
    assert cache.status() == 0
    table[0, 1] = 4                  # one past the pool
    T.tria_quantize_kv(K[:, :, :Tb + 1].contiguous(), V[:, :, :Tb + 1].contiguous(), cache)
    assert cache.status() == T.TRIA_ERR_BOUNDS
    q = seeded((B, Hq, D), 43).cuda()
    T.tria_decode(q, cache, np.array([4 * Tb], np.int32), [0, 1], [4, 4])
    torch.cuda.synchronize()
    assert cache.status() == T.TRIA_ERR_BOUNDS
    assert cache.status() == 0       # read and cleared
