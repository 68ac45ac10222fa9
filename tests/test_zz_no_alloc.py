"""The allocation-free decode entry point (tria_decode_static).

Some callers cannot allocate device memory (a plugin whose host application
has budgeted all device memory in advance, a latency-critical loop that must
not call cudaMalloc). For them the library offers tria_decode_static, which
uses a fixed scratch array compiled into the library instead of a caller
workspace. This test calls it through the C ABI (ctypes on the raw symbol)
twice in a row, on two different problems, and checks each result against the
workspace-taking tria_decode within the parity tolerances; it also checks that
a problem needing more scratch than the fixed array holds is rejected. The
file is named to be collected last, and it runs the same alone or after the
other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity import compare_lse, compare_o

pytestmark = pytest.mark.gpu


def _seeded(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def test_static_scratch_decode_matches_workspace_decode():
    from block_sparse_mixed_b200.build import build
    build()
    from block_sparse_mixed_b200 import tria
    assert torch.cuda.is_available(), "GPU test"
    L = tria.lib()
    P = ctypes.c_void_p
    L.tria_decode_static.argtypes = [P, ctypes.POINTER(tria.tria_kv_cache), P, ctypes.c_int, P, P, P, P, P]
    L.tria_decode_static.restype = ctypes.c_int
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    host = lambda a: np.ascontiguousarray(a, np.int32)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    cases = [  # (B, Hq, Hkv, D, T, cap, kv_len, hi, keep, seed): two different problems, back to back
        (3, 8, 2, 128, 128, 2048, [2048, 1000, 129], [4, 1, 0, 2, 6, 1, 3, 0], [9, 3, 0, 16, 6, 2, 7, 5], 11),
        (2, 4, 1, 128, 64, 1024, [1024, 65], [1, 2, 0, 3], [3, 9, 1, 4], 12),
    ]
    for B, Hq, Hkv, D, T, cap, kv_len, hi, keep, seed in cases:
        q = _seeded((B, Hq, D), seed).cuda()
        K, V = _seeded((B, Hkv, cap, D), seed + 1).cuda(), _seeded((B, Hkv, cap, D), seed + 2).cuda()
        cache = tria.CompressedKVCache(B, Hkv, D, T, cap)
        tria.tria_quantize_kv(K, V, cache)
        kv, h, k = host(kv_len), host(hi), host(keep)
        O_ref, L_ref = tria.tria_decode(q, cache, kv, h, k)
        O = torch.full_like(q, float("nan"))
        LSE = torch.full((B, Hq), float("nan"), device="cuda")
        st = L.tria_decode_static(ptr(q), ctypes.byref(cache.struct), kv.ctypes.data_as(P), Hq,
                                  h.ctypes.data_as(P), k.ctypes.data_as(P), ptr(O), ptr(LSE), stream)
        assert st == tria.TRIA_OK, tria.tria_status_string(st)
        torch.cuda.synchronize()
        compare_o(O, O_ref.double().cpu().numpy(), "static scratch decode")
        compare_lse(LSE, L_ref.double().cpu().numpy(), "static scratch decode")

        # the fixed array's error word: clear after a call that completed normally
        L.tria_decode_static_status.argtypes = [P]
        L.tria_decode_static_status.restype = ctypes.c_int
        assert L.tria_decode_static_status(stream) == tria.TRIA_OK

    # A problem whose decode scratch exceeds the fixed array is refused before any
    # work. Its buffers are real allocations of the right sizes, so that a
    # regression in the size check would give a wrong status, never a launch on
    # made-up addresses.
    Bb, Hqb, Hkvb, Db, Tb, capb = 1024, 32, 2, 128, 128, 128
    assert tria.tria_decode_workspace_bytes(Bb, Hqb, Hkvb, Db, Tb, capb) > (40 << 20)
    big = tria.CompressedKVCache(Bb, Hkvb, Db, Tb, capb)
    qb = torch.zeros((Bb, Hqb, Db), dtype=torch.bfloat16, device="cuda")
    Ob = torch.zeros_like(qb)
    Lb = torch.zeros((Bb, Hqb), dtype=torch.float32, device="cuda")
    kv = host([capb] * Bb)
    h = host([1] * Hqb)
    st = L.tria_decode_static(ptr(qb), ctypes.byref(big.struct), kv.ctypes.data_as(P), Hqb, h.ctypes.data_as(P),
                              h.ctypes.data_as(P), ptr(Ob), ptr(Lb), stream)
    assert st == tria.TRIA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert int(Ob.view(torch.int16).abs().sum()) == 0 and float(Lb.abs().sum()) == 0.0   # nothing written
