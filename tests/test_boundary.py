"""C-ABI boundary checks that need no GPU: the library loads, exports every
function include/tria.h declares, and its host-side logic (sizes, cache
carving, tile counting, argument validation) behaves as documented."""
import ctypes

import numpy as np
import pytest

from block_sparse_mixed_b200 import tria
from block_sparse_mixed_b200.build import build


@pytest.fixture(scope="module")
def L():
    build()
    return tria.lib()


EXPECTED = {
    "tria_status_string", "tria_cache_bytes", "tria_cache_init", "tria_quantize_rows", "tria_quantize_kv",
    "tria_count_tiles", "tria_prefill_load_plan", "tria_decode_plan", "tria_prefill_workspace_bytes", "tria_prefill",
    "tria_prefill_prepare", "tria_prefill_attend", "tria_decode_workspace_bytes", "tria_decode",
    "tria_decode_static", "tria_decode_static_status", "tria_workspace_status",
    "tria_paged_cache_bytes", "tria_paged_cache_init", "tria_cache_status",
    "tria_calibration_costs", "tria_calibrate_workspace_bytes", "tria_calibrate", "tria_allocate",
    "tria_prefill_gqa", "tria_prefill_host_staging_bytes", "tria_prefill_host_workspace_bytes", "tria_prefill_host",
}


def test_every_declared_symbol_is_exported(L):
    names = tria.declared_functions()
    assert set(names) == EXPECTED, sorted(set(names) ^ EXPECTED)
    for n in names:
        assert hasattr(L, n), f"{n} declared in tria.h but not exported"


def test_status_strings(L):
    for s in range(7):
        assert tria.tria_status_string(s)
    assert tria.tria_status_string(0) == "ok"


def test_cache_sizes_and_carving(L):
    B, Hkv, D, T, cap = 2, 3, 128, 64, 256
    n = L.tria_cache_bytes(B, Hkv, D, T, cap)
    rows = B * Hkv * cap
    assert n >= 2 * (rows * D + rows * D // 2 + 2 * rows * 4)
    assert L.tria_cache_bytes(B, Hkv, 96, T, cap) == 0          # unsupported D
    assert L.tria_cache_bytes(B, Hkv, D, T, cap + 1) == 0       # capacity not a multiple of T
    c = tria.tria_kv_cache()
    base = 1 << 40                                             # never dereferenced
    assert L.tria_cache_init(ctypes.byref(c), ctypes.c_void_p(base), n, B, Hkv, D, T, cap) == 0
    ptrs = [c.k8, c.k4, c.k8_scale, c.k4_scale, c.v8, c.v4, c.v8_scale, c.v4_scale]
    assert c.status == base and ptrs[0] >= base + 4 and all(p % 256 == 0 for p in ptrs)
    assert c.block_table is None and c.capacity == cap
    sizes = [rows * D, rows * D // 2, rows * 4, rows * 4] * 2
    for p, q, s in zip(ptrs, ptrs[1:], sizes):
        assert q - p >= s                                      # planes do not overlap
    assert ptrs[-1] + rows * 4 <= base + n
    assert L.tria_cache_init(ctypes.byref(c), ctypes.c_void_p(base + 16), n, B, Hkv, D, T, cap) == 1
    assert L.tria_cache_init(ctypes.byref(c), ctypes.c_void_p(base), n - 1, B, Hkv, D, T, cap) == 1


def test_paged_cache_sizes_and_carving(L):
    pages, Hkv, D, T, B, mb = 37, 2, 64, 128, 3, 5
    n = L.tria_paged_cache_bytes(pages, Hkv, D, T)
    rows = pages * Hkv * T
    assert n >= 4 + 2 * (rows * D + rows * D // 2 + 2 * rows * 4)
    assert L.tria_paged_cache_bytes(0, Hkv, D, T) == 0
    assert L.tria_paged_cache_bytes(pages, Hkv, D, 96) == 0
    c = tria.tria_kv_cache()
    base, table = 1 << 40, 1 << 41                             # never dereferenced
    assert L.tria_paged_cache_init(ctypes.byref(c), ctypes.c_void_p(base), n, B, Hkv, D, T, pages,
                                   ctypes.c_void_p(table), mb) == 0
    assert c.block_table == table and c.max_blocks == mb and c.num_pages == pages and c.capacity == mb * T
    ptrs = [c.k8, c.k4, c.k8_scale, c.k4_scale, c.v8, c.v4, c.v8_scale, c.v4_scale]
    sizes = [rows * D, rows * D // 2, rows * 4, rows * 4] * 2
    for p, q, sz in zip(ptrs, ptrs[1:], sizes):
        assert q - p >= sz
    assert ptrs[-1] + rows * 4 <= base + n
    # no table, a short buffer, a misaligned base
    assert L.tria_paged_cache_init(ctypes.byref(c), ctypes.c_void_p(base), n, B, Hkv, D, T, pages, None, mb) == 1
    assert L.tria_paged_cache_init(ctypes.byref(c), ctypes.c_void_p(base), n - 1, B, Hkv, D, T, pages,
                                   ctypes.c_void_p(table), mb) == 1
    assert L.tria_paged_cache_init(ctypes.byref(c), ctypes.c_void_p(base + 16), n, B, Hkv, D, T, pages,
                                   ctypes.c_void_p(table), mb) == 1


def test_tile_counts_match_oracle(L, oracle_mod):
    for nb in (1, 2, 7, 16, 33):
        for hi in range(0, 6):
            for keep in range(hi, hi + 8):
                assert tria.tria_count_tiles(nb, hi, keep) == oracle_mod.action_counts(nb, hi, keep)
    with pytest.raises(tria.TriaError):
        tria.tria_count_tiles(8, 3, 2)


def test_workspace_sizes(L):
    assert tria.tria_prefill_workspace_bytes(1, 32, 8, 8192, 128, 64) > 0
    assert tria.tria_prefill_workspace_bytes(1, 32, 8, 8192 + 1, 128, 64) == 0   # S % T
    assert tria.tria_prefill_workspace_bytes(1, 30, 8, 8192, 128, 64) == 0       # Hq % Hkv
    assert tria.tria_prefill_workspace_bytes(1, 32, 8, 8192, 80, 64) == 0        # D
    assert tria.tria_decode_workspace_bytes(64, 32, 8, 128, 128, 32768) > 0
    assert tria.tria_decode_workspace_bytes(64, 64, 2, 128, 128, 32768) == 0     # 32 heads per group


def _fake_cache(B=1, Hkv=2, D=128, T=64, cap=512):
    c = tria.tria_kv_cache()
    n = tria.lib().tria_cache_bytes(B, Hkv, D, T, cap)
    assert tria.lib().tria_cache_init(ctypes.byref(c), ctypes.c_void_p(1 << 40), n, B, Hkv, D, T, cap) == 0
    return c


def test_host_validation_rejects_bad_arguments(L):
    fake = ctypes.c_void_p(1 << 41)
    c = _fake_cache()
    i32 = lambda v: np.ascontiguousarray(v, np.int32)
    hi, keep = i32([1, 2, 1, 2]), i32([3, 5, 3, 5])
    P = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    ws = ctypes.c_void_p(1 << 42)
    # quantize_kv: start + S beyond capacity, null pointers
    assert L.tria_quantize_kv(fake, fake, 600, 0, ctypes.byref(c), None) == tria.TRIA_ERR_INVALID_ARG
    assert L.tria_quantize_kv(None, fake, 10, 0, ctypes.byref(c), None) == tria.TRIA_ERR_INVALID_ARG
    assert L.tria_quantize_kv(fake, fake, 10, -1, ctypes.byref(c), None) == tria.TRIA_ERR_INVALID_ARG
    # prefill: S % T, keep < hi, negative hi, unsupported D, workspace too small
    d = tria.tria_dims(1, 4, 2, 500, 128, 64)
    assert L.tria_prefill(fake, ctypes.byref(c), ctypes.byref(d), P(hi), P(keep), fake, fake, ws, 1 << 40,
                          None) == tria.TRIA_ERR_INVALID_ARG
    d = tria.tria_dims(1, 4, 2, 512, 128, 64)
    assert L.tria_prefill(fake, ctypes.byref(c), ctypes.byref(d), P(i32([2, 2, 2, 2])), P(i32([1, 5, 5, 5])),
                          fake, fake, ws, 1 << 40, None) == tria.TRIA_ERR_INVALID_ARG
    assert L.tria_prefill(fake, ctypes.byref(c), ctypes.byref(d), P(i32([-1, 2, 2, 2])), P(keep),
                          fake, fake, ws, 1 << 40, None) == tria.TRIA_ERR_INVALID_ARG
    assert L.tria_prefill(fake, ctypes.byref(c), ctypes.byref(d), P(hi), P(keep), fake, fake, ws, 16,
                          None) == tria.TRIA_ERR_WORKSPACE
    d96 = tria.tria_dims(1, 4, 2, 512, 96, 64)
    assert L.tria_prefill(fake, ctypes.byref(c), ctypes.byref(d96), P(hi), P(keep), fake, fake, ws, 1 << 40,
                          None) == tria.TRIA_ERR_UNSUPPORTED
    big = tria.tria_dims(1, 4, 2, 1024, 128, 64)          # S beyond the cache capacity
    assert L.tria_prefill(fake, ctypes.byref(c), ctypes.byref(big), P(hi), P(keep), fake, fake, ws, 1 << 40,
                          None) == tria.TRIA_ERR_INVALID_ARG
    # decode: kv_len out of range, head ratio
    assert L.tria_decode(fake, ctypes.byref(c), P(i32([513])), 4, P(hi), P(keep), fake, fake, ws, 1 << 40,
                         None) == tria.TRIA_ERR_INVALID_ARG
    assert L.tria_decode(fake, ctypes.byref(c), P(i32([0])), 4, P(hi), P(keep), fake, fake, ws, 1 << 40,
                         None) == tria.TRIA_ERR_INVALID_ARG
    assert L.tria_decode(fake, ctypes.byref(c), P(i32([10])), 3, P(hi), P(keep), fake, fake, ws, 1 << 40,
                         None) == tria.TRIA_ERR_INVALID_ARG
    # codec: unsupported width, unaligned pointer
    assert L.tria_quantize_rows(fake, 4, 96, fake, fake, fake, fake, None) == tria.TRIA_ERR_UNSUPPORTED
    assert L.tria_quantize_rows(ctypes.c_void_p((1 << 41) + 2), 4, 128, fake, fake, fake, fake,
                                None) == tria.TRIA_ERR_INVALID_ARG


def test_host_prefill_validation_before_any_cuda_call(L):
    """tria_prefill_host checks every argument on the host before it creates an event
    or queues a copy, so these calls return at once, here without a GPU."""
    P = ctypes.c_void_p
    f = L.tria_prefill_host
    f.argtypes = [P, P, P, ctypes.POINTER(tria.tria_kv_cache), ctypes.POINTER(tria.tria_dims), P, P, P, P,
                  P, ctypes.c_size_t, P, ctypes.c_size_t, P, P, P]
    f.restype = ctypes.c_int
    for fn in ("tria_prefill_host_staging_bytes", "tria_prefill_host_workspace_bytes"):
        getattr(L, fn).argtypes = [ctypes.POINTER(tria.tria_dims)]
        getattr(L, fn).restype = ctypes.c_size_t
    c = _fake_cache(B=1, Hkv=2, D=128, T=64, cap=512)
    d = tria.tria_dims(1, 4, 2, 512, 128, 64)
    i32 = lambda v: np.ascontiguousarray(v, np.int32)
    hi, keep = i32([1, 2, 1, 2]), i32([3, 5, 3, 5])
    host = P(1 << 30)
    staging, ws = P(1 << 41), P(1 << 42)
    sbytes = L.tria_prefill_host_staging_bytes(ctypes.byref(d))
    wbytes = L.tria_prefill_host_workspace_bytes(ctypes.byref(d))
    # two slots of (Q of 2 heads, K, V, O of 2 heads, LSE of 2 heads) at S = 512, D = 128
    assert sbytes == 2 * (2 * 262144 + 2 * 131072 + 4096)
    assert wbytes == tria.tria_prefill_workspace_bytes(1, 2, 1, 512, 128, 64) > 0
    s1, s2, s3 = P(1), P(2), P(3)

    def call(hQ=host, cache=c, dims=d, st=staging, sb=sbytes, wb=wbytes, streams=(s1, s2, s3)):
        return f(hQ, host, host, ctypes.byref(cache), ctypes.byref(dims), hi.ctypes.data_as(P),
                 keep.ctypes.data_as(P), host, host, st, sb, ws, wb, *streams)

    assert call(hQ=None) == tria.TRIA_ERR_INVALID_ARG
    assert call(streams=(s1, s2, s2)) == tria.TRIA_ERR_INVALID_ARG          # one stream for both copies
    assert call(streams=(s1, s1, s3)) == tria.TRIA_ERR_INVALID_ARG          # copies on the compute stream
    assert call(st=P((1 << 41) + 16)) == tria.TRIA_ERR_INVALID_ARG          # staging not 256-byte aligned
    assert call(sb=sbytes - 1) == tria.TRIA_ERR_INVALID_ARG
    assert call(wb=wbytes - 1) == tria.TRIA_ERR_INVALID_ARG
    assert call(dims=tria.tria_dims(1, 4, 2, 1024, 128, 64)) == tria.TRIA_ERR_INVALID_ARG   # S > capacity
    assert call(dims=tria.tria_dims(1, 4, 1, 512, 128, 64)) == tria.TRIA_ERR_INVALID_ARG    # Hkv differs
    paged = tria.tria_kv_cache()
    ctypes.memmove(ctypes.byref(paged), ctypes.byref(c), ctypes.sizeof(c))
    paged.block_table = P(1 << 43)
    assert call(cache=paged) == tria.TRIA_ERR_UNSUPPORTED


def test_calibration_costs_match_oracle(L):
    from oracle import calibration as cal
    for nb, T, D in ((8, 64, 128), (37, 128, 64), (1, 64, 64)):
        hi = [0, 1, 2, 5, nb, 3]
        keep = [0, 3, 2, 9, nb, 40]
        assert tria.tria_calibration_costs(nb, T, D, hi, keep).tolist() == \
            cal.candidate_costs(nb, T, D, hi, keep).tolist()
    with pytest.raises(tria.TriaError):
        tria.tria_calibration_costs(8, 64, 128, [3], [2])


def test_allocator_matches_oracle(L):
    """The library's greedy allocator takes the same decisions as the oracle's on the same
    (error, cost) tables: the hand-worked example and random tables with ties."""
    from oracle import calibration as cal
    err = np.array([[9.0, 4.0, 6.0], [3.0, 3.0, 5.0], [1.0, 0.0, 0.5]])
    cost = np.array([[10, 10, 10], [20, 20, 20], [40, 40, 40]], np.int64)
    for budget in (30, 45, 80, 1000):
        assert tria.tria_allocate(err, cost, budget).tolist() == cal.allocate(err, cost, budget)
    rng = np.random.RandomState(7)
    for _ in range(300):
        C, H = rng.randint(1, 7), rng.randint(1, 9)
        cost = rng.randint(1, 12, (C, H)).astype(np.int64)          # small ranges: many ties
        err = rng.randint(0, 6, (C, H)).astype(np.float64) / 4.0
        budget = int(rng.randint(0, 80))
        assert tria.tria_allocate(err, cost, budget).tolist() == cal.allocate(err, cost, budget)
