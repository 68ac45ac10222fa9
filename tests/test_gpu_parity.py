"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Every input is seeded and synthetic (block_sparse_mixed_b200.workloads); the
oracle never sees anything the GPU computed. Codes and scales must match bit
for bit; O and LSE within the tolerances in tests/parity.py.
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


def seeded(shape, seed, device="cpu", scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16).to(device)


# ---------------------------------------------------------------- codec

def test_codec_bit_exact(T, oracle_mod):
    for D in (64, 128):
        x = seeded((4099, D), 100 + D)
        x[0] = 0                                    # zero row
        x[1] = (x[1].float() * 1e-30).to(torch.bfloat16)   # tiny magnitudes
        x[2] = -x[2].abs()
        x[3, :8] = torch.tensor([127, 45.5, -37.5, 0.5, -0.5, 1.5, 2.5, -2.5])   # exact ties (s8 = 1)
        x[3, 8:] = 0
        x[4, :8] = torch.tensor([7, 4.5, 2.5, -0.5, 1.5, -5.5, 6.5, 0.25])       # exact ties (s4 = 1)
        x[4, 8:] = 0
        c8, s8, c4, s4 = T.tria_quantize_rows(x.cuda())
        r8, rs8, r4, rs4 = oracle_mod.quantize_rows(x, D)
        assert np.array_equal(c8.cpu().numpy(), r8)
        assert np.array_equal(s8.cpu().numpy().view(np.uint32), rs8.view(np.uint32))
        assert np.array_equal(s4.cpu().numpy().view(np.uint32), rs4.view(np.uint32))
        assert np.array_equal(c4.cpu().numpy(), oracle_mod.pack_int4(r4))


def test_codec_ties_and_scales_bit_exact(T, oracle_mod):
    """Rows whose 8-bit quotients sit exactly on half-integers at many binary scales
    (amax = 127 * 2^e, so s8 = 2^e and x = (k + 1/2) 2^e), and a million random rows
    spread over 2^-40 .. 2^40 in magnitude: codes and scales bit for bit."""
    D = 64
    ties = []
    for e in range(-30, 31, 3):
        for k0 in range(0, 126, 63):
            row = torch.zeros(D)
            row[0] = 127.0 * 2.0 ** e
            ks = torch.arange(k0, k0 + D - 1) % 127
            row[1:] = (ks.float() + 0.5) * 2.0 ** e * torch.where(ks % 2 == 0, 1.0, -1.0)
            ties.append(row)
    ties32 = torch.stack(ties)
    ties = ties32.to(torch.bfloat16)
    assert torch.equal(ties.float(), ties32)   # bf16 holds every tie exactly
    # Rows around the smallest maximum of the division-free path (2^-100) and far
    # below it, down to bf16 subnormals, where the kernel divides exactly; the first
    # two maxima (0x1.dep-118, 0x1.54p-120) with x = amax / 2 are pairs the
    # division-free step would round wrongly.
    gt = torch.Generator().manual_seed(321)
    tiny = []
    for amax in (2.0 ** -99, 2.0 ** -100, 2.0 ** -101, float.fromhex("0x1.dep-118"), float.fromhex("0x1.54p-120"),
                 2.0 ** -126, 2.0 ** -130, 2.0 ** -133):
        row = (torch.rand(D, generator=gt) * 2 - 1) * amax
        row[0] = amax
        row[1] = amax / 2
        row[2] = -amax / 2
        tiny.append(row)
    ties = torch.cat([ties, torch.stack(tiny).to(torch.bfloat16)])
    g = torch.Generator().manual_seed(123)
    rnd = torch.randn((1 << 20, D), generator=g)
    rnd = rnd * torch.pow(2.0, torch.randint(-40, 41, (1 << 20, 1), generator=g).float())
    x = torch.cat([ties, rnd.to(torch.bfloat16)])
    c8, s8, c4, s4 = T.tria_quantize_rows(x.cuda())
    r8, rs8, r4, rs4 = oracle_mod.quantize_rows(x, D)
    assert np.array_equal(s8.cpu().numpy().view(np.uint32), rs8.view(np.uint32))
    assert np.array_equal(s4.cpu().numpy().view(np.uint32), rs4.view(np.uint32))
    assert np.array_equal(c8.cpu().numpy(), r8)
    assert np.array_equal(c4.cpu().numpy(), oracle_mod.pack_int4(r4))


def test_cache_write_and_append_bit_exact(T, oracle_mod):
    B, Hkv, D, Tb, cap = 2, 3, 128, 64, 320
    cache = T.CompressedKVCache(B, Hkv, D, Tb, cap)
    cache.buffer.fill_(0x5A)
    K, V = seeded((B, Hkv, 200, D), 7), seeded((B, Hkv, 200, D), 8)
    T.tria_quantize_kv(K.cuda(), V.cuda(), cache, start=0)
    k1, v1 = seeded((B, Hkv, 1, D), 9), seeded((B, Hkv, 1, D), 10)
    T.tria_quantize_kv(k1.cuda(), v1.cuda(), cache, start=200)          # one-token append
    torch.cuda.synchronize()
    Kall, Vall = torch.cat([K, k1], 2), torch.cat([V, v1], 2)
    for X, p in ((Kall, "k"), (Vall, "v")):
        r8, rs8, r4, rs4 = oracle_mod.quantize_rows(X, D)
        r8 = r8.reshape(B, Hkv, 201, D)
        r4p = oracle_mod.pack_int4(r4).reshape(B, Hkv, 201, D // 2)
        assert np.array_equal(cache.plane(p + "8")[:, :, :201].cpu().numpy(), r8)
        assert np.array_equal(cache.plane(p + "4")[:, :, :201].cpu().numpy(), r4p)
        assert np.array_equal(cache.plane(p + "8_scale")[:, :, :201].cpu().numpy().reshape(-1).view(np.uint32),
                              rs8.view(np.uint32))
        assert np.array_equal(cache.plane(p + "4_scale")[:, :, :201].cpu().numpy().reshape(-1).view(np.uint32),
                              rs4.view(np.uint32))
        assert (cache.plane(p + "8")[:, :, 201:].cpu().view(torch.uint8) == 0x5A).all()  # untouched


def test_cache_write_more_groups_than_one_launch_bit_exact(T, oracle_mod):
    """A one-token write into B * Hkv = 65,544 (batch, KV head) groups: more than the
    65,535 grid rows of one codec launch, so the write is split over two launches."""
    B, Hkv, D, Tb, cap, start = 8193, 8, 64, 64, 64, 37
    cache = T.CompressedKVCache(B, Hkv, D, Tb, cap)
    cache.buffer.fill_(0x5A)
    K, V = seeded((B, Hkv, 1, D), 11), seeded((B, Hkv, 1, D), 12)
    T.tria_quantize_kv(K.cuda(), V.cuda(), cache, start=start)
    torch.cuda.synchronize()
    for X, p in ((K, "k"), (V, "v")):
        r8, rs8, r4, rs4 = oracle_mod.quantize_rows(X, D)
        got8 = cache.plane(p + "8")[:, :, start].cpu().numpy().reshape(-1, D)
        got4 = cache.plane(p + "4")[:, :, start].cpu().numpy().reshape(-1, D // 2)
        assert np.array_equal(got8, r8)
        assert np.array_equal(got4, oracle_mod.pack_int4(r4))
        assert np.array_equal(cache.plane(p + "8_scale")[:, :, start].cpu().numpy().reshape(-1).view(np.uint32),
                              rs8.view(np.uint32))
        assert np.array_equal(cache.plane(p + "4_scale")[:, :, start].cpu().numpy().reshape(-1).view(np.uint32),
                              rs4.view(np.uint32))
        # the rows next to the written token are untouched, in the first and the last group
        for b in (0, B - 1):
            assert (cache.plane(p + "8")[b, :, start - 1].cpu().view(torch.uint8) == 0x5A).all()
            assert (cache.plane(p + "8")[b, :, start + 1].cpu().view(torch.uint8) == 0x5A).all()
    del cache
    torch.cuda.empty_cache()


# ---------------------------------------------------------------- prefill

def run_prefill(T, Q, K, V, Tb, hi, keep, cap=None):
    B, Hq, S, D = Q.shape
    Hkv = K.shape[1]
    cache = T.CompressedKVCache(B, Hkv, D, Tb, cap or S)
    T.tria_quantize_kv(K.cuda(), V.cuda(), cache)
    ws = torch.empty(T.tria_prefill_workspace_bytes(B, Hq, Hkv, S, D, Tb), dtype=torch.uint8, device="cuda")
    O, L = T.tria_prefill(Q.cuda(), cache, hi, keep, workspace=ws)
    torch.cuda.synchronize()
    assert T.tria_workspace_status(ws) == 0
    return O, L, cache


PREFILL_CASES = {
    # name: (B, Hq, Hkv, S, D, T, policies)
    "tiny_512_d64_t64": (1, 2, 2, 512, 64, 64, [(1, 3), (2, 5)]),
    "gqa_t128_d128": (1, 4, 1, 1280, 128, 128, [(1, 3), (2, 6), (0, 2), (4, 4)]),
    "ragged_tile_t64": (2, 4, 2, 576, 128, 64, [(1, 2), (3, 9), (0, 0), (2, 4)]),
    "d64_t128": (1, 2, 1, 768, 64, 128, [(2, 3), (1, 6)]),
    "protected_only": (1, 2, 2, 640, 128, 64, [(0, 0), (0, 1)]),
    "dense_int8": (1, 2, 1, 512, 128, 128, [(4, 4), (9, 9)]),
    "all_int4_band": (1, 2, 1, 512, 128, 64, [(0, 20), (1, 20)]),
    # head pairs with equal boundaries: the GQA-shared kernel (its staged O stores),
    # with a last tile of one query block at T = 64
    "gqa_shared_ragged_t64": (2, 4, 2, 576, 128, 64, [(1, 2), (1, 2), (3, 9), (3, 9)]),
    "gqa_shared_d64_t64": (1, 4, 1, 704, 64, 64, [(2, 5), (2, 5), (0, 3), (0, 3)]),
    "gqa_shared_d64_t128": (1, 4, 2, 896, 64, 128, [(1, 4), (1, 4), (2, 7), (2, 7)]),
}


@pytest.mark.parametrize("name", list(PREFILL_CASES))
def test_prefill_matches_oracle(T, oracle_mod, name):
    B, Hq, Hkv, S, D, Tb, pol = PREFILL_CASES[name]
    hi = np.array([p[0] for p in pol], np.int32)
    keep = np.array([p[1] for p in pol], np.int32)
    seed = sum(map(ord, name))
    Q, K, V = seeded((B, Hq, S, D), seed), seeded((B, Hkv, S, D), seed + 1), seeded((B, Hkv, S, D), seed + 2)
    O, L, _ = run_prefill(T, Q, K, V, Tb, hi, keep)
    O_ref, L_ref = oracle_mod.prefill_rows(Q, K, V, Tb, hi, keep)
    compare_o(O, O_ref.reshape(B, Hq, S, D), name)
    compare_lse(L, L_ref.reshape(B, Hq, S), name)


def test_prefill_tiny_workload(T, oracle_mod):
    w = W.WORKLOADS["tiny_prefill"]
    Q, K, V = W.prefill_inputs(w)
    hi, keep = W.policy(w)
    O, L, _ = run_prefill(T, Q, K, V, w.T, hi, keep)
    O_ref, L_ref = oracle_mod.prefill_rows(Q, K, V, w.T, hi, keep)
    compare_o(O, O_ref.reshape(O.shape), "tiny")
    compare_lse(L, L_ref.reshape(L.shape), "tiny")


def test_prefill_llama_workload_sampled_rows(T, oracle_mod):
    """Full-size 8192-token GQA workload; the oracle checks sampled rows."""
    w = W.WORKLOADS["llama_prefill"]
    Q, K, V = W.prefill_inputs(w)
    hi, keep = W.policy(w)
    O, L, _ = run_prefill(T, Q, K, V, w.T, hi, keep)
    rng = np.random.RandomState(0)
    picks = [(0, h, t) for h in range(w.Hq) for t in (0, 63, 64, w.S - 1)]
    picks += [(0, int(rng.randint(w.Hq)), int(rng.randint(w.S))) for _ in range(256)]
    rows = rows_of(w.B, w.Hq, w.S, picks)
    O_ref, L_ref = oracle_mod.prefill_rows(Q, K, V, w.T, hi, keep, rows=rows)
    idx = torch.from_numpy(rows)
    compare_o(O.reshape(-1, w.D).cpu()[idx], O_ref, "llama sampled")
    compare_lse(L.reshape(-1).cpu()[idx], L_ref, "llama sampled")


@pytest.mark.parametrize("name", ["llama_prefill", "llama_prefill_gqa", "long_prefill_b1"])
def test_prefill_is_deterministic(T, name):
    """Two calls on the same cache give the same bits. The per-head kernel splits a
    tile's loads between two accumulators by the parity of the CTA's running load
    count, which depends on which tiles the CTA drew from the tile counter; the two
    partial results are merged commutatively, so the bits must not depend on it.
    long_prefill_b1: one sequence of the 32,768-token workload (T = 128, 55 tiles per CTA)."""
    w = W.scaled(W.WORKLOADS["long_prefill"], B=1) if name == "long_prefill_b1" else W.WORKLOADS[name]
    Q, K, V = W.prefill_inputs(w)
    hi, keep = W.policy(w)
    cache = T.CompressedKVCache(w.B, w.Hkv, w.D, w.T, w.S)
    T.tria_quantize_kv(K.cuda(), V.cuda(), cache)
    Qd = Q.cuda()
    outs = []
    for _ in range(3):
        O = torch.full_like(Qd, float("nan"))
        L = torch.full((w.B, w.Hq, w.S), float("nan"), dtype=torch.float32, device="cuda")
        T.tria_prefill(Qd, cache, hi, keep, O=O, LSE=L)
        outs.append((O, L))
    torch.cuda.synchronize()
    for O, L in outs[1:]:
        assert torch.equal(O.view(torch.int16), outs[0][0].view(torch.int16)), name
        assert torch.equal(L.view(torch.int32), outs[0][1].view(torch.int32)), name
    assert not torch.isnan(outs[0][0].float()).any() and not torch.isnan(outs[0][1]).any()


@pytest.mark.parametrize("Tb", [64, 128])
def test_prefill_many_short_tiles_sampled_rows(T, oracle_mod, Tb):
    """Tiles of one to three loads each, about 17 per CTA: each CTA runs through
    its 16-entry tile ring more than once and meets every tile boundary case
    (a tile whose only load belongs to one pair, lone blocks of either plane)."""
    B, Hq, Hkv, S, D = 1, 16, 4, 20480, 128
    pol = [(0, 0), (0, 1), (1, 2), (0, 2)] * 4
    hi = np.array([p[0] for p in pol], np.int32)
    keep = np.array([p[1] for p in pol], np.int32)
    Q, K, V = seeded((B, Hq, S, D), 71), seeded((B, Hkv, S, D), 72), seeded((B, Hkv, S, D), 73)
    O, L, _ = run_prefill(T, Q, K, V, Tb, hi, keep)
    rng = np.random.RandomState(Tb)
    picks = [(0, h, t) for h in range(Hq) for t in (0, Tb - 1, Tb, 2 * Tb + 5, S - 1)]
    picks += [(0, int(rng.randint(Hq)), int(rng.randint(S))) for _ in range(384)]
    rows = rows_of(B, Hq, S, picks)
    O_ref, L_ref = oracle_mod.prefill_rows(Q, K, V, Tb, hi, keep, rows=rows)
    idx = torch.from_numpy(rows)
    compare_o(O.reshape(-1, D).cpu()[idx], O_ref, f"short tiles T{Tb}")
    compare_lse(L.reshape(-1).cpu()[idx], L_ref, f"short tiles T{Tb}")


def test_prefill_skipped_blocks_are_never_read(T, oracle_mod):
    """Overwrite the cache codes of one key block: rows whose tile with it is
    skipped must come out bit-identical; rows that keep it must change."""
    B, Hq, Hkv, S, D, Tb = 1, 2, 1, 1024, 128, 64
    hi = np.array([1, 2], np.int32)
    keep = np.array([3, 5], np.int32)
    Q, K, V = seeded((B, Hq, S, D), 61), seeded((B, Hkv, S, D), 62), seeded((B, Hkv, S, D), 63)
    O1, L1, cache = run_prefill(T, Q, K, V, Tb, hi, keep)
    j0 = 4
    K2, V2 = K.clone(), V.clone()
    K2[:, :, j0 * Tb:(j0 + 1) * Tb] = seeded((B, Hkv, Tb, D), 64, scale=3.0)
    V2[:, :, j0 * Tb:(j0 + 1) * Tb] = seeded((B, Hkv, Tb, D), 65, scale=3.0)
    O2, L2, _ = run_prefill(T, Q, K2, V2, Tb, hi, keep)
    nb = S // Tb
    for h in range(Hq):
        amap = oracle_mod.action_map(nb, int(hi[h]), int(keep[h]))
        for i in range(nb):
            same = torch.equal(O1[0, h, i * Tb:(i + 1) * Tb], O2[0, h, i * Tb:(i + 1) * Tb])
            assert same == (amap[i, j0] not in (4, 8)), (h, i, amap[i, j0])


# ---------------------------------------------------------------- decode

DECODE_CASES = {
    # name: (B, Hq, Hkv, D, T, cap, kv_len, policies per head)
    "t128_ragged": (3, 8, 2, 128, 128, 2048, [2048, 1000, 129],
                    [(4, 9), (1, 3), (0, 0), (2, 16), (6, 6), (1, 2), (3, 7), (0, 5)]),
    "t64_d64": (2, 4, 1, 64, 64, 640, [640, 65], [(1, 3), (2, 9), (0, 1), (3, 4)]),
    "single_block": (2, 2, 2, 128, 128, 256, [1, 128], [(1, 4), (0, 2)]),
    "g16": (1, 16, 1, 128, 64, 1024, [777], [(h % 4, 2 + h) for h in range(16)]),
    "g12_t128": (1, 12, 1, 128, 128, 2048, [1999], [(h % 5, 1 + 2 * h) for h in range(12)]),
    "t128_d64_g8": (2, 16, 2, 64, 128, 1536, [1536, 700], [((3 * h) % 4, 2 + (h % 7)) for h in range(16)]),
    # one long sequence and one KV group: about 65 kept blocks, one work item each, so
    # the group has more than 256 partials and the merge splits its columns over CTAs
    "long_one_group_t128": (1, 4, 1, 128, 128, 8192, [8192], [(2, 60), (5, 64), (0, 40), (9, 63)]),
    "long_one_group_d64": (1, 2, 1, 64, 64, 4096, [4000], [(1, 62), (3, 50)]),
}


def test_decode_large_values(T, oracle_mod):
    """V of magnitude ~500: 4-bit V scales near 200 force the running maximum to
    move more often so that P * s_v stays finite in fp16."""
    B, Hq, Hkv, D, Tb, cap = 2, 8, 2, 128, 128, 4096
    hi = np.array([1, 2, 0, 3, 1, 4, 2, 0], np.int32)
    keep = np.array([6, 9, 3, 32, 2, 12, 20, 5], np.int32)
    q, K = seeded((B, Hq, D), 71), seeded((B, Hkv, cap, D), 72)
    V = (seeded((B, Hkv, cap, D), 73).float() * 128.0).to(torch.bfloat16)
    kv = np.array([4096, 3001], np.int32)
    O, L = run_decode(T, q, K, V, Tb, kv, hi, keep)
    O_ref, L_ref = oracle_mod.decode(q, K, V, Tb, kv, hi, keep)
    # outputs scale with V: the bound is relative to the V magnitude (bf16 rounding of O included)
    ref = torch.from_numpy(O_ref).double()
    err = (O.double().cpu() - ref).abs()
    assert float(err.max()) <= 128.0 * 1e-2 + 2.0 ** -8 * float(ref.abs().max()), float(err.max())
    compare_lse(L, L_ref, "large_values")


def run_decode(T, q, K, V, Tb, kv_len, hi, keep):
    B, Hkv, cap, D = K.shape
    cache = T.CompressedKVCache(B, Hkv, D, Tb, cap)
    T.tria_quantize_kv(K.cuda(), V.cuda(), cache)
    qd = q.cuda()
    ws = torch.empty(T.tria_decode_workspace_bytes(B, q.shape[1], Hkv, D, Tb, cap), dtype=torch.uint8, device="cuda")
    for _ in range(2):   # a second call on the same workspace must work as well
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        O, L = T.tria_decode(qd, cache, kv_len, hi, keep, workspace=ws)
        t1.record()
        torch.cuda.synchronize()
        assert T.tria_workspace_status(ws) == 0
        # a pipeline wait that ran out would take seconds even if it left no error
        assert t0.elapsed_time(t1) < 500.0, t0.elapsed_time(t1)
    return O, L


@pytest.mark.parametrize("name", list(DECODE_CASES))
def test_decode_matches_oracle(T, oracle_mod, name):
    B, Hq, Hkv, D, Tb, cap, kv_len, pol = DECODE_CASES[name]
    hi = np.array([p[0] for p in pol], np.int32)
    keep = np.array([p[1] for p in pol], np.int32)
    seed = sum(map(ord, name))
    q, K, V = seeded((B, Hq, D), seed), seeded((B, Hkv, cap, D), seed + 1), seeded((B, Hkv, cap, D), seed + 2)
    kv = np.array(kv_len, np.int32)
    O, L = run_decode(T, q, K, V, Tb, kv, hi, keep)
    O_ref, L_ref = oracle_mod.decode(q, K, V, Tb, kv, hi, keep)
    compare_o(O, O_ref, name)
    compare_lse(L, L_ref, name)


def test_decode_workload_four_sequences(T, oracle_mod):
    """The 32768-token decode workload's shapes and policy, 4 of its 64 sequences."""
    w = W.scaled(W.WORKLOADS["decode"], B=4)
    q, K, V, kv = W.decode_inputs(w)
    hi, keep = W.policy(w)
    O, L = run_decode(T, q, K, V, w.T, kv, hi, keep)
    O_ref, L_ref = oracle_mod.decode(q, K, V, w.T, kv, hi, keep)
    compare_o(O, O_ref, "decode workload")
    compare_lse(L, L_ref, "decode workload")


def test_decode_is_deterministic(T):
    """Two decode calls on the same cache give the same bits, whichever CTA draws which
    work item: every (item, warp) partial has its own slot and the merge adds them in
    slot order."""
    w = W.scaled(W.WORKLOADS["decode"], B=16)
    q, K, V, kv = W.decode_inputs(w)
    hi, keep = W.policy(w)
    cache = T.CompressedKVCache(w.B, w.Hkv, w.D, w.T, K.shape[2])
    T.tria_quantize_kv(K.cuda(), V.cuda(), cache)
    qd = q.cuda()
    outs = [T.tria_decode(qd, cache, kv, hi, keep) for _ in range(3)]
    torch.cuda.synchronize()
    for O, L in outs[1:]:
        assert torch.equal(O.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(L.view(torch.int32), outs[0][1].view(torch.int32))


def test_decode_equals_last_prefill_row(T):
    """Same cache, same policy: decode of token S-1 reproduces prefill row S-1."""
    B, Hq, Hkv, S, D, Tb = 2, 4, 1, 1024, 128, 128
    hi = np.array([1, 2, 0, 3], np.int32)
    keep = np.array([3, 4, 5, 3], np.int32)
    Q, K, V = seeded((B, Hq, S, D), 71), seeded((B, Hkv, S, D), 72), seeded((B, Hkv, S, D), 73)
    O, L, cache = run_prefill(T, Q, K, V, Tb, hi, keep)
    Od, Ld = T.tria_decode(Q[:, :, S - 1].contiguous().cuda(), cache, np.full(B, S, np.int32), hi, keep)
    torch.cuda.synchronize()
    assert (Od.float() - O[:, :, S - 1].float()).abs().max().item() <= 1e-2
    assert (Ld - L[:, :, S - 1]).abs().max().item() <= 1e-3


def test_prepare_then_attend_equals_prefill(T):
    """tria_prefill_prepare + tria_prefill_attend on one stream give tria_prefill's bits."""
    B, Hq, Hkv, S, D, Tb = 1, 4, 2, 1024, 128, 128
    hi = np.array([1, 2, 0, 3], np.int32)
    keep = np.array([3, 5, 2, 4], np.int32)
    Q, K, V = seeded((B, Hq, S, D), 81, "cuda"), seeded((B, Hkv, S, D), 82, "cuda"), seeded((B, Hkv, S, D), 83, "cuda")
    cache = T.CompressedKVCache(B, Hkv, D, Tb, S)
    T.tria_quantize_kv(K, V, cache)
    ws = torch.empty(T.tria_prefill_workspace_bytes(B, Hq, Hkv, S, D, Tb), dtype=torch.uint8, device="cuda")
    O1, L1 = T.tria_prefill(Q, cache, hi, keep, workspace=ws)
    O2, L2 = torch.empty_like(O1), torch.empty_like(L1)
    T.tria_prefill_prepare(Q, cache, ws)
    T.tria_prefill_attend(cache, hi, keep, ws, O2, L2)
    torch.cuda.synchronize()
    assert T.tria_workspace_status(ws) == 0
    assert torch.equal(O1, O2) and torch.equal(L1, L2)
