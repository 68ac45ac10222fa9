"""Pins of the CPU oracle against what the pages and the mathematics fix.

The oracle is the parity reference for the GPU library, so it is first checked
against things other than itself: hand-worked fixtures (tests/golden/), closed
forms for the tile counts, library routines for the special cases that reduce
to textbook attention (torch SDPA in float64), and invariants (rows of P sum to
one, skipped blocks never contribute, decode equals the last prefill row,
log-sum-exp merge of any split equals the unsplit result).

Sources: the rit.work TriAttention page, section "Какие связи можно не считать,
а какие нельзя удалять" (three actions by distance to the diagonal, protected
first key block and diagonal, two boundaries per head) and section "Как
калибровка распределяет вычисления между головами", last paragraph (one
normalised result; the compressed cache read by decode).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from conftest import GOLDEN

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


# ---------------------------------------------------------------- helpers

def bf16(values) -> torch.Tensor:
    t = torch.tensor(values, dtype=torch.float64).to(torch.bfloat16)
    assert torch.equal(t.double(), torch.tensor(values, dtype=torch.float64)), "not bf16-exact"
    return t


def parse_rows(path):
    rows = []
    for line in open(path, encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        rows.append([f.strip() for f in line.split("|")])
    return rows


def token_mask(oracle_mod, S, T, hi, keep):
    """[Hq, S, S] bool: key u takes part in query t's softmax (from the action map)."""
    nb = (S + T - 1) // T
    masks = []
    t_idx = torch.arange(S)
    for h, k in zip(hi, keep):
        amap = torch.from_numpy(oracle_mod.action_map(nb, int(h), int(k)))
        kept_block = (amap == 8) | (amap == 4)
        m = kept_block[t_idx[:, None] // T, t_idx[None, :] // T]
        m &= t_idx[None, :] <= t_idx[:, None]
        masks.append(m)
    return torch.stack(masks)


def sdpa_reference(Q, K, V, mask=None):
    """Library attention in float64 (torch SDPA) with GQA and an optional [Hq,S,S] mask."""
    Qd, Kd, Vd = Q.double(), K.double(), V.double()
    G = Qd.shape[1] // Kd.shape[1]
    Kd = Kd.repeat_interleave(G, dim=1)
    Vd = Vd.repeat_interleave(G, dim=1)
    S, D = Qd.shape[2], Qd.shape[3]
    if mask is None:
        mask = torch.tril(torch.ones(S, S, dtype=torch.bool))[None].expand(Qd.shape[1], S, S)
    O = F.scaled_dot_product_attention(Qd, Kd, Vd, attn_mask=mask[None])
    scores = (Qd @ Kd.transpose(-1, -2)) / math.sqrt(D)
    scores = scores.masked_fill(~mask[None], float("-inf"))
    return O.numpy(), torch.logsumexp(scores, dim=-1).numpy()


def seeded(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


# ---------------------------------------------------------------- codec

def test_codec_golden_rows(oracle_mod):
    for name, xs, a8, c8s, a4, c4s in parse_rows(GOLDEN / "codec_rows.txt"):
        x = bf16([float(v) for v in xs.split()])
        c8, s8, c4, s4 = oracle_mod.quantize_rows(x, x.numel())
        exp_s8 = np.float32(float(a8)) / np.float32(127.0)
        exp_s4 = np.float32(float(a4)) / np.float32(7.0)
        assert s8[0] == exp_s8, name
        assert s4[0] == exp_s4, name
        assert c8[0].tolist() == [int(v) for v in c8s.split()], name
        assert c4[0].tolist() == [int(v) for v in c4s.split()], name


def test_int4_packing_golden(oracle_mod):
    for codes, hexbytes in parse_rows(GOLDEN / "int4_packing.txt"):
        c = np.array([int(v) for v in codes.split()], np.int8)
        assert oracle_mod.pack_int4(c).tolist() == [int(h, 16) for h in hexbytes.split()]


def test_codec_error_bound_and_symmetry(oracle_mod):
    D = 128
    x = seeded((512, D), 7)
    x[3] = 0                               # zero row
    x[5] = x[5] * 1e-30                    # tiny magnitudes (normal bf16 range)
    x[9] = -x[9].abs()                     # all negative
    c8, s8, c4, s4 = oracle_mod.quantize_rows(x, D)
    xd = x.double().numpy()
    for c, s, lim in ((c8, s8, 127), (c4, s4, 7)):
        assert np.abs(c).max() <= lim
        rec = c.astype(np.float64) * s.astype(np.float64)[:, None]
        # round-to-nearest: every value within half a step of its code, plus the
        # rounding of the fp32 quotient x/s (half an ulp of a number below 128)
        assert np.all(np.abs(xd - rec) <= (0.5 + 2.0 ** -17) * s.astype(np.float64)[:, None])
        # the largest magnitude of each non-zero row maps to the end of the range
        nz = s > 0
        assert np.all(np.abs(c[nz]).max(axis=1) == lim)
    assert s8[3] == 0 and s4[3] == 0 and not c8[3].any() and not c4[3].any()
    # odd symmetry: q(-x) = -q(x), same scales
    n8, ns8, n4, ns4 = oracle_mod.quantize_rows(-x, D)
    assert np.array_equal(n8, -c8) and np.array_equal(n4, -c4)
    assert np.array_equal(ns8, s8) and np.array_equal(ns4, s4)
    # power-of-two scaling commutes with IEEE division: same codes, scales x2
    d8, ds8, d4, ds4 = oracle_mod.quantize_rows((x.float() * 2).to(torch.bfloat16), D)
    assert np.array_equal(d8, c8) and np.array_equal(d4, c4)
    assert np.array_equal(ds8, s8 * 2) and np.array_equal(ds4, s4 * 2)


# ---------------------------------------------------------------- policy

def test_action_map_golden(oracle_mod):
    sym = {"8": 8, "4": 4, ".": 0, "-": -1}
    rows = [line.split() for line in open(GOLDEN / "action_map_nb8_hi1_keep3.txt", encoding="utf-8")
            if line.strip() and not line.startswith("#")]
    expected = np.array([[sym[c] for c in r] for r in rows], np.int32)
    assert np.array_equal(oracle_mod.action_map(8, 1, 3), expected)


def closed_form_counts(nb, hi, keep):
    """Tile counts from the band widths (the diagonal is always int8, so hi=0 acts as hi=1)."""
    h = max(min(hi, nb), 1)
    k = max(min(keep, nb), h)
    n8 = sum(nb - d for d in range(h)) + (nb - h)
    n4 = sum(nb - d for d in range(h, k)) - (k - h)
    return n8, n4, nb * (nb + 1) // 2 - n8 - n4


def test_action_counts_closed_form(oracle_mod):
    for nb in range(1, 11):
        for hi in range(0, nb + 2):
            for keep in range(hi, nb + 3):
                assert oracle_mod.action_counts(nb, hi, keep) == closed_form_counts(nb, hi, keep), (nb, hi, keep)
    # the 512-token workload: nb = 8, heads (1,3) and (2,5)
    assert oracle_mod.action_counts(8, 1, 3) == (15, 11, 10)
    assert oracle_mod.action_counts(8, 2, 5) == (21, 12, 3)


def test_protected_blocks(oracle_mod):
    for hi, keep in ((0, 0), (0, 1), (1, 1), (3, 3)):
        amap = oracle_mod.action_map(12, hi, keep)
        assert np.all(amap[:, 0] == 8)                 # sink block
        assert np.all(np.diag(amap) == 8)              # diagonal
        assert np.all(amap[np.triu_indices(12, 1)] == -1)


# ---------------------------------------------------------------- attention special cases

def test_dense_reference_equals_sdpa(oracle_mod):
    B, Hq, Hkv, S, D = 2, 4, 2, 48, 16
    Q, K, V = seeded((B, Hq, S, D), 1), seeded((B, Hkv, S, D), 2), seeded((B, Hkv, S, D), 3)
    O_ref, L_ref = sdpa_reference(Q, K, V)
    O, L = oracle_mod.dense_attention(Q, K, V)
    assert np.abs(O - O_ref).max() < 1e-12 and np.abs(L - L_ref).max() < 1e-12
    # bypassed codec + every causal tile kept (hi = keep = nb) is dense attention
    T = 8
    nb = S // T
    hi = np.full(Hq, nb, np.int32)
    O2, L2 = oracle_mod.prefill_rows(Q, K, V, T, hi, hi, flags=oracle_mod.FLAG_BYPASS_QUANT)
    assert np.abs(O2.reshape(O_ref.shape) - O_ref).max() < 1e-12
    assert np.abs(L2.reshape(L_ref.shape) - L_ref).max() < 1e-12


@pytest.mark.parametrize("S,T,D", [(24, 4, 8), (20, 4, 4), (16, 1, 2), (18, 2, 4)])
def test_sparse_bypass_equals_masked_sdpa_all_policies(oracle_mod, S, T, D):
    nb = (S + T - 1) // T
    Q, K, V = seeded((1, 1, S, D), 11), seeded((1, 1, S, D), 12), seeded((1, 1, S, D), 13)
    for hi in range(0, nb + 2):
        for keep in range(hi, nb + 2):
            h = np.array([hi], np.int32)
            k = np.array([keep], np.int32)
            O, L = oracle_mod.prefill_rows(Q, K, V, T, h, k, flags=oracle_mod.FLAG_BYPASS_QUANT)
            O_ref, L_ref = sdpa_reference(Q, K, V, token_mask(oracle_mod, S, T, h, k))
            assert np.abs(O - O_ref.reshape(O.shape)).max() < 1e-12, (hi, keep)
            assert np.abs(L - L_ref.reshape(L.shape)).max() < 1e-12, (hi, keep)


def test_exactly_representable_inputs_match_masked_sdpa(oracle_mod):
    """Rows made of 0 and +-a dequantise to themselves in both planes (up to the
    fp32 rounding of the scale), so the quantised oracle must equal library
    attention under the policy's mask: pins how codes and scales enter Q.K and P.V."""
    B, Hq, Hkv, S, D, T = 1, 4, 2, 64, 16, 8
    g = torch.Generator().manual_seed(5)

    def rows(shape):
        sign = torch.randint(-1, 2, shape, generator=g).double()
        sign[..., 0] = 1.0                                       # no all-zero row
        mag = 2.0 ** torch.randint(-3, 3, shape[:-1] + (1,), generator=g).double()
        return (sign * mag).to(torch.bfloat16)

    Q, K, V = rows((B, Hq, S, D)), rows((B, Hkv, S, D)), rows((B, Hkv, S, D))
    hi = np.array([1, 2, 0, 3], np.int32)
    keep = np.array([3, 5, 2, 3], np.int32)
    O, L = oracle_mod.prefill_rows(Q, K, V, T, hi, keep)
    O_ref, L_ref = sdpa_reference(Q, K, V, token_mask(oracle_mod, S, T, hi, keep))
    assert np.abs(O - O_ref.reshape(O.shape)).max() < 1e-5
    assert np.abs(L - L_ref.reshape(L.shape)).max() < 1e-5


def test_plane_example_golden(oracle_mod):
    lines = {r[0]: r[1:] for r in parse_rows(GOLDEN / "plane_example.txt")}
    Q, K, V = (bf16([[float(v) for v in r.split()] for r in lines[n]]).reshape(1, 1, 4, 2)
               for n in ("Q", "K", "V"))
    O, L = oracle_mod.prefill_rows(Q, K, V, 1, np.array([1], np.int32), np.array([2], np.int32))
    r2 = 1.0 / math.sqrt(2.0)
    v0, v3 = np.array([1.0, 0.0]), np.array([0.0, -1.0])
    v1_8, v1_4 = np.array([-100.0, 51 * 100 / 127]), np.array([-100.0, 3 * 100 / 7])
    v2_8, v2_4 = np.array([7.0, 36 * 7 / 127]), np.array([7.0, 2.0])

    def row(scores, values):
        w = np.exp(np.array(scores) - max(scores))
        return (w[:, None] * np.array(values)).sum(0) / w.sum(), max(scores) + math.log(w.sum())

    expect = [
        row([2 * r2], [v0]),
        row([2 * r2, 100 * r2], [v0, v1_8]),
        row([0.0, 0.0, (36 * 7 / 127) * r2], [v0, v1_4, v2_8]),
        row([2 * r2, 9 * r2, 1 * r2], [v0, v2_4, v3]),
    ]
    for t, (o, lse) in enumerate(expect):
        assert np.allclose(O[t], o, rtol=1e-6, atol=1e-9), (t, O[t], o)
        assert abs(L[t] - lse) <= 1e-6 * max(1.0, abs(lse)), (t, L[t], lse)


# ---------------------------------------------------------------- invariants

def test_rows_of_p_sum_to_one(oracle_mod):
    B, Hq, Hkv, S, D, T = 1, 2, 1, 40, 8, 4
    Q, K = seeded((B, Hq, S, D), 21), seeded((B, Hkv, S, D), 22)
    V = torch.ones((B, Hkv, S, D), dtype=torch.bfloat16)
    O, _ = oracle_mod.prefill_rows(Q, K, V, T, np.array([1, 0], np.int32), np.array([3, 2], np.int32))
    assert np.abs(O - 1.0).max() < 1e-6


def test_skipped_blocks_do_not_contribute(oracle_mod):
    B, Hq, Hkv, S, D, T = 1, 2, 2, 64, 8, 8
    nb = S // T
    hi = np.array([1, 2], np.int32)
    keep = np.array([2, 4], np.int32)
    Q, K, V = seeded((B, Hq, S, D), 31), seeded((B, Hkv, S, D), 32), seeded((B, Hkv, S, D), 33)
    O, L = oracle_mod.prefill_rows(Q, K, V, T, hi, keep)
    j0 = 3
    K2, V2 = K.clone(), V.clone()
    K2[:, :, j0 * T:(j0 + 1) * T] = seeded((B, Hkv, T, D), 34, 5.0)
    V2[:, :, j0 * T:(j0 + 1) * T] = seeded((B, Hkv, T, D), 35, 5.0)
    O2, L2 = oracle_mod.prefill_rows(Q, K2, V2, T, hi, keep)
    O, O2 = O.reshape(Hq, S, D), O2.reshape(Hq, S, D)
    for h in range(Hq):
        amap = oracle_mod.action_map(nb, int(hi[h]), int(keep[h]))
        for t in range(S):
            a = amap[t // T, j0]
            same = np.array_equal(O[h, t], O2[h, t])
            assert same == (a not in (4, 8)), (h, t, a)


@pytest.mark.parametrize("t", [0, 5, 7, 8, 21, 39])
def test_decode_equals_last_prefill_row(oracle_mod, t):
    B, Hq, Hkv, S, D, T = 2, 4, 2, 40, 8, 4
    Q, K, V = seeded((B, Hq, S, D), 41), seeded((B, Hkv, S, D), 42), seeded((B, Hkv, S, D), 43)
    hi = np.array([1, 0, 2, 3], np.int32)
    keep = np.array([2, 3, 2, 6], np.int32)
    rows = np.array([(b * Hq + h) * S + t for b in range(B) for h in range(Hq)], np.int64)
    O, L = oracle_mod.prefill_rows(Q, K, V, T, hi, keep, rows=rows)
    q = Q[:, :, t].contiguous()
    Od, Ld = oracle_mod.decode(q, K, V, T, np.full(B, t + 1, np.int32), hi, keep)
    assert np.array_equal(Od.reshape(-1, D), O) and np.array_equal(Ld.reshape(-1), L)


def test_lse_merge_of_any_split_equals_unsplit(oracle_mod):
    B, Hq, Hkv, S, D, T = 3, 4, 1, 96, 8, 4
    q = seeded((B, Hq, D), 51)
    K, V = seeded((B, Hkv, S, D), 52), seeded((B, Hkv, S, D), 53)
    kv_len = np.array([96, 61, 5], np.int32)
    hi = np.array([1, 2, 0, 4], np.int32)
    keep = np.array([5, 9, 30, 4], np.int32)
    O0, L0 = oracle_mod.decode(q, K, V, T, kv_len, hi, keep)
    for nsplit in (1, 2, 3, 7, 40):
        O1, L1 = oracle_mod.decode(q, K, V, T, kv_len, hi, keep, nsplit=nsplit)
        assert np.abs(O1 - O0).max() < 1e-12 and np.abs(L1 - L0).max() < 1e-12, nsplit


def test_invalid_dimensions_rejected(oracle_mod):
    Q, K, V = seeded((1, 3, 8, 4), 1), seeded((1, 2, 8, 4), 2), seeded((1, 2, 8, 4), 3)
    with pytest.raises(ValueError):
        oracle_mod.prefill_rows(Q, K, V, 2, np.zeros(3, np.int32), np.zeros(3, np.int32))
    q = seeded((1, 2, 4), 4)
    K2, V2 = seeded((1, 2, 8, 4), 2), seeded((1, 2, 8, 4), 3)
    with pytest.raises(ValueError):
        oracle_mod.decode(q, K2, V2, 2, np.array([9], np.int32), np.zeros(2, np.int32), np.zeros(2, np.int32))
