"""The fused prefill's load plan, checked on the host against the oracle's tile
policy (rit.work TriAttention page, section on which links may be skipped and
which must be kept: block 0 and the diagonal at 8 bits, d < hi at 8 bits,
d < keep at 4 bits, the rest skipped).

The plan decides which (key block, plane) tiles the kernel computes at all, so a
dropped or doubled entry would be a wrong result even where the arithmetic is
right. Every query tile must load each tile its rows need exactly once, at the
needed plane, with no load left half empty beyond one lone block per plane.
"""
import numpy as np
import pytest

from block_sparse_mixed_b200 import tria


def needed(amap, i0, nq):
    """{(j, plane)} that some query block of the tile [i0, i0 + nq) needs."""
    out = set()
    for i in range(i0, i0 + nq):
        for j in range(i + 1):
            a = int(amap[i, j])
            if a in (4, 8):
                out.add((j, a))
    return out


def check_plan(oracle_mod, nb, T, hi, keep):
    plan = tria.tria_prefill_load_plan(nb, T, hi, keep)
    amap = oracle_mod.action_map(nb, hi, keep)
    nq = 128 // T
    tiles = {}
    for i0, j0, j1, plane in plan.tolist():
        tiles.setdefault(i0, []).append((j0, j1, plane))
    assert sorted(tiles) == list(range(0, nb, nq))
    assert list(plan[:, 0]) == sorted(plan[:, 0])          # tiles in ascending order
    for i0, loads in tiles.items():
        q = min(nq, nb - i0)
        got = []
        for j0, j1, plane in loads:
            assert plane in (4, 8)
            if T == 128:
                assert j1 == j0
                got.append((j0, plane))
            else:
                assert j1 != j0
                got.append((j0, plane))
                if j1 >= 0:
                    got.append((j1, plane))
        need = needed(amap, i0, q)
        assert len(got) == len(set(got)), (i0, loads)       # nothing loaded twice
        assert set(got) == need, (i0, loads, need)          # nothing missing, nothing extra
        planes = [p for _, _, p in loads]
        assert planes == sorted(planes, reverse=True)       # all 8-bit loads before the 4-bit ones
        for p in (8, 4):
            n = sum(1 for (_, pl) in need if pl == p)
            lone = sum(1 for j0, j1, pl in loads if pl == p and j1 < 0)
            if T == 64:
                assert lone == n % 2, (i0, p, loads)        # at most one lone block per plane
                assert sum(1 for _, _, pl in loads if pl == p) == (n + 1) // 2
            else:
                assert sum(1 for _, _, pl in loads if pl == p) == n
    return plan


@pytest.mark.parametrize("T", [64, 128])
@pytest.mark.parametrize("nb,hi,keep", [
    (0, 0, 0), (1, 0, 0), (1, 3, 5), (2, 0, 1), (7, 0, 0), (9, 1, 1),
    (13, 2, 5), (16, 4, 4), (17, 1, 64), (33, 5, 11), (40, 16, 40),
])
def test_load_plan_edge_cases(oracle_mod, nb, T, hi, keep):
    check_plan(oracle_mod, nb, T, hi, keep)


def test_load_plan_random_policies(oracle_mod):
    rng = np.random.RandomState(7)
    for _ in range(150):
        T = int(rng.choice([64, 128]))
        nb = int(rng.randint(1, 48))
        hi = int(rng.randint(0, 12))
        keep = hi + int(rng.randint(0, 40))
        check_plan(oracle_mod, nb, T, hi, keep)


def test_load_plan_counts_match_tile_counts(oracle_mod):
    # at T = 128 every load is one kept tile, so the plan has exactly as many
    # loads as the policy keeps tiles
    for nb, hi, keep in [(64, 16, 64), (256, 17, 35), (100, 3, 100)]:
        n8, n4, _ = oracle_mod.action_counts(nb, hi, keep)
        assert len(tria.tria_prefill_load_plan(nb, 128, hi, keep)) == n8 + n4


def test_load_plan_rejects_bad_arguments():
    for args in [(-1, 64, 0, 0), (8, 96, 0, 0), (8, 64, -1, 0), (8, 64, 3, 2)]:
        with pytest.raises(RuntimeError):
            tria.tria_prefill_load_plan(*args)
