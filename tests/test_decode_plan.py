"""The decode's work plan (tria_decode_plan, the host side of tria_decode), on the CPU.

Checked against definitions written here from the tile action of the rit.work
TriAttention page (section on which links may be skipped and which must be kept):
a group's kept blocks at its query position are every block that at least one of its
query heads keeps; the plan must split exactly those, within the workspace's partial
slots, and hand the groups' first splits out in non-increasing cost. The device side
of the mapping (which work item takes which blocks) is restated from its description
in the header, and every kept block of every group must be taken exactly once.
"""
import numpy as np
import pytest

from block_sparse_mixed_b200 import tria
from block_sparse_mixed_b200 import workloads as W


def kept_union(ib, hi, keep):
    """Blocks j <= ib that some head (hi_h, keep_h) keeps at query block ib."""
    out = []
    for j in range(ib + 1):
        d = ib - j
        if j == 0 or d == 0 or any(d < k for k in keep) or any(d < max(h, 1) for h in hi):
            out.append(j)
    return out


def check_plan(B, Hq, Hkv, T, cap, kv_len, hi, keep, sms):
    G = Hq // Hkv
    plan = tria.tria_decode_plan(B, Hq, Hkv, T, cap, kv_len, hi, keep, sms)
    groups = B * Hkv
    nk, ss, fo = plan["nkept"], plan["split_start"], plan["first_order"]
    bps, n_items = plan["blocks_per_split"], plan["n_items"]
    # kept blocks: the union of the group's heads, a contiguous run from the widest band
    # plus block 0
    for b in range(B):
        ib = (int(kv_len[b]) - 1) // T
        for k in range(Hkv):
            blocks = kept_union(ib, hi[k * G:(k + 1) * G], keep[k * G:(k + 1) * G])
            assert nk[b * Hkv + k] == len(blocks), (b, k)
    # splits: ceil(nkept / bps) per group, consecutive, within the slots
    assert ss[0] == 0 and ss[groups] == n_items
    assert all(ss[g + 1] - ss[g] == -(-int(nk[g]) // bps) for g in range(groups))
    slots = max(2 * groups, 512)
    assert n_items <= slots and bps >= 4
    target = max(4, -(-int(nk.sum()) // (6 * sms)))
    if bps > target:   # enlarged only as far as the slots require
        assert sum(-(-int(n) // (bps - 1)) for n in nk) > slots
    # the last phase: every group once, non-increasing cost
    assert sorted(fo.tolist()) == list(range(groups))
    def cost(g):
        n = int(ss[g + 1] - ss[g])
        first = int(nk[g]) - (n - 1) * bps
        band = max(hi[(g % Hkv) * G:(g % Hkv + 1) * G]) if n == 1 else 0
        return min(first + band, 8191)
    costs = [cost(int(g)) for g in fo]
    assert all(costs[i] >= costs[i + 1] for i in range(groups - 1))
    # the items as the kernel maps them: full splits of every group first (group-major,
    # the positions nearest the diagonal), then each group's first positions, in
    # first_order; every position of every group exactly once, every slot exactly once
    n_full = n_items - groups
    cover = [np.zeros(int(n), np.int32) for n in nk]
    seen = np.zeros(n_items, np.int32)
    for item in range(n_items):
        if item < n_full:
            g = max(x for x in range(groups) if ss[x] - x <= item)
            slot = int(ss[g]) + 1 + (item - (int(ss[g]) - g))
        else:
            g = int(fo[item - n_full])
            slot = int(ss[g])
        split = slot - int(ss[g])
        first = int(nk[g]) - (int(ss[g + 1] - ss[g]) - 1) * bps
        p0, p1 = (0, first) if split == 0 else (first + (split - 1) * bps, first + split * bps)
        cover[g][p0:p1] += 1
        seen[slot] += 1
    assert all((c == 1).all() for c in cover) and (seen == 1).all()
    return plan


def test_decode_workload_plan():
    w = W.WORKLOADS["decode"]
    hi, keep = W.policy(w)
    kv = np.full(w.B, w.S, np.int32)
    plan = check_plan(w.B, w.Hq, w.Hkv, w.T, w.S, kv, hi, keep, 148)
    # about six items per SM, each group in one or two items
    assert 5 * 148 <= plan["n_items"] <= 2 * w.B * w.Hkv


@pytest.mark.parametrize("seed", range(6))
def test_random_plans(seed):
    rng = np.random.RandomState(seed)
    Hkv = int(rng.choice([1, 2, 8]))
    G = int(rng.choice([1, 2, 4, 8]))
    B, T = int(rng.randint(1, 40)), int(rng.choice([64, 128]))
    cap = T * int(rng.randint(1, 300))
    kv = rng.randint(1, cap + 1, size=B).astype(np.int32)
    hi = rng.randint(0, 20, size=Hkv * G).astype(np.int32)
    keep = (hi + rng.randint(0, 200, size=Hkv * G)).astype(np.int32)
    check_plan(B, Hkv * G, Hkv, T, cap, kv, hi, keep, int(rng.choice([1, 20, 148])))


def test_plan_rejects_bad_arguments():
    with pytest.raises(tria.TriaError):
        tria.tria_decode_plan(1, 4, 3, 128, 1024, [10], [1, 1, 1, 1], [2, 2, 2, 2], 148)   # Hq % Hkv
    with pytest.raises(tria.TriaError):
        tria.tria_decode_plan(1, 4, 1, 128, 1024, [2000], [1] * 4, [2] * 4, 148)         # kv_len > capacity
    with pytest.raises(tria.TriaError):
        tria.tria_decode_plan(1, 4, 1, 128, 1024, [10], [3] * 4, [2] * 4, 148)           # keep < hi
