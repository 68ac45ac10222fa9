"""Pins of the calibration oracle (per-head error after the output projection, block
cost, greedy global allocator) against closed forms, a hand-worked allocation and
properties that any mistake in the slicing of W_O, the normalisation or the
allocator's rule would break.

Source: rit.work TriAttention page, section "Как калибровка распределяет
вычисления между головами", paragraphs one to three.
"""
import numpy as np
import torch

from conftest import GOLDEN
from oracle import calibration as cal

ERR = np.array([[9.0, 4.0, 6.0], [3.0, 3.0, 5.0], [1.0, 0.0, 0.5]])
COST = np.array([[10, 10, 10], [20, 20, 20], [40, 40, 40]], np.int64)


def seeded(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def test_allocation_golden():
    n = 0
    for line in open(GOLDEN / "allocation_example.txt", encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        budget, choice = line.split("|")
        assert cal.allocate(ERR, COST, int(budget)) == [int(x) for x in choice.split()], line
        n += 1
    assert n == 4


def test_allocation_properties():
    rng = np.random.RandomState(5)
    for _ in range(200):
        C, H = rng.randint(1, 6), rng.randint(1, 7)
        cost = rng.randint(1, 50, (C, H)).astype(np.int64)
        err = rng.rand(C, H)
        budget = int(rng.randint(0, 300))
        choice = cal.allocate(err, cost, budget)
        start = [min(range(C), key=lambda c: (cost[c, h], err[c, h], c)) for h in range(H)]
        spent = sum(cost[choice[h], h] for h in range(H))
        assert spent <= max(budget, sum(cost[start[h], h] for h in range(H)))
        # every move made a head costlier and better than its start
        for h in range(H):
            assert choice[h] == start[h] or (cost[choice[h], h] > cost[start[h], h] and err[choice[h], h] < err[start[h], h])
        # with candidates whose error falls as cost rises and an unlimited budget, every
        # head ends at its most precise candidate
        order = np.argsort(cost, axis=0, kind="stable")
        mono_err = np.empty_like(err)
        for h in range(H):
            mono_err[order[:, h], h] = np.sort(err[:, h])[::-1]
        cost_u = cost.copy()
        for h in range(H):
            cost_u[order[:, h], h] = np.arange(1, C + 1) * 7 + h
        choice = cal.allocate(mono_err, cost_u, 10 ** 9)
        assert all(choice[h] == int(np.argmin(mono_err[:, h])) for h in range(H))


def test_tile_costs_hand_counted():
    # T = 2, D = 4: query-key product 2*2*2*4 = 32 operations, value aggregation 32,
    # normalisation 4 per score x 4 scores = 16; at 4 bits the products count half
    assert cal.tile_costs(2, 4) == (80, 48)
    # every causal tile of nb = 5 kept at 8 bits: 15 tiles
    assert cal.candidate_costs(5, 2, 4, [5], [5]).tolist() == [15 * 80]
    # hi = 1, keep = 3 over nb = 8: 15 tiles at 8 bits, 11 at 4 bits (the tile-count pins)
    assert cal.candidate_costs(8, 2, 4, [1], [3]).tolist() == [15 * 80 + 11 * 48]


def test_errors_after_projection(oracle_mod):
    B, Hq, Hkv, S, D, T = 1, 4, 2, 256, 16, 32
    Q, K, V = seeded((B, Hq, S, D), 1), seeded((B, Hkv, S, D), 2), seeded((B, Hkv, S, D), 3)
    nb = S // T
    hi, keep = [nb, 1, 2, 0], [nb, 3, 4, 2]
    # identity projection: the error is the plain squared difference of the head outputs
    W = torch.eye(Hq * D, dtype=torch.float64)
    E, energy = cal.head_output_errors(Q, K, V, T, W, hi, keep)
    O_ref = oracle_mod.prefill_rows(Q, K, V, T, np.full(Hq, nb, np.int32), np.full(Hq, nb, np.int32))[0]
    O_ref = O_ref.reshape(B, Hq, S, D)
    assert np.all(E[0] == 0.0)                                  # the reference candidate itself
    for c in range(1, 4):
        O_c = oracle_mod.prefill_rows(Q, K, V, T, np.full(Hq, hi[c], np.int32), np.full(Hq, keep[c], np.int32))[0]
        d = O_c.reshape(B, Hq, S, D) - O_ref
        for h in range(Hq):
            assert abs(E[c, h] - np.sum(d[:, h] ** 2)) <= 1e-9 * max(1.0, E[c, h])
    for h in range(Hq):
        assert abs(energy[h] - np.sum(O_ref[:, h] ** 2)) <= 1e-9 * energy[h]
    # a projection that only head 2 feeds: every other head has zero error and energy
    W2 = torch.zeros(Hq * D, 8, dtype=torch.float64)
    W2[2 * D:3 * D] = torch.randn(D, 8, dtype=torch.float64, generator=torch.Generator().manual_seed(4))
    E2, en2 = cal.head_output_errors(Q, K, V, T, W2, hi, keep)
    assert np.all(E2[:, [0, 1, 3]] == 0.0) and np.all(en2[[0, 1, 3]] == 0.0)
    assert en2[2] > 0 and np.all(E2[1:, 2] > 0)
    # scaling W_O by 3 scales errors and energy by 9: the normalised error is unchanged
    E3, en3 = cal.head_output_errors(Q, K, V, T, 3 * W2, hi, keep)
    assert np.allclose(E3 / en3.sum(), E2 / en2.sum(), rtol=1e-12, atol=0)
