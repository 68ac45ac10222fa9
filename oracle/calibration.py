"""CPU oracle of the synthetic per-head calibration and the global allocator.

TEST INFRASTRUCTURE ONLY, like the rest of this package: the tests and the
benchmark's CPU leg are its only callers, and it shares no code with the GPU
library.

What it follows (rit.work TriAttention page, section "Как калибровка распределяет
вычисления между головами", paragraphs one to three):
  * a set of boundary pairs (hi, keep) is tried for every head separately;
  * the error of a candidate is measured after the output projection W_O, where
    the head's result reaches the next layer, and is normalised by the energy of
    the layer's output so that heads can be compared directly;
  * every candidate has a compute cost that counts whole processed blocks: the
    query-key product, the normalisation of the weights and the aggregation of the
    values;
  * a global allocator then spends extra work where it lowers the error most.

Readings (the page gives no formulas):
  * reference output: the same attention with nothing skipped and every tile at
    8 bits (hi = keep = number of blocks); a candidate's error is therefore what its
    4-bit tiles and skipped blocks add;
  * error of head h under candidate c: E[c, h] = sum over rows of
    ||(O_c[h] - O_ref[h]) W_O[h]||^2, with W_O[h] the D rows of W_O that head h
    feeds; the layer energy is sum_h sum over rows of ||O_ref[h] W_O[h]||^2 (the
    heads' contributions, cross terms between heads dropped, as they are in the
    summed error);
  * cost of a candidate: per kept tile, the query-key product (2 T^2 D operations)
    and the aggregation of values (2 T^2 D) at 8 bits, half of each at 4 bits, and
    4 T^2 for the normalisation (scale, maximum, exponential, sum of every score);
  * allocator: every head starts at its cheapest candidate; then, while the budget
    allows, the single move of one head to a costlier candidate with a lower error
    that has the largest error decrease per unit of added cost is taken (the first
    such move in head-then-candidate order on equal ratios).

Parity pins: tests/test_calibration_pins.py (closed forms, hand-worked golden
allocation, brute force on tiny instances).
"""
from __future__ import annotations

import numpy as np

from . import prefill_rows, action_counts


def tile_costs(T: int, D: int) -> tuple[int, int]:
    """(8-bit tile, 4-bit tile) cost: query-key product + value aggregation at the plane's
    width (4 bits: half the 8-bit operations) + normalisation of the T*T scores."""
    qk_pv_8 = 2 * T * T * D + 2 * T * T * D
    norm = 4 * T * T
    return qk_pv_8 + norm, qk_pv_8 // 2 + norm


def candidate_costs(nb: int, T: int, D: int, cand_hi, cand_keep) -> np.ndarray:
    """Cost of each candidate for one head over nb x nb causal blocks (int64 [C])."""
    c8, c4 = tile_costs(T, D)
    out = []
    for h, k in zip(cand_hi, cand_keep):
        n8, n4, _ = action_counts(nb, int(h), int(k))
        out.append(n8 * c8 + n4 * c4)
    return np.array(out, np.int64)


def head_output_errors(Q, K, V, T: int, W_O, cand_hi, cand_keep, nthreads=None):
    """Per-candidate, per-head error after the output projection, and per-head energy.

    Q [B, Hq, S, D], K/V [B, Hkv, S, D] (bf16), W_O [Hq*D, d_model] (bf16 or float).
    Returns (E [C, Hq] float64, energy [Hq] float64); the normalised error is
    E / energy.sum()."""
    import torch
    B, Hq, S, D = Q.shape
    nb = (S + T - 1) // T
    W = torch.as_tensor(W_O).to(torch.float64).numpy().reshape(Hq, D, -1)

    def outputs(hi, keep):
        O, _ = prefill_rows(Q, K, V, T, np.full(Hq, hi, np.int32), np.full(Hq, keep, np.int32), nthreads=nthreads)
        return O.reshape(B, Hq, S, D)

    O_ref = outputs(nb, nb)
    energy = np.array([np.sum((O_ref[:, h].reshape(-1, D) @ W[h]) ** 2) for h in range(Hq)])
    E = np.zeros((len(cand_hi), Hq))
    for c, (hi, keep) in enumerate(zip(cand_hi, cand_keep)):
        dO = outputs(int(hi), int(keep)) - O_ref
        for h in range(Hq):
            E[c, h] = np.sum((dO[:, h].reshape(-1, D) @ W[h]) ** 2)
    return E, energy


def allocate(err, cost, budget: int) -> list[int]:
    """Greedy global allocation of candidates to heads.

    err [C, H] (float), cost [C, H] (integer), budget: the largest total cost.
    Returns the chosen candidate index of every head."""
    err = [[float(x) for x in row] for row in np.asarray(err, np.float64)]
    cost = [[int(x) for x in row] for row in np.asarray(cost, np.int64)]
    C, H = len(err), len(err[0])
    choice = []
    for h in range(H):
        choice.append(min(range(C), key=lambda c: (cost[c][h], err[c][h], c)))
    spent = sum(cost[choice[h]][h] for h in range(H))
    while True:
        best = None
        for h in range(H):
            for c in range(C):
                added = cost[c][h] - cost[choice[h]][h]
                gain = err[choice[h]][h] - err[c][h]
                if added <= 0 or gain <= 0 or spent + added > budget:
                    continue
                ratio = gain / added
                if best is None or ratio > best[0]:
                    best = (ratio, h, c)
        if best is None:
            return choice
        _, h, c = best
        spent += cost[c][h] - cost[choice[h]][h]
        choice[h] = c
