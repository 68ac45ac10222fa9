"""GPU parity of the synthetic per-head calibration and the global allocator.

The rit.work TriAttention page (section "Как калибровка распределяет вычисления
между головами", paragraphs one to three) calibrates each head's boundary pair by
the error it adds after the output projection, normalised by the layer's output
energy, prices candidates by the work of the blocks they keep, and lets a global
allocator spend extra work where it lowers the error most. Here a synthetic layer
(seeded N(0,1) Q/K/V and a random W_O; no trained weights) is calibrated through
the C ABI (tria_calibrate) and checked three ways:
  * the library's errors equal the same quantity formed in float64 from the GPU's
    own prefill outputs (so the quadratic-form kernel is exact up to fp32 sums);
  * they agree with the oracle's float64 errors within the bound that the outputs'
    own parity differences imply (triangle inequality on ||dO W_O[h]||);
  * the library's allocator (tria_allocate) makes the oracle allocator's decisions
    on the same error and cost tables, for a range of budgets.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    from block_sparse_mixed_b200.build import build
    build()
    from block_sparse_mixed_b200 import tria
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return tria


def seeded(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("D,Tb", [(128, 64), (64, 128)])
def test_calibration_errors_and_allocation(T, oracle_mod, D, Tb):
    from oracle import calibration as cal
    B, Hq, Hkv, S, d_model = 1, 4, 2, 1024, 192
    nb = S // Tb
    Q, K, V = seeded((B, Hq, S, D), 51), seeded((B, Hkv, S, D), 52), seeded((B, Hkv, S, D), 53)
    W = seeded((Hq * D, d_model), 54, scale=D ** -0.5)
    cand_hi = np.array([0, 1, 1, 2, 3, nb // 2, nb], np.int32)
    cand_keep = np.array([0, 2, 4, 6, nb // 2, nb, nb], np.int32)
    cache = T.CompressedKVCache(B, Hkv, D, Tb, S)
    T.tria_quantize_kv(K.cuda(), V.cuda(), cache)
    err, energy = T.tria_calibrate(Q.cuda(), cache, W.cuda(), cand_hi, cand_keep)
    assert np.all(np.isfinite(err)) and np.all(energy > 0)
    assert np.all(err[-1] == 0.0)                  # the last candidate is the reference itself

    # 1. the same quantity from the GPU's own outputs, in float64
    Wd = W.double().numpy().reshape(Hq, D, d_model)
    full = np.full(Hq, nb, np.int32)
    O_ref_g = T.tria_prefill(Q.cuda(), cache, full, full)[0].double().cpu().numpy()
    O_c_g = [T.tria_prefill(Q.cuda(), cache, np.full(Hq, h, np.int32), np.full(Hq, k, np.int32))[0]
             .double().cpu().numpy() for h, k in zip(cand_hi, cand_keep)]
    for h in range(Hq):
        e_ref = np.sum((O_ref_g[0, h] @ Wd[h]) ** 2)
        assert abs(energy[h] - e_ref) <= 1e-4 * e_ref
        for c in range(len(cand_hi)):
            e = np.sum(((O_c_g[c][0, h] - O_ref_g[0, h]) @ Wd[h]) ** 2)
            assert abs(err[c, h] - e) <= 1e-4 * e + 1e-9 * e_ref, (c, h, err[c, h], e)

    # 2. the oracle's float64 errors, within the bound the outputs' parity implies
    E_o, energy_o = cal.head_output_errors(Q, K, V, Tb, W, cand_hi, cand_keep)
    O_ref_o = oracle_mod.prefill_rows(Q, K, V, Tb, full, full)[0].reshape(B, Hq, S, D)
    for h in range(Hq):
        wn = np.linalg.norm(Wd[h], 2)
        d_ref = np.sqrt(np.sum((O_ref_g[0, h] - O_ref_o[0, h]) ** 2))
        assert abs(np.sqrt(energy[h]) - np.sqrt(energy_o[h])) <= wn * d_ref * 1.001 + 1e-6
        for c in range(len(cand_hi)):
            O_c_o = oracle_mod.prefill_rows(Q, K, V, Tb, np.full(Hq, cand_hi[c], np.int32),
                                            np.full(Hq, cand_keep[c], np.int32))[0].reshape(B, Hq, S, D)
            d_c = np.sqrt(np.sum((O_c_g[c][0, h] - O_c_o[0, h]) ** 2))
            bound = wn * (d_c + d_ref) * 1.001 + 1e-6
            assert abs(np.sqrt(err[c, h]) - np.sqrt(E_o[c, h])) <= bound, (c, h)

    # 3. allocations: the library's and the oracle's allocator on the same tables
    cost1 = T.tria_calibration_costs(nb, Tb, D, cand_hi, cand_keep)
    assert cost1.tolist() == cal.candidate_costs(nb, Tb, D, cand_hi, cand_keep).tolist()
    cost = np.repeat(cost1[:, None], Hq, axis=1)
    norm_g = err / energy.sum()
    norm_o = E_o / energy_o.sum()
    cheapest, dearest = int(cost1.min()) * Hq, int(cost1.max()) * Hq
    for frac in np.linspace(0.0, 1.0, 11):
        budget = int(cheapest + frac * (dearest - cheapest))
        for table in (norm_g, norm_o):
            assert T.tria_allocate(table, cost, budget).tolist() == cal.allocate(table, cost, budget)
