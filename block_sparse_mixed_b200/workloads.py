"""Seeded synthetic workloads: shapes, bf16 N(0,1) tensors and per-head policies.

This module only draws inputs. It holds none of the attention arithmetic, so the
CPU oracle (test infrastructure) and the GPU library can both be fed from it.

The pages measure TriAttention on Llama, Qwen and Ministral models with prompts
up to 65,536 tokens on unnamed QA suites (rit.work TriAttention page, section
"Когда TriAttention меняет планы инфраструктуры"). Neither those models nor
those suites are available here; the five workloads below are synthetic
stand-ins with the shapes of such models (GQA 32/8 heads, head dim 128).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str          # "prefill" or "decode"
    B: int
    Hq: int
    Hkv: int
    D: int
    S: int             # prefill: sequence length; decode: KV length per sequence
    T: int             # block size (tokens per block)
    seed: int
    policy: str        # how (hi, keep) per query head is drawn
    k_outlier: float = 1.0   # per-channel outlier gain on K (1.0 = none)
    k_outlier_frac: float = 0.0
    fixed_policy: tuple = field(default=())

    @property
    def nb(self) -> int:
        return (self.S + self.T - 1) // self.T


WORKLOADS = {
    "tiny_prefill": Workload("tiny_prefill", "prefill", B=1, Hq=2, Hkv=2, D=64, S=512, T=64,
                             seed=1, policy="fixed", fixed_policy=((1, 3), (2, 5))),
    "llama_prefill": Workload("llama_prefill", "prefill", B=1, Hq=32, Hkv=8, D=128, S=8192,
                              T=64, seed=2, policy="llama", k_outlier=4.0, k_outlier_frac=0.02),
    "long_prefill": Workload("long_prefill", "prefill", B=2, Hq=32, Hkv=8, D=128, S=32768,
                             T=128, seed=3, policy="quarter"),
    "max_prefill": Workload("max_prefill", "prefill", B=1, Hq=32, Hkv=8, D=128, S=65536,
                            T=128, seed=4, policy="maxctx"),
    "decode": Workload("decode", "decode", B=64, Hq=32, Hkv=8, D=128, S=32768, T=128,
                       seed=5, policy="decode"),
    # the 8,192-token shapes with one (hi, keep) per KV head, shared by its 4 query heads
    # (the case the GQA-shared prefill serves)
    "llama_prefill_gqa": Workload("llama_prefill_gqa", "prefill", B=1, Hq=32, Hkv=8, D=128, S=8192,
                                  T=64, seed=6, policy="llama_kv", k_outlier=4.0, k_outlier_frac=0.02),
    # the 65,536-token shape with the max-context distributions drawn once per KV head
    "max_prefill_gqa": Workload("max_prefill_gqa", "prefill", B=1, Hq=32, Hkv=8, D=128, S=65536,
                                T=128, seed=7, policy="maxctx_kv"),
}


def policy(w: Workload) -> tuple[np.ndarray, np.ndarray]:
    """Per-query-head (hi, keep) as two int32 arrays of length Hq (integers inclusive)."""
    rng = np.random.RandomState(1000 + w.seed)
    if w.policy == "fixed":
        hi = np.array([p[0] for p in w.fixed_policy], np.int32)
        keep = np.array([p[1] for p in w.fixed_policy], np.int32)
        return hi, keep
    hi = np.empty(w.Hq, np.int32)
    keep = np.empty(w.Hq, np.int32)
    if w.policy == "llama_kv":         # hi ~ U{1..16}, keep ~ U{hi+1..64} per KV head
        G = w.Hq // w.Hkv
        for k in range(w.Hkv):
            hi[k * G:(k + 1) * G] = rng.randint(1, 17)
            keep[k * G:(k + 1) * G] = rng.randint(hi[k * G] + 1, 65)
        return hi, keep
    if w.policy == "maxctx_kv":        # hi ~ U{2..32}, keep ~ U{hi+8..256} per KV head
        G = w.Hq // w.Hkv
        for k in range(w.Hkv):
            hi[k * G:(k + 1) * G] = rng.randint(2, 33)
            keep[k * G:(k + 1) * G] = rng.randint(hi[k * G] + 8, 257)
        return hi, keep
    for h in range(w.Hq):
        if w.policy == "llama":        # hi ~ U{1..16}, keep ~ U{hi+1..64}
            hi[h] = rng.randint(1, 17)
            keep[h] = rng.randint(hi[h] + 1, 65)
        elif w.policy == "quarter":    # ~25% of causal tiles kept, ~half of them int4
            keep[h] = rng.randint(32, 38)
            hi[h] = rng.randint(15, 19)
        elif w.policy == "maxctx":     # hi ~ U{2..32}, keep ~ U{hi+8..256}
            hi[h] = rng.randint(2, 33)
            keep[h] = rng.randint(hi[h] + 8, 257)
        elif w.policy == "decode":     # hi ~ U{4..16}, keep ~ U{32..128}
            hi[h] = rng.randint(4, 17)
            keep[h] = rng.randint(32, 129)
        else:
            raise ValueError(w.policy)
    return hi, keep


def randn_bf16(shape, seed: int, device="cpu", gain_channels=None, gain: float = 1.0,
               chunk_rows: int = 1 << 22) -> torch.Tensor:
    """N(0,1) draws rounded to bf16, from a torch generator seeded with `seed`.

    gain_channels: optional bool mask over the last dim (or a [lead..., D] mask
    broadcastable over the leading dims); those channels are multiplied by `gain`
    before the bf16 rounding. Large tensors are drawn in row chunks to bound the
    fp32 staging memory.
    """
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    D = shape[-1]
    flat = out.view(-1, D)
    rows = flat.shape[0]
    mask = None
    if gain_channels is not None:
        mask = torch.as_tensor(gain_channels, device=device)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        x = torch.randn((r1 - r0, D), generator=g, device=device, dtype=torch.float32)
        if mask is not None:
            if mask.dim() == 1:
                x[:, mask] *= gain
            else:  # per-row-group mask: [groups, D] with rows laid out group-major
                rows_per_group = rows // mask.shape[0]
                gidx = torch.arange(r0, r1, device=device) // rows_per_group
                x = torch.where(mask[gidx], x * gain, x)
        flat[r0:r1] = x.to(torch.bfloat16)
    return out


def outlier_mask(w: Workload) -> np.ndarray | None:
    """Seeded per-KV-head channel mask: ceil(frac * D) channels per KV head."""
    if w.k_outlier_frac <= 0.0:
        return None
    rng = np.random.RandomState(2000 + w.seed)
    n = int(math.ceil(w.k_outlier_frac * w.D))
    m = np.zeros((w.B * w.Hkv, w.D), dtype=bool)
    for g in range(w.B * w.Hkv):
        m[g, rng.choice(w.D, size=n, replace=False)] = True
    return m


def prefill_inputs(w: Workload, device="cpu"):
    """(Q [B,Hq,S,D], K [B,Hkv,S,D], V [B,Hkv,S,D]) bf16 for a prefill workload."""
    Q = randn_bf16((w.B, w.Hq, w.S, w.D), 10 * w.seed + 1, device)
    mask = outlier_mask(w)
    K = randn_bf16((w.B, w.Hkv, w.S, w.D), 10 * w.seed + 2, device,
                   gain_channels=mask, gain=w.k_outlier)
    V = randn_bf16((w.B, w.Hkv, w.S, w.D), 10 * w.seed + 3, device)
    return Q, K, V


def decode_inputs(w: Workload, device="cpu", kv_len=None):
    """(q [B,Hq,D], K [B,Hkv,S,D], V [B,Hkv,S,D], kv_len [B] int32) for a decode workload."""
    q = randn_bf16((w.B, w.Hq, w.D), 10 * w.seed + 1, device)
    K = randn_bf16((w.B, w.Hkv, w.S, w.D), 10 * w.seed + 2, device)
    V = randn_bf16((w.B, w.Hkv, w.S, w.D), 10 * w.seed + 3, device)
    if kv_len is None:
        kv_len = np.full(w.B, w.S, np.int32)
    return q, K, V, np.ascontiguousarray(kv_len, np.int32)


def scaled(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields replaced (smaller parity cases)."""
    d = dict(w.__dict__)
    d.update(changes)
    return Workload(**d)
