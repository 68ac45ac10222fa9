"""Benchmark of the block-sparse mixed-precision attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--legs LIST] [--impl reference]

One step = one pass of the whole path over one batch of the workload: write
the compressed KV cache (int8/int4 codes + scales) from bf16 K/V, the fused
block-sparse mixed-precision prefill (Q codec, operand preparation, tcgen05
kernel), and one decode call for the last token over the cache just written.
For the decode workload a step is the decode call over a pre-written cache.

The default workload is the largest single-GPU one: 65,536-token prefill with
cache write (B1, 32/8 heads, D128, T128). The same run also times, as rows of
the line, the 64-sequence decode over a 32,768-token compressed cache, the
8,192-token prefill, the 8,192-token and 65,536-token prefills with one policy per KV
head (the GQA-shared kernel's case) and the two-sequence 32,768-token prefill;
`--legs none` skips them.

Printed: one JSON line on rank 0. `value` is whole-job throughput with inputs
resident in HBM; `e2e` times the same calls with the inputs copied from pinned
host memory and the outputs copied back inside the timed region. `roofline`
is for the dominant kernel (the fused prefill: int8 QK ops at the measured
int8 tensor peak plus bf16 P.V flops at the measured bf16 peak, over kept
tiles; decode: kept compressed bytes at the HBM copy bandwidth).
`cpu_baseline` is the CPU oracle on a fixed subset of the same workload, on
this host's cores, extrapolated to the whole workload by its exact share of
the work.

Multi-GPU (torchrun): each rank runs its own independent copy of the workload
(no collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

import numpy as np
import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

from block_sparse_mixed_b200 import workloads as W  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 2.0   # nominal dense ratio 4.5 POPS int8 / 2.25 PFLOPS bf16: used only if the measurement fails
DEFAULT_LEGS = ("decode", "llama_prefill", "llama_prefill_gqa", "long_prefill", "max_prefill_gqa")


def load_peaks():
    """Measured HBM copy and bf16 GEMM peaks when the measured-peaks file is present and
    readable (top-level keys hbm_gbs, bf16_tflops, optional bf16_tflops_sustained),
    else the fallback figures."""
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        try:
            d = json.loads(p.read_text())
            out = {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"])}
            out["bf16_tflops_sustained"] = float(d.get("bf16_tflops_sustained", out["bf16_tflops"]))
            return out, "measured"
        except (ValueError, KeyError, TypeError) as e:
            print(f"bench: MEASURED_PEAKS.json not usable ({e!r}); fallback peaks", file=sys.stderr)
    return dict(PEAKS_FALLBACK), "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled during the timed region.

    NVML (read-only queries) every 5 ms from a thread; nvidia-smi every 200 ms when
    NVML is not importable."""

    # NVML clock-event reason bits
    REASONS = {0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.sm, self.mx, self.reasons = [], [], set()
        self._nv = None
        self._stop = threading.Event()
        self._t = None

    def _run_nvml(self, nv):
        h = nv.nvmlDeviceGetHandleByIndex(self.idx)
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self._stop.is_set():
            self.sm.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
            self.mx.append(float(mx))
            bits = int(get_reasons(h))
            self.reasons.update(name for bit, name in self.REASONS.items() if bits & bit)
            other = bits & ~(0x1 | sum(self.REASONS))   # 0x1: idle
            if other:
                self.reasons.add(f"other_{other:#x}")
            self._stop.wait(0.005)

    def _run_smi(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                     timeout=5).stdout.strip()
                f = [x.strip() for x in out.split(",")]
                if len(f) >= 9:
                    self.sm.append(float(f[1]))
                    self.mx.append(float(f[2]))
                    self.reasons.update(names[k] for k in range(4) if f[5 + k].lower() == "active")
            except Exception:
                pass
            self._stop.wait(0.2)

    def _run(self):
        if self._nv is None:
            self._run_smi()
            return
        try:
            self._run_nvml(self._nv)
        finally:
            self._nv.nvmlShutdown()

    def __enter__(self):
        try:   # NVML is brought up before the timed region starts
            import pynvml as nv
            nv.nvmlInit()
            self._nv = nv
        except Exception:
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        t0 = time.time()
        while not self.sm and time.time() - t0 < 2.0:   # first sample taken before timing starts
            time.sleep(0.001)
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._t.join(timeout=10)

    def summary(self):
        if not self.sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(self.sm), "sm_max_mhz": max(self.mx),
                "reasons": sorted(self.reasons), "samples": len(self.sm)}


# ---------------------------------------------------------------- ncu traffic

def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch (read + write) of `kernel` on `workload`, from the ncu
    summary table in profiles/traffic.md, or None when there is no entry or the
    kernel's sources have changed since the counters were taken (hash mismatch: the
    digest covers the kernel's file and the headers every kernel includes)."""
    import re
    table = ROOT / "profiles" / "traffic.md"
    if not table.exists():
        return None
    for line in table.read_text().splitlines():
        m = re.match(r"^\|\s*(\w+)\s*\|\s*([\w.]+)\s*\|\s*([0-9.eE+]+)\s*\|\s*([\w/.]+)\s*\|\s*([0-9a-f]{12})\s*\|",
                     line)
        if not m or m.group(1) != kernel or m.group(2) != workload:
            continue
        if kernel_digest(m.group(4)) != m.group(5):
            return None
        return float(m.group(3))
    return None


KERNEL_HEADERS = ("common.cuh", "kernels.h", "load_plan.cuh", "prefill_common.cuh")


def kernel_digest(name: str):
    """First 12 hex digits of the SHA-256 of a kernel source file followed by the shared
    headers (in the order of KERNEL_HEADERS), or None if a file is missing."""
    import hashlib
    csrc = ROOT / "block_sparse_mixed_b200" / "csrc"
    h = hashlib.sha256()
    for f in (name,) + KERNEL_HEADERS:
        p = csrc / f
        if not p.exists():
            return None
        h.update(p.read_bytes())
    return h.hexdigest()[:12]


# ---------------------------------------------------------------- accounting

def prefill_work(w: W.Workload, hi, keep, tria):
    """Kept tiles and algorithmic ops: 2*T*T*D int8 ops (QK) + 2*T*T*D bf16 flops (P.V) per kept tile."""
    n8 = n4 = 0
    for h, k in zip(hi.tolist(), keep.tolist()):
        c = tria.tria_count_tiles(w.nb, h, k)
        n8 += c[0]
        n4 += c[1]
    tiles = w.B * (n8 + n4)
    per = 2 * w.T * w.T * w.D
    # diagonal tiles (one per query block, always 8-bit) count whole, as executed; the
    # causal count keeps only their T (T + 1) / 2 visible (query, key) pairs
    diag = w.B * len(hi) * w.nb
    causal = (tiles - diag) * per + diag * per * (w.T + 1) / (2 * w.T)
    return {"tiles_int8": w.B * n8, "tiles_int4": w.B * n4, "ops_int8": tiles * per, "flop_bf16": tiles * per,
            "tiles_diagonal": diag, "ops_int8_causal": causal, "flop_bf16_causal": causal,
            "kept_fraction": (n8 + n4) / (len(hi) * w.nb * (w.nb + 1) / 2), "int4_share": n4 / max(1, n8 + n4)}


def decode_bytes(B, Hq, Hkv, D, T, kv_len, hi, keep):
    """Kept compressed bytes a decode call must read, plus q in and O/LSE out."""
    G = Hq // Hkv
    total = 0
    for b in range(B):
        ib = (int(kv_len[b]) - 1) // T
        for k in range(Hkv):
            for j in range(ib + 1):
                acts = set()
                for h in range(G):
                    hh, kk = int(hi[k * G + h]), int(keep[k * G + h])
                    d = ib - j
                    a = 8 if (j == 0 or j == ib or d < hh) else (4 if d < kk else 0)
                    acts.add(a)
                tok = min(T, int(kv_len[b]) - j * T)
                if 8 in acts:
                    total += 2 * tok * D + 2 * tok * 4
                if 4 in acts:
                    total += 2 * tok * D // 2 + 2 * tok * 4
    total += B * Hq * D * 2 + B * Hq * (D * 2 + 4)
    return total


def measure_int8_peak(device, n: int = 8192, reps: int = 10):
    """Dense int8 tensor throughput of this GPU: torch._int_mm (cuBLASLt) on n^3, best of
    `reps` CUDA-event timings after warm-up. Returns (TOPS, how) or (None, reason)."""
    try:
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device)
        best = None
        for name, bb in (("B row-major", b), ("B column-major", b.t().contiguous().t())):
            for _ in range(3):
                torch._int_mm(a, bb)
            torch.cuda.synchronize()
            for _ in range(reps):
                s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                s.record()
                torch._int_mm(a, bb)
                e.record()
                e.synchronize()
                tops = 2 * n ** 3 / (s.elapsed_time(e) / 1e3) / 1e12
                if best is None or tops > best[0]:
                    best = (tops, f"torch._int_mm int8 {n}^3, {name}, best of {reps}")
        del a, b
        return best
    except Exception as ex:   # no int8 GEMM on this build: caller falls back to the nominal ratio
        return None, f"int8 GEMM unavailable ({type(ex).__name__})"


# ---------------------------------------------------------------- GPU arm

def max_over_ranks(x: float, world: int, device) -> float:
    """The largest x over all ranks: a job's step takes as long as its slowest rank."""
    if world <= 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Units that all ranks processed, per second of the slowest rank's time."""
    return units_per_rank * world / (ms / 1e3)


def _ev():
    return torch.cuda.Event(enable_timing=True)


def _timed(step, steps, warmup, flush, clocks=None):
    """Run `step(times)` warmup + steps times (L2 flushed before each, outside the
    events); returns [steps, segments] ms from the events each step recorded."""
    for _ in range(warmup):
        step([])
        flush.zero_()
    torch.cuda.synchronize()
    times = []
    if clocks is not None:
        clocks.__enter__()
    try:
        for _ in range(steps):
            flush.zero_()
            step(times)
        torch.cuda.synchronize()
    finally:
        if clocks is not None:
            clocks.__exit__(None, None, None)
    return np.array([[t[i].elapsed_time(t[i + 1]) for i in range(len(t) - 1)] for t in times])


def _e2e(e2e_step, steps, warmup, flush, stream):
    for _ in range(max(1, warmup)):
        e2e_step()
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        flush.zero_()
        a, b = _ev(), _ev()
        a.record(stream)
        e2e_step()
        b.record(stream)
        b.synchronize()
        ms.append(a.elapsed_time(b))
    return float(np.mean(ms))


def prefill_leg(tria, w, args, flush, stream, clocks=None, e2e=True):
    """Time the prefill step of workload w: cache write, prefill (prepare, attend), last-token decode."""
    hi, keep = W.policy(w)
    device = flush.device
    Q, K, V = W.prefill_inputs(w, device=device)
    cache = tria.CompressedKVCache(w.B, w.Hkv, w.D, w.T, w.S, device=device)
    ws = torch.empty(tria.tria_prefill_workspace_bytes(w.B, w.Hq, w.Hkv, w.S, w.D, w.T), dtype=torch.uint8,
                     device=device)
    dws = torch.empty(tria.tria_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, w.T, w.S), dtype=torch.uint8,
                      device=device)
    O = torch.empty_like(Q)
    LSE = torch.empty((w.B, w.Hq, w.S), dtype=torch.float32, device=device)
    q_last = Q[:, :, w.S - 1].contiguous()
    kv_len = np.full(w.B, w.S, np.int32)
    Od = torch.empty_like(q_last)
    Ld = torch.empty((w.B, w.Hq), dtype=torch.float32, device=device)

    def step(times):
        # tria_prefill in its two halves, so that the fused kernel is timed alone
        e = [_ev() for _ in range(5)]
        e[0].record(stream)
        tria.tria_quantize_kv(K, V, cache)
        e[1].record(stream)
        tria.tria_prefill_prepare(Q, cache, ws)
        e[2].record(stream)
        tria.tria_prefill_attend(cache, hi, keep, ws, O, LSE)
        e[3].record(stream)
        tria.tria_decode(q_last, cache, kv_len, hi, keep, workspace=dws, O=Od, LSE=Ld)
        e[4].record(stream)
        times.append(e)

    seg = _timed(step, args.steps, args.warmup, flush, clocks)
    for buf in (ws, dws):
        st = tria.tria_workspace_status(buf)
        if st != 0:
            raise RuntimeError(f"{w.name}: device-side error during the timed steps: {tria.tria_status_string(st)}")
    q_ms, prep_ms, att_ms, d_ms = (float(seg[:, i].mean()) for i in range(4))
    out = {"step_ms": float(seg.sum(axis=1).mean()), "quantize_kv_ms": q_ms, "prepare_ms": prep_ms,
           "attend_ms": att_ms, "attend_ms_min": float(seg[:, 2].min()), "decode_ms": d_ms,
           "work": prefill_work(w, hi, keep, tria),
           "decode_bytes": decode_bytes(w.B, w.Hq, w.Hkv, w.D, w.T, kv_len, hi, keep),
           "codec_bytes": 2 * (K.numel() * 2) + 2 * (K.numel() + K.numel() // 2) + 4 * 4 * K.numel() // w.D,
           # cache write (one launch for K and V), Q codec + preparation, fused kernel,
           # decode + merge
           "launches_per_step": 1 + 2 + 1 + 2}
    if e2e:
        # The user's call from host memory: tria_prefill_host writes the cache and runs the
        # prefill group by group, its copies in and out overlapping the kernels; then the
        # last token's decode from its host query row.
        hQ, hK, hV = (t.cpu().pin_memory() for t in (Q, K, V))
        hq_last = q_last.cpu().pin_memory()
        hO = torch.empty(O.shape, dtype=O.dtype).pin_memory()
        hL = torch.empty(LSE.shape, dtype=LSE.dtype).pin_memory()
        hOd = torch.empty(Od.shape, dtype=Od.dtype).pin_memory()
        del O, LSE, ws
        torch.cuda.empty_cache()
        host_prefill = tria.HostPrefill(w.B, w.Hq, w.Hkv, w.S, w.D, w.T, device=device)

        def e2e_step():
            host_prefill(hQ, hK, hV, cache, hi, keep, hO, hL, stream=stream)
            q_last.copy_(hq_last, non_blocking=True)
            tria.tria_decode(q_last, cache, kv_len, hi, keep, workspace=dws, O=Od, LSE=Ld)
            hOd.copy_(Od, non_blocking=True)

        out["e2e_ms"] = _e2e(e2e_step, args.steps, args.warmup, flush, stream)
        st = tria.tria_workspace_status(host_prefill.workspace)
        if st != 0:
            raise RuntimeError(f"{w.name}: device-side error in the host-buffer prefill: {tria.tria_status_string(st)}")
        out["h2d"] = sum(t.numel() * t.element_size() for t in (hQ, hK, hV, hq_last))
        out["d2h"] = sum(t.numel() * t.element_size() for t in (hO, hL, hOd))
    return out


def decode_leg(tria, w, args, flush, stream, clocks=None, e2e=True):
    """Time the decode call of workload w over a cache written before the timed region."""
    hi, keep = W.policy(w)
    device = flush.device
    q, K, V, kv_len = W.decode_inputs(w, device=device)
    cache = tria.CompressedKVCache(w.B, w.Hkv, w.D, w.T, w.S, device=device)
    tria.tria_quantize_kv(K, V, cache)
    del K, V
    dws = torch.empty(tria.tria_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, w.T, w.S), dtype=torch.uint8,
                      device=device)
    Od = torch.empty_like(q)
    Ld = torch.empty((w.B, w.Hq), dtype=torch.float32, device=device)

    def step(times):
        e = [_ev() for _ in range(2)]
        e[0].record(stream)
        tria.tria_decode(q, cache, kv_len, hi, keep, workspace=dws, O=Od, LSE=Ld)
        e[1].record(stream)
        times.append(e)

    seg = _timed(step, args.steps, args.warmup, flush, clocks)
    st = tria.tria_workspace_status(dws)
    if st != 0:
        raise RuntimeError(f"{w.name}: device-side error during the timed steps: {tria.tria_status_string(st)}")
    out = {"step_ms": float(seg[:, 0].mean()), "decode_ms": float(seg[:, 0].mean()),
           "decode_ms_min": float(seg[:, 0].min()),
           "decode_bytes": decode_bytes(w.B, w.Hq, w.Hkv, w.D, w.T, kv_len, hi, keep), "launches_per_step": 2}
    if e2e:
        hq = q.cpu().pin_memory()
        hO = torch.empty(Od.shape, dtype=Od.dtype).pin_memory()
        hL = torch.empty(Ld.shape, dtype=Ld.dtype).pin_memory()

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            tria.tria_decode(q, cache, kv_len, hi, keep, workspace=dws, O=Od, LSE=Ld)
            hO.copy_(Od, non_blocking=True); hL.copy_(Ld, non_blocking=True)

        out["e2e_ms"] = _e2e(e2e_step, args.steps, args.warmup, flush, stream)
        out["h2d"] = hq.numel() * 2
        out["d2h"] = hO.numel() * 2 + hL.numel() * 4
    return out


def prefill_roofline(w, r, peaks):
    """Roofline of the fused prefill kernel on kept tiles: t_roof = ops_i8 / P_i8 + flop_bf16 / P_bf16."""
    work = r["work"]
    p_i8, p_bf16 = peaks["int8_tops"], peaks["bf16_tflops"]
    t_roof = work["ops_int8"] / (p_i8 * 1e12) + work["flop_bf16"] / (p_bf16 * 1e12)
    ops = work["ops_int8"] + work["flop_bf16"]
    achieved = ops / (r["attend_ms"] / 1e3) / 1e12
    peak = ops / t_roof / 1e12
    return achieved, peak


def prefill_rows(w, r, peaks):
    achieved, peak = prefill_roofline(w, r, peaks)
    ops = r["work"]["ops_int8"] + r["work"]["flop_bf16"]
    p_ms = r["prepare_ms"] + r["attend_ms"]
    hbm = peaks["hbm_gbs"]
    return {
        "step_ms": r["step_ms"], "tokens_per_s": w.B * w.S / (r["step_ms"] / 1e3),
        "quantize_kv": {"ms": r["quantize_kv_ms"], "GB/s": r["codec_bytes"] / (r["quantize_kv_ms"] / 1e3) / 1e9,
                        "frac_hbm": r["codec_bytes"] / (r["quantize_kv_ms"] / 1e3) / 1e9 / hbm},
        "prefill": {"ms": p_ms, "prepare_ms": r["prepare_ms"], "attend_ms": r["attend_ms"],
                    "attend_ms_min": r["attend_ms_min"], "TOPS_kept": achieved, "frac_roofline": achieved / peak,
                    "TOPS_kept_whole_call": ops / (p_ms / 1e3) / 1e12,
                    "TOPS_kept_causal": (r["work"]["ops_int8_causal"] + r["work"]["flop_bf16_causal"])
                    / (r["attend_ms"] / 1e3) / 1e12, **r["work"]},
        "decode_last_token": {"ms": r["decode_ms"], "kept_bytes": r["decode_bytes"],
                              "GB/s": r["decode_bytes"] / (r["decode_ms"] / 1e3) / 1e9},
    }


def decode_rows(w, r, peaks):
    gbs = r["decode_bytes"] / (r["decode_ms"] / 1e3) / 1e9
    return {"workload": describe(w), "ms": r["decode_ms"], "ms_min": r["decode_ms_min"],
            "kept_bytes": r["decode_bytes"], "GB/s": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
            "traffic": recorded_traffic("decode_kernel", w.name)}


def run_gpu(args, rank, world, device):
    from block_sparse_mixed_b200 import tria
    from block_sparse_mixed_b200.build import build
    build()
    w = W.WORKLOADS[args.workload]
    peaks, peak_src = load_peaks()
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    i8, i8_note = measure_int8_peak(device)
    if i8 is None:
        i8, i8_note = peaks["bf16_tflops"] * INT8_OVER_BF16, f"assumed {peak_src} bf16 x {INT8_OVER_BF16:g} ({i8_note})"
    else:
        i8_note = "measured live: " + i8_note
    peaks["int8_tops"] = i8

    clk = ClockSampler(torch.cuda.current_device())
    res = {}
    if w.kind == "prefill":
        r = prefill_leg(tria, w, args, flush, stream, clocks=clk)
        step_ms = max_over_ranks(r["step_ms"], world, device)
        res["value"] = whole_job_rate(w.B * w.S, world, step_ms)
        achieved, peak = prefill_roofline(w, r, peaks)
        # context only: the same roofline with both peaks scaled to the sustained (power-capped) bf16 figure
        sus = peaks["bf16_tflops_sustained"] / peaks["bf16_tflops"]
        res["roofline"] = {"bound": "tensor", "kernel": "prefill_kernel (tria_prefill_attend, fused tcgen05)",
                           "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                           "frac_vs_sustained_peaks": achieved / (peak * sus),
                           "traffic": recorded_traffic("prefill_kernel", w.name),
                           "peak_note": f"of measured: int8 {i8:.1f} TOPS ({i8_note}) for QK; bf16 "
                                        f"{peaks['bf16_tflops']} TFLOP/s ({peak_src}, burst) for P.V; "
                                        f"achieved = kept-tile ops / mean attend time; frac_vs_sustained_peaks "
                                        f"scales both peaks by the sustained/burst bf16 ratio {sus:.3f}"}
        res["rows"] = prefill_rows(w, r, peaks)
        e2e_val, e2e_unit = whole_job_rate(w.B * w.S, world, max_over_ranks(r["e2e_ms"], world, device)), "tokens/s"
    else:
        r = decode_leg(tria, w, args, flush, stream, clocks=clk)
        step_ms = max_over_ranks(r["step_ms"], world, device)
        res["value"] = whole_job_rate(r["decode_bytes"], world, step_ms) / 1e9
        gbs = r["decode_bytes"] / (r["decode_ms"] / 1e3) / 1e9
        res["roofline"] = {"bound": "hbm", "kernel": "tria_decode (decode_kernel + decode_merge_kernel)",
                           "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                           "traffic": recorded_traffic("decode_kernel", w.name),
                           "peak_note": f"of measured: HBM copy bandwidth ({peak_src})"}
        res["rows"] = {"decode": decode_rows(w, r, peaks)}
        e2e_val = whole_job_rate(r["decode_bytes"], world, max_over_ranks(r["e2e_ms"], world, device)) / 1e9
        e2e_unit = "GB/s"
    res["ms_per_step"] = step_ms
    res["clocks"] = clk.summary()
    res["gpu_launches"] = r["launches_per_step"] * args.steps
    res["e2e"] = {"value": e2e_val, "unit": e2e_unit, "h2d_bytes_per_step": r["h2d"],
                  "d2h_bytes_per_step": r["d2h"], "ms_per_step": r["e2e_ms"]}
    res["peaks"] = {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"], "int8_tops": i8,
                    "int8_note": i8_note, "source": peak_src}
    del r
    torch.cuda.empty_cache()

    # Other workloads of the same path, timed in the same run (rows, not the headline).
    for name in args.legs:
        if name == args.workload:
            continue
        lw = W.WORKLOADS[name]
        lclk = ClockSampler(torch.cuda.current_device())
        if lw.kind == "decode":
            lr = decode_leg(tria, lw, args, flush, stream, clocks=lclk, e2e=False)
            res["rows"][f"{name}_workload"] = {**decode_rows(lw, lr, peaks), "clocks": lclk.summary()}
        else:
            lr = prefill_leg(tria, lw, args, flush, stream, clocks=lclk, e2e=False)
            achieved, peak = prefill_roofline(lw, lr, peaks)
            res["rows"][f"{name}_workload"] = {"workload": describe(lw), **prefill_rows(lw, lr, peaks),
                                               "frac_roofline": achieved / peak,
                                               "traffic": recorded_traffic("prefill_kernel", lw.name),
                                               "clocks": lclk.summary()}
        del lr
        torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- oracle (CPU baseline / reference arm)

def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def kept_keys_of_rows(w: W.Workload, hi, keep, picks):
    """Keys each sampled query row attends to (the oracle's work per row), from the oracle's
    own tile actions: every kept block below the diagonal gives T keys, the diagonal t % T + 1."""
    import oracle
    maps = {}
    out = np.empty(len(picks), np.int64)
    for n, (b, h, t) in enumerate(picks):
        key = (int(hi[h]), int(keep[h]))
        if key not in maps:
            amap = oracle.action_map(w.nb, *key)
            kept = (amap == oracle.INT8) | (amap == oracle.INT4)
            maps[key] = kept.sum(axis=1) - 1          # kept blocks below the diagonal, per query block
        i = t // w.T
        out[n] = maps[key][i] * w.T + (t % w.T) + 1
    return out


def prefill_subset(w: W.Workload, block_phase: int, block_stride: int = 16, row_stride: int = 8):
    """A fixed deterministic subset of query rows: query blocks i = block_phase mod block_stride
    of every (batch, head), every row_stride-th row inside each (all rows when the workload is
    small enough for the oracle to take whole)."""
    if w.B * w.Hq * w.S <= 1 << 14:
        return [(b, h, t) for b in range(w.B) for h in range(w.Hq) for t in range(w.S)]
    blocks = [i for i in range(w.nb) if i % block_stride == block_phase % block_stride]
    return [(b, h, i * w.T + r) for b in range(w.B) for h in range(w.Hq) for i in blocks
            for r in range(row_stride - 1, w.T, row_stride)]


def oracle_prefill_sample(w: W.Workload, inputs, picks, nthreads):
    """Time the oracle on `picks` and extrapolate to the whole workload.

    Every oracle call quantises all of K and V once (single-threaded) before its rows;
    the whole workload would do that once, so the extrapolation is
    t_quant + (t_sample - t_quant) / (work share of the sample), t_quant timed on a
    one-row call and the share counted in kept keys per row."""
    import oracle
    Q, K, V = inputs
    hi, keep = W.policy(w)
    t0 = time.perf_counter()
    oracle.prefill_rows(Q, K, V, w.T, hi, keep, rows=np.array([0], np.int64), nthreads=1)
    t_quant = time.perf_counter() - t0
    rows = np.array([(b * w.Hq + h) * w.S + t for b, h, t in picks], np.int64)
    t0 = time.perf_counter()
    oracle.prefill_rows(Q, K, V, w.T, hi, keep, rows=rows, nthreads=nthreads)
    t_sample = time.perf_counter() - t0
    all_rows = [(0, h, t) for h in range(w.Hq) for t in range(w.S)]    # batches repeat the policy
    share = kept_keys_of_rows(w, hi, keep, picks).sum() / (w.B * kept_keys_of_rows(w, hi, keep, all_rows).sum())
    t_full = t_quant + max(t_sample - t_quant, 0.0) / share
    return w.B * w.S / t_full, t_sample, t_full, share, len(picks)


def oracle_decode_sample(w: W.Workload, n_seq: int, nthreads: int):
    import oracle
    hi, keep = W.policy(w)
    sub = W.scaled(w, B=n_seq)
    q, K, V, kv = W.decode_inputs(sub)
    t0 = time.perf_counter()
    oracle.decode(q, K, V, w.T, kv, hi, keep, nthreads=nthreads)
    el = time.perf_counter() - t0
    db = decode_bytes(n_seq, w.Hq, w.Hkv, w.D, w.T, kv, hi, keep)
    return db / el / 1e9, el


def cpu_baseline(w: W.Workload):
    """The oracle as it stands on this host's cores: a fixed subset of the workload, all cores,
    plus a single-core time of a smaller subset; both extrapolated to the whole workload."""
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    model = cpu_model()
    if w.kind == "prefill":
        inputs = W.prefill_inputs(w)
        picks = prefill_subset(w, block_phase=15)
        v, t_s, t_f, share, n = oracle_prefill_sample(w, inputs, picks, cores)
        v1, t1, t1f, share1, n1 = oracle_prefill_sample(w, inputs, picks[::16] if len(picks) > 4096 else picks, 1)
        note = (f"extrapolated: {n} query rows (query blocks i = 15 mod 16 of every batch and head, every 8th "
                f"row; {share:.4f} of the workload's kept keys) in {t_s:.1f} s on {cores} threads -> "
                f"{t_f:.0f} s for the whole workload")
        return {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": note,
                "cpu_model": model, "single_core": {"value": v1, "unit": "tokens/s", "rows": n1,
                                                    "sample_s": t1, "extrapolated_s": t1f}}
    n_seq = min(w.B, 2)
    v, el = oracle_decode_sample(w, n_seq, cores)
    v1, el1 = oracle_decode_sample(w, 1, 1)
    note = f"{n_seq} of {w.B} sequences over their full kept cache, {el:.1f} s on {cores} threads"
    return {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": note, "cpu_model": model,
            "single_core": {"value": v1, "unit": "GB/s", "sequences": 1, "sample_s": el1}}


def describe(w):
    return (f"{w.name}: B{w.B} Hq{w.Hq}/Hkv{w.Hkv} D{w.D} "
            f"{'S' if w.kind == 'prefill' else 'kv_len'}{w.S} T{w.T}")


def metric_name(w):
    return ("prefill tokens/s and kept-tile TOPS % roofline; decode kept-KV GB/s % HBM" if w.kind == "prefill"
            else "decode kept-KV GB/s % HBM")


def config_of(w, args, world):
    return {"workload": describe(w), "global_batch": w.B * world, "seq_len": w.S,
            "parallelism": f"replicas{world}", "l2": "flushed between timed steps (256 MiB write)"}


def reference_arm(w, args):
    """The CPU oracle as it stands, on this host's cores: each step times it on a fixed subset of
    the workload (query blocks of one residue mod 16, every 16th row; or one decode sequence) and
    extrapolates to the whole workload by the subset's exact share of the work."""
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    vals, secs = [], []
    inputs = W.prefill_inputs(w) if w.kind == "prefill" else None
    for k in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        if w.kind == "prefill":
            picks = prefill_subset(w, block_phase=k, row_stride=16)
            v, _, _, share, n = oracle_prefill_sample(w, inputs, picks, cores)
            unit = "tokens/s"
            note = (f"per step: {n} query rows (query blocks of one residue mod 16, every 16th row; "
                    f"~{share:.4f} of the kept keys), extrapolated to the whole workload")
        else:
            v, _ = oracle_decode_sample(w, 1, cores)
            unit = "GB/s"
            note = f"per step: 1 of {w.B} sequences over its full kept cache"
        if k >= args.warmup:
            secs.append(time.perf_counter() - t0)
            vals.append(v)
    v = float(np.mean(vals))
    # n_gpus 0: this arm is the CPU oracle; a step is one bounded sample of the workload
    print(json.dumps({"impl": "reference", "metric": metric_name(w), "value": v, "unit": unit, "n_gpus": 0,
                      "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * float(np.mean(secs)),
                      "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                      "dtype": "f64 softmax / int codes", "data": "synthetic", "config": config_of(w, args, 1),
                      "cpu_baseline": {"value": v, "unit": unit, "cores": cores, "kind": "oracle", "sample": note,
                                       "cpu_model": cpu_model()},
                      "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="max_prefill", choices=sorted(W.WORKLOADS))
    ap.add_argument("--legs", default=",".join(DEFAULT_LEGS),
                    help="other workloads timed in the same run, as rows ('none' for none)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=1.0, help="0 skips the CPU baseline")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (smaller profiling cases)")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the number of query heads, keeping the head ratio (smaller profiling cases)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    args.legs = [] if args.legs in ("", "none") else [x for x in args.legs.split(",") if x]
    for name in args.legs:
        if name not in W.WORKLOADS:
            ap.error(f"unknown leg {name}")
    if args.batch > 0 or args.heads > 0:
        w0 = W.WORKLOADS[args.workload]
        ch = {}
        if args.batch > 0:
            ch["B"] = args.batch
        if args.heads > 0:
            ch["Hq"] = args.heads
            ch["Hkv"] = max(1, args.heads * w0.Hkv // w0.Hq)
        # a slice is named apart from its workload, so that nothing recorded for the
        # full workload (the DRAM traffic of profiles/traffic.md) is reported for it
        ch["name"] = f"{w0.name}_slice"
        W.WORKLOADS[args.workload] = W.scaled(w0, **ch)
    w = W.WORKLOADS[args.workload]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            reference_arm(w, args)
        return

    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=300))
    device = torch.device("cuda", local)
    res = run_gpu(args, rank, world, device)
    if rank == 0:
        line = {"metric": metric_name(w), "value": res["value"],
                "unit": "tokens/s" if w.kind == "prefill" else "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "int8/int4 QK, bf16 PV, fp32 softmax",
                "data": "synthetic (seeded N(0,1) bf16; no weights or datasets)", "config": config_of(w, args, world),
                "roofline": res["roofline"], "rows": res.get("rows"), "e2e": res["e2e"],
                "gpu_launches": res["gpu_launches"], "clocks": res["clocks"], "peaks": res["peaks"]}
        if world == 1 and args.cpu_budget > 0:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
