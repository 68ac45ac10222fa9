"""Benchmark of the block-sparse mixed-precision attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the whole path over one batch of the workload: write
the compressed KV cache (int8/int4 codes + scales) from bf16 K/V, the fused
block-sparse mixed-precision prefill (Q codec, operand preparation, tcgen05
kernel), and one decode call for the last token over the cache just written.
For the decode workload a step is the decode call over a pre-written cache.

Printed: one JSON line on rank 0. `value` is whole-job throughput with inputs
resident in HBM; `e2e` times the same calls with the inputs copied from pinned
host memory and the outputs copied back inside the timed region. `roofline`
is for the dominant call (prefill: int8 QK ops at the int8 tensor peak plus
bf16 P.V flops at the bf16 peak, over kept tiles; decode: kept compressed
bytes at the HBM copy bandwidth). `cpu_baseline` is the CPU oracle on a
bounded sample of the same workload, on this host's cores.

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
INT8_OVER_BF16 = 2.0   # nominal dense ratio: 4.5 POPS int8 / 2.25 PFLOPS bf16


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"])}, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled during the timed region.

    NVML (read-only queries) every 5 ms from a thread; nvidia-smi every 200 ms when
    NVML is not importable."""

    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}
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
    kernel source has changed since the counters were taken (hash mismatch)."""
    import hashlib
    import re
    table = ROOT / "profiles" / "traffic.md"
    if not table.exists():
        return None
    for line in table.read_text().splitlines():
        m = re.match(r"^\|\s*(\w+)\s*\|\s*([\w.]+)\s*\|\s*([0-9.eE+]+)\s*\|\s*([\w/.]+)\s*\|\s*([0-9a-f]{12})\s*\|",
                     line)
        if not m or m.group(1) != kernel or m.group(2) != workload:
            continue
        src = ROOT / "block_sparse_mixed_b200" / "csrc" / m.group(4)
        if not src.exists() or hashlib.sha256(src.read_bytes()).hexdigest()[:12] != m.group(5):
            return None
        return float(m.group(3))
    return None


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
    return {"tiles_int8": w.B * n8, "tiles_int4": w.B * n4, "ops_int8": tiles * per, "flop_bf16": tiles * per,
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


def run_gpu(args, rank, world, device):
    from block_sparse_mixed_b200 import tria
    from block_sparse_mixed_b200.build import build
    build()
    w = W.WORKLOADS[args.workload]
    hi, keep = W.policy(w)
    peaks, peak_src = load_peaks()
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    ev = lambda: torch.cuda.Event(enable_timing=True)
    launches_per_step = 0
    if w.kind == "prefill":
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
        work = prefill_work(w, hi, keep, tria)
        dbytes = decode_bytes(w.B, w.Hq, w.Hkv, w.D, w.T, kv_len, hi, keep)
        launches_per_step = 2 + 3 + 2

        def step(times):
            # tria_prefill in its two halves, so that the fused kernel is timed alone
            e = [ev() for _ in range(5)]
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
    else:
        q, K, V, kv_len = W.decode_inputs(w, device=device)
        cache = tria.CompressedKVCache(w.B, w.Hkv, w.D, w.T, w.S, device=device)
        tria.tria_quantize_kv(K, V, cache)
        del K, V
        dws = torch.empty(tria.tria_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, w.T, w.S), dtype=torch.uint8,
                          device=device)
        Od = torch.empty_like(q)
        Ld = torch.empty((w.B, w.Hq), dtype=torch.float32, device=device)
        dbytes = decode_bytes(w.B, w.Hq, w.Hkv, w.D, w.T, kv_len, hi, keep)
        launches_per_step = 2

        def step(times):
            e = [ev() for _ in range(2)]
            e[0].record(stream)
            tria.tria_decode(q, cache, kv_len, hi, keep, workspace=dws, O=Od, LSE=Ld)
            e[1].record(stream)
            times.append(e)

    for _ in range(args.warmup):
        step([])
        flush.zero_()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    times = []
    with ClockSampler(torch.cuda.current_device()) as clk:
        for _ in range(args.steps):
            flush.zero_()           # L2 flush between timed steps (outside the events)
            step(times)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()

    for buf in ([ws, dws] if w.kind == "prefill" else [dws]):
        st = tria.tria_workspace_status(buf)
        if st != 0:
            raise RuntimeError(f"device-side error during the timed steps: {tria.tria_status_string(st)}")
    seg = np.array([[times[k][i].elapsed_time(times[k][i + 1]) for i in range(len(times[k]) - 1)]
                    for k in range(len(times))])          # ms per segment per step
    step_ms = float(seg.sum(axis=1).mean())
    step_ms_max = max_over_ranks(step_ms, world, device)

    res = {"clocks": clk.summary(), "ms_per_step": step_ms_max}
    if w.kind == "prefill":
        tokens = w.B * w.S
        res["value"] = whole_job_rate(tokens, world, step_ms_max)
        q_ms, prep_ms, att_ms, d_ms = (float(seg[:, i].mean()) for i in range(4))
        p_ms = prep_ms + att_ms
        p_i8 = peaks["bf16_tflops"] * INT8_OVER_BF16
        t_roof = work["ops_int8"] / (p_i8 * 1e12) + work["flop_bf16"] / (peaks["bf16_tflops"] * 1e12)
        ops = work["ops_int8"] + work["flop_bf16"]
        achieved = ops / (att_ms / 1e3) / 1e12
        peak = ops / t_roof / 1e12
        res["roofline"] = {"bound": "tensor", "kernel": "prefill_kernel (tria_prefill_attend, fused tcgen05)",
                           "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                           "traffic": recorded_traffic("prefill_kernel", w.name),
                           "peak_note": f"int8 {p_i8:.1f} TOPS (= {peak_src} bf16 burst x {INT8_OVER_BF16:g} nominal "
                                        f"ratio) for QK, bf16 {peaks['bf16_tflops']} TFLOP/s ({peak_src}) for P.V"}
        qkv_bytes = 2 * (K.numel() * 2) + 2 * (K.numel() + K.numel() // 2) + 4 * 4 * K.numel() // w.D
        res["rows"] = {
            "quantize_kv": {"ms": q_ms, "GB/s": qkv_bytes / (q_ms / 1e3) / 1e9,
                            "frac_hbm": qkv_bytes / (q_ms / 1e3) / 1e9 / peaks["hbm_gbs"]},
            "prefill": {"ms": p_ms, "prepare_ms": prep_ms, "attend_ms": att_ms, "TOPS_kept": achieved,
                        "frac_roofline": achieved / peak,
                        "TOPS_kept_whole_call": ops / (p_ms / 1e3) / 1e12, **work},
            "decode": {"ms": d_ms, "kept_bytes": dbytes, "GB/s": dbytes / (d_ms / 1e3) / 1e9,
                       "frac_hbm": dbytes / (d_ms / 1e3) / 1e9 / peaks["hbm_gbs"]},
        }
    else:
        d_ms = float(seg[:, 0].mean())
        gbs = dbytes / (d_ms / 1e3) / 1e9
        res["value"] = whole_job_rate(dbytes, world, step_ms_max) / 1e9
        res["roofline"] = {"bound": "hbm", "kernel": "tria_decode (decode_kernel + decode_merge_kernel)",
                           "achieved": gbs, "peak": peaks["hbm_gbs"],
                           "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                           "traffic": recorded_traffic("decode_kernel", w.name),
                           "peak_note": f"HBM copy bandwidth ({peak_src})"}
        res["rows"] = {"decode": {"ms": d_ms, "kept_bytes": dbytes}}
    res["gpu_launches"] = launches_per_step * args.steps

    # ---- end to end through the same C-ABI calls, host buffers in and out ----
    if w.kind == "prefill":
        hQ, hK, hV = (t.cpu().pin_memory() for t in (Q, K, V))
        hO = torch.empty(O.shape, dtype=O.dtype).pin_memory()
        hL = torch.empty(LSE.shape, dtype=LSE.dtype).pin_memory()
        hOd = torch.empty(Od.shape, dtype=Od.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hQ, hK, hV))
        d2h = sum(t.numel() * t.element_size() for t in (hO, hL, hOd))

        def e2e_step():
            Q.copy_(hQ, non_blocking=True); K.copy_(hK, non_blocking=True); V.copy_(hV, non_blocking=True)
            tria.tria_quantize_kv(K, V, cache)
            tria.tria_prefill(Q, cache, hi, keep, workspace=ws, O=O, LSE=LSE)
            q_last.copy_(Q[:, :, w.S - 1])
            tria.tria_decode(q_last, cache, kv_len, hi, keep, workspace=dws, O=Od, LSE=Ld)
            hO.copy_(O, non_blocking=True); hL.copy_(LSE, non_blocking=True); hOd.copy_(Od, non_blocking=True)
        units = w.B * w.S
    else:
        hq = q.cpu().pin_memory()
        hO = torch.empty(Od.shape, dtype=Od.dtype).pin_memory()
        hL = torch.empty(Ld.shape, dtype=Ld.dtype).pin_memory()
        h2d = hq.numel() * 2
        d2h = hO.numel() * 2 + hL.numel() * 4

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            tria.tria_decode(q, cache, kv_len, hi, keep, workspace=dws, O=Od, LSE=Ld)
            hO.copy_(Od, non_blocking=True); hL.copy_(Ld, non_blocking=True)
        units = None
    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    e_ms = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = ev(), ev()
        a.record(stream)
        e2e_step()
        b.record(stream)
        b.synchronize()
        e_ms.append(a.elapsed_time(b))
    e2e_ms = max_over_ranks(float(np.mean(e_ms)), world, device)
    if units is not None:
        e2e_val, e2e_unit = whole_job_rate(units, world, e2e_ms), "tokens/s"
    else:
        e2e_val, e2e_unit = whole_job_rate(dbytes, world, e2e_ms) / 1e9, "GB/s"
    res["e2e"] = {"value": e2e_val, "unit": e2e_unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                  "ms_per_step": e2e_ms}
    return res


# ---------------------------------------------------------------- oracle (CPU baseline / reference arm)

def oracle_sample(w: W.Workload, budget_s: float, seed: int = 0):
    """Run the CPU oracle on a bounded sample of the workload. Returns (value, unit, sample note, cores)."""
    import oracle
    oracle.build()
    hi, keep = W.policy(w)
    cores = os.cpu_count() or 1
    rng = np.random.RandomState(seed)
    if w.kind == "prefill":
        Q, K, V = W.prefill_inputs(w)
        n_rows, t0, done = 64, time.perf_counter(), 0
        while True:
            picks = rng.randint(0, w.B * w.Hq * w.S, size=n_rows).astype(np.int64)
            a = time.perf_counter()
            oracle.prefill_rows(Q, K, V, w.T, hi, keep, rows=picks, nthreads=cores)
            done += n_rows
            el = time.perf_counter() - a
            if time.perf_counter() - t0 > budget_s:
                break
            n_rows = int(min(8192, max(64, n_rows * 2 if el < budget_s / 4 else n_rows)))
        elapsed = time.perf_counter() - t0
        rows_per_s = done / elapsed
        return rows_per_s / w.Hq, "tokens/s", f"{done} query rows drawn at random with replacement " \
                                               f"(the workload has {w.B * w.Hq * w.S}), " \
                                               f"{elapsed:.1f} s; tokens/s = rows/s / Hq", cores
    # decode: a subset of sequences, each over its full kept cache
    nb = max(1, min(w.B, 2))
    sub = W.scaled(w, B=nb)
    q, K, V, kv = W.decode_inputs(sub)
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.decode(q, K, V, w.T, kv, hi, keep, nthreads=cores)
        reps += 1
        if time.perf_counter() - t0 > budget_s:
            break
    elapsed = time.perf_counter() - t0
    db = decode_bytes(nb, w.Hq, w.Hkv, w.D, w.T, kv, hi, keep) * reps
    return db / elapsed / 1e9, "GB/s", f"{reps} decode calls over {nb} of {w.B} sequences, {elapsed:.1f} s", cores


def metric_name(w):
    return ("prefill tokens/s and kept-tile TOPS % roofline; decode kept-KV GB/s % HBM" if w.kind == "prefill"
            else "decode kept-KV GB/s % HBM")


def config_of(w, args, world):
    return {"workload": f"{w.name}: B{w.B} Hq{w.Hq}/Hkv{w.Hkv} D{w.D} "
                        f"{'S' if w.kind == 'prefill' else 'kv_len'}{w.S} T{w.T}",
            "global_batch": w.B * world, "seq_len": w.S, "parallelism": f"replicas{world}",
            "l2": "flushed between timed steps (256 MiB write)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama_prefill", choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (smaller profiling cases)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.batch > 0:
        W.WORKLOADS[args.workload] = W.scaled(W.WORKLOADS[args.workload], B=args.batch)
    w = W.WORKLOADS[args.workload]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        vals, secs = [], []
        for _ in range(args.warmup):
            oracle_sample(w, budget_s=2.0)
        for k in range(args.steps):
            t0 = time.perf_counter()
            v, unit, note, cores = oracle_sample(w, budget_s=args.cpu_budget / max(1, args.steps), seed=k + 1)
            secs.append(time.perf_counter() - t0)
            vals.append(v)
        v = float(np.mean(vals))
        # n_gpus 0: this arm is the CPU oracle; a step is one bounded sample of the workload
        print(json.dumps({"impl": "reference", "metric": metric_name(w), "value": v, "unit": unit, "n_gpus": 0,
                          "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": 1e3 * float(np.mean(secs)), "higher_is_better": True,
                          "scaling": "weak", "vs_baseline": None, "dtype": "f64 softmax / int codes",
                          "data": "synthetic", "config": config_of(w, args, 1),
                          "cpu_baseline": {"value": v, "unit": unit, "cores": cores, "kind": "oracle",
                                           "sample": note},
                          "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
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
                "gpu_launches": res["gpu_launches"], "clocks": res["clocks"]}
        if world == 1 and args.cpu_budget > 0:
            v, unit, note, cores = oracle_sample(w, budget_s=args.cpu_budget)
            line["cpu_baseline"] = {"value": v, "unit": unit, "cores": cores, "kind": "oracle", "sample": note}
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
