"""ctypes binding of libtria.so (include/tria.h), same names as the C entry points.

Argument marshalling only: tensors are passed as device pointers with the
current CUDA stream; every step of the computation runs in the library's
kernels. torch is used for device memory and streams. If the library is
missing this module raises at first use -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import re
from pathlib import Path

import numpy as np
import torch

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libtria.so"
HEADER = _PKG.parent / "include" / "tria.h"

TRIA_OK, TRIA_ERR_INVALID_ARG, TRIA_ERR_UNSUPPORTED, TRIA_ERR_CUDA = 0, 1, 2, 3
TRIA_ERR_TIMEOUT, TRIA_ERR_BOUNDS, TRIA_ERR_WORKSPACE = 4, 5, 6


class TriaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {tria_status_string(status)} (status {status})")
        self.status = status


class tria_kv_cache(ctypes.Structure):
    _fields_ = [("k8", ctypes.c_void_p), ("k4", ctypes.c_void_p), ("k8_scale", ctypes.c_void_p),
                ("k4_scale", ctypes.c_void_p), ("v8", ctypes.c_void_p), ("v4", ctypes.c_void_p),
                ("v8_scale", ctypes.c_void_p), ("v4_scale", ctypes.c_void_p),
                ("B", ctypes.c_int), ("Hkv", ctypes.c_int), ("D", ctypes.c_int), ("T", ctypes.c_int),
                ("capacity", ctypes.c_int), ("block_table", ctypes.c_void_p), ("max_blocks", ctypes.c_int),
                ("num_pages", ctypes.c_int), ("status", ctypes.c_void_p)]


class tria_dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("S", ctypes.c_int),
                ("D", ctypes.c_int), ("T", ctypes.c_int)]


_lib = None


def lib():
    """Load libtria.so (raises FileNotFoundError if it has not been built)."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise FileNotFoundError(f"{LIB_PATH} is missing: build it with python -m block_sparse_mixed_b200.build")
        L = ctypes.CDLL(str(LIB_PATH))
        P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        L.tria_status_string.argtypes = [I]
        L.tria_status_string.restype = ctypes.c_char_p
        L.tria_cache_bytes.argtypes = [I, I, I, I, I]
        L.tria_cache_bytes.restype = SZ
        L.tria_cache_init.argtypes = [ctypes.POINTER(tria_kv_cache), P, SZ, I, I, I, I, I]
        L.tria_cache_init.restype = I
        L.tria_paged_cache_bytes.argtypes = [I, I, I, I]
        L.tria_paged_cache_bytes.restype = SZ
        L.tria_paged_cache_init.argtypes = [ctypes.POINTER(tria_kv_cache), P, SZ, I, I, I, I, I, P, I]
        L.tria_paged_cache_init.restype = I
        L.tria_cache_status.argtypes = [ctypes.POINTER(tria_kv_cache), P]
        L.tria_cache_status.restype = I
        L.tria_quantize_rows.argtypes = [P, I64, I, P, P, P, P, P]
        L.tria_quantize_rows.restype = I
        L.tria_quantize_kv.argtypes = [P, P, I, I, ctypes.POINTER(tria_kv_cache), P]
        L.tria_quantize_kv.restype = I
        L.tria_count_tiles.argtypes = [I, I, I, P]
        L.tria_count_tiles.restype = I
        L.tria_prefill_load_plan.argtypes = [I, I, I, I, P, I64, P]
        L.tria_prefill_load_plan.restype = I
        L.tria_decode_plan.argtypes = [I, I, I, I, I, P, P, P, I, P, P, P, P, P]
        L.tria_decode_plan.restype = I
        L.tria_prefill_workspace_bytes.argtypes = [ctypes.POINTER(tria_dims)]
        L.tria_prefill_workspace_bytes.restype = SZ
        L.tria_prefill.argtypes = [P, ctypes.POINTER(tria_kv_cache), ctypes.POINTER(tria_dims), P, P, P, P, P,
                                   SZ, P]
        L.tria_prefill.restype = I
        L.tria_prefill_prepare.argtypes = [P, ctypes.POINTER(tria_kv_cache), ctypes.POINTER(tria_dims), P, SZ, P]
        L.tria_prefill_prepare.restype = I
        L.tria_prefill_attend.argtypes = [ctypes.POINTER(tria_kv_cache), ctypes.POINTER(tria_dims), P, P, P, P, P,
                                          SZ, P]
        L.tria_prefill_attend.restype = I
        L.tria_decode_workspace_bytes.argtypes = [I, I, I, I, I, I]
        L.tria_decode_workspace_bytes.restype = SZ
        L.tria_decode.argtypes = [P, ctypes.POINTER(tria_kv_cache), P, I, P, P, P, P, P, SZ, P]
        L.tria_decode.restype = I
        L.tria_workspace_status.argtypes = [P, P]
        L.tria_workspace_status.restype = I
        _lib = L
    return _lib


def declared_functions() -> list[str]:
    """Names of the functions include/tria.h declares."""
    text = HEADER.read_text()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+[\s\*]+(tria_\w+)\s*\(", text, flags=re.M)))


def tria_status_string(status: int) -> str:
    return lib().tria_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != TRIA_OK:
        raise TriaError(fn, status)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev_ptr(t: torch.Tensor) -> ctypes.c_void_p:
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _host_i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _aligned_empty(nbytes: int, device) -> torch.Tensor:
    """A byte buffer whose start is 256-byte aligned (torch's allocator already aligns to 512)."""
    buf = torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)
    assert buf.data_ptr() % 256 == 0
    return buf


class CompressedKVCache:
    """Caller-owned compressed cache: one device buffer carved by tria_cache_init
    (contiguous [B, Hkv, capacity] rows)."""

    def __init__(self, B: int, Hkv: int, D: int, T: int, capacity: int, device="cuda"):
        n = lib().tria_cache_bytes(B, Hkv, D, T, capacity)
        if n == 0:
            raise TriaError("tria_cache_bytes", TRIA_ERR_INVALID_ARG)
        self.buffer = _aligned_empty(n, device)
        self.buffer[:256].zero_()                  # the status word
        self.struct = tria_kv_cache()
        _check("tria_cache_init", lib().tria_cache_init(ctypes.byref(self.struct), _dev_ptr(self.buffer), n,
                                                         B, Hkv, D, T, capacity))
        self.B, self.Hkv, self.D, self.T, self.capacity = B, Hkv, D, T, capacity
        self.lead = (B, Hkv, capacity)

    def plane(self, name: str) -> torch.Tensor:
        """View of one plane: k8/v8 int8 [*lead, D], k4/v4 uint8 [*lead, D/2], *_scale fp32 [*lead]
        (lead = (B, Hkv, capacity) contiguous, (num_pages, Hkv, T) paged)."""
        base = self.buffer.data_ptr()
        off = getattr(self.struct, name) - base
        rows = int(np.prod(self.lead))
        if name in ("k8", "v8"):
            return self.buffer[off:off + rows * self.D].view(torch.int8).view(*self.lead, self.D)
        if name in ("k4", "v4"):
            return self.buffer[off:off + rows * self.D // 2].view(*self.lead, self.D // 2)
        return self.buffer[off:off + rows * 4].view(torch.float32).view(*self.lead)

    def status(self, stream=None) -> int:
        """The cache's device error word (synchronises; clears it)."""
        return int(lib().tria_cache_status(ctypes.byref(self.struct), _stream(stream)))


class PagedKVCache(CompressedKVCache):
    """Caller-owned paged compressed cache: a pool of `num_pages` pages of T tokens x Hkv
    heads carved by tria_paged_cache_init, addressed through `block_table` (a device int32
    tensor [B, max_blocks] of page ids that the caller owns and may update between calls)."""

    def __init__(self, B: int, Hkv: int, D: int, T: int, num_pages: int, block_table: torch.Tensor,
                 device="cuda"):
        n = lib().tria_paged_cache_bytes(num_pages, Hkv, D, T)
        if n == 0:
            raise TriaError("tria_paged_cache_bytes", TRIA_ERR_INVALID_ARG)
        if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != B:
            raise ValueError("block_table must be a device int32 tensor [B, max_blocks]")
        self.block_table = block_table
        self.buffer = _aligned_empty(n, device)
        self.buffer[:256].zero_()
        self.struct = tria_kv_cache()
        mb = block_table.shape[1]
        _check("tria_paged_cache_init", lib().tria_paged_cache_init(
            ctypes.byref(self.struct), _dev_ptr(self.buffer), n, B, Hkv, D, T, num_pages, _dev_ptr(block_table), mb))
        self.B, self.Hkv, self.D, self.T, self.capacity = B, Hkv, D, T, mb * T
        self.num_pages, self.max_blocks = num_pages, mb
        self.lead = (num_pages, Hkv, T)


def tria_quantize_rows(X: torch.Tensor, int4: bool = True, stream=None):
    """Codec over the rows of X (bf16 [..., D]): (c8 int8, s8 fp32, c4 uint8 packed, s4 fp32)."""
    D = X.shape[-1]
    rows = X.numel() // D
    c8 = torch.empty((rows, D), dtype=torch.int8, device=X.device)
    s8 = torch.empty(rows, dtype=torch.float32, device=X.device)
    c4 = torch.empty((rows, D // 2), dtype=torch.uint8, device=X.device) if int4 else None
    s4 = torch.empty(rows, dtype=torch.float32, device=X.device) if int4 else None
    _check("tria_quantize_rows", lib().tria_quantize_rows(
        _dev_ptr(X), rows, D, _dev_ptr(c8), _dev_ptr(s8), _dev_ptr(c4) if int4 else None,
        _dev_ptr(s4) if int4 else None, _stream(stream)))
    return c8, s8, c4, s4


def tria_quantize_kv(K: torch.Tensor, V: torch.Tensor, cache: CompressedKVCache, start: int = 0, stream=None):
    """Write K/V (bf16 [B,Hkv,S,D]) into cache positions [start, start+S)."""
    S = K.shape[2]
    _check("tria_quantize_kv", lib().tria_quantize_kv(_dev_ptr(K), _dev_ptr(V), S, start,
                                                      ctypes.byref(cache.struct), _stream(stream)))


def tria_count_tiles(nb: int, hi: int, keep: int):
    out = np.zeros(3, np.int64)
    _check("tria_count_tiles", lib().tria_count_tiles(nb, hi, keep, out.ctypes.data_as(ctypes.c_void_p)))
    return tuple(int(v) for v in out)


def tria_prefill_load_plan(nb: int, T: int, hi: int, keep: int) -> np.ndarray:
    """The fused prefill's loads for one query head: int32 [n, 4] rows of
    (first query block of the tile, j0, j1, plane), in issue order."""
    n = ctypes.c_int64(0)
    _check("tria_prefill_load_plan", lib().tria_prefill_load_plan(nb, T, hi, keep, None, 0, ctypes.byref(n)))
    out = np.zeros((n.value, 4), np.int32)
    _check("tria_prefill_load_plan", lib().tria_prefill_load_plan(nb, T, hi, keep, out.ctypes.data_as(ctypes.c_void_p),
                                                                  n.value, ctypes.byref(n)))
    return out


def tria_decode_plan(B: int, Hq: int, Hkv: int, T: int, capacity: int, kv_len, hi, keep, num_sms: int) -> dict:
    """The decode's work plan: {'nkept', 'split_start', 'first_order', 'blocks_per_split', 'n_items'}."""
    groups = B * Hkv
    ss = np.zeros(groups + 1, np.int32)
    fo = np.zeros(groups, np.int32)
    nk = np.zeros(groups, np.int32)
    bps, n = ctypes.c_int32(0), ctypes.c_int32(0)
    P = ctypes.c_void_p
    kv_a, hi_a, keep_a = _host_i32(kv_len), _host_i32(hi), _host_i32(keep)
    _check("tria_decode_plan", lib().tria_decode_plan(
        B, Hq, Hkv, T, capacity, kv_a.ctypes.data_as(P), hi_a.ctypes.data_as(P), keep_a.ctypes.data_as(P), num_sms,
        ss.ctypes.data_as(P), fo.ctypes.data_as(P), nk.ctypes.data_as(P), ctypes.byref(bps), ctypes.byref(n)))
    return {"nkept": nk, "split_start": ss, "first_order": fo, "blocks_per_split": bps.value, "n_items": n.value}


def tria_prefill_workspace_bytes(B, Hq, Hkv, S, D, T) -> int:
    d = tria_dims(B, Hq, Hkv, S, D, T)
    return int(lib().tria_prefill_workspace_bytes(ctypes.byref(d)))


def tria_prefill(Q: torch.Tensor, cache: CompressedKVCache, hi, keep, workspace: torch.Tensor | None = None,
                 O: torch.Tensor | None = None, LSE: torch.Tensor | None = None, stream=None):
    """Fused prefill. Q bf16 [B,Hq,S,D]; the cache holds tokens [0,S). Returns (O bf16, LSE fp32)."""
    B, Hq, S, D = Q.shape
    dims = tria_dims(B, Hq, cache.Hkv, S, D, cache.T)
    need = int(lib().tria_prefill_workspace_bytes(ctypes.byref(dims)))
    if workspace is None:
        workspace = _aligned_empty(need, Q.device)
    if O is None:
        O = torch.empty_like(Q)
    if LSE is None:
        LSE = torch.empty((B, Hq, S), dtype=torch.float32, device=Q.device)
    hi_a, keep_a = _host_i32(hi), _host_i32(keep)
    _check("tria_prefill", lib().tria_prefill(
        _dev_ptr(Q), ctypes.byref(cache.struct), ctypes.byref(dims), hi_a.ctypes.data_as(ctypes.c_void_p),
        keep_a.ctypes.data_as(ctypes.c_void_p), _dev_ptr(O), _dev_ptr(LSE), _dev_ptr(workspace),
        workspace.numel(), _stream(stream)))
    return O, LSE


def tria_prefill_prepare(Q: torch.Tensor, cache: CompressedKVCache, workspace: torch.Tensor, stream=None):
    """First half of tria_prefill: Q codec and operand tiles into `workspace`."""
    B, Hq, S, D = Q.shape
    dims = tria_dims(B, Hq, cache.Hkv, S, D, cache.T)
    _check("tria_prefill_prepare", lib().tria_prefill_prepare(
        _dev_ptr(Q), ctypes.byref(cache.struct), ctypes.byref(dims), _dev_ptr(workspace), workspace.numel(),
        _stream(stream)))


def tria_prefill_attend(cache: CompressedKVCache, hi, keep, workspace: torch.Tensor, O: torch.Tensor,
                        LSE: torch.Tensor, stream=None):
    """Second half of tria_prefill: the fused kernel over a prepared workspace; writes O and LSE."""
    B, Hq, S, D = O.shape
    dims = tria_dims(B, Hq, cache.Hkv, S, D, cache.T)
    hi_a, keep_a = _host_i32(hi), _host_i32(keep)
    _check("tria_prefill_attend", lib().tria_prefill_attend(
        ctypes.byref(cache.struct), ctypes.byref(dims), hi_a.ctypes.data_as(ctypes.c_void_p),
        keep_a.ctypes.data_as(ctypes.c_void_p), _dev_ptr(O), _dev_ptr(LSE), _dev_ptr(workspace),
        workspace.numel(), _stream(stream)))
    return O, LSE


def tria_decode_workspace_bytes(B, Hq, Hkv, D, T, capacity) -> int:
    return int(lib().tria_decode_workspace_bytes(B, Hq, Hkv, D, T, capacity))


def tria_decode(q: torch.Tensor, cache: CompressedKVCache, kv_len, hi, keep, workspace: torch.Tensor | None = None,
                O: torch.Tensor | None = None, LSE: torch.Tensor | None = None, stream=None):
    """Split-KV decode. q bf16 [B,Hq,D]; kv_len host ints [B]. Returns (O bf16 [B,Hq,D], LSE fp32 [B,Hq])."""
    B, Hq, D = q.shape
    need = tria_decode_workspace_bytes(B, Hq, cache.Hkv, D, cache.T, cache.capacity)
    if workspace is None:
        workspace = _aligned_empty(need, q.device)
    if O is None:
        O = torch.empty_like(q)
    if LSE is None:
        LSE = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    kv, hi_a, keep_a = _host_i32(kv_len), _host_i32(hi), _host_i32(keep)
    _check("tria_decode", lib().tria_decode(
        _dev_ptr(q), ctypes.byref(cache.struct), kv.ctypes.data_as(ctypes.c_void_p), Hq,
        hi_a.ctypes.data_as(ctypes.c_void_p), keep_a.ctypes.data_as(ctypes.c_void_p), _dev_ptr(O), _dev_ptr(LSE),
        _dev_ptr(workspace), workspace.numel(), _stream(stream)))
    return O, LSE


def tria_workspace_status(workspace: torch.Tensor, stream=None) -> int:
    return int(lib().tria_workspace_status(_dev_ptr(workspace), _stream(stream)))


def tria_decode_static(q: torch.Tensor, cache: CompressedKVCache, kv_len, hi, keep, O: torch.Tensor | None = None,
                       LSE: torch.Tensor | None = None, stream=None):
    """tria_decode with the library's fixed device scratch instead of a caller workspace
    (for callers that cannot allocate device memory; see include/tria.h)."""
    L = lib()
    if not getattr(L.tria_decode_static, "_typed", False):
        P = ctypes.c_void_p
        L.tria_decode_static.argtypes = [P, ctypes.POINTER(tria_kv_cache), P, ctypes.c_int, P, P, P, P, P]
        L.tria_decode_static.restype = ctypes.c_int
        L.tria_decode_static._typed = True
    B, Hq, D = q.shape
    if O is None:
        O = torch.empty_like(q)
    if LSE is None:
        LSE = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    kv, hi_a, keep_a = _host_i32(kv_len), _host_i32(hi), _host_i32(keep)
    _check("tria_decode_static", L.tria_decode_static(
        _dev_ptr(q), ctypes.byref(cache.struct), kv.ctypes.data_as(ctypes.c_void_p), Hq,
        hi_a.ctypes.data_as(ctypes.c_void_p), keep_a.ctypes.data_as(ctypes.c_void_p), _dev_ptr(O), _dev_ptr(LSE),
        _stream(stream)))
    return O, LSE


def tria_decode_static_status(stream=None) -> int:
    """Error word of the fixed scratch tria_decode_static uses in the current context (synchronises)."""
    L = lib()
    if not getattr(L.tria_decode_static_status, "_typed", False):
        L.tria_decode_static_status.argtypes = [ctypes.c_void_p]
        L.tria_decode_static_status.restype = ctypes.c_int
        L.tria_decode_static_status._typed = True
    return int(L.tria_decode_static_status(_stream(stream)))


# ---------------------------------------------------------------- calibration

def _typed(name, argtypes, restype):
    f = getattr(lib(), name)
    if not getattr(f, "_typed", False):
        f.argtypes, f.restype, f._typed = argtypes, restype, True
    return f


def tria_calibration_costs(nb: int, T: int, D: int, cand_hi, cand_keep) -> np.ndarray:
    """Cost of each candidate (hi, keep) for one head over nb x nb causal blocks (int64 [C])."""
    P = ctypes.c_void_p
    f = _typed("tria_calibration_costs", [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int, P],
               ctypes.c_int)
    h, k = _host_i32(cand_hi), _host_i32(cand_keep)
    out = np.zeros(len(h), np.int64)
    _check("tria_calibration_costs", f(nb, T, D, h.ctypes.data_as(P), k.ctypes.data_as(P), len(h),
                                       out.ctypes.data_as(P)))
    return out


def tria_calibrate(Q: torch.Tensor, cache: CompressedKVCache, W_O: torch.Tensor, cand_hi, cand_keep,
                   workspace: torch.Tensor | None = None, stream=None):
    """Per-candidate, per-head error after the output projection and per-head energy
    (float64 numpy [C, Hq] and [Hq]); the normalised error is err / energy.sum()."""
    P, I = ctypes.c_void_p, ctypes.c_int
    B, Hq, S, D = Q.shape
    dims = tria_dims(B, Hq, cache.Hkv, S, D, cache.T)
    d_model = W_O.shape[1]
    need = _typed("tria_calibrate_workspace_bytes", [ctypes.POINTER(tria_dims), I], ctypes.c_size_t)(
        ctypes.byref(dims), d_model)
    if need == 0:
        raise TriaError("tria_calibrate_workspace_bytes", TRIA_ERR_INVALID_ARG)
    if workspace is None:
        workspace = _aligned_empty(need, Q.device)
    h, k = _host_i32(cand_hi), _host_i32(cand_keep)
    err = np.zeros((len(h), Hq), np.float64)
    energy = np.zeros(Hq, np.float64)
    f = _typed("tria_calibrate", [P, ctypes.POINTER(tria_kv_cache), ctypes.POINTER(tria_dims), P, I, P, P, I, P, P,
                                  P, ctypes.c_size_t, P], I)
    _check("tria_calibrate", f(_dev_ptr(Q), ctypes.byref(cache.struct), ctypes.byref(dims), _dev_ptr(W_O), d_model,
                               h.ctypes.data_as(P), k.ctypes.data_as(P), len(h), err.ctypes.data_as(P),
                               energy.ctypes.data_as(P), _dev_ptr(workspace), workspace.numel(), _stream(stream)))
    return err, energy


def tria_allocate(err, cost, budget: int) -> np.ndarray:
    """Greedy global allocation: err [C, H] float64, cost [C, H] int64 -> chosen candidate per head."""
    P = ctypes.c_void_p
    f = _typed("tria_allocate", [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int64, P], ctypes.c_int)
    e = np.ascontiguousarray(err, np.float64)
    c = np.ascontiguousarray(cost, np.int64)
    C, H = e.shape
    out = np.zeros(H, np.int32)
    _check("tria_allocate", f(e.ctypes.data_as(P), c.ctypes.data_as(P), C, H, int(budget), out.ctypes.data_as(P)))
    return out


def tria_prefill_gqa(enable: bool) -> bool:
    """Allow (True) or forbid (False) the GQA-shared fused prefill; returns the previous setting."""
    f = _typed("tria_prefill_gqa", [ctypes.c_int], ctypes.c_int)
    return bool(f(1 if enable else 0))


def _host_ptr(t: torch.Tensor) -> ctypes.c_void_p:
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous host tensor")
    return ctypes.c_void_p(t.data_ptr())


def tria_prefill_host_staging_bytes(B, Hq, Hkv, S, D, T) -> int:
    f = _typed("tria_prefill_host_staging_bytes", [ctypes.POINTER(tria_dims)], ctypes.c_size_t)
    return int(f(ctypes.byref(tria_dims(B, Hq, Hkv, S, D, T))))


def tria_prefill_host_workspace_bytes(B, Hq, Hkv, S, D, T) -> int:
    f = _typed("tria_prefill_host_workspace_bytes", [ctypes.POINTER(tria_dims)], ctypes.c_size_t)
    return int(f(ctypes.byref(tria_dims(B, Hq, Hkv, S, D, T))))


class HostPrefill:
    """Device buffers and the two copy streams of tria_prefill_host for one shape, kept
    across calls (the library itself allocates nothing)."""

    def __init__(self, B, Hq, Hkv, S, D, T, device="cuda", slots=2):
        """slots: staging slots (2 to 4); with more, the copies in run further ahead."""
        self.dims = tria_dims(B, Hq, Hkv, S, D, T)
        self.shape = (B, Hq, Hkv, S, D, T)
        per_slot = tria_prefill_host_staging_bytes(*self.shape) // 2
        self.staging = _aligned_empty(per_slot * max(2, min(4, int(slots))), device)
        self.workspace = _aligned_empty(tria_prefill_host_workspace_bytes(*self.shape), device)
        self.copy_in = torch.cuda.Stream(device=device)
        self.copy_out = torch.cuda.Stream(device=device)

    def __call__(self, hQ, hK, hV, cache: CompressedKVCache, hi, keep, hO, hLSE, stream=None):
        """Cache write and prefill from host tensors hQ/hK/hV into host hO/hLSE (queued on
        `stream`; synchronise it before reading hO)."""
        P = ctypes.c_void_p
        f = _typed("tria_prefill_host", [P, P, P, ctypes.POINTER(tria_kv_cache), ctypes.POINTER(tria_dims), P, P, P,
                                         P, P, ctypes.c_size_t, P, ctypes.c_size_t, P, P, P], ctypes.c_int)
        hi_a, keep_a = _host_i32(hi), _host_i32(keep)
        _check("tria_prefill_host", f(
            _host_ptr(hQ), _host_ptr(hK), _host_ptr(hV), ctypes.byref(cache.struct), ctypes.byref(self.dims),
            hi_a.ctypes.data_as(P), keep_a.ctypes.data_as(P), _host_ptr(hO), _host_ptr(hLSE),
            _dev_ptr(self.staging), self.staging.numel(), _dev_ptr(self.workspace), self.workspace.numel(),
            _stream(stream), _stream(self.copy_in), _stream(self.copy_out)))
        return hO, hLSE
