"""CPU oracle for block-sparse mixed-precision causal attention (TriAttention).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers. The GPU library never
imports this package, and this package never imports the GPU library.

The arithmetic lives in ``tria_oracle.cpp`` (plain C++17, fp32 codec, exact
integer dot products, float64 softmax and P.V); this module only builds it with
g++ and marshals numpy arrays through ctypes. bf16 tensors travel as their raw
16-bit patterns (numpy ``uint16``).

What each entry point follows is stated in the C++ header comment (the rit.work
TriAttention page, sections "Какие связи можно не считать, а какие нельзя
удалять" and "Как калибровка распределяет вычисления между головами"; the GQA
head mapping from llmis.ru chapter 3.5, section 4).

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
(closed-form tile counts, hand-worked codec and attention fixtures under
``tests/golden/``, library SDPA special cases, invariants). No function is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "tria_oracle.cpp"
_LIB = _HERE / "liboracle.so"

FLAG_BYPASS_QUANT = 1
NONE, SKIP, INT4, INT8 = -1, 0, 4, 8

_lib = None


def build(force: bool = False) -> Path:
    """Compile the oracle shared library with g++ (no FMA contraction)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.tmp{os.getpid()}")
        cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-pthread", str(_SRC), "-o", str(tmp)]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(str(_LIB))
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int, ctypes.c_int64
        lib.oracle_quantize_rows.argtypes = [P, i64, i32, P, P, P, P]
        lib.oracle_quantize_rows.restype = None
        lib.oracle_pack_int4.argtypes = [P, i64, P]
        lib.oracle_pack_int4.restype = None
        lib.oracle_action.argtypes = [i32, i32, i32, i32]
        lib.oracle_action.restype = i32
        lib.oracle_action_map.argtypes = [i32, i32, i32, P]
        lib.oracle_action_map.restype = None
        lib.oracle_action_counts.argtypes = [i32, i32, i32, P]
        lib.oracle_action_counts.restype = None
        lib.oracle_prefill_rows.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, P, P, i32,
                                            P, i64, P, P, i32]
        lib.oracle_prefill_rows.restype = i32
        lib.oracle_dense_attention.argtypes = [P, P, P, i32, i32, i32, i32, i32, P, P, i32]
        lib.oracle_dense_attention.restype = i32
        lib.oracle_decode.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, P, P, P, i32, i32,
                                      P, P, i32]
        lib.oracle_decode.restype = i32
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    """Accept a numpy uint16 array of bf16 bits or a torch bf16 tensor."""
    if isinstance(a, np.ndarray):
        assert a.dtype == np.uint16
        return np.ascontiguousarray(a)
    import torch  # local: only to accept torch tensors
    assert a.dtype == torch.bfloat16
    return np.ascontiguousarray(a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _threads(n: int | None) -> int:
    return int(n) if n else (os.cpu_count() or 1)


def quantize_rows(x, D: int):
    """Both planes of every D-wide row: (c8, s8, c4, s4), codes unpacked int8."""
    x = _u16(x).reshape(-1)
    rows = x.size // D
    c8 = np.empty((rows, D), np.int8)
    c4 = np.empty((rows, D), np.int8)
    s8 = np.empty(rows, np.float32)
    s4 = np.empty(rows, np.float32)
    _load().oracle_quantize_rows(_ptr(x), rows, D, _ptr(c8), _ptr(s8), _ptr(c4), _ptr(s4))
    return c8, s8, c4, s4


def pack_int4(c4: np.ndarray) -> np.ndarray:
    """Two int4 codes per byte: even element low nibble, odd element high nibble."""
    c4 = np.ascontiguousarray(c4, dtype=np.int8)
    out = np.empty(c4.shape[:-1] + (c4.shape[-1] // 2,), np.uint8)
    _load().oracle_pack_int4(_ptr(c4), c4.size, _ptr(out))
    return out


def action(i: int, j: int, hi: int, keep: int) -> int:
    return int(_load().oracle_action(i, j, hi, keep))


def action_map(nb: int, hi: int, keep: int) -> np.ndarray:
    out = np.empty((nb, nb), np.int32)
    _load().oracle_action_map(nb, hi, keep, _ptr(out))
    return out


def action_counts(nb: int, hi: int, keep: int):
    """(int8, int4, skip) tile counts over the nb(nb+1)/2 causal tiles, by enumeration."""
    out = np.zeros(3, np.int64)
    _load().oracle_action_counts(nb, hi, keep, _ptr(out))
    return tuple(int(v) for v in out)


def prefill_rows(Q, K, V, T: int, hi, keep, rows=None, flags: int = 0, nthreads=None):
    """Attention rows of a prefill.

    Q [B,Hq,S,D], K/V [B,Hkv,S,D] (bf16 bits or torch bf16); hi/keep per query
    head. ``rows`` are flat ids (b*Hq + hq)*S + t (default: every row).
    Returns (O [n, D] float64, LSE [n] float64).
    """
    Q, K, V = _u16(Q), _u16(K), _u16(V)
    B, Hq, S, D = Q.shape
    Hkv = K.shape[1]
    assert K.shape == (B, Hkv, S, D) and V.shape == K.shape
    hi = np.ascontiguousarray(hi, np.int32)
    keep = np.ascontiguousarray(keep, np.int32)
    assert hi.shape == (Hq,) and keep.shape == (Hq,)
    if rows is None:
        rows = np.arange(B * Hq * S, dtype=np.int64)
    rows = np.ascontiguousarray(rows, np.int64)
    O = np.empty((rows.size, D), np.float64)
    LSE = np.empty(rows.size, np.float64)
    rc = _load().oracle_prefill_rows(_ptr(Q), _ptr(K), _ptr(V), B, Hq, Hkv, S, D, T,
                                     _ptr(hi), _ptr(keep), flags, _ptr(rows), rows.size,
                                     _ptr(O), _ptr(LSE), _threads(nthreads))
    if rc:
        raise ValueError("oracle_prefill_rows: invalid dimensions")
    return O, LSE


def dense_attention(Q, K, V, nthreads=None):
    """Textbook dense causal softmax attention in float64 (GQA), no codes or tiles."""
    Q, K, V = _u16(Q), _u16(K), _u16(V)
    B, Hq, S, D = Q.shape
    Hkv = K.shape[1]
    O = np.empty((B, Hq, S, D), np.float64)
    LSE = np.empty((B, Hq, S), np.float64)
    rc = _load().oracle_dense_attention(_ptr(Q), _ptr(K), _ptr(V), B, Hq, Hkv, S, D,
                                        _ptr(O), _ptr(LSE), _threads(nthreads))
    if rc:
        raise ValueError("oracle_dense_attention: invalid dimensions")
    return O, LSE


def decode(q, K, V, T: int, kv_len, hi, keep, flags: int = 0, nsplit: int = 0, nthreads=None):
    """One query token per sequence over its K/V (capacity S, kv_len[b] valid).

    q [B,Hq,D]; K/V [B,Hkv,S,D]. nsplit >= 1 reduces contiguous runs of kept key
    blocks separately and merges them by log-sum-exp. Returns (O [B,Hq,D], LSE [B,Hq]).
    """
    q, K, V = _u16(q), _u16(K), _u16(V)
    B, Hq, D = q.shape
    Hkv, S = K.shape[1], K.shape[2]
    kv_len = np.ascontiguousarray(kv_len, np.int32)
    hi = np.ascontiguousarray(hi, np.int32)
    keep = np.ascontiguousarray(keep, np.int32)
    O = np.empty((B, Hq, D), np.float64)
    LSE = np.empty((B, Hq), np.float64)
    rc = _load().oracle_decode(_ptr(q), _ptr(K), _ptr(V), B, Hq, Hkv, S, D, T, _ptr(kv_len),
                               _ptr(hi), _ptr(keep), flags, nsplit, _ptr(O), _ptr(LSE),
                               _threads(nthreads))
    if rc:
        raise ValueError("oracle_decode: invalid arguments")
    return O, LSE
