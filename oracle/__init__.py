"""CPU oracle for Condensate attention (test infrastructure).

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of
`bench.py` may import this package.  The product path (the CUDA library and
its binding) never imports it, and it imports nothing from the product.

The arithmetic lives in `condensate_oracle.c` (double precision, one row at a
time, standard library sort), built by `build()` with gcc into
`liboracle.so` next to this file.  This module only marshals arrays.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "condensate_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

DIAG_NAMES = [
    "m", "size", "anchor_mass", "window_mass", "topk_mass", "excluded_mass",
    "cos", "err_l2", "vmax_l2", "tau_min", "best_unsel", "gap", "bound",
    "win_lo", "lse",
]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP over independent rows)."""
    if force or not os.path.exists(_LIB) or \
            os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load(path):
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    L.oracle_rows.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, P, P,
                              P, P, ctypes.c_int64, ctypes.c_int, P, P, P,
                              P, P, ctypes.c_int]
    L.oracle_rows.restype = ctypes.c_int
    L.oracle_diag_count.restype = ctypes.c_int
    L.oracle_max_threads.restype = ctypes.c_int
    assert L.oracle_diag_count() == len(DIAG_NAMES)
    return L


@contextlib.contextmanager
def using_library(path: str):
    """Temporarily route every oracle call through another build of the C
    source (the tests use it to check that planted mistakes are caught)."""
    global _lib
    saved = _lib
    _lib = _load(path)
    try:
        yield
    finally:
        _lib = saved


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = _load(_LIB)
    return _lib




def max_threads() -> int:
    return int(lib().oracle_max_threads())


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def rows(Q, K, V, k: int, q_off, kv_off, pos, win, C_max: int,
         with_full: bool = True, threads: int = 0) -> dict:
    """Run the oracle on explicit rows (see `oracle_rows` in the C source)."""
    Q = np.ascontiguousarray(Q, dtype=np.float32)
    K = np.ascontiguousarray(K, dtype=np.float32)
    V = np.ascontiguousarray(V, dtype=np.float32)
    d = K.shape[-1]
    q_off = np.ascontiguousarray(q_off, dtype=np.int64)
    kv_off = np.ascontiguousarray(kv_off, dtype=np.int64)
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    win = np.ascontiguousarray(win, dtype=np.int32)
    R = len(pos)
    C = np.empty((R, C_max), dtype=np.int32)
    cnt = np.empty(R, dtype=np.int32)
    o = np.empty((R, d), dtype=np.float64)
    of = np.empty((R, d), dtype=np.float64) if with_full else None
    dg = np.empty((R, len(DIAG_NAMES)), dtype=np.float64)
    rc = lib().oracle_rows(_ptr(Q), _ptr(K), _ptr(V), d, int(k), _ptr(q_off),
                           _ptr(kv_off), _ptr(pos), _ptr(win), R, int(C_max),
                           _ptr(C), _ptr(cnt), _ptr(o), _ptr(of), _ptr(dg),
                           int(threads))
    if rc != 0:
        raise ValueError("a row's Condensate Set does not fit C_max")
    out = {"idx": C, "count": cnt, "o": o, "diag": dg}
    if with_full:
        out["o_full"] = of
    for z, name in enumerate(DIAG_NAMES):
        out[name] = dg[:, z]
    return out


def prefill(Q, K, V, W: int, k: int, W_i=None, sel=None, C_max=None,
            with_full: bool = True, threads: int = 0) -> dict:
    """Oracle for causal prefill.

    Q: [B, Hq, n, d]; K, V: [B, Hkv, n, d] (float32 holding the exact input
    values).  W_i: optional int [B, n] per-query windows.  sel: optional
    int array [R, 3] of (b, h, i) rows; default is every row.
    Results are in row order of `sel` (or b, h, i order).
    """
    B, Hq, n, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    if sel is None:
        b, h, i = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(n),
                              indexing="ij")
        sel = np.stack([b.ravel(), h.ravel(), i.ravel()], axis=1)
    sel = np.asarray(sel, dtype=np.int64).reshape(-1, 3)
    b, h, i = sel[:, 0], sel[:, 1], sel[:, 2]
    q_off = ((b * Hq + h) * n + i) * d
    kv_off = (b * Hkv + h // G) * n * d
    if W_i is not None:
        win = np.asarray(W_i, dtype=np.int32).reshape(B, n)[b, i]
        wmax = int(np.max(W_i))
    else:
        win = np.full(len(i), W, dtype=np.int32)
        wmax = W
    if C_max is None:
        C_max = 1 + wmax + k
    out = rows(Q, K, V, k, q_off, kv_off, i, win, C_max, with_full, threads)
    out["sel"] = sel
    return out


def decode(q, K, V, W: int, k: int, W_i=None, C_max=None,
           with_full: bool = True, threads: int = 0) -> dict:
    """Oracle for decode: q [B, Hq, d] at position L-1 over K, V [B, Hkv, L, d].

    Results are in (b, h) order: idx [B*Hq, C_max], o [B*Hq, d], ...
    """
    B, Hq, d = q.shape
    Hkv, L = K.shape[1], K.shape[2]
    G = Hq // Hkv
    b, h = np.meshgrid(np.arange(B), np.arange(Hq), indexing="ij")
    b, h = b.ravel(), h.ravel()
    q_off = (b * Hq + h) * d
    kv_off = (b * Hkv + h // G) * L * d
    pos = np.full(len(b), L - 1, dtype=np.int64)
    if W_i is not None:
        win = np.asarray(W_i, dtype=np.int32).reshape(B)[b]
        wmax = int(np.max(W_i))
    else:
        win = np.full(len(b), W, dtype=np.int32)
        wmax = W
    if C_max is None:
        C_max = 1 + wmax + k
    return rows(q, K, V, k, q_off, kv_off, pos, win, C_max, with_full, threads)
