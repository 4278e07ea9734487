"""CPU oracle for block-sparse attention driven by a per-input mask.

TEST INFRASTRUCTURE ONLY: only tests/, the package smoke check and bench.py's
cpu_baseline / reference arm may import this module.  The product path (the
CUDA library and its Python binding) never imports, loads or calls it, and the
two share no code; they meet only through the seeded generators in workloads/.

Thin numpy wrapper over oracle.c (plain fp64 C, built with gcc by
``build_oracle``).  Every function states the passage it follows in oracle.c.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

PIN, SPARSE, DROP = 0, 1, 2
PAT_RADIAL, PAT_WINDOW_GLOBAL, PAT_DILATED, PAT_RANDOM = 0, 1, 2, 3


def build_oracle(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain gcc, fp64, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build_oracle())
        P = ctypes.c_void_p
        i, f, dbl = ctypes.c_int, ctypes.c_float, ctypes.c_double
        _lib.oracle_layout.argtypes = [P, i, i, i, P]
        _lib.oracle_layout.restype = i
        _lib.oracle_pool.argtypes = [P, i, i, i, i, P]
        _lib.oracle_scores.argtypes = [P, P, i, i, i, i, i, P]
        _lib.oracle_budget.argtypes = [f, i]
        _lib.oracle_budget.restype = i
        _lib.oracle_select.argtypes = [P, P, i, i, i, f, P, i, P, P]
        _lib.oracle_pattern.argtypes = [P, i, i, i, i, i, i, f, i, i, P, i, P, P, ctypes.c_uint64]
        _lib.oracle_pattern.restype = i
        _lib.oracle_attention.argtypes = [P, P, P, i, i, i, i, i, i, P, P, i, P, P, dbl, P, ctypes.c_int64, P]
        _lib.oracle_density.argtypes = [P, i, i, i, P, P, P]
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def layout(segments: Sequence[Tuple[int, int, int]], N: int, block: int = 64) -> np.ndarray:
    """Per-block class (PIN / SPARSE / DROP) from token segments."""
    lib = _load()
    segs = np.ascontiguousarray(np.array(segments, dtype=np.int32).reshape(-1, 3))
    cls = np.zeros(N // block if block > 0 else 0, dtype=np.uint8)
    rc = lib.oracle_layout(_ptr(segs), len(segments), N, block, _ptr(cls))
    if rc != 0:
        raise ValueError("segments do not tile [0, N) in order")
    return cls


def pool(X: np.ndarray, block: int = 64) -> np.ndarray:
    """Block means in fp64; X is uint16 bf16 bits [..., N, d]."""
    lib = _load()
    X = np.ascontiguousarray(X, dtype=np.uint16)
    N, d = X.shape[-2], X.shape[-1]
    BH = int(np.prod(X.shape[:-2])) if X.ndim > 2 else 1
    out = np.zeros((BH, N // block, d), dtype=np.float64)
    lib.oracle_pool(_ptr(X), BH, N, d, block, _ptr(out))
    return out.reshape(X.shape[:-2] + (N // block, d))


def _kv_heads(H: int, q_size: int, k_size: int) -> int:
    """Key/value heads when a query tensor of q_size elements has H heads and
    the key tensor k_size elements (same batch, length and head size)."""
    if k_size * H % q_size != 0:
        raise ValueError("key tensor does not hold a whole number of heads")
    Hkv = k_size * H // q_size
    if Hkv < 1 or H % Hkv != 0:
        raise ValueError("query heads %d are not a multiple of key/value heads %d" % (H, Hkv))
    return Hkv


def scores(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """s[i][j] = qbar_i . kbar_j in fp64 (no scale, no softmax), on query heads.

    qbar [..., H, nB, d]; kbar [..., Hkv, nB, d] with H a multiple of Hkv
    (grouped heads: query head h scores against key head h // (H / Hkv))."""
    lib = _load()
    qbar = np.ascontiguousarray(qbar, dtype=np.float64)
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    nB, d = qbar.shape[-2], qbar.shape[-1]
    BH = int(np.prod(qbar.shape[:-2])) if qbar.ndim > 2 else 1
    H = qbar.shape[-3] if qbar.ndim > 2 else 1
    Hkv = _kv_heads(H, qbar.size, kbar.size)
    out = np.zeros((BH, nB, nB), dtype=np.float64)
    lib.oracle_scores(_ptr(qbar), _ptr(kbar), BH, H, Hkv, nB, d, _ptr(out))
    return out.reshape(qbar.shape[:-2] + (nB, nB))


def budget(density: float, C: int) -> int:
    return int(_load().oracle_budget(ctypes.c_float(density), C))


def cap_of(cls: np.ndarray) -> int:
    return int(np.sum(cls != DROP))


def select(sc: np.ndarray, cls: np.ndarray, H: int, density: float,
           head_mask: Optional[np.ndarray] = None, cap: Optional[int] = None):
    """Rank-select block lists from scores [BH, nB, nB] (fp64 or widened fp32)."""
    lib = _load()
    nB = cls.shape[0]
    sc = np.ascontiguousarray(sc, dtype=np.float64).reshape(-1, nB, nB)
    BH = sc.shape[0]
    cap = cap_of(cls) if cap is None else cap
    cls = np.ascontiguousarray(cls, dtype=np.uint8)
    hm = None if head_mask is None else np.ascontiguousarray(head_mask, dtype=np.uint8)
    idx = np.full((BH, nB, max(cap, 1)), -1, dtype=np.int32)
    counts = np.zeros((BH, nB), dtype=np.int32)
    lib.oracle_select(_ptr(sc), _ptr(cls), BH, H, nB, ctypes.c_float(density), _ptr(hm), max(cap, 1),
                      _ptr(idx), _ptr(counts))
    return idx, counts


def pattern(cls: np.ndarray, kind: int, BH: int, H: int, window: int = 0, n_global: int = 0,
            dilation: int = 1, density: float = 1.0, head_mask: Optional[np.ndarray] = None,
            cap: Optional[int] = None, block: int = 64, seed: int = 0):
    """Radial / window+global / dilated / random block lists at the layout's pins and drops
    (seed: the random pattern's SplitMix64 seed)."""
    lib = _load()
    nB = cls.shape[0]
    cap = cap_of(cls) if cap is None else cap
    cls = np.ascontiguousarray(cls, dtype=np.uint8)
    hm = None if head_mask is None else np.ascontiguousarray(head_mask, dtype=np.uint8)
    idx = np.full((BH, nB, max(cap, 1)), -1, dtype=np.int32)
    counts = np.zeros((BH, nB), dtype=np.int32)
    rc = lib.oracle_pattern(_ptr(cls), nB, block, kind, window, n_global, dilation, ctypes.c_float(density),
                            BH, H, _ptr(hm), max(cap, 1), _ptr(idx), _ptr(counts), ctypes.c_uint64(seed))
    if rc != 0:
        raise ValueError("bad pattern")
    return idx, counts


def attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, H: int, idx: np.ndarray, counts: np.ndarray,
              head_mask: Optional[np.ndarray] = None, scale: Optional[float] = None,
              rows: Optional[np.ndarray] = None, block: int = 64,
              key_mask: Optional[np.ndarray] = None) -> np.ndarray:
    """fp64 attention over the kept tiles; Q uint16 bf16 bits [B, H, N, d],
    K and V [B, Hkv, N, d] with H a multiple of Hkv (query head h reads
    key/value head h // (H / Hkv)).

    rows: flat row ids (b*H + h)*N + n to compute (None = all); returns
    [len(rows), d] (or [B, H, N, d] when rows is None).
    key_mask: optional token-level mask over keys, [B, N] (nonzero = may be
    attended), applied inside the kept tiles; a row left with no key gives 0."""
    lib = _load()
    Q = np.ascontiguousarray(Q, dtype=np.uint16)
    K = np.ascontiguousarray(K, dtype=np.uint16)
    V = np.ascontiguousarray(V, dtype=np.uint16)
    N, d = Q.shape[-2], Q.shape[-1]
    BH = int(np.prod(Q.shape[:-2]))
    Hkv = _kv_heads(H, Q.size, K.size)
    if V.size != K.size:
        raise ValueError("K and V differ in size")
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    cap = idx.shape[-1]
    hm = None if head_mask is None else np.ascontiguousarray(head_mask, dtype=np.uint8)
    sc = 1.0 / np.sqrt(d) if scale is None else float(scale)
    km = None
    if key_mask is not None:
        km = np.ascontiguousarray(np.asarray(key_mask) != 0, dtype=np.uint8)
        if km.size != (BH // H) * N:
            raise ValueError("key_mask must be [B, N]")
    if rows is None:
        out = np.zeros((BH * N, d), dtype=np.float64)
        lib.oracle_attention(_ptr(Q), _ptr(K), _ptr(V), BH, H, Hkv, N, d, block, _ptr(idx), _ptr(counts), cap,
                             _ptr(hm), _ptr(km), sc, None, BH * N, _ptr(out))
        return out.reshape(Q.shape)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.zeros((rows.shape[0], d), dtype=np.float64)
    lib.oracle_attention(_ptr(Q), _ptr(K), _ptr(V), BH, H, Hkv, N, d, block, _ptr(idx), _ptr(counts), cap,
                         _ptr(hm), _ptr(km), sc, _ptr(rows), rows.shape[0], _ptr(out))
    return out


def density(counts: np.ndarray, H: int, nB: int, head_mask: Optional[np.ndarray] = None):
    lib = _load()
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    BH = counts.size // nB
    hm = None if head_mask is None else np.ascontiguousarray(head_mask, dtype=np.uint8)
    a = ctypes.c_double()
    b = ctypes.c_double()
    lib.oracle_density(_ptr(counts), BH, H, nB, _ptr(hm), ctypes.byref(a), ctypes.byref(b))
    return a.value, b.value
