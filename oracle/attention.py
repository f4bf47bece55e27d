"""ctypes wrapper over the C oracle (``attention_oracle.c``).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .routing import tile_offsets

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention_oracle.c")
_LIB = os.path.join(_HERE, "_attention_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle next to this file (plain gcc -O2, OpenMP, IEEE)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_attention_rows.restype = I
        lib.oracle_attention_rows.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I,
                                              I, I, P, ctypes.c_double, P, ctypes.c_int64, P, P]
        lib.oracle_attention_rows_fmt.restype = I
        lib.oracle_attention_rows_fmt.argtypes = lib.oracle_attention_rows.argtypes + [I]
        lib.oracle_int_scores.restype = I
        lib.oracle_int_scores.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P, P]
        lib.oracle_half_to_double.restype = ctypes.c_double
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        _lib = lib
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def all_rows(lengths, hq):
    """(sequence, head, row) triples of every output row."""
    out = []
    for s, L in enumerate(lengths):
        for h in range(hq):
            for i in range(L):
                out.append((s, h, i))
    return np.array(out, dtype=np.int64).reshape(-1, 3)


def attention_rows(q, k, v, q8, q_scale, k8, k_scale, masks, g, lengths, causal,
                   kv_map=None, scale=None, rows=None, low="int8"):
    """fp64 output rows and LSE of tile-routed attention.

    q [T,hq,d], k/v [T,hk,d] float16; q8/k8 the low-precision codes in the
    same layouts (int8, or e4m3 bytes when low == "fp8");
    q_scale [hq, total_qtiles], k_scale [hk, total_ktiles] float32;
    masks [total_qtiles, hk] uint64; g one grouping factor per sequence;
    rows: [n, 3] (sequence, head, row) or None for every row.
    Returns (O [n, d] float64, lse [n] float64)."""
    lib = _load()
    T, hq, d = q.shape
    hk = k.shape[1]
    lengths = [int(x) for x in lengths]
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    cu_q, cu_k = tile_offsets(lengths)
    if kv_map is None:
        kv_map = np.arange(hq) // (hq // hk)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if rows is None:
        rows = all_rows(lengths, hq)
    rows = _c(rows, np.int64).reshape(-1, 3)
    n = rows.shape[0]
    out = np.zeros((n, d), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    if low not in ("int8", "fp8"):
        raise ValueError(low)
    args = [_c(q, np.float16).view(np.uint16), _c(k, np.float16).view(np.uint16),
            _c(v, np.float16).view(np.uint16), _c(q8, q8.dtype).view(np.int8),
            _c(q_scale, np.float32), _c(k8, k8.dtype).view(np.int8), _c(k_scale, np.float32),
            _c(masks, np.uint64),
            _c(g, np.int32), cu, cu_q, cu_k]
    keep = args + [_c(kv_map, np.int32), rows, out, lse]
    rc = lib.oracle_attention_rows_fmt(
        *[a.ctypes.data for a in args], len(lengths), int(cu_q[-1]), int(cu_k[-1]), hq, hk, d,
        int(bool(causal)), keep[12].ctypes.data, float(scale), rows.ctypes.data, n,
        out.ctypes.data, lse.ctypes.data, int(low == "fp8"))
    if rc != 0:
        raise RuntimeError("oracle_attention_rows failed: %d" % rc)
    return out, lse


def int_scores(q8, k8, masks, g, lengths, s, h, hq, hk, causal, kv_map=None):
    """Exact int64 INT8-path scores of (sequence s, head h): [L, L] with -2**62 on
    entries that are illegal or FP16-routed."""
    lib = _load()
    d = q8.shape[2]
    lengths = [int(x) for x in lengths]
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    cu_q, _ = tile_offsets(lengths)
    if kv_map is None:
        kv_map = np.arange(hq) // (hq // hk)
    L = lengths[s]
    a = np.full((L, L), -(2 ** 62), dtype=np.int64)
    arrs = [_c(q8, np.int8), _c(k8, np.int8), _c(masks, np.uint64), _c(g, np.int32), cu, cu_q]
    km = _c(kv_map, np.int32)
    rc = lib.oracle_int_scores(*[x.ctypes.data for x in arrs], s, h, hq, hk, d,
                               int(bool(causal)), km.ctypes.data, a.ctypes.data)
    if rc != 0:
        raise RuntimeError("oracle_int_scores failed: %d" % rc)
    return a


def half_to_double(bits: int) -> float:
    return float(_load().oracle_half_to_double(bits))
