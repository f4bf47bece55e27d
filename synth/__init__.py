"""Seeded synthetic inputs for tile-routed mixed-precision prefill attention.

This module only draws numbers.  It holds none of the attention method's
arithmetic (no quantisation, no routing, no softmax), so that both the CUDA
path and the CPU oracle can be fed the same tensors.

Generator
---------
splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014): the state advances by the golden-ratio constant
GAMMA and each output is the state passed through the finaliser ``mix64``.
Because the k-th output (k >= 1) of a stream started at state ``s`` is
``mix64(s + k*GAMMA)``, a stream is a counter-based generator and is
parallel over ``k`` (``_synth.c``).

Streams: stream ``id`` of seed ``seed`` starts at state ``draw(seed, id + 1)``,
i.e. at the (id+1)-th output of the master stream of ``seed``.

Normals: Box-Muller in fp64.  Draw pair (2m+1, 2m+2) of a stream gives
u1 = (top53(a) + 1) * 2^-53 in (0, 1] and u2 = top53(b) * 2^-53 in [0, 1);
r = sqrt(-2 ln u1); element 2m = r cos(2 pi u2), element 2m+1 = r sin(2 pi u2).
fp16 tensors are these fp64 values rounded to nearest-even by numpy.

Tensor stream ids: Q = 1, K = 2, V = 3, outlier channel picks = 4,
low-rank basis W = 5, low-rank query weights = 6, low-rank key weights = 7.
Variable sequence lengths use stream 0.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB

STREAM_LENGTHS = 0
STREAM_Q = 1
STREAM_K = 2
STREAM_V = 3
STREAM_OUTLIER = 4
STREAM_LOWRANK_W = 5
STREAM_LOWRANK_ZQ = 6
STREAM_LOWRANK_ZK = 7

_CHUNK = 1 << 24  # elements per block (bounds host memory)
_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "_synth.c")
_LIB = os.path.join(_HERE, "_synth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C draw kernel next to this file (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.synth_draw.restype = ctypes.c_uint64
        lib.synth_draw.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_normals.restype = None
        lib.synth_normals.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_void_p]
        _lib = lib
    return _lib


def mix64_int(z: int) -> int:
    """splitmix64 output finaliser on a Python int."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * _M1) & MASK64
    z = ((z ^ (z >> 27)) * _M2) & MASK64
    return z ^ (z >> 31)


def draw(seed: int, k: int) -> int:
    """k-th output (k >= 1) of the splitmix64 stream started at state ``seed``."""
    return mix64_int(seed + k * GAMMA)


def substream(seed: int, stream: int) -> int:
    """Start state of stream ``stream`` of ``seed``."""
    return draw(seed, stream + 1)


def normals(seed: int, stream: int, n: int, start: int = 0) -> np.ndarray:
    """Elements start .. start+n-1 of the N(0,1) sequence of (seed, stream), fp64."""
    out = np.empty(n, dtype=np.float64)
    if n:
        _load().synth_normals(substream(seed, stream), start, n, out.ctypes.data)
    return out


def fp16_normal(seed: int, stream: int, shape) -> np.ndarray:
    """fp16 tensor of N(0,1) values (fp64 Box-Muller rounded to nearest-even)."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float16)
    for pos in range(0, n, _CHUNK):
        m = min(_CHUNK, n - pos)
        out[pos:pos + m] = normals(seed, stream, m, start=pos).astype(np.float16)
    return out.reshape(shape)


def partial_fisher_yates(seed_state: int, n: int, count: int, start: int = 0):
    """First ``count`` entries of a partial Fisher-Yates shuffle of range(n).

    Draw number start+i+1 of the stream picks j = i + (draw mod (n - i)).
    Returns (picks, draws_used).  The modulo bias is accepted.
    """
    a = list(range(n))
    for i in range(count):
        r = draw(seed_state, start + i + 1)
        j = i + r % (n - i)
        a[i], a[j] = a[j], a[i]
    return a[:count], count


def varlen_lengths(seed: int, nseq: int, lo: int = 1024, hi: int = 16384,
                   multiple: int = 64) -> list:
    """Lengths uniform in [lo, hi] (modulo draw), rounded to the nearest multiple
    of ``multiple`` with ties rounding up."""
    s = substream(seed, STREAM_LENGTHS)
    span = hi - lo + 1
    out = []
    for i in range(nseq):
        L = lo + draw(s, i + 1) % span
        L = ((L + multiple // 2) // multiple) * multiple
        out.append(int(L))
    return out


def cu_seqlens_of(lengths) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


def default_kv_map(hq: int, hk: int) -> np.ndarray:
    return (np.arange(hq) // (hq // hk)).astype(np.int32)


def outlier_channels(seed: int, hk: int, d: int, per_head: int = 4) -> np.ndarray:
    """Distinct channel picks per KV head, drawn consecutively from stream 4."""
    s = substream(seed, STREAM_OUTLIER)
    out = np.zeros((hk, per_head), dtype=np.int64)
    used = 0
    for kv in range(hk):
        picks, n = partial_fisher_yates(s, d, per_head, start=used)
        used += n
        out[kv] = picks
    return out


def make_qkv(seed: int, total_tokens: int, hq: int, hk: int, d: int,
             outliers: int = 0, outlier_scale: float = 8.0, lowrank: int = 0):
    """Q [T,hq,d], K [T,hk,d], V [T,hk,d] as fp16.

    outliers > 0: that many channels per KV head (shared with the KV head's
    query heads) are multiplied by ``outlier_scale`` in Q and K before rounding.
    lowrank > 0: Q += zq @ W[kv], K += zk @ W[kv] with W ~ N(0,1) [hk, r, d] and
    zq, zk ~ N(0, 1/r) per token and head, added before rounding.  V is plain.
    """
    T = total_tokens
    kvmap = default_kv_map(hq, hk)
    v = fp16_normal(seed, STREAM_V, (T, hk, d))
    if outliers == 0 and lowrank == 0:
        q = fp16_normal(seed, STREAM_Q, (T, hq, d))
        k = fp16_normal(seed, STREAM_K, (T, hk, d))
        return q, k, v
    scale_q = np.ones((hq, d))
    scale_k = np.ones((hk, d))
    if outliers:
        ch = outlier_channels(seed, hk, d, outliers)
        for kv in range(hk):
            scale_k[kv, ch[kv]] = outlier_scale
        for h in range(hq):
            scale_q[h, ch[kvmap[h]]] = outlier_scale
    W = None
    if lowrank:
        W = normals(seed, STREAM_LOWRANK_W, hk * lowrank * d).reshape(hk, lowrank, d)
    q = np.empty((T, hq, d), dtype=np.float16)
    k = np.empty((T, hk, d), dtype=np.float16)
    rows = max(1, _CHUNK // (hq * d))
    zs = 1.0 / np.sqrt(lowrank) if lowrank else 0.0
    for t0 in range(0, T, rows):
        t1 = min(T, t0 + rows)
        n = t1 - t0
        xq = normals(seed, STREAM_Q, n * hq * d, start=t0 * hq * d).reshape(n, hq, d)
        xk = normals(seed, STREAM_K, n * hk * d, start=t0 * hk * d).reshape(n, hk, d)
        xq *= scale_q[None]
        xk *= scale_k[None]
        if lowrank:
            zq = normals(seed, STREAM_LOWRANK_ZQ, n * hq * lowrank,
                         start=t0 * hq * lowrank).reshape(n, hq, lowrank) * zs
            zk = normals(seed, STREAM_LOWRANK_ZK, n * hk * lowrank,
                         start=t0 * hk * lowrank).reshape(n, hk, lowrank) * zs
            xq += np.matmul(zq.transpose(1, 0, 2), W[kvmap]).transpose(1, 0, 2)
            xk += np.matmul(zk.transpose(1, 0, 2), W).transpose(1, 0, 2)
        q[t0:t1] = xq.astype(np.float16)
        k[t0:t1] = xk.astype(np.float16)
    return q, k, v


# ---------------------------------------------------------------------------
# The five workloads (shapes, distributions and routing choices).
# ---------------------------------------------------------------------------

WORKLOADS = {
    "tiny_l256": dict(lengths=[256], hq=1, hk=1, d=64, causal=True, g="1",
                      template="band", percent=50, outliers=0, lowrank=0,
                      routing_seed=0),
    "llama3b_4k_b8": dict(lengths=[4096] * 8, hq=24, hk=8, d=128, causal=True, g="1",
                          template="sptrans", percent=75, outliers=4, lowrank=0,
                          routing_seed=0),
    "sweep_8k_b8": dict(lengths=[8192] * 8, hq=24, hk=8, d=128, causal=True, g="2",
                        template="band", percent=25, outliers=0, lowrank=0,
                        routing_seed=0),
    "varlen_qwen7b": dict(lengths="varlen", hq=28, hk=4, d=128, causal=True, g="auto",
                          template="bigbird", percent=50, outliers=0, lowrank=0,
                          routing_seed=0),
    "long_64k": dict(lengths=[65536], hq=32, hk=8, d=128, causal=True, g="16",
                     template="row_random", percent=25, outliers=0, lowrank=16,
                     routing_seed=0),
}


def workload_lengths(name: str) -> list:
    w = WORKLOADS[name]
    if w["lengths"] == "varlen":
        return varlen_lengths(7, 12)
    return list(w["lengths"])
