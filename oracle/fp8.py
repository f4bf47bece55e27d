"""Oracle for the FP8 (e4m3) low path: the codec and the block quantiser.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages name FP8 (and INT4) as an open alternative to the INT8 low path,
with scale handling to be redone ("TileMix: Tile-Centric Mixed-Precision
Attention for LLM Inference Acceleration", agihunt.info summary, limitations
paragraph; "Precision Has a Map", cognaptus.com, "The A100 result should not
be exported unchanged").  Reading used here: the INT8 path with its codes
replaced by FP8 e4m3 values, everything else unchanged -- Q blocks of 128 x d
and K blocks of 64 x d, symmetric, s = fp32(absmax / 448) (448 is the largest
finite e4m3 value), code = e4m3(fp32(x / s)) rounded to nearest, ties to even,
saturating to +-448; a zero block has s = 0 and codes 0; the score of an FP8
tile is (sum over channels of decoded q code x decoded k code) x s_q x s_k /
sqrt(d).

e4m3 (the OCP 8-bit format with 4 exponent bits, bias 7, 3 mantissa bits, no
infinities): sign s, exponent e, mantissa m; e = 0 gives m / 8 x 2^-6, the
other exponents (1 + m / 8) x 2^(e - 7), except e = 15, m = 7, which is NaN.
"""
from __future__ import annotations

import math

import numpy as np

from .routing import BLOCK_M, BLOCK_N

E4M3_MAX = 448.0


def e4m3_decode(code: int) -> float:
    s, e, m = (code >> 7) & 1, (code >> 3) & 15, code & 7
    if e == 15 and m == 7:
        return math.nan
    v = math.ldexp(m, -9) if e == 0 else math.ldexp(8 + m, e - 10)
    return -v if s else v


DECODE = np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)
_POS = DECODE[:0x7F]  # codes 0x00..0x7E: 0 .. 448, ascending


def e4m3_encode(y) -> np.ndarray:
    """float32 array -> uint8 codes (round to nearest, ties to even code,
    saturate to +-448; the sign of zero is kept)."""
    y = np.asarray(y, dtype=np.float32)
    a = np.minimum(np.abs(y).astype(np.float64), E4M3_MAX)
    hi = np.searchsorted(_POS, a, side="left")          # first value >= a
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    dlo = a - _POS[lo]
    dhi = _POS[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    mag = np.where(a == _POS[hi], hi, np.where(pick_hi, hi, lo)).astype(np.uint8)
    return np.where(np.signbit(y), mag | np.uint8(0x80), mag).astype(np.uint8)


def quantize_blocks_fp8(x16: np.ndarray, lengths, block: int):
    """x16 [T, H, d] float16 -> (codes uint8 [T, H, d], scales float32 [H, total_blocks])."""
    if x16.dtype != np.float16 or x16.ndim != 3:
        raise ValueError("expected float16 [T, H, d]")
    T, H, d = x16.shape
    nblk = [(L + block - 1) // block for L in lengths]
    codes = np.zeros((T, H, d), dtype=np.uint8)
    scales = np.zeros((H, sum(nblk)), dtype=np.float32)
    t0 = col = 0
    with np.errstate(invalid="ignore", divide="ignore", over="ignore"):
        for L, nb in zip(lengths, nblk):
            for b in range(nb):
                r0 = t0 + b * block
                r1 = min(t0 + L, r0 + block)
                blk = x16[r0:r1].astype(np.float32)
                a = np.abs(blk).max(axis=(0, 2))
                s = (a / np.float32(E4M3_MAX)).astype(np.float32)      # IEEE fp32 division
                y = (blk / s[None, :, None]).astype(np.float32)          # IEEE fp32 division
                c = e4m3_encode(np.nan_to_num(y, nan=0.0))
                c = np.where((a == 0)[None, :, None], np.uint8(0), c)
                codes[r0:r1] = c
                scales[:, col + b] = s
            t0 += L
            col += nb
    return codes, scales


def quantize_q_fp8(q16, lengths):
    return quantize_blocks_fp8(q16, lengths, BLOCK_M)


def quantize_k_fp8(k16, lengths):
    return quantize_blocks_fp8(k16, lengths, BLOCK_N)


__all__ = ["DECODE", "E4M3_MAX", "e4m3_decode", "e4m3_encode", "quantize_blocks_fp8",
           "quantize_k_fp8", "quantize_q_fp8"]
