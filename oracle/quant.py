"""Oracle block quantiser for the INT8 score path.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

"TileMix: Tile-Centric Mixed-Precision Attention for LLM Inference
Acceleration" (agihunt.info summary, method paragraphs): only Q and K are
quantised, Q in 128 x d blocks and K in 64 x d blocks, symmetric, absmax / 127.

Readings: a block is the rows [b*block, min((b+1)*block, L)) of one sequence
and one head (it never crosses a sequence; a short tail block uses its valid
rows only).  a = max |x| over the block (x is the fp16 value, exact in fp32);
s = fp32(a / 127) with IEEE division; code = clamp(round_half_even(fp32(x / s)),
-127, 127); a block with a == 0 has s = 0 and all codes 0.

INT4 codes (the 4-bit format the same pages name as an open alternative to
INT8: agihunt, limitations paragraph; 59188saintaubert.com explainer, closing
section): the same blocks and rule with 7 in place of 127, s = fp32(a / 7) and
codes in [-7, 7] (kept one per byte).
"""
from __future__ import annotations

import numpy as np

from .routing import BLOCK_M, BLOCK_N


def quantize_blocks(x16: np.ndarray, lengths, block: int, qmax: int = 127):
    """x16 [T, H, d] float16 -> (codes int8 [T, H, d], scales float32 [H, total_blocks]);
    qmax = 127 for INT8 codes, 7 for INT4 codes."""
    if x16.dtype != np.float16 or x16.ndim != 3:
        raise ValueError("expected float16 [T, H, d]")
    T, H, d = x16.shape
    nblk = [(L + block - 1) // block for L in lengths]
    total = sum(nblk)
    codes = np.zeros((T, H, d), dtype=np.int8)
    scales = np.zeros((H, total), dtype=np.float32)
    t0 = 0
    col = 0
    with np.errstate(invalid="ignore", divide="ignore", over="ignore"):
        for L, nb in zip(lengths, nblk):
            for b in range(nb):
                r0 = t0 + b * block
                r1 = min(t0 + L, r0 + block)
                blk = x16[r0:r1].astype(np.float32)             # exact
                a = np.abs(blk).max(axis=(0, 2))                  # [H]
                s = (a / np.float32(qmax)).astype(np.float32)     # IEEE fp32 division
                q = blk / s[None, :, None]                        # IEEE fp32 division
                c = np.clip(np.rint(q), -qmax, qmax)              # half-to-even
                c = np.where((a == 0)[None, :, None], 0, c)
                c = np.nan_to_num(c, nan=0.0)
                codes[r0:r1] = c.astype(np.int8)
                scales[:, col + b] = s
            t0 += L
            col += nb
    return codes, scales


def quantize_q(q16, lengths):
    return quantize_blocks(q16, lengths, BLOCK_M)


def quantize_k(k16, lengths):
    return quantize_blocks(k16, lengths, BLOCK_N)


def quantize_q_int4(q16, lengths):
    return quantize_blocks(q16, lengths, BLOCK_M, qmax=7)


def quantize_k_int4(k16, lengths):
    return quantize_blocks(k16, lengths, BLOCK_N, qmax=7)
