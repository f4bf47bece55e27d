"""Oracle of the decode step with the INT8 K cache (one new query token per
sequence).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages name decode with the INT8 KV cache as the step after prefill ("TileMix:
Tile-Centric Mixed-Precision Attention for LLM Inference Acceleration",
agihunt.info summary; "Precision Has a Map: TileMix Routes INT8 Inside Dense
Attention", cognaptus.com, last section) but give no algorithm for it.  The
reading here is the prefill method applied to one row:

- sequence s holds L = seq_len[s] cached tokens at cache rows
  [seq_start[s], seq_start[s] + L); the new token is at position t = L - 1 and
  attends to positions 0..t;
- its routing word is the one of its query-tile row t // 128 (row
  qtile_start[s] + t // 128 of ``masks``);
- the K cache is quantised in 64-key blocks from the sequence's first token,
  the last block over its valid rows (the prefill blocks, ``quantize_k``);
- the query row is quantised as a block of its own (earlier queries are not
  cached), with the same absmax / 127 rules.

The attention itself is the pinned row oracle (``attention_rows``) run on the
sequence with the new query placed at row t; nothing is recomputed here.
"""
from __future__ import annotations

import numpy as np

from .attention import attention_rows
from .quant import quantize_blocks, quantize_k
from .routing import BLOCK_M


def quantize_rows(x16):
    """Each row of x16 [n, H, d] float16 as a block of its own:
    (codes int8 [n, H, d], scales float32 [n, H])."""
    n = x16.shape[0]
    codes, scales = quantize_blocks(x16, [1] * n, 1)
    return codes, np.ascontiguousarray(scales.T)


def decode_rows(q_new, k_cache, v_cache, seq_start, seq_len, masks, qtile_start, g,
                kv_map=None, scale=None):
    """O [nseq, hq, d] float64 of the decode step and the LSE [nseq, hq]."""
    q_new = np.asarray(q_new, dtype=np.float16)
    nseq, hq, d = q_new.shape
    hk = k_cache.shape[1]
    q8_new, qs_new = quantize_rows(q_new)
    out = np.zeros((nseq, hq, d))
    lse = np.zeros((nseq, hq))
    for s in range(nseq):
        a, L = int(seq_start[s]), int(seq_len[s])
        t = L - 1
        k_s = np.ascontiguousarray(k_cache[a:a + L])
        v_s = np.ascontiguousarray(v_cache[a:a + L])
        k8_s, ks_s = quantize_k(k_s, [L])
        nqt = (L + BLOCK_M - 1) // BLOCK_M
        q_s = np.zeros((L, hq, d), dtype=np.float16)
        q_s[t] = q_new[s]
        q8_s = np.zeros((L, hq, d), dtype=np.int8)
        q8_s[t] = q8_new[s]
        qs_s = np.zeros((hq, nqt), dtype=np.float32)
        qs_s[:, t // BLOCK_M] = qs_new[s]
        m_s = np.ascontiguousarray(masks[int(qtile_start[s]):int(qtile_start[s]) + nqt])
        rows = np.array([(0, h, t) for h in range(hq)], dtype=np.int64)
        o, l = attention_rows(q_s, k_s, v_s, q8_s, qs_s, k8_s, ks_s, m_s,
                              np.array([int(g[s])], dtype=np.int32), [L], True,
                              kv_map=kv_map, scale=scale, rows=rows)
        out[s] = o
        lse[s] = l
    return out, lse
