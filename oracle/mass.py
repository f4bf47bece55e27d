"""Oracle for the importance-mass exposure probe.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages report, for static SpTrans routing at 25% INT8 coverage, that only
about 8.5% of the selected high-importance attention mass lands on INT8-routed
regions ("Precision Has a Map: TileMix Routes INT8 Inside Dense Attention",
cognaptus.com, last section; "TileMix: Tile-Centric Mixed-Precision Attention
for LLM Inference Acceleration", agihunt.info summary, appendix sentence of
the results paragraph; the 59188saintaubert.com explainer, 实验说了什么).  They
do not say how interactions are selected.  Reading used here:

  P_i       = softmax over row i's legal keys of the full-precision scores
              q_i . k_j / sqrt(d) (fp16 inputs, exact products);
  H_i       = the row's high-importance keys: P_ij >= 2^-delta * max_j P_ij,
              i.e. score_ij >= max_j score_ij - delta * ln 2 (delta = 4: keys
              within a factor 16 of the row's most attended key);
  m8_i      = sum of P_ij over INT8-routed legal keys (the row's INT8 mass);
  h_i       = sum of P_ij over H_i;     h8_i = over H_i and INT8-routed.
A batch's exposure is sum_i h8_i / sum_i h_i (every row's P sums to one, so
rows weigh equally); its INT8 mass share is the mean of m8_i.  INT8-routed
means the row's routing word has the bit of the key's group set (the words
of the attention path, bit (kt / g) of word (query-tile row, KV head)).

Everything here is fp64.  ``probe_rows`` also returns, per row, the bounds of
h and h8 over every choice of membership for keys whose score is within
``band`` of the threshold, for comparing with an fp32 computation.
"""
from __future__ import annotations

import math

import numpy as np

from .routing import BLOCK_M, BLOCK_N, n_qtiles

LN2 = math.log(2.0)


def probe_rows(q16, k16, masks, g, lengths, causal, delta=4.0, kv_map=None, band=0.0):
    """Per (head, token) arrays [hq, T]: m8, h, h8, and h/h8 lower and upper
    bounds over the memberships of keys within ``band`` (natural-log units) of
    the selection threshold."""
    q = np.asarray(q16).astype(np.float64)
    k = np.asarray(k16).astype(np.float64)
    T, hq, d = q.shape
    hk = k.shape[1]
    masks = np.asarray(masks, dtype=np.uint64)
    out = {key: np.zeros((hq, T)) for key in ("m8", "h", "h8", "h_lo", "h_hi", "h8_lo", "h8_hi")}
    start = 0
    cq = 0
    for s, L in enumerate(lengths):
        if L == 0:  # no rows, nothing to write
            continue
        gs = int(g[s])
        for h in range(hq):
            kv = h // (hq // hk) if kv_map is None else int(kv_map[h])
            Q = q[start:start + L, h]
            K = k[start:start + L, kv]
            S = (Q @ K.T) / math.sqrt(d)
            i = np.arange(L)[:, None]
            j = np.arange(L)[None, :]
            legal = (j <= i) if causal else np.ones((L, L), dtype=bool)
            S = np.where(legal, S, -np.inf)
            m = S.max(axis=1, keepdims=True)
            P = np.exp(S - m)
            P = P / P.sum(axis=1, keepdims=True)
            words = masks[cq + np.arange(L) // BLOCK_M, kv].astype(np.uint64)
            grp = (np.arange(L) // BLOCK_N) // gs
            bit = ((words[:, None] >> grp[None, :].astype(np.uint64)) & np.uint64(1)).astype(bool)
            int8 = bit & legal
            thr = m - delta * LN2
            H = legal & (S >= thr)
            amb = legal & (np.abs(S - thr) <= band)
            col = start + np.arange(L)
            out["m8"][h, col] = (P * int8).sum(axis=1)
            out["h"][h, col] = (P * H).sum(axis=1)
            out["h8"][h, col] = (P * (H & int8)).sum(axis=1)
            out["h_lo"][h, col] = (P * (H & ~amb)).sum(axis=1)
            out["h_hi"][h, col] = (P * (H | amb)).sum(axis=1)
            out["h8_lo"][h, col] = (P * (H & ~amb & int8)).sum(axis=1)
            out["h8_hi"][h, col] = (P * ((H | amb) & int8)).sum(axis=1)
        start += L
        cq += n_qtiles(L)
    return out


def exposure(h, h8):
    """Batch exposure: the INT8 share of the selected high-importance mass."""
    h = np.asarray(h, dtype=np.float64)
    return float(np.asarray(h8, dtype=np.float64).sum() / h.sum()) if h.sum() > 0 else 0.0


__all__ = ["exposure", "probe_rows"]
