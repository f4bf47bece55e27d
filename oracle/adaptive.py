"""Oracle for content-aware (adaptive) routing through the routing-word ABI.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Shares no code with
the library's routing kernels.

The pages say the mask interface can carry adaptive, content-aware policies
and evaluate none ("TileMix: Tile-Centric Mixed-Precision Attention for LLM
Inference Acceleration", agihunt.info summary, limitations paragraph;
"Precision Has a Map: TileMix Routes INT8 Inside Dense Attention",
cognaptus.com, "Placement can matter more than the nominal percentage").  The
policy here is this library's reading, the plainest content signal the method
already has at tile granularity:

pooled-score routing.  For query-tile row r = (s, qt) and KV head kv:
  qbar      = mean of q over the row's valid query rows and the KV head's
              query heads,
  kbar_kt   = mean of k over key tile kt's valid keys (KV head kv),
  score_kt  = qbar . kbar_kt for every legal key tile kt of the row,
  score_b   = max of score_kt over the legal tiles of group b,
  INT8      = the row's k_r lowest-scoring legal groups (ties: the lower group
              first), k_r from the static templates' proportional quota, so a
              sequence gets the same INT8 group count as under any template.
All arithmetic is fp32 in a fixed order, which is part of the definition (the
device computes the same words bit for bit):
  a mean adds its items (q: head-major, heads in ascending index, then rows
  ascending; k: rows ascending) into 8 interleaved partial sums (item m into
  sum m mod 8, in ascending m), adds the partial sums in order 0..7 and
  divides by the item count; no items gives a zero mean;
  a dot adds fl(qbar_c * kbar_c) over channels c ascending, rounding each
  product and each sum to fp32 (no fused multiply-add).
"""
from __future__ import annotations

import numpy as np

from .routing import (BLOCK_M, BLOCK_N, MAX_GROUPS, _quota, int8_target, last_legal_tile,
                      legal_groups, n_ktiles, n_qtiles)

F32 = np.float32


def interleaved_mean(items):
    """items: float32 [..., M, d] -> float32 [..., d] in the fixed order."""
    items = np.asarray(items, dtype=F32)
    M = items.shape[-2]
    shape = items.shape[:-2] + (8, items.shape[-1])
    acc = np.zeros(shape, dtype=F32)
    for m in range(M):
        acc[..., m % 8, :] = acc[..., m % 8, :] + items[..., m, :]
    tot = acc[..., 0, :].copy()
    for j in range(1, 8):
        tot = tot + acc[..., j, :]
    if M == 0:
        return tot
    return tot / F32(M)


def ordered_dot(qbar, kbar):
    """qbar float32 [d], kbar float32 [n, d] -> float32 [n]."""
    qbar = np.asarray(qbar, dtype=F32)
    kbar = np.asarray(kbar, dtype=F32)
    s = np.zeros(kbar.shape[0], dtype=F32)
    for c in range(kbar.shape[1]):
        s = s + qbar[c] * kbar[:, c]
    return s


def heads_of(kv, hq, hk, kv_map):
    if kv_map is None:
        G = hq // hk
        return list(range(kv * G, kv * G + G))
    return [h for h in range(hq) if int(kv_map[h]) == kv]


def pooled_means(q16, k16, lengths, hq, hk, kv_map=None):
    """qbar [total_qtiles, hk, d] and kbar [total_ktiles, hk, d] (float32)."""
    q = np.asarray(q16).astype(F32)
    k = np.asarray(k16).astype(F32)
    d = q.shape[-1]
    qb, kb = [], []
    start = 0
    for L in lengths:
        for qt in range(n_qtiles(L)):
            r0, r1 = start + qt * BLOCK_M, start + min((qt + 1) * BLOCK_M, L)
            row = []
            for kv in range(hk):
                hs = heads_of(kv, hq, hk, kv_map)
                items = q[r0:r1][:, hs, :].transpose(1, 0, 2).reshape(-1, d)  # head-major
                row.append(interleaved_mean(items))
            qb.append(row)
        for kt in range(n_ktiles(L)):
            r0, r1 = start + kt * BLOCK_N, start + min((kt + 1) * BLOCK_N, L)
            kb.append([interleaved_mean(k[r0:r1, kv, :]) for kv in range(hk)])
        start += L
    return (np.array(qb, dtype=F32).reshape(-1, hk, d),
            np.array(kb, dtype=F32).reshape(-1, hk, d))


def choose_int8(scores, k):
    """Indices of the k lowest scores, ties to the lower index."""
    order = sorted(range(len(scores)), key=lambda b: (float(scores[b]), b))
    return set(order[:k])


def route_pooled(q16, k16, lengths, hq, hk, g, causal, percent, kv_map=None):
    """Routing words [total_qtiles, hk] (uint64) of the pooled-score policy."""
    if not 0 <= percent <= 100:
        raise ValueError(percent)
    qbar, kbar = pooled_means(q16, k16, lengths, hq, hk, kv_map)
    words = []
    cq = ck = 0
    for s, L in enumerate(lengths):
        gs = int(g[s])
        n = [legal_groups(qt, L, gs, causal) for qt in range(n_qtiles(L))]
        if n and max(n) > MAX_GROUPS:
            raise ValueError("more than 64 routing groups in a row")
        quota = _quota(n, percent)
        for qt in range(n_qtiles(L)):
            lt = last_legal_tile(qt, L, causal)
            row = []
            for kv in range(hk):
                sc_t = ordered_dot(qbar[cq + qt, kv], kbar[ck:ck + lt + 1, kv])
                sc_b = [max(float(x) for x in sc_t[b * gs:min((b + 1) * gs, lt + 1)])
                        for b in range(n[qt])]
                w = 0
                for b in choose_int8(sc_b, quota[qt]):
                    w |= 1 << b
                row.append(w)
            words.append(row)
        cq += n_qtiles(L)
        ck += n_ktiles(L)
    if not words:
        return np.zeros((0, hk), dtype=np.uint64)
    return np.array(words, dtype=np.uint64).reshape(-1, hk)


__all__ = ["choose_int8", "heads_of", "interleaved_mean", "ordered_dot", "pooled_means",
           "route_pooled", "int8_target"]
