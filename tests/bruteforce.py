"""Brute-force fp64 references used to pin the oracle (tests only).

Written as whole-matrix numpy, independently of the oracle's row loop: scores
as matrix products, masking by boolean matrices, softmax along rows.
"""
import numpy as np

BM, BN = 128, 64


def _offsets(lengths):
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lengths)
    return cu


def _legal(L, causal):
    if causal:
        return np.tril(np.ones((L, L), dtype=bool))
    return np.ones((L, L), dtype=bool)


def _softmax_out(S, legal, V):
    S = np.where(legal, S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    P = np.where(legal, np.exp(S - m), 0.0)
    l = P.sum(axis=1, keepdims=True)
    return (P @ V) / l, (m + np.log(l))[:, 0]


def naive_attention(q, k, v, lengths, causal, kv_map=None, scale=None):
    """Softmax attention in fp64: O [T, hq, d], lse [hq, T]."""
    T, hq, d = q.shape
    hk = k.shape[1]
    if kv_map is None:
        kv_map = np.arange(hq) // (hq // hk)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    cu = _offsets(lengths)
    O = np.zeros((T, hq, d))
    lse = np.zeros((hq, T))
    for s, L in enumerate(lengths):
        a, b = cu[s], cu[s + 1]
        for h in range(hq):
            Q = q[a:b, h].astype(np.float64)
            K = k[a:b, kv_map[h]].astype(np.float64)
            V = v[a:b, kv_map[h]].astype(np.float64)
            O[a:b, h], lse[h, a:b] = _softmax_out((Q @ K.T) * scale, _legal(L, causal), V)
    return O, lse


def _block_index(L, block):
    return np.arange(L) // block


def int8_keys_of_word(word, L, g):
    """Boolean [L] of keys whose group bit is set: expand groups into keys."""
    out = np.zeros(L, dtype=bool)
    for b in range(64):
        if (int(word) >> b) & 1:
            lo = b * g * BN
            hi = min((b + 1) * g * BN, L)
            if lo < hi:
                out[lo:hi] = True
    return out


def routed_attention(q, k, v, q8, qs, k8, ks, masks, g, lengths, causal, kv_map=None,
                     scale=None):
    """Brute force with per-key routing: for every query-tile row the INT8 key
    set is expanded from the word; INT8 scores are exact integer matrix
    products times the two block scales, FP16 scores are fp64 matrix products."""
    T, hq, d = q.shape
    hk = k.shape[1]
    if kv_map is None:
        kv_map = np.arange(hq) // (hq // hk)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    cu = _offsets(lengths)
    O = np.zeros((T, hq, d))
    lse = np.zeros((hq, T))
    qt_base = 0
    kt_base = 0
    for s, L in enumerate(lengths):
        a, b = cu[s], cu[s + 1]
        tm = (L + BM - 1) // BM
        tn = (L + BN - 1) // BN
        for h in range(hq):
            kv = kv_map[h]
            Q = q[a:b, h].astype(np.float64)
            K = k[a:b, kv].astype(np.float64)
            V = v[a:b, kv].astype(np.float64)
            A = q8[a:b, h].astype(np.int64) @ k8[a:b, kv].astype(np.int64).T
            sq = qs[h, qt_base + _block_index(L, BM)].astype(np.float64)
            sk = ks[kv, kt_base + _block_index(L, BN)].astype(np.float64)
            S_int = A.astype(np.float64) * sq[:, None] * sk[None, :] * scale
            S_fp = (Q @ K.T) * scale
            use_int = np.zeros((L, L), dtype=bool)
            for r in range(tm):
                word = masks[qt_base + r, kv]
                use_int[r * BM:(r + 1) * BM] = int8_keys_of_word(word, L, int(g[s]))[None, :]
            S = np.where(use_int, S_int, S_fp)
            O[a:b, h], lse[h, a:b] = _softmax_out(S, _legal(L, causal), V)
        qt_base += tm
        kt_base += tn
    return O, lse
