"""Oracle routing: legality counts and the six static routing templates.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Written from the
pages' description and the readings below; shares no code with the C++
routing builder in the library.

Geometry ("TileMix: Tile-Centric Mixed-Precision Attention for LLM Inference
Acceleration", agihunt.info summary, method paragraphs): the score matrix is cut
into 128 x 64 (BLOCK_M x BLOCK_N) tiles; along the key axis g adjacent tiles
form one routing group with one bit, 1 = INT8 and 0 = FP16; one 64-bit word per
(KV head, query-tile row); g keeps a row at <= 64 bits.  Coverage is the share
of *legal* tile groups routed INT8, not a FLOP share; the same template is
reused across KV heads.

Readings (the pages name the templates with one phrase each):
  bit b (LSB = 0) <-> group b = key tiles [b*g, (b+1)*g).
  legal groups of row qt: n = last_legal_tile // g + 1, where the last legal
    key tile is min((qt+1)*128 - 1, L - 1) // 64 when causal, else Tn - 1.
  INT8 target per sequence: K = floor((p * N + 50) / 100) with N = sum of n.
  Band (keeps the diagonal local): largest width w with sum_r min(w, n_r) <= F
    (F = N - K FP16 groups); the rightmost min(w, n_r) groups of each row are
    FP16, and the F - sum left over go one each, in ascending row order, to the
    rows with n_r > w as one more group left of the band.
  Global (keeps designated positions): Band mirrored, leftmost groups.
  Proportional quota (Aligned-Sparse, Row-Random, BigBird, SpTrans): row r
    gets k_r = floor(p * n_r / 100) INT8 groups; the K - sum k_r left over go
    one each to the rows with the largest remainder p * n_r mod 100 (ties to the
    lower row); f_r = n_r - k_r FP16 groups.
  Aligned-Sparse (right-aligned extension): FP16 = the rightmost f_r groups.
  Row-Random (each row keeps random FP16): FP16 = the first f_r picks of a
    partial Fisher-Yates shuffle of 0..n_r-1 driven by the row's stream.
  BigBird (union of Band, Global and Row-Random): the leftmost ceil(f/3); then
    the rightmost ceil((f - ceil(f/3)) / 2); the rest random from the unchosen
    middle (partial Fisher-Yates over the ascending middle list, row stream).
  SpTrans (stride plus tail): FP16 priority = the last two legal groups, then
    groups with b mod 8 == 7, then 6, ..., 0, each class right to left; the
    first f_r distinct groups of that order are FP16.
  Row stream of row qt: splitmix64 state draw(seed, qt + 1); the shuffle step
    i takes j = i + (draw(state, i + 1) mod (len - i)).
"""
from __future__ import annotations

import math

import numpy as np

BLOCK_M = 128
BLOCK_N = 64
MAX_GROUPS = 64
TEMPLATES = ("band", "global", "row_random", "aligned_sparse", "bigbird", "sptrans")

_MASK64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15


def _mix64(z: int) -> int:
    # splitmix64 finaliser (Steele, Lea & Flood 2014).
    z &= _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def _draw(state: int, k: int) -> int:
    return _mix64(state + k * _GAMMA)


def n_qtiles(L: int) -> int:
    return (L + BLOCK_M - 1) // BLOCK_M


def n_ktiles(L: int) -> int:
    return (L + BLOCK_N - 1) // BLOCK_N


def last_legal_tile(qt: int, L: int, causal: bool) -> int:
    if causal:
        return min((qt + 1) * BLOCK_M - 1, L - 1) // BLOCK_N
    return n_ktiles(L) - 1


def legal_groups(qt: int, L: int, g: int, causal: bool) -> int:
    return last_legal_tile(qt, L, causal) // g + 1


def auto_g(L: int) -> int:
    return max(1, math.ceil(n_ktiles(L) / MAX_GROUPS))


def tile_offsets(lengths):
    cu_q = [0]
    cu_k = [0]
    for L in lengths:
        cu_q.append(cu_q[-1] + n_qtiles(L))
        cu_k.append(cu_k[-1] + n_ktiles(L))
    return np.array(cu_q, dtype=np.int32), np.array(cu_k, dtype=np.int32)


def int8_target(percent: int, N: int) -> int:
    return (percent * N + 50) // 100


def _fixed_width(n, F):
    """Per-row FP16 counts of the fixed-width rule (Band / Global)."""
    w = 0
    while n and w < max(n) and sum(min(w + 1, x) for x in n) <= F:
        w += 1
    left = F - sum(min(w, x) for x in n)
    widths = []
    for x in n:
        c = min(w, x)
        if x > w and left > 0:
            c += 1
            left -= 1
        widths.append(c)
    assert left == 0
    return widths


def _quota(n, percent):
    """Per-row INT8 counts of the proportional rule."""
    k = [percent * x // 100 for x in n]
    rem = [percent * x % 100 for x in n]
    left = int8_target(percent, sum(n)) - sum(k)
    order = sorted(range(len(n)), key=lambda r: (-rem[r], r))
    for r in order[:left]:
        k[r] += 1
    return k


def _shuffle_prefix(items, count, state):
    a = list(items)
    for i in range(count):
        j = i + _draw(state, i + 1) % (len(a) - i)
        a[i], a[j] = a[j], a[i]
    return a[:count]


def fp16_groups(template: str, percent: int, seed: int, n):
    """FP16 group sets of each q-tile row of one sequence (n = legal groups)."""
    if template not in TEMPLATES:
        raise ValueError(template)
    if not 0 <= percent <= 100:
        raise ValueError(percent)
    N = sum(n)
    K = int8_target(percent, N)
    if template in ("band", "global"):
        widths = _fixed_width(n, N - K)
        if template == "band":
            return [set(range(x - c, x)) for x, c in zip(n, widths)]
        return [set(range(0, c)) for c, x in zip(widths, n)]
    k = _quota(n, percent)
    out = []
    for qt, (x, kr) in enumerate(zip(n, k)):
        f = x - kr
        state = _draw(seed, qt + 1)
        if template == "aligned_sparse":
            out.append(set(range(x - f, x)))
        elif template == "row_random":
            out.append(set(_shuffle_prefix(range(x), f, state)))
        elif template == "bigbird":
            a = -(-f // 3)
            b = -(-(f - a) // 2)
            chosen = set(range(0, a)) | set(range(x - b, x))
            middle = [y for y in range(a, x - b)]
            chosen |= set(_shuffle_prefix(middle, f - a - b, state))
            out.append(chosen)
        else:  # sptrans
            order = []
            for y in (x - 1, x - 2):
                if y >= 0 and y not in order:
                    order.append(y)
            for res in range(7, -1, -1):
                for y in range(x - 1, -1, -1):
                    if y % 8 == res and y not in order:
                        order.append(y)
            out.append(set(order[:f]))
    return out


def build_routing(template: str, percent: int, seed: int, lengths, hk: int, g, causal: bool):
    """Routing words [total_qtiles, hk] (uint64) plus per-sequence legal and INT8
    group counts.  ``g`` is one grouping factor per sequence."""
    words = []
    legal = []
    int8 = []
    for s, L in enumerate(lengths):
        gs = int(g[s])
        n = [legal_groups(qt, L, gs, causal) for qt in range(n_qtiles(L))]
        if n and max(n) > MAX_GROUPS:
            raise ValueError("more than 64 routing groups in a row")
        fp = fp16_groups(template, percent, seed, n)
        cnt = 0
        for x, f in zip(n, fp):
            w = 0
            for b in range(x):
                if b not in f:
                    w |= 1 << b
                    cnt += 1
            words.append([w] * hk)
        legal.append(sum(n))
        int8.append(cnt)
    arr = np.array(words, dtype=np.uint64).reshape(-1, hk) if words else np.zeros((0, hk), np.uint64)
    return arr, np.array(legal, dtype=np.int64), np.array(int8, dtype=np.int64)
