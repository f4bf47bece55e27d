"""Pins of the CPU oracle against brute force, closed forms, hand-derived
words and the invariants the TileMix pages state.  CPU only."""
import math
import os

import numpy as np
import pytest

import oracle
import synth
from tests import bruteforce as bf

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [x.strip() for x in f if x.strip() and not x.startswith("#")]


def _inputs(lengths, hq, hk, d, seed=0):
    T = sum(lengths)
    q, k, v = synth.make_qkv(seed, T, hq, hk, d)
    q8, qs = oracle.quantize_q(q, lengths)
    k8, ks = oracle.quantize_k(k, lengths)
    return q, k, v, q8, qs, k8, ks


def _words(lengths, hk, value):
    tm = sum(oracle.n_qtiles(L) for L in lengths)
    return np.full((tm, hk), value, dtype=np.uint64)


def _run(inp, masks, g, lengths, causal, kv_map=None, scale=None):
    q, k, v, q8, qs, k8, ks = inp
    O, lse = oracle.attention_rows(q, k, v, q8, qs, k8, ks, masks, g, lengths, causal,
                                   kv_map=kv_map, scale=scale)
    T, hq, d = q.shape
    rows = oracle.all_rows(lengths, hq)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    full = np.zeros((T, hq, d))
    full_lse = np.zeros((hq, T))
    t = cu[rows[:, 0]] + rows[:, 2]
    full[t, rows[:, 1]] = O
    full_lse[rows[:, 1], t] = lse
    return full, full_lse


# --------------------------------------------------------------------------
# generator pins
# --------------------------------------------------------------------------

def test_splitmix64_reference_outputs():
    want = [int(x, 16) for x in _golden_lines("splitmix64_state0.txt")]
    assert [synth.draw(0, k) for k in (1, 2, 3)] == want
    assert [oracle.routing._draw(0, k) for k in (1, 2, 3)] == want
    lib = synth._load()
    assert [lib.synth_draw(0, k) for k in (1, 2, 3)] == want


def test_box_muller_moments():
    x = synth.normals(123, 1, 1 << 20)
    assert abs(x.mean()) < 5e-3
    assert abs(x.std() - 1.0) < 5e-3
    # fourth moment of N(0,1) is 3
    assert abs((x ** 4).mean() - 3.0) < 0.05
    # any window equals the same slice of a longer draw
    assert np.array_equal(synth.normals(123, 1, 77, start=1001), x[1001:1078])


def test_half_to_double_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


# --------------------------------------------------------------------------
# quantiser pins
# --------------------------------------------------------------------------

def test_quantiser_hand_cases():
    for line in _golden_lines("quant_hand_cases.txt"):
        vals, codes = line.split(";")
        vals = np.array([float(x) for x in vals.split()], dtype=np.float64)
        codes = np.array([int(x) for x in codes.split()], dtype=np.int64)
        x = np.zeros((64, 1, vals.size), dtype=np.float16)
        x[0, 0] = vals
        x[1, 0, 0] = 127.0   # absmax of the block is 127 -> scale 1
        c, s = oracle.quantize_k(x, [64])
        assert s[0, 0] == np.float32(1.0)
        assert np.array_equal(c[0, 0].astype(np.int64), codes)


def test_quantiser_zero_block_and_tails():
    # zero block: scale 0, codes 0
    x = np.zeros((64, 2, 8), dtype=np.float16)
    x[:, 1] = 1.0
    c, s = oracle.quantize_k(x, [64])
    assert s[0, 0] == 0 and not c[:, 0].any()
    assert s[1, 0] == np.float32(1.0) / np.float32(127.0) and (c[:, 1] == 127).all()
    # tail block of a 100-row sequence uses rows 64..99 only; a second
    # sequence's rows never enter the first sequence's blocks
    lengths = [100, 50]
    x = np.zeros((150, 1, 4), dtype=np.float16)
    x[:64] = 1.0
    x[64:100] = 0.5
    x[99, 0, 3] = -2.0     # absmax of seq 0 block 1 sits in its last row
    x[100, 0, 0] = 1000.0  # first row of seq 1
    c, s = oracle.quantize_k(x, lengths)
    assert s.shape == (1, 2 + 1)
    assert s[0, 1] == np.float32(2.0) / np.float32(127.0)
    assert c[99, 0, 3] == -127 and c[64, 0, 0] == round(0.5 / float(s[0, 1]))
    assert s[0, 2] == np.float32(1000.0) / np.float32(127.0)
    # Q blocks are 128 rows
    cq, sq = oracle.quantize_q(x, lengths)
    assert sq.shape == (1, 1 + 1)
    assert sq[0, 0] == np.float32(2.0) / np.float32(127.0)


def test_quantiser_error_bound_random():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((300, 3, 64)) * rng.uniform(0.01, 50, (1, 3, 1))).astype(np.float16)
    lengths = [130, 170]
    for block, fn in ((64, oracle.quantize_k), (128, oracle.quantize_q)):
        c, s = fn(x, lengths)
        t0, col = 0, 0
        for L in lengths:
            nb = -(-L // block)
            for b in range(nb):
                r0, r1 = t0 + b * block, min(t0 + L, t0 + (b + 1) * block)
                for h in range(3):
                    blk = x[r0:r1, h].astype(np.float64)
                    cc = c[r0:r1, h].astype(np.float64)
                    sc = float(s[h, col + b])
                    assert np.abs(cc).max() == 127
                    assert np.all(np.abs(cc) <= 127)
                    # |code * s - x| <= s / 2 up to fp32 rounding of x / s
                    assert np.all(np.abs(cc * sc - blk) <= sc * (0.5 + 1e-5))
            t0 += L
            col += nb


def test_int4_quantiser_hand_cases():
    for line in _golden_lines("quant_int4_hand_cases.txt"):
        vals, codes = line.split(";")
        vals = np.array([float(x) for x in vals.split()], dtype=np.float64)
        codes = np.array([int(x) for x in codes.split()], dtype=np.int64)
        x = np.zeros((64, 1, vals.size), dtype=np.float16)
        x[0, 0] = vals
        x[1, 0, 0] = 7.0   # absmax of the block is 7 -> scale 1
        c, s = oracle.quantize_k_int4(x, [64])
        assert s[0, 0] == np.float32(1.0)
        assert np.array_equal(c[0, 0].astype(np.int64), codes)


def test_int4_quantiser_bounds_zero_blocks_and_tails():
    x = np.zeros((64, 2, 8), dtype=np.float16)
    x[:, 1] = -3.0
    c, s = oracle.quantize_k_int4(x, [64])
    assert s[0, 0] == 0 and not c[:, 0].any()
    assert s[1, 0] == np.float32(3.0) / np.float32(7.0) and (c[:, 1] == -7).all()
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((300, 3, 64)) * rng.uniform(0.01, 50, (1, 3, 1))).astype(np.float16)
    lengths = [130, 170]
    for block, fn in ((64, oracle.quantize_k_int4), (128, oracle.quantize_q_int4)):
        c, s = fn(x, lengths)
        t0, col = 0, 0
        for L in lengths:
            nb = -(-L // block)
            for b in range(nb):
                r0, r1 = t0 + b * block, min(t0 + L, t0 + (b + 1) * block)
                for h in range(3):
                    blk = x[r0:r1, h].astype(np.float64)
                    cc = c[r0:r1, h].astype(np.float64)
                    sc = float(s[h, col + b])
                    # the block's largest |x| maps to 7; every code within +-7
                    assert np.abs(cc).max() == 7 and np.all(np.abs(cc) <= 7)
                    assert sc == float(np.float32(np.abs(blk).max()) / np.float32(7.0))
                    # |code * s - x| <= s / 2 up to fp32 rounding of x / s
                    assert np.all(np.abs(cc * sc - blk) <= sc * (0.5 + 1e-5))
            t0 += L
            col += nb


def test_int4_codes_through_the_routed_attention():
    # INT4 codes take the INT8 path's arithmetic (exact integer dots times the
    # two block scales): the oracle fed INT4 codes equals the per-key brute
    # force on the same codes, and all-INT4 words deviate from all-FP16 more
    # than all-INT8 words do
    lengths = [100, 300, 64]
    hq, hk, d = 4, 2, 64
    q, k, v, _, _, _, _ = _inputs(lengths, hq, hk, d, seed=4)
    q4, qs4 = oracle.quantize_q_int4(q, lengths)
    k4, ks4 = oracle.quantize_k_int4(k, lengths)
    assert np.abs(q4).max() <= 7 and np.abs(k4).max() <= 7
    inp4 = (q, k, v, q4, qs4, k4, ks4)
    tm = sum(oracle.n_qtiles(L) for L in lengths)
    rng = np.random.default_rng(3)
    masks = rng.integers(0, 2 ** 63, size=(tm, hk), dtype=np.uint64) * np.uint64(2) + \
        rng.integers(0, 2, size=(tm, hk), dtype=np.uint64)
    gs = [1] * len(lengths)
    O, lse = _run(inp4, masks, gs, lengths, True)
    Or, lr = bf.routed_attention(*inp4, masks, gs, lengths, True)
    assert np.abs(O - Or).max() < 1e-12 and np.abs(lse - lr).max() < 1e-12
    ones = _words(lengths, hk, (1 << 64) - 1)
    base, _ = _run(inp4, _words(lengths, hk, 0), gs, lengths, True)
    dev4 = np.abs(_run(inp4, ones, gs, lengths, True)[0] - base).mean()
    dev8 = np.abs(_run(_inputs(lengths, hq, hk, d, seed=4), ones, gs, lengths, True)[0] - base).mean()
    assert dev4 > 4 * dev8


# --------------------------------------------------------------------------
# routing pins
# --------------------------------------------------------------------------

def test_geometry_closed_forms():
    # L = 4096, g = 1: row qt has 2qt + 2 legal groups, N = 1056 per sequence
    assert [oracle.legal_groups(qt, 4096, 1, True) for qt in (0, 1, 31)] == [2, 4, 64]
    assert sum(oracle.legal_groups(qt, 4096, 1, True) for qt in range(32)) == 1056
    # L = 8192, g = 2: n = qt + 1, N = 2080;  L = 65536, g = 16: N = 16640
    assert sum(oracle.legal_groups(qt, 8192, 2, True) for qt in range(64)) == 2080
    assert sum(oracle.legal_groups(qt, 65536, 16, True) for qt in range(512)) == 16640
    # ragged: L = 100 -> one q-tile, key tiles 0..1
    assert oracle.last_legal_tile(0, 100, True) == 1
    assert oracle.last_legal_tile(0, 100, False) == 1
    assert [oracle.auto_g(L) for L in (64, 4096, 4097, 8192, 65536, 16384)] == [1, 1, 2, 2, 16, 4]
    cu_q, cu_k = oracle.tile_offsets([100, 256, 64])
    assert list(cu_q) == [0, 1, 3, 4] and list(cu_k) == [0, 2, 6, 7]


def test_band_tiny_golden():
    want = [int(x, 16) for x in _golden_lines("band_tiny_l256.txt")]
    m, legal, int8 = oracle.build_routing("band", 50, 0, [256], 1, [1], True)
    assert [int(x) for x in m[:, 0]] == want
    assert list(legal) == [6] and list(int8) == [3]


# Hand-derived routing words (derivation in each file's header): SpTrans's
# stride and tail, the proportional quota's remainder rule with ties, and the
# seeded Row-Random / BigBird shuffles at seed 0.
TEMPLATE_GOLDENS = [
    ("sptrans_l640_p75.txt", "sptrans", 75, 640),
    ("sptrans_l1024_p50.txt", "sptrans", 50, 1024),
    ("aligned_sparse_l1024_p25.txt", "aligned_sparse", 25, 1024),
    ("aligned_sparse_l1024_p30.txt", "aligned_sparse", 30, 1024),
    ("row_random_l640_p50_seed0.txt", "row_random", 50, 640),
    ("bigbird_l640_p50_seed0.txt", "bigbird", 50, 640),
]


@pytest.mark.parametrize("fname,template,percent,L", TEMPLATE_GOLDENS, ids=lambda x: str(x))
def test_template_hand_golden(fname, template, percent, L):
    want = [int(x, 16) for x in _golden_lines(fname)]
    m, legal, int8 = oracle.build_routing(template, percent, 0, [L], 2, [1], True)
    assert [int(x) for x in m[:, 0]] == want
    assert [int(x) for x in m[:, 1]] == want
    assert int(legal[0]) == sum(2 * qt + 2 for qt in range(L // 128))
    assert int(int8[0]) == sum(bin(w).count("1") for w in want)


def test_row_streams_are_the_splitmix64_sequence():
    # row qt's stream state draw(0, qt + 1) is the (qt+1)-th splitmix64 output
    # from state 0, the values of splitmix64_state0.txt
    want = [int(x, 16) for x in _golden_lines("splitmix64_state0.txt")]
    assert [oracle.routing._draw(0, qt + 1) for qt in range(3)] == want


def _workload_geometry(name):
    w = synth.WORKLOADS[name]
    lengths = synth.workload_lengths(name)
    if w["g"] == "auto":
        g = [oracle.auto_g(L) for L in lengths]
    else:
        g = [int(w["g"])] * len(lengths)
    return lengths, g, w


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
@pytest.mark.parametrize("template", oracle.TEMPLATES)
def test_coverage_exact(name, template):
    lengths, g, w = _workload_geometry(name)
    for p in (0, 25, 50, 75, 100):
        m, legal, int8 = oracle.build_routing(template, p, 3, lengths, 2, g, w["causal"])
        row = 0
        for s, L in enumerate(lengths):
            n = [oracle.legal_groups(qt, L, g[s], w["causal"]) for qt in range(oracle.n_qtiles(L))]
            assert max(n) <= 64
            assert legal[s] == sum(n)
            cnt = 0
            for qt, x in enumerate(n):
                wd = int(m[row + qt, 0])
                assert int(m[row + qt, 1]) == wd                      # same word per KV head
                assert wd >> x == 0                                   # no bits beyond legal groups
                cnt += bin(wd).count("1")
            K = (p * sum(n) + 50) // 100
            assert cnt == K == int8[s]
            assert abs(100.0 * cnt / sum(n) - p) <= 50.0 / sum(n) + 1e-9
            if p == 0:
                assert not m[row:row + len(n)].any()
            if p == 100:
                assert all(int(m[row + qt, 0]) == (1 << x) - 1 for qt, x in enumerate(n))
            row += len(n)


def _fp16_sets(template, p, n, seed=0):
    return oracle.fp16_groups(template, p, seed, n)


def test_template_structure():
    n = [2 * qt + 2 for qt in range(32)]               # L = 4096, g = 1
    for p in (25, 50, 75):
        band = _fp16_sets("band", p, n)
        glob = _fp16_sets("global", p, n)
        al = _fp16_sets("aligned_sparse", p, n)
        for x, b, gl, a in zip(n, band, glob, al):
            assert b == set(range(x - len(b), x))             # suffix at the diagonal
            assert gl == set(range(0, len(gl)))               # prefix at the sink keys
            assert a == set(range(x - len(a), x))
            if x >= 2:
                assert {0, 1} <= gl
        # Band is a fixed width: rows differ by at most one group (plus short rows)
        widths = sorted({len(b) for x, b in zip(n, band) if x > len(b)})
        assert len(widths) <= 2
    # SpTrans at a full 64-group row and 75%: exactly residues {6, 7} of each 8
    st = _fp16_sets("sptrans", 75, [64])
    assert st[0] == {b for b in range(64) if b % 8 in (6, 7)}
    # BigBird contains its leftmost and rightmost parts, and the random part varies
    n = [64] * 4
    bb0 = _fp16_sets("bigbird", 50, n, seed=1)
    bb1 = _fp16_sets("bigbird", 50, n, seed=2)
    for s in bb0:
        f = len(s)
        a = -(-f // 3)
        b = -(-(f - a) // 2)
        assert set(range(a)) <= s and set(range(64 - b, 64)) <= s
    assert bb0 != bb1
    rr = _fp16_sets("row_random", 25, n, seed=1)
    assert all(len(s) == 48 for s in rr) and rr[0] != rr[1]


def test_global_workload_width():
    # 8k, g = 2, 75%: width 8 plus one extra for rows 8..43
    n = [qt + 1 for qt in range(64)]
    gl = _fp16_sets("global", 75, n)
    for qt, s in enumerate(gl):
        want = min(8, n[qt]) + (1 if 8 <= qt <= 43 else 0)
        assert s == set(range(want))


# --------------------------------------------------------------------------
# attention pins
# --------------------------------------------------------------------------

SHAPES = [([64], 1, 1, 64), ([100], 1, 1, 64), ([256], 4, 2, 64), ([100, 200, 64], 4, 2, 64),
          ([130], 2, 2, 128)]


@pytest.mark.parametrize("lengths,hq,hk,d", SHAPES)
@pytest.mark.parametrize("causal", [True, False])
def test_all_fp16_equals_softmax_attention(lengths, hq, hk, d, causal):
    inp = _inputs(lengths, hq, hk, d)
    g = [1] * len(lengths)
    O, lse = _run(inp, _words(lengths, hk, 0), g, lengths, causal)
    Or, lr = bf.naive_attention(inp[0], inp[1], inp[2], lengths, causal)
    assert np.abs(O - Or).max() < 1e-12
    assert np.abs(lse - lr).max() < 1e-12


@pytest.mark.parametrize("lengths,hq,hk,d", SHAPES)
def test_all_int8_equals_uniform_int8(lengths, hq, hk, d):
    inp = _inputs(lengths, hq, hk, d)
    g = [1] * len(lengths)
    ones = _words(lengths, hk, (1 << 64) - 1)
    O, lse = _run(inp, ones, g, lengths, True)
    Or, lr = bf.routed_attention(*inp, ones, g, lengths, True)
    assert np.abs(O - Or).max() < 1e-12
    assert np.abs(lse - lr).max() < 1e-12
    # and it is really the INT8 path: it differs from the FP16 result
    O0, _ = _run(inp, _words(lengths, hk, 0), g, lengths, True)
    assert np.abs(O - O0).max() > 1e-6


@pytest.mark.parametrize("g", [1, 2, 3])
def test_mixed_words_equal_per_key_bruteforce(g):
    lengths = [100, 300, 64]
    hq, hk, d = 4, 2, 64
    inp = _inputs(lengths, hq, hk, d, seed=9)
    tm = sum(oracle.n_qtiles(L) for L in lengths)
    rng = np.random.default_rng(g)
    masks = rng.integers(0, 2 ** 63, size=(tm, hk), dtype=np.uint64) * np.uint64(2) + \
        rng.integers(0, 2, size=(tm, hk), dtype=np.uint64)
    gs = [g] * len(lengths)
    for causal in (True, False):
        O, lse = _run(inp, masks, gs, lengths, causal)
        Or, lr = bf.routed_attention(*inp, masks, gs, lengths, causal)
        assert np.abs(O - Or).max() < 1e-12
        assert np.abs(lse - lr).max() < 1e-12


def test_bits_beyond_legal_groups_are_ignored():
    lengths = [300]
    inp = _inputs(lengths, 2, 1, 64)
    m, _, _ = oracle.build_routing("sptrans", 75, 0, lengths, 1, [1], True)
    full = m.copy()
    for qt in range(m.shape[0]):
        n = oracle.legal_groups(qt, 300, 1, True)
        full[qt] = np.uint64(int(m[qt, 0]) | (((1 << 64) - 1) ^ ((1 << n) - 1)))
    a, _ = _run(inp, m, [1], lengths, True)
    b, _ = _run(inp, full, [1], lengths, True)
    assert np.array_equal(a, b)


def test_illegal_entries_never_contribute():
    # NaN in every K/V block after the last legal tile of q-tile row 0, and in
    # the neighbouring sequences: rows 0..127 of the middle sequence unchanged.
    lengths = [64, 384, 128]
    hq, hk, d = 2, 1, 64
    inp = list(_inputs(lengths, hq, hk, d))
    m = oracle.build_routing("bigbird", 50, 1, lengths, hk, [1, 1, 1], True)[0]
    base, _ = _run(inp, m, [1, 1, 1], lengths, True)
    q, k, v = inp[0].copy(), inp[1].copy(), inp[2].copy()
    t0 = 64
    last = oracle.last_legal_tile(0, 384, True)         # = 1
    k[t0 + (last + 1) * 64:t0 + 384] = np.nan
    v[t0 + (last + 1) * 64:t0 + 384] = np.inf
    k[:64] = np.nan
    v[:64] = np.nan
    k[448:] = np.nan
    v[448:] = np.nan
    q8, qs = oracle.quantize_q(q, lengths)
    k8, ks = oracle.quantize_k(k, lengths)
    got, _ = _run([q, k, v, q8, qs, k8, ks], m, [1, 1, 1], lengths, True)
    assert np.isfinite(got[t0:t0 + 128]).all()
    assert np.array_equal(got[t0:t0 + 128], base[t0:t0 + 128])


def test_gqa_heads_share_their_kv_word():
    lengths = [256, 130]
    hq, hk, d = 4, 2, 64
    inp = _inputs(lengths, hq, hk, d, seed=4)
    tm = sum(oracle.n_qtiles(L) for L in lengths)
    rng = np.random.default_rng(0)
    masks = rng.integers(0, 16, size=(tm, hk), dtype=np.uint64)
    assert (masks[:, 0] != masks[:, 1]).any()
    g = [1, 1]
    O, _ = _run(inp, masks, g, lengths, True)
    q, k, v, q8, qs, k8, ks = inp
    for h in range(hq):
        kv = h // 2
        sub = (q[:, h:h + 1], k[:, kv:kv + 1], v[:, kv:kv + 1], q8[:, h:h + 1], qs[h:h + 1],
               k8[:, kv:kv + 1], ks[kv:kv + 1])
        Oh, _ = _run(sub, masks[:, kv:kv + 1], g, lengths, True)
        assert np.array_equal(Oh[:, 0], O[:, h])
    # permuting query heads inside a KV group permutes the outputs
    perm = [1, 0, 3, 2]
    sub = (q[:, perm], k, v, q8[:, perm], qs[perm], k8, ks)
    Op, _ = _run(sub, masks, g, lengths, True)
    assert np.array_equal(Op, O[:, perm])


def test_scale_exact_inputs_make_paths_agree():
    # values c * 2^-5 with |c| <= 127 and one |c| = 127 in every block: the
    # quantiser is exact, so INT8 and FP16 scores are the same real number.
    lengths = [256, 100]
    hq, hk, d = 2, 1, 64
    T = sum(lengths)
    rng = np.random.default_rng(11)

    def codes(H):
        c = rng.integers(-127, 128, size=(T, H, d))
        for t in range(0, T, 64):
            c[t, :, 0] = 127 * (1 if (t // 64) % 2 else -1)
        return c

    cq, ck = codes(hq), codes(hk)
    q = (cq * 2.0 ** -5).astype(np.float16)
    k = (ck * 2.0 ** -5).astype(np.float16)
    v = rng.standard_normal((T, hk, d)).astype(np.float16)
    q8, qs = oracle.quantize_q(q, lengths)
    k8, ks = oracle.quantize_k(k, lengths)
    assert np.array_equal(q8, cq) and np.array_equal(k8, ck)
    assert (qs == np.float32(2.0 ** -5)).all() and (ks == np.float32(2.0 ** -5)).all()
    inp = (q, k, v, q8, qs, k8, ks)
    a, la = _run(inp, _words(lengths, hk, (1 << 64) - 1), [1, 1], lengths, True)
    b, lb = _run(inp, _words(lengths, hk, 0), [1, 1], lengths, True)
    assert np.abs(a - b).max() <= 1e-12 and np.abs(la - lb).max() <= 1e-12


def test_int_scores_exact():
    lengths = [200]
    inp = _inputs(lengths, 1, 1, 64)
    q8, k8 = inp[3], inp[5]
    m = oracle.build_routing("band", 50, 0, lengths, 1, [1], True)[0]
    A = oracle.int_scores(q8, k8, m, [1], lengths, 0, 0, 1, 1, True)
    full = q8[:, 0].astype(np.int64) @ k8[:, 0].astype(np.int64).T
    for i in range(200):
        keys = bf.int8_keys_of_word(m[i // 128, 0], 200, 1)
        for j in range(200):
            if j <= i and keys[j]:
                assert A[i, j] == full[i, j]
            else:
                assert A[i, j] == -(2 ** 62)
    assert np.abs(full).max() < 2 ** 22


def test_deviation_grows_with_coverage():
    # not a parity pin: the trend the pages report (deviation from all-FP16
    # rises with INT8 coverage), checked on one seeded case
    lengths = [512]
    inp = _inputs(lengths, 2, 1, 64, seed=2)
    base, _ = _run(inp, _words(lengths, 1, 0), [1], lengths, True)
    mads = []
    for p in (0, 25, 50, 75, 100):
        m = oracle.build_routing("sptrans", p, 0, lengths, 1, [1], True)[0]
        O, _ = _run(inp, m, [1], lengths, True)
        mads.append(np.abs(O - base).mean())
    assert mads[0] == 0.0
    assert all(b >= a for a, b in zip(mads, mads[1:]))


# ------------------------------------------------------------------ decode ---
# The decode step (one new query row per sequence attending to its cache) is
# the prefill row oracle composed with a single-row query block; these pins
# check the composition against whole-matrix brute force.

def _decode_case(lengths, hq, hk, d, seed, slack=5):
    rng = np.random.default_rng(seed)
    starts, a = [], 0
    for L in lengths:
        starts.append(a)
        a += L + slack                      # caches with capacity slack between sequences
    rows = a
    k = rng.standard_normal((rows, hk, d)).astype(np.float16)
    v = rng.standard_normal((rows, hk, d)).astype(np.float16)
    q = rng.standard_normal((len(lengths), hq, d)).astype(np.float16)
    qt = [0]
    for L in lengths:
        qt.append(qt[-1] + (L + 127) // 128)
    return q, k, v, np.array(starts), np.array(lengths), np.array(qt[:-1]), qt[-1]


@pytest.mark.parametrize("lengths,hq,hk,d", [([1, 64, 65, 200], 4, 2, 64), ([130, 7], 3, 1, 128)])
def test_decode_all_fp16_equals_softmax_of_the_new_row(lengths, hq, hk, d):
    q, k, v, st, ln, qts, nqt = _decode_case(lengths, hq, hk, d, 1)
    masks = np.zeros((nqt, hk), dtype=np.uint64)
    o, lse = oracle.decode_rows(q, k, v, st, ln, masks, qts, np.ones(len(lengths), np.int32))
    for s, L in enumerate(lengths):
        qs = np.zeros((L, hq, d), dtype=np.float16)
        qs[L - 1] = q[s]
        want, wl = bf.naive_attention(qs, k[st[s]:st[s] + L], v[st[s]:st[s] + L], [L], True)
        assert np.abs(o[s] - want[L - 1]).max() < 1e-12
        assert np.abs(lse[s] - wl[:, L - 1]).max() < 1e-12


@pytest.mark.parametrize("lengths,hq,hk,d", [([1, 63, 64, 129], 2, 2, 64), ([300], 4, 2, 128)])
def test_decode_all_int8_equals_integer_bruteforce(lengths, hq, hk, d):
    q, k, v, st, ln, qts, nqt = _decode_case(lengths, hq, hk, d, 2)
    masks = np.full((nqt, hk), np.uint64(2 ** 64 - 1), dtype=np.uint64)
    o, _ = oracle.decode_rows(q, k, v, st, ln, masks, qts, np.ones(len(lengths), np.int32))
    scale = 1.0 / math.sqrt(d)
    for s, L in enumerate(lengths):
        K, V = k[st[s]:st[s] + L], v[st[s]:st[s] + L]
        k8, ks = oracle.quantize_k(K, [L])              # pinned above
        for h in range(hq):
            kv = h // (hq // hk)
            x = q[s, h].astype(np.float32)
            a = np.float32(np.abs(x).max())
            sq = np.float32(a / np.float32(127.0))
            q8 = np.clip(np.rint(x / sq), -127, 127).astype(np.int64)
            dots = k8[:, kv].astype(np.int64) @ q8       # exact integers, [L]
            sk = ks[kv, np.arange(L) // 64].astype(np.float64)
            S = dots.astype(np.float64) * float(sq) * sk * scale
            P = np.exp(S - S.max())
            want = (P @ V[:, kv].astype(np.float64)) / P.sum()
            assert np.abs(o[s, h] - want).max() < 1e-12


def test_decode_matches_prefill_row_when_the_query_tile_is_the_new_row():
    # with an all-FP16 word the query quantisation plays no part: the decode of
    # position t equals the prefill oracle's row t of the same sequence
    L, hq, hk, d = 100, 2, 1, 64
    q, k, v, st, ln, qts, nqt = _decode_case([L], hq, hk, d, 3, slack=0)
    qs = np.zeros((L, hq, d), dtype=np.float16)
    qs[L - 1] = q[0]
    masks = np.zeros((nqt, hk), dtype=np.uint64)
    o, _ = oracle.decode_rows(q, k, v, st, ln, masks, qts, np.ones(1, np.int32))
    q8, qsc = oracle.quantize_q(qs, [L])
    k8, ksc = oracle.quantize_k(k, [L])
    want, _ = oracle.attention_rows(qs, k, v, q8, qsc, k8, ksc, masks, np.ones(1, np.int32), [L],
                                    True, rows=np.array([(0, h, L - 1) for h in range(hq)]))
    assert np.abs(o[0] - want).max() < 1e-12


def test_decode_reads_the_word_of_the_new_rows_query_tile():
    # row 0 of the sequence's words says all INT8, row 1 (where t = 199 lives)
    # all FP16: the result is the FP16 one
    L, hq, hk, d = 200, 2, 1, 64
    q, k, v, st, ln, qts, nqt = _decode_case([L], hq, hk, d, 4, slack=0)
    masks = np.array([[2 ** 64 - 1], [0]], dtype=np.uint64)
    o, _ = oracle.decode_rows(q, k, v, st, ln, masks, qts, np.ones(1, np.int32))
    o16, _ = oracle.decode_rows(q, k, v, st, ln, np.zeros_like(masks), qts, np.ones(1, np.int32))
    assert np.abs(o - o16).max() == 0.0


def test_decode_query_rows_are_their_own_blocks():
    x = np.zeros((2, 1, 64), dtype=np.float16)
    x[0, 0, :3] = [127.0, -63.5, 0.5]       # a = 127 -> s = 1: rne(-63.5) = -64, rne(0.5) = 0
    x[1, 0, 0] = 2.0                        # a second row with its own scale
    c, s = oracle.quantize_rows(x)
    assert list(c[0, 0, :3]) == [127, -64, 0] and s[0, 0] == np.float32(1.0)
    assert c[1, 0, 0] == 127 and s[1, 0] == np.float32(np.float32(2.0) / np.float32(127.0))


# ---------------------------------------------------------- adaptive routing --
# Pins of oracle/adaptive.py (the pooled-score policy): hand-derived fp32
# values for the stated summation order, closed-form words for constructed
# inputs, the static templates' quota, and the aligned-sparse layout that the
# policy must reproduce when the scores grow with the key position.

from oracle import adaptive as ad  # noqa: E402


def test_adaptive_mean_uses_interleaved_partial_sums():
    # item 0 = 2^24, items 1 and 9 = 1: partial sum 1 holds 1 + 1 = 2 exactly,
    # so the total is 2^24 + 2; a running sum would lose both ones (ties to even)
    items = np.zeros((10, 1), dtype=np.float32)
    items[0, 0] = 2.0 ** 24
    items[1, 0] = 1.0
    items[9, 0] = 1.0
    got = ad.interleaved_mean(items)
    assert got.dtype == np.float32
    assert got[0] == np.float32(16777218.0) / np.float32(10.0)
    seq = np.float32(0.0)
    for x in items[:, 0]:
        seq = np.float32(seq + x)
    assert seq == np.float32(2.0 ** 24)      # what the order rules out
    assert np.array_equal(ad.interleaved_mean(np.zeros((0, 3), np.float32)), np.zeros(3, np.float32))
    # exact small integers: the mean is exact
    v = np.arange(24, dtype=np.float32).reshape(24, 1)
    assert ad.interleaved_mean(v)[0] == np.float32(11.5)


def test_adaptive_dot_rounds_each_product():
    a = np.float32(1.0 + 2.0 ** -12)
    # a*a = 1 + 2^-11 + 2^-24 rounds to 1 + 2^-11 (tie to even); a*(-a) the
    # same with a minus sign: separately rounded the dot is 0, a fused
    # multiply-add in the second step would give -2^-24
    got = ad.ordered_dot(np.array([a, a], np.float32), np.array([[a, -a]], np.float32))
    assert got[0] == np.float32(0.0)
    assert math.copysign(1.0, float(np.float32(a) * np.float32(a) - np.float64(a) * np.float64(a))) < 0


def test_adaptive_choose_ties_go_to_the_lower_group():
    assert ad.choose_int8([0.0] * 6, 3) == {0, 1, 2}
    assert ad.choose_int8([3.0, 1.0, 1.0, 2.0], 2) == {1, 2}
    assert ad.choose_int8([3.0, 1.0, 1.0, 2.0], 3) == {1, 2, 3}
    assert ad.choose_int8([1.0, -0.0, 0.0], 1) == {1}  # -0 == 0: the lower index


def _ramp_keys(lengths, hk, d, slope):
    """K rows whose channel 0 holds slope * (key tile index + 1), other channels 0."""
    T = sum(lengths)
    k = np.zeros((T, hk, d), dtype=np.float16)
    start = 0
    for L in lengths:
        for j in range(L):
            k[start + j, :, 0] = np.float16(slope * (j // 64 + 1))
        start += L
    return k


@pytest.mark.parametrize("percent", [0, 25, 50, 75, 100])
def test_adaptive_rising_scores_give_the_aligned_sparse_layout(percent):
    # q = e0 and k tiles rising along the key axis: the score grows with the
    # tile, so each row's lowest-scoring groups are its leftmost ones and the
    # FP16 groups are the rightmost f_r: the aligned-sparse template's words
    lengths, hq, hk, d = [300, 1000, 64], 4, 2, 64
    T = sum(lengths)
    q = np.zeros((T, hq, d), dtype=np.float16)
    q[:, :, 0] = np.float16(0.5)
    k = _ramp_keys(lengths, hk, d, 0.25)
    g = [1, 2, 1]
    for causal in (True, False):
        got = ad.route_pooled(q, k, lengths, hq, hk, g, causal, percent)
        want, _, _ = oracle.build_routing("aligned_sparse", percent, 0, lengths, hk, g, causal)
        assert np.array_equal(got, want), (percent, causal)


def test_adaptive_falling_scores_keep_the_left_groups():
    # scores falling along the key axis: the INT8 groups are the rightmost k_r
    lengths, hq, hk, d = [1000], 2, 1, 64
    q = np.zeros((1000, hq, d), dtype=np.float16)
    q[:, :, 0] = np.float16(-1.0)
    k = _ramp_keys(lengths, hk, d, 0.125)
    got = ad.route_pooled(q, k, lengths, hq, hk, [1], True, 50)
    n = [oracle.legal_groups(qt, 1000, 1, True) for qt in range(oracle.n_qtiles(1000))]
    kq = ad._quota(n, 50)
    for qt, (x, kr) in enumerate(zip(n, kq)):
        want = sum(1 << b for b in range(x - kr, x))
        assert int(got[qt, 0]) == want, qt


@pytest.mark.parametrize("percent", [10, 33, 75])
def test_adaptive_quota_and_legality(percent):
    rng = np.random.default_rng(7)
    lengths, hq, hk, d = [129, 777, 2048], 6, 2, 64
    T = sum(lengths)
    q = rng.standard_normal((T, hq, d)).astype(np.float16)
    k = rng.standard_normal((T, hk, d)).astype(np.float16)
    g = [1, 1, 2]
    got = ad.route_pooled(q, k, lengths, hq, hk, g, True, percent)
    cq = 0
    for s, L in enumerate(lengths):
        n = [oracle.legal_groups(qt, L, g[s], True) for qt in range(oracle.n_qtiles(L))]
        kq = ad._quota(n, percent)
        for qt, (x, kr) in enumerate(zip(n, kq)):
            for kv in range(hk):
                w = int(got[cq + qt, kv])
                assert w >> x == 0                      # no bits past the legal groups
                assert bin(w).count("1") == kr          # the templates' per-row quota
        assert sum(kq) == oracle.int8_target(percent, sum(n))
        cq += oracle.n_qtiles(L)


def test_adaptive_pooled_means_by_brute_force():
    rng = np.random.default_rng(3)
    lengths, hq, hk, d = [130, 64], 6, 2, 64
    T = sum(lengths)
    q = rng.standard_normal((T, hq, d)).astype(np.float16)
    k = rng.standard_normal((T, hk, d)).astype(np.float16)
    kv_map = np.array([1, 0, 0, 1, 1, 0], dtype=np.int32)
    qb, kb = ad.pooled_means(q, k, lengths, hq, hk, kv_map)
    assert qb.shape == (3, hk, d) and kb.shape == (4, hk, d)
    # q tile 1 of sequence 0 is rows 128..129 of heads {1, 2, 5} for KV head 0
    items = [q[r, h].astype(np.float64) for h in (1, 2, 5) for r in (128, 129)]
    np.testing.assert_allclose(qb[1, 0], np.mean(items, axis=0), rtol=1e-6, atol=1e-6)
    # key tile 2 of sequence 0 is rows 128..129
    np.testing.assert_allclose(kb[2, 1], k[128:130, 1].astype(np.float64).mean(axis=0),
                               rtol=1e-6, atol=1e-6)
    # key tile 3 is the 64 rows of sequence 1
    np.testing.assert_allclose(kb[3, 0], k[130:194, 0].astype(np.float64).mean(axis=0),
                               rtol=1e-5, atol=1e-6)


# ------------------------------------------------------- importance-mass probe --
from oracle import mass as om  # noqa: E402


def _words_all(lengths, hk, bit):
    n = sum(oracle.n_qtiles(L) for L in lengths)
    return np.full((n, hk), np.uint64((1 << 64) - 1 if bit else 0), dtype=np.uint64)


def test_mass_probe_all_fp16_and_all_int8_words():
    rng = np.random.default_rng(11)
    lengths, hq, hk, d = [200, 70], 2, 1, 64
    q = rng.standard_normal((270, hq, d)).astype(np.float16)
    k = rng.standard_normal((270, hk, d)).astype(np.float16)
    r0 = om.probe_rows(q, k, _words_all(lengths, hk, 0), [1, 1], lengths, True)
    assert np.all(r0["m8"] == 0) and np.all(r0["h8"] == 0)
    r1 = om.probe_rows(q, k, _words_all(lengths, hk, 1), [1, 1], lengths, True)
    np.testing.assert_allclose(r1["m8"], 1.0, atol=1e-12)
    np.testing.assert_allclose(r1["h8"], r1["h"], atol=1e-12)
    assert np.all(r1["h"] <= 1 + 1e-12) and np.all(r1["h"] > 0)


def test_empty_sequences_change_nothing():
    """Zero-length sequences hold no rows and no tiles: a batch with them
    inserted gives the same mass-probe rows and adaptive words as without."""
    rng = np.random.default_rng(5)
    hq, hk, d = 2, 1, 64
    q = rng.standard_normal((194, hq, d)).astype(np.float16)
    k = rng.standard_normal((194, hk, d)).astype(np.float16)
    plain, padded = [130, 64], [0, 130, 0, 64, 0]
    g_plain, g_padded = [1, 1], [1, 1, 1, 1, 1]
    m_plain = oracle.build_routing("sptrans", 75, 0, plain, hk, g_plain, True)[0]
    m_padded = oracle.build_routing("sptrans", 75, 0, padded, hk, g_padded, True)[0]
    assert np.array_equal(m_plain, m_padded)
    a = om.probe_rows(q, k, m_plain, g_plain, plain, True)
    b = om.probe_rows(q, k, m_padded, g_padded, padded, True)
    for key in a:
        assert np.array_equal(a[key], b[key]), key
    w_plain = ad.route_pooled(q, k, plain, hq, hk, g_plain, True, 50)
    w_padded = ad.route_pooled(q, k, padded, hq, hk, g_padded, True, 50)
    assert np.array_equal(w_plain, w_padded)


def test_mass_probe_uniform_scores_closed_form():
    # q = 0: every legal key scores 0, P is uniform over the i + 1 legal keys,
    # every key is high-importance, and the INT8 mass is the INT8 key count
    # over i + 1
    lengths, hq, hk, d = [300], 1, 1, 64
    q = np.zeros((300, hq, d), dtype=np.float16)
    k = np.random.default_rng(1).standard_normal((300, hk, d)).astype(np.float16)
    words = np.array([[0b101], [0b1010], [0b10001]], dtype=np.uint64)  # one word per 128 rows
    r = om.probe_rows(q, k, words, [1], lengths, True)
    for i in range(300):
        w = int(words[i // 128, 0])
        n8 = sum(1 for j in range(i + 1) if (w >> (j // 64)) & 1)
        assert abs(r["m8"][0, i] - n8 / (i + 1)) < 1e-12
        assert abs(r["h"][0, i] - 1.0) < 1e-12
        assert abs(r["h8"][0, i] - n8 / (i + 1)) < 1e-12


def test_mass_probe_two_key_hand_case():
    # row 1 sees keys 0 and 1 with scores 0 and a: P = (1, e^a) / (1 + e^a);
    # with a = 4 ln 2 + 0.1 key 0 falls below the 2^-4 threshold (delta 4)
    d = 64
    a = 4 * math.log(2) + 0.1
    q = np.zeros((2, 1, d), dtype=np.float16)
    k = np.zeros((2, 1, d), dtype=np.float16)
    q[1, 0, 0] = np.float16(1.0)
    k[1, 0, 0] = np.float16(a * math.sqrt(d))
    k_eff = float(np.float16(a * math.sqrt(d))) / math.sqrt(d)      # the fp16-rounded score
    words = np.array([[0b1]], dtype=np.uint64)                       # tile 0 (both keys) INT8
    r = om.probe_rows(q, k, words, [1], [2], True)
    p1 = math.exp(k_eff) / (1 + math.exp(k_eff))
    assert k_eff > 4 * math.log(2)
    assert abs(r["m8"][0, 1] - 1.0) < 1e-12
    assert abs(r["h"][0, 1] - p1) < 1e-12
    assert abs(r["h8"][0, 1] - p1) < 1e-12
    assert abs(om.exposure(r["h"], r["h8"]) - 1.0) < 1e-12


def test_mass_probe_matches_python_loops():
    rng = np.random.default_rng(5)
    lengths, hq, hk, d = [150, 9], 2, 1, 64
    T = sum(lengths)
    q = (rng.standard_normal((T, hq, d)) * 0.5).astype(np.float16)
    k = rng.standard_normal((T, hk, d)).astype(np.float16)
    words = np.array([[0b01], [0b10], [0b1]], dtype=np.uint64)
    r = om.probe_rows(q, k, words, [1, 1], lengths, True, delta=2.0)
    start, cq = 0, 0
    for s, L in enumerate(lengths):
        for h in range(hq):
            for i in range(0, L, 7):
                sc = [sum(float(q[start + i, h, c]) * float(k[start + j, 0, c]) for c in range(d))
                      / 8.0 for j in range(i + 1)]
                mx = max(sc)
                e = [math.exp(x - mx) for x in sc]
                tot = sum(e)
                w = int(words[cq + i // 128, 0])
                m8 = sum(e[j] for j in range(i + 1) if (w >> (j // 64)) & 1) / tot
                hh = sum(e[j] for j in range(i + 1) if sc[j] >= mx - 2 * math.log(2)) / tot
                h8 = sum(e[j] for j in range(i + 1)
                         if sc[j] >= mx - 2 * math.log(2) and (w >> (j // 64)) & 1) / tot
                assert abs(r["m8"][h, start + i] - m8) < 1e-10
                assert abs(r["h"][h, start + i] - hh) < 1e-10
                assert abs(r["h8"][h, start + i] - h8) < 1e-10
        start += L
        cq += oracle.n_qtiles(L)


# ------------------------------------------------------------- FP8 low path --
from oracle import fp8 as of8  # noqa: E402


def test_e4m3_table_fixed_points():
    D = of8.DECODE
    assert D[0x00] == 0.0 and D[0x80] == 0.0 and math.copysign(1, D[0x80]) < 0
    assert D[0x01] == 2.0 ** -9                    # smallest subnormal
    assert D[0x07] == 7 * 2.0 ** -9                # largest subnormal
    assert D[0x08] == 2.0 ** -6                    # smallest normal
    assert D[0x38] == 1.0 and D[0x40] == 2.0 and D[0x30] == 0.5
    assert D[0x7E] == 448.0 and D[0xFE] == -448.0  # largest finite
    assert math.isnan(D[0x7F]) and math.isnan(D[0xFF])
    pos = D[:0x7F]
    assert np.all(np.diff(pos) > 0)                # strictly increasing codes 0..0x7E
    assert np.array_equal(D[0x80:0xFF], -pos)      # sign symmetry


def test_e4m3_encode_round_trip_ties_and_saturation():
    pos = of8.DECODE[:0x7F]
    codes = np.arange(0x7F, dtype=np.uint8)
    assert np.array_equal(of8.e4m3_encode(pos.astype(np.float32)), codes)
    assert np.array_equal(of8.e4m3_encode(-pos[1:].astype(np.float32)), codes[1:] | 0x80)
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)   # exact in fp32
    assert np.all(mids.astype(np.float64) == (pos[:-1] + pos[1:]) / 2)
    got = of8.e4m3_encode(mids).astype(int)
    lower = np.arange(0x7E)
    assert np.array_equal(got, np.where(lower % 2 == 0, lower, lower + 1))   # ties to even
    just_above = np.nextafter(mids, np.float32(1000))
    assert np.array_equal(of8.e4m3_encode(just_above).astype(int), lower + 1)
    sat = of8.e4m3_encode(np.array([448.0, 463.9, 464.0, 1e6, -1e6], np.float32))
    assert list(sat) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_fp8_block_quantiser():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((200, 2, 64)) * 3).astype(np.float16)
    x[5, 1, 7] = np.float16(-40.0)                 # the block's absmax, negative
    codes, sc = of8.quantize_blocks_fp8(x, [200], 64)
    assert codes.dtype == np.uint8 and sc.shape == (2, 4)
    assert sc[1, 0] == np.float32(40.0) / np.float32(448.0)
    assert codes[5, 1, 7] == 0xFE                  # -absmax -> -448
    back = of8.DECODE[codes] * sc[np.arange(2)[None, :, None], (np.arange(200) // 64)[:, None, None]]
    err = np.abs(back - x.astype(np.float64))
    # e4m3 keeps 3 mantissa bits: half an ulp is at most 2^-4 of the value
    # (normal range); below 2^-6 s the subnormal spacing 2^-9 s bounds it
    bound = np.maximum(np.abs(x.astype(np.float64)) * 2.0 ** -4,
                       2.0 ** -10 * sc[np.arange(2)[None, :, None], (np.arange(200) // 64)[:, None, None]])
    assert np.all(err <= bound * (1 + 1e-6))
    z = np.zeros((10, 1, 64), np.float16)
    c0, s0 = of8.quantize_blocks_fp8(z, [10], 64)
    assert np.all(c0 == 0) and s0[0, 0] == 0.0


def test_fp8_scale_exact_inputs_make_paths_agree():
    # every block holds values whose ratio to the block scale is an exact e4m3
    # value: the FP8 scores equal the FP16 scores, so all-FP8 routing gives
    # the all-FP16 output
    rng = np.random.default_rng(9)
    lengths, hq, hk, d = [130, 64], 2, 1, 64
    T = sum(lengths)
    grid = of8.DECODE[rng.integers(0x30, 0x50, size=(T, hq + 2 * hk, d))]   # 0.5 .. 8, exact
    sign = rng.choice([-1.0, 1.0], size=grid.shape)
    vals = (grid * sign * 0.125).astype(np.float16)                        # exact in fp16
    q, k = vals[:, :hq], vals[:, hq:hq + hk]
    for blk_rows, arr in ((128, q), (64, k)):
        start = 0
        for L in lengths:
            for b in range(0, L, blk_rows):
                arr[start + b, :, 0] = np.float16(56.0)   # absmax 56 = 448 * 0.125 per block
            start += L
    v = rng.standard_normal((T, hk, d)).astype(np.float16)
    q8, qs = of8.quantize_q_fp8(q, lengths)
    k8, ks = of8.quantize_k_fp8(k, lengths)
    assert np.all(qs[qs > 0] == np.float32(0.125)) and np.all(ks[ks > 0] == np.float32(0.125))
    ones, _, _ = oracle.build_routing("band", 100, 0, lengths, hk, [1, 1], True)
    zeros, _, _ = oracle.build_routing("band", 0, 0, lengths, hk, [1, 1], True)
    o8, l8 = oracle.attention_rows(q, k, v, q8, qs, k8, ks, ones, [1, 1], lengths, True, low="fp8")
    o16, l16 = oracle.attention_rows(q, k, v, q8, qs, k8, ks, zeros, [1, 1], lengths, True, low="fp8")
    np.testing.assert_allclose(o8, o16, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l8, l16, rtol=0, atol=1e-12)
    # and the INT8 reading of the same bytes differs (the flag is used)
    oi, _ = oracle.attention_rows(q, k, v, q8.view(np.int8), qs, k8.view(np.int8), ks, ones,
                                  [1, 1], lengths, True)
    assert np.max(np.abs(oi - o16)) > 1e-3
