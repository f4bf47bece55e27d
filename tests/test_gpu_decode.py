"""GPU parity of the decode step with the INT8 K cache (tilemix_decode_fwd)
against the oracle: the re-quantised last K blocks bit for bit, O within
max-abs 2e-3 / mean-abs 2e-4."""
import numpy as np
import pytest

import oracle
import synth
from tests import gpu_cases as gc

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gc.set_test_timeout()


def _run(lengths, hq, hk, d, masks_fn, g, seed, slack=37, kv_map=None, tiles_per_split=0):
    import tile_routed_mixed_b200 as tm
    rng = np.random.default_rng(seed)
    nseq = len(lengths)
    starts, ktiles, a, kt = [], [], 0, 0
    for L in lengths:
        starts.append(a)
        ktiles.append(kt)
        a += L + slack                       # cache capacity beyond the current length
        kt += (L + slack + 63) // 64
    rows, total_kt = a, kt
    k = synth.fp16_normal(seed, 2, (rows, hk, d))
    v = synth.fp16_normal(seed, 3, (rows, hk, d))
    q = synth.fp16_normal(seed, 1, (nseq, hq, d))
    qt = np.zeros(nseq + 1, dtype=np.int64)
    qt[1:] = np.cumsum([(L + 127) // 128 for L in lengths])
    masks = masks_fn(int(qt[-1]))
    # INT8 K cache as the previous steps left it: every block current except
    # the one holding the new key, which is stale
    k8 = np.zeros((rows, hk, d), dtype=np.int8)
    ks = np.zeros((hk, total_kt), dtype=np.float32)
    want_k8, want_ks = k8.copy(), ks.copy()
    for s, L in enumerate(lengths):
        c, sc = oracle.quantize_k(np.ascontiguousarray(k[starts[s]:starts[s] + L]), [L])
        want_k8[starts[s]:starts[s] + L] = c
        want_ks[:, ktiles[s]:ktiles[s] + sc.shape[1]] = sc
        k8[starts[s]:starts[s] + L] = c
        ks[:, ktiles[s]:ktiles[s] + sc.shape[1]] = sc
        if L == 0:
            continue
        b = (L - 1) // 64
        k8[starts[s] + 64 * b:starts[s] + L] = 99
        ks[:, ktiles[s] + b] = -1.0
    dev = "cuda"
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    dec = tm.TileMixDecode(starts, lengths, ktiles, qt[:-1], hq, hk, d, masks, g, total_kt,
                           kv_head_of_q=kv_map, device=dev, tiles_per_split=tiles_per_split)
    qd, kd, vd, k8d, ksd = t(q), t(k), t(v), t(k8), t(ks)
    o = dec(qd, kd, vd, k8d, ksd, o=torch.full_like(qd, float("nan")))
    torch.cuda.synchronize()
    assert tm.tilemix_get_error() == tm.OK
    got_k8, got_ks = k8d.cpu().numpy(), ksd.cpu().numpy()
    for s, L in enumerate(lengths):
        assert np.array_equal(got_k8[starts[s]:starts[s] + L], want_k8[starts[s]:starts[s] + L])
    assert np.array_equal(got_ks.view(np.uint32), want_ks.view(np.uint32))
    # an empty sequence has no token: nothing is computed for it and its O
    # rows keep what they held
    live = [s for s, L in enumerate(lengths) if L > 0]
    got = o.cpu().numpy().astype(np.float64)
    for s, L in enumerate(lengths):
        if L == 0:
            assert np.isnan(got[s]).all()
    want, _ = oracle.decode_rows(q[live], k, v, [starts[s] for s in live], [lengths[s] for s in live],
                                 masks, qt[:-1][live], g[live], kv_map=kv_map)
    got = got[live]
    assert np.isfinite(got).all()
    mx, mn = gc.errors(got.reshape(-1, d), want.reshape(-1, d))
    assert mx <= gc.MAX_ABS and mn <= gc.MEAN_ABS, (mx, mn)
    return mx, mn


def _template(name, percent, lengths, hk, g):
    def f(nqt):
        m, _, _ = oracle.build_routing(name, percent, 0, lengths, hk, g, True)
        assert m.shape == (nqt, hk)
        return m
    return f


@pytest.mark.parametrize("lengths", [[1, 63, 64, 65, 200, 1000], [4096] * 8])
def test_decode_sptrans_ragged(lengths):
    g = np.ones(len(lengths), dtype=np.int32)
    _run(lengths, 24 if len(lengths) == 8 else 6, 8 if len(lengths) == 8 else 2, 128,
         _template("sptrans", 75, lengths, 8 if len(lengths) == 8 else 2, g), g, seed=5)


def test_decode_d64_gqa4_bigbird_g2():
    lengths = [129, 640, 33]
    g = np.full(len(lengths), 2, dtype=np.int32)
    _run(lengths, 4, 1, 64, _template("bigbird", 50, lengths, 1, g), g, seed=6)


@pytest.mark.parametrize("word", [0, 2 ** 64 - 1])
def test_decode_all_fp16_and_all_int8(word):
    lengths = [77, 300]
    g = np.ones(2, dtype=np.int32)
    _run(lengths, 8, 2, 128, lambda n: np.full((n, 2), np.uint64(word), dtype=np.uint64), g, seed=7)


def test_decode_custom_head_map():
    lengths = [150, 90]
    g = np.ones(2, dtype=np.int32)
    kv_map = np.array([1, 0, 1, 0, 0, 1], dtype=np.int32)
    _run(lengths, 6, 2, 128, _template("row_random", 50, lengths, 2, g), g, seed=8, kv_map=kv_map)


def test_decode_long_context():
    lengths = [16384, 5000]
    g = np.array([oracle.auto_g(L) for L in lengths], dtype=np.int32)
    _run(lengths, 8, 2, 128, _template("row_random", 25, lengths, 2, g), g, seed=9)


@pytest.mark.parametrize("group,d", [(1, 128), (2, 64), (5, 128), (7, 64), (8, 128), (12, 64),
                                     (16, 128)])
def test_decode_group_sizes(group, d):
    """Every compiled group size, and the generic path (12, 16) that takes any
    count up to 16."""
    lengths = [70, 257, 1]
    g = np.ones(len(lengths), dtype=np.int32)
    _run(lengths, 2 * group, 2, d, _template("sptrans", 75, lengths, 2, g), g, seed=10 + group)


def test_decode_zero_length_sequences():
    lengths = [0, 70, 0, 200, 0]
    g = np.ones(len(lengths), dtype=np.int32)
    _run(lengths, 4, 2, 128, _template("sptrans", 75, lengths, 2, g), g, seed=11)


@pytest.mark.parametrize("tps", [1, 3, 5, 16, 64])
def test_decode_tiles_per_split(tps):
    """Splits of several tiles: the copy ring wraps (tiles past the number of
    stages), splits end ragged, and one split may hold a whole sequence."""
    lengths = [1000, 64, 3000, 129]
    g = np.ones(len(lengths), dtype=np.int32)
    _run(lengths, 12, 4, 128, _template("sptrans", 75, lengths, 4, g), g, seed=30 + tps,
         tiles_per_split=tps)
