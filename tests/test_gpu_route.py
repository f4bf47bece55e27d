"""GPU parity of pooled-score adaptive routing (tilemix_route_pooled) with the
oracle: the routing words bit for bit, and prefill on those words within the
attention tolerance."""
import numpy as np
import pytest

import oracle
from oracle import adaptive
import synth
from tests import gpu_cases as gc

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gc.set_test_timeout()


def _words(lengths, hq, hk, d, g, causal, percent, seed, kv_map=None, outliers=0):
    import tile_routed_mixed_b200 as tm
    T = sum(lengths)
    q, k, _ = synth.make_qkv(seed, T, hq, hk, d, outliers=outliers, lowrank=False)
    got = tm.route_pooled(torch.from_numpy(q).cuda(), torch.from_numpy(k).cuda(), lengths, hq,
                          hk, g, causal, percent, kv_head_of_q=kv_map)
    torch.cuda.synchronize()
    assert tm.tilemix_get_error() == tm.OK
    want = adaptive.route_pooled(q, k, lengths, hq, hk, g, causal, percent, kv_map=kv_map)
    got = got.cpu().numpy().view(np.uint64)
    assert got.shape == want.shape
    bad = np.argwhere(got != want)
    assert bad.size == 0, (bad[:5], got[tuple(bad[0])], want[tuple(bad[0])])
    return q, k, got


@pytest.mark.parametrize("percent", [0, 25, 75, 100])
def test_route_ragged_causal_bit_exact(percent):
    lengths = [1, 64, 65, 300, 1000, 2048]
    _words(lengths, 6, 2, 128, [1] * 6, True, percent, seed=21)


def test_route_noncausal_d64_g2_bit_exact():
    lengths = [700, 129, 4096]
    _words(lengths, 8, 2, 64, [2, 1, 2], False, 50, seed=22)


def test_route_head_map_and_outliers_bit_exact():
    lengths = [513, 1200]
    kv_map = np.array([2, 0, 1, 1, 0, 2, 0, 1, 1], dtype=np.int32)
    _words(lengths, 9, 3, 128, [1, 1], True, 33, seed=23, kv_map=kv_map, outliers=4)


def test_route_benchmark_shape_bit_exact():
    lengths = [4096] * 2
    _words(lengths, 24, 8, 128, [1, 1], True, 75, seed=24)


def test_prefill_on_adaptive_words_matches_oracle():
    """The words feed the prefill path unchanged (same mask ABI)."""
    import tile_routed_mixed_b200 as tm
    lengths, hq, hk, d = [300, 1000], 4, 2, 128
    g = [1, 1]
    q, k, words = _words(lengths, hq, hk, d, g, True, 75, seed=25)
    T = sum(lengths)
    v = synth.fp16_normal(25, 9, (T, hk, d))
    pf = tm.TileMixPrefill(lengths, hq, hk, d, words, g, causal=True, device="cuda")
    o = pf(torch.from_numpy(q).cuda(), torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    torch.cuda.synchronize()
    assert tm.tilemix_get_error() == tm.OK
    q8, qs = oracle.quantize_q(q, lengths)
    k8, ks = oracle.quantize_k(k, lengths)
    want, _ = oracle.attention_rows(q, k, v, q8, qs, k8, ks, words, g, lengths, True)
    got = o.cpu().numpy().astype(np.float64)
    rows = oracle.all_rows(lengths, hq)          # (sequence, head, row), sequence-major
    starts = np.cumsum([0] + lengths[:-1])
    got = np.stack([got[starts[s] + i, h] for s, h, i in rows])
    mx, mn = gc.errors(got, want)
    assert mx <= gc.MAX_ABS and mn <= gc.MEAN_ABS, (mx, mn)
