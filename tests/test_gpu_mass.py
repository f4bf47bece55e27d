"""GPU parity of the importance-mass exposure probe (tilemix_mass_probe) with
the fp64 oracle: per (head, token) INT8 mass m8 within 1e-3, and the
high-importance sums h, h8 within 1e-3 of the oracle's bounds over the
memberships of keys whose score lies within 1e-3 (natural-log units) of the
selection threshold (an fp32 score can fall on either side of it).

Tolerance: the fractions are sums of fp32 exponentials of fp32 scores; the
scores' error is below 1e-4 here (d <= 128 products of fp16 values, fp32
accumulation) and the sums' relative error below L * 2^-24 < 1e-3 for
L <= 16384."""
import numpy as np
import pytest

import oracle
from oracle import mass as om
import synth
from tests import gpu_cases as gc

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 1e-3
BAND = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gc.set_test_timeout()


def _run(lengths, hq, hk, d, template, percent, g, causal, seed, kv_map=None, outliers=0,
         lowrank=0, delta=4.0):
    import tile_routed_mixed_b200 as tm
    T = sum(lengths)
    q, k, _ = synth.make_qkv(seed, T, hq, hk, d, outliers=outliers, lowrank=lowrank)
    masks, _, _ = oracle.build_routing(template, percent, seed, lengths, hk, g, causal)
    m8, h, h8 = tm.mass_probe(torch.from_numpy(q).cuda(), torch.from_numpy(k).cuda(), masks,
                              lengths, hq, hk, g, causal=causal, delta_log2=delta,
                              kv_head_of_q=kv_map)
    torch.cuda.synchronize()
    assert tm.tilemix_get_error() == tm.OK
    want = om.probe_rows(q, k, masks, g, lengths, causal, delta=delta, kv_map=kv_map, band=BAND)
    m8, h, h8 = (x.cpu().numpy().astype(np.float64) for x in (m8, h, h8))
    assert np.all(np.isfinite(m8)) and np.all(np.isfinite(h)) and np.all(np.isfinite(h8))
    assert np.max(np.abs(m8 - want["m8"])) <= TOL
    assert np.all(h >= want["h_lo"] - TOL) and np.all(h <= want["h_hi"] + TOL)
    assert np.all(h8 >= want["h8_lo"] - TOL) and np.all(h8 <= want["h8_hi"] + TOL)
    return om.exposure(h, h8), om.exposure(want["h"], want["h8"])


def test_mass_probe_ragged_sptrans():
    got, want = _run([1, 65, 300, 1000], 4, 2, 128, "sptrans", 25, [1, 1, 1, 1], True, seed=31)
    assert abs(got - want) <= TOL


def test_mass_probe_noncausal_d64_bigbird_g2():
    _run([700, 129], 4, 1, 64, "bigbird", 50, [2, 1], False, seed=32)


def test_mass_probe_head_map_and_peaked_inputs():
    kv_map = np.array([1, 0, 0, 1], dtype=np.int32)
    _run([513, 900], 4, 2, 128, "row_random", 75, [1, 1], True, seed=33, kv_map=kv_map,
         lowrank=16)


def test_mass_probe_outliers_and_delta():
    _run([2048], 6, 2, 128, "band", 50, [1], True, seed=34, outliers=4, delta=1.0)
