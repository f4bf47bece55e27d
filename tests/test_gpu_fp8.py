"""GPU parity of the FP8 (e4m3) low path with the oracle: the e4m3 codes and
scales bit for bit (tilemix_quantize_qk_fp8), and prefill with FP8 low tiles
within max-abs 2e-3 / mean-abs 2e-4 of the oracle's FP8 reading."""
import numpy as np
import pytest

import oracle
from oracle import fp8 as of8
from tests import gpu_cases as gc

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gc.set_test_timeout()


@pytest.mark.parametrize("d,outliers", [(128, 0), (64, 4), (128, 4)])
def test_fp8_codes_bit_exact(d, outliers):
    import tile_routed_mixed_b200 as tm
    case = gc.Case([1, 63, 64, 65, 129, 1000], 6, 2, d, outliers=outliers, seed=41)
    q, k, _ = case.inputs()
    cu = np.concatenate([[0], np.cumsum(case.lengths)]).astype(np.int32)
    cq, ck = oracle.tile_offsets(case.lengths)
    T = case.total_tokens
    dev = "cuda"
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    q8 = torch.zeros((T, 6, d), dtype=torch.uint8, device=dev)
    k8 = torch.zeros((T, 2, d), dtype=torch.uint8, device=dev)
    qs = torch.zeros((6, int(cq[-1])), dtype=torch.float32, device=dev)
    ks = torch.zeros((2, int(ck[-1])), dtype=torch.float32, device=dev)
    tm.tilemix_quantize_qk_fp8(t(q), t(k), t(cu), t(cq), t(ck), len(case.lengths), T, int(cq[-1]),
                               int(ck[-1]), 6, 2, d, q8, qs, k8, ks)
    torch.cuda.synchronize()
    wq8, wqs = of8.quantize_q_fp8(q, case.lengths)
    wk8, wks = of8.quantize_k_fp8(k, case.lengths)
    assert np.array_equal(q8.cpu().numpy(), wq8)
    assert np.array_equal(k8.cpu().numpy(), wk8)
    assert np.array_equal(qs.cpu().numpy().view(np.uint32), wqs.view(np.uint32))
    assert np.array_equal(ks.cpu().numpy().view(np.uint32), wks.view(np.uint32))


def _prefill_fp8(case, rows=None, words=None):
    import tile_routed_mixed_b200 as tm
    q, k, v = case.inputs()
    masks = case.masks(words)
    pf = tm.TileMixPrefill(case.lengths, case.hq, case.hk, case.d, masks, case.g,
                           causal=case.causal, kv_head_of_q=case.kv_map, low="fp8")
    qd, kd, vd = (torch.from_numpy(x).cuda() for x in (q, k, v))
    od = torch.full_like(qd, float("nan"))
    pf(qd, kd, vd, od)
    assert tm.tilemix_get_error() == tm.OK
    if rows is None:
        rows = oracle.all_rows(case.lengths, case.hq)
    q8, qs = of8.quantize_q_fp8(q, case.lengths)
    k8, ks = of8.quantize_k_fp8(k, case.lengths)
    want, _ = oracle.attention_rows(q, k, v, q8, qs, k8, ks, masks, case.g, case.lengths,
                                    case.causal, kv_map=case.kv_map, rows=rows, low="fp8")
    got = gc.gather(case, od.cpu().numpy(), rows)
    assert np.all(np.isfinite(got))
    mx, mn = gc.errors(got, want)
    assert mx <= gc.MAX_ABS and mn <= gc.MEAN_ABS, (mx, mn)
    return mx, mn


def test_fp8_prefill_ragged_sptrans():
    _prefill_fp8(gc.Case([1, 65, 300, 1000], 6, 2, 128, template="sptrans", percent=75, seed=42))


def test_fp8_prefill_all_fp8_d64_gqa4():
    _prefill_fp8(gc.Case([129, 640, 33], 4, 1, 64, seed=43), words=(1 << 64) - 1)


def test_fp8_prefill_bigbird_g2_outliers_noncausal():
    _prefill_fp8(gc.Case([700, 1100], 8, 2, 128, causal=False, template="bigbird", percent=50,
                         g=2, outliers=4, seed=44))


def test_fp8_prefill_benchmark_shape_sampled():
    case = gc.Case.workload("llama3b_4k_b8")
    rows = gc.sample_rows(case.lengths, case.hq, seed=5, per_head_random=8, heads=(0, 13, 23),
                          tiles_per_head=8)
    _prefill_fp8(case, rows=rows)


def test_fp8_and_int8_paths_differ_on_the_same_words():
    """The flag reaches the kernel: all-low words give different outputs."""
    import tile_routed_mixed_b200 as tm
    case = gc.Case([300], 2, 1, 128, seed=45)
    q, k, v = case.inputs()
    masks = case.masks((1 << 64) - 1)
    outs = []
    for low in ("int8", "fp8"):
        pf = tm.TileMixPrefill(case.lengths, 2, 1, 128, masks, case.g, low=low)
        qd, kd, vd = (torch.from_numpy(x).cuda() for x in (q, k, v))
        outs.append(pf(qd, kd, vd).cpu().numpy().astype(np.float64))
    assert np.max(np.abs(outs[0] - outs[1])) > 1e-3


def test_fp8_zero_length_sequences_and_custom_head_map():
    # the FP8 flag with empty sequences in a packed batch and a
    # non-contiguous head map
    case = gc.Case([0, 300, 0, 129, 0], 4, 2, 128, template="bigbird", percent=50,
                   kv_map=np.array([1, 0, 1, 0], dtype=np.int32), outliers=4, seed=46)
    _prefill_fp8(case)
