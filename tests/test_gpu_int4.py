"""GPU parity of the INT4 low path with the oracle: the INT4 codes (in [-7, 7],
one per byte) and scales bit for bit (tilemix_quantize_qk_int4), the INT32
tile scores of INT4-routed tiles bit for bit, and prefill with INT4 low tiles
within max-abs 2e-3 / mean-abs 2e-4 of the oracle fed the same codes."""
import numpy as np
import pytest

import oracle
from tests import gpu_cases as gc

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gc.set_test_timeout()


@pytest.mark.parametrize("lengths,hq,hk,d,outliers", [
    ([1, 63, 64, 65, 129, 1000], 6, 2, 128, 0),
    ([1, 63, 64, 65, 129, 1000], 6, 2, 64, 4),
    ([4096] * 8, 24, 8, 128, 4),
])
def test_int4_codes_bit_exact(lengths, hq, hk, d, outliers):
    import tile_routed_mixed_b200 as tm
    case = gc.Case(lengths, hq, hk, d, outliers=outliers, seed=51)
    q, k, _ = case.inputs()
    cu = np.concatenate([[0], np.cumsum(case.lengths)]).astype(np.int32)
    cq, ck = oracle.tile_offsets(case.lengths)
    T = case.total_tokens
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    q4 = torch.zeros((T, hq, d), dtype=torch.int8, device="cuda")
    k4 = torch.zeros((T, hk, d), dtype=torch.int8, device="cuda")
    qs = torch.zeros((hq, int(cq[-1])), dtype=torch.float32, device="cuda")
    ks = torch.zeros((hk, int(ck[-1])), dtype=torch.float32, device="cuda")
    tm.tilemix_quantize_qk_int4(t(q), t(k), t(cu), t(cq), t(ck), len(lengths), T, int(cq[-1]),
                                int(ck[-1]), hq, hk, d, q4, qs, k4, ks)
    torch.cuda.synchronize()
    wq4, wqs = oracle.quantize_q_int4(q, lengths)
    wk4, wks = oracle.quantize_k_int4(k, lengths)
    assert np.array_equal(q4.cpu().numpy(), wq4)
    assert np.array_equal(k4.cpu().numpy(), wk4)
    assert np.array_equal(qs.cpu().numpy().view(np.uint32), wqs.view(np.uint32))
    assert np.array_equal(ks.cpu().numpy().view(np.uint32), wks.view(np.uint32))
    assert int(q4.abs().max()) == 7


def test_int4_rounding_ties_bit_exact():
    # values on and next to the half-integers of x / s: one K block whose
    # absmax is 7 (scale 1) and one whose absmax is 3.5 (scale 0.5)
    import tile_routed_mixed_b200 as tm
    d = 64
    x = np.zeros((128, 1, d), dtype=np.float16)
    ties = np.array([-6.5, -5.5, -4.5, -3.5, -2.5, -1.5, -0.5, 0.5, 1.5, 2.5, 3.5, 4.5, 5.5, 6.5],
                    dtype=np.float64)
    x[0, 0, :ties.size] = ties
    x[1, 0, :ties.size] = np.nextafter(ties.astype(np.float16), np.float16(np.inf))
    x[2, 0, :ties.size] = np.nextafter(ties.astype(np.float16), np.float16(-np.inf))
    x[3, 0, 0] = 7.0
    x[64:67, 0, :ties.size] = (x[0:3, 0, :ties.size].astype(np.float32) * 0.5).astype(np.float16)
    x[67, 0, 0] = 3.5
    lengths = [128]
    cu = np.array([0, 128], dtype=np.int32)
    cq, ck = oracle.tile_offsets(lengths)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    k4 = torch.zeros((128, 1, d), dtype=torch.int8, device="cuda")
    ks = torch.zeros((1, int(ck[-1])), dtype=torch.float32, device="cuda")
    q4 = torch.zeros((128, 1, d), dtype=torch.int8, device="cuda")
    qs = torch.zeros((1, int(cq[-1])), dtype=torch.float32, device="cuda")
    tm.tilemix_quantize_qk_int4(t(x), t(x), t(cu), t(cq), t(ck), 1, 128, int(cq[-1]), int(ck[-1]),
                                1, 1, d, q4, qs, k4, ks)
    torch.cuda.synchronize()
    wk4, wks = oracle.quantize_k_int4(x, lengths)
    wq4, wqs = oracle.quantize_q_int4(x, lengths)
    assert np.array_equal(k4.cpu().numpy(), wk4) and np.array_equal(q4.cpu().numpy(), wq4)
    assert np.array_equal(ks.cpu().numpy().view(np.uint32), wks.view(np.uint32))
    assert list(wk4[0, 0, :ties.size]) == [-6, -6, -4, -4, -2, -2, 0, 0, 2, 2, 4, 4, 6, 6]


def _prefill_int4(case, rows=None, words=None, debug=False):
    import tile_routed_mixed_b200 as tm
    q, k, v = case.inputs()
    masks = case.masks(words)
    pf = tm.TileMixPrefill(case.lengths, case.hq, case.hk, case.d, masks, case.g,
                           causal=case.causal, kv_head_of_q=case.kv_map, low="int4")
    qd, kd, vd = (torch.from_numpy(x).cuda() for x in (q, k, v))
    od = torch.full_like(qd, float("nan"))
    dbg = None
    if debug:
        cols = (max(case.lengths) + 63) // 64 * 64
        dbg = torch.full((case.hq, case.total_tokens, cols), -(2 ** 31), dtype=torch.int32,
                         device="cuda")
    pf(qd, kd, vd, od, debug_int32_scores=dbg)
    torch.cuda.synchronize()
    assert tm.tilemix_get_error() == tm.OK
    if rows is None:
        rows = oracle.all_rows(case.lengths, case.hq)
    q4, qs = oracle.quantize_q_int4(q, case.lengths)
    k4, ks = oracle.quantize_k_int4(k, case.lengths)
    want, _ = oracle.attention_rows(q, k, v, q4, qs, k4, ks, masks, case.g, case.lengths,
                                    case.causal, kv_map=case.kv_map, rows=rows)
    got = gc.gather(case, od.cpu().numpy(), rows)
    assert np.all(np.isfinite(got))
    mx, mn = gc.errors(got, want)
    assert mx <= gc.MAX_ABS and mn <= gc.MEAN_ABS, (mx, mn)
    if debug:
        dump = dbg.cpu().numpy()
        cu = np.concatenate([[0], np.cumsum(case.lengths)])
        checked = 0
        for s, L in enumerate(case.lengths):
            for h in range(case.hq):
                A = oracle.int_scores(q4, k4, masks, case.g, case.lengths, s, h, case.hq, case.hk,
                                      case.causal, kv_map=case.kv_map)
                legal = A > -(2 ** 62)
                got_s = dump[h, cu[s]:cu[s] + L, :L].astype(np.int64)
                assert np.array_equal(got_s[legal], A[legal])
                checked += int(legal.sum())
        assert checked > 0
    return mx, mn


def test_int4_prefill_ragged_sptrans_int32_scores():
    _prefill_int4(gc.Case([1, 65, 300, 513], 4, 2, 128, template="sptrans", percent=75, seed=52),
                  debug=True)


def test_int4_prefill_all_int4_d64_gqa4():
    _prefill_int4(gc.Case([129, 640, 33], 4, 1, 64, seed=53), words=(1 << 64) - 1)


def test_int4_prefill_bigbird_g2_outliers_noncausal():
    _prefill_int4(gc.Case([700, 1100], 8, 2, 128, causal=False, template="bigbird", percent=50,
                          g=2, outliers=4, seed=54))


def test_int4_prefill_benchmark_shape_sampled():
    case = gc.Case.workload("llama3b_4k_b8")
    rows = gc.sample_rows(case.lengths, case.hq, seed=6, per_head_random=8, heads=(0, 13, 23),
                          tiles_per_head=8)
    _prefill_int4(case, rows=rows)


def test_int4_and_int8_paths_differ_on_the_same_words():
    """The flag reaches the quantiser: all-low words give different outputs."""
    import tile_routed_mixed_b200 as tm
    case = gc.Case([300], 2, 1, 128, seed=55)
    q, k, v = case.inputs()
    masks = case.masks((1 << 64) - 1)
    outs = []
    for low in ("int8", "int4"):
        pf = tm.TileMixPrefill(case.lengths, 2, 1, 128, masks, case.g, low=low)
        qd, kd, vd = (torch.from_numpy(x).cuda() for x in (q, k, v))
        outs.append(pf(qd, kd, vd).cpu().numpy().astype(np.float64))
    assert np.max(np.abs(outs[0] - outs[1])) > 1e-3


def test_int4_zero_length_sequences_custom_head_map_and_host_call():
    # the INT4 flag through the remaining entry shapes: empty sequences in a
    # packed batch, a non-contiguous head map, and the host-buffer call in
    # runs of whole sequences (bit-equal to the device call)
    import tile_routed_mixed_b200 as tm
    kv_map = np.array([1, 0, 1, 0], dtype=np.int32)
    case = gc.Case([0, 300, 0, 129, 0, 77], 4, 2, 128, template="sptrans", percent=75,
                   kv_map=kv_map, outliers=4, seed=56)
    q, k, v = case.inputs()
    masks = case.masks()
    pf = tm.TileMixPrefill(case.lengths, 4, 2, 128, masks, case.g, kv_head_of_q=kv_map,
                           low="int4")
    qd, kd, vd = (torch.from_numpy(x).cuda() for x in (q, k, v))
    od = torch.full_like(qd, float("nan"))
    pf(qd, kd, vd, od)
    torch.cuda.synchronize()
    assert tm.tilemix_get_error() == tm.OK
    dev = od.cpu().numpy()
    rows = oracle.all_rows(case.lengths, case.hq)
    q4, qs = oracle.quantize_q_int4(q, case.lengths)
    k4, ks = oracle.quantize_k_int4(k, case.lengths)
    want, _ = oracle.attention_rows(q, k, v, q4, qs, k4, ks, masks, case.g, case.lengths,
                                    case.causal, kv_map=kv_map, rows=rows)
    mx, mn = gc.errors(gc.gather(case, dev, rows), want)
    assert mx <= gc.MAX_ABS and mn <= gc.MEAN_ABS, (mx, mn)
    qh, kh, vh = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
    for chunks in (1, 4):
        oh = torch.full(q.shape, float("nan"), dtype=torch.float16).pin_memory()
        qd2, kd2, vd2 = (torch.empty(x.shape, dtype=torch.float16, device="cuda") for x in (q, k, v))
        od2 = torch.empty(q.shape, dtype=torch.float16, device="cuda")
        pf.from_host(qh, kh, vh, oh, qd2, kd2, vd2, od2, chunks=chunks)
        torch.cuda.current_stream().synchronize()
        assert tm.tilemix_get_error() == tm.OK
        assert np.array_equal(oh.numpy().view(np.uint16), dev.view(np.uint16))
