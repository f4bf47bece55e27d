"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.  Integer stages (codes, scales, INT32 tile scores) are
compared bit for bit; fp16 outputs within max-abs 2e-3 / mean-abs 2e-4."""
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
    import tile_routed_mixed_b200 as tm
    tm.lib()


def _check_out(case, got_full, want, rows, max_abs=gc.MAX_ABS, mean_abs=gc.MEAN_ABS):
    got = gc.gather(case, got_full, rows)
    assert np.isfinite(got).all()
    mx, mn = gc.errors(got, want)
    assert mx <= max_abs and mn <= mean_abs, (mx, mn)
    return mx, mn


# ------------------------------------------------------------ quantiser ---

@pytest.mark.parametrize("lengths,hq,hk,d", [([256], 1, 1, 64), ([100, 300, 1, 64], 4, 2, 128),
                                            ([4096] * 8, 24, 8, 128)])
def test_quantize_bit_exact(lengths, hq, hk, d):
    import tile_routed_mixed_b200 as tm
    case = gc.Case(lengths, hq, hk, d, outliers=4 if hk == 8 else 0)
    q, k, _ = case.inputs()
    q8o, qso = oracle.quantize_q(q, lengths)
    k8o, kso = oracle.quantize_k(k, lengths)
    cu = synth.cu_seqlens_of(lengths)
    cq, ck = tm.tilemix_tile_offsets(cu)
    dev = "cuda"
    T = sum(lengths)
    qd, kd = torch.from_numpy(q).to(dev), torch.from_numpy(k).to(dev)
    q8 = torch.zeros((T, hq, d), dtype=torch.int8, device=dev)
    k8 = torch.zeros((T, hk, d), dtype=torch.int8, device=dev)
    qs = torch.zeros((hq, int(cq[-1])), dtype=torch.float32, device=dev)
    ks = torch.zeros((hk, int(ck[-1])), dtype=torch.float32, device=dev)
    t = lambda a: torch.from_numpy(a).to(dev)
    tm.tilemix_quantize_qk(qd, kd, t(cu), t(cq), t(ck), len(lengths), T, int(cq[-1]), int(ck[-1]),
                           hq, hk, d, q8, qs, k8, ks)
    torch.cuda.synchronize()
    assert np.array_equal(q8.cpu().numpy(), q8o)
    assert np.array_equal(k8.cpu().numpy(), k8o)
    assert np.array_equal(qs.cpu().numpy().view(np.uint32), qso.view(np.uint32))
    assert np.array_equal(ks.cpu().numpy().view(np.uint32), kso.view(np.uint32))


def _near_half_integers(lengths, heads, d, block, seed):
    """fp16 values whose quotient x / s sits on or next to a half-integer, per
    block: the rounding cases where a reciprocal-multiply shortcut and the
    IEEE quotient can disagree.  One block in three has a = 127 (s = 1, so the
    ties are exact and rne must pick the even code)."""
    rng = np.random.default_rng(seed)
    T = sum(lengths)
    x = np.zeros((T, heads, d), dtype=np.float16)
    t0 = 0
    for L in lengths:
        for r0 in range(0, L, block):
            rows = min(block, L - r0)
            for h in range(heads):
                a = np.float16(127.0) if rng.integers(3) == 0 else np.float16(rng.uniform(0.05, 9.0))
                s = np.float32(np.float32(a) / np.float32(127.0))
                kk = rng.integers(-127, 127, size=(rows, d))
                tgt = ((kk + 0.5) * np.float64(s)).astype(np.float16)
                bump = rng.integers(-1, 2, size=(rows, d))
                up = np.nextafter(tgt, np.float16(np.inf))
                dn = np.nextafter(tgt, np.float16(-np.inf))
                v = np.where(bump > 0, up, np.where(bump < 0, dn, tgt))
                v = np.clip(v, -a, a)
                v[0, 0] = a
                x[t0 + r0:t0 + r0 + rows, h, :] = v
        t0 += L
    return x


@pytest.mark.parametrize("d", [64, 128])
def test_quantize_rounding_boundaries_bit_exact(d):
    import tile_routed_mixed_b200 as tm
    lengths, hq, hk = [256, 77, 130], 3, 2
    q = _near_half_integers(lengths, hq, d, 128, seed=11)
    k = _near_half_integers(lengths, hk, d, 64, seed=12)
    q8o, qso = oracle.quantize_q(q, lengths)
    k8o, kso = oracle.quantize_k(k, lengths)
    cu = synth.cu_seqlens_of(lengths)
    cq, ck = tm.tilemix_tile_offsets(cu)
    dev = "cuda"
    T = sum(lengths)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    q8 = torch.zeros((T, hq, d), dtype=torch.int8, device=dev)
    k8 = torch.zeros((T, hk, d), dtype=torch.int8, device=dev)
    qs = torch.zeros((hq, int(cq[-1])), dtype=torch.float32, device=dev)
    ks = torch.zeros((hk, int(ck[-1])), dtype=torch.float32, device=dev)
    tm.tilemix_quantize_qk(t(q), t(k), t(cu), t(cq), t(ck), len(lengths), T, int(cq[-1]),
                           int(ck[-1]), hq, hk, d, q8, qs, k8, ks)
    torch.cuda.synchronize()
    assert np.array_equal(q8.cpu().numpy(), q8o)
    assert np.array_equal(k8.cpu().numpy(), k8o)
    assert np.array_equal(qs.cpu().numpy().view(np.uint32), qso.view(np.uint32))
    assert np.array_equal(ks.cpu().numpy().view(np.uint32), kso.view(np.uint32))


# --------------------------------------------------------- INT32 scores ---

@pytest.mark.parametrize("case", [
    gc.Case([256], 1, 1, 64, template="band", percent=50, g=1),
    gc.Case([300, 130], 4, 2, 128, template="row_random", percent=75, g=2, seed=3),
    gc.Case([200], 2, 1, 64, template="sptrans", percent=100, g=1, causal=False),
], ids=["tiny", "ragged_gqa_g2", "noncausal_all_int8"])
def test_int32_tile_scores_bit_exact(case):
    q, k, v = case.inputs()
    masks = case.masks()
    out = gc.run_gpu(case, q, k, v, masks, debug=True)
    q8, _ = oracle.quantize_q(q, case.lengths)
    k8, _ = oracle.quantize_k(k, case.lengths)
    cu = np.concatenate([[0], np.cumsum(case.lengths)])
    checked = 0
    for s, L in enumerate(case.lengths):
        for h in range(case.hq):
            A = oracle.int_scores(q8, k8, masks, case.g, case.lengths, s, h, case.hq, case.hk,
                                  case.causal)
            got = out["dbg"][h, cu[s]:cu[s] + L, :L].astype(np.int64)
            legal = A != -(2 ** 62)
            assert np.array_equal(got[legal], A[legal])
            checked += int(legal.sum())
    assert checked > 0


# ------------------------------------------------------------- outputs ---

SMALL = [
    ("tiny_band50", gc.Case.workload("tiny_l256")),
    ("ragged_gqa_sptrans75", gc.Case([100, 300, 1, 513], 4, 2, 128, template="sptrans", percent=75)),
    ("ragged_d64_bigbird50", gc.Case([77, 640, 200], 2, 1, 64, template="bigbird", percent=50,
                                     seed=5)),
    ("noncausal_rowrandom25", gc.Case([200, 333], 2, 2, 128, causal=False, template="row_random",
                                      percent=25, seed=2)),
    ("g3_global75", gc.Case([1500, 700], 3, 1, 128, template="global", percent=75, g=3)),
    ("aligned_sparse_90", gc.Case([1024, 512], 6, 2, 128, template="aligned_sparse", percent=90,
                                  outliers=4)),
    ("band_0", gc.Case([1024], 2, 2, 128, template="band", percent=0)),
    ("band_100", gc.Case([1024], 2, 2, 128, template="band", percent=100)),
]


@pytest.mark.parametrize("name,case", SMALL, ids=[n for n, _ in SMALL])
def test_prefill_small_full_parity(name, case):
    q, k, v = case.inputs()
    masks = case.masks()
    out = gc.run_gpu(case, q, k, v, masks, lse=True)
    rows = oracle.all_rows(case.lengths, case.hq)
    want, lse, _ = gc.oracle_rows(case, q, k, v, masks, rows)
    _check_out(case, out["o"], want, rows)
    cu = np.concatenate([[0], np.cumsum(case.lengths)])
    got_lse = out["lse"][rows[:, 1], cu[rows[:, 0]] + rows[:, 2]]
    assert np.abs(got_lse - lse).max() < 2e-3


def test_all_fp16_and_all_int8_words():
    case = gc.Case([700, 256], 4, 2, 128, seed=8)
    q, k, v = case.inputs()
    rows = oracle.all_rows(case.lengths, case.hq)
    for words in (0, (1 << 64) - 1):
        masks = case.masks(words)
        out = gc.run_gpu(case, q, k, v, masks)
        want, _, _ = gc.oracle_rows(case, q, k, v, masks, rows)
        _check_out(case, out["o"], want, rows)


def test_illegal_entries_never_reach_outputs():
    # NaN / Inf in K and V blocks past the last legal tile of q-tile row 0 of
    # the middle sequence and in both neighbouring sequences: that row block's
    # outputs are bit-identical to the clean run.
    case = gc.Case([64, 384, 100], 2, 1, 128, template="bigbird", percent=50, routing_seed=1)
    q, k, v = case.inputs()
    masks = case.masks()
    clean = gc.run_gpu(case, q, k, v, masks)["o"]
    k2, v2 = k.copy(), v.copy()
    t0 = 64
    last = oracle.last_legal_tile(0, 384, True)
    k2[t0 + (last + 1) * 64:t0 + 384] = np.nan
    v2[t0 + (last + 1) * 64:t0 + 384] = np.inf
    k2[:t0] = np.nan
    v2[:t0] = np.nan
    k2[t0 + 384:] = np.inf
    v2[t0 + 384:] = np.nan
    dirty = gc.run_gpu(case, q, k2, v2, masks)["o"]
    blk = slice(t0, t0 + 128)
    assert np.isfinite(dirty[blk]).all()
    assert np.array_equal(dirty[blk].view(np.uint16), clean[blk].view(np.uint16))


def test_ragged_tail_keys_from_next_sequence_are_zeroed():
    # The last key tile of sequence 0 (L = 100) also holds rows of sequence 1:
    # NaN there must not leak into sequence 0 through P.V.
    case = gc.Case([100, 156], 2, 2, 64, template="band", percent=50)
    q, k, v = case.inputs()
    masks = case.masks()
    clean = gc.run_gpu(case, q, k, v, masks)["o"]
    v2 = v.copy()
    v2[100:] = np.nan
    k2 = k.copy()
    k2[100:] = np.inf
    dirty = gc.run_gpu(case, q, k2, v2, masks)["o"]
    assert np.array_equal(dirty[:100].view(np.uint16), clean[:100].view(np.uint16))


def test_gqa_head_map():
    # explicit kv_head_of_q (non-contiguous groups) and words that differ per KV head
    kv_map = [1, 0, 1, 0]
    case = gc.Case([300, 200], 4, 2, 128, kv_map=np.array(kv_map, np.int32), seed=6)
    q, k, v = case.inputs()
    tm = sum(oracle.n_qtiles(L) for L in case.lengths)
    rng = np.random.default_rng(1)
    masks = rng.integers(0, 16, size=(tm, 2), dtype=np.uint64)
    out = gc.run_gpu(case, q, k, v, masks)
    rows = oracle.all_rows(case.lengths, case.hq)
    want, _, _ = gc.oracle_rows(case, q, k, v, masks, rows)
    _check_out(case, out["o"], want, rows)


# -------------------------------------------- full workloads, sampled rows ---

# The coverage x layout sweep: every template at 25, 50 and 75% INT8.
SWEEP = [("sweep_8k_b8", dict(template=t, percent=pct))
         for t in ("band", "global", "row_random", "aligned_sparse", "bigbird", "sptrans")
         for pct in (25, 50, 75)]

WORKLOAD_RUNS = [
    ("llama3b_4k_b8", dict()),
    ("llama3b_4k_b8", dict(percent=0)),
    ("llama3b_4k_b8", dict(percent=100)),
] + SWEEP + [
    ("varlen_qwen7b", dict()),
    ("long_64k", dict()),
]


@pytest.mark.parametrize("name,over", WORKLOAD_RUNS,
                         ids=["%s-%s" % (n, "-".join("%s%s" % kv for kv in o.items()) or "default")
                              for n, o in WORKLOAD_RUNS])
def test_workload_sampled_rows(name, over):
    case = gc.Case.workload(name, **over)
    q, k, v = case.inputs()
    masks = case.masks()
    out = gc.run_gpu(case, q, k, v, masks)
    if name == "long_64k":
        rows = gc.sample_rows(case.lengths, case.hq, per_head_random=16, heads={0, 13, 31},
                              tiles_per_head=64)
    elif name == "varlen_qwen7b":
        rows = gc.sample_rows(case.lengths, case.hq, per_head_random=16, heads={0, 9, 27})
    elif name == "sweep_8k_b8":
        rows = gc.sample_rows(case.lengths, case.hq, per_head_random=16, heads={0, 11, 23})
    else:
        rows = gc.sample_rows(case.lengths, case.hq, per_head_random=32)
    want, _, _ = gc.oracle_rows(case, q, k, v, masks, rows)
    _check_out(case, out["o"], want, rows)


# ------------------------------------------------------ packed batches ---

def test_zero_length_sequences_in_a_batch():
    # Empty sequences hold no tiles, rows or words; the device's sequence
    # lookups skip them.  Full parity on every row, and the host-buffer call
    # (runs of whole sequences, some of them empty) equals the device call.
    import tile_routed_mixed_b200 as tm
    case = gc.Case([0, 300, 0, 0, 129, 0], 4, 2, 128, template="sptrans", percent=75, seed=12)
    q, k, v = case.inputs()
    masks = case.masks()
    out = gc.run_gpu(case, q, k, v, masks, lse=True)
    rows = oracle.all_rows(case.lengths, case.hq)
    want, lse, _ = gc.oracle_rows(case, q, k, v, masks, rows)
    _check_out(case, out["o"], want, rows)
    cu = np.concatenate([[0], np.cumsum(case.lengths)])
    assert np.abs(out["lse"][rows[:, 1], cu[rows[:, 0]] + rows[:, 2]] - lse).max() < 2e-3
    pf = tm.TileMixPrefill(case.lengths, case.hq, case.hk, case.d, masks, case.g)
    qh, kh, vh = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
    for chunks in (1, 3, 6):
        oh = torch.full(q.shape, float("nan"), dtype=torch.float16).pin_memory()
        qd, kd, vd = (torch.empty(x.shape, dtype=torch.float16, device="cuda") for x in (q, k, v))
        od = torch.empty(q.shape, dtype=torch.float16, device="cuda")
        pf.from_host(qh, kh, vh, oh, qd, kd, vd, od, chunks=chunks)
        torch.cuda.current_stream().synchronize()
        assert tm.tilemix_get_error() == tm.OK
        assert np.array_equal(oh.numpy().view(np.uint16), out["o"].view(np.uint16))


def test_head_map_entry_out_of_range_is_reported_and_skipped():
    # Query head 2 names KV head 2 of 2: its work items are skipped (its O
    # rows stay as they were) and the status word reports INVALID_ARG; the
    # other heads are computed as usual.
    import tile_routed_mixed_b200 as tm
    kv_map = np.array([0, 1, 2, 1], dtype=np.int32)
    good_map = np.array([0, 1, 0, 1], dtype=np.int32)
    case = gc.Case([300, 200], 4, 2, 128, kv_map=good_map, seed=13)
    q, k, v = case.inputs()
    masks = case.masks()
    pf = tm.TileMixPrefill(case.lengths, case.hq, case.hk, case.d, masks, case.g,
                           kv_head_of_q=kv_map)
    qd, kd, vd = (torch.from_numpy(x).cuda() for x in (q, k, v))
    od = torch.full_like(qd, float("nan"))
    pf(qd, kd, vd, od)
    assert tm.tilemix_get_error() == tm.ERR_INVALID_ARG
    assert tm.tilemix_get_error() == tm.OK
    got = od.cpu().numpy()
    assert np.isnan(got[:, 2]).all()
    rows = oracle.all_rows(case.lengths, case.hq)
    rows = rows[rows[:, 1] != 2]
    want, _, _ = gc.oracle_rows(case, q, k, v, masks, rows)
    _check_out(case, got, want, rows)


# ------------------------------------------------------------- failures ---

def test_bounded_wait_expires_and_is_reported():
    # a barrier nothing signals: the wait gives up after 50 ms, the status
    # word reports TIMEOUT once, and the context still runs the kernel
    import tile_routed_mixed_b200 as tm
    tm.tilemix_selftest_wait_timeout(50)
    assert tm.tilemix_get_error() == tm.ERR_TIMEOUT
    assert tm.tilemix_get_error() == tm.OK
    case = gc.Case([200], 2, 1, 64, template="band", percent=50)
    q, k, v = case.inputs()
    masks = case.masks()
    out = gc.run_gpu(case, q, k, v, masks)
    rows = oracle.all_rows(case.lengths, case.hq)
    want, _, _ = gc.oracle_rows(case, q, k, v, masks, rows)
    _check_out(case, out["o"], want, rows)
    with pytest.raises(tm.TileMixError):
        tm.tilemix_selftest_wait_timeout(0)


def test_row_with_too_many_groups_is_reported():
    # g = 1 on an 8192-token sequence needs 128 groups per row: the device
    # rejects the rows it cannot encode and reports INVALID_ARG
    import tile_routed_mixed_b200 as tm
    case = gc.Case([8192], 1, 1, 64, template="band", percent=0, g=2)
    q, k, v = case.inputs()
    masks = case.masks()
    bad = gc.Case([8192], 1, 1, 64, template="band", percent=0, g=1)
    with pytest.raises(tm.TileMixError) as e:
        gc.run_gpu(bad, q, k, v, masks)
    assert e.value.status == tm.ERR_INVALID_ARG
    assert tm.tilemix_get_error() == tm.OK
