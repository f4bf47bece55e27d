"""CPU checks of the work counts behind bench.py's roofline figures: the
algorithmic FLOPs and bytes are recomputed by brute force over every legal
(query, key) pair, or from closed forms, so that a miscount in the bench's
tile-level bookkeeping fails here."""
import numpy as np
import pytest

import bench
import oracle


def _brute_prefill(lengths, hq, hk, d, masks, g, causal, kv_map=None):
    """FP16 FLOPs and INT8 ops, pair by pair: QK 2d in the routed precision,
    PV 2d in FP16, for every legal pair of every query head."""
    f16 = i8 = 0
    cq = 0
    for s, L in enumerate(lengths):
        for h in range(hq):
            kv = h // (hq // hk)
            for i in range(L):
                w = int(masks[cq + i // 128, kv])
                for j in range(i + 1 if causal else L):
                    if (w >> ((j // 64) // g[s])) & 1:
                        i8 += 2 * d
                    else:
                        f16 += 2 * d
                    f16 += 2 * d
        cq += (L + 127) // 128
    return f16, i8


@pytest.mark.parametrize("lengths,hq,hk,g,causal,template,percent", [
    ([200], 2, 1, [1], True, "sptrans", 75),
    ([129, 64, 300], 4, 2, [1, 1, 2], True, "bigbird", 50),
    ([190, 70], 3, 3, [2, 1], False, "band", 40),
])
def test_prefill_work_matches_pair_brute_force(lengths, hq, hk, g, causal, template, percent):
    masks = oracle.build_routing(template, percent, 3, lengths, hk, g, causal)[0]
    d = 16  # counts scale with d; a small d keeps the brute force fast
    f16, i8, nbytes = bench.algorithmic_work(lengths, hq, hk, d, masks, g, causal)
    bf16, bi8 = _brute_prefill(lengths, hq, hk, d, masks, g, causal)
    assert (f16, i8) == (bf16, bi8)
    T = sum(lengths)
    assert nbytes == T * (2 * hq + 2 * hk) * d * 2


def test_prefill_work_closed_form_at_the_benchmark_shape():
    """8 x 4096, 24 query heads, d 128, causal: every legal pair costs 4d
    operations whatever its precision, and there are L (L + 1) / 2 of them."""
    lengths, hq, hk, d = [4096] * 8, 24, 8, 128
    g = [1] * 8
    masks = oracle.build_routing("sptrans", 75, 0, lengths, hk, g, True)[0]
    f16, i8, nbytes = bench.algorithmic_work(lengths, hq, hk, d, masks, g, True)
    assert f16 + i8 == 8 * hq * (4096 * 4097 // 2) * 4 * d
    assert nbytes == 8 * 4096 * (2 * hq + 2 * hk) * d * 2
    # INT8 covers 0.75 of the legal groups, not of the pairs: the FP16 groups
    # under SpTrans include the diagonal ones, which are only partly legal, so
    # the INT8 share of the QK pairs is a little above 0.75
    assert 0.75 < i8 / (f16 + i8) * 2 < 0.8


@pytest.mark.parametrize("L,causal", [(1, True), (63, True), (64, True), (200, True), (200, False),
                                      (4096, True)])
def test_legal_pairs_tiles_sum_to_the_pair_count(L, causal):
    p = bench.legal_pairs(L, causal)
    assert p.shape == ((L + 127) // 128, (L + 63) // 64)
    assert int(p.sum()) == (L * (L + 1) // 2 if causal else L * L)
    assert (p >= 0).all() and (p <= 128 * 64).all()


def test_decode_bytes_by_brute_force():
    lengths, hq, hk, d = [70, 200, 1], 4, 2, 32
    g = np.array([1, 2, 1], dtype=np.int32)
    masks = oracle.build_routing("sptrans", 75, 0, lengths, hk, g, True)[0]
    step, attn = bench.decode_bytes(lengths, hq, hk, d, masks, g)
    keys = values = requant = 0
    cq = 0
    for s, L in enumerate(lengths):
        t = L - 1
        for kv in range(hk):
            w = int(masks[cq + t // 128, kv])
            for j in range(L):
                keys += d * (1 if (w >> ((j // 64) // int(g[s]))) & 1 else 2)
                values += 2 * d
            requant += (L - 64 * (t // 64)) * d * 3  # the new key's block: fp16 in, codes out
        cq += (L + 127) // 128
    q_rows = len(lengths) * hq * d
    assert attn == keys + values + q_rows * 3                      # query fp16 + codes
    assert step == keys + values + requant + q_rows * 2 * 2       # query in, O out


def test_mass_flops_closed_form():
    # causal: 64-row block b scores tiles 0..b, so sum_b (b + 1) tiles of 64 x 64 per sweep
    L, hq, d = 4096, 24, 128
    nb = L // 64
    tiles = nb * (nb + 1) // 2
    assert bench.mass_flops([L], hq, d, True) == 2 * hq * tiles * 64 * 64 * 2 * d
    assert bench.mass_flops([L], hq, d, False) == 2 * hq * nb * nb * 64 * 64 * 2 * d


def test_workload_seqs_keeps_the_first_sequences():
    # --seqs N: the first N sequences of a configuration, with their own
    # grouping factors (the small cases the profiler captures run)
    import synth
    for name in synth.WORKLOADS:
        w, lengths, g = bench.workload(name)
        for n in (1, 2):
            w2, l2, g2 = bench.workload(name, seqs=n)
            assert l2 == lengths[:n] and g2 == g[:n]
            assert (w2["hq"], w2["hk"], w2["d"], w2["template"]) == (w["hq"], w["hk"], w["d"],
                                                                      w["template"])
        assert bench.workload(name, seqs=None)[1] == lengths
