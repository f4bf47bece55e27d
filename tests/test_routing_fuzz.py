"""Randomised agreement of the library's host routing code with the oracle:
random packed batches (zero-length and ragged sequences, per-sequence
grouping factors, GQA widths), every template, any coverage and seed.  The
words, the legal-group counts and the INT8-group counts must agree bit for
bit, every INT8 bit must be a legal group, and each sequence must carry
exactly floor((p N + 50) / 100) INT8 groups."""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
import synth
import tile_routed_mixed_b200 as tm


@st.composite
def batches(draw):
    lengths = draw(st.lists(st.integers(0, 3000), min_size=1, max_size=5))
    g = [max(tm.tilemix_auto_g(L), draw(st.integers(1, 3))) for L in lengths]
    return lengths, g


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(batch=batches(), template=st.sampled_from(list(tm.TEMPLATES)),
       percent=st.integers(0, 100), seed=st.integers(0, 2 ** 32 - 1),
       hk=st.integers(1, 3), causal=st.booleans())
def test_routing_builder_agrees_with_oracle(batch, template, percent, seed, hk, causal):
    lengths, g = batch
    cu = synth.cu_seqlens_of(lengths)
    m, legal, int8 = tm.tilemix_build_routing(template, percent, seed, cu, hk, g, causal)
    mo, lo, io = oracle.build_routing(template, percent, seed, lengths, hk, g, causal)
    assert np.array_equal(m, mo)
    assert np.array_equal(legal, lo) and np.array_equal(int8, io)
    row = 0
    for s, L in enumerate(lengths):
        n_rows = oracle.n_qtiles(L)
        total_int8 = 0
        for qt in range(n_rows):
            n = oracle.legal_groups(qt, L, g[s], causal)
            for kv in range(hk):
                w = int(m[row + qt, kv])
                assert w >> n == 0          # no bit past the row's legal groups
                assert w == int(m[row + qt, 0])  # one word for every KV head
            total_int8 += bin(int(m[row + qt, 0])).count("1")
        assert total_int8 == int8[s] == (percent * legal[s] + 50) // 100
        row += n_rows
