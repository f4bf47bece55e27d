"""The C-ABI library: load, exported symbols, host-side helpers against the
oracle, and synchronous argument checks.  No GPU needed (no device calls)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import synth
import tile_routed_mixed_b200 as tm
from tile_routed_mixed_b200 import build as tmbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    tmbuild.build()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "tilemix.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tilemix_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert "tilemix_prefill_fwd" in names and len(names) >= 9
    L = ctypes.CDLL(tm.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    assert tm.tilemix_version() == 1
    assert tm.status_string(tm.ERR_TIMEOUT) == "device wait timed out"


def test_auto_g_and_offsets_match_oracle():
    for L in (0, 1, 63, 64, 65, 4096, 4097, 8192, 12096, 16384, 65536, 65537):
        assert tm.tilemix_auto_g(L) == oracle.auto_g(L)
    lengths = [100, 0, 256, 64, 4097]
    cu = synth.cu_seqlens_of(lengths)
    cq, ck = tm.tilemix_tile_offsets(cu)
    oq, ok = oracle.tile_offsets(lengths)
    assert np.array_equal(cq, oq) and np.array_equal(ck, ok)


def _geometries():
    out = []
    for name in synth.WORKLOADS:
        w = synth.WORKLOADS[name]
        lengths = synth.workload_lengths(name)
        g = ([oracle.auto_g(L) for L in lengths] if w["g"] == "auto"
             else [int(w["g"])] * len(lengths))
        out.append((name, lengths, g, True))
    out.append(("ragged", [100, 300, 1, 513, 2000], [1, 1, 1, 1, 1], True))
    out.append(("ragged_noncausal", [100, 300, 513], [1, 1, 1], False))
    out.append(("g3", [5000, 3000], [3, 2], True))
    # zero-length sequences have no query-tile rows and so no words
    out.append(("empty_seqs", [0, 300, 0, 64, 0], [1, 1, 1, 1, 1], True))
    out.append(("only_empty", [0, 0], [1, 1], True))
    return out


@pytest.mark.parametrize("geom", _geometries(), ids=lambda g: g[0])
@pytest.mark.parametrize("template", list(tm.TEMPLATES))
def test_routing_builder_bit_exact_vs_oracle(geom, template):
    _, lengths, g, causal = geom
    cu = synth.cu_seqlens_of(lengths)
    for p in (0, 10, 25, 50, 75, 90, 100):
        for seed in (0, 12345):
            m, legal, int8 = tm.tilemix_build_routing(template, p, seed, cu, 3, g, causal)
            mo, lo, io = oracle.build_routing(template, p, seed, lengths, 3, g, causal)
            assert np.array_equal(m, mo), (template, p, seed)
            assert np.array_equal(legal, lo) and np.array_equal(int8, io)


@pytest.mark.parametrize("fname,template,percent,L", [
    ("sptrans_l640_p75.txt", "sptrans", 75, 640),
    ("sptrans_l1024_p50.txt", "sptrans", 50, 1024),
    ("aligned_sparse_l1024_p25.txt", "aligned_sparse", 25, 1024),
    ("aligned_sparse_l1024_p30.txt", "aligned_sparse", 30, 1024),
    ("row_random_l640_p50_seed0.txt", "row_random", 50, 640),
    ("bigbird_l640_p50_seed0.txt", "bigbird", 50, 640),
    ("band_tiny_l256.txt", "band", 50, 256),
], ids=lambda x: str(x))
def test_routing_builder_hand_golden(fname, template, percent, L):
    # the library's host builder against the hand-derived words directly
    with open(os.path.join(ROOT, "tests", "golden", fname)) as f:
        want = [int(x, 16) for x in f if x.strip() and not x.startswith("#")]
    m, _, _ = tm.tilemix_build_routing(template, percent, 0, synth.cu_seqlens_of([L]), 1, [1],
                                       True)
    assert [int(x) for x in m[:, 0]] == want


def test_routing_builder_rejects_bad_arguments():
    cu = synth.cu_seqlens_of([8192])
    with pytest.raises(tm.TileMixError) as e:
        tm.tilemix_build_routing("band", 50, 0, cu, 1, [1], True)   # 128 groups in a row
    assert e.value.status == tm.ERR_INVALID_ARG
    for bad in (-1, 101):
        with pytest.raises(tm.TileMixError):
            tm.tilemix_build_routing("band", bad, 0, cu, 1, [2], True)
    with pytest.raises(tm.TileMixError):
        tm.tilemix_build_routing(7, 50, 0, cu, 1, [2], True)
    with pytest.raises(tm.TileMixError):
        tm.tilemix_build_routing("band", 50, 0, cu, 0, [2], True)
    with pytest.raises(tm.TileMixError):
        tm.tilemix_build_routing("band", 50, 0, cu, 1, [0], True)
    L = tm.lib()
    assert L.tilemix_auto_g(-1, ctypes.byref(ctypes.c_int())) == tm.ERR_INVALID_ARG
    assert L.tilemix_auto_g(5, None) == tm.ERR_INVALID_ARG
    bad_cu = np.array([0, 10, 5], dtype=np.int32)
    q = np.zeros(3, np.int32)
    assert L.tilemix_tile_offsets(bad_cu.ctypes.data, 2, q.ctypes.data, q.ctypes.data) == \
        tm.ERR_INVALID_ARG


def _fake_args(**over):
    a = tm.PrefillArgs()
    a.q = a.k = a.v = a.o = 4096
    a.cu_seqlens = a.cu_qtiles = a.cu_ktiles = a.masks = a.g = 4096
    a.nseq, a.total_tokens, a.total_qtiles, a.total_ktiles, a.max_seqlen = 1, 256, 2, 4, 256
    a.hq, a.hk, a.d = 4, 2, 128
    a.causal = 1
    for k, v in over.items():
        setattr(a, k, v)
    return a


def test_prefill_argument_checks_are_synchronous():
    L = tm.lib()
    n = ctypes.c_size_t(0)
    assert L.tilemix_workspace_size(ctypes.byref(_fake_args()), ctypes.byref(n)) == tm.OK
    # q8 [256*4*128] + q scales [4*2 floats] + k8 [256*2*128] + k scales, each 256-aligned,
    # + 256 bytes for the fused kernel's work-item ticket
    assert n.value == 131072 + 256 + 65536 + 256 + 256
    assert L.tilemix_workspace_size(ctypes.byref(_fake_args(k_i8=4096, k_scale=4096)),
                                    ctypes.byref(n)) == tm.OK
    assert n.value == 131072 + 256 + 256
    cases = [
        (dict(d=96), tm.ERR_UNSUPPORTED),
        (dict(low_format=3), tm.ERR_INVALID_ARG),
        (dict(low_format=-1), tm.ERR_INVALID_ARG),
        (dict(low_format=1, debug_int32_scores=4096), tm.ERR_UNSUPPORTED),
        (dict(hq=3, hk=2), tm.ERR_INVALID_ARG),
        (dict(hk=0), tm.ERR_INVALID_ARG),
        (dict(causal=2), tm.ERR_INVALID_ARG),
        (dict(q=None), tm.ERR_INVALID_ARG),
        (dict(masks=None), tm.ERR_INVALID_ARG),
        (dict(q=4100), tm.ERR_INVALID_ARG),            # not 16-byte aligned
        (dict(k_i8=4096), tm.ERR_INVALID_ARG),         # codes without scales
        (dict(softmax_scale=-1.0), tm.ERR_INVALID_ARG),
        (dict(max_seqlen=0), tm.ERR_INVALID_ARG),
        (dict(), tm.ERR_WORKSPACE),                    # no workspace given
        (dict(workspace=4096, workspace_bytes=10), tm.ERR_WORKSPACE),
        (dict(workspace=4100, workspace_bytes=1 << 30), tm.ERR_WORKSPACE),
    ]
    for over, want in cases:
        assert L.tilemix_prefill_fwd(ctypes.byref(_fake_args(**over)), None) == want, over
    # empty batches are a no-op
    assert L.tilemix_prefill_fwd(ctypes.byref(_fake_args(nseq=0)), None) == tm.OK
    assert L.tilemix_quantize_qk(None, None, None, None, None, 0, 0, 0, 0, 1, 1, 128, None, None,
                                 None, None, None) == tm.OK
    assert L.tilemix_quantize_qk(None, None, None, None, None, 1, 10, 1, 1, 1, 1, 80, None,
                                 None, None, None, None) == tm.ERR_UNSUPPORTED


def test_prefill_host_argument_checks_are_synchronous():
    """tilemix_prefill_host validates everything it reads on the host before
    it enqueues anything (no device is touched by these calls)."""
    L = tm.lib()
    cu = np.array([0, 100, 256], dtype=np.int32)   # 2 sequences: 1 + 2 query tiles, 2 + 3 key tiles
    events = (ctypes.c_void_p * 7)(*([4096] * 7))

    def host(cu_arr=cu, **over):
        h = tm.PrefillHostArgs()
        h.dev = _fake_args(nseq=2, total_qtiles=3, total_ktiles=5, workspace=4096,
                           workspace_bytes=1 << 30)
        h.cu_seqlens_h = cu_arr.ctypes.data
        h.q_h = h.k_h = h.v_h = h.o_h = 8192
        h.chunks = 2
        h.stream_in = h.stream_out = 16
        h.events = ctypes.cast(events, ctypes.c_void_p).value
        for k, v in over.items():
            if k.startswith("dev_"):
                setattr(h.dev, k[4:], v)
            else:
                setattr(h, k, v)
        return h

    assert L.tilemix_prefill_host(None, None) == tm.ERR_INVALID_ARG
    cases = [
        (dict(dev_d=96), tm.ERR_UNSUPPORTED),           # the device arguments' own checks
        (dict(dev_q=None), tm.ERR_INVALID_ARG),
        (dict(q_h=None), tm.ERR_INVALID_ARG),
        (dict(o_h=None), tm.ERR_INVALID_ARG),
        (dict(stream_in=None), tm.ERR_INVALID_ARG),
        (dict(events=None), tm.ERR_INVALID_ARG),
        (dict(chunks=0), tm.ERR_INVALID_ARG),
        (dict(chunks=(1 << 20) + 1), tm.ERR_INVALID_ARG),  # 3 * chunks + 1 events must fit
        (dict(after_previous=2), tm.ERR_INVALID_ARG),
        (dict(cu_seqlens_h=None), tm.ERR_INVALID_ARG),
        (dict(dev_total_qtiles=4), tm.ERR_INVALID_ARG),  # disagrees with the host offsets
        (dict(dev_total_ktiles=4), tm.ERR_INVALID_ARG),
        (dict(dev_max_seqlen=155), tm.ERR_INVALID_ARG),  # shorter than sequence 1 (156)
        (dict(dev_workspace=None), tm.ERR_WORKSPACE),
    ]
    for over, want in cases:
        assert L.tilemix_prefill_host(ctypes.byref(host(**over)), None) == want, over
    bad = np.array([0, 300, 256], dtype=np.int32)    # decreasing offsets
    assert L.tilemix_prefill_host(ctypes.byref(host(bad)), None) == tm.ERR_INVALID_ARG
    short = np.array([0, 100, 200], dtype=np.int32)  # ends before total_tokens
    assert L.tilemix_prefill_host(ctypes.byref(host(short)), None) == tm.ERR_INVALID_ARG
    # an empty batch is a no-op
    assert L.tilemix_prefill_host(ctypes.byref(host(dev_nseq=0)), None) == tm.OK


def _runs_reference(lengths, chunks):
    """The host-buffer call's cut rule restated: with n = min(chunks, nseq),
    run c ends before the first sequence whose start offset reaches
    (c + 1) / n of the tokens; the last run takes the rest."""
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    nseq = len(lengths)
    n = min(chunks, nseq)
    starts, s0 = [0], 0
    for c in range(n):
        if s0 >= nseq:
            break
        s1 = s0 + 1
        while s1 < nseq and (c == n - 1 or cu[s1] < cu[-1] * (c + 1) // n):
            s1 += 1
        starts.append(s1)
        s0 = s1
    return starts


@pytest.mark.parametrize("lengths,chunks", [
    ([4096] * 8, 8), ([4096] * 8, 3), ([4096] * 8, 16), ([100, 1, 3000, 7, 7, 512], 4),
    ([5000, 10, 10, 10], 2), ([1], 5), ([0, 0, 64, 0], 3), ([300, 1, 777, 128, 197], 3),
])
def test_host_runs_cut_rule(lengths, chunks):
    starts = tm.tilemix_host_runs(np.concatenate([[0], np.cumsum(lengths)]), chunks)
    assert list(starts) == _runs_reference(lengths, chunks)
    # every sequence in exactly one run, in order, no empty run
    assert starts[0] == 0 and starts[-1] == len(lengths)
    assert all(b > a for a, b in zip(starts[:-1], starts[1:]))
    assert len(starts) - 1 <= min(chunks, len(lengths))


def test_host_runs_equal_sequences_split_evenly():
    starts = tm.tilemix_host_runs(np.arange(0, 8 * 4096 + 1, 4096), 4)
    assert list(starts) == [0, 2, 4, 6, 8]


def test_host_runs_rejects_bad_arguments():
    L = tm.lib()
    cu = np.array([0, 10, 5], dtype=np.int32)   # decreasing
    out = np.zeros(4, dtype=np.int32)
    n = ctypes.c_int(0)
    assert L.tilemix_host_runs(cu.ctypes.data, 2, 2, out.ctypes.data, ctypes.byref(n)) == \
        tm.ERR_INVALID_ARG
    ok = np.array([0, 10, 15], dtype=np.int32)
    assert L.tilemix_host_runs(ok.ctypes.data, 2, 0, out.ctypes.data, ctypes.byref(n)) == \
        tm.ERR_INVALID_ARG
    assert L.tilemix_host_runs(None, 2, 2, out.ctypes.data, ctypes.byref(n)) == tm.ERR_INVALID_ARG


def _fake_decode(**over):
    a = tm.DecodeArgs()
    for f in ("q", "k", "v", "k_i8", "k_scale", "o", "seq_start", "seq_len", "ktile_start",
              "qtile_start", "masks", "g"):
        setattr(a, f, 4096)
    a.nseq, a.max_seqlen, a.total_ktiles, a.cache_rows = 2, 300, 10, 600
    a.hq, a.hk, a.d = 6, 2, 128
    for k, v in over.items():
        setattr(a, k, v)
    return a


def test_decode_argument_checks_are_synchronous():
    L = tm.lib()
    n = ctypes.c_size_t(0)
    assert L.tilemix_decode_workspace_size(ctypes.byref(_fake_decode()), ctypes.byref(n)) == tm.OK
    assert n.value > 0
    cases = [
        (dict(d=80), tm.ERR_UNSUPPORTED),
        (dict(hq=6, hk=4), tm.ERR_INVALID_ARG),
        (dict(hq=34, hk=2), tm.ERR_UNSUPPORTED),        # 17 query heads per KV head
        (dict(max_seqlen=0), tm.ERR_INVALID_ARG),
        (dict(nseq=-1), tm.ERR_INVALID_ARG),
        (dict(k_i8=None), tm.ERR_INVALID_ARG),
        (dict(q=4097), tm.ERR_INVALID_ARG),             # misaligned
        (dict(softmax_scale=-1.0), tm.ERR_INVALID_ARG),
        (dict(tiles_per_split=-1), tm.ERR_INVALID_ARG),
        (dict(cache_rows=0), tm.ERR_INVALID_ARG),
        (dict(workspace=None), tm.ERR_WORKSPACE),
        (dict(workspace=4096 + 128, workspace_bytes=1 << 30), tm.ERR_WORKSPACE),  # misaligned
    ]
    for over, want in cases:
        assert L.tilemix_decode_fwd(ctypes.byref(_fake_decode(**over)), None) == want, over
    # nothing to do: OK without touching any pointer
    assert L.tilemix_decode_fwd(ctypes.byref(_fake_decode(nseq=0, q=None)), None) == tm.OK


def _fake_route(cu, g, **over):
    a = tm.RouteArgs()
    for f in ("q", "k", "cu_seqlens", "cu_qtiles", "cu_ktiles", "g", "masks"):
        setattr(a, f, 4096)
    a.cu_seqlens_h = cu.ctypes.data_as(ctypes.c_void_p)
    a.g_h = g.ctypes.data_as(ctypes.c_void_p)
    a.nseq, a.hq, a.hk, a.d, a.causal, a.int8_percent = len(g), 6, 2, 128, 1, 50
    for k, v in over.items():
        setattr(a, k, v)
    return a


def test_route_argument_checks_are_synchronous():
    """Every argument error of tilemix_route_pooled returns before any launch
    (fake device pointers; nothing is dereferenced on these paths)."""
    L = ctypes.CDLL(tm.LIB_PATH)
    L.tilemix_route_pooled.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    L.tilemix_route_workspace_size.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    cu = np.array([0, 300, 1300], dtype=np.int32)
    g = np.array([1, 1], dtype=np.int32)
    n = ctypes.c_size_t(0)
    assert L.tilemix_route_workspace_size(ctypes.byref(_fake_route(cu, g)), ctypes.byref(n)) == tm.OK
    # 3 + 8 query tiles and 5 + 16 key tiles, 2 KV heads, d 128, fp32 means
    assert n.value == (11 * 2 * 128 * 4 + 255) // 256 * 256 + (21 * 2 * 128 * 4 + 255) // 256 * 256
    long_seq = np.array([0, 64 * 64 + 1], dtype=np.int32)   # 65 groups at g = 1
    cases = [
        (dict(d=80), tm.ERR_UNSUPPORTED),
        (dict(int8_percent=101), tm.ERR_INVALID_ARG),
        (dict(int8_percent=-1), tm.ERR_INVALID_ARG),
        (dict(causal=2), tm.ERR_INVALID_ARG),
        (dict(hq=6, hk=4), tm.ERR_INVALID_ARG),
        (dict(hq=600, hk=2), tm.ERR_UNSUPPORTED),
        (dict(q=None), tm.ERR_INVALID_ARG),
        (dict(k=4100), tm.ERR_INVALID_ARG),            # misaligned
        (dict(masks=4100), tm.ERR_INVALID_ARG),        # not 8-byte aligned
        (dict(cu_seqlens_h=None), tm.ERR_INVALID_ARG),
        (dict(workspace=None), tm.ERR_WORKSPACE),
        (dict(workspace=4096 + 64, workspace_bytes=1 << 30), tm.ERR_WORKSPACE),
    ]
    for over, want in cases:
        assert L.tilemix_route_pooled(ctypes.byref(_fake_route(cu, g, **over)), None) == want, over
    bad_g = np.array([1, 0], dtype=np.int32)
    assert L.tilemix_route_pooled(ctypes.byref(_fake_route(cu, bad_g)), None) == tm.ERR_INVALID_ARG
    one = np.array([1], dtype=np.int32)
    assert L.tilemix_route_pooled(ctypes.byref(_fake_route(long_seq, one)), None) == tm.ERR_INVALID_ARG
    two = np.array([2], dtype=np.int32)                    # g = 2 brings it to 33 groups
    a = _fake_route(long_seq, two, workspace=None)
    assert L.tilemix_route_pooled(ctypes.byref(a), None) == tm.ERR_WORKSPACE
    dec = np.array([0, 300, 200], dtype=np.int32)          # decreasing offsets
    assert L.tilemix_route_pooled(ctypes.byref(_fake_route(dec, g)), None) == tm.ERR_INVALID_ARG
    empty = np.array([0], dtype=np.int32)
    a = _fake_route(empty, np.zeros(0, np.int32), q=None, k=None)
    a.nseq = 0
    assert L.tilemix_route_pooled(ctypes.byref(a), None) == tm.OK


def test_mass_probe_argument_checks_are_synchronous():
    L = ctypes.CDLL(tm.LIB_PATH)
    L.tilemix_mass_probe.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    cu = np.array([0, 300, 1300], dtype=np.int32)
    g = np.array([1, 1], dtype=np.int32)

    def fake(**over):
        a = tm.MassArgs()
        for f in ("q", "k", "cu_seqlens", "cu_qtiles", "cu_ktiles", "g", "masks", "m8", "h", "h8"):
            setattr(a, f, 4096)
        a.cu_seqlens_h = cu.ctypes.data_as(ctypes.c_void_p)
        a.g_h = g.ctypes.data_as(ctypes.c_void_p)
        a.nseq, a.hq, a.hk, a.d, a.causal, a.delta_log2 = 2, 6, 2, 128, 1, 4.0
        for k, v in over.items():
            setattr(a, k, v)
        return a

    cases = [
        (dict(d=96), tm.ERR_UNSUPPORTED),
        (dict(delta_log2=0.0), tm.ERR_INVALID_ARG),
        (dict(delta_log2=float("inf")), tm.ERR_INVALID_ARG),
        (dict(delta_log2=float("nan")), tm.ERR_INVALID_ARG),
        (dict(softmax_scale=-1.0), tm.ERR_INVALID_ARG),
        (dict(causal=3), tm.ERR_INVALID_ARG),
        (dict(hq=5, hk=2), tm.ERR_INVALID_ARG),
        (dict(h8=None), tm.ERR_INVALID_ARG),
        (dict(q=4104), tm.ERR_INVALID_ARG),
        (dict(g_h=None), tm.ERR_INVALID_ARG),
    ]
    for over, want in cases:
        assert L.tilemix_mass_probe(ctypes.byref(fake(**over)), None) == want, over
    long_seq = np.array([0, 64 * 64 + 1], dtype=np.int32)
    one = np.array([1], dtype=np.int32)
    a = fake(nseq=1)
    a.cu_seqlens_h = long_seq.ctypes.data_as(ctypes.c_void_p)
    a.g_h = one.ctypes.data_as(ctypes.c_void_p)
    assert L.tilemix_mass_probe(ctypes.byref(a), None) == tm.ERR_INVALID_ARG   # 65 groups
    empty = np.array([0, 0], dtype=np.int32)
    a = fake(nseq=1, q=None, k=None)
    a.cu_seqlens_h = empty.ctypes.data_as(ctypes.c_void_p)
    a.g_h = one.ctypes.data_as(ctypes.c_void_p)
    assert L.tilemix_mass_probe(ctypes.byref(a), None) == tm.OK                # nothing to do


def test_plain_c_program_against_the_header(tmp_path):
    """tests/abi_check.c, compiled as C99 with gcc against include/tilemix.h and
    linked to the library: the ABI needs no Python and no C++ on the caller's
    side (host entry points and argument checks only; no GPU is touched)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(tm.LIB_PATH)
    exe = str(tmp_path / "abi_check")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-O1",
                           "-I" + os.path.join(root, "include"),
                           os.path.join(root, "tests", "abi_check.c"), "-L" + libdir, "-ltilemix",
                           "-Wl,-rpath," + libdir, "-o", exe])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
