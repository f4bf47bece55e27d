"""tilemix_prefill_fwd_noalloc: the entry point for callers that cannot call
cudaMalloc (for example inside a host application that owns all device memory
through its own pool, or on a latency-critical path where an allocation may
synchronise the device).  It keeps its INT8 scratch in a fixed 64 MiB array
inside the library instead of a caller workspace, and runs the same kernels
as tilemix_prefill_fwd, so its outputs must equal that entry point's bit for
bit.

Collected last on purpose, so that a run stopping at the first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest

import oracle
from tests import gpu_cases as gc

torch = pytest.importorskip("torch")

LIMIT = 64 << 20


def _lib():
    import tile_routed_mixed_b200 as tm
    return tm


def _fake_args(tm, total_tokens):
    # Pointers that are never dereferenced: every call below returns before
    # any launch, or runs only where there is no CUDA device.
    a = tm.PrefillArgs()
    a.q = a.k = a.v = a.o = 4096
    a.cu_seqlens = a.cu_qtiles = a.cu_ktiles = a.masks = a.g = 4096
    a.k_i8 = a.k_scale = 4096  # caller-supplied K codes: the scratch holds Q only
    a.nseq, a.total_tokens, a.max_seqlen = 1, total_tokens, total_tokens
    a.total_qtiles, a.total_ktiles = 64, 64
    a.hq, a.hk, a.d, a.causal = 1, 1, 64, 1
    return a


def test_rejects_inputs_beyond_its_scratch():
    # host-side check only: nothing is launched for an oversized request
    tm = _lib()
    a = tm.PrefillArgs()
    a.q = a.k = a.v = a.o = 4096
    a.cu_seqlens = a.cu_qtiles = a.cu_ktiles = a.masks = a.g = 4096
    a.nseq, a.total_tokens, a.max_seqlen = 1, 1 << 20, 1 << 20
    a.total_qtiles, a.total_ktiles = 1 << 13, 1 << 14
    a.hq, a.hk, a.d, a.causal = 8, 8, 128, 1
    rc = tm.lib().tilemix_prefill_fwd_noalloc(ctypes.byref(a), None)
    assert rc == tm.ERR_TOO_LARGE
    assert "64 MiB" in tm.status_string(rc)


def test_limit_is_exact_to_the_byte():
    # Workspace pieces (Q codes, Q scales, work counter) sized to fill the
    # scratch exactly: 64 * T + 4 * 64 (one 256-byte piece) + 256 = 2^26.
    tm = _lib()
    t_at = (LIMIT - 512) // 64
    at = _fake_args(tm, t_at)
    assert tm.tilemix_workspace_size(at) == LIMIT
    over = _fake_args(tm, t_at + 4)  # 256 bytes more
    assert tm.tilemix_workspace_size(over) == LIMIT + 256
    assert tm.lib().tilemix_prefill_fwd_noalloc(ctypes.byref(over), None) == tm.ERR_TOO_LARGE
    if torch.cuda.is_available():
        pytest.skip("the at-limit call would launch on the fake pointers")
    # accepted by the size check; with no CUDA device the scratch lookup fails
    rc = tm.lib().tilemix_prefill_fwd_noalloc(ctypes.byref(at), None)
    assert rc == tm.ERR_CUDA


def _noalloc(tm, pf, qd, kd, vd, stream, **kw):
    o = torch.full_like(qd, float("nan"))
    args = pf.args(qd, kd, vd, o, **kw)
    args.workspace = None
    args.workspace_bytes = 0
    rc = tm.lib().tilemix_prefill_fwd_noalloc(ctypes.byref(args),
                                               ctypes.c_void_p(stream.cuda_stream))
    assert rc == tm.OK
    assert tm.tilemix_get_error() == tm.OK
    return o


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gc.set_test_timeout()
    tm = _lib()
    dev = "cuda"
    stream = torch.cuda.current_stream()
    # calls in a row on different inputs: the shared scratch keeps the
    # previous call's contents, which must not leak into the next result; the
    # third passes its own K codes, so the scratch holds only Q's
    cases = [gc.Case([300, 1000, 77], 6, 2, 128, template="sptrans", percent=75, seed=3),
             gc.Case([512, 200], 4, 4, 64, template="bigbird", percent=50, seed=4),
             gc.Case([640, 129], 4, 2, 128, template="row_random", percent=25, seed=5)]
    for i, case in enumerate(cases):
        q, k, v = case.inputs()
        masks = case.masks()
        pf = tm.TileMixPrefill(case.lengths, case.hq, case.hk, case.d, masks, case.g,
                               device=dev)
        qd, kd, vd = (torch.from_numpy(x).to(dev) for x in (q, k, v))
        kw = {}
        if i == 2:
            T = case.total_tokens
            k8 = torch.zeros((T, case.hk, case.d), dtype=torch.int8, device=dev)
            ks = torch.zeros((case.hk, pf.total_ktiles), dtype=torch.float32, device=dev)
            tm.tilemix_quantize_qk(None, kd, pf.cu_seqlens, pf.cu_qtiles, pf.cu_ktiles, pf.nseq,
                                   T, pf.total_qtiles, pf.total_ktiles, case.hq, case.hk,
                                   case.d, None, None, k8, ks)
            kw = dict(k_i8=k8, k_scale=ks)
        ref = pf(qd, kd, vd, **kw)  # existing entry point, caller workspace
        need = tm.tilemix_workspace_size(pf.args(qd, kd, vd, ref, **kw))
        assert need <= tm.NOALLOC_SCRATCH_BYTES
        got = _noalloc(tm, pf, qd, kd, vd, stream, **kw)
        # same kernels on the same inputs: identical bits
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
        rows = oracle.all_rows(case.lengths, case.hq)
        want, _, _ = gc.oracle_rows(case, q, k, v, masks, rows)
        mx, mn = gc.errors(gc.gather(case, got.cpu().numpy(), rows), want)
        assert mx <= gc.MAX_ABS and mn <= gc.MEAN_ABS, (mx, mn)
