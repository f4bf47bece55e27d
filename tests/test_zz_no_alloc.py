"""tilemix_prefill_fwd_noalloc: the entry point for callers that cannot call
cudaMalloc (for example inside a host application that owns all device memory
through its own pool, or on a latency-critical path where an allocation may
synchronise the device).  It keeps its INT8 scratch in a fixed 64 MiB array
inside the library instead of a caller workspace.

Collected last on purpose, so that a run stopping at the first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest

from tests import gpu_cases as gc

torch = pytest.importorskip("torch")


def _lib():
    import tile_routed_mixed_b200 as tm
    return tm


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


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gc.set_test_timeout()
    tm = _lib()
    dev = "cuda"
    stream = torch.cuda.current_stream()
    outs = []
    # two calls in a row on different inputs: the shared scratch keeps the
    # previous call's contents, which must not leak into the next result
    for case in (gc.Case([300, 1000, 77], 6, 2, 128, template="sptrans", percent=75, seed=3),
                 gc.Case([512, 200], 4, 4, 64, template="bigbird", percent=50, seed=4)):
        q, k, v = case.inputs()
        masks = case.masks()
        pf = tm.TileMixPrefill(case.lengths, case.hq, case.hk, case.d, masks, case.g,
                               device=dev)
        qd, kd, vd = (torch.from_numpy(x).to(dev) for x in (q, k, v))
        ref = pf(qd, kd, vd)  # existing entry point, caller workspace
        need = tm.tilemix_workspace_size(pf.args(qd, kd, vd, ref))
        assert need <= tm.NOALLOC_SCRATCH_BYTES
        o = torch.full_like(qd, float("nan"))
        args = pf.args(qd, kd, vd, o)
        args.workspace = None
        args.workspace_bytes = 0
        rc = tm.lib().tilemix_prefill_fwd_noalloc(ctypes.byref(args),
                                                   ctypes.c_void_p(stream.cuda_stream))
        assert rc == tm.OK
        assert tm.tilemix_get_error() == tm.OK
        got = o.cpu().numpy().astype(np.float64)
        want = ref.cpu().numpy().astype(np.float64)
        mx, mn = gc.errors(got, want)
        assert np.isfinite(got).all()
        assert mx <= gc.MAX_ABS and mn <= gc.MEAN_ABS, (mx, mn)
        outs.append(mx)
    assert len(outs) == 2
