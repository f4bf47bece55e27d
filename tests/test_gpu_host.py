"""GPU: prefill from host buffers (tilemix_prefill_host), the batch cut into
runs of whole sequences whose uploads, kernels and downloads overlap.  Every
output row is computed exactly as by tilemix_prefill_fwd on device buffers, so
the two are compared bit for bit, and the host result against the oracle
(fp16 max-abs 2e-3 / mean-abs 2e-4)."""
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
    import tile_routed_mixed_b200 as tm
    tm.lib()


CASES = [
    ("ragged5_d128", gc.Case([300, 1, 777, 128, 197], 6, 2, 128, template="sptrans",
                             percent=75, outliers=4)),
    ("ragged4_d64", gc.Case([64, 513, 90, 1000], 4, 4, 64, template="band", percent=50)),
]


def _host_run(case, q, k, v, masks, chunks, repeat=1):
    import tile_routed_mixed_b200 as tm
    pf = tm.TileMixPrefill(case.lengths, case.hq, case.hk, case.d, masks, case.g,
                           causal=case.causal, kv_head_of_q=case.kv_map)
    qh, kh, vh = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
    oh = torch.full(q.shape, float("nan"), dtype=torch.float16).pin_memory()
    qd, kd, vd = (torch.empty(x.shape, dtype=torch.float16, device="cuda") for x in (q, k, v))
    od = torch.empty(q.shape, dtype=torch.float16, device="cuda")
    for _ in range(repeat):
        pf.from_host(qh, kh, vh, oh, qd, kd, vd, od, chunks=chunks)
    torch.cuda.current_stream().synchronize()
    rc = tm.tilemix_get_error()
    if rc != tm.OK:
        raise tm.TileMixError(rc, "device status")
    return oh.numpy().copy()


@pytest.mark.parametrize("name,case", CASES, ids=[n for n, _ in CASES])
@pytest.mark.parametrize("chunks", [1, 3, 16])
def test_host_prefill_equals_device_call_and_oracle(name, case, chunks):
    q, k, v = case.inputs()
    masks = case.masks()
    want_dev = gc.run_gpu(case, q, k, v, masks)["o"]
    got = _host_run(case, q, k, v, masks, chunks)
    assert np.array_equal(got.view(np.uint16), want_dev.view(np.uint16))
    rows = oracle.all_rows(case.lengths, case.hq)
    want, _, _ = gc.oracle_rows(case, q, k, v, masks, rows)
    mx, mn = gc.errors(gc.gather(case, got, rows), want)
    assert mx <= gc.MAX_ABS and mn <= gc.MEAN_ABS, (mx, mn)


def test_host_prefill_back_to_back_calls():
    """Calls enqueued back to back reuse the same device rows: each call's
    uploads wait for the previous call's kernels and downloads."""
    case = CASES[0][1]
    q, k, v = case.inputs()
    masks = case.masks()
    want = gc.run_gpu(case, q, k, v, masks)["o"]
    got = _host_run(case, q, k, v, masks, chunks=4, repeat=3)
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


def test_host_prefill_chained_calls_keep_each_batch():
    """Calls chained with after_previous reuse the device rows while the
    previous batch is still in flight: each batch's uploads wait only for the
    previous batch's kernels of the same run.  Three different batches, each
    downloaded into its own host buffer, must each equal its own device
    result."""
    import tile_routed_mixed_b200 as tm
    case = CASES[0][1]
    masks = case.masks()
    batches = []
    for seed in (11, 12, 13):
        c = gc.Case(case.lengths, case.hq, case.hk, case.d, template=case.template,
                    percent=case.percent, outliers=case.outliers, seed=seed)
        q, k, v = c.inputs()
        batches.append((q, k, v, gc.run_gpu(c, q, k, v, masks)["o"]))
    pf = tm.TileMixPrefill(case.lengths, case.hq, case.hk, case.d, masks, case.g,
                           causal=case.causal)
    shape_q, shape_k = batches[0][0].shape, batches[0][1].shape
    qd = torch.empty(shape_q, dtype=torch.float16, device="cuda")
    kd = torch.empty(shape_k, dtype=torch.float16, device="cuda")
    vd = torch.empty(shape_k, dtype=torch.float16, device="cuda")
    od = torch.empty(shape_q, dtype=torch.float16, device="cuda")
    hosts = []
    for i, (q, k, v, _) in enumerate(batches):
        qh, kh, vh = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
        oh = torch.full(shape_q, float("nan"), dtype=torch.float16).pin_memory()
        hosts.append((qh, kh, vh, oh))
        pf.from_host(qh, kh, vh, oh, qd, kd, vd, od, chunks=3, after_previous=i > 0)
    torch.cuda.current_stream().synchronize()
    assert tm.tilemix_get_error() == tm.OK
    for (_, _, _, want), (_, _, _, oh) in zip(batches, hosts):
        assert np.array_equal(oh.numpy().view(np.uint16), want.view(np.uint16))


def test_host_prefill_workload_equals_device_call():
    """The 4k x b8 benchmark workload (one sequence per run), bit for bit
    against the device-buffer call."""
    case = gc.Case.workload("llama3b_4k_b8")
    q, k, v = case.inputs()
    masks = case.masks()
    want = gc.run_gpu(case, q, k, v, masks)["o"]
    got = _host_run(case, q, k, v, masks, chunks=8)
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


def test_host_prefill_fp8_lse_and_head_map_equal_device_call():
    """The FP8 low path, the LSE output (left on the device) and a custom
    query-to-KV head map go through the host-buffer call unchanged."""
    import tile_routed_mixed_b200 as tm
    case = gc.Case([77, 640, 129, 300], 4, 2, 128, template="bigbird", percent=60, seed=5,
                   kv_map=[1, 0, 0, 1])
    q, k, v = case.inputs()
    masks = case.masks()
    pf = tm.TileMixPrefill(case.lengths, case.hq, case.hk, case.d, masks, case.g,
                           causal=case.causal, kv_head_of_q=case.kv_map, low="fp8")
    qd, kd, vd = (torch.from_numpy(x).cuda() for x in (q, k, v))
    od = torch.empty_like(qd)
    lse_dev = torch.zeros((case.hq, case.total_tokens), dtype=torch.float32, device="cuda")
    pf(qd, kd, vd, od, lse=lse_dev)
    torch.cuda.synchronize()
    want_o, want_lse = od.cpu().numpy(), lse_dev.cpu().numpy()
    qh, kh, vh = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
    oh = torch.full(q.shape, float("nan"), dtype=torch.float16).pin_memory()
    q2, k2, v2, o2 = (torch.empty_like(x) for x in (qd, kd, vd, od))
    lse2 = torch.zeros_like(lse_dev)
    pf.from_host(qh, kh, vh, oh, q2, k2, v2, o2, chunks=3, lse=lse2)
    torch.cuda.current_stream().synchronize()
    assert tm.tilemix_get_error() == tm.OK
    assert np.array_equal(oh.numpy().view(np.uint16), want_o.view(np.uint16))
    assert np.array_equal(lse2.cpu().numpy().view(np.uint32), want_lse.view(np.uint32))
