"""Python binding of libtilemix.so: tile-routed FP16/INT8 causal prefill
attention for B200 (sm_100a).

Argument marshalling only: every step of the attention path runs in the CUDA
library.  PyTorch supplies device memory and streams.  If the library is
missing this module raises on first use; there is no fallback.

Names mirror the C ABI of ``include/tilemix.h``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtilemix.so")

BLOCK_M = 128
BLOCK_N = 64
MAX_GROUPS = 64

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE, ERR_TOO_LARGE = range(7)
NOALLOC_SCRATCH_BYTES = 64 << 20
TEMPLATES = {"band": 0, "global": 1, "row_random": 2, "aligned_sparse": 3, "bigbird": 4,
             "sptrans": 5}


class TileMixError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (what, status_string(status), status))


class PrefillArgs(ctypes.Structure):
    """Mirror of ``tilemix_prefill_args``."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("cu_seqlens", ctypes.c_void_p), ("cu_qtiles", ctypes.c_void_p),
        ("cu_ktiles", ctypes.c_void_p),
        ("nseq", ctypes.c_int), ("total_tokens", ctypes.c_int), ("total_qtiles", ctypes.c_int),
        ("total_ktiles", ctypes.c_int), ("max_seqlen", ctypes.c_int),
        ("hq", ctypes.c_int), ("hk", ctypes.c_int), ("d", ctypes.c_int),
        ("kv_head_of_q", ctypes.c_void_p), ("masks", ctypes.c_void_p), ("g", ctypes.c_void_p),
        ("causal", ctypes.c_int), ("softmax_scale", ctypes.c_float),
        ("k_i8", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("debug_int32_scores", ctypes.c_void_p),
        ("event_kernel_begin", ctypes.c_void_p), ("event_kernel_end", ctypes.c_void_p),
        ("low_format", ctypes.c_int),
    ]


LOW_FORMATS = {"int8": 0, "fp8": 1, "int4": 2}


class PrefillHostArgs(ctypes.Structure):
    """Mirror of ``tilemix_prefill_host_args``."""
    _fields_ = [
        ("dev", PrefillArgs), ("cu_seqlens_h", ctypes.c_void_p),
        ("q_h", ctypes.c_void_p), ("k_h", ctypes.c_void_p), ("v_h", ctypes.c_void_p),
        ("o_h", ctypes.c_void_p), ("chunks", ctypes.c_int),
        ("stream_in", ctypes.c_void_p), ("stream_out", ctypes.c_void_p),
        ("events", ctypes.c_void_p), ("after_previous", ctypes.c_int),
    ]


class DecodeArgs(ctypes.Structure):
    """Mirror of ``tilemix_decode_args``."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("k_i8", ctypes.c_void_p), ("k_scale", ctypes.c_void_p), ("o", ctypes.c_void_p),
        ("seq_start", ctypes.c_void_p), ("seq_len", ctypes.c_void_p),
        ("ktile_start", ctypes.c_void_p), ("qtile_start", ctypes.c_void_p),
        ("masks", ctypes.c_void_p), ("g", ctypes.c_void_p), ("kv_head_of_q", ctypes.c_void_p),
        ("nseq", ctypes.c_int), ("max_seqlen", ctypes.c_int), ("total_ktiles", ctypes.c_int),
        ("cache_rows", ctypes.c_int),
        ("hq", ctypes.c_int), ("hk", ctypes.c_int), ("d", ctypes.c_int),
        ("softmax_scale", ctypes.c_float), ("tiles_per_split", ctypes.c_int),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("event_kernel_begin", ctypes.c_void_p), ("event_kernel_end", ctypes.c_void_p),
    ]


class RouteArgs(ctypes.Structure):
    """Mirror of ``tilemix_route_args``."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p),
        ("cu_seqlens_h", ctypes.c_void_p), ("g_h", ctypes.c_void_p),
        ("cu_seqlens", ctypes.c_void_p), ("cu_qtiles", ctypes.c_void_p),
        ("cu_ktiles", ctypes.c_void_p), ("g", ctypes.c_void_p), ("kv_head_of_q", ctypes.c_void_p),
        ("nseq", ctypes.c_int), ("hq", ctypes.c_int), ("hk", ctypes.c_int), ("d", ctypes.c_int),
        ("causal", ctypes.c_int), ("int8_percent", ctypes.c_int),
        ("masks", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("event_begin", ctypes.c_void_p), ("event_end", ctypes.c_void_p),
    ]


class MassArgs(ctypes.Structure):
    """Mirror of ``tilemix_mass_args``."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p),
        ("cu_seqlens_h", ctypes.c_void_p), ("g_h", ctypes.c_void_p),
        ("cu_seqlens", ctypes.c_void_p), ("cu_qtiles", ctypes.c_void_p),
        ("cu_ktiles", ctypes.c_void_p), ("g", ctypes.c_void_p), ("masks", ctypes.c_void_p),
        ("kv_head_of_q", ctypes.c_void_p),
        ("nseq", ctypes.c_int), ("hq", ctypes.c_int), ("hk", ctypes.c_int), ("d", ctypes.c_int),
        ("causal", ctypes.c_int), ("softmax_scale", ctypes.c_float),
        ("delta_log2", ctypes.c_float),
        ("m8", ctypes.c_void_p), ("h", ctypes.c_void_p), ("h8", ctypes.c_void_p),
        ("event_begin", ctypes.c_void_p), ("event_end", ctypes.c_void_p),
    ]


_lib = None


def lib():
    """The loaded library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libtilemix.so is missing at %s: run "
                              "`python -m tile_routed_mixed_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        P, I = ctypes.c_void_p, ctypes.c_int
        L.tilemix_version.restype = I
        L.tilemix_status_string.restype = ctypes.c_char_p
        L.tilemix_status_string.argtypes = [I]
        L.tilemix_auto_g.restype = I
        L.tilemix_auto_g.argtypes = [I, P]
        L.tilemix_tile_offsets.restype = I
        L.tilemix_tile_offsets.argtypes = [P, I, P, P]
        L.tilemix_host_runs.restype = I
        L.tilemix_host_runs.argtypes = [P, I, I, P, P]
        L.tilemix_build_routing.restype = I
        L.tilemix_build_routing.argtypes = [I, I, ctypes.c_uint64, P, I, I, P, I, P, P, P]
        L.tilemix_quantize_qk.restype = I
        L.tilemix_quantize_qk.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, P, P]
        L.tilemix_quantize_qk_fp8.restype = I
        L.tilemix_quantize_qk_fp8.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, P, P]
        L.tilemix_quantize_qk_int4.restype = I
        L.tilemix_quantize_qk_int4.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, P, P]
        L.tilemix_workspace_size.restype = I
        L.tilemix_workspace_size.argtypes = [ctypes.POINTER(PrefillArgs),
                                             ctypes.POINTER(ctypes.c_size_t)]
        L.tilemix_prefill_fwd.restype = I
        L.tilemix_prefill_fwd.argtypes = [ctypes.POINTER(PrefillArgs), P]
        L.tilemix_prefill_fwd_noalloc.restype = I
        L.tilemix_prefill_fwd_noalloc.argtypes = [ctypes.POINTER(PrefillArgs), P]
        L.tilemix_prefill_host.restype = I
        L.tilemix_prefill_host.argtypes = [ctypes.POINTER(PrefillHostArgs), P]
        L.tilemix_mma_rate.restype = I
        L.tilemix_mma_rate.argtypes = [I, I, I, I, P, P]
        L.tilemix_decode_workspace_size.restype = I
        L.tilemix_decode_workspace_size.argtypes = [ctypes.POINTER(DecodeArgs),
                                                    ctypes.POINTER(ctypes.c_size_t)]
        L.tilemix_decode_fwd.restype = I
        L.tilemix_decode_fwd.argtypes = [ctypes.POINTER(DecodeArgs), P]
        L.tilemix_route_workspace_size.restype = I
        L.tilemix_route_workspace_size.argtypes = [ctypes.POINTER(RouteArgs),
                                                   ctypes.POINTER(ctypes.c_size_t)]
        L.tilemix_route_pooled.restype = I
        L.tilemix_route_pooled.argtypes = [ctypes.POINTER(RouteArgs), P]
        L.tilemix_mass_probe.restype = I
        L.tilemix_mass_probe.argtypes = [ctypes.POINTER(MassArgs), P]
        L.tilemix_selftest_wait_timeout.restype = I
        L.tilemix_selftest_wait_timeout.argtypes = [I, P]
        L.tilemix_get_error.restype = I
        L.tilemix_get_error.argtypes = [P]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().tilemix_status_string(int(status)).decode()


tilemix_status_string = status_string


def _check(rc: int, what: str):
    if rc != OK:
        raise TileMixError(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ------------------------------------------------------------------- host ---

def tilemix_version() -> int:
    return int(lib().tilemix_version())


def tilemix_auto_g(seqlen: int) -> int:
    g = ctypes.c_int(0)
    _check(lib().tilemix_auto_g(int(seqlen), ctypes.byref(g)), "tilemix_auto_g")
    return g.value


def tilemix_tile_offsets(cu_seqlens):
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    nseq = cu.size - 1
    cq = np.zeros(nseq + 1, dtype=np.int32)
    ck = np.zeros(nseq + 1, dtype=np.int32)
    _check(lib().tilemix_tile_offsets(cu.ctypes.data, nseq, cq.ctypes.data, ck.ctypes.data),
           "tilemix_tile_offsets")
    return cq, ck


def tilemix_host_runs(cu_seqlens, chunks: int):
    """First sequence of each run tilemix_prefill_host cuts the batch into,
    plus nseq at the end (so run r is run_start[r] .. run_start[r + 1] - 1)."""
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    nseq = cu.size - 1
    starts = np.zeros(max(1, min(int(chunks), nseq)) + 1, dtype=np.int32)
    n = ctypes.c_int(0)
    _check(lib().tilemix_host_runs(cu.ctypes.data, nseq, int(chunks), starts.ctypes.data,
                                   ctypes.byref(n)), "tilemix_host_runs")
    return starts[:n.value + 1].copy()


def tilemix_build_routing(template, int8_percent: int, seed: int, cu_seqlens, n_kv_heads: int,
                          g, causal: bool = True):
    """Routing words [total_qtiles, n_kv_heads] (uint64) and per-sequence
    (legal groups, INT8 groups)."""
    tpl = TEMPLATES[template] if isinstance(template, str) else int(template)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    nseq = cu.size - 1
    gg = np.ascontiguousarray(g, dtype=np.int32)
    if gg.size != nseq:
        raise ValueError("one grouping factor per sequence")
    cq, _ = tilemix_tile_offsets(cu)
    masks = np.zeros((int(cq[-1]), int(n_kv_heads)), dtype=np.uint64)
    legal = np.zeros(nseq, dtype=np.int64)
    int8 = np.zeros(nseq, dtype=np.int64)
    _check(lib().tilemix_build_routing(tpl, int(int8_percent), ctypes.c_uint64(seed & (2**64 - 1)),
                                       cu.ctypes.data, nseq, int(n_kv_heads), gg.ctypes.data,
                                       int(bool(causal)), masks.ctypes.data, legal.ctypes.data,
                                       int8.ctypes.data),
           "tilemix_build_routing")
    return masks, legal, int8


# ----------------------------------------------------------------- device ---

def tilemix_quantize_qk(q, k, cu_seqlens, cu_qtiles, cu_ktiles, nseq, total_tokens,
                        total_qtiles, total_ktiles, hq, hk, d, q_i8, q_scale, k_i8, k_scale,
                        stream=None):
    _check(lib().tilemix_quantize_qk(_ptr(q), _ptr(k), _ptr(cu_seqlens), _ptr(cu_qtiles),
                                     _ptr(cu_ktiles), int(nseq), int(total_tokens),
                                     int(total_qtiles), int(total_ktiles), int(hq), int(hk),
                                     int(d), _ptr(q_i8), _ptr(q_scale), _ptr(k_i8),
                                     _ptr(k_scale), _stream_handle(stream)),
           "tilemix_quantize_qk")


def tilemix_quantize_qk_fp8(q, k, cu_seqlens, cu_qtiles, cu_ktiles, nseq, total_tokens,
                            total_qtiles, total_ktiles, hq, hk, d, q_codes, q_scale, k_codes,
                            k_scale, stream=None):
    """The FP8 (e4m3) low path's codes (bytes in int8/uint8 tensors) and scales."""
    _check(lib().tilemix_quantize_qk_fp8(_ptr(q), _ptr(k), _ptr(cu_seqlens), _ptr(cu_qtiles),
                                         _ptr(cu_ktiles), int(nseq), int(total_tokens),
                                         int(total_qtiles), int(total_ktiles), int(hq), int(hk),
                                         int(d), _ptr(q_codes), _ptr(q_scale), _ptr(k_codes),
                                         _ptr(k_scale), _stream_handle(stream)),
           "tilemix_quantize_qk_fp8")


def tilemix_quantize_qk_int4(q, k, cu_seqlens, cu_qtiles, cu_ktiles, nseq, total_tokens,
                             total_qtiles, total_ktiles, hq, hk, d, q_codes, q_scale, k_codes,
                             k_scale, stream=None):
    """The INT4 low path's codes (in [-7, 7], one per int8 element) and scales."""
    _check(lib().tilemix_quantize_qk_int4(_ptr(q), _ptr(k), _ptr(cu_seqlens), _ptr(cu_qtiles),
                                          _ptr(cu_ktiles), int(nseq), int(total_tokens),
                                          int(total_qtiles), int(total_ktiles), int(hq), int(hk),
                                          int(d), _ptr(q_codes), _ptr(q_scale), _ptr(k_codes),
                                          _ptr(k_scale), _stream_handle(stream)),
           "tilemix_quantize_qk_int4")


def make_args(q, k, v, o, cu_seqlens, cu_qtiles, cu_ktiles, nseq, total_tokens, total_qtiles,
              total_ktiles, max_seqlen, masks, g, causal=True, softmax_scale=0.0,
              kv_head_of_q=None, lse=None, k_i8=None, k_scale=None, workspace=None,
              debug_int32_scores=None, events=None, low="int8") -> PrefillArgs:
    T, hq, d = q.shape
    hk = k.shape[1]
    a = PrefillArgs()
    a.q, a.k, a.v, a.o = (x.data_ptr() for x in (q, k, v, o))
    a.lse = lse.data_ptr() if lse is not None else None
    a.cu_seqlens, a.cu_qtiles, a.cu_ktiles = (x.data_ptr() for x in (cu_seqlens, cu_qtiles,
                                                                       cu_ktiles))
    a.nseq, a.total_tokens, a.total_qtiles, a.total_ktiles = (int(nseq), int(total_tokens),
                                                               int(total_qtiles),
                                                               int(total_ktiles))
    a.max_seqlen = int(max_seqlen)
    a.hq, a.hk, a.d = int(hq), int(hk), int(d)
    a.kv_head_of_q = kv_head_of_q.data_ptr() if kv_head_of_q is not None else None
    a.masks = masks.data_ptr()
    a.g = g.data_ptr()
    a.causal = int(bool(causal))
    a.softmax_scale = float(softmax_scale)
    a.k_i8 = k_i8.data_ptr() if k_i8 is not None else None
    a.k_scale = k_scale.data_ptr() if k_scale is not None else None
    if workspace is not None:
        a.workspace = workspace.data_ptr()
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    a.debug_int32_scores = (debug_int32_scores.data_ptr()
                            if debug_int32_scores is not None else None)
    if events is not None:  # (begin, end) torch.cuda.Event pair around the fused kernel
        a.event_kernel_begin = events[0].cuda_event
        a.event_kernel_end = events[1].cuda_event
    a.low_format = LOW_FORMATS[low]
    return a


def tilemix_workspace_size(args: PrefillArgs) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().tilemix_workspace_size(ctypes.byref(args), ctypes.byref(n)),
           "tilemix_workspace_size")
    return int(n.value)


def tilemix_prefill_fwd(args: PrefillArgs, stream=None):
    _check(lib().tilemix_prefill_fwd(ctypes.byref(args), _stream_handle(stream)),
           "tilemix_prefill_fwd")


def tilemix_prefill_fwd_noalloc(args: PrefillArgs, stream=None):
    """tilemix_prefill_fwd without a caller workspace: the library's fixed
    64 MiB scratch array is used instead (see include/tilemix.h)."""
    _check(lib().tilemix_prefill_fwd_noalloc(ctypes.byref(args), _stream_handle(stream)),
           "tilemix_prefill_fwd_noalloc")


def tilemix_prefill_host(args: PrefillHostArgs, stream=None):
    """Host-buffer prefill with overlapped copies (see include/tilemix.h)."""
    _check(lib().tilemix_prefill_host(ctypes.byref(args), _stream_handle(stream)),
           "tilemix_prefill_host")


MMA_FORMS = {"f16": 0, "i8": 1, "f16_tmem_a": 2, "f8": 3}


def tilemix_mma_rate(form, n, iters, ctas, cycles, stream=None):
    """Diagnostic: back-to-back tcgen05.mma of one form (see include/tilemix.h);
    ``cycles`` is a device int64 tensor of 2 * ctas (issue, completion cycles
    per CTA)."""
    _check(lib().tilemix_mma_rate(MMA_FORMS[form] if isinstance(form, str) else int(form),
                                  int(n), int(iters), int(ctas), _ptr(cycles),
                                  _stream_handle(stream)), "tilemix_mma_rate")


def mma_rate(form, n, iters=4096, ctas=None, device="cuda"):
    """Measured rate of one MMA form on every SM: returns a dict with the SM
    cycles per MMA (issue and completion, median over CTAs), the wall time and
    the dense rate in TFLOP/s (TOP/s for INT8) over all CTAs.  M = 128, K = 16
    (f16) or 32 (i8, f8) per MMA."""
    import torch
    dev = torch.device(device)
    if ctas is None:
        ctas = torch.cuda.get_device_properties(dev).multi_processor_count
    cyc = torch.zeros(2 * ctas, dtype=torch.int64, device=dev)
    tilemix_mma_rate(form, n, 16, ctas, cyc)  # warm-up (module load, clocks)
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    tilemix_mma_rate(form, n, iters, ctas, cyc)
    b.record()
    torch.cuda.synchronize(dev)
    c = cyc.cpu().numpy().reshape(ctas, 2)
    if (c[:, 1] < 0).any():
        raise TileMixError(ERR_TIMEOUT, "tilemix_mma_rate")
    nmma = 4 * iters
    k = 16 if (form in ("f16", "f16_tmem_a", 0, 2)) else 32
    ms = a.elapsed_time(b)
    ops = 2.0 * 128 * n * k * nmma * ctas
    return {"form": form, "n": int(n), "issue_cycles_per_mma": float(np.median(c[:, 0])) / nmma,
            "cycles_per_mma": float(np.median(c[:, 1])) / nmma, "ms": ms,
            "tera_ops_per_s": ops / (ms * 1e-3) / 1e12, "ctas": int(ctas)}


def tilemix_selftest_wait_timeout(timeout_ms: int, stream=None):
    _check(lib().tilemix_selftest_wait_timeout(int(timeout_ms), _stream_handle(stream)),
           "tilemix_selftest_wait_timeout")


def tilemix_get_error(stream=None) -> int:
    return int(lib().tilemix_get_error(_stream_handle(stream)))


def tilemix_decode_workspace_size(args: DecodeArgs) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().tilemix_decode_workspace_size(ctypes.byref(args), ctypes.byref(n)),
           "tilemix_decode_workspace_size")
    return int(n.value)


def tilemix_decode_fwd(args: DecodeArgs, stream=None):
    _check(lib().tilemix_decode_fwd(ctypes.byref(args), _stream_handle(stream)),
           "tilemix_decode_fwd")


def tilemix_route_workspace_size(args: RouteArgs) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().tilemix_route_workspace_size(ctypes.byref(args), ctypes.byref(n)),
           "tilemix_route_workspace_size")
    return int(n.value)


def tilemix_route_pooled(args: RouteArgs, stream=None):
    _check(lib().tilemix_route_pooled(ctypes.byref(args), _stream_handle(stream)),
           "tilemix_route_pooled")


def route_pooled(q, k, lengths, hq, hk, g, causal, int8_percent, kv_head_of_q=None,
                 stream=None, events=None, workspace=None):
    """Pooled-score routing words [total_qtiles, hk] (int64 view of uint64) on
    q's device for the packed batch ``lengths``."""
    import numpy as np
    import torch
    dev = q.device
    lengths = [int(x) for x in lengths]
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    cq, ck = tilemix_tile_offsets(cu)
    gh = np.ascontiguousarray(np.asarray(g, dtype=np.int32))
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    cud, cqd, ckd, gd = to(cu), to(cq), to(ck), to(gh)
    masks = torch.empty((int(cq[-1]), int(hk)), dtype=torch.int64, device=dev)
    a = RouteArgs()
    a.q, a.k = _ptr(q), _ptr(k)
    a.cu_seqlens_h = cu.ctypes.data_as(ctypes.c_void_p)
    a.g_h = gh.ctypes.data_as(ctypes.c_void_p)
    a.cu_seqlens, a.cu_qtiles, a.cu_ktiles, a.g = _ptr(cud), _ptr(cqd), _ptr(ckd), _ptr(gd)
    km = None
    if kv_head_of_q is not None:
        km = to(kv_head_of_q)
        a.kv_head_of_q = _ptr(km)
    a.nseq, a.hq, a.hk, a.d = len(lengths), int(hq), int(hk), int(q.shape[-1])
    a.causal, a.int8_percent = int(bool(causal)), int(int8_percent)
    a.masks = _ptr(masks)
    need = tilemix_route_workspace_size(a)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    a.workspace, a.workspace_bytes = _ptr(workspace), workspace.numel()
    if events is not None:
        a.event_begin, a.event_end = events[0].cuda_event, events[1].cuda_event
    tilemix_route_pooled(a, stream)
    # keep the device metadata alive until the launches have read it
    masks._route_keepalive = (cud, cqd, ckd, gd, km, workspace)
    return masks


def tilemix_mass_probe(args: MassArgs, stream=None):
    _check(lib().tilemix_mass_probe(ctypes.byref(args), _stream_handle(stream)),
           "tilemix_mass_probe")


def mass_probe(q, k, masks, lengths, hq, hk, g, causal=True, delta_log2=4.0, kv_head_of_q=None,
               softmax_scale=0.0, stream=None, events=None):
    """Per (query head, token) m8, h, h8 (fp32 tensors [hq, T]) on q's device."""
    import numpy as np
    import torch
    dev = q.device
    lengths = [int(x) for x in lengths]
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    cq, ck = tilemix_tile_offsets(cu)
    gh = np.ascontiguousarray(np.asarray(g, dtype=np.int32))
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    cud, cqd, ckd, gd = to(cu), to(cq), to(ck), to(gh)
    if isinstance(masks, np.ndarray):
        masks = torch.from_numpy(np.ascontiguousarray(masks, dtype=np.uint64).view(np.int64)).to(dev)
    T = int(cu[-1])
    out = [torch.empty((int(hq), T), dtype=torch.float32, device=dev) for _ in range(3)]
    a = MassArgs()
    a.q, a.k = _ptr(q), _ptr(k)
    a.cu_seqlens_h = cu.ctypes.data_as(ctypes.c_void_p)
    a.g_h = gh.ctypes.data_as(ctypes.c_void_p)
    a.cu_seqlens, a.cu_qtiles, a.cu_ktiles, a.g = _ptr(cud), _ptr(cqd), _ptr(ckd), _ptr(gd)
    a.masks = _ptr(masks)
    km = None
    if kv_head_of_q is not None:
        km = to(kv_head_of_q)
        a.kv_head_of_q = _ptr(km)
    a.nseq, a.hq, a.hk, a.d = len(lengths), int(hq), int(hk), int(q.shape[-1])
    a.causal, a.softmax_scale, a.delta_log2 = int(bool(causal)), float(softmax_scale), float(delta_log2)
    a.m8, a.h, a.h8 = _ptr(out[0]), _ptr(out[1]), _ptr(out[2])
    if events is not None:
        a.event_begin, a.event_end = events[0].cuda_event, events[1].cuda_event
    tilemix_mass_probe(a, stream)
    out[0]._mass_keepalive = (cud, cqd, ckd, gd, km, masks)
    return tuple(out)


from .prefill import TileMixPrefill  # noqa: E402  (convenience wrapper)
from .decode import TileMixDecode  # noqa: E402  (convenience wrapper)

__all__ = [
    "BLOCK_M", "BLOCK_N", "DecodeArgs", "MAX_GROUPS", "PrefillArgs", "RouteArgs", "TEMPLATES",
    "TileMixError", "route_pooled", "tilemix_route_pooled", "tilemix_route_workspace_size",
    "LOW_FORMATS", "tilemix_quantize_qk_fp8", "tilemix_quantize_qk_int4",
    "MassArgs", "mass_probe", "tilemix_mass_probe",
    "TileMixDecode", "TileMixPrefill", "lib", "make_args", "status_string", "tilemix_auto_g",
    "tilemix_build_routing", "tilemix_decode_fwd", "tilemix_decode_workspace_size",
    "tilemix_get_error", "tilemix_prefill_fwd",
    "tilemix_prefill_fwd_noalloc", "tilemix_quantize_qk", "tilemix_selftest_wait_timeout",
    "PrefillHostArgs", "tilemix_prefill_host", "tilemix_host_runs",
    "tilemix_status_string", "tilemix_tile_offsets", "tilemix_version",
    "tilemix_workspace_size", "tilemix_mma_rate", "mma_rate",
]
