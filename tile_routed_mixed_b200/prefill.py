"""Reusable call site for ``tilemix_prefill_fwd``: keeps a batch's device-side
metadata (offsets, routing words, grouping factors) and the workspace, so a
step only marshals the four tensor pointers."""
from __future__ import annotations

import numpy as np
import torch

import ctypes

from . import (BLOCK_M, PrefillHostArgs, make_args, tilemix_prefill_fwd, tilemix_prefill_host,
               tilemix_tile_offsets, tilemix_workspace_size)


class TileMixPrefill:
    def __init__(self, lengths, hq, hk, d, masks, g, causal=True, softmax_scale=0.0,
                 kv_head_of_q=None, device="cuda", low="int8"):
        self.lengths = [int(x) for x in lengths]
        self.hq, self.hk, self.d = int(hq), int(hk), int(d)
        cu = np.zeros(len(self.lengths) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(self.lengths)
        cq, ck = tilemix_tile_offsets(cu)
        self.nseq = len(self.lengths)
        self.total_tokens = int(cu[-1])
        self.total_qtiles = int(cq[-1])
        self.total_ktiles = int(ck[-1])
        self.max_seqlen = max(self.lengths) if self.lengths else 0
        self.causal = bool(causal)
        self.softmax_scale = float(softmax_scale)
        self.low = str(low)  # low-precision path of bit-1 tiles: "int8", "fp8" (e4m3) or "int4"
        self.device = torch.device(device)
        masks = np.ascontiguousarray(masks, dtype=np.uint64)
        if masks.shape != (self.total_qtiles, self.hk):
            raise ValueError("masks must be [total_qtiles, hk] = [%d, %d]"
                             % (self.total_qtiles, self.hk))
        self.cu_seqlens = torch.from_numpy(cu).to(self.device)
        self.cu_qtiles = torch.from_numpy(cq).to(self.device)
        self.cu_ktiles = torch.from_numpy(ck).to(self.device)
        self.masks = torch.from_numpy(masks.view(np.int64)).to(self.device)
        self.g = torch.as_tensor(np.asarray(g, dtype=np.int32)).to(self.device)
        self.kv_head_of_q = (None if kv_head_of_q is None else
                             torch.as_tensor(np.asarray(kv_head_of_q, dtype=np.int32)).to(self.device))
        self.workspace = None
        self.cu_host = cu
        self._host_side = None  # (chunks, stream_in, stream_out, events, handle array)

    @property
    def max_qtiles(self):
        return (self.max_seqlen + BLOCK_M - 1) // BLOCK_M

    def args(self, q, k, v, o, lse=None, k_i8=None, k_scale=None, debug_int32_scores=None,
             events=None):
        return make_args(q, k, v, o, self.cu_seqlens, self.cu_qtiles, self.cu_ktiles, self.nseq,
                         self.total_tokens, self.total_qtiles, self.total_ktiles,
                         self.max_seqlen, self.masks, self.g, causal=self.causal,
                         softmax_scale=self.softmax_scale, kv_head_of_q=self.kv_head_of_q,
                         lse=lse, k_i8=k_i8, k_scale=k_scale, workspace=self.workspace,
                         debug_int32_scores=debug_int32_scores, events=events, low=self.low)

    def ensure_workspace(self, q, k, v, o, **kw):
        a = self.args(q, k, v, o, **kw)
        need = tilemix_workspace_size(a)
        if self.workspace is None or self.workspace.numel() < need:
            self.workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=self.device)
        return self.workspace

    def __call__(self, q, k, v, o=None, lse=None, stream=None, **kw):
        if o is None:
            o = torch.empty_like(q)
        self.ensure_workspace(q, k, v, o, lse=lse, **kw)
        tilemix_prefill_fwd(self.args(q, k, v, o, lse=lse, **kw), stream)
        return o

    def host_args(self, q_h, k_h, v_h, o_h, q, k, v, o, chunks=8, after_previous=False,
                  lse=None):
        """Arguments of ``tilemix_prefill_host``: host tensors q_h, k_h, v_h, o_h
        (page-locked for the copies to overlap) and the device buffers q, k, v,
        o of the same shapes.  The side streams and events are kept here, so
        ``after_previous`` may chain a call to the previous one made through
        this object with the same device buffers and chunks.  ``lse``, if
        given, is a device buffer and stays on the device."""
        for name, t in (("q_h", q_h), ("k_h", k_h), ("v_h", v_h), ("o_h", o_h)):
            if t.device.type != "cpu" or not t.is_contiguous() or t.dtype != torch.float16:
                raise ValueError("%s must be a contiguous fp16 CPU tensor" % name)
        chunks = int(chunks)
        if self._host_side is None or self._host_side[0] != chunks:
            s_in = torch.cuda.Stream(device=self.device)
            s_out = torch.cuda.Stream(device=self.device)
            evs = [torch.cuda.Event() for _ in range(3 * chunks + 1)]
            for e in evs:  # creates the CUDA event
                e.record(s_in)
            handles = (ctypes.c_void_p * len(evs))(*[e.cuda_event for e in evs])
            self._host_side = (chunks, s_in, s_out, evs, handles)
        _, s_in, s_out, _, handles = self._host_side
        self.ensure_workspace(q, k, v, o, lse=lse)
        h = PrefillHostArgs()
        h.dev = self.args(q, k, v, o, lse=lse)
        h.cu_seqlens_h = self.cu_host.ctypes.data
        h.q_h, h.k_h, h.v_h, h.o_h = (t.data_ptr() for t in (q_h, k_h, v_h, o_h))
        h.chunks = chunks
        h.stream_in = s_in.cuda_stream
        h.stream_out = s_out.cuda_stream
        h.events = ctypes.cast(handles, ctypes.c_void_p).value
        h.after_previous = 1 if after_previous else 0
        return h

    @property
    def upload_stream(self):
        """The stream the host-buffer call uploads on (None before its first use)."""
        return None if self._host_side is None else self._host_side[1]

    def from_host(self, q_h, k_h, v_h, o_h, q, k, v, o, chunks=8, after_previous=False,
                  lse=None, stream=None):
        """O of host inputs into host o_h through tilemix_prefill_host; work
        enqueued on `stream` afterwards sees o_h complete."""
        tilemix_prefill_host(self.host_args(q_h, k_h, v_h, o_h, q, k, v, o, chunks,
                                            after_previous, lse), stream)
        return o_h
