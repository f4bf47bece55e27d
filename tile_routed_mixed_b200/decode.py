"""Reusable call site for ``tilemix_decode_fwd``: keeps a batch's device-side
metadata (cache extents, tile offsets, routing words, grouping factors) and the
workspace, so a step only marshals the tensor pointers."""
from __future__ import annotations

import numpy as np
import torch

from . import DecodeArgs, _ptr, tilemix_decode_fwd, tilemix_decode_workspace_size


class TileMixDecode:
    """Sequence s holds seq_len[s] cached tokens (the new one last) in cache
    rows [seq_start[s], seq_start[s] + seq_len[s]); its K block scales start at
    column ktile_start[s] of k_scale and its routing words at row
    qtile_start[s] of masks ([total_qtiles, hk])."""

    def __init__(self, seq_start, seq_len, ktile_start, qtile_start, hq, hk, d, masks, g,
                 total_ktiles, softmax_scale=0.0, kv_head_of_q=None, device="cuda",
                 tiles_per_split=0):
        self.device = torch.device(device)
        to = lambda a, dt: torch.as_tensor(np.ascontiguousarray(a, dtype=dt)).to(self.device)
        self.seq_len_h = [int(x) for x in seq_len]
        self.nseq = len(self.seq_len_h)
        self.hq, self.hk, self.d = int(hq), int(hk), int(d)
        self.max_seqlen = max(self.seq_len_h) if self.seq_len_h else 1
        self.total_ktiles = int(total_ktiles)
        self.softmax_scale = float(softmax_scale)
        self.tiles_per_split = int(tiles_per_split)
        self.seq_start = to(seq_start, np.int32)
        self.seq_len = to(seq_len, np.int32)
        self.ktile_start = to(ktile_start, np.int32)
        self.qtile_start = to(qtile_start, np.int32)
        self.masks = to(np.ascontiguousarray(masks, dtype=np.uint64).view(np.int64), np.int64)
        self.g = to(g, np.int32)
        self.kv_head_of_q = None if kv_head_of_q is None else to(kv_head_of_q, np.int32)
        self.workspace = None

    def args(self, q, k, v, k_i8, k_scale, o, events=None):
        a = DecodeArgs()
        a.q, a.k, a.v = _ptr(q), _ptr(k), _ptr(v)
        a.k_i8, a.k_scale, a.o = _ptr(k_i8), _ptr(k_scale), _ptr(o)
        a.seq_start, a.seq_len = _ptr(self.seq_start), _ptr(self.seq_len)
        a.ktile_start, a.qtile_start = _ptr(self.ktile_start), _ptr(self.qtile_start)
        a.masks, a.g = _ptr(self.masks), _ptr(self.g)
        a.kv_head_of_q = _ptr(self.kv_head_of_q) if self.kv_head_of_q is not None else None
        a.nseq, a.max_seqlen, a.total_ktiles = self.nseq, self.max_seqlen, self.total_ktiles
        a.cache_rows = int(k.shape[0]) if k is not None else 0
        a.hq, a.hk, a.d = self.hq, self.hk, self.d
        a.softmax_scale = self.softmax_scale
        a.tiles_per_split = self.tiles_per_split
        if self.workspace is not None:
            a.workspace, a.workspace_bytes = _ptr(self.workspace), self.workspace.numel()
        if events is not None:  # (begin, end) torch.cuda.Event pair around the attention kernel
            a.event_kernel_begin = events[0].cuda_event
            a.event_kernel_end = events[1].cuda_event
        return a

    def __call__(self, q, k, v, k_i8, k_scale, o=None, stream=None, events=None):
        if o is None:
            o = torch.empty_like(q)
        a = self.args(q, k, v, k_i8, k_scale, o, events)
        need = tilemix_decode_workspace_size(a)
        if self.workspace is None or self.workspace.numel() < need:
            self.workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=self.device)
            a = self.args(q, k, v, k_i8, k_scale, o, events)
        tilemix_decode_fwd(a, stream)
        return o
