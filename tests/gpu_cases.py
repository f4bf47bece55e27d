"""Shared GPU-vs-oracle machinery for the parity tests and the smoke check."""
from __future__ import annotations

import math
import os

import numpy as np

import oracle
import synth

# fp16 output tolerances of the parity bar (max-abs, mean-abs against the
# fp64 oracle).
MAX_ABS = 2e-3
MEAN_ABS = 2e-4


_INPUTS = {}


class Case:
    def __init__(self, lengths, hq, hk, d, causal=True, template="band", percent=50, g=None,
                 outliers=0, lowrank=0, seed=0, routing_seed=0, kv_map=None):
        self.lengths = [int(x) for x in lengths]
        self.hq, self.hk, self.d = hq, hk, d
        self.causal = causal
        self.template, self.percent = template, percent
        if g is None or g == "auto":
            g = [oracle.auto_g(L) for L in self.lengths]
        elif isinstance(g, int):
            g = [g] * len(self.lengths)
        self.g = list(g)
        self.outliers, self.lowrank = outliers, lowrank
        self.seed, self.routing_seed = seed, routing_seed
        self.kv_map = kv_map

    @classmethod
    def workload(cls, name, **over):
        w = synth.WORKLOADS[name]
        lengths = synth.workload_lengths(name)
        g = "auto" if w["g"] == "auto" else int(w["g"])
        kw = dict(lengths=lengths, hq=w["hq"], hk=w["hk"], d=w["d"], causal=w["causal"],
                  template=w["template"], percent=w["percent"], g=g, outliers=w["outliers"],
                  lowrank=w["lowrank"], seed=0, routing_seed=w["routing_seed"])
        kw.update(over)
        return cls(**kw)

    @property
    def total_tokens(self):
        return sum(self.lengths)

    def inputs(self):
        # one draw per process and shape: the workload sweeps reuse it
        key = (self.seed, self.total_tokens, self.hq, self.hk, self.d, self.outliers,
               self.lowrank)
        if key not in _INPUTS:
            if len(_INPUTS) >= 2:
                _INPUTS.clear()
            _INPUTS[key] = synth.make_qkv(*key[:5], outliers=self.outliers, lowrank=self.lowrank)
        return _INPUTS[key]

    def masks(self, words=None):
        if words is not None:
            tm = sum(oracle.n_qtiles(L) for L in self.lengths)
            return np.full((tm, self.hk), words, dtype=np.uint64)
        return oracle.build_routing(self.template, self.percent, self.routing_seed, self.lengths,
                                    self.hk, self.g, self.causal)[0]


def sample_rows(lengths, hq, seed=0, per_head_random=64, heads=None, tiles_per_head=None):
    """Every q-tile's first, middle and last row (optionally only on `heads`)
    plus `per_head_random` seeded rows per (sequence, head)."""
    rng = np.random.default_rng(seed)
    rows = []
    for s, L in enumerate(lengths):
        for h in range(hq):
            picks = set()
            if heads is None or h in heads:
                ntile = math.ceil(L / 128)
                tiles = range(ntile)
                if tiles_per_head is not None and ntile > tiles_per_head:
                    tiles = np.unique(np.linspace(0, ntile - 1, tiles_per_head).astype(int))
                for qt in tiles:
                    r0 = qt * 128
                    r1 = min(L, r0 + 128) - 1
                    picks |= {r0, (r0 + r1) // 2, r1}
            picks |= set(int(x) for x in rng.integers(0, L, size=per_head_random))
            rows += [(s, h, i) for i in sorted(picks)]
    return np.array(rows, dtype=np.int64).reshape(-1, 3)


def oracle_rows(case, q, k, v, masks, rows):
    q8, qs = oracle.quantize_q(q, case.lengths)
    k8, ks = oracle.quantize_k(k, case.lengths)
    O, lse = oracle.attention_rows(q, k, v, q8, qs, k8, ks, masks, case.g, case.lengths,
                                   case.causal, kv_map=case.kv_map, rows=rows)
    return O, lse, (q8, qs, k8, ks)


def gather(case, o_full, rows):
    """Rows [n, d] of a [T, hq, d] array at (sequence, head, row) triples."""
    cu = np.concatenate([[0], np.cumsum(case.lengths)])
    t = cu[rows[:, 0]] + rows[:, 2]
    return o_full[t, rows[:, 1]]


def errors(got, want):
    diff = np.abs(got.astype(np.float64) - want)
    return float(diff.max()) if diff.size else 0.0, float(diff.mean()) if diff.size else 0.0


def run_gpu(case, q, k, v, masks, lse=False, debug=False, device="cuda"):
    """Run tilemix_prefill_fwd through the C ABI; returns numpy O (and LSE, dbg)."""
    import torch

    import tile_routed_mixed_b200 as tm
    pf = tm.TileMixPrefill(case.lengths, case.hq, case.hk, case.d, masks, case.g,
                           causal=case.causal, kv_head_of_q=case.kv_map, device=device)
    qd = torch.from_numpy(q).to(device)
    kd = torch.from_numpy(k).to(device)
    vd = torch.from_numpy(v).to(device)
    od = torch.full_like(qd, float("nan"))
    lsed = torch.zeros((case.hq, case.total_tokens), dtype=torch.float32, device=device) if lse else None
    dbg = None
    if debug:
        cols = (pf.max_seqlen + 63) // 64 * 64
        dbg = torch.full((case.hq, case.total_tokens, cols), -(2 ** 31), dtype=torch.int32,
                         device=device)
    pf(qd, kd, vd, od, lse=lsed, debug_int32_scores=dbg)
    rc = tm.tilemix_get_error()
    if rc != tm.OK:
        raise tm.TileMixError(rc, "device status")
    out = {"o": od.cpu().numpy()}
    if lse:
        out["lse"] = lsed.cpu().numpy()
    if debug:
        out["dbg"] = dbg.cpu().numpy()
    return out


def set_test_timeout():
    os.environ.setdefault("TILEMIX_WAIT_TIMEOUT_MS", "1000")
