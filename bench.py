#!/usr/bin/env python
"""Throughput of tile-routed FP16/INT8 causal prefill attention on B200.

One step = one pass of the whole hot path over one batch: K block
quantisation, Q block quantisation and the fused routed attention kernel,
launched through the C ABI (tilemix_prefill_fwd).  Default workload: LLaMA-3.2-3B
attention shape, batch 8 x 4096 tokens, 24 query / 8 KV heads, head dim 128,
causal, SpTrans routing at 75% INT8 of legal tile groups, synthetic N(0,1)
inputs with four x8 outlier channels per KV head.

Prints one JSON line (rank 0).  Multi-GPU (torchrun): every rank runs its own
batch (weak scaling, no collective on the data path); timing is the max over
ranks.  ``--impl reference`` times the CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "attention prefill tok/s at 4k b8 (3B GQA shape); % of mixed tensor roofline"
UNIT = "tok/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_F16 = 4.5 / 2.25  # nominal dense INT8 : FP16 tensor rate on B200 (context only)


# ----------------------------------------------------------------- helpers ---

def workload(name, template=None, percent=None, seqs=None):
    """A configuration's sizes; `seqs` keeps only its first sequences (a
    smaller case of the same shapes, for profiler captures)."""
    w = dict(synth.WORKLOADS[name])
    if template:
        w["template"] = template
    if percent is not None:
        w["percent"] = int(percent)
    lengths = synth.workload_lengths(name)
    if seqs:
        lengths = lengths[:int(seqs)]
    if w["g"] == "auto":
        g = [max(1, math.ceil(math.ceil(L / 64) / 64)) for L in lengths]
    else:
        g = [int(w["g"])] * len(lengths)
    return w, lengths, g


def legal_pairs(L, causal):
    """[Tm, Tn] legal (query, key) pair counts of one sequence's tile grid."""
    tm, tn = math.ceil(L / 128), math.ceil(L / 64)
    out = np.zeros((tm, tn), dtype=np.int64)
    for qt in range(tm):
        rows = np.arange(qt * 128, min(L, qt * 128 + 128))
        for kt in range(tn):
            k0, k1 = kt * 64, min(L, kt * 64 + 64)
            if causal:
                out[qt, kt] = np.clip(rows - k0 + 1, 0, k1 - k0).sum()
            else:
                out[qt, kt] = len(rows) * (k1 - k0)
    return out


def algorithmic_work(lengths, hq, hk, d, masks, g, causal):
    """FP16 FLOPs, INT8 ops and HBM bytes of one batch (legal pairs only:
    2d per pair for QK in the routed precision, 2d FP16 for PV; bytes = Q, K,
    V read once and O written once in fp16)."""
    f16 = 0
    i8 = 0
    row = 0
    group = hq // hk
    for s, L in enumerate(lengths):
        pairs = legal_pairs(L, causal)
        for qt in range(pairs.shape[0]):
            for kv in range(hk):
                w = int(masks[row + qt, kv])
                bits = np.array([(w >> (kt // g[s])) & 1 for kt in range(pairs.shape[1])], bool)
                p_int = int(pairs[qt, bits].sum())
                p_all = int(pairs[qt].sum())
                i8 += group * 2 * d * p_int
                f16 += group * 2 * d * (p_all - p_int) + group * 2 * d * p_all
        row += pairs.shape[0]
    T = sum(lengths)
    nbytes = T * (2 * hq + 2 * hk) * d * 2
    return f16, i8, nbytes


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p["bf16_tflops_sustained"]),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK, source="fallback")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples of this GPU, every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = os.path.join("/tmp", "tilemix_clocks_%d_%d.csv" % (os.getpid(), time.time_ns()))

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id,
                                          "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity when not
    distributed).  Timing of multi-GPU runs is the slowest rank's."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def low_over_f16(low="int8"):
    """Measured dense rate ratio of the low-precision MMA form to the FP16 one
    on this GPU: tcgen05.mma M128 N256 issued back to back on every SM
    (tilemix_mma_rate), kind::i8 (or kind::f8f6f4) with K = 32 against
    kind::f16 with K = 16, from the SM cycles per MMA.  Returns the ratio and
    the two measurements."""
    import tile_routed_mixed_b200 as tm
    f16 = tm.mma_rate("f16", 256, iters=2048)
    lo = tm.mma_rate("f8" if low == "fp8" else "i8", 256, iters=2048)  # INT4 codes: kind::i8
    per_cycle_f16 = 2 * 128 * 256 * 16 / f16["cycles_per_mma"]
    per_cycle_lo = 2 * 128 * 256 * 32 / lo["cycles_per_mma"]
    return per_cycle_lo / per_cycle_f16, f16, lo


def whole_job_tokens(tokens_per_rank, world):
    """Weak scaling: every rank processes its own full batch."""
    return int(tokens_per_rank) * int(world)


def kernel_traffic(workload_name, kernel="prefill_fwd_kernel<128>"):
    """DRAM bytes per launch of `kernel` from the committed ncu record, or None
    if the record is for another workload or one of the kernel's source files
    changed since it was captured."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel]
        h = hashlib.sha256()
        for name in rec["sources"]:
            with open(os.path.join(ROOT, "tile_routed_mixed_b200", "csrc", name), "rb") as f:
                h.update(f.read())
        if rec["workload"] != workload_name or h.hexdigest()[:16] != rec["sources_sha256_16"]:
            return None
        return float(rec["dram_bytes_per_launch"])
    except Exception:
        return None


def affinity_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def host_cores():
    """Threads the oracle's OpenMP loops run on: OMP_NUM_THREADS when set,
    else every core this process may use."""
    try:
        n = int(os.environ.get("OMP_NUM_THREADS", "").split(",")[0])
        if n > 0:
            return n
    except ValueError:
        pass
    return affinity_cores()


# ------------------------------------------------------------ oracle side ---

def oracle_sample(q, k, v, lengths, hq, hk, masks, g, causal, rows, quant=None):
    """Run the CPU oracle on `rows` and return (seconds, quant seconds)."""
    import oracle
    tq = 0.0
    if quant is None:
        t = time.perf_counter()
        q8, qs = oracle.quantize_q(q, lengths)
        k8, ks = oracle.quantize_k(k, lengths)
        tq = time.perf_counter() - t
        quant = (q8, qs, k8, ks)
    q8, qs, k8, ks = quant
    t = time.perf_counter()
    oracle.attention_rows(q, k, v, q8, qs, k8, ks, masks, g, lengths, causal, rows=rows)
    return time.perf_counter() - t, tq, quant


def random_rows(lengths, hq, n, rng):
    s = rng.integers(0, len(lengths), size=n)
    h = rng.integers(0, hq, size=n)
    L = np.asarray(lengths)[s]
    i = (rng.random(n) * L).astype(np.int64)
    return np.stack([s, h, i], axis=1).astype(np.int64)


def cpu_baseline(q, k, v, lengths, hq, hk, masks, g, causal, budget_s=15.0):
    """Oracle throughput on a bounded random-row sample, in prefill tokens/s
    (one token = all hq heads of a row; quantisation cost charged pro rata)."""
    rng = np.random.default_rng(1234)
    T = sum(lengths)
    cal = random_rows(lengths, hq, 256, rng)
    t_cal, t_quant, quant = oracle_sample(q, k, v, lengths, hq, hk, masks, g, causal, cal)
    n = int(max(256, min(1000000, 256 * budget_s / max(t_cal, 1e-3))))
    rows = random_rows(lengths, hq, n, rng)
    t_rows, _, _ = oracle_sample(q, k, v, lengths, hq, hk, masks, g, causal, rows, quant=quant)
    t = t_rows + t_quant * n / (T * hq)
    return {"value": (n / hq) / t, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
            "sample": "%d uniformly random (sequence, head, row) outputs of the workload, fp64 "
                      "oracle rows plus the numpy quantisation pro rata (%.1f s)" % (n, t)}


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, timed step by step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        # the launcher pins every rank to one OpenMP thread; rank 0 works
        # alone here, so give the oracle every core (before any OpenMP
        # runtime loads)
        os.environ["OMP_NUM_THREADS"] = str(affinity_cores())
    w, lengths, g = workload(args.workload, args.template, args.percent, args.seqs)
    hq, hk, d, causal = w["hq"], w["hk"], w["d"], w["causal"]
    T = sum(lengths)
    q, k, v = synth.make_qkv(0, T, hq, hk, d, outliers=w["outliers"], lowrank=w["lowrank"])
    import oracle
    masks = oracle.build_routing(w["template"], w["percent"], w["routing_seed"], lengths, hk, g,
                                 causal)[0]
    rng = np.random.default_rng(99)
    cal = random_rows(lengths, hq, 64, rng)
    t_cal, t_quant, quant = oracle_sample(q, k, v, lengths, hq, hk, masks, g, causal, cal)
    per_step_budget = max(0.02, 90.0 / max(1, args.steps + args.warmup))
    n = int(max(16, min(100000, 64 * per_step_budget / max(t_cal, 1e-4))))
    for _ in range(args.warmup):
        oracle_sample(q, k, v, lengths, hq, hk, masks, g, causal, random_rows(lengths, hq, n, rng),
                      quant=quant)
    total = 0.0
    for _ in range(args.steps):
        rows = random_rows(lengths, hq, n, rng)
        t, _, _ = oracle_sample(q, k, v, lengths, hq, hk, masks, g, causal, rows, quant=quant)
        total += t + t_quant * n / (T * hq)
    ms = 1e3 * total / args.steps
    value = (n / hq) / (total / args.steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64+i64",
        "data": "synthetic", "config": bench_config(args, w, lengths, g),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
                         "sample": "%d random (sequence, head, row) outputs per step" % n},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def bench_config(args, w, lengths, g):
    return {"workload": args.workload, "batch": len(lengths), "seq_len": lengths[0]
            if len(set(lengths)) == 1 else "varlen", "hq": w["hq"], "hk": w["hk"],
            "head_dim": w["d"], "causal": w["causal"], "template": w["template"],
            "int8_percent": w["percent"], "g": g[0] if len(set(g)) == 1 else "per-sequence",
            "block_m": 128, "block_n": 64, "low_precision": getattr(args, "low", "int8"),
            "l2": "no flush: inputs and output (%.0f MB per step) exceed the 126 MB L2"
                  % (sum(lengths) * (2 * w["hq"] + 2 * w["hk"]) * w["d"] * 2 / 1e6)}


# ---------------------------------------------------------------- GPU side ---

def run_gpu(args):
    import torch
    import torch.distributed as dist

    import tile_routed_mixed_b200 as tm

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    w, lengths, g = workload(args.workload, args.template, args.percent, args.seqs)
    hq, hk, d, causal = w["hq"], w["hk"], w["d"], w["causal"]
    T = sum(lengths)
    q, k, v = synth.make_qkv(rank, T, hq, hk, d, outliers=w["outliers"], lowrank=w["lowrank"])
    cu = synth.cu_seqlens_of(lengths)
    masks, legal, int8 = tm.tilemix_build_routing(w["template"], w["percent"],
                                                  w["routing_seed"], cu, hk, g, causal)
    pf = tm.TileMixPrefill(lengths, hq, hk, d, masks, g, causal=causal, device=dev, low=args.low)
    qd, kd, vd = (torch.from_numpy(x).to(dev) for x in (q, k, v))
    od = torch.empty_like(qd)
    pf.ensure_workspace(qd, kd, vd, od)
    stream = torch.cuda.current_stream(dev)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for a, b in ev:  # torch creates the CUDA event on first record: force it now
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    args_plain = pf.args(qd, kd, vd, od)
    args_timed = [pf.args(qd, kd, vd, od, events=e) for e in ev]

    for _ in range(args.warmup):
        tm.tilemix_prefill_fwd(args_plain, stream)
    rc = tm.tilemix_get_error(stream)
    if rc != tm.OK:
        raise tm.TileMixError(rc, "warm-up")

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)  # let the sampler take its first sample
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        tm.tilemix_prefill_fwd(args_timed[i], stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    rc = tm.tilemix_get_error(stream)
    if rc != tm.OK:
        raise tm.TileMixError(rc, "timed steps")
    ms = e0.elapsed_time(e1) / args.steps
    kern_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    ms, kern_ms = max_over_ranks([ms, kern_ms], device=dev)

    # end to end through the public host-buffer call (tilemix_prefill_host):
    # pinned inputs uploaded, O downloaded, by runs of sequences overlapped
    # with the kernels; `stream` ends with the last download
    qh, kh, vh = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
    oh = torch.empty(od.shape, dtype=od.dtype).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    nrun = min(len(lengths), 8)
    first_args = pf.host_args(qh, kh, vh, oh, qd, kd, vd, od, chunks=nrun)
    # later steps chain to the previous one: a step's uploads start while the
    # previous step's last runs finish
    host_args = pf.host_args(qh, kh, vh, oh, qd, kd, vd, od, chunks=nrun, after_previous=True)

    def e2e_step(args=host_args):
        tm.tilemix_prefill_host(args, stream)

    e2e_step(first_args)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0.record(stream)
    pf.upload_stream.wait_event(e0)  # the chained uploads start after e0
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks([e0.elapsed_time(e1) / e2e_steps], device=dev)[0]
    if not torch.equal(oh, od.cpu()):
        raise RuntimeError("host-buffer output differs from the device buffer")
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    f16, i8, nbytes = algorithmic_work(lengths, hq, hk, d, masks, g, causal)
    pk = peaks()
    p16 = pk["bf16_tflops"] * 1e12
    ratio, r16, rlo = low_over_f16(args.low)
    p8 = p16 * ratio
    t_tensor = f16 / p16 + i8 / p8
    t_mem = nbytes / (pk["hbm_gbs"] * 1e9)
    bound = "tensor" if t_tensor >= t_mem else "hbm"
    t_k = kern_ms / 1e3
    if bound == "tensor":
        achieved = (f16 + i8 * p16 / p8) / t_k / 1e12   # FP16-equivalent TFLOP/s
        peak, unit = p16 / 1e12, "TFLOP/s"
    else:
        achieved, peak, unit = nbytes / t_k / 1e9, pk["hbm_gbs"], "GB/s"
    tokens = whole_job_tokens(T, world)
    line = {
        "metric": METRIC,
        "value": tokens / (ms / 1e3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": {"int8": "f16+i8", "fp8": "f16+e4m3", "int4": "f16+i4(in i8)"}[args.low],
        "data": "synthetic",
        "config": bench_config(args, w, lengths, g),
        "roofline": {
            "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak,
            "traffic": kernel_traffic(args.workload) if not args.seqs else None,
            "traffic_unit": "bytes per launch (ncu)",
            "kernel": "prefill_fwd_kernel<128>",
            "kernel_ms": kern_ms,
            "peak_kind": "burst (%s)" % pk["source"],
            "fp16_flops": f16, "int8_ops": i8, "hbm_bytes": nbytes,
            "mixed_roof_ms": 1e3 * max(t_tensor, t_mem),
            "tflops_raw": (f16 + i8) / t_k / 1e12,
            "int8_share_of_legal_groups": float(int8.sum() / legal.sum()),
            "low_over_fp16_rate": {
                "measured": ratio, "nominal": INT8_OVER_F16,
                "how": "tcgen05.mma M128 N256 back to back on every SM: %s %.1f cycles per MMA "
                       "(K 32), kind::f16 %.1f (K 16)" % (
                           "kind::f8f6f4" if args.low == "fp8" else "kind::i8",
                           rlo["cycles_per_mma"], r16["cycles_per_mma"])},
        },
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": int(q.nbytes + k.nbytes + v.nbytes),
                "d2h_bytes_per_step": int(q.nbytes)},
        "gpu_launches": 2 * args.steps,  # quantiser + fused attention
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(q, k, v, lengths, hq, hk, masks, g, causal)
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ decode path ---

DECODE_METRIC = "attention decode tok/s at 4k b8 (3B GQA shape), INT8 K cache; % of HBM roofline"


def tile_starts(lengths):
    """First query tile (128 rows) and key tile (64 keys) of each sequence."""
    cq = np.zeros(len(lengths) + 1, dtype=np.int32)
    ck = np.zeros(len(lengths) + 1, dtype=np.int32)
    cq[1:] = np.cumsum([(L + 127) // 128 for L in lengths])
    ck[1:] = np.cumsum([(L + 63) // 64 for L in lengths])
    return cq, ck


def decode_bytes(lengths, hq, hk, d, masks, g):
    """Algorithmic HBM bytes of one decode step, and of its split attention
    kernel.  The step: every cached key once in its routed precision (INT8
    codes or fp16), every cached value once (fp16), the K block re-quantised
    (fp16 in, codes out), the new query rows and O.  The attention kernel: the
    keys and values, and the query rows in fp16 and as codes (its partial
    results are scratch and not counted)."""
    cq, ck = tile_starts(lengths)
    total = 0
    requant = 0
    for s, L in enumerate(lengths):
        t = L - 1
        nt = t // 64 + 1
        for kv in range(hk):
            w = int(masks[cq[s] + t // 128, kv])
            for kt in range(nt):
                keys = min(64, L - 64 * kt)
                total += keys * d * (1 if (w >> (kt // int(g[s]))) & 1 else 2) + keys * d * 2
            last = L - 64 * (t // 64)
            requant += last * d * 3
    attn = total + len(lengths) * hq * d * 3
    return total + requant + len(lengths) * hq * d * 2 * 2, attn


DECODE_CACHES = 4  # copies of the decode cache the steps rotate over


def run_decode(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference" and rank != 0:
        return
    w, lengths, g = workload(args.workload, args.template, args.percent, args.seqs)
    hq, hk, d = w["hq"], w["hk"], w["d"]
    if args.impl != "reference":
        import torch
        import torch.distributed as dist

        import tile_routed_mixed_b200 as tm
    cu = synth.cu_seqlens_of(lengths)
    cq, ck = tile_starts(lengths)
    if args.impl == "reference":
        import oracle
        masks, _, _ = oracle.build_routing(w["template"], w["percent"], w["routing_seed"],
                                           lengths, hk, g, True)
    else:
        masks, _, _ = tm.tilemix_build_routing(w["template"], w["percent"], w["routing_seed"],
                                               cu, hk, g, True)
    T = int(cu[-1])
    q, k, v = synth.make_qkv(rank, T, hq, hk, d, outliers=w["outliers"], lowrank=w["lowrank"])
    q_new = np.ascontiguousarray(q[cu[1:] - 1])          # the last position's query
    nbytes, attn_bytes = decode_bytes(lengths, hq, hk, d, masks, g)
    config = dict(bench_config(args, w, lengths, g), path="decode",
                  l2="inputs larger than L2: the steps rotate over %d copies of the cache "
                     "(%.0f MB; the step moves %.0f MB), no flush" % (
                         DECODE_CACHES, DECODE_CACHES * nbytes / 1e6, nbytes / 1e6))
    if args.impl == "reference":
        if rank == 0:
            t0 = time.perf_counter()
            steps = 0
            while steps < args.steps + args.warmup and (steps < 2 or time.perf_counter() - t0 < 60):
                oracle.decode_rows(q_new, k, v, cu[:-1], lengths, masks, cq[:-1], g)
                steps += 1
            dt = (time.perf_counter() - t0) / steps
            val = len(lengths) / dt
            print(json.dumps({"impl": "reference", "metric": DECODE_METRIC, "value": val,
                              "unit": "tok/s", "n_gpus": world, "steps": steps, "warmup": 0,
                              "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
                              "vs_baseline": None, "dtype": "f16+i8", "data": "synthetic",
                              "config": config,
                              "cpu_baseline": {"value": val, "unit": "tok/s", "cores": host_cores(),
                                               "kind": "oracle",
                                               "sample": "%d full decode steps" % steps},
                              "e2e": {"value": val, "unit": "tok/s", "h2d_bytes_per_step": 0,
                                      "d2h_bytes_per_step": 0}}), flush=True)
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    kd, vd, qd = t(k), t(v), t(q_new)
    k8 = torch.empty((T, hk, d), dtype=torch.int8, device=dev)
    ks = torch.empty((hk, int(ck[-1])), dtype=torch.float32, device=dev)
    cud, cqd, ckd = t(cu.astype(np.int32)), t(cq.astype(np.int32)), t(ck.astype(np.int32))
    tm.tilemix_quantize_qk(None, kd, cud, cqd, ckd, len(lengths), T, int(cq[-1]), int(ck[-1]),
                           hq, hk, d, None, None, k8, ks)     # the cache as prefill leaves it
    dec = tm.TileMixDecode(cu[:-1], lengths, ck[:-1], cq[:-1], hq, hk, d, masks, g, int(ck[-1]),
                           device=dev)
    od = torch.empty_like(qd)
    # Copies of the cache, used in turn: each step reads a cache the L2 has
    # not held since DECODE_CACHES - 1 other caches were read (the decode
    # inputs alone fit the L2).  A 256 MB write flush is measured too: it also
    # charges the step for writing the flushed lines back.
    caches = [(kd, vd, k8, ks)] + [(kd.clone(), vd.clone(), k8.clone(), ks.clone())
                                   for _ in range(DECODE_CACHES - 1)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for it in range(args.warmup):
        dec(qd, *caches[it % DECODE_CACHES], od)
    rc = tm.tilemix_get_error(stream)
    if rc != tm.OK:
        raise tm.TileMixError(rc, "warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for a, b in ev + kev:  # torch creates the CUDA event on first record: force it now
        a.record(stream)
        b.record(stream)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    for it, ((a, b), e) in enumerate(zip(ev, kev)):
        a.record(stream)
        dec(qd, *caches[it % DECODE_CACHES], od, events=e)
        b.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    # the same kernel after a 256 MB write flush (for comparison)
    n_fl = max(args.steps // 4, 3)
    kfl = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_fl)]
    for a, b in kfl:
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    for e in kfl:
        flush.zero_()
        dec(qd, kd, vd, k8, ks, od, events=e)
    torch.cuda.synchronize(dev)
    kern_ms_flush = max_over_ranks([sum(a.elapsed_time(b) for a, b in kfl) / n_fl], device=dev)[0]
    rc = tm.tilemix_get_error(stream)
    if rc != tm.OK:
        raise tm.TileMixError(rc, "timed steps")
    per_step = [a.elapsed_time(b) for a, b in ev]
    ms = sum(per_step) / args.steps
    kern_ms = sum(a.elapsed_time(b) for a, b in kev) / args.steps
    ms, kern_ms = max_over_ranks([ms, kern_ms], device=dev)
    # end to end: the new queries from pinned host memory in, O back out
    qh = torch.from_numpy(q_new).pin_memory()
    oh = torch.empty(q_new.shape, dtype=torch.float16).pin_memory()
    n_e2e = max(args.steps // 4, 3)
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_e2e)]
    torch.cuda.synchronize(dev)
    for it, (a, b) in enumerate(ev2):
        a.record(stream)
        qd.copy_(qh, non_blocking=True)
        dec(qd, *caches[it % DECODE_CACHES], od)
        oh.copy_(od, non_blocking=True)
        b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in ev2) / n_e2e], device=dev)[0]
    pk = peaks()
    tokens = whole_job_tokens(len(lengths), world)
    achieved = attn_bytes / (kern_ms / 1e3) / 1e9
    line = {
        "metric": DECODE_METRIC, "value": tokens / (ms / 1e3), "unit": "tok/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16+i8",
        "data": "synthetic", "config": config,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"],
                     "traffic": (kernel_traffic(args.workload, "decode_attn_kernel<128>")
                                 if not args.seqs else None),
                     "kernel": "decode_attn_kernel<128>", "kernel_ms": kern_ms,
                     "peak_kind": "copy bandwidth (%s)" % pk["source"],
                     "algorithmic_bytes": attn_bytes, "step_bytes": nbytes,
                     "kernel_ms_after_write_flush": kern_ms_flush,
                     "frac_after_write_flush": attn_bytes / (kern_ms_flush / 1e3) / 1e9 / pk["hbm_gbs"],
                     "step_frac": nbytes / (ms / 1e3) / 1e9 / pk["hbm_gbs"]},
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tok/s",
                "h2d_bytes_per_step": int(q_new.nbytes), "d2h_bytes_per_step": int(q_new.nbytes)},
        "gpu_launches": args.steps,  # one decode kernel per step (plus a memset of its counters)
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        import oracle
        t0 = time.perf_counter()
        n = 0
        while n < 1 or time.perf_counter() - t0 < 10.0:
            oracle.decode_rows(q_new, k, v, cu[:-1], lengths, masks, cq[:-1], g)
            n += 1
        dt = (time.perf_counter() - t0) / n
        line["cpu_baseline"] = {"value": len(lengths) / dt, "unit": "tok/s", "cores": host_cores(),
                                "kind": "oracle",
                                "sample": "%d full decode steps of the workload" % n}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------------- route path ---

ROUTE_METRIC = "pooled-score adaptive routing tok/s at 4k b8 (3B GQA shape); % of HBM roofline"


def run_route(args):
    """Pooled-score routing words for the whole batch per step.  Its inputs
    (Q and K, fp16) exceed the 126 MB L2, so no flush."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference" and rank != 0:
        return
    w, lengths, g = workload(args.workload, args.template, args.percent, args.seqs)
    hq, hk, d = w["hq"], w["hk"], w["d"]
    T = sum(lengths)
    q, k, _ = synth.make_qkv(rank, T, hq, hk, d, outliers=w["outliers"], lowrank=w["lowrank"])
    cq, ck = tile_starts(lengths)
    # algorithmic bytes: Q and K read once, the fp32 means written and read
    # once, the words written
    nbytes = (q.nbytes + k.nbytes + 2 * (int(cq[-1]) + int(ck[-1])) * hk * d * 4 +
              int(cq[-1]) * hk * 8)
    config = dict(bench_config(args, w, lengths, g), path="route",
                  l2="no flush: Q and K (%.0f MB per step) exceed the 126 MB L2"
                     % ((q.nbytes + k.nbytes) / 1e6))
    sample = lengths[:1]
    if args.impl == "reference" or not args.no_cpu_baseline:
        from oracle import adaptive
        Ts = sample[0]
        t0 = time.perf_counter()
        n = 0
        while n < 1 or time.perf_counter() - t0 < (60.0 if args.impl == "reference" else 10.0):
            adaptive.route_pooled(q[:Ts], k[:Ts], sample, hq, hk, g[:1], w["causal"],
                                  w["percent"])
            n += 1
        cpu_val = Ts / ((time.perf_counter() - t0) / n)
        cpu_base = {"value": cpu_val, "unit": "tok/s", "cores": 1, "kind": "oracle",
                    "sample": "%d runs on the first sequence (%d tokens) of the batch" % (n, Ts)}
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "metric": ROUTE_METRIC, "value": cpu_val,
                              "unit": "tok/s", "n_gpus": world, "steps": n, "warmup": 0,
                              "ms_per_step": T / cpu_val * 1e3, "higher_is_better": True,
                              "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                              "data": "synthetic", "config": config, "cpu_baseline": cpu_base,
                              "e2e": {"value": cpu_val, "unit": "tok/s", "h2d_bytes_per_step": 0,
                                      "d2h_bytes_per_step": 0}}), flush=True)
            return
    import torch
    import torch.distributed as dist

    import tile_routed_mixed_b200 as tm
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    qd, kd = torch.from_numpy(q).to(dev), torch.from_numpy(k).to(dev)
    stream = torch.cuda.current_stream(dev)
    ws = None
    for _ in range(args.warmup):
        m = tm.route_pooled(qd, kd, lengths, hq, hk, g, w["causal"], w["percent"], workspace=ws)
        ws = m._route_keepalive[-1]
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for a, b in ev:
        a.record(stream)
        b.record(stream)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for e in ev:
        tm.route_pooled(qd, kd, lengths, hq, hk, g, w["causal"], w["percent"], events=e,
                        workspace=ws)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    rc = tm.tilemix_get_error(stream)
    if rc != tm.OK:
        raise tm.TileMixError(rc, "timed steps")
    ms = e0.elapsed_time(e1) / args.steps
    kern_ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    ms, kern_ms = max_over_ranks([ms, kern_ms], device=dev)
    # end to end: Q and K from pinned host memory in, the words back out
    qh, kh = torch.from_numpy(q).pin_memory(), torch.from_numpy(k).pin_memory()
    n_e2e = max(args.steps // 4, 3)
    words_h = None
    torch.cuda.synchronize(dev)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(n_e2e):
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        m = tm.route_pooled(qd, kd, lengths, hq, hk, g, w["causal"], w["percent"], workspace=ws)
        words_h = m.to("cpu", non_blocking=True)
    e3.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks([e2.elapsed_time(e3) / n_e2e], device=dev)[0]
    pk = peaks()
    tokens = whole_job_tokens(T, world)
    achieved = nbytes / (kern_ms / 1e3) / 1e9
    line = {
        "metric": ROUTE_METRIC, "value": tokens / (ms / 1e3), "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"],
                     "traffic": None, "kernel": "route_pool_kernel x2 + route_words_kernel",
                     "kernel_ms": kern_ms, "peak_kind": "copy bandwidth (%s)" % pk["source"],
                     "algorithmic_bytes": nbytes},
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tok/s",
                "h2d_bytes_per_step": int(q.nbytes + k.nbytes),
                "d2h_bytes_per_step": int(words_h.numel() * 8)},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_base
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# -------------------------------------------------------------- mass path ---

MASS_METRIC = "importance-mass exposure probe tok/s at 4k b8 (3B GQA shape); % of FP16 tensor peak"


def mass_flops(lengths, hq, d, causal):
    """Score FLOPs of the probe: two sweeps over each 64-row block's legal key tiles."""
    f = 0
    for L in lengths:
        for b in range((L + 63) // 64):
            last = ((min(64 * b + 64, L) - 1) // 64) if causal else (L - 1) // 64
            f += (last + 1) * 64 * 64 * 2 * d
    return 2 * f * hq


def run_mass(args):
    """The probe over the whole batch per step (the bench's routing words),
    plus the batch exposure for several routings (computed once, untimed)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference" and rank != 0:
        return
    w, lengths, g = workload(args.workload, args.template, args.percent, args.seqs)
    hq, hk, d, causal = w["hq"], w["hk"], w["d"], w["causal"]
    T = sum(lengths)
    q, k, _ = synth.make_qkv(rank, T, hq, hk, d, outliers=w["outliers"], lowrank=w["lowrank"])
    config = dict(bench_config(args, w, lengths, g), path="mass", delta_log2=4.0,
                  l2="no flush: Q and K (%.0f MB per step) exceed the 126 MB L2"
                     % ((q.nbytes + k.nbytes) / 1e6))
    flops = mass_flops(lengths, hq, d, causal)
    cpu_base = None
    if args.impl == "reference" or not args.no_cpu_baseline:
        import oracle
        from oracle import mass as om
        Ls = min(lengths[0], 1024)
        sm, _, _ = oracle.build_routing(w["template"], w["percent"], w["routing_seed"], [Ls], hk,
                                        g[:1], causal)
        t0 = time.perf_counter()
        n = 0
        while n < 1 or time.perf_counter() - t0 < 10.0:
            om.probe_rows(q[:Ls], k[:Ls], sm, g[:1], [Ls], causal)
            n += 1
        dt = (time.perf_counter() - t0) / n
        # tokens/s scaled by the causal work: a 4096-row sequence costs 16x a 1024-row one
        scale = sum((L / Ls) ** 2 for L in lengths)
        cpu_val = T / (dt * scale)
        cpu_base = {"value": cpu_val, "unit": "tok/s", "cores": host_cores(), "kind": "oracle",
                    "sample": "%d runs on the first %d tokens of sequence 0, scaled by the batch's "
                              "quadratic work" % (n, Ls)}
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "metric": MASS_METRIC, "value": cpu_val,
                              "unit": "tok/s", "n_gpus": world, "steps": n, "warmup": 0,
                              "ms_per_step": T / cpu_val * 1e3, "higher_is_better": True,
                              "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                              "data": "synthetic", "config": config, "cpu_baseline": cpu_base,
                              "e2e": {"value": cpu_val, "unit": "tok/s", "h2d_bytes_per_step": 0,
                                      "d2h_bytes_per_step": 0}}), flush=True)
            return
    import torch
    import torch.distributed as dist

    import tile_routed_mixed_b200 as tm
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    cu = synth.cu_seqlens_of(lengths)
    masks, _, _ = tm.tilemix_build_routing(w["template"], w["percent"], w["routing_seed"], cu, hk,
                                           g, causal)
    qd, kd = torch.from_numpy(q).to(dev), torch.from_numpy(k).to(dev)
    md = torch.from_numpy(np.ascontiguousarray(masks).view(np.int64)).to(dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        tm.mass_probe(qd, kd, md, lengths, hq, hk, g, causal)
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for a, b in ev:
        a.record(stream)
        b.record(stream)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for e in ev:
        tm.mass_probe(qd, kd, md, lengths, hq, hk, g, causal, events=e)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    rc = tm.tilemix_get_error(stream)
    if rc != tm.OK:
        raise tm.TileMixError(rc, "timed steps")
    ms = e0.elapsed_time(e1) / args.steps
    kern_ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    ms, kern_ms = max_over_ranks([ms, kern_ms], device=dev)
    # end to end: Q and K from pinned host memory in, the three row arrays out
    qh, kh = torch.from_numpy(q).pin_memory(), torch.from_numpy(k).pin_memory()
    n_e2e = max(args.steps // 4, 3)
    torch.cuda.synchronize(dev)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    out_bytes = 0
    for _ in range(n_e2e):
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        outs = tm.mass_probe(qd, kd, md, lengths, hq, hk, g, causal)
        hosts = [x.to("cpu", non_blocking=True) for x in outs]
        out_bytes = sum(x.numel() * 4 for x in hosts)
    e3.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks([e2.elapsed_time(e3) / n_e2e], device=dev)[0]
    # exposure of several routings of this batch (untimed)
    expo = {}
    for tpl, pct in (("sptrans", 25), ("sptrans", 50), ("sptrans", 75), ("adaptive", 25),
                     ("adaptive", 75)):
        if tpl == "adaptive":
            mw = tm.route_pooled(qd, kd, lengths, hq, hk, g, causal, pct)
        else:
            mm, _, _ = tm.tilemix_build_routing(tpl, pct, w["routing_seed"], cu, hk, g, causal)
            mw = torch.from_numpy(np.ascontiguousarray(mm).view(np.int64)).to(dev)
        m8, hh, h8 = tm.mass_probe(qd, kd, mw, lengths, hq, hk, g, causal)
        expo["%s%d" % (tpl, pct)] = {
            "int8_share_of_high_importance_mass": float(h8.double().sum() / hh.double().sum()),
            "int8_share_of_all_mass": float(m8.double().mean())}
    pk = peaks()
    tokens = whole_job_tokens(T, world)
    achieved = flops / (kern_ms / 1e3) / 1e12
    line = {
        "metric": MASS_METRIC, "value": tokens / (ms / 1e3), "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": config,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"], "traffic": None,
                     "kernel": "mass_probe_kernel<128>", "kernel_ms": kern_ms,
                     "peak_kind": "dense bf16 burst (%s), fp16 taken at the same rate" % pk["source"],
                     "score_flops": flops},
        "exposure": expo,
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tok/s",
                "h2d_bytes_per_step": int(q.nbytes + k.nbytes), "d2h_bytes_per_step": int(out_bytes)},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and cpu_base is not None:
        line["cpu_baseline"] = cpu_base
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# --------------------------------------------------------------- mad path ---

def run_mad(args):
    """Mean absolute deviation of the GPU prefill output from the all-FP16
    oracle (fp64) at each coverage of the workload's template, for INT8 and
    FP8 low tiles, on sampled rows (every q-tile's first, middle and last row
    of three heads plus random rows).  A report, not a timed bench line."""
    import torch

    import oracle
    import tile_routed_mixed_b200 as tm
    from oracle import fp8 as of8
    from tests import gpu_cases as gc

    w, lengths, g = workload(args.workload, args.template, args.percent, args.seqs)
    case = gc.Case.workload(args.workload)
    q, k, v = case.inputs()
    rows = gc.sample_rows(case.lengths, case.hq, seed=3, per_head_random=16,
                          heads={0, case.hq // 2, case.hq - 1}, tiles_per_head=16)
    zero = case.masks(0)
    q8, qs = oracle.quantize_q(q, case.lengths)
    k8, ks = oracle.quantize_k(k, case.lengths)
    ref, _ = oracle.attention_rows(q, k, v, q8, qs, k8, ks, zero, case.g, case.lengths,
                                   case.causal, rows=rows)
    qd, kd, vd = (torch.from_numpy(x).cuda() for x in (q, k, v))
    out = {}
    for low in ("int8", "fp8", "int4"):
        for pct in (0, 10, 25, 50, 75, 100):
            masks = oracle.build_routing(case.template, pct, case.routing_seed, case.lengths,
                                         case.hk, case.g, case.causal)[0]
            pf = tm.TileMixPrefill(case.lengths, case.hq, case.hk, case.d, masks, case.g,
                                   causal=case.causal, low=low)
            o = pf(qd, kd, vd).cpu().numpy()
            got = gc.gather(case, o, rows).astype(np.float64)
            out["%s_%d" % (low, pct)] = float(np.mean(np.abs(got - ref)))
    print(json.dumps({"report": "mean abs deviation of the fp16 output from the all-FP16 oracle",
                      "workload": args.workload, "template": case.template,
                      "rows_sampled": int(rows.shape[0]), "mad": out}), flush=True)


def run_mma(args):
    """Dense rate of each MMA form the fused kernel issues (tcgen05.mma, M128,
    issued back to back by one thread per CTA on every SM; tilemix_mma_rate):
    SM cycles per MMA and TFLOP/s (TOP/s) at the clock the run saw, and the
    INT8 : FP16 and FP8 : FP16 rate ratios the mixed roofline uses."""
    import torch
    import tile_routed_mixed_b200 as tm
    torch.cuda.init()
    uuid = str(torch.cuda.get_device_properties(0).uuid)
    smi = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    smi.start()
    rows = []
    for form, k in (("f16", 16), ("i8", 32), ("f8", 32), ("f16_tmem_a", 16)):
        for n in (64, 128, 256):
            r = tm.mma_rate(form, n, iters=4096)
            r["k"] = k
            r["macs_per_cycle"] = 128 * n * k / r["cycles_per_mma"]
            rows.append(r)
    clocks = smi.stop()
    by = {(r["form"], r["n"]): r for r in rows}
    ratio = lambda a, b: by[(a, 256)]["macs_per_cycle"] / by[(b, 256)]["macs_per_cycle"]
    line = {"metric": "tcgen05.mma dense rate of the fused kernel's MMA forms (M128, every SM)",
            "value": ratio("i8", "f16"), "unit": "INT8 : FP16 rate (N256)",
            "fp8_over_fp16": ratio("f8", "f16"), "forms": rows, "clocks": clocks,
            "n_gpus": 1, "data": "synthetic"}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["tilemix", "reference"], default="tilemix")
    ap.add_argument("--workload", default="llama3b_4k_b8", choices=list(synth.WORKLOADS))
    ap.add_argument("--template", default=None)
    ap.add_argument("--percent", type=int, default=None)
    ap.add_argument("--low", choices=["int8", "fp8", "int4"], default="int8",
                    help="low-precision path of bit-1 tiles in the prefill bench (fp8 = e4m3)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seqs", type=int, default=None,
                    help="keep only the first N sequences of the workload (profiler captures)")
    ap.add_argument("--path", choices=["prefill", "decode", "route", "mass", "mad", "mma"],
                    default="prefill",
                    help="prefill (the headline metric), the decode step with the INT8 K "
                         "cache, pooled-score adaptive routing, the importance-mass probe, "
                         "the deviation table, or the tcgen05 rate of the kernel's MMA forms")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.path == "decode":
        run_decode(args)
    elif args.path == "route":
        run_route(args)
    elif args.path == "mass":
        run_mass(args)
    elif args.path == "mad":
        run_mad(args)
    elif args.path == "mma":
        run_mma(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
