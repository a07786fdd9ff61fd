#!/usr/bin/env python
"""Throughput benchmark of the LoLA hybrid-attention inference step on B200.

One step = one pass of the whole hot path over one batch: reset the state, then
one chunkwise prefill call over the workload's sequence (feature map, SRE
scoring, top-lambda selection, fold, attention output, cache/window update).
`value` is whole-job prefill tokens/s with inputs resident in HBM; `e2e` is the
same through the C ABI with host buffers (H2D of q,k,v and D2H of the output
inside the timed region). Decode measurements (batched decode, and single-
sequence decode after the long-context prefill) are attached under "decode".
Every timed number comes from CUDA events on the launching stream, with L2
flushed (a 256 MiB write) between timed iterations.

The default workload is the 8B-shaped prefill (B 4, 32/8 heads, head dim 128,
16384 tokens), the configuration the tensor-peak target is stated on.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from hybrid_linear_attention_lola_b200 import workloads as wl  # noqa: E402
from hybrid_linear_attention_lola_b200.lola import SCHEDULES  # noqa: E402

METRIC = "LoLA prefill & decode tokens/sec on 1xB200; % of tensor/HBM roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes per launch of a kernel, copied from ncu captures (profiles/dram_traffic.json);
# an entry counts only while the kernel's source file is unchanged since its capture
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")
_CSRC = "hybrid_linear_attention_lola_b200/csrc/"
_HEADERS = (_CSRC + "umma.cuh", _CSRC + "lola_internal.cuh")
KERNEL_SOURCES = {"attn": (_CSRC + "attn_ws.cu",) + _HEADERS,
                  "chain": (_CSRC + "chain_tc.cu", _CSRC + "scoring.cuh") + _HEADERS,
                  "decode": (_CSRC + "decode.cu",) + _HEADERS}


# ---------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def host_cores() -> int:
    return len(os.sched_getaffinity(0))


def source_sha(rels) -> str:
    """Hash of a kernel's source files (its .cu and the headers it includes)."""
    import hashlib
    h = hashlib.sha256()
    for rel in ((rels,) if isinstance(rels, str) else rels):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def captured_traffic(kernel: str, workload: str, units=None):
    """DRAM bytes (read + write) per launch of `kernel` on `workload` from the
    committed ncu summary, or (None, reason) when there is none for the current
    source of the kernel. An entry that stores bytes per unit of work (one interval
    of one stream) is scaled to a launch of `units` such units."""
    try:
        with open(TRAFFIC_FILE) as f:
            entries = json.load(f)
    except (OSError, ValueError):
        return None, "no ncu capture committed"
    for e in entries:
        if e.get("kernel") == kernel and e.get("workload") == workload:
            src = KERNEL_SOURCES.get(kernel)
            if src is None or e.get("source_sha") != source_sha(src):
                return None, "kernel changed since its ncu capture"
            if units is not None and e.get("dram_bytes_per_unit") is not None:
                return (round(e["dram_bytes_per_unit"] * units),
                        f"ncu capture (profiles/dram_traffic.json) of {e['captured_launch']}, "
                        f"scaled to this launch by its {units} units ({e['unit']})")
            if e.get("dram_bytes_per_launch") is None:
                return None, "no ncu capture of the kernel's current launch form"
            return e["dram_bytes_per_launch"], "ncu capture (profiles/dram_traffic.json)"
    return None, "no ncu capture for this kernel and workload"


def interval_sizes(w, T, lam=None):
    """Per-interval (nS_before, nL, nK) of a fresh-state prefill of T tokens."""
    lam = w.lambda_ if lam is None else lam
    out = []
    nS = 0
    for t0 in range(0, T, w.chunk):
        t1 = t0 + w.chunk
        lo = max(0, t0 - w.window)
        hi = max(lo, t1 - w.window)
        nL = hi - lo
        nK = min(lam, nS + nL)
        out.append((nS, nL, nK))
        nS = nK
    return out


def prefill_flops(w, T):
    """Algorithmic FLOPs of one prefill call, per phase (exact interval sizes):
    attn: 4 d (|cache| + window) softmax + 2 D (d+1) readout + (C+1)(D+d+1) band linear,
          per query head and token;
    chain: 2 D (d+1) per scored candidate (SRE) and per folded pair (fold), per kv-head;
    phi: 2 d D/2 per q and k row."""
    B, Hq, Hkv, d, D, C = w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.feat_dim, w.chunk
    attn = chain = 0.0
    for ci, (nS, nL, nK) in enumerate(interval_sizes(w, T)):
        t0 = ci * C
        win = min(w.window, t0)
        attn += C * B * Hq * (4 * d * (nK + win) + 2 * D * (d + 1) + (C + 1) * (D + d + 1))
        nQ = nS + nL
        chain += B * Hkv * 2 * D * (d + 1) * (nQ + (nQ - nK))
    phi = 2.0 * d * (D // 2) * B * T * (Hq + Hkv)
    return {"attn": attn, "chain": chain, "phi": phi}


def decode_bytes_per_step(w):
    """Algorithmic HBM bytes of one decode step (all streams), steady state:
    cache K/V + band K/V + [H|s] fp32 + q/out + new k/v, plus the interval
    update amortised over its decode_interval steps."""
    d, D, lam, eta, Cd = w.head_dim, w.feat_dim, w.lambda_, w.window, w.decode_interval
    e = 2 if w.dtype == "bf16" else 4
    g = w.group
    per = (lam * 2 * d * e + (eta + (Cd + 1) / 2) * 2 * d * e + D * (d + 1) * 4
           + 2 * g * d * e + 2 * d * e)
    per += ((lam + Cd) * 2 * d * e + 2 * D * (d + 1) * 4 + Cd * 2 * d * e) / Cd
    return per * w.batch * w.n_kv_heads


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    Q = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    # raw samples go to LOLA_CLOCKS_DIR (default: the system temp directory)
    def __init__(self, bus_id=None):
        self.bus_id = (bus_id or "").lower()
        self.proc = None
        out_dir = os.environ.get("LOLA_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"lola_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                if self.bus_id and self.bus_id not in parts[1].lower():
                    continue
                rows.append(parts)
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- distributed

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = os.environ.get("LOLA_BENCH_BACKEND", "nccl")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (identity at world size 1)."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, ws: int, seconds_max: float) -> float:
    """Weak scaling: every rank processes the same amount of independent work."""
    return units_per_rank * ws / seconds_max


# ---------------------------------------------------------------- oracle baseline

def cpu_baseline(w, budget_s=15.0, threads=None, single_thread=True):
    """Times the oracle, as it stands, on a bounded sample of the workload:
    a subset of (batch, kv-head) streams over a prefix of the sequence."""
    import numpy as np
    import oracle
    cores = threads or host_cores()
    T = w.seq_len
    # rough fp64 cost per stream to size the sample
    d, D, lam, eta, g = w.head_dim, w.feat_dim, w.lambda_, w.window, w.group
    per_tok = g * (4 * d * (lam + eta) + 2 * D * d) + 2 * D * d * (lam + w.chunk) / w.chunk
    rate = 1.0e9  # fp64 FLOP/s per thread, conservative
    Ts = T
    while Ts > w.chunk * 4 and per_tok * Ts / rate > budget_s:
        Ts //= 2
    Ts -= Ts % w.chunk
    ns_total = w.batch * w.n_kv_heads
    n_streams = max(1, min(ns_total, cores))
    q, k, v, _ = wl.make_inputs(w, T=Ts, batch=1)
    W = wl.make_W(w)
    hsel = list(range(min(n_streams, w.n_kv_heads)))
    qsel = [h * g + r for h in hsel for r in range(g)]
    qs, ks, vs = q[:, :, qsel], k[:, :, hsel], v[:, :, hsel]
    ints = [w.chunk] * (Ts // w.chunk)
    t = time.perf_counter()
    oracle.run(qs, ks, vs, W, window=w.window, lambda_=w.lambda_, intervals=ints, eps=w.eps, threads=cores)
    dt = time.perf_counter() - t
    frac = len(hsel) / w.n_kv_heads
    tokens = Ts * frac            # prefill tokens of one sequence, all heads equivalent
    out = {"value": tokens / dt, "unit": UNIT, "cores": min(cores, len(hsel)), "kind": "oracle",
           "sample": f"{w.name}: batch 1 of {w.batch}, kv-heads {len(hsel)} of {w.n_kv_heads} "
                     f"(with their {g} query heads each), first {Ts} of {T} tokens; "
                     f"{dt:.2f} s wall, fp64 C oracle"}
    if single_thread and len(hsel) > 1:
        # the same prefix of one stream on one thread
        t = time.perf_counter()
        oracle.run(qs[:, :, :g], ks[:, :, :1], vs[:, :, :1], W, window=w.window, lambda_=w.lambda_,
                   intervals=ints, eps=w.eps, threads=1)
        dt1 = time.perf_counter() - t
        out["single_thread"] = {"value": (Ts / w.n_kv_heads) / dt1, "unit": UNIT, "cores": 1,
                                "sample": f"kv-head 0 of batch 0, first {Ts} tokens; {dt1:.2f} s wall"}
    return out


# ---------------------------------------------------------------- roofline

def prefill_roofline(w, T, ms_step, phase_ms, steps, peaks, peak_src, launch_intervals=None):
    """Headline: the whole prefill step's algorithmic FLOPs over its time, against the
    measured bf16 tensor peak (burst; the sustained figure beside it). Per phase: the
    attention (tensor-bound contractions) and the chain (sequential per stream: its
    FLOPs over its time are a latency figure, not a tensor-pipe one)."""
    fl = prefill_flops(w, T)
    total = sum(fl.values())
    burst = float(peaks["bf16_tflops"])
    sust = float(peaks.get("bf16_tflops_sustained", burst))
    ach = total / (ms_step / 1e3) / 1e12
    per_call = {ph: v[0] / steps for ph, v in phase_ms.items() if v[1]}
    phases = {}
    for ph, bound in (("attn", "tensor"), ("chain", "latency (sequential intervals per stream)"),
                      ("phi", "hbm")):
        if ph not in per_call:
            continue
        a = fl[ph] / (per_call[ph] / 1e3) / 1e12
        phases[ph] = {"ms_per_call": round(per_call[ph], 4), "tflop_per_call": round(fl[ph] / 1e12, 5),
                      "achieved_tflops": round(a, 3), "frac_of_burst": round(a / burst, 5),
                      "frac_of_sustained": round(a / sust, 5), "bound": bound}
    # traffic of the dominant kernel (the phase with the most device time)
    dom = max((p for p in ("attn", "chain") if p in per_call), key=per_call.get, default="attn")
    streams = w.batch * w.n_kv_heads
    units = launch_intervals * streams if launch_intervals else None
    traffic, tsrc = captured_traffic(dom, w.name, units)
    if w != wl.WORKLOADS.get(w.name):
        traffic, tsrc = None, "workload overridden on the command line (no capture for it)"
    return {"bound": "tensor", "kernel": f"whole prefill step (dominant kernel: {dom})",
            "achieved": round(ach, 3), "peak": burst, "unit": "TFLOP/s", "frac": round(ach / burst, 5),
            "frac_of_sustained": round(ach / sust, 5), "peak_sustained": sust,
            "traffic": traffic, "traffic_kernel": dom, "traffic_source": tsrc,
            "traffic_launch": (f"{launch_intervals} intervals x {streams} streams" if launch_intervals else None),
            "peak_source": f"{peak_src} bf16 dense (burst; sustained beside it)",
            "algorithmic_tflop_per_step": round(total / 1e12, 5), "phases": phases,
            "phase_ms": {ph: round(v, 4) for ph, v in per_call.items()}}


def memory_report(w, cfg_bytes_per_stream):
    """State + cache bytes (constant in T) against a full key/value cache of the
    same heads at the workload's length."""
    e = 2 if w.dtype == "bf16" else 4
    per_seq = cfg_bytes_per_stream * w.n_kv_heads
    full = w.seq_len * w.n_kv_heads * w.head_dim * 2 * e
    return {"state_cache_bytes_per_stream": cfg_bytes_per_stream,
            "state_cache_bytes_per_sequence": per_seq,
            "full_kv_bytes_per_sequence": full, "seq_len": w.seq_len,
            "full_kv_over_state_cache": round(full / per_seq, 3)}


# ---------------------------------------------------------------- engine arm

def run_engine(args, ws, rank, local):
    import numpy as np
    import torch
    from hybrid_linear_attention_lola_b200 import build as B
    from hybrid_linear_attention_lola_b200 import lola as L

    B.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    w = wl.WORKLOADS[args.workload]
    if args.batch:
        w = w.replace(batch=args.batch)
    T = w.seq_len
    q, k, v, _ = wl.make_inputs(w, T=T)
    W = wl.make_W(w)
    w_job = w                    # the whole job's workload (all ranks)
    shard = None
    if args.shard and ws > 1:
        # this rank's block of the batch's (sequence, kv-head) streams (strong scaling)
        from hybrid_linear_attention_lola_b200 import shard as SH
        shard = SH.partition(w.batch, w.n_q_heads, w.n_kv_heads, ws, rank)
        q = np.ascontiguousarray(q[shard.b0:shard.b1, :, shard.h0 * shard.g:shard.h1 * shard.g])
        k = np.ascontiguousarray(k[shard.b0:shard.b1, :, shard.h0:shard.h1])
        v = np.ascontiguousarray(v[shard.b0:shard.b1, :, shard.h0:shard.h1])
        if w.w_per_head:
            W = np.ascontiguousarray(W[shard.h0:shard.h1])
        w = w.replace(batch=shard.batch, n_kv_heads=shard.n_kv_heads, n_q_heads=shard.n_q_heads)
    cfg = L.config_from_workload(w, max_prefill_tokens=T)
    S = L.LolaState(cfg, torch.from_numpy(W), dev)
    S.set_prefill_schedule(args.prefill_schedule, args.segment_intervals)
    mode, seg_len, nseg = L.lola_prefill_plan(cfg, T, args.prefill_schedule, args.segment_intervals,
                                              torch.cuda.get_device_properties(dev).multi_processor_count)
    sched = (f"{args.prefill_schedule}: {mode}, {nseg} segments of {seg_len} intervals per call"
             if nseg > 1 else f"{args.prefill_schedule}: one segment")
    dt = S.dtype
    qd = torch.from_numpy(q).to(dev, dt)
    kd = torch.from_numpy(k).to(dev, dt)
    vd = torch.from_numpy(v).to(dev, dt)
    out = torch.empty_like(qd)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        S.reset()
        S.prefill(qd, kd, vd, out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    L.lola_timing_read(S.handle)
    L.lola_set_timing(S.handle, True)
    phase_ms = {}
    props = torch.cuda.get_device_properties(dev)
    bus = None
    if isinstance(getattr(props, "pci_bus_id", None), int):
        bus = f"{props.pci_bus_id:02x}:{getattr(props, 'pci_device_id', 0):02x}."
    clocks = ClockSampler(bus).start() if rank == 0 else None
    barrier(ws)
    torch.cuda.synchronize(dev)
    launches0 = L.lola_launch_count()
    times = []
    for _ in range(args.steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
        for ph, (ms, n) in L.lola_timing_read(S.handle).items():
            a = phase_ms.setdefault(ph, [0.0, 0])
            a[0] += ms
            a[1] += n
    torch.cuda.synchronize(dev)
    launches = L.lola_launch_count() - launches0
    barrier(ws)
    clk = clocks.stop() if clocks else None
    L.lola_set_timing(S.handle, False)
    ms_step = max_over_ranks(sum(times) / len(times), ws, dev)
    # tokens of the whole job: every rank's own batch (replicas), or one batch split
    # over the ranks (shard)
    job_tokens = w_job.batch * T if shard is not None else w.batch * T * ws
    value = job_tokens / (ms_step / 1e3)

    roofline = prefill_roofline(w, T, ms_step, phase_ms, args.steps, peaks, peak_src,
                                launch_intervals=seg_len if nseg > 1 else T // w.chunk)

    # end to end through the C ABI from pinned host memory: lola_prefill_host copies every
    # input to the device and every output back inside the timed region, overlapping the
    # copies of one piece of the sequence with the compute of the next
    qh = torch.from_numpy(q).to(dt).pin_memory()
    kh = torch.from_numpy(k).to(dt).pin_memory()
    vh = torch.from_numpy(v).to(dt).pin_memory()
    oh = torch.empty(qh.shape, dtype=dt).pin_memory()
    h2d = qh.numel() * qh.element_size() + kh.numel() * kh.element_size() * 2
    d2h = oh.numel() * oh.element_size()
    piece = max(w.chunk, (T // max(1, args.e2e_pieces)) // w.chunk * w.chunk)
    staging = torch.empty(L.lola_prefill_host_staging_bytes(S.cfg, piece), dtype=torch.uint8, device=dev)

    def e2e_step():
        S.reset()
        S.prefill_host(qh, kh, vh, oh, piece, staging)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier(ws)
    et = []
    for _ in range(args.steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_step()
        e1.record(stream)
        e1.synchronize()
        et.append(e0.elapsed_time(e1))
    barrier(ws)
    e2e_ms = max_over_ranks(sum(et) / len(et), ws, dev)
    e2e = {"value": job_tokens / (e2e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
           "api": "lola_prefill_host", "piece_tokens": piece}
    S.close()
    del qd, kd, vd, out

    decode = []
    for dname in [x for x in args.decode_workload.split(",") if x and x != "none"]:
        dres = run_decode(args, dname, ws, rank, dev, flush, peaks, peak_src)
        launches += dres.pop("_launches")
        decode.append(dres)
    sb = L.lola_state_stream_bytes(cfg)

    line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "strong" if shard is not None else "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": f"{w_job.name} prefill", "batch": w_job.batch,
                       "seq_len": T, "n_q_heads": w_job.n_q_heads, "n_kv_heads": w_job.n_kv_heads,
                       "head_dim": w.head_dim, "feat_dim": w.feat_dim, "window": w.window,
                       "lambda": w.lambda_, "chunk": w.chunk,
                       "prefill_schedule": sched,
                       "parallelism": (f"streams sharded over {ws} ranks by {shard.by} (no collective on the "
                                       f"data path)" if shard is not None
                                       else f"replicas x{ws} (independent streams, no collective)"),
                       "l2": "flushed (256 MiB write) before every timed step"},
            "roofline": roofline, "e2e": e2e, "gpu_launches": launches, "clocks": clk,
            "decode": decode, "memory": memory_report(w, sb)}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_decode(args, name, ws, rank, dev, flush, peaks, peak_src):
    """Decode on workload `name`: prefill the prefix (untimed), then time every decode
    step (L2 flushed before each). Tokens/s = batch / step time."""
    import torch
    from hybrid_linear_attention_lola_b200 import lola as L
    w = wl.WORKLOADS[name]
    if args.decode_prefix:
        w = w.replace(seq_len=args.decode_prefix)
    if args.decode_steps:
        w = w.replace(decode_steps=min(args.decode_steps, w.decode_steps))
    Tp, n_dec = w.seq_len, w.decode_steps
    q, k, v, _ = wl.make_inputs(w, T=Tp)
    qn, kn, vn, _ = wl.make_inputs(w, part="decode")
    W = wl.make_W(w)
    piece = min(Tp, 512)          # the untimed prefix is prefilled in calls of this many tokens
    cfg = L.config_from_workload(w, max_prefill_tokens=piece)
    S = L.LolaState(cfg, torch.from_numpy(W), dev)
    dt = S.dtype
    qd, kd, vd = (torch.from_numpy(x).to(dev, dt) for x in (q, k, v))
    qs, ks, vs = (torch.from_numpy(x).to(dev, dt) for x in (qn, kn, vn))
    outp = torch.empty_like(qd[:, :piece])
    outd = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=dt, device=dev)
    stream = torch.cuda.current_stream(dev)
    qsteps = [qs[:, t].contiguous() for t in range(n_dec)]
    ksteps = [ks[:, t].contiguous() for t in range(n_dec)]
    vsteps = [vs[:, t].contiguous() for t in range(n_dec)]

    def prefix():
        S.reset()
        for t0 in range(0, Tp, piece):
            S.prefill(qd[:, t0:t0 + piece].contiguous(), kd[:, t0:t0 + piece].contiguous(),
                      vd[:, t0:t0 + piece].contiguous(), outp)

    for _ in range(max(1, args.warmup)):          # warm-up passes over the decode steps
        prefix()
        for t in range(n_dec):
            S.decode(qsteps[t], ksteps[t], vsteps[t], outd)
    prefix()
    torch.cuda.synchronize(dev)
    L.lola_timing_read(S.handle)
    L.lola_set_timing(S.handle, True)
    barrier(ws)
    l0 = L.lola_launch_count()
    times = []
    ph = {}
    for t in range(n_dec):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        S.decode(qsteps[t], ksteps[t], vsteps[t], outd)
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
        for name, (ms, n) in L.lola_timing_read(S.handle).items():
            a = ph.setdefault(name, [0.0, 0])
            a[0] += ms
            a[1] += n
    launches = L.lola_launch_count() - l0
    barrier(ws)
    L.lola_set_timing(S.handle, False)
    ms_step = max_over_ranks(sum(times) / len(times), ws, dev)
    sb = L.lola_state_stream_bytes(cfg)
    bytes_step = decode_bytes_per_step(w)
    dec_ms = ph["decode"][0] / ph["decode"][1]
    upd = ph.get("update", [0.0, 0])
    achieved = bytes_step / (ms_step / 1e3) / 1e9
    peak = float(peaks["hbm_gbs"])
    S.close()
    return {"workload": f"{w.name}: prefix {Tp} prefilled, "
                        f"{n_dec} timed decode steps, interval {w.decode_interval}",
            "prefix_prefill_calls_of": piece,
            "value": round(whole_job_rate(w.batch, ws, ms_step / 1e3), 1), "unit": UNIT,
            "ms_per_step": round(ms_step, 5), "batch": w.batch,
            "roofline": {"bound": "hbm", "kernel": "whole decode step", "achieved": round(achieved, 1),
                         "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": captured_traffic("decode", w.name)[0],
                         "traffic_source": captured_traffic("decode", w.name)[1],
                         "peak_source": f"{peak_src} HBM copy",
                         "algorithmic_bytes_per_step": bytes_step,
                         "phase_ms": {"decode_attn": round(dec_ms, 5),
                                      "interval_update_per_interval": round(upd[0] / max(upd[1], 1), 5),
                                      "append": round(ph["append"][0] / ph["append"][1], 5)}},
            "memory": memory_report(w, sb),
            "l2": "flushed before every timed step", "_launches": launches}


# ---------------------------------------------------------------- reference arm

def run_reference(args, ws, rank):
    """The oracle, as it stands, on the host cores: each step is a bounded
    sample of the workload (see cpu_baseline); rank 0 only."""
    if rank != 0:
        return
    w = wl.WORKLOADS[args.workload]
    for _ in range(args.warmup):
        cpu_baseline(w, budget_s=4.0, single_thread=False)
    vals = []
    t0 = time.perf_counter()
    last = None
    for _ in range(args.steps):
        last = cpu_baseline(w, budget_s=4.0, single_thread=False)
        vals.append(last["value"])
    wall = time.perf_counter() - t0
    value = statistics.mean(vals)
    line = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "impl": "reference",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(wall / args.steps * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{w.name} prefill", "batch": w.batch,
                       "seq_len": w.seq_len, "parallelism": "host threads"},
            "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": last["cores"],
                             "kind": "oracle", "sample": last["sample"]},
            "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="engine", choices=["engine", "reference"])
    ap.add_argument("--workload", default="prefill-8b", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--decode-workload", default="decode-batched,long-context",
                    help="comma-separated decode workloads (or none)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", action="store_true",
                    help="with N > 1 ranks, split one batch's streams over the ranks (strong "
                         "scaling) instead of running N replicas")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the prefill workload's batch (smaller cases for profiling)")
    ap.add_argument("--decode-prefix", type=int, default=None,
                    help="override the decode workloads' prefilled prefix length")
    ap.add_argument("--e2e-pieces", type=int, default=8,
                    help="pieces the end-to-end prefill from host buffers is cut into (copies of one "
                         "piece overlap the compute of the next)")
    ap.add_argument("--prefill-schedule", default="auto", choices=sorted(SCHEDULES),
                    help="how a prefill call overlaps its chain and its attention (lola_set_prefill_schedule)")
    ap.add_argument("--segment-intervals", type=int, default=0,
                    help="update intervals per prefill segment (0: the library's choice)")
    ap.add_argument("--decode-steps", type=int, default=None,
                    help="override the number of timed decode steps")
    args = ap.parse_args(argv)
    ws, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, ws, rank)
        else:
            run_engine(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
