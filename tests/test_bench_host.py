"""Host-side logic of bench.py: algorithmic work counts and the multi-rank
aggregation (max over ranks, weak-scaling whole-job rate) on 2 gloo ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
from hybrid_linear_attention_lola_b200 import workloads as wl


def test_prefill_flops_match_steady_state_formula():
    # 8B-shaped: 31.56 MFLOP per token at steady state (|S| = lambda)
    w = wl.WORKLOADS["prefill-8b"]
    T = 64 * 64
    fl = bench.prefill_flops(w.replace(batch=1), T)
    late = bench.prefill_flops(w.replace(batch=1), T + 64)
    per_tok = sum(late[k] - fl[k] for k in fl) / 64
    assert abs(per_tok / 31.56e6 - 1) < 0.01


def test_interval_sizes_fill_cache_then_steady():
    w = wl.WORKLOADS["prefill-1b"]
    sizes = bench.interval_sizes(w, 4096)
    assert sizes[0] == (0, 0, 0)            # nothing has left the 64-token window yet
    assert sizes[1] == (0, 64, 64)
    assert sizes[-1] == (512, 64, 512)


def test_decode_bytes_per_step():
    w = wl.WORKLOADS["decode-batched"]
    per_stream = bench.decode_bytes_per_step(w) / (w.batch * w.n_kv_heads)
    assert abs(per_stream / 193.9e3 - 1) < 0.02


def test_attention_traffic_scales_with_the_launch():
    # the committed capture is per unit (one interval of one stream); a launch of n units
    # reads n times that, and the 8-interval launch at batch 4 is the stored per-launch figure
    e = next(x for x in __import__("json").load(open(bench.TRAFFIC_FILE)) if x["kernel"] == "attn")
    t8, src = bench.captured_traffic("attn", "prefill-8b", 8 * 32)
    assert abs(t8 / e["dram_bytes_per_launch"] - 1) < 1e-6 and "scaled" in src
    t16, _ = bench.captured_traffic("attn", "prefill-8b", 16 * 32)
    assert abs(t16 / t8 - 2) < 1e-6
    assert bench.captured_traffic("attn", "prefill-8b")[0] == e["dram_bytes_per_launch"]
    assert bench.captured_traffic("chain", "prefill-8b", 512)[0] is None


def test_traffic_is_null_once_the_kernel_changes(monkeypatch):
    monkeypatch.setattr(bench, "source_sha", lambda rels: "0" * 16)
    t, why = bench.captured_traffic("attn", "prefill-8b", 512)
    assert t is None and "changed" in why


def test_prefill_roofline_reports_the_launch_it_scales_to():
    w = wl.WORKLOADS["prefill-8b"]
    phases = {"attn": [180.0, 160], "chain": [106.0, 160], "phi": [2.7, 10]}   # 10 steps
    peaks = {"bf16_tflops": 1717.8, "bf16_tflops_sustained": 1424.0}
    r = bench.prefill_roofline(w, w.seq_len, 11.97, phases, 10, peaks, "measured", launch_intervals=16)
    assert r["traffic_kernel"] == "attn" and r["traffic_launch"] == "16 intervals x 32 streams"
    assert r["traffic"] == bench.captured_traffic("attn", "prefill-8b", 16 * 32)[0]
    assert abs(r["frac"] - r["achieved"] / 1717.8) < 1e-4


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE="2", LOCAL_RANK=str(rank), LOLA_BENCH_BACKEND="gloo")
    ws, r, _ = bench.dist_setup()
    mx = bench.max_over_ranks(1.5 + rank, ws)
    bench.barrier(ws)
    rate = bench.whole_job_rate(4096, ws, mx / 1e3)
    q.put((r, mx, rate))
    dist.destroy_process_group()


def test_two_rank_aggregation_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(2))
    for r, mx, rate in res:
        assert mx == 2.5                      # max over ranks, not the local value
        assert abs(rate - 2 * 4096 / 2.5e-3) < 1e-6
