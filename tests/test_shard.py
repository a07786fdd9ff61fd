"""Sharding a batch's (batch, kv-head) streams over ranks: the partition, the slicing
of inputs and feature maps, and the gather of outputs, run as two gloo ranks on the
CPU. Each rank's compute is the fp64 oracle on its shard (the test stands in for the
GPU engine with the reference definition); the gathered output must equal the oracle
on the whole batch, since streams are independent."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from hybrid_linear_attention_lola_b200 import shard as SH
from hybrid_linear_attention_lola_b200 import workloads as wl


def test_partition_by_batch_then_by_heads():
    s = [SH.partition(4, 32, 8, 2, r) for r in range(2)]
    assert [(x.by, x.b0, x.b1, x.h0, x.h1) for x in s] == [("batch", 0, 2, 0, 8), ("batch", 2, 4, 0, 8)]
    s = [SH.partition(1, 32, 8, 4, r) for r in range(4)]
    assert [(x.by, x.h0, x.h1, x.n_q_heads) for x in s] == [("kv_heads", 2 * r, 2 * r + 2, 8) for r in range(4)]
    with pytest.raises(ValueError):
        SH.partition(3, 12, 3, 2, 0)
    # every stream exactly once
    for B, Hkv, world in [(4, 8, 2), (4, 8, 4), (1, 8, 8), (2, 8, 4)]:
        seen = []
        for r in range(world):
            x = SH.partition(B, Hkv * 2, Hkv, world, r)
            seen += [(b, h) for b in range(x.b0, x.b1) for h in range(x.h0, x.h1)]
        assert sorted(seen) == [(b, h) for b in range(B) for h in range(Hkv)]


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, case, result_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = case
        q, k, v, _ = wl.make_inputs(w, T=w.seq_len)
        W = wl.make_W(w)
        sh = SH.partition(w.batch, w.n_q_heads, w.n_kv_heads, world, rank)
        Ws = SH.slice_W(sh, torch.from_numpy(W), w.w_per_head).numpy()
        ints = [w.chunk] * (w.seq_len // w.chunk)

        def compute(qs, ks, vs):
            r = oracle.run(qs.numpy(), ks.numpy(), vs.numpy(), Ws, window=w.window, lambda_=w.lambda_,
                           intervals=ints, eps=w.eps, threads=1)
            return torch.from_numpy(r.out)

        full = SH.run_sharded(sh, torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), compute)
        if rank == 0:
            np.save(result_path, full.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("by", ["batch", "kv_heads"])
def test_two_gloo_ranks_gather_equals_whole_batch(by, tmp_path):
    base = dict(name="shard", wid=14, n_q_heads=4, head_dim=16, feat_dim=16, window=6, lambda_=5,
                chunk=4, decode_interval=4, seq_len=40, decode_steps=0, dtype="f32", w_per_head=True)
    w = wl.Workload(batch=2, n_kv_heads=1, **base) if by == "batch" else wl.Workload(batch=1, n_kv_heads=2, **base)
    out_path = str(tmp_path / "full.npy")
    mp.start_processes(_rank_main, args=(2, _port(), w, out_path), nprocs=2, join=True, start_method="spawn")
    full = np.load(out_path)
    q, k, v, _ = wl.make_inputs(w, T=w.seq_len)
    r = oracle.run(q, k, v, wl.make_W(w), window=w.window, lambda_=w.lambda_,
                   intervals=[w.chunk] * (w.seq_len // w.chunk), eps=w.eps)
    np.testing.assert_allclose(full, r.out, rtol=1e-12, atol=1e-14)
