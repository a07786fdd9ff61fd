"""lola_decode_step_static: the decode step for callers that cannot obtain
device memory on demand (a plugin whose host framework owns all device memory,
or code running during CUDA graph capture). Its per-step temporaries live in a
fixed array inside the library instead of the workspace.

Checked through the C ABI against lola_decode_step on two calls in a row (one
that opens an update interval, one inside it), in float32 and bfloat16, with the
output tolerances the parity tests use, and for the size limit. Collected last on purpose: if it
fails, a run that stops at the first failure has already run everything else.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from hybrid_linear_attention_lola_b200 import lola as L
from hybrid_linear_attention_lola_b200 import workloads as wl


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_linear_attention_lola_b200 import build
    build.build()


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return np.linalg.norm(a - b) / np.linalg.norm(b)


TOL = {"f32": 1e-4, "bf16": 2e-2}


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_static_decode_matches_decode_step_twice(dtype):
    # bfloat16 runs the streaming decode kernel, whose fp32 query features also
    # live in the library's array (after the partial sums)
    w = wl.Workload("noalloc", 12, batch=2, n_q_heads=4, n_kv_heads=2, head_dim=64, feat_dim=64,
                    window=16, lambda_=24, chunk=32, decode_interval=16, seq_len=64,
                    decode_steps=2, dtype=dtype)
    q, k, v, _ = wl.make_inputs(w, T=w.seq_len + 2)
    W = torch.from_numpy(wl.make_W(w))
    dev = torch.device("cuda")
    cfg = L.config_from_workload(w, max_prefill_tokens=w.seq_len)
    A = L.LolaState(cfg, W, dev)
    Bst = L.LolaState(cfg, W, dev)
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    qd, kd, vd = (torch.from_numpy(x).to(dev, dt) for x in (q, k, v))
    T = w.seq_len
    for S in (A, Bst):
        S.prefill(qd[:, :T].contiguous(), kd[:, :T].contiguous(), vd[:, :T].contiguous())
    stream = torch.cuda.current_stream().cuda_stream
    for t in (T, T + 1):          # first call opens an update interval, second is inside it
        qs, ks, vs = (x[:, t].contiguous() for x in (qd, kd, vd))
        out_ref = torch.empty_like(qs)
        out_static = torch.full_like(qs, float("nan"))
        L.lola_decode_step(A.handle, qs.data_ptr(), ks.data_ptr(), vs.data_ptr(),
                           out_ref.data_ptr(), stream)
        L.lola_decode_step_static(Bst.handle, qs.data_ptr(), ks.data_ptr(), vs.data_ptr(),
                                  out_static.data_ptr(), stream)
        torch.cuda.synchronize()
        assert torch.isfinite(out_static).all()
        assert _rel(out_static, out_ref) <= TOL[dtype]
        assert L.lola_position(Bst.handle) == L.lola_position(A.handle) == t + 1
    A.sync()
    Bst.sync()
    A.close()
    Bst.close()


def test_static_decode_rejects_scratch_beyond_limit():
    # 128 sequences x 64 query heads (8 per kv-head), head_dim 128, feat_dim 256:
    # the fp32 query features alone (8 MiB) plus the partials exceed the 8 MiB array
    cfg = L.make_config(batch=128, n_q_heads=64, n_kv_heads=8, head_dim=128, feat_dim=256,
                        window=1, lambda_=0, chunk=1, decode_interval=1, max_prefill_tokens=1,
                        eps=1e-6, dtype="bf16")
    S = L.LolaState(cfg, torch.zeros(128, 128), torch.device("cuda"))
    x = torch.zeros((128, 64, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((128, 8, 128), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    with pytest.raises(L.LolaError) as ei:
        L.lola_decode_step_static(S.handle, x.data_ptr(), kv.data_ptr(), kv.data_ptr(),
                                  x.data_ptr(), stream)
    assert ei.value.code == 5                 # LOLA_ERR_WORKSPACE, nothing enqueued
    assert L.lola_position(S.handle) == 0
    S.sync()
    S.close()
