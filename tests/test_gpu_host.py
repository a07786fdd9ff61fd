"""GPU: lola_prefill_host (host buffers, copies overlapped with the compute piece by
piece) gives exactly what the same prefill calls give on device buffers."""
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


@pytest.mark.parametrize("n,piece", [(256, 64), (224, 64), (128, 128)], ids=["4 pieces", "ragged", "1 piece"])
def test_host_prefill_equals_device_calls(n, piece):
    w = wl.Workload("host", 21, batch=2, n_q_heads=8, n_kv_heads=2, head_dim=64, feat_dim=128, window=16,
                    lambda_=40, chunk=32, decode_interval=8, seq_len=n, decode_steps=0, dtype="bf16")
    q, k, v, _ = wl.make_inputs(w, T=n)
    W = wl.make_W(w)
    dev = torch.device("cuda:0")
    S = L.LolaState(L.config_from_workload(w, max_prefill_tokens=piece), torch.from_numpy(W), dev)
    qd, kd, vd = (torch.from_numpy(x).to(dev, S.dtype) for x in (q, k, v))
    # the same pieces through lola_prefill_chunk on device buffers
    ref = []
    for t0 in range(0, n, piece):
        t1 = min(n, t0 + piece)
        ref.append(S.prefill(qd[:, t0:t1].contiguous(), kd[:, t0:t1].contiguous(), vd[:, t0:t1].contiguous()))
    ref = torch.cat(ref, 1).cpu()
    pos_dev = S.position
    S.reset()
    qh, kh, vh = (t.cpu().pin_memory() for t in (qd, kd, vd))
    oh = torch.empty(qh.shape, dtype=S.dtype).pin_memory()
    S.prefill_host(qh, kh, vh, oh, piece)
    torch.cuda.current_stream(dev).synchronize()
    S.sync()
    assert S.position == pos_dev == n
    assert torch.equal(oh, ref)
    S.close()
