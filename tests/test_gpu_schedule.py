"""GPU: every prefill schedule (one chain launch per call with per-segment counts, or one
chain launch per segment; any segment length) gives the same outputs and the same cache,
bit for bit. The default schedule is checked against the oracle by the parity tests, so
this extends that parity to the others."""
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


# (mode, intervals per segment) on a call of 64 intervals
SCHEDULES = [("auto", 0), ("one-chain", 8), ("one-chain", 5), ("one-chain", 1), ("one-chain", 64),
             ("segments", 16), ("segments", 3), ("segments", 0)]


def _run(S, qd, kd, vd, calls):
    """Prefill in `calls` equal calls from a reset state; returns (out, cache ids, counts)."""
    S.reset()
    n = qd.shape[1]
    step = n // calls
    outs = []
    for t0 in range(0, n, step):
        outs.append(S.prefill(qd[:, t0:t0 + step].contiguous(), kd[:, t0:t0 + step].contiguous(),
                              vd[:, t0:t0 + step].contiguous()))
    idx, cnt = S.cache_indices()
    torch.cuda.current_stream(S.device).synchronize()
    S.sync()
    return torch.cat(outs, 1).cpu(), idx.cpu(), cnt.cpu()


@pytest.mark.parametrize("calls", [1, 2], ids=["one call", "two calls"])
def test_prefill_schedules_agree(calls):
    # the prefill-1b heads (warp-specialised attention, tensor-core chain), 64 intervals
    w = wl.WORKLOADS["prefill-1b"]
    T = w.seq_len
    q, k, v, _ = wl.make_inputs(w, T=T)
    dev = torch.device("cuda:0")
    S = L.LolaState(L.config_from_workload(w, max_prefill_tokens=T), torch.from_numpy(wl.make_W(w)), dev)
    qd, kd, vd = (torch.from_numpy(x).to(dev, S.dtype) for x in (q, k, v))
    ref = None
    for mode, seg in SCHEDULES:
        S.set_prefill_schedule(mode, seg)
        got = _run(S, qd, kd, vd, calls)
        assert S.position == T
        if ref is None:
            ref = got
            assert int(got[2].min()) == w.lambda_
            continue
        for a, b, what in zip(got, ref, ("output", "cache ids", "cache counts")):
            assert torch.equal(a, b), f"{mode} / {seg} intervals per segment: {what} differ"
    S.close()


def test_prefill_schedule_rejects_bad_arguments():
    w = wl.WORKLOADS["tiny"]
    S = L.LolaState(L.config_from_workload(w, max_prefill_tokens=w.seq_len), torch.from_numpy(wl.make_W(w)),
                    torch.device("cuda:0"))
    for mode, seg in ((3, 0), (-1, 0), (1, -2)):
        with pytest.raises(L.LolaError) as e:
            L.lola_set_prefill_schedule(S.handle, mode, seg)
        assert e.value.code == 1
    S.close()
