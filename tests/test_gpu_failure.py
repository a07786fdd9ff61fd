"""Failure detection on the GPU without faulting it.

A bounded device wait is made to run out (a test hook arms one wait on an
mbarrier that nothing arrives at, with a 1 ms limit), and a device-side bounds
check is tripped by a host-injected inconsistent selection override. In each
case the kernel records its error word and leaves its work, lola_sync reports
LOLA_ERR_TIMEOUT / LOLA_ERR_DEVICE, the CUDA context stays usable, and the state
computes correct results again afterwards (checked against the fp64 oracle).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle
from hybrid_linear_attention_lola_b200 import lola as L
from hybrid_linear_attention_lola_b200 import workloads as wl
from tests import parity as P

LIMIT_NS = 1_000_000          # 1 ms: the armed wait gives up after this
TOL = 2e-2                    # bfloat16 inputs, fp32 accumulation


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_linear_attention_lola_b200 import build
    build.build()


def _w(**kw):
    base = dict(name="failure", wid=13, batch=2, n_q_heads=4, n_kv_heads=2, head_dim=64, feat_dim=64,
                window=16, lambda_=200, chunk=32, decode_interval=16, seq_len=320, decode_steps=48,
                dtype="bf16")
    base.update(kw)
    return wl.Workload(**base)


def _oracle(w, q, k, v, ints):
    return oracle.run(q, k, v, wl.make_W(w), window=w.window, lambda_=w.lambda_, intervals=ints, eps=w.eps,
                      want_cands=True)


def _dev(*xs):
    return [torch.from_numpy(x).to("cuda", torch.bfloat16) for x in xs]


def _status_of(fn):
    try:
        fn()
    except L.LolaError as e:
        return e.code
    return 0


def test_chain_wait_runs_out_then_reset_state_is_correct():
    w = _w()
    T = w.seq_len
    q, k, v, _ = wl.make_inputs(w, T=T)
    qd, kd, vd = _dev(q, k, v)
    S = L.LolaState(L.config_from_workload(w, max_prefill_tokens=T), torch.from_numpy(wl.make_W(w)), "cuda")
    L.lola_set_fault_injection(S.handle, 1, LIMIT_NS)
    S.prefill(qd, kd, vd)
    assert _status_of(S.sync) == 7            # LOLA_ERR_TIMEOUT
    assert _status_of(S.sync) == 0            # reported once, then cleared
    # the context is usable and a reset state computes the right outputs and kept sets
    ints = P.intervals_for([("prefill", T)], w.chunk, w.decode_interval)
    r = _oracle(w, q, k, v, ints)
    S.reset()
    log = S.enable_selection_log(len(ints))
    S.set_selection_override(torch.from_numpy(P.override_from(r, w.lambda_, only_under_margin=True)))
    out = S.prefill(qd, kd, vd).float().cpu().numpy()
    S.sync()
    checked, exact, under, hard = P.compare_selections(log.cpu().numpy(), r, w.lambda_)
    assert not hard and checked == len(ints) * w.batch * w.n_kv_heads
    assert P.rel_l2(out, r.out) <= TOL
    S.close()


def test_decode_wait_runs_out_then_following_steps_are_correct():
    # one warp of the streaming decode kernel gives up before counting its partial;
    # lola_sync restarts the per-stream counters, so later steps merge correctly
    w = _w()
    T, n_dec = w.seq_len, w.decode_steps
    q, k, v, _ = wl.make_inputs(w, T=T + n_dec)
    ints = P.intervals_for([("prefill", T), ("decode", n_dec)], w.chunk, w.decode_interval)
    r = _oracle(w, q, k, v, ints)
    qd, kd, vd = _dev(q, k, v)
    S = L.LolaState(L.config_from_workload(w, max_prefill_tokens=T), torch.from_numpy(wl.make_W(w)), "cuda")
    S.set_selection_override(torch.from_numpy(P.override_from(r, w.lambda_, only_under_margin=True)))
    S.prefill(qd[:, :T].contiguous(), kd[:, :T].contiguous(), vd[:, :T].contiguous())
    bad = T + 5                                # a step inside an open decode interval
    outs = {}
    for t in range(T, T + n_dec):
        if t == bad:
            L.lola_set_fault_injection(S.handle, 2, LIMIT_NS)
        o = S.decode(qd[:, t].contiguous(), kd[:, t].contiguous(), vd[:, t].contiguous())
        if t == bad:
            assert _status_of(S.sync) == 7    # LOLA_ERR_TIMEOUT
        else:
            outs[t] = o.float().cpu().numpy()
    S.sync()
    steps = sorted(t for t in outs if t > bad)
    got = np.stack([outs[t] for t in steps], 1)
    want = r.out[:, steps]
    assert P.rel_l2(got, want) <= TOL
    assert P.row_rel_l2_max(got, want) <= TOL
    S.close()


def test_bounds_word_from_inconsistent_override():
    # an override whose kept count disagrees with the cache size trips the chain's
    # bounds check; lola_sync reports LOLA_ERR_DEVICE, and a reset state is correct
    w = _w()
    T = w.seq_len
    q, k, v, _ = wl.make_inputs(w, T=T)
    ints = P.intervals_for([("prefill", T)], w.chunk, w.decode_interval)
    r = _oracle(w, q, k, v, ints)
    qd, kd, vd = _dev(q, k, v)
    S = L.LolaState(L.config_from_workload(w, max_prefill_tokens=T), torch.from_numpy(wl.make_W(w)), "cuda")
    ovr = P.override_from(r, w.lambda_)
    ci = len(ints) - 2                         # an interval with a full cache
    assert ovr[ci, 0, 0] == w.lambda_
    ovr[ci, 0, 0] = w.lambda_ - 1              # one kept pair fewer than the cache holds
    ovr[ci, 0, w.lambda_] = -1
    S.set_selection_override(torch.from_numpy(ovr))
    S.prefill(qd, kd, vd)
    assert _status_of(S.sync) == 8             # LOLA_ERR_DEVICE
    S.set_selection_override(torch.from_numpy(P.override_from(r, w.lambda_, only_under_margin=True)))
    S.reset()
    out = S.prefill(qd, kd, vd).float().cpu().numpy()
    S.sync()
    assert P.rel_l2(out, r.out) <= TOL
    S.close()
