"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle on
identical seeded inputs.

Tolerances: relative L2 over the compared outputs <= 1e-4 for float32 inputs
and <= 2e-2 for bfloat16 inputs (fp32 accumulation); the kept set of every
update interval equals the oracle's wherever the oracle's lambda-th vs
(lambda+1)-th SRE margin exceeds 1e-3 relative, and is a valid top-lambda
within that band elsewhere (counted). "Forced" runs feed the oracle's kept
sets to the engine (lola_set_selection_override) so that a numerically
ambiguous choice cannot move the GPU off the reference trajectory; the GPU's
own choice is still logged and checked.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle
from hybrid_linear_attention_lola_b200 import lola as L
from hybrid_linear_attention_lola_b200 import workloads as wl
from tests import parity as P

TOL = {"f32": 1e-4, "bf16": 2e-2}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_linear_attention_lola_b200 import build
    build.build()


def _case(w, plan, *, forced=True, unforced=False, subset=None, qmask_every=None,
          T=None, seed_inputs=None):
    """Runs plan on the GPU and the oracle; returns a dict of metrics and asserts
    the parity bar. subset=(batches, kv_heads) restricts the oracle's streams."""
    T = sum(n for _, n in plan) if T is None else T
    q, k, v, _ = seed_inputs if seed_inputs is not None else wl.make_inputs(w, T=T)
    W = wl.make_W(w)
    ints = P.intervals_for(plan, w.chunk, w.decode_interval)
    n_pre = max([n for kind, n in plan if kind == "prefill"] + [w.chunk])
    cfg = L.config_from_workload(w, max_prefill_tokens=n_pre)
    # oracle on the chosen streams
    bsel = list(range(w.batch)) if subset is None else subset[0]
    hsel = list(range(w.n_kv_heads)) if subset is None else subset[1]
    g = w.group
    qsel = [hk * g + r for hk in hsel for r in range(g)]
    qo = q[bsel][:, :, qsel]
    ko = k[bsel][:, :, hsel]
    vo = v[bsel][:, :, hsel]
    qmask = None
    if qmask_every:
        qmask = np.zeros(T, np.uint8)
        qmask[::qmask_every] = 1
        qmask[-1] = 1
    r = oracle.run(qo, ko, vo, W, window=w.window, lambda_=w.lambda_, intervals=ints,
                   eps=w.eps, qmask=qmask, want_cands=True)
    smap = [b * w.n_kv_heads + h for b in bsel for h in hsel]
    res = {}
    runs = []
    if forced:
        runs.append(("forced", P.override_from(r, w.lambda_, w.batch * w.n_kv_heads, smap)))
    if unforced:
        runs.append(("unforced", None))
    for name, ovr in runs:
        out, log = P.run_gpu(cfg, W, q, k, v, plan, override=ovr, log_cap=len(ints))
        go = out[bsel][:, :, qsel]
        if qmask is not None:
            go = go[:, qmask == 1]
            oo = r.out[:, qmask == 1]
        else:
            oo = r.out
        assert np.all(np.isfinite(go))
        err = P.rel_l2(go, oo)
        checked, exact, under, hard = P.compare_selections(log, r, w.lambda_, smap)
        res[name] = dict(rel_l2=err, checked=checked, exact=exact, under=under, hard=hard)
        print(f"{w.name} {name}: rel_l2={err:.3e} intervals={checked} exact={exact} "
              f"under-margin={under} hard={len(hard)}")
        if name == "forced":
            assert not hard, hard[:4]
            assert err <= TOL[w.dtype], err
    if unforced:
        u = res["unforced"]
        # the product path without forcing: identical unless an ambiguous choice moved it
        if u["exact"] == u["checked"]:
            assert u["rel_l2"] <= TOL[w.dtype], u
    return res


def _small(**kw):
    base = dict(name="small", wid=11, batch=1, n_q_heads=2, n_kv_heads=2, head_dim=32,
                feat_dim=32, window=8, lambda_=12, chunk=16, decode_interval=8, seq_len=128,
                decode_steps=0, dtype="f32")
    base.update(kw)
    return wl.Workload(**base)


# ---------------------------------------------------------------- tiny (fp32)

def test_tiny_prefill_parity():
    w = wl.WORKLOADS["tiny"]
    res = _case(w, [("prefill", 512)], forced=True, unforced=True)
    assert res["unforced"]["exact"] == res["unforced"]["checked"]
    assert res["unforced"]["rel_l2"] <= 1e-4


def test_tiny_prefill_then_decode_parity():
    w = wl.WORKLOADS["tiny"]
    _case(w, [("prefill", 256), ("decode", 256)], forced=True, unforced=True)


def test_tiny_split_calls_equal_single_call():
    w = wl.WORKLOADS["tiny"]
    _case(w, [("prefill", 128), ("prefill", 64), ("prefill", 320)], forced=True, unforced=True)


def test_decode_then_prefill_then_decode():
    w = _small(decode_interval=8)
    _case(w, [("prefill", 32), ("decode", 24), ("prefill", 48), ("decode", 20)],
          forced=True, unforced=True)


# ---------------------------------------------------------------- edge cases (fp32)

def test_no_window_no_cache_is_linear_attention():
    w = _small(window=0, lambda_=0, decode_interval=1)
    _case(w, [("prefill", 64), ("decode", 16)], forced=False, unforced=True)


def test_window_covering_everything_is_softmax():
    w = _small(window=200, lambda_=0, decode_interval=16)
    _case(w, [("prefill", 128), ("decode", 32)], forced=False, unforced=True)


def test_cache_holding_everything():
    w = _small(window=4, lambda_=256, decode_interval=4)
    _case(w, [("prefill", 96), ("decode", 32)], forced=False, unforced=True)


def test_chunk_longer_than_window_ragged_tiles():
    # leaving pairs come from the current chunk; lambda and C off the 32/64 tile grid
    w = _small(window=5, lambda_=37, chunk=48, decode_interval=6, head_dim=64, feat_dim=64)
    _case(w, [("prefill", 240), ("decode", 13)], forced=True, unforced=True)


def test_zero_window_with_cache():
    w = _small(window=0, lambda_=9, chunk=8, decode_interval=1)
    _case(w, [("prefill", 80), ("decode", 5)], forced=True, unforced=True)


def test_gqa_group_of_eight_and_eps_zero():
    w = _small(n_q_heads=16, n_kv_heads=2, eps=0.0, head_dim=128, feat_dim=128, lambda_=20,
               chunk=32, window=16)
    _case(w, [("prefill", 160)], forced=True, unforced=True)


# ---------------------------------------------------------------- edge cases (bfloat16)
# head_dim 64 keeps these on the tensor-core chain and attention and the streaming decode

def _small_bf16(**kw):
    base = dict(head_dim=64, feat_dim=64, dtype="bf16")
    base.update(kw)
    return _small(**base)


def test_bf16_no_window_no_cache_is_linear_attention():
    w = _small_bf16(window=0, lambda_=0, decode_interval=1)
    _case(w, [("prefill", 64), ("decode", 16)], forced=False, unforced=True)


def test_bf16_chunk_longer_than_window_ragged_tiles():
    # partial cache and window tiles, query rows past the interval, and kept leaving
    # pairs that are later than some queries of their interval (chunk > window)
    w = _small_bf16(window=5, lambda_=37, chunk=48, decode_interval=6)
    _case(w, [("prefill", 240), ("decode", 13)], forced=True, unforced=True)


def test_bf16_zero_window_with_cache():
    w = _small_bf16(window=0, lambda_=9, chunk=8, decode_interval=1)
    _case(w, [("prefill", 80), ("decode", 5)], forced=True, unforced=True)


def test_bf16_gqa_group_of_eight():
    w = _small_bf16(n_q_heads=16, n_kv_heads=2, head_dim=128, feat_dim=128, lambda_=20, chunk=32, window=16)
    _case(w, [("prefill", 160)], forced=True, unforced=True)


# ---------------------------------------------------------------- bf16 workloads

def test_prefill_1b_full():
    w = wl.WORKLOADS["prefill-1b"]
    res = _case(w, [("prefill", w.seq_len)], forced=True, unforced=True)
    assert res["forced"]["exact"] + res["forced"]["under"] == res["forced"]["checked"]


def test_decode_batched_subset():
    w = wl.WORKLOADS["decode-batched"]
    qp, kp, vp, _ = wl.make_inputs(w, part="prefill")
    qd, kd, vd, _ = wl.make_inputs(w, part="decode")
    inputs = (np.concatenate([qp, qd], 1), np.concatenate([kp, kd], 1),
              np.concatenate([vp, vd], 1), None)
    _case(w, [("prefill", w.seq_len), ("decode", w.decode_steps)], forced=True,
          subset=([0, 37], [0, 5]), seed_inputs=inputs)


def test_prefill_8b_sampled():
    w = wl.WORKLOADS["prefill-8b"]
    _case(w, [("prefill", w.seq_len)], forced=True, subset=([1], [0, 6]), qmask_every=97)


def test_long_context_sampled():
    w = wl.WORKLOADS["long-context"]
    T = w.seq_len
    qp, kp, vp, _ = wl.make_inputs(w, part="prefill")
    qd, kd, vd, _ = wl.make_inputs(w, part="decode")
    inputs = (np.concatenate([qp, qd], 1), np.concatenate([kp, kd], 1),
              np.concatenate([vp, vd], 1), None)
    plan = [("prefill", 16384)] * (T // 16384) + [("decode", w.decode_steps)]
    _case(w, plan, forced=True, subset=([0], [3]), qmask_every=251, seed_inputs=inputs)


# ---------------------------------------------------------------- next rows: the pages' setting, C = 1

def test_pages_cache_setting_prefill_then_decode():
    # window 256, sparse cache 256, 4K context with needles, then decode steps
    w = wl.WORKLOADS["pages-4k"]
    qp, kp, vp, _ = wl.make_inputs(w, part="prefill")
    qd, kd, vd, _ = wl.make_inputs(w, part="decode")
    inputs = (np.concatenate([qp, qd], 1), np.concatenate([kp, kd], 1),
              np.concatenate([vp, vd], 1), None)
    res = _case(w, [("prefill", w.seq_len), ("decode", w.decode_steps)], forced=True, unforced=True,
                seed_inputs=inputs)
    assert res["forced"]["exact"] + res["forced"]["under"] == res["forced"]["checked"]


def test_token_by_token_intervals():
    # every token is its own update interval, in prefill (C = 1) and in decode (C_dec = 1)
    w = wl.WORKLOADS["token-by-token"]
    res = _case(w, [("prefill", w.seq_len), ("decode", w.decode_steps)], forced=True, unforced=True)
    assert res["unforced"]["exact"] == res["unforced"]["checked"]
