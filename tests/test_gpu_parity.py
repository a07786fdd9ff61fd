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


ROW_TOL = {"f32": 1e-4, "bf16": 2e-2}


def _case(w, plan, *, modes=("forced", "own"), subset=None, qmask_every=None,
          T=None, seed_inputs=None, scores=False, name=None):
    """Runs plan on the GPU (once per mode, see tests/parity.py) and the oracle once;
    asserts the parity bar, records the counts, and returns a dict of metrics per
    mode. subset=(batches, kv_heads) restricts the oracle's streams."""
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
    qo = np.ascontiguousarray(q[bsel][:, :, qsel])
    ko = np.ascontiguousarray(k[bsel][:, :, hsel])
    vo = np.ascontiguousarray(v[bsel][:, :, hsel])
    qmask = rows = None
    if qmask_every:
        qmask = np.zeros(T, np.uint8)
        qmask[::qmask_every] = 1
        qmask[-1] = 1
        rows = np.flatnonzero(qmask)
    r = oracle.run(qo, ko, vo, W, window=w.window, lambda_=w.lambda_, intervals=ints,
                   eps=w.eps, qmask=qmask, want_cands=True, compact=qmask is not None,
                   scorer=w.scorer)
    smap = [b * w.n_kv_heads + h for b in bsel for h in hsel]
    ns = w.batch * w.n_kv_heads
    res = {}
    for mode in modes:
        ovr = None
        if mode == "forced":
            ovr = P.override_from(r, w.lambda_, ns, smap)
        elif mode == "own":
            ovr = P.override_from(r, w.lambda_, ns, smap, only_under_margin=True)
        out, log, sc = P.run_gpu(cfg, W, q, k, v, plan, override=ovr, log_cap=len(ints), rows=rows,
                                 score_cap=len(ints) if (scores and mode == "forced") else None)
        go = out[bsel][:, :, qsel]
        assert np.all(np.isfinite(go))
        err = P.rel_l2(go, r.out)
        rmax = P.row_rel_l2_max(go, r.out)
        checked, exact, under, hard = P.compare_selections(log, r, w.lambda_, smap)
        u = dict(rel_l2=err, row_rel_l2_max=rmax, intervals_checked=checked, exact=exact,
                 under_margin_differ=under, hard=len(hard),
                 forced_intervals=int(np.sum(ovr[:, smap, 0] >= 0)) if ovr is not None else 0)
        if sc is not None:
            u["sre_vs_oracle"] = P.score_errors(sc, r, smap)
        res[mode] = u
        print(f"{w.name} {mode}: {u}")
        if mode in ("forced", "own"):
            assert not hard, hard[:4]
            assert err <= TOL[w.dtype], u
            assert rmax <= ROW_TOL[w.dtype], u
        elif exact == checked:
            # the product path without any forcing: identical unless an ambiguous choice moved it
            assert err <= TOL[w.dtype] and rmax <= ROW_TOL[w.dtype], u
    P.record(name or w.name, {"workload": w.name, "dtype": w.dtype, "plan": [list(x) for x in plan],
                              "streams_compared": len(smap), "streams_total": ns,
                              "outputs_compared": "every position" if rows is None
                              else f"every {qmask_every}th position and the last ({len(rows)})",
                              "tolerance": {"rel_l2": TOL[w.dtype], "row_rel_l2": ROW_TOL[w.dtype],
                                            "selection_margin": P.MARGIN},
                              "oracle_margins": P.margin_summary(r), "runs": res})
    return res


def _small(**kw):
    base = dict(name="small", wid=11, batch=1, n_q_heads=2, n_kv_heads=2, head_dim=32,
                feat_dim=32, window=8, lambda_=12, chunk=16, decode_interval=8, seq_len=128,
                decode_steps=0, dtype="f32")
    base.update(kw)
    return wl.Workload(**base)


# ---------------------------------------------------------------- tiny (fp32)

ALL = ("forced", "own", "free")


def test_tiny_prefill_parity():
    w = wl.WORKLOADS["tiny"]
    res = _case(w, [("prefill", 512)], modes=ALL)
    assert res["free"]["exact"] == res["free"]["intervals_checked"]
    assert res["free"]["rel_l2"] <= 1e-4


def test_tiny_prefill_then_decode_parity():
    w = wl.WORKLOADS["tiny"]
    _case(w, [("prefill", 256), ("decode", 256)], modes=ALL, name="tiny prefill+decode")


def test_tiny_split_calls_equal_single_call():
    w = wl.WORKLOADS["tiny"]
    _case(w, [("prefill", 128), ("prefill", 64), ("prefill", 320)], modes=ALL, name="tiny split calls")


def test_decode_then_prefill_then_decode():
    w = _small(decode_interval=8)
    _case(w, [("prefill", 32), ("decode", 24), ("prefill", 48), ("decode", 20)], modes=ALL,
          name="f32 decode/prefill interleaved")


# ---------------------------------------------------------------- edge cases (fp32)

def test_no_window_no_cache_is_linear_attention():
    w = _small(window=0, lambda_=0, decode_interval=1)
    _case(w, [("prefill", 64), ("decode", 16)], modes=("free",), name="f32 linear only")


def test_window_covering_everything_is_softmax():
    w = _small(window=200, lambda_=0, decode_interval=16)
    _case(w, [("prefill", 128), ("decode", 32)], modes=("free",), name="f32 softmax only")


def test_cache_holding_everything():
    w = _small(window=4, lambda_=256, decode_interval=4)
    _case(w, [("prefill", 96), ("decode", 32)], modes=("free",), name="f32 cache holds all")


def test_chunk_longer_than_window_ragged_tiles():
    # leaving pairs come from the current chunk; lambda and C off the 32/64 tile grid
    w = _small(window=5, lambda_=37, chunk=48, decode_interval=6, head_dim=64, feat_dim=64)
    _case(w, [("prefill", 240), ("decode", 13)], modes=ALL, name="f32 chunk > window, ragged")


def test_zero_window_with_cache():
    w = _small(window=0, lambda_=9, chunk=8, decode_interval=1)
    _case(w, [("prefill", 80), ("decode", 5)], modes=ALL, name="f32 zero window")


def test_gqa_group_of_eight_and_eps_zero():
    w = _small(n_q_heads=16, n_kv_heads=2, eps=0.0, head_dim=128, feat_dim=128, lambda_=20,
               chunk=32, window=16)
    _case(w, [("prefill", 160)], modes=ALL, name="f32 GQA 8, eps 0")


# ---------------------------------------------------------------- edge cases (bfloat16)
# head_dim 64 keeps these on the tensor-core chain and attention and the streaming decode.
# Feature dim 64 (feature half 32) takes the single-tile attention kernel. The
# warp-specialised one takes feature dim 128 with intervals of more than 128 query rows
# (two query tiles per CTA): WS marks the cases whose shape gives it those.

ATTN = pytest.mark.parametrize("feat", [64, 128], ids=["tile-attn", "ws-attn"])


def _small_bf16(**kw):
    base = dict(head_dim=64, feat_dim=64, dtype="bf16")
    base.update(kw)
    return _small(**base)


@ATTN
def test_bf16_no_window_no_cache_is_linear_attention(feat):
    w = _small_bf16(window=0, lambda_=0, decode_interval=1, feat_dim=feat)
    _case(w, [("prefill", 64), ("decode", 16)], modes=("free",), name=f"bf16 linear only D{feat}")


@ATTN
def test_bf16_chunk_longer_than_window_ragged_tiles(feat):
    # partial cache and window tiles, query rows past the interval (192 rows: the second
    # query tile half full), and kept leaving pairs that are later than some queries of
    # their interval (chunk > window)
    w = _small_bf16(window=5, lambda_=37, chunk=48, decode_interval=6, n_q_heads=8, n_kv_heads=2, feat_dim=feat)
    _case(w, [("prefill", 240), ("decode", 13)], modes=ALL, name=f"bf16 chunk > window, ragged D{feat}")


@ATTN
def test_bf16_zero_window_with_cache(feat):
    w = _small_bf16(window=0, lambda_=9, chunk=8, decode_interval=1, feat_dim=feat)
    _case(w, [("prefill", 80), ("decode", 5)], modes=ALL, name=f"bf16 zero window D{feat}")


def test_bf16_gqa_group_of_eight():
    w = _small_bf16(n_q_heads=16, n_kv_heads=2, head_dim=128, feat_dim=128, lambda_=20, chunk=32, window=16)
    _case(w, [("prefill", 160)], modes=ALL, name="bf16 GQA 8")


@ATTN
def test_bf16_token_by_token(feat):
    # C = C_dec = 1 on the tensor-core chain and attention and the streaming decode
    w = _small_bf16(window=16, lambda_=24, chunk=1, decode_interval=1, n_q_heads=4, n_kv_heads=2, feat_dim=feat)
    _case(w, [("prefill", 96), ("decode", 32)], modes=ALL, name=f"bf16 token-by-token D{feat}")


@ATTN
def test_bf16_decode_then_prefill_then_decode(feat):
    # the second prefill call starts with window and band rows from the ring (16-byte
    # gathers instead of tiled loads) and cached pairs of the earlier calls; 256 query
    # rows per interval
    w = _small_bf16(window=16, lambda_=40, chunk=32, decode_interval=8, n_q_heads=16, n_kv_heads=2,
                    batch=2, feat_dim=feat)
    _case(w, [("prefill", 64), ("decode", 24), ("prefill", 64), ("decode", 20)], modes=ALL,
          name=f"bf16 decode/prefill interleaved D{feat}")


@ATTN
def test_bf16_long_chunk_two_band_chunks(feat):
    # chunk 128 > 64: two band chunks per interval and four query tiles per interval
    w = _small_bf16(window=64, lambda_=96, chunk=128, decode_interval=32, n_q_heads=8, n_kv_heads=2,
                    feat_dim=feat)
    _case(w, [("prefill", 512), ("decode", 64)], modes=ALL, name=f"bf16 chunk 128 D{feat}")


def test_bf16_head_dim_32():
    # head_dim 32 runs the SIMT attention beside the tensor-core chain
    w = _small_bf16(head_dim=32, feat_dim=64, window=8, lambda_=40, chunk=16, decode_interval=8)
    _case(w, [("prefill", 192), ("decode", 24)], modes=ALL, name="bf16 head_dim 32")


# ---------------------------------------------------------------- bf16 workloads

def _with_decode(w, T=None):
    qp, kp, vp, _ = wl.make_inputs(w, part="prefill", T=T)
    qd, kd, vd, _ = wl.make_inputs(w, part="decode")
    return (np.concatenate([qp, qd], 1), np.concatenate([kp, kd], 1), np.concatenate([vp, vd], 1), None)


def test_prefill_1b_full():
    w = wl.WORKLOADS["prefill-1b"]
    res = _case(w, [("prefill", w.seq_len)], modes=ALL, scores=True)
    f = res["forced"]
    assert f["exact"] + f["under_margin_differ"] == f["intervals_checked"]


def test_decode_batched_subset():
    # 64 of the 512 streams: batches 0, 9, ..., 63 with all eight kv-heads
    w = wl.WORKLOADS["decode-batched"]
    _case(w, [("prefill", w.seq_len), ("decode", w.decode_steps)], modes=("forced", "own"),
          subset=(list(range(0, 64, 9)), list(range(8))), seed_inputs=_with_decode(w))


def test_prefill_8b_sampled():
    # 8 of the 32 streams (every batch, kv-heads 0 and 5), every 97th position
    w = wl.WORKLOADS["prefill-8b"]
    _case(w, [("prefill", w.seq_len)], modes=("forced", "own"), subset=([0, 1, 2, 3], [0, 5]),
          qmask_every=97, scores=True)


def _long_context(name, every):
    w = wl.WORKLOADS[name]
    T = w.seq_len
    plan = [("prefill", 16384)] * (T // 16384) + [("decode", w.decode_steps)]
    _case(w, plan, modes=("forced", "own"), qmask_every=every, seed_inputs=_with_decode(w),
          scores=True)


def test_long_context_64k():
    _long_context("long-context", 251)


def test_long_context_128k():
    _long_context("long-context-128k", 503)


def test_long_context_256k():
    _long_context("long-context-256k", 1009)


# ---------------------------------------------------------------- next rows: the pages' setting, C = 1

def test_pages_cache_setting_prefill_then_decode():
    # window 256, sparse cache 256, 4K context with needles, then decode steps
    w = wl.WORKLOADS["pages-4k"]
    res = _case(w, [("prefill", w.seq_len), ("decode", w.decode_steps)], modes=ALL,
                seed_inputs=_with_decode(w))
    f = res["forced"]
    assert f["exact"] + f["under_margin_differ"] == f["intervals_checked"]


def test_token_by_token_intervals():
    # every token is its own update interval, in prefill (C = 1) and in decode (C_dec = 1)
    w = wl.WORKLOADS["token-by-token"]
    res = _case(w, [("prefill", w.seq_len), ("decode", w.decode_steps)], modes=ALL)
    assert res["free"]["exact"] == res["free"]["intervals_checked"]


# ---------------------------------------------------------------- the pages' ablation scorers, FIFO

@pytest.mark.parametrize("scorer", ["attention-weight", "softmax-error", "fifo"])
def test_ablation_scorer_bf16(scorer):
    # tensor-core chain on a two-CTA cluster per stream (the scores are computed by
    # every CTA, no key exchange), then decode intervals scored at their first step
    w = _small_bf16(n_q_heads=4, n_kv_heads=2, window=16, lambda_=150, chunk=32, decode_interval=16,
                    scorer=scorer)
    _case(w, [("prefill", 256), ("decode", 40)], modes=ALL, scores=True, name=f"bf16 scorer {scorer}")


@pytest.mark.parametrize("scorer", ["attention-weight", "softmax-error", "fifo"])
def test_ablation_scorer_f32(scorer):
    w = _small(n_q_heads=4, n_kv_heads=2, window=8, lambda_=20, chunk=16, decode_interval=8,
               head_dim=64, feat_dim=64, scorer=scorer)
    _case(w, [("prefill", 128), ("decode", 24)], modes=ALL, scores=True, name=f"f32 scorer {scorer}")


# ---------------------------------------------------------------- one feature map per kv-head

def test_per_head_feature_maps_bf16():
    # tensor-core feature map (grid rows by kv-head), chain, attention, decode preparation
    w = _small_bf16(n_q_heads=8, n_kv_heads=4, window=16, lambda_=150, chunk=32, decode_interval=16,
                    w_per_head=True)
    _case(w, [("prefill", 256), ("decode", 40)], modes=ALL, name="bf16 per-head W")


def test_per_head_feature_maps_bf16_query_kernel():
    # no cache: SIMT chain with the tensor-core query feature map (grid rows by kv-head)
    w = _small_bf16(n_q_heads=8, n_kv_heads=4, window=12, lambda_=0, chunk=16, decode_interval=8,
                    w_per_head=True)
    _case(w, [("prefill", 128), ("decode", 24)], modes=("free",), name="bf16 per-head W, no cache")


def test_per_head_feature_maps_f32_with_softmax_error():
    w = _small(n_q_heads=6, n_kv_heads=3, window=8, lambda_=20, chunk=16, decode_interval=8,
               head_dim=64, feat_dim=64, w_per_head=True, scorer="softmax-error")
    _case(w, [("prefill", 128), ("decode", 24)], modes=ALL, name="f32 per-head W, softmax-error")
