"""Pins of the CPU oracle against facts other than itself.

Each test ties one part of the oracle to a closed form, a library routine, a
special case that reduces to textbook attention, or the independent set-based
restatement in oracle/brute.py. Together they cover the feature map, the SRE,
the selection rule and its tie-break, the fold into (H, s), the window
boundary, the causal mask and the shared-normaliser output combination
(LoLA, arXiv 2505.23666; gist.science technical summary, "Methodologie",
"Het Self-Recall Error (SRE) Mechanisme", "Inferentiestrategie").
"""
import itertools

import numpy as np
import pytest
import torch
from scipy.special import softmax

import oracle
from oracle import brute
from hybrid_linear_attention_lola_b200 import workloads as wl


def _rand(shape, seed, scale=1.0):
    return wl.make_random(shape, seed, "f32", scale)


def _qkvw(B, T, Hq, Hkv, d, D, seed, wscale=1.0):
    q = _rand((B, T, Hq, d), seed)
    k = _rand((B, T, Hkv, d), seed + 1)
    v = _rand((B, T, Hkv, d), seed + 2)
    W = _rand((d, D // 2), seed + 3, wscale / np.sqrt(d))
    return q, k, v, W


def _phi_lib(x, W):
    z = np.asarray(x, np.float64) @ np.asarray(W, np.float64)
    return np.concatenate([softmax(z, axis=-1), softmax(-z, axis=-1)], axis=-1)


# ---------------------------------------------------------------- feature map

def test_phi_identity_W_is_plain_softmax_pair():
    x = _rand((16,), 11, 2.0).astype(np.float64)
    out = oracle.phi(x, np.eye(16))
    np.testing.assert_allclose(out[:16], softmax(x), rtol=1e-14, atol=0)
    np.testing.assert_allclose(out[16:], softmax(-x), rtol=1e-14, atol=0)


def test_phi_random_W_matches_library_softmax_and_is_positive():
    W = _rand((32, 24), 12, 1 / np.sqrt(32))
    for seed in range(5):
        x = _rand((32,), 100 + seed, 3.0)
        out = oracle.phi(x, W)
        np.testing.assert_allclose(out, _phi_lib(x, W), rtol=1e-13, atol=0)
        assert np.all(out > 0)
        assert abs(out[:24].sum() - 1) < 1e-14 and abs(out[24:].sum() - 1) < 1e-14


def test_phi_zero_input_is_uniform():
    out = oracle.phi(np.zeros(8), _rand((8, 5), 13))
    np.testing.assert_allclose(out, np.full(10, 0.2), rtol=1e-15)


# ---------------------------------------------------------------- SRE

def test_sre_single_pair_closed_form():
    """A pair folded alone into an empty state: H = phi v^T, s = phi, so
    pred = (phi.phi) v / (phi.phi + eps) and SRE = (eps / (phi.phi + eps))^2 ||v||^2."""
    W = _rand((8, 6), 14, 1 / np.sqrt(8))
    k = _rand((8,), 15)
    v = _rand((8,), 16)
    ph = _phi_lib(k, W)
    for eps in (0.0, 1e-6, 1e-2, 0.3):
        got = oracle.sre(ph, v, np.outer(ph, v), ph, eps)
        pp = float(ph @ ph)
        want = (eps / (pp + eps)) ** 2 * float(v.astype(np.float64) @ v)
        assert abs(got - want) <= 1e-15 + 1e-12 * want


def test_sre_empty_state_is_value_norm():
    v = _rand((8,), 17)
    ph = _phi_lib(_rand((8,), 18), _rand((8, 4), 19))
    got = oracle.sre(ph, v, np.zeros((8, 8)), np.zeros(8), 1e-6)
    assert abs(got - float(v.astype(np.float64) @ v)) < 1e-12


def test_sre_in_the_run_single_pair_and_tie_break():
    """lambda=1, eta=0, interval 1. Tokens 0 and 1 carry the same (k, v):
    interval 1 scores both against the empty state (equal SRE = ||v||^2) and the
    tie keeps the lower index, so token 1 is folded alone. Interval 2 then
    scores token 0 against that single-pair state: the closed form above."""
    d, D, eps = 8, 8, 1e-2
    W = _rand((d, D // 2), 20, 1 / np.sqrt(d))
    k = _rand((1, 3, 1, d), 21)
    v = _rand((1, 3, 1, d), 22)
    k[0, 1] = k[0, 0]
    v[0, 1] = v[0, 0]
    q = _rand((1, 3, 1, d), 23)
    r = oracle.run(q, k, v, W, window=0, lambda_=1, intervals=[1, 1, 1], eps=eps,
                   want_cands=True)
    assert r.kept[1, 0, 0] == 0 and r.nkept[1, 0] == 1       # tie -> lower index kept
    ph = _phi_lib(k[0, 0, 0], W)
    pp = float(ph @ ph)
    want = (eps / (pp + eps)) ** 2 * float(v[0, 0, 0].astype(np.float64) @ v[0, 0, 0])
    toks = list(r.cand_tok[2, 0])
    got = r.cand_sre[2, 0, toks.index(0)]
    assert abs(got - want) <= 1e-12 * max(want, 1e-30)


# ---------------------------------------------------------------- special cases

def _causal_softmax(q, k, v):
    """Exact causal softmax attention (scale 1/sqrt(d)) via torch's SDPA in fp64."""
    B, T, Hq, d = q.shape
    g = Hq // k.shape[2]
    Q = torch.from_numpy(q.astype(np.float64)).permute(0, 2, 1, 3)
    K = torch.from_numpy(np.repeat(k, g, axis=2).astype(np.float64)).permute(0, 2, 1, 3)
    V = torch.from_numpy(np.repeat(v, g, axis=2).astype(np.float64)).permute(0, 2, 1, 3)
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("lam,C", [(0, 4), (3, 1), (5, 7), (64, 16)])
def test_unbounded_window_is_causal_softmax(lam, C):
    B, T, Hq, Hkv, d, D = 2, 56, 4, 2, 16, 12
    q, k, v, W = _qkvw(B, T, Hq, Hkv, d, D, 30 + lam)
    ints = [C] * (T // C) + ([T % C] if T % C else [])
    r = oracle.run(q, k, v, W, window=T, lambda_=lam, intervals=ints, eps=0.0)
    np.testing.assert_allclose(r.out, _causal_softmax(q, k, v), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("eta,C", [(0, 4), (3, 1), (2, 8), (5, 5)])
def test_cache_holding_every_pair_is_causal_softmax(eta, C):
    B, T, Hq, Hkv, d, D = 1, 48, 2, 2, 8, 8
    q, k, v, W = _qkvw(B, T, Hq, Hkv, d, D, 40 + eta)
    ints = [C] * (T // C) + ([T % C] if T % C else [])
    r = oracle.run(q, k, v, W, window=eta, lambda_=T, intervals=ints, eps=0.0,
                   want_state=True)
    np.testing.assert_allclose(r.out, _causal_softmax(q, k, v), rtol=1e-11, atol=1e-12)
    assert np.all(r.H == 0) and np.all(r.s == 0)


def _causal_linear(q, k, v, W, eps):
    """Inclusive causal linear attention with feature map phi, via cumulative sums."""
    B, T, Hq, d = q.shape
    g = Hq // k.shape[2]
    pq = _phi_lib(q, W)                                   # [B,T,Hq,D]
    pk = np.repeat(_phi_lib(k, W), g, axis=2)             # [B,T,Hq,D]
    vv = np.repeat(v.astype(np.float64), g, axis=2)
    Hc = np.cumsum(np.einsum("bthi,bthc->bthic", pk, vv), axis=1)
    sc = np.cumsum(pk, axis=1)
    num = np.einsum("bthi,bthic->bthc", pq, Hc)
    den = np.einsum("bthi,bthi->bth", pq, sc) + eps
    return num / den[..., None]


@pytest.mark.parametrize("C", [1, 3, 8, 13])
def test_no_window_no_cache_is_linear_attention(C):
    B, T, Hq, Hkv, d, D = 2, 39, 4, 2, 8, 10
    q, k, v, W = _qkvw(B, T, Hq, Hkv, d, D, 50 + C, wscale=2.0)
    ints = [C] * (T // C) + ([T % C] if T % C else [])
    eps = 1e-3
    r = oracle.run(q, k, v, W, window=0, lambda_=0, intervals=ints, eps=eps)
    np.testing.assert_allclose(r.out, _causal_linear(q, k, v, W, eps), rtol=1e-11, atol=1e-13)


def _window_plus_linear(q, k, v, W, eta, eps):
    """lambda = 0 direct form: softmax over the window (p-eta, p], linear over j <= p-eta."""
    B, T, Hq, d = q.shape
    g = Hq // k.shape[2]
    out = np.zeros((B, T, Hq, d))
    pq = _phi_lib(q, W)
    pk = _phi_lib(k, W)
    p_idx = np.arange(T)[:, None]
    j_idx = np.arange(T)[None, :]
    win = (j_idx <= p_idx) & (j_idx > p_idx - eta)
    lin = j_idx <= p_idx - eta
    for b in range(B):
        for hq in range(Hq):
            hk = hq // g
            Q = q[b, :, hq].astype(np.float64)
            K = k[b, :, hk].astype(np.float64)
            V = v[b, :, hk].astype(np.float64)
            Wt = np.where(win, np.exp(Q @ K.T / np.sqrt(d)), 0.0)
            Wt = Wt + np.where(lin, pq[b, :, hq] @ pk[b, :, hk].T, 0.0)
            out[b, :, hq] = (Wt @ V) / (Wt.sum(1) + eps)[:, None]
    return out


@pytest.mark.parametrize("eta,C", [(5, 1), (5, 3), (5, 8), (1, 4), (7, 16)])
def test_no_cache_is_window_softmax_plus_linear(eta, C):
    B, T, Hq, Hkv, d, D = 1, 47, 4, 2, 8, 8
    q, k, v, W = _qkvw(B, T, Hq, Hkv, d, D, 60 + eta + C)
    ints = [C] * (T // C) + ([T % C] if T % C else [])
    r = oracle.run(q, k, v, W, window=eta, lambda_=0, intervals=ints, eps=1e-6)
    np.testing.assert_allclose(r.out, _window_plus_linear(q, k, v, W, eta, 1e-6),
                               rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------- mixed regime

MIXED = [
    # (eta, lam, intervals)
    (5, 4, [4] * 10),
    (5, 4, [1] * 40),
    (3, 6, [8] * 5),
    (0, 3, [4] * 10),
    (6, 2, [2, 5, 1, 7, 4, 4, 1, 1, 8, 7]),
    (4, 5, [4] * 4 + [1] * 24),           # chunked prefill then token-by-token decode
    (2, 9, [10] * 4),
]


@pytest.mark.parametrize("eta,lam,ints", MIXED)
def test_matches_set_based_bruteforce(eta, lam, ints):
    T = sum(ints)
    B, Hq, Hkv, d, D = 1, 4, 2, 8, 8
    q, k, v, W = _qkvw(B, T, Hq, Hkv, d, D, 70 + eta * 7 + lam)
    # planted collision: a later key nearly equal to an earlier one, fresh value
    k[0, 25] = 0.95 * k[0, 3] + 0.05 * k[0, 25]
    eps = 1e-6
    r = oracle.run(q, k, v, W, window=eta, lambda_=lam, intervals=ints, eps=eps,
                   want_cands=True)
    out_b, kept_b, sre_b = brute.run(q, k, v, W, window=eta, lambda_=lam, intervals=ints, eps=eps)
    np.testing.assert_allclose(r.out, out_b, rtol=1e-10, atol=1e-12)
    for ci in range(len(ints)):
        for st in range(B * Hkv):
            got = [t for t in r.kept[ci, st] if t >= 0] if lam else []
            assert got == kept_b[ci][st], (ci, st)
            for t, s in zip(r.cand_tok[ci, st], r.cand_sre[ci, st]):
                if t >= 0:
                    assert abs(s - sre_b[ci][st][t]) <= 1e-10 * max(1.0, abs(s))


def test_selection_is_top_lambda_with_lower_index_tie_break():
    """Exchange property on every interval: each kept candidate beats each folded
    one in (SRE desc, index asc); brute force over all subsets of tiny candidate
    sets confirms it is the unique such set."""
    T, eta, lam = 36, 3, 4
    q, k, v, W = _qkvw(1, T, 2, 2, 8, 8, 90)
    v[0, 10] = v[0, 2]      # planted exact SRE ties at the start
    v[0, 11] = v[0, 2]
    r = oracle.run(q, k, v, W, window=eta, lambda_=lam, intervals=[3] * 12, want_cands=True)
    for ci in range(12):
        for st in range(2):
            toks = [t for t in r.cand_tok[ci, st] if t >= 0]
            sres = {t: s for t, s in zip(r.cand_tok[ci, st], r.cand_sre[ci, st]) if t >= 0}
            kept = set(t for t in r.kept[ci, st] if t >= 0)
            assert len(kept) == min(lam, len(toks))
            rank = lambda t: (-sres[t], t)
            for a in kept:
                for f in set(toks) - kept:
                    assert rank(a) < rank(f)
            if len(toks) <= 12:
                best = min(itertools.combinations(toks, len(kept)),
                           key=lambda c: sorted(rank(t) for t in c))
                assert set(best) == kept


def test_margin_log():
    T, eta, lam = 40, 4, 3
    q, k, v, W = _qkvw(1, T, 2, 1, 8, 8, 95)
    r = oracle.run(q, k, v, W, window=eta, lambda_=lam, intervals=[4] * 10, want_cands=True)
    for ci in range(10):
        toks = [t for t in r.cand_tok[0 + ci, 0] if t >= 0]
        s = sorted((x for x in r.cand_sre[ci, 0] if not np.isnan(x)), reverse=True)
        if len(toks) <= lam:
            assert np.isinf(r.margin[ci, 0])
        else:
            assert abs(r.margin[ci, 0] - (s[lam - 1] - s[lam]) / s[lam - 1]) < 1e-15


def test_gqa_equals_mha_with_repeated_kv():
    T, eta, lam = 40, 4, 3
    q, k, v, W = _qkvw(1, T, 4, 2, 8, 8, 96)
    ints = [4] * 10
    ra = oracle.run(q, k, v, W, window=eta, lambda_=lam, intervals=ints)
    rb = oracle.run(q, np.repeat(k, 2, axis=2), np.repeat(v, 2, axis=2), W, window=eta,
                    lambda_=lam, intervals=ints)
    np.testing.assert_allclose(ra.out, rb.out, rtol=1e-13, atol=0)
    np.testing.assert_array_equal(np.repeat(ra.kept, 2, axis=1), rb.kept)


def test_interval_partition_is_irrelevant_when_nothing_folds():
    T = 48
    q, k, v, W = _qkvw(1, T, 2, 2, 8, 8, 97)
    outs = [oracle.run(q, k, v, W, window=4, lambda_=T, intervals=ints).out
            for ints in ([48], [1] * 48, [8] * 6, [5, 3, 16, 1, 1, 22])]
    for o in outs[1:]:
        np.testing.assert_allclose(o, outs[0], rtol=1e-12, atol=1e-14)


def test_final_state_is_sum_over_folded_set():
    """After the last interval, (H, s) = sum over every pair that left the window
    and is not in the cache, recomputed directly."""
    T, eta, lam = 44, 5, 4
    q, k, v, W = _qkvw(2, T, 2, 2, 8, 6, 98)
    ints = [4] * 11
    r = oracle.run(q, k, v, W, window=eta, lambda_=lam, intervals=ints, want_state=True)
    for b in range(2):
        for hk in range(2):
            st = b * 2 + hk
            S = set(int(t) for t in r.kept[-1, st] if t >= 0)
            folded = [j for j in range(T) if j + eta < T and j not in S]
            pk = _phi_lib(k[b, :, hk], W)
            H = sum(np.outer(pk[j], v[b, j, hk].astype(np.float64)) for j in folded)
            s = sum(pk[j] for j in folded)
            np.testing.assert_allclose(r.H[st], H, rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(r.s[st], s, rtol=1e-12, atol=1e-14)


def test_qmask_rows_equal_full_run():
    T = 40
    q, k, v, W = _qkvw(1, T, 2, 1, 8, 8, 99)
    full = oracle.run(q, k, v, W, window=3, lambda_=4, intervals=[4] * 10)
    mask = np.zeros(T, np.uint8)
    mask[[0, 7, 13, 39]] = 1
    part = oracle.run(q, k, v, W, window=3, lambda_=4, intervals=[4] * 10, qmask=mask)
    np.testing.assert_array_equal(part.out[:, mask == 1], full.out[:, mask == 1])
    assert np.all(part.out[:, mask == 0] == 0)
    np.testing.assert_array_equal(part.kept, full.kept)


def test_rejects_bad_intervals():
    q, k, v, W = _qkvw(1, 8, 2, 1, 8, 8, 100)
    with pytest.raises(ValueError):
        oracle.run(q, k, v, W, window=2, lambda_=2, intervals=[4, 3])       # short of T
    with pytest.raises(ValueError):
        oracle.run(q, k, v, W, window=2, lambda_=2, intervals=[4, 4, 2])    # interval past T
    with pytest.raises(ValueError):
        oracle.run(q, k, v, W, window=2, lambda_=2, intervals=[4, 8])       # scores unseen pairs


def test_open_last_interval_matches_bruteforce():
    """A decode interval still open at the end: its candidates are all known
    (interval length <= eta + 1) and its queries stop at T."""
    T, eta, lam = 37, 5, 4
    q, k, v, W = _qkvw(1, T, 4, 2, 8, 8, 101)
    ints = [4] * 7 + [6, 6]          # covers 40 >= 37, last interval opened at 34
    r = oracle.run(q, k, v, W, window=eta, lambda_=lam, intervals=ints)
    out_b, kept_b, _ = brute.run(q, k, v, W, window=eta, lambda_=lam, intervals=ints)
    np.testing.assert_allclose(r.out, out_b, rtol=1e-10, atol=1e-12)
    assert [t for t in r.kept[-1, 1] if t >= 0] == kept_b[-1][1]


# ---------------------------------------------------------------- ablation scorers and FIFO

@pytest.mark.parametrize("scorer", ["attention-weight", "softmax-error", "fifo"])
@pytest.mark.parametrize("eta,lam,ints", [(5, 4, [4] * 10), (3, 6, [8] * 5), (4, 5, [4] * 4 + [1] * 24)])
def test_scorers_match_set_based_bruteforce(scorer, eta, lam, ints):
    T = sum(ints)
    B, Hq, Hkv, d, D = 1, 4, 2, 8, 8
    q, k, v, W = _qkvw(B, T, Hq, Hkv, d, D, 170 + eta * 7 + lam)
    eps = 1e-6
    r = oracle.run(q, k, v, W, window=eta, lambda_=lam, intervals=ints, eps=eps, want_cands=True,
                   scorer=scorer)
    out_b, kept_b, sc_b = brute.run(q, k, v, W, window=eta, lambda_=lam, intervals=ints, eps=eps,
                                    scorer=scorer)
    np.testing.assert_allclose(r.out, out_b, rtol=1e-10, atol=1e-12)
    for ci in range(len(ints)):
        for st in range(B * Hkv):
            assert [t for t in r.kept[ci, st] if t >= 0] == kept_b[ci][st], (ci, st)
            for t, s in zip(r.cand_tok[ci, st], r.cand_sre[ci, st]):
                if t >= 0:
                    assert abs(s - sc_b[ci][st][t]) <= 1e-10 * max(1.0, abs(s))


@pytest.mark.parametrize("eta,lam", [(5, 4), (2, 7), (0, 3)])
def test_fifo_token_by_token_is_a_wider_window(eta, lam):
    # keeping the most recent pairs with one-token intervals leaves exactly the
    # last eta + lam pairs in softmax and everything older in the linear state:
    # the no-cache direct form with window eta + lam
    B, T, Hq, Hkv, d, D = 1, 41, 4, 2, 8, 8
    q, k, v, W = _qkvw(B, T, Hq, Hkv, d, D, 190 + eta + lam)
    r = oracle.run(q, k, v, W, window=eta, lambda_=lam, intervals=[1] * T, eps=1e-6, scorer="fifo")
    np.testing.assert_allclose(r.out, _window_plus_linear(q, k, v, W, eta + lam, 1e-6),
                               rtol=1e-11, atol=1e-13)


def test_attention_weight_one_head_keeps_the_largest_logits():
    # with one query head per kv-head the softmax is monotone in q.k: the kept set
    # of every interval is the lambda candidates with the largest q_t0 . k
    B, T, Hq, Hkv, d, D = 1, 60, 2, 2, 8, 8
    q, k, v, W = _qkvw(B, T, Hq, Hkv, d, D, 211)
    ints, lam = [6] * 10, 5
    r = oracle.run(q, k, v, W, window=4, lambda_=lam, intervals=ints, eps=1e-6, want_cands=True,
                   scorer="attention-weight")
    t0 = 0
    for ci, C in enumerate(ints):
        for st in range(Hkv):
            toks = [int(t) for t in r.cand_tok[ci, st] if t >= 0]
            if len(toks) > lam:
                logit = {j: float(q[0, t0, st] @ k[0, j, st]) for j in toks}
                want = sorted(sorted(toks, key=lambda j: (-logit[j], j))[:lam])
                assert [int(t) for t in r.kept[ci, st] if t >= 0] == want
        t0 += C


# ---------------------------------------------------------------- one feature map per kv-head

def test_per_head_feature_maps_match_set_based_bruteforce():
    B, Hq, Hkv, d, D = 1, 4, 2, 8, 8
    ints = [4] * 10
    T = sum(ints)
    q, k, v, W0 = _qkvw(B, T, Hq, Hkv, d, D, 230)
    W = np.stack([W0, _rand((d, D // 2), 234, 1.0 / np.sqrt(d))])
    r = oracle.run(q, k, v, W, window=5, lambda_=4, intervals=ints, eps=1e-6, want_cands=True)
    out_b, kept_b, _ = brute.run(q, k, v, W, window=5, lambda_=4, intervals=ints, eps=1e-6)
    np.testing.assert_allclose(r.out, out_b, rtol=1e-10, atol=1e-12)
    for ci in range(len(ints)):
        for st in range(B * Hkv):
            assert [t for t in r.kept[ci, st] if t >= 0] == kept_b[ci][st]


def test_per_head_feature_maps_are_separable_by_head():
    # each kv-head (with its query heads and its own W) run alone equals its slice of
    # the joint run: the head -> matrix mapping of keys and queries
    B, Hq, Hkv, d, D = 2, 6, 3, 8, 8
    ints = [5] * 8
    T = sum(ints)
    q, k, v, _ = _qkvw(B, T, Hq, Hkv, d, D, 240)
    W = np.stack([_rand((d, D // 2), 250 + h, 1.0 / np.sqrt(d)) for h in range(Hkv)])
    r = oracle.run(q, k, v, W, window=4, lambda_=5, intervals=ints, eps=1e-6)
    g = Hq // Hkv
    for h in range(Hkv):
        rh = oracle.run(q[:, :, h * g:(h + 1) * g], k[:, :, h:h + 1], v[:, :, h:h + 1], W[h], window=4,
                        lambda_=5, intervals=ints, eps=1e-6)
        np.testing.assert_allclose(r.out[:, :, h * g:(h + 1) * g], rh.out, rtol=1e-13, atol=1e-15)
        for b in range(B):
            np.testing.assert_array_equal(r.kept[:, b * Hkv + h], rh.kept[:, b])
