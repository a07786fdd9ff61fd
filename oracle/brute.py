"""Set-based brute-force restatement of the LoLA inference step (tiny inputs).

TEST INFRASTRUCTURE ONLY. It pins the C oracle to a second, non-recurrent
formulation of the same method (LoLA, arXiv 2505.23666; gist.science technical
summary, sections "Het Self-Recall Error (SRE) Mechanisme" and
"Inferentiestrategie"):

  * The recurrent state is never updated incrementally. At each interval start
    t0 it is rebuilt from scratch as the sum over the folded set
    F* = { j < t0 - eta } minus the sparse cache S, i.e. H = sum phi(k_j) v_j^T
    and s = sum phi(k_j) over F*.
  * Selection sorts the candidates with Python's sort on (-score, index). The
    score is the SRE, or one of the ablation scores (see `scores`).
  * Each output row classifies every earlier key j <= p directly: softmax when
    j is inside the window of p (j > p - eta) or j is in the kept set of the
    interval; linear (weight phi(q).phi(k_j)) otherwise. The row is
    (sum_softmax e^{score} v + sum_linear w v) / (sum_softmax e^{score} + sum_linear w + eps),
    evaluated without the max shift (inputs here are small).
The feature map uses scipy's softmax: phi(x) = [softmax(xW), softmax(-xW)].
"""
from __future__ import annotations

import numpy as np
from scipy.special import softmax


def phi_rows(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    z = np.asarray(x, np.float64) @ np.asarray(W, np.float64)
    return np.concatenate([softmax(z, axis=-1), softmax(-z, axis=-1)], axis=-1)


def scores(scorer, cands, qrows, keys, phik, H, s, vv, eps):
    """Score of every candidate token, NumPy: "sre" -- ||phi(k)H/(phi(k)s+eps) - v||^2;
    "attention-weight" -- over the heads of the group, the softmax (over the
    candidates) of q.k/sqrt(d) for the interval's first query; "softmax-error" --
    over the heads, the squared gap between that weight and phi(q).phi(k) divided
    by its sum over the candidates; "fifo" -- the token index."""
    d = vv.shape[1]
    if not cands:
        return {}
    if scorer == "fifo":
        return {j: float(j) for j in cands}
    if scorer == "sre":
        out = {}
        for j in cands:
            den = float(phik[j] @ s) + eps
            pred = (phik[j] @ H) / den if den != 0.0 else np.zeros(d)
            out[j] = float(np.sum((pred - vv[j]) ** 2))
        return out
    tot = np.zeros(len(cands))
    for qh in qrows:
        a = softmax(np.array([float(qh @ keys[j]) for j in cands]) / np.sqrt(d))
        if scorer == "attention-weight":
            tot += a
        else:
            pq = phi_rows(qh[None, :], _W_for_scores)[0]
            lw = np.array([float(pq @ phik[j]) for j in cands])
            tot += (a - lw / lw.sum()) ** 2
    return {j: float(x) for j, x in zip(cands, tot)}


_W_for_scores = None


def run(q, k, v, W, *, window: int, lambda_: int, intervals, eps: float = 1e-6, scorer: str = "sre"):
    """Returns (out [B,T,Hq,d], kept list per interval per stream, score dict per interval)."""
    global _W_for_scores
    _W_for_scores = np.asarray(W, np.float64)
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    eta, lam = window, lambda_
    out = np.zeros((B, T, Hq, d))
    kept_log = []       # [interval][stream] -> sorted list of kept token ids
    sre_log = []        # [interval][stream] -> {token: sre}
    S = [[] for _ in range(B * Hkv)]
    bounds = np.cumsum([0] + list(intervals))
    for ci in range(len(intervals)):
        t0, t1 = int(bounds[ci]), int(bounds[ci + 1])
        kept_log.append([])
        sre_log.append([])
        for b in range(B):
            for hk in range(Hkv):
                st = b * Hkv + hk
                Wh = W[hk] if np.ndim(W) == 3 else W       # one matrix per kv-head, or shared
                _W_for_scores = np.asarray(Wh, np.float64)
                pk = phi_rows(k[b, :, hk, :], Wh)           # [T, D]
                vv = v[b, :, hk, :]
                cache = set(S[st])
                folded = [j for j in range(0, max(0, t0 - eta)) if j not in cache]
                H = sum((np.outer(pk[j], vv[j]) for j in folded), np.zeros((pk.shape[1], d)))
                s = sum((pk[j] for j in folded), np.zeros(pk.shape[1]))
                leaving = [j for j in range(T) if t0 <= j + eta < t1]
                cands = sorted(cache) + leaving
                qrows = [q[b, t0, hk * g + r, :] for r in range(g)]
                sres = scores(scorer, cands, qrows, k[b, :, hk, :], pk, H, s, vv, eps)
                order = sorted(cands, key=lambda j: (-sres[j], j))
                K = set(order[:min(lam, len(order))])
                kept_log[-1].append(sorted(K))
                sre_log[-1].append(sres)
                for p in range(t0, min(t1, T)):
                    for r in range(g):
                        hq = hk * g + r
                        qp = q[b, p, hq, :]
                        pq = phi_rows(qp[None, :], Wh)[0]
                        num = np.zeros(d)
                        den = eps
                        for j in range(0, p + 1):
                            if j > p - eta or j in K:
                                w = np.exp(float(qp @ k[b, j, hk, :]) / np.sqrt(d))
                            else:
                                w = float(pq @ pk[j])
                            num += w * vv[j]
                            den += w
                        out[b, p, hq, :] = num / den
                S[st] = sorted(K)
    return out, kept_log, sre_log
