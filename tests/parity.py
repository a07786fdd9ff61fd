"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the CPU oracle on the same seeded inputs, and compare them.

Selection rule for comparisons (the top-lambda choice is a discrete decision
taken on floating-point SREs): where the oracle's lambda-th vs (lambda+1)-th
SRE margin exceeds 1e-3 relative, the GPU's kept set must equal the oracle's
exactly; under that margin the GPU's set must be a valid top-lambda within the
band (every token on which the two sets differ has an oracle SRE within 1e-3
relative of the oracle's lambda-th SRE) and the case is counted.

Runs of the engine against one oracle run:
  forced -- every interval's kept set is the oracle's (the engine still computes
            and logs its own choice, which is checked);
  own    -- the engine keeps its own choice wherever the oracle's margin exceeds
            1e-3, and takes the oracle's set only on the intervals under that
            margin, so the outputs compared are the product path's own;
  free   -- no forcing at all.
No value computed on the GPU ever enters the oracle.
"""
from __future__ import annotations

import json
import os

import numpy as np

import oracle

MARGIN = 1e-3
COUNTS_FILE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "profiles",
                           "parity_counts.json")


def intervals_for(plan, chunk, decode_interval, pos0=0):
    """Interval lengths of a plan [("prefill", n) | ("decode", steps)], mirroring
    the engine: prefill runs n/chunk intervals; decode opens an interval of
    decode_interval steps whenever the position reaches the end of the last."""
    ints = []
    pos, iend = pos0, pos0
    for kind, n in plan:
        if kind == "prefill":
            assert pos == iend and n % chunk == 0
            ints += [chunk] * (n // chunk)
            pos += n
            iend = pos
        else:
            for _ in range(n):
                if pos == iend:
                    ints.append(decode_interval)
                    iend = pos + decode_interval
                pos += 1
    return ints


def override_from(r, lam, ns_gpu=None, stream_map=None, only_under_margin=False):
    """Engine override buffer [n_int, ns_gpu, lam+1] from an oracle run. Streams
    the oracle did not run (subset runs) get count -1: not forced. With
    only_under_margin, only the intervals whose oracle margin is <= MARGIN are
    forced; all others keep the engine's own choice."""
    n_int, ns = r.nkept.shape
    ns_gpu = ns if ns_gpu is None else ns_gpu
    smap = list(range(ns)) if stream_map is None else stream_map
    buf = np.full((n_int, ns_gpu, lam + 1), -1, np.int32)
    for so, sg in enumerate(smap):
        rows = np.ones(n_int, bool) if not only_under_margin else (r.margin[:, so] <= MARGIN)
        buf[rows, sg, 0] = r.nkept[rows, so]
        if lam:
            buf[rows, sg, 1:] = r.kept[rows, so]
    return buf


def run_gpu(cfg, W, q, k, v, plan, override=None, log_cap=None, device="cuda", rows=None,
            score_cap=None):
    """Runs the plan through the C ABI. q,k,v are float32 numpy arrays on the
    dtype grid, [B, T, H, d] with T = all prefill + decode tokens in order.
    rows (sorted positions) keeps only those outputs (gathered on the device).
    Returns (out float32 [B, T or len(rows), Hq, d], selection log or None,
    score log (sre, tok) or None)."""
    import torch
    from hybrid_linear_attention_lola_b200.lola import LolaState

    S = LolaState(cfg, torch.from_numpy(W), device)
    log = S.enable_selection_log(log_cap) if log_cap else None
    scores = S.enable_score_log(score_cap) if score_cap else None
    if override is not None:
        S.set_selection_override(torch.from_numpy(override))
    dt = S.dtype
    qd = torch.from_numpy(q).to(device=device, dtype=dt)
    kd = torch.from_numpy(k).to(device=device, dtype=dt)
    vd = torch.from_numpy(v).to(device=device, dtype=dt)
    keep = None if rows is None else np.asarray(rows)
    outs = []
    t = 0

    def take(o, t0, n):
        # o: [B, n, Hq, d] outputs of positions [t0, t0 + n)
        if keep is None:
            return o.float().cpu()
        lo, hi = np.searchsorted(keep, [t0, t0 + n])
        if hi == lo:
            return None
        idx = torch.as_tensor(keep[lo:hi] - t0, device=o.device)
        return o.index_select(1, idx).float().cpu()

    for kind, n in plan:
        if kind == "prefill":
            o = S.prefill(qd[:, t:t + n].contiguous(), kd[:, t:t + n].contiguous(),
                          vd[:, t:t + n].contiguous())
            outs.append(take(o, t, n))
            t += n
        else:
            for _ in range(n):
                o = S.decode(qd[:, t].contiguous(), kd[:, t].contiguous(), vd[:, t].contiguous())
                outs.append(take(o[:, None], t, 1))
                t += 1
    S.sync()
    out = torch.cat([o for o in outs if o is not None], dim=1).numpy()
    lg = log.cpu().numpy() if log is not None else None
    sc = (scores[0].cpu().numpy(), scores[1].cpu().numpy()) if scores is not None else None
    S.close()
    return out, lg, sc


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def row_rel_l2_max(a, b):
    """Largest relative L2 error over the output rows (one row = one query head of
    one position of one sequence)."""
    a = np.asarray(a, np.float64).reshape(-1, a.shape[-1])
    b = np.asarray(b, np.float64).reshape(-1, b.shape[-1])
    num = np.linalg.norm(a - b, axis=1)
    den = np.maximum(np.linalg.norm(b, axis=1), 1e-300)
    return float(np.max(num / den)) if len(num) else 0.0


def compare_selections(gpu_log, r, lam, stream_map=None):
    """Returns (n_checked, n_exact, n_under_margin_diff, hard_mismatches list).
    stream_map: oracle stream index -> GPU stream index (subset runs)."""
    n_int, ns_o = r.nkept.shape
    checked = exact = under = 0
    hard = []
    for ci in range(n_int):
        for so in range(ns_o):
            sg = so if stream_map is None else stream_map[so]
            row = gpu_log[ci, sg]
            cnt = int(row[0])
            gset = set(int(x) for x in row[1:1 + cnt])
            oset = set(int(x) for x in r.kept[ci, so] if x >= 0) if lam else set()
            checked += 1
            if gset == oset and cnt == r.nkept[ci, so]:
                exact += 1
                continue
            m = r.margin[ci, so]
            if m > MARGIN or r.cand_sre is None:
                hard.append((ci, so, float(m), sorted(gset ^ oset)[:8]))
                continue
            toks = list(r.cand_tok[ci, so])
            sres = {int(t): float(s) for t, s in zip(toks, r.cand_sre[ci, so]) if t >= 0}
            ordered = sorted(sres.values(), reverse=True)
            s_lam = ordered[lam - 1]
            ok = len(gset) == len(oset) and all(
                t in sres and abs(sres[t] - s_lam) <= MARGIN * s_lam for t in gset ^ oset)
            if ok:
                under += 1
            else:
                hard.append((ci, so, float(m), sorted(gset ^ oset)[:8]))
    return checked, exact, under, hard


def margin_summary(r):
    """Counts of the oracle's selection margins (intervals where |Q| > lambda)."""
    m = r.margin[np.isfinite(r.margin)]
    return {"intervals_with_selection": int(m.size),
            "margin_le_1e-3": int(np.sum(m <= MARGIN)),
            "margin_le_1e-2": int(np.sum(m <= 1e-2)),
            "min_margin": float(m.min()) if m.size else None}


def score_errors(gpu_scores, r, stream_map=None):
    """Relative error of the engine's SRE against the oracle's, candidate by
    candidate (matched by token) on a forced run, where both score the same
    candidate sets against states built from the same kept sets."""
    sre_g, tok_g = gpu_scores
    n_int = r.cand_tok.shape[0]
    smap = list(range(r.cand_tok.shape[1])) if stream_map is None else stream_map
    rels = []
    mism = 0
    for so, sg in enumerate(smap):
        tg = tok_g[:n_int, sg]
        sg_ = sre_g[:n_int, sg]
        to = r.cand_tok[:, so]
        so_ = r.cand_sre[:, so]
        # sort both by token per interval (-1 padding first) and align
        ig = np.argsort(np.where(tg < 0, -1, tg), axis=1, kind="stable")
        io = np.argsort(np.where(to < 0, -1, to), axis=1, kind="stable")
        tg2 = np.take_along_axis(tg, ig, 1)
        sg2 = np.take_along_axis(sg_, ig, 1)
        to2 = np.take_along_axis(to, io, 1)
        so2 = np.take_along_axis(so_, io, 1)
        # right-align the valid entries (both have the same number of candidates)
        ng = (tg2 >= 0).sum(1)
        no = (to2 >= 0).sum(1)
        mism += int(np.sum(ng != no))
        w = min(tg2.shape[1], to2.shape[1])
        tg3, sg3, to3, so3 = tg2[:, -w:], sg2[:, -w:], to2[:, -w:], so2[:, -w:]
        valid = (to3 >= 0) & (tg3 == to3)
        mism += int(np.sum((to3 >= 0) & (tg3 != to3)))
        o = so3[valid]
        gv = sg3[valid].astype(np.float64)
        rels.append(np.abs(gv - o) / np.maximum(np.abs(o), 1e-30))
    rel = np.concatenate(rels) if rels else np.zeros(0)
    edges = [1e-5, 1e-4, 1e-3, 1e-2]
    hist = {f"<{e:g}": int(np.sum(rel < e)) for e in edges}
    hist[">=1e-2"] = int(np.sum(rel >= 1e-2))
    return {"candidates": int(rel.size), "token_mismatches": mism,
            "max_rel_err": float(rel.max()) if rel.size else 0.0,
            "p99_rel_err": float(np.quantile(rel, 0.99)) if rel.size else 0.0,
            "median_rel_err": float(np.median(rel)) if rel.size else 0.0,
            "histogram": hist}


def record(name: str, entry: dict) -> None:
    """Adds one test's measured counts to the committed record of parity counts
    (written by the GPU parity tests themselves)."""
    try:
        with open(COUNTS_FILE) as f:
            data = json.load(f)
    except (OSError, ValueError):
        data = {}
    data[name] = entry
    os.makedirs(os.path.dirname(COUNTS_FILE), exist_ok=True)
    tmp = COUNTS_FILE + f".{os.getpid()}.tmp"
    with open(tmp, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
    os.replace(tmp, COUNTS_FILE)
